// mla_lib.cu -- host side of libmla.so: the C ABI declared in include/mla.h.
// Validates arguments, plans the split-KV work, builds TMA descriptors and
// launches the kernels of simt_kernels.cuh and decode_tc.cuh. It allocates no
// device memory and never synchronises a stream except in mla_check_status.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "mla.h"
#include "common.cuh"
#include "ptx.cuh"
#include "simt_kernels.cuh"
#include "decode_tc.cuh"
#include "gemm_tc.cuh"
#include "decode_2sm.cuh"
#include "cache_write.cuh"
#include "fp8_kernels.cuh"
#include "prefill.cuh"

namespace {

thread_local std::string g_last_error;
std::atomic<int32_t> g_policy{MLA_POLICY_AUTO};
std::atomic<uint64_t> g_timeout_ns{2000000000ull};
// The planner's estimate of what merging split queries costs, in pages of decode work
// (mla_set_plan_combine_cost); negative: plans always cut queries where slots fill up.
std::atomic<double> g_combine_cost_pages{-1.0};
unsigned long long* g_trace = nullptr;  // event trace buffer (MLA_TRACE builds only)
std::atomic<int32_t> g_drop_load{-1};   // testing hook, see mla_debug_drop_page_load

mla_status fail(mla_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

mla_status ok() {
  g_last_error.clear();
  return MLA_OK;
}

#define MLA_CUDA_TRY(expr)                                                               \
  do {                                                                                   \
    cudaError_t e_ = (expr);                                                             \
    if (e_ != cudaSuccess)                                                               \
      return fail(MLA_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));          \
  } while (0)

mla_status check_dims(const mla_dims& d) {
  const int32_t v[] = {d.H, d.Dn, d.Dr, d.Dv, d.R, d.page_size};
  const char* names[] = {"H", "Dn", "Dr", "Dv", "R", "page_size"};
  for (int i = 0; i < 6; ++i)
    if (v[i] <= 0) return fail(MLA_ERR_INVALID, "dims.%s must be positive, got %d", names[i], v[i]);
  if (d.dtype != MLA_BF16 && d.dtype != MLA_F32)
    return fail(MLA_ERR_INVALID, "dims.dtype must be MLA_BF16 or MLA_F32, got %d", d.dtype);
  if (d.R + d.Dr > 16384) return fail(MLA_ERR_UNSUPPORTED, "R + Dr = %d is too wide", d.R + d.Dr);
  return MLA_OK;
}


// Geometry the tensor-core decode kernel is written for.
bool decode_tc_ok(const mla_dims& d) {
  return d.dtype == MLA_BF16 && d.R == mla::tc::kR && d.Dr == mla::tc::kDr &&
         d.page_size == mla::tc::kPage && d.H % mla::tc::kHeads == 0;
}

bool use_tc_decode(const mla_dims& d) {
  const int32_t pol = g_policy.load();
  return pol != MLA_POLICY_SIMT && decode_tc_ok(d);
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

mla_status launch_check(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MLA_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return ok();
}

// ---------------------------------------------------------------- TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D bf16 tensor [rows][cols] (row pitch `pitch_bytes`), box = box_rows rows x 64 cols,
// 128-byte swizzle, zero fill out of bounds.
// 2-D bf16 tensor map, boxes of box_cols x box_rows; box_cols = 64 uses the 128-byte
// swizzle, box_cols = 32 the 64-byte swizzle (one box row = one swizzle row).
mla_status make_map_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch_bytes,
                       uint32_t box_rows = 64, uint32_t box_cols = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0)
    return fail(MLA_ERR_INVALID, "tensor base %p is not 16-byte aligned", base);
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  if (box_cols != 64 && box_cols != 32) return fail(MLA_ERR_INVALID, "unsupported box width %u", box_cols);
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MLA_OK;
}

// 2-D tensor map of one-byte elements (E4M3 codes): boxes of 128 x box_rows with the
// 128-byte swizzle. Columns of a box past `cols` read as zero.
mla_status make_map_u8_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t pitch_bytes,
                          uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0)
    return fail(MLA_ERR_INVALID, "tensor base %p is not 16-byte aligned", base);
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (codes) failed (%d)", (int)r);
  return MLA_OK;
}

// 2-D tensor map without swizzle (boxes stored row-major in shared memory), for the
// decode kernel's output stores: bf16 or fp32 elements, boxes of box_cols x box_rows.
mla_status make_store_map_2d(CUtensorMap* m, const void* base, bool f32, uint64_t cols, uint64_t rows,
                             uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0)
    return fail(MLA_ERR_INVALID, "tensor base %p is not 16-byte aligned", base);
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (store map) failed (%d)", (int)r);
  return MLA_OK;
}

// Per-device one-time kernel attributes (large dynamic shared memory).
mla_status ensure_smem_attr(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, int>> done;  // (kernel, device)
  int dev = 0;
  MLA_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(mu);
  for (auto& e : done)
    if (e.first == kernel && e.second == dev) return MLA_OK;
  MLA_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  done.emplace_back(kernel, dev);
  return MLA_OK;
}

// Geometry the tensor-core projections are instantiated for.
bool absorb_tc_ok(const mla_dims& d) { return d.dtype == MLA_BF16 && d.Dn == 128 && d.R == 512; }
bool outproj_tc_ok(const mla_dims& d) { return d.dtype == MLA_BF16 && d.R == 512 && d.Dv == 128; }

template <int KBLK, int N, bool B_MN, int STAGES>
mla_status launch_proj(const void* A, const void* Bw, void* out, int32_t T, const mla_dims& d, int32_t a_cols,
                       int32_t b_rows, int32_t b_cols, int32_t n_total, cudaStream_t st, const char* what) {
  using C = mla::gemm::Cfg<KBLK, N, B_MN, STAGES>;
  CUtensorMap ta, tb;
  if (mla_status s = make_map_2d(&ta, A, (uint64_t)d.H * a_cols, (uint64_t)T, (uint64_t)d.H * a_cols * 2, 128))
    return s;
  if (mla_status s = make_map_2d(&tb, Bw, (uint64_t)b_cols, (uint64_t)b_rows, (uint64_t)b_cols * 2, 64)) return s;
  auto kern = mla::gemm::proj_kernel<KBLK, N, B_MN, STAGES>;
  if (mla_status s = ensure_smem_attr((const void*)kern, C::kSmemBytes)) return s;
  mla::gemm::Params p;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.T = T;
  p.H = d.H;
  p.n_total = n_total;
  p.timeout_ns = g_timeout_ns.load();
  const dim3 grid(d.H, (T + mla::gemm::kM - 1) / mla::gemm::kM, n_total / N);
  kern<<<grid, 128, C::kSmemBytes, st>>>(ta, tb, p);
  return launch_check(what);
}

// The output projection with fp32 o_lat (see gemm::proj_a32_kernel): A boxes of 32 fp32
// columns x 128 rows with the 128-byte swizzle, weights as for launch_proj.
template <int KBLK, int N, int STAGES>
mla_status launch_proj_a32(const void* A, const void* Bw, void* out, int32_t T, const mla_dims& d, cudaStream_t st) {
  using C = mla::gemm::CfgA32<KBLK, N, STAGES>;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  if (reinterpret_cast<uintptr_t>(A) % 16 != 0) return fail(MLA_ERR_INVALID, "o_lat %p is not 16-byte aligned", A);
  CUtensorMap ta, tb;
  const cuuint64_t dims[2] = {(cuuint64_t)d.H * d.R, (cuuint64_t)T};
  const cuuint64_t strides[1] = {(cuuint64_t)d.H * d.R * 4};
  const cuuint32_t box[2] = {32, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(A), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuTensorMapEncodeTiled (fp32 A) failed (%d)", (int)r);
  if (mla_status s = make_map_2d(&tb, Bw, (uint64_t)d.R, (uint64_t)d.H * d.Dv, (uint64_t)d.R * 2, 64)) return s;
  auto kern = mla::gemm::proj_a32_kernel<KBLK, N, STAGES>;
  if (mla_status s = ensure_smem_attr((const void*)kern, C::kSmemBytes)) return s;
  mla::gemm::Params p;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.T = T;
  p.H = d.H;
  p.n_total = d.Dv;
  p.timeout_ns = g_timeout_ns.load();
  const dim3 grid(d.H, (T + mla::gemm::kM - 1) / mla::gemm::kM, d.Dv / N);
  kern<<<grid, mla::gemm::kA32Threads, C::kSmemBytes, st>>>(ta, tb, p);
  return launch_check("out_proj (tcgen05, fp32 o_lat)");
}

// The SM-pair kernel serves 128 rows per cluster: all heads of one query token for
// H=128, or the heads of up to two consecutive query tokens of a sequence for H=64
// (with one query token per sequence the odd CTA's rows are idle).
bool pair_decode(const mla_dims& d, int32_t q_len) {
  (void)q_len;
  return use_tc_decode(d) && (d.H == mla::duo::kRows || d.H == mla::duo::kRows / 2);
}

// CTAs per slot (the plan has num_sms / head_groups slots).
int32_t head_groups_for(const mla_dims& d, int32_t q_len) {
  if (pair_decode(d, q_len)) return 2;
  return decode_tc_ok(d) ? d.H / mla::tc::kHeads : 1;
}

// Work a unit costs beyond its pages, in pages, for the split planner: the SM-pair
// kernel stages each unit's query, runs its epilogue and refills its load pipeline at the
// unit's boundaries (measured at about six pages' time); the other kernels are planned on
// pages alone.
// Work the SM-pair kernel spends on a unit beyond its pages, in pages: a unit boundary
// (the next query staged in TMEM, the previous unit's epilogue, the pipeline refilled)
// measured ~18.9K cycles against ~2.45K per page in steady state on B200.
double unit_cost_pages(const mla_dims& d, int32_t q_len) { return pair_decode(d, q_len) ? 7.5 : 0.0; }

// Query tokens per plan unit (consecutive tokens of one sequence).
int32_t items_per_unit_for(const mla_dims& d, int32_t q_len) {
  return pair_decode(d, q_len) && q_len >= 2 ? mla::duo::kRows / d.H : 1;
}

}  // namespace

// =============================================================================== C ABI
extern "C" {

int32_t mla_abi_version(void) { return MLA_ABI_VERSION; }

#ifdef MLA_TRACE
// Trace builds only (not declared in mla.h): device buffer of 1024 uint64 per CTA.
void mla_debug_set_trace(void* dev_buf) { g_trace = static_cast<unsigned long long*>(dev_buf); }
#endif

const char* mla_last_error(void) { return g_last_error.c_str(); }

mla_status mla_set_policy(int32_t policy) {
  if (policy < MLA_POLICY_AUTO || policy > MLA_POLICY_TCGEN05)
    return fail(MLA_ERR_INVALID, "unknown policy %d", policy);
  g_policy.store(policy);
  return ok();
}

mla_status mla_set_plan_combine_cost(double pages) {
  if (!(pages == pages)) return fail(MLA_ERR_INVALID, "combine cost is NaN");
  g_combine_cost_pages.store(pages);
  return ok();
}

mla_status mla_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return fail(MLA_ERR_INVALID, "timeout must be positive");
  g_timeout_ns.store(ns);
  return ok();
}

mla_status mla_debug_drop_page_load(int32_t ordinal) {
  g_drop_load.store(ordinal < 0 ? -1 : ordinal);
  return ok();
}

mla_status mla_check_status(void* stream) {
  MLA_CUDA_TRY(cudaStreamSynchronize(as_stream(stream)));
  unsigned int v = 0, zero = 0;
  MLA_CUDA_TRY(cudaMemcpyFromSymbol(&v, mla::g_status, sizeof(v)));
  MLA_CUDA_TRY(cudaMemcpyToSymbol(mla::g_status, &zero, sizeof(zero)));
  if (v & mla::kStatusTimeout) return fail(MLA_ERR_TIMEOUT, "a kernel wait ran out (status 0x%x)", v);
  if (v & mla::kStatusBadPage)
    return fail(MLA_ERR_INVALID, "a block_table entry was outside [0, num_pages) (status 0x%x)", v);
  if (g_drop_load.load() >= 0)
    return fail(MLA_ERR_INVALID, "the test-only mla_debug_drop_page_load hook is still set (ordinal %d)",
                g_drop_load.load());
  return ok();
}

// ------------------------------------------------------------------------------- append
mla_status mla_cache_append(void* kv_cache, const int32_t* block_table, const int32_t* seq_lens,
                            const void* new_ckr, int32_t B, int32_t q_len, int32_t max_pages,
                            int32_t num_pages, mla_dims d, void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (B < 0 || q_len <= 0 || max_pages <= 0 || num_pages <= 0)
    return fail(MLA_ERR_INVALID, "bad sizes B=%d q_len=%d max_pages=%d num_pages=%d", B, q_len, max_pages,
                num_pages);
  if (B == 0) return ok();
  if (!kv_cache || !block_table || !seq_lens || !new_ckr) return fail(MLA_ERR_INVALID, "null pointer");
  const int32_t row = d.R + d.Dr;
  const size_t row_bytes = (size_t)row * (d.dtype == MLA_BF16 ? 2 : 4);
  if (row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(kv_cache) % 16 == 0 &&
      reinterpret_cast<uintptr_t>(new_ckr) % 16 == 0) {
    const int32_t items = B * q_len;
    mla::simt::cache_append_vec_kernel<<<(items + 3) / 4, 128, 0, as_stream(stream)>>>(
        static_cast<uint4*>(kv_cache), block_table, seq_lens, static_cast<const uint4*>(new_ckr), items, q_len,
        max_pages, num_pages, (int32_t)(row_bytes / 16), d.page_size);
    return launch_check("cache_append");
  }
  const dim3 grid(B * q_len);
  if (d.dtype == MLA_BF16)
    mla::simt::cache_append_kernel<__nv_bfloat16><<<grid, 128, 0, as_stream(stream)>>>(
        static_cast<__nv_bfloat16*>(kv_cache), block_table, seq_lens,
        static_cast<const __nv_bfloat16*>(new_ckr), q_len, max_pages, num_pages, row, d.page_size);
  else
    mla::simt::cache_append_kernel<float><<<grid, 128, 0, as_stream(stream)>>>(
        static_cast<float*>(kv_cache), block_table, seq_lens, static_cast<const float*>(new_ckr), q_len,
        max_pages, num_pages, row, d.page_size);
  return launch_check("cache_append");
}

// ------------------------------------------------------------------------------- cache-write prologue
size_t mla_cache_write_workspace_size(int32_t T, int32_t M) {
  if (T <= 0 || M <= 0 || M % mla::cw::kKB != 0) return 0;
  return (size_t)mla::cw::slices_for(M) * (size_t)T * mla::cw::kRow * sizeof(float);
}

mla_status mla_cache_write(const void* hidden, const void* W_DKV, const void* kv_gain, int32_t M,
                           void* kv_cache, const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                           int32_t q_len, int32_t max_pages, int32_t num_pages, void* q_rope, float eps,
                           float rope_base, void* workspace, size_t workspace_bytes, mla_dims d, void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (B < 0 || q_len <= 0 || max_pages <= 0 || num_pages <= 0 || M <= 0)
    return fail(MLA_ERR_INVALID, "bad sizes B=%d q_len=%d max_pages=%d num_pages=%d M=%d", B, q_len, max_pages,
                num_pages, M);
  if (!(eps >= 0.f) || !std::isfinite(eps)) return fail(MLA_ERR_INVALID, "eps must be finite and >= 0");
  if (!(rope_base > 1.f) || !std::isfinite(rope_base)) return fail(MLA_ERR_INVALID, "rope_base must be > 1");
  if (d.dtype != MLA_BF16 || d.R != mla::cw::kR || d.Dr != mla::cw::kDr || d.page_size != mla::cw::kPage ||
      M % mla::cw::kKB != 0)
    return fail(MLA_ERR_UNSUPPORTED, "the cache-write prologue needs bf16, R=512, Dr=64, page_size=64, M %% 64 == 0");
  if (g_policy.load() == MLA_POLICY_SIMT)
    return fail(MLA_ERR_UNSUPPORTED, "the cache-write prologue has only a tensor-core kernel");
  if (B == 0) return ok();
  if (!hidden || !W_DKV || !kv_gain || !kv_cache || !block_table || !seq_lens)
    return fail(MLA_ERR_INVALID, "null pointer");
  const int32_t T = B * q_len;
  const size_t need = mla_cache_write_workspace_size(T, M);
  if (!workspace || workspace_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) % 16 != 0) return fail(MLA_ERR_INVALID, "workspace not 16-byte aligned");
  CUtensorMap ta, tb;
  if (mla_status s = make_map_2d(&ta, hidden, (uint64_t)M, (uint64_t)T, (uint64_t)M * 2, 128)) return s;
  if (mla_status s = make_map_2d(&tb, W_DKV, (uint64_t)M, (uint64_t)(d.R + d.Dr), (uint64_t)M * 2, 64)) return s;
  mla::cw::Params p;
  p.kv = static_cast<__nv_bfloat16*>(kv_cache);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.gain = static_cast<const __nv_bfloat16*>(kv_gain);
  p.part = static_cast<float*>(workspace);
  p.T = T;
  p.q_len = q_len;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.kblk = M / mla::cw::kKB;
  p.slices = mla::cw::slices_for(M);
  p.eps = eps;
  p.rope_base = rope_base;
  p.timeout_ns = g_timeout_ns.load();
  cudaStream_t st = as_stream(stream);
  if (mla_status s = ensure_smem_attr((const void*)mla::cw::cache_write_gemm_kernel, mla::cw::Cfg::kSmemBytes))
    return s;
  const dim3 grid((T + mla::cw::kM - 1) / mla::cw::kM, mla::cw::kColBlocks, p.slices);
  mla::cw::cache_write_gemm_kernel<<<grid, 128, mla::cw::Cfg::kSmemBytes, st>>>(ta, tb, p);
  if (mla_status s = launch_check("cache_write (down projection)")) return s;
  mla::cw::cache_write_finish_kernel<<<T, mla::cw::kFinishThreads, 0, st>>>(
      p, static_cast<__nv_bfloat16*>(q_rope), d.H);
  return launch_check("cache_write (norm, rotation, append)");
}

// ------------------------------------------------------------------------------- absorb
mla_status mla_absorb_q(const void* q_nope, const void* W_UK, void* q_lat, int32_t T, mla_dims d,
                        void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (T < 0) return fail(MLA_ERR_INVALID, "T=%d", T);
  if (T == 0) return ok();
  if (!q_nope || !W_UK || !q_lat) return fail(MLA_ERR_INVALID, "null pointer");
  const int32_t pol = g_policy.load();
  if (pol == MLA_POLICY_TCGEN05 && !absorb_tc_ok(d))
    return fail(MLA_ERR_UNSUPPORTED, "tensor-core absorb needs bf16, Dn=128, R=512");
  if (pol != MLA_POLICY_SIMT && absorb_tc_ok(d)) {
    // up to 64 rows the weights dominate: four 128-column blocks per head (65 KB of shared
    // memory, three CTAs per SM) spread them over more SMs than two 256-column blocks do
    if (T <= 64)
      return launch_proj<2, 128, true, 2>(q_nope, W_UK, q_lat, T, d, d.Dn, d.H * d.Dn, d.R, d.R,
                                          as_stream(stream), "absorb_q (tcgen05)");
    return launch_proj<2, 256, true, 2>(q_nope, W_UK, q_lat, T, d, d.Dn, d.H * d.Dn, d.R, d.R, as_stream(stream),
                                        "absorb_q (tcgen05)");
  }
  const dim3 grid((d.R + 127) / 128, d.H, (T + mla::simt::kTT - 1) / mla::simt::kTT);
  const size_t smem = sizeof(float) * mla::simt::kTT * d.Dn;
  if (smem > 48 * 1024) return fail(MLA_ERR_UNSUPPORTED, "Dn=%d too large", d.Dn);
  if (d.dtype == MLA_BF16)
    mla::simt::absorb_kernel<__nv_bfloat16><<<grid, 128, smem, as_stream(stream)>>>(
        static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(W_UK),
        static_cast<__nv_bfloat16*>(q_lat), T, d.H, d.Dn, d.R);
  else
    mla::simt::absorb_kernel<float><<<grid, 128, smem, as_stream(stream)>>>(
        static_cast<const float*>(q_nope), static_cast<const float*>(W_UK), static_cast<float*>(q_lat), T,
        d.H, d.Dn, d.R);
  return launch_check("absorb_q");
}

// ------------------------------------------------------------------------------- out proj
mla_status mla_out_proj(const void* o_lat, const void* W_UV, void* out, int32_t T, mla_dims d,
                        void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (T < 0) return fail(MLA_ERR_INVALID, "T=%d", T);
  if (T == 0) return ok();
  if (!o_lat || !W_UV || !out) return fail(MLA_ERR_INVALID, "null pointer");
  const int32_t pol = g_policy.load();
  if (pol == MLA_POLICY_TCGEN05 && !outproj_tc_ok(d))
    return fail(MLA_ERR_UNSUPPORTED, "tensor-core output projection needs bf16, R=512, Dv=128");
  if (pol != MLA_POLICY_SIMT && outproj_tc_ok(d))
    return launch_proj_a32<8, 128, 4>(o_lat, W_UV, out, T, d, as_stream(stream));
  const dim3 grid(d.H, (T + mla::simt::kTT - 1) / mla::simt::kTT);
  const size_t smem = sizeof(float) * mla::simt::kTT * d.R;
  if (smem > 48 * 1024) return fail(MLA_ERR_UNSUPPORTED, "R=%d too large", d.R);
  if (d.dtype == MLA_BF16)
    mla::simt::outproj_kernel<__nv_bfloat16><<<grid, 256, smem, as_stream(stream)>>>(
        static_cast<const float*>(o_lat), static_cast<const __nv_bfloat16*>(W_UV),
        static_cast<__nv_bfloat16*>(out), T, d.H, d.Dv, d.R);
  else
    mla::simt::outproj_kernel<float><<<grid, 256, smem, as_stream(stream)>>>(
        static_cast<const float*>(o_lat), static_cast<const float*>(W_UV), static_cast<float*>(out), T, d.H,
        d.Dv, d.R);
  return launch_check("out_proj");
}

// ------------------------------------------------------------------------------- planning
size_t mla_plan_capacity(int32_t B, int32_t q_len, int32_t num_sms) {
  if (B < 0 || q_len <= 0 || num_sms <= 0) return 0;
  const size_t items = (size_t)B * q_len;
  const size_t slots = (size_t)num_sms;
  const size_t units = items + slots + 1;
  return mla::kPlanHeader + mla::kUnitWords * units + (slots + 1) + 2 * items;
}

mla_status mla_plan_splits(const int32_t* seq_lens_host, int32_t B, int32_t q_len, int32_t max_pages,
                           mla_dims d, int32_t num_sms, int32_t* plan_host, size_t capacity,
                           mla_plan_info* info) {
  if (mla_status s = check_dims(d)) return s;
  if (B < 0 || q_len <= 0 || max_pages <= 0 || num_sms <= 0)
    return fail(MLA_ERR_INVALID, "bad sizes B=%d q_len=%d max_pages=%d num_sms=%d", B, q_len, max_pages,
                num_sms);
  if ((B > 0 && !seq_lens_host) || !plan_host || !info) return fail(MLA_ERR_INVALID, "null pointer");
  if (capacity < mla_plan_capacity(B, q_len, num_sms))
    return fail(MLA_ERR_WORKSPACE, "plan capacity %zu < %zu words", capacity,
                mla_plan_capacity(B, q_len, num_sms));
  const int32_t ps = d.page_size;
  const int32_t G = head_groups_for(d, q_len);
  const int32_t ipu = items_per_unit_for(d, q_len);
  const int32_t slots_max = std::max(1, num_sms / G);
  const int32_t items = B * q_len;
  std::vector<int32_t> pages(items);
  for (int32_t b = 0; b < B; ++b) {
    const int32_t L = seq_lens_host[b];
    if (L < 0 || (int64_t)L > (int64_t)max_pages * ps)
      return fail(MLA_ERR_INVALID, "seq_lens[%d]=%d outside [0, max_pages*page_size=%lld]", b, L,
                  (long long)max_pages * ps);
    for (int32_t i = 0; i < q_len; ++i) {
      const int32_t n = mla::visible_tokens(L, q_len, i);
      pages[b * q_len + i] = (n + ps - 1) / ps;
    }
  }
  // Units cover groups of ipu consecutive query tokens of one sequence; a group's page
  // count is its last token's (which sees the most).
  int64_t total = 0;
  const int32_t groups_per_seq = (q_len + ipu - 1) / ipu;
  auto group_pages = [&](int32_t b, int32_t k) {
    const int32_t last = std::min(q_len, (k + 1) * ipu) - 1;
    return pages[b * q_len + last];
  };
  for (int32_t b = 0; b < B; ++b)
    for (int32_t k = 0; k < groups_per_seq; ++k) total += group_pages(b, k);
  struct U { int32_t item, b, pb, pe, slot, n; };
  std::vector<U> units;
  const int64_t S = std::max<int64_t>(1, std::min<int64_t>(slots_max, total));
  units.reserve(items + S);
  const double cost = unit_cost_pages(d, q_len);
  if (cost <= 0.0) {
    // Slot s covers flattened pages [s*total/S, (s+1)*total/S): page counts differ by at most one.
    auto bound = [&](int64_t s) { return s * total / S; };
    int32_t slot = 0;
    int64_t flat = 0;  // flattened index of the next page
    for (int32_t b = 0; b < B; ++b) {
      for (int32_t k = 0; k < groups_per_seq; ++k) {
        const int32_t it = b * q_len + k * ipu;
        const int32_t n = std::min(ipu, q_len - k * ipu);
        int32_t left = group_pages(b, k), pb = 0;
        if (left == 0) {
          units.push_back({it, b, 0, 0, slot, n});
          continue;
        }
        while (left > 0) {
          while (slot + 1 < S && flat >= bound(slot + 1)) ++slot;
          const int64_t room = (slot + 1 < S) ? bound(slot + 1) - flat : left;
          const int32_t take = (int32_t)std::min<int64_t>(left, room);
          units.push_back({it, b, pb, pb + take, slot, n});
          pb += take;
          left -= take;
          flat += take;
        }
      }
    }
  } else {
    // Every unit also costs `cost` pages of work (its query, its epilogue, a pipeline
    // refill). Units are laid out in order and each slot takes work up to a capacity C
    // (a group is cut where a slot fills up); C is the smallest capacity whose fill
    // needs at most S slots, found by bisection, so the heaviest slot is as light as
    // this contiguous layout allows.
    // A layout is a sequence of groups (b, k) laid out in order over the slots
    // [slot0, slot0 + ns).
    struct Grp { int32_t b, k; };
    auto fill = [&](const std::vector<Grp>& order, int64_t slot0, double C, bool emit) -> int64_t {
      int64_t slot = 0;
      double acc = 0.0;
      bool used = false;
      for (const Grp& g : order) {
        const int32_t b = g.b, k = g.k;
        const int32_t it = b * q_len + k * ipu;
        const int32_t n = std::min(ipu, q_len - k * ipu);
        int32_t left = group_pages(b, k), pb = 0;
        if (left == 0) {
          if (emit) units.push_back({it, b, 0, 0, (int32_t)(slot0 + slot), n});
          continue;
        }
        while (left > 0) {
          const double room = C - acc - cost;
          if (used && room < 1.0) {   // not even one more page fits: the next slot
            ++slot;
            acc = 0.0;
            used = false;
            continue;
          }
          const int32_t take = (int32_t)std::min<double>(left, std::max(1.0, std::floor(room)));
          if (emit) units.push_back({it, b, pb, pb + take, (int32_t)(slot0 + slot), n});
          used = true;
          pb += take;
          left -= take;
          acc += cost + take;
        }
      }
      return slot + 1;
    };
    // The same layout with every group whole: a group that does not fit in what is left
    // of a slot's capacity C starts the next slot (a group larger than C fills one alone).
    auto fill_whole = [&](const std::vector<Grp>& order, int64_t slot0, double C, bool emit) -> int64_t {
      int64_t slot = 0;
      double acc = 0.0;
      bool used = false;
      for (const Grp& g : order) {
        const int32_t it = g.b * q_len + g.k * ipu;
        const int32_t n = std::min(ipu, q_len - g.k * ipu);
        const int32_t pg = group_pages(g.b, g.k);
        if (pg > 0 && used && acc + cost + pg > C) {
          ++slot;
          acc = 0.0;
          used = false;
        }
        if (emit) units.push_back({it, g.b, 0, pg, (int32_t)(slot0 + slot), n});
        if (pg > 0) {
          used = true;
          acc += cost + pg;
        }
      }
      return slot + 1;
    };
    // the heaviest slot of the units emitted from index u0 on, and whether a group was cut
    auto heaviest = [&](size_t u0, bool* cut) {
      std::vector<double> load;
      *cut = false;
      for (size_t k = u0; k < units.size(); ++k) {
        const U& u = units[k];
        if ((size_t)u.slot >= load.size()) load.resize(u.slot + 1, 0.0);
        if (u.pe > u.pb) load[u.slot] += cost + (u.pe - u.pb);
        if (u.pb > 0) *cut = true;
      }
      double m = 0.0;
      for (double x : load) m = std::max(m, x);
      return m;
    };
    // the smallest capacity whose fill of `order` needs at most ns slots (bisection)
    auto bisect = [&](const std::vector<Grp>& order, int64_t slot0, int64_t ns, double lo, double hi, bool whole) {
      for (int it = 0; it < 48 && hi - lo > 0.25; ++it) {
        const double mid = 0.5 * (lo + hi);
        if ((whole ? fill_whole(order, slot0, mid, false) : fill(order, slot0, mid, false)) <= ns) hi = mid;
        else lo = mid;
      }
      return hi;
    };
    const double combine_cost = g_combine_cost_pages.load();
    auto layout = [&](const std::vector<Grp>& order, int64_t slot0, int64_t ns) {
      int64_t pages = 0, groups = 0;
      int32_t largest = 0;
      for (const Grp& g : order) {
        const int32_t pg = group_pages(g.b, g.k);
        pages += pg;
        groups += pg > 0;
        largest = std::max(largest, pg);
      }
      // below lo the pages and one cost per group do not fit in ns slots; hi fits in one
      const double lo = std::max(cost, ((double)pages + cost * (double)groups) / (double)ns - 1.0);
      const double hi = (double)pages + cost * (double)(groups + ns) + 1.0;
      const size_t u0 = units.size();
      fill(order, slot0, bisect(order, slot0, ns, lo, hi, false), true);
      if (combine_cost < 0.0) return;
      // With a combine cost set: the layout that keeps every group whole is taken instead
      // when its heaviest slot is no heavier than the cut layout's plus the merge of the
      // cut queries' parts (which only the cut layout needs).
      bool cut = false;
      const double cut_load = heaviest(u0, &cut);
      if (!cut) return;
      const double lo_w = std::max(lo, cost + (double)largest - 1.0);
      const size_t u1 = units.size();
      fill_whole(order, slot0, bisect(order, slot0, ns, lo_w, std::max(hi, lo_w + 1.0), true), true);
      bool cut_w = false;
      const double whole_load = heaviest(u1, &cut_w);
      if (units.back().slot - slot0 < ns && whole_load <= cut_load + combine_cost)
        units.erase(units.begin() + (std::ptrdiff_t)u0, units.begin() + (std::ptrdiff_t)u1);
      else
        units.resize(u1);
    };
    if (ipu == 1 && q_len >= 2 && S >= 2 * q_len) {
      // Several query tokens per sequence, one per unit (128 heads fill the pair's rows):
      // the last token's pages (it sees the most) are laid out on a block of S / q_len
      // slots, and every token gets a copy of that layout on a block of its own (the
      // kernel clips each unit to the pages its token sees). The tokens of a sequence
      // then stream the same pages on slot j of every block at about the same time:
      // each page is read from DRAM once and served to the other tokens' slots by L2.
      const int64_t ns = S / q_len;
      std::vector<Grp> order;
      order.reserve(B);
      for (int32_t b = 0; b < B; ++b) order.push_back({b, q_len - 1});
      const size_t u0 = units.size();
      layout(order, 0, ns);
      const std::vector<U> base(units.begin() + (std::ptrdiff_t)u0, units.end());
      units.resize(u0);
      for (int32_t k = 0; k < q_len; ++k)
        for (U u : base) {
          u.item = u.b * q_len + k;
          u.slot += (int32_t)(k * ns);
          units.push_back(u);
        }
    } else {
      std::vector<Grp> order;
      order.reserve((size_t)B * groups_per_seq);
      for (int32_t b = 0; b < B; ++b)
        for (int32_t k = 0; k < groups_per_seq; ++k) order.push_back({b, k});
      layout(order, 0, S);
    }
  }
  const int32_t num_slots = units.empty() ? 0 : units.back().slot + 1;
  // parts: items with more than one unit (every token of a split group is split)
  std::vector<int32_t> count(items, 0);
  for (const U& u : units)
    for (int32_t j = 0; j < u.n; ++j) count[u.item + j]++;
  std::vector<int32_t> first(items, -1);
  int32_t parts = 0;
  for (int32_t it = 0; it < items; ++it)
    if (count[it] > 1) {
      first[it] = parts;
      parts += count[it];
    }
  const size_t words = mla::kPlanHeader + mla::kUnitWords * units.size() + (num_slots + 1) + 2 * (size_t)items;
  if (words > capacity) return fail(MLA_ERR_WORKSPACE, "plan needs %zu words", words);
  std::memset(plan_host, 0, words * sizeof(int32_t));
  plan_host[0] = mla::kPlanMagic;
  plan_host[1] = B;
  plan_host[2] = q_len;
  plan_host[3] = (int32_t)units.size();
  plan_host[4] = num_slots;
  plan_host[5] = parts;
  plan_host[6] = G;
  plan_host[7] = d.H;
  plan_host[8] = ps;
  plan_host[9] = ipu;
  int32_t* uw = plan_host + mla::kPlanHeader;
  std::vector<int32_t> next(items, 0);
  for (size_t k = 0; k < units.size(); ++k) {
    const U& u = units[k];
    int32_t part[2] = {-1, -1};
    for (int32_t j = 0; j < u.n; ++j)
      if (count[u.item + j] > 1) part[j] = first[u.item + j] + next[u.item + j]++;
    int32_t* w = uw + mla::kUnitWords * k;
    w[0] = u.item;
    w[1] = u.b;
    w[2] = u.pb;
    w[3] = u.pe;
    w[4] = part[0];
    w[5] = u.slot;
    w[6] = part[1];
    w[7] = u.n;
  }
  int32_t* sb = uw + mla::kUnitWords * units.size();
  {
    size_t k = 0;  // units are ordered by slot: sb[s] = first unit of slot s
    for (int32_t s = 0; s <= num_slots; ++s) {
      while (k < units.size() && units[k].slot < s) ++k;
      sb[s] = (int32_t)k;
    }
  }
  int32_t* ip = sb + num_slots + 1;
  for (int32_t it = 0; it < items; ++it) {
    ip[2 * it] = count[it] > 1 ? first[it] : -1;
    ip[2 * it + 1] = count[it] > 1 ? count[it] : 0;
  }
  info->num_items = items;
  info->num_units = (int32_t)units.size();
  info->num_slots = num_slots;
  info->num_parts = parts;
  info->head_groups = G;
  info->plan_words = (int32_t)words;
  info->max_pages = max_pages;
  return ok();
}

size_t mla_workspace_size(const mla_plan_info* info, mla_dims d) {
  if (!info || check_dims(d) != MLA_OK) return 0;
  const size_t parts = (size_t)std::max(0, info->num_parts);
  size_t o = parts * d.H * d.R * sizeof(float);
  o = (o + 255) / 256 * 256;
  return o + parts * d.H * sizeof(float);
}

static mla_status split_workspace(const mla_plan_info* info, const mla_dims& d, void* ws, size_t bytes,
                                  float** o_part, float** lse_part) {
  *o_part = nullptr;
  *lse_part = nullptr;
  if (info->num_parts == 0) return MLA_OK;
  const size_t need = mla_workspace_size(info, d);
  if (!ws || bytes < need) return fail(MLA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", bytes, need);
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(MLA_ERR_INVALID, "workspace not 256-byte aligned");
  size_t o = (size_t)info->num_parts * d.H * d.R * sizeof(float);
  o = (o + 255) / 256 * 256;
  *o_part = static_cast<float*>(ws);
  *lse_part = reinterpret_cast<float*>(static_cast<char*>(ws) + o);
  return MLA_OK;
}

static mla_status check_info(const mla_plan_info* info, int32_t B, int32_t q_len, int32_t max_pages,
                             const mla_dims& d) {
  if (!info) return fail(MLA_ERR_INVALID, "null plan info");
  if (info->num_items != B * q_len)
    return fail(MLA_ERR_INVALID, "plan covers %d query tokens, call has %d", info->num_items, B * q_len);
  // the plan's page ranges index block_table rows of the length it was cut for
  if (info->max_pages != max_pages)
    return fail(MLA_ERR_INVALID, "plan was made for max_pages=%d, call has %d", info->max_pages, max_pages);
  if (info->head_groups != head_groups_for(d, q_len))
    return fail(MLA_ERR_INVALID,
                "plan was made for %d CTAs per slot, these dims, q_len and kernel policy need %d (plan "
                "again after changing the policy)",
                info->head_groups, head_groups_for(d, q_len));
  return MLA_OK;
}

// ------------------------------------------------------------------------------- decode
mla_status mla_decode_attn(const void* q_lat, const void* q_rope, const void* kv_cache,
                           const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                           int32_t q_len, int32_t max_pages, int32_t num_pages, float scale,
                           const int32_t* plan_dev, const mla_plan_info* info, void* o_lat,
                           float* lse, void* workspace, size_t workspace_bytes, mla_dims d,
                           void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (B < 0 || q_len <= 0 || max_pages <= 0 || num_pages <= 0)
    return fail(MLA_ERR_INVALID, "bad sizes B=%d q_len=%d max_pages=%d num_pages=%d", B, q_len, max_pages,
                num_pages);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MLA_ERR_INVALID, "scale must be positive");
  if (mla_status s = check_info(info, B, q_len, max_pages, d)) return s;
  if (B == 0 || info->num_units == 0) return ok();
  if (!q_lat || !q_rope || !kv_cache || !block_table || !seq_lens || !plan_dev || !o_lat)
    return fail(MLA_ERR_INVALID, "null pointer");
  float *o_part, *lse_part;
  if (mla_status s = split_workspace(info, d, workspace, workspace_bytes, &o_part, &lse_part)) return s;
  const int32_t pol = g_policy.load();
  if (pol == MLA_POLICY_TCGEN05 && !decode_tc_ok(d))
    return fail(MLA_ERR_UNSUPPORTED, "tensor-core decode needs bf16, R=512, Dr=64, page_size=64, H%%64==0");
  cudaStream_t st = as_stream(stream);
  if (use_tc_decode(d)) {
    const int64_t T = (int64_t)B * q_len;
    CUtensorMap tq, tr, tk;
    if (mla_status s = make_map_2d(&tq, q_lat, d.R, (uint64_t)T * d.H, (uint64_t)d.R * 2)) return s;
    if (mla_status s = make_map_2d(&tr, q_rope, d.Dr, (uint64_t)T * d.H, (uint64_t)d.Dr * 2)) return s;
    if (mla_status s = make_map_2d(&tk, kv_cache, d.R + d.Dr, (uint64_t)num_pages * d.page_size,
                                   (uint64_t)(d.R + d.Dr) * 2))
      return s;
    if (mla_status s = ensure_smem_attr((const void*)mla::tc::decode_kernel, mla::tc::kSmemBytes)) return s;
    mla::tc::Params p;
    p.plan = plan_dev;
    p.block_table = block_table;
    p.seq_lens = seq_lens;
    p.max_pages = max_pages;
    p.num_pages = num_pages;
    p.H = d.H;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o_lat = static_cast<float*>(o_lat);
    p.lse = lse;
    p.o_part = o_part;
    p.lse_part = lse_part;
    p.kv = static_cast<const __nv_bfloat16*>(kv_cache);
    p.q_lat = static_cast<const __nv_bfloat16*>(q_lat);
    p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
    p.timeout_ns = g_timeout_ns.load();
    p.trace = g_trace;
    p.drop_load = g_drop_load.load();
    const dim3 grid(info->num_slots * info->head_groups);
    if (pair_decode(d, q_len)) {
      // a pair of SMs per slot: 32-row boxes of the cache (half a page), 64-row boxes of
      // the queries (one CTA's rows)
      CUtensorMap tk32, to, top;
      if (mla_status s = make_map_2d(&tk32, kv_cache, d.R + d.Dr, (uint64_t)num_pages * d.page_size,
                                     (uint64_t)(d.R + d.Dr) * 2, 32, 64))
        return s;
      // output stores: fp32 blocks of 16 rows x 32 columns, final rows and partial rows
      if (mla_status s = make_store_map_2d(&to, o_lat, true, d.R, (uint64_t)T * d.H, (uint64_t)d.R * 4, 32, 16))
        return s;
      if (info->num_parts > 0) {
        if (mla_status s = make_store_map_2d(&top, o_part, true, d.R, (uint64_t)info->num_parts * d.H,
                                             (uint64_t)d.R * 4, 32, 16))
          return s;
      } else {
        top = to;   // never used: the plan has no partial outputs
      }
      if (mla_status s = ensure_smem_attr((const void*)mla::duo::decode_2sm_kernel<false>, mla::duo::kSmemBytes))
        return s;
      mla::duo::decode_2sm_kernel<false><<<grid, mla::duo::kThreads, mla::duo::kSmemBytes, st>>>(
          tk32, tq, tr, to, top, tq, p);
      return launch_check("decode_attn (tcgen05, SM pair)");
    }
    mla::tc::decode_kernel<<<grid, 256, mla::tc::kSmemBytes, st>>>(tq, tr, tk, p);
    return launch_check("decode_attn (tcgen05)");
  }
  mla::simt::DecodeSimtArgs a;
  a.plan = plan_dev;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.H = d.H;
  a.R = d.R;
  a.Dr = d.Dr;
  a.page_size = d.page_size;
  a.scale = scale;
  a.o_lat = o_lat;
  a.lse = lse;
  a.o_part = o_part;
  a.lse_part = lse_part;
  const size_t smem = sizeof(float) * ((size_t)(d.R + d.Dr) + 4 * (size_t)d.R + 8);
  if (smem > 200 * 1024) return fail(MLA_ERR_UNSUPPORTED, "R=%d too large for the SIMT decode", d.R);
  const dim3 grid(info->num_units, d.H);
  if (d.dtype == MLA_BF16) {
    if (mla_status s = ensure_smem_attr((const void*)mla::simt::decode_kernel<__nv_bfloat16>, (int)smem)) return s;
    mla::simt::decode_kernel<__nv_bfloat16><<<grid, 128, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q_lat), static_cast<const __nv_bfloat16*>(q_rope),
        static_cast<const __nv_bfloat16*>(kv_cache), a);
  } else {
    if (mla_status s = ensure_smem_attr((const void*)mla::simt::decode_kernel<float>, (int)smem)) return s;
    mla::simt::decode_kernel<float><<<grid, 128, smem, st>>>(static_cast<const float*>(q_lat),
                                                             static_cast<const float*>(q_rope),
                                                             static_cast<const float*>(kv_cache), a);
  }
  return launch_check("decode_attn (SIMT)");
}

// ------------------------------------------------------------------------------- combine
// ------------------------------------------------------------------------------- 8-bit cache
static bool fp8_dims_ok(const mla_dims& d) {
  return d.dtype == MLA_BF16 && d.R == 512 && d.Dr == 64 && d.page_size == 64;
}

mla_status mla_quantize_rows_fp8(const void* rows, void* codes, void* scales, int64_t n, mla_dims d,
                                 void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (!fp8_dims_ok(d)) return fail(MLA_ERR_UNSUPPORTED, "the 8-bit cache needs bf16 rows with R=512, Dr=64");
  if (n < 0) return fail(MLA_ERR_INVALID, "bad row count %lld", (long long)n);
  if (n == 0) return ok();
  if (!rows || !codes || !scales) return fail(MLA_ERR_INVALID, "null pointer");
  if (reinterpret_cast<uintptr_t>(rows) % 16 != 0 || reinterpret_cast<uintptr_t>(codes) % 8 != 0)
    return fail(MLA_ERR_INVALID, "rows must be 16-byte and codes 8-byte aligned");
  mla::f8::quantise_rows_kernel<<<(unsigned)((n + 7) / 8), 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(rows), static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales), n,
      nullptr, nullptr, 1, 1, 1, d.page_size);
  return launch_check("quantize_rows_fp8");
}

mla_status mla_cache_append_fp8(void* kv_codes, void* kv_scales, const int32_t* block_table,
                                const int32_t* seq_lens, const void* new_ckr, int32_t B, int32_t q_len,
                                int32_t max_pages, int32_t num_pages, mla_dims d, void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (!fp8_dims_ok(d)) return fail(MLA_ERR_UNSUPPORTED, "the 8-bit cache needs bf16 rows with R=512, Dr=64, page 64");
  if (B < 0 || q_len <= 0 || max_pages <= 0 || num_pages <= 0)
    return fail(MLA_ERR_INVALID, "bad sizes B=%d q_len=%d max_pages=%d num_pages=%d", B, q_len, max_pages,
                num_pages);
  if (B == 0) return ok();
  if (!kv_codes || !kv_scales || !block_table || !seq_lens || !new_ckr) return fail(MLA_ERR_INVALID, "null pointer");
  if (reinterpret_cast<uintptr_t>(new_ckr) % 16 != 0 || reinterpret_cast<uintptr_t>(kv_codes) % 8 != 0)
    return fail(MLA_ERR_INVALID, "new_ckr must be 16-byte and kv_codes 8-byte aligned");
  const int64_t n = (int64_t)B * q_len;
  mla::f8::quantise_rows_kernel<<<(unsigned)((n + 7) / 8), 256, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(new_ckr), static_cast<uint8_t*>(kv_codes), static_cast<uint8_t*>(kv_scales),
      n, block_table, seq_lens, q_len, max_pages, num_pages, d.page_size);
  return launch_check("cache_append_fp8");
}

// The 8-bit decode's workspace: the split partials (as mla_workspace_size), then the
// split query [2][T*H][576] codes and its row scales [T*H] fp32.
static size_t fp8_query_offset(const mla_plan_info* info, const mla_dims& d) {
  return (mla_workspace_size(info, d) + 255) / 256 * 256;
}

size_t mla_workspace_size_fp8(const mla_plan_info* info, mla_dims d) {
  if (!info || check_dims(d) != MLA_OK) return 0;
  const size_t rows = (size_t)std::max(0, info->num_items) * d.H;
  return fp8_query_offset(info, d) + (2 * rows * 576 + 255) / 256 * 256 + rows * sizeof(float);
}

mla_status mla_decode_attn_fp8(const void* q_lat, const void* q_rope, const void* kv_codes, const void* kv_scales,
                               const int32_t* block_table, const int32_t* seq_lens, int32_t B, int32_t q_len,
                               int32_t max_pages, int32_t num_pages, float scale, const int32_t* plan_dev,
                               const mla_plan_info* info, void* o_lat, float* lse, void* workspace,
                               size_t workspace_bytes, mla_dims d, void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (B < 0 || q_len <= 0 || max_pages <= 0 || num_pages <= 0)
    return fail(MLA_ERR_INVALID, "bad sizes B=%d q_len=%d max_pages=%d num_pages=%d", B, q_len, max_pages,
                num_pages);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MLA_ERR_INVALID, "scale must be positive");
  if (!fp8_dims_ok(d) || !pair_decode(d, q_len))
    return fail(MLA_ERR_UNSUPPORTED,
                "the 8-bit cache decode runs on the SM-pair tensor-core kernel: bf16 queries, R=512, Dr=64, "
                "page_size=64, H=64 or 128, and a policy other than SIMT");
  if (mla_status s = check_info(info, B, q_len, max_pages, d)) return s;
  if (B == 0 || info->num_units == 0) return ok();
  if (!q_lat || !q_rope || !kv_codes || !kv_scales || !block_table || !seq_lens || !plan_dev || !o_lat)
    return fail(MLA_ERR_INVALID, "null pointer");
  if (reinterpret_cast<uintptr_t>(kv_scales) % 16 != 0)
    return fail(MLA_ERR_INVALID, "kv_scales must be 16-byte aligned (each page's 64 bytes are bulk-copied)");
  const size_t need = mla_workspace_size_fp8(info, d);
  if (!workspace || workspace_bytes < need)
    return fail(MLA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return fail(MLA_ERR_INVALID, "workspace not 256-byte aligned");
  float *o_part, *lse_part;
  if (mla_status s = split_workspace(info, d, workspace, workspace_bytes, &o_part, &lse_part)) return s;
  const int64_t T = (int64_t)B * q_len, rows = T * d.H;
  uint8_t* q8 = static_cast<uint8_t*>(workspace) + fp8_query_offset(info, d);
  float* q_scale = reinterpret_cast<float*>(q8 + (2 * (size_t)rows * 576 + 255) / 256 * 256);
  cudaStream_t st = as_stream(stream);
  CUtensorMap tk32, tk64, tqh, tql, to, top;
  const uint64_t cache_rows = (uint64_t)num_pages * d.page_size;
  if (mla_status s = make_map_u8_2d(&tk32, kv_codes, 576, cache_rows, 576, 32)) return s;
  if (mla_status s = make_map_u8_2d(&tk64, kv_codes, 576, cache_rows, 576, 64)) return s;
  if (mla_status s = make_map_u8_2d(&tqh, q8, 576, (uint64_t)rows, 576, 64)) return s;
  if (mla_status s = make_map_u8_2d(&tql, q8 + (size_t)rows * 576, 576, (uint64_t)rows, 576, 64)) return s;
  if (mla_status s = make_store_map_2d(&to, o_lat, true, d.R, (uint64_t)rows, (uint64_t)d.R * 4, 32, 16)) return s;
  if (info->num_parts > 0) {
    if (mla_status s = make_store_map_2d(&top, o_part, true, d.R, (uint64_t)info->num_parts * d.H,
                                         (uint64_t)d.R * 4, 32, 16))
      return s;
  } else {
    top = to;   // never used: the plan has no partial outputs
  }
  mla::f8::split_query_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q_lat), static_cast<const __nv_bfloat16*>(q_rope), q8, q_scale, rows);
  if (mla_status s = launch_check("decode_attn_fp8 (split query)")) return s;
  mla::tc::Params p;
  p.plan = plan_dev;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.H = d.H;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_lat = static_cast<float*>(o_lat);
  p.lse = lse;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.kv = nullptr;
  p.q_lat = static_cast<const __nv_bfloat16*>(q_lat);
  p.q_rope = static_cast<const __nv_bfloat16*>(q_rope);
  p.timeout_ns = g_timeout_ns.load();
  p.trace = g_trace;
  p.drop_load = g_drop_load.load();
  p.kv_scale = static_cast<const uint8_t*>(kv_scales);
  p.q8 = q8;
  p.q_scale = q_scale;
  if (mla_status s = ensure_smem_attr((const void*)mla::duo::decode_2sm_kernel<true>, mla::duo::kSmemBytesF8))
    return s;
  const dim3 grid(info->num_slots * info->head_groups);
  mla::duo::decode_2sm_kernel<true><<<grid, mla::duo::kThreadsF8, mla::duo::kSmemBytesF8, st>>>(tk32, tqh, tk64, to,
                                                                                               top, tql, p);
  return launch_check("decode_attn_fp8 (tcgen05, SM pair)");
}

// ------------------------------------------------------------------------------- prefill (non-absorbed)
static bool prefill_dims_ok(const mla_dims& d) {
  return d.dtype == MLA_BF16 && d.R == 512 && d.Dr == 64 && d.Dn == 128 && d.Dv == 128 && d.H % 2 == 0;
}

size_t mla_prefill_workspace_size(int32_t N, mla_dims d) {
  if (N <= 0 || check_dims(d) != MLA_OK || !prefill_dims_ok(d)) return 0;
  return 2 * (((size_t)N * d.H * 128 * 2 + 255) / 256 * 256);
}

mla_status mla_prefill_attn(const void* ckr, const void* q_nope, const void* q_rope, const void* W_UK,
                            const void* W_UV, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int32_t B,
                            float scale, void* out, void* workspace, size_t workspace_bytes, mla_dims d,
                            void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (!prefill_dims_ok(d))
    return fail(MLA_ERR_UNSUPPORTED, "prefill needs bf16, R=512, Dr=64, Dn=Dv=128 and an even head count");
  if (g_policy.load() == MLA_POLICY_SIMT)
    return fail(MLA_ERR_UNSUPPORTED, "prefill has only a tensor-core kernel (policy is SIMT)");
  if (B < 0) return fail(MLA_ERR_INVALID, "bad B=%d", B);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(MLA_ERR_INVALID, "scale must be positive");
  if (B == 0) return ok();
  if (!cu_seqlens_host || !cu_seqlens) return fail(MLA_ERR_INVALID, "null cu_seqlens");
  if (cu_seqlens_host[0] != 0) return fail(MLA_ERR_INVALID, "cu_seqlens[0] must be 0");
  int32_t max_qtiles = 0, tiles = 0;
  for (int32_t b = 0; b < B; ++b) {
    const int32_t L = cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    if (L < 0) return fail(MLA_ERR_INVALID, "cu_seqlens must not decrease (sequence %d)", b);
    const int32_t t = (L + mla::pf::kM - 1) / mla::pf::kM;
    max_qtiles = std::max(max_qtiles, t);
    tiles += t;
  }
  const int32_t N = cu_seqlens_host[B];
  if (N == 0) return ok();
  if (!ckr || !q_nope || !q_rope || !W_UK || !W_UV || !out) return fail(MLA_ERR_INVALID, "null pointer");
  const size_t need = mla_prefill_workspace_size(N, d);
  if (!workspace || workspace_bytes < need) return fail(MLA_ERR_WORKSPACE, "workspace %zu bytes < %zu needed",
                                                        workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return fail(MLA_ERR_INVALID, "workspace not 256-byte aligned");
  __nv_bfloat16* kc = static_cast<__nv_bfloat16*>(workspace);
  __nv_bfloat16* vv = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(workspace) + need / 2);
  cudaStream_t st = as_stream(stream);
  const int32_t HD = d.H * 128;
  // up-projections: K_c = C W_UK^T and V = C W_UV^T for all heads at once (one GEMM each,
  // A = the latent columns of the packed rows, B = the weights as [H*128][512], K-major)
  {
    // two stages (97 KiB): two CTAs per SM, one's epilogue under the other's main loop
    using C = mla::gemm::Cfg<8, 256, false, 2>;
    auto kern = mla::gemm::proj_kernel<8, 256, false, 2>;
    if (mla_status s = ensure_smem_attr((const void*)kern, C::kSmemBytes)) return s;
    CUtensorMap ta;
    if (mla_status s = make_map_2d(&ta, ckr, 512, (uint64_t)N, 576 * 2, 128)) return s;
    const void* W[2] = {W_UK, W_UV};
    __nv_bfloat16* O[2] = {kc, vv};
    for (int i = 0; i < 2; ++i) {
      CUtensorMap tb;
      if (mla_status s = make_map_2d(&tb, W[i], 512, (uint64_t)HD, 512 * 2, 64)) return s;
      mla::gemm::Params gp;
      gp.out = O[i];
      gp.T = N;
      gp.H = 1;
      gp.n_total = HD;
      gp.timeout_ns = g_timeout_ns.load();
      const dim3 grid(1, (N + mla::gemm::kM - 1) / mla::gemm::kM, HD / 256);
      kern<<<grid, 128, C::kSmemBytes, st>>>(ta, tb, gp);
      if (mla_status s = launch_check("prefill (up-projection)")) return s;
    }
  }
  CUtensorMap tqn, tqr, tkc, tkr, tv;
  if (mla_status s = make_map_2d(&tqn, q_nope, HD, (uint64_t)N, (uint64_t)HD * 2, 128)) return s;
  if (mla_status s = make_map_2d(&tqr, q_rope, (uint64_t)d.H * 64, (uint64_t)N, (uint64_t)d.H * 64 * 2, 128)) return s;
  if (mla_status s = make_map_2d(&tkc, kc, HD, (uint64_t)N, (uint64_t)HD * 2, 128)) return s;
  if (mla_status s = make_map_2d(&tkr, ckr, 576, (uint64_t)N, 576 * 2, 128)) return s;
  if (mla_status s = make_map_2d(&tv, vv, HD, (uint64_t)N, (uint64_t)HD * 2, 128)) return s;
  if (mla_status s = ensure_smem_attr((const void*)mla::pf::prefill_attn_kernel, mla::pf::kSmemBytes)) return s;
  mla::pf::Params pp;
  pp.cu_seqlens = cu_seqlens;
  pp.B = B;
  pp.H = d.H;
  pp.max_qtiles = max_qtiles;
  pp.scale_log2 = scale * 1.4426950408889634f;
  pp.out = static_cast<__nv_bfloat16*>(out);
  pp.timeout_ns = g_timeout_ns.load();
  const dim3 grid(tiles, d.H);
  mla::pf::prefill_attn_kernel<<<grid, mla::pf::kThreads, mla::pf::kSmemBytes, st>>>(tqn, tqr, tkc, tkr, tv, pp);
  return launch_check("prefill (attention)");
}

mla_status mla_combine(const int32_t* plan_dev, const mla_plan_info* info, const void* workspace,
                       size_t workspace_bytes, void* o_lat, float* lse, mla_dims d, void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (!info) return fail(MLA_ERR_INVALID, "null plan info");
  if (info->num_parts == 0) return ok();
  if (!plan_dev || !o_lat) return fail(MLA_ERR_INVALID, "null pointer");
  float *o_part, *lse_part;
  if (mla_status s = split_workspace(info, d, const_cast<void*>(workspace), workspace_bytes, &o_part, &lse_part))
    return s;
  if (d.R <= 512 && d.R % 4 == 0) {
    // parts per query, at least: a few queries cut into many parts spread their parts over
    // the warps of a block; otherwise one warp per (query, head)
    const int32_t per_item = info->num_items > 0 ? info->num_parts / info->num_items : 0;
    if (per_item >= 3) {
      const dim3 gw(info->num_items, d.H);
      if (per_item >= 8)
        mla::simt::combine_wide_kernel<8><<<gw, 256, 0, as_stream(stream)>>>(
            plan_dev, o_part, lse_part, static_cast<float*>(o_lat), lse, d.H, d.R);
      else
        mla::simt::combine_wide_kernel<4><<<gw, 128, 0, as_stream(stream)>>>(
            plan_dev, o_part, lse_part, static_cast<float*>(o_lat), lse, d.H, d.R);
      return launch_check("combine");
    }
    const dim3 gv(info->num_items, (d.H + 3) / 4);
    mla::simt::combine_vec_kernel<<<gv, 128, 0, as_stream(stream)>>>(plan_dev, o_part, lse_part,
                                                                      static_cast<float*>(o_lat), lse, d.H, d.R);
    return launch_check("combine");
  }
  const dim3 grid(info->num_items, d.H);
  mla::simt::combine_kernel<<<grid, 128, 0, as_stream(stream)>>>(plan_dev, o_part, lse_part,
                                                                 static_cast<float*>(o_lat), lse, d.H, d.R);
  return launch_check("combine");
}

// ------------------------------------------------------------------------------- allocation-free decode
// Scratch for the partial outputs of mla_decode_attn_noalloc. It is a file-scope
// device array, so every GPU that loads this library holds kNoAllocScratchBytes
// until the process exits. Host code must not use the symbol as an address: the
// device address comes from cudaGetSymbolAddress, looked up once per CUDA context
// and kept under the context's driver id (unique for the life of the process), so a
// context created again after a reset is looked up afresh.
}  // extern "C"

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(48) << 20;
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
std::mutex g_noalloc_mu;
std::vector<std::pair<unsigned long long, void*>> g_noalloc_ptr;   // (context id, scratch address)

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static mla_status noalloc_scratch(void** out) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return fail(MLA_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId not available");
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) {
    // no context yet on this thread: the runtime makes the device's primary context
    // current on its first call that needs one
    void* p = nullptr;
    MLA_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return fail(MLA_ERR_CUDA, "no current CUDA context");
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return fail(MLA_ERR_CUDA, "cuCtxGetId failed");
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  for (const auto& e : g_noalloc_ptr)
    if (e.first == id) {
      *out = e.second;
      return MLA_OK;
    }
  void* p = nullptr;
  MLA_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));
  g_noalloc_ptr.emplace_back(id, p);
  *out = p;
  return MLA_OK;
}

extern "C" {

mla_status mla_decode_attn_noalloc(const void* q_lat, const void* q_rope, const void* kv_cache,
                                   const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                                   int32_t q_len, int32_t max_pages, int32_t num_pages, float scale,
                                   const int32_t* plan_dev, const mla_plan_info* info, void* o_lat,
                                   float* lse, mla_dims d, void* stream) {
  if (mla_status s = check_dims(d)) return s;
  if (mla_status s = check_info(info, B, q_len, max_pages, d)) return s;
  const size_t need = mla_workspace_size(info, d);
  if (need > kNoAllocScratchBytes)
    return fail(MLA_ERR_WORKSPACE,
                "plan has %d partial outputs needing %zu bytes of scratch; mla_decode_attn_noalloc "
                "holds at most %zu bytes (use mla_decode_attn with a caller workspace)",
                info->num_parts, need, kNoAllocScratchBytes);
  void* ws = nullptr;
  if (info->num_parts > 0)
    if (mla_status s = noalloc_scratch(&ws)) return s;
  if (mla_status s = mla_decode_attn(q_lat, q_rope, kv_cache, block_table, seq_lens, B, q_len, max_pages,
                                     num_pages, scale, plan_dev, info, o_lat, lse, ws,
                                     ws ? kNoAllocScratchBytes : 0, d, stream))
    return s;
  return mla_combine(plan_dev, info, ws, ws ? kNoAllocScratchBytes : 0, o_lat, lse, d, stream);
}

}  // extern "C"
