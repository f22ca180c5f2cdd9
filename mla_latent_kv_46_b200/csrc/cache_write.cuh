// cache_write.cuh -- the cache-write prologue of a decode step on sm_100a tensor cores.
//
// For each new token t (hidden state h_t, width M):
//   f_t = W_DKV h_t                      the down projection M -> R + Dr (one matrix: the
//                                        compressed KV feature and the shared key)
//   c_t = f_t[:R] / sqrt(mean(f_t[:R]^2) + eps) * kv_gain          (RMSNorm)
//   k_t = rope(f_t[R:], pos_t)           dims i and i + Dr/2 turned by pos_t * base^(-2i/Dr)
// and [c_t ; k_t] is written, in bf16, to the token's row of its page. Token i of
// sequence b sits at pos = seq_lens[b] - q_len + i.
//
// Two kernels. The down projection at decode sizes (a few hundred tokens, M in the
// thousands) has little work per output and much per K, so it is split over K:
// cache_write_gemm_kernel computes 128 tokens x 64 output columns over one slice of K
// (grid: token tiles x 9 column blocks x K slices) on the tensor cores (TMA stages of
// 64-wide K blocks, one elected lane issuing tcgen05.mma M=128 N=64, fp32 in TMEM) and
// writes its fp32 partial to the caller's workspace [slices][T][576].
// cache_write_finish_kernel (one CTA per token) adds the slices, normalises the latent
// part, turns the shared key, writes the bf16 row into the token's page, and turns the
// token's query rope planes in place.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace cw {

constexpr int kM = 128;       // tokens per CTA
constexpr int kKB = 64;       // K elements per block (one 128-byte swizzle row)
constexpr int kN = 64;        // output columns per CTA
constexpr int kR = 512, kDr = 64, kRow = kR + kDr, kPage = 64;
constexpr int kColBlocks = kRow / kN;   // 9
constexpr int kStages = 8;      // a slice's K blocks (up to 8) all in flight at once
constexpr int kMaxSlices = 16;

// K slices for hidden width M (a multiple of 64): enough CTAs to cover the GPU for a
// 128-token tile, each slice at least two 64-wide blocks.
__host__ __device__ constexpr int slices_for(int M) {
  return (M / kKB) >= 2 * kMaxSlices ? kMaxSlices : ((M / kKB) / 2 > 0 ? (M / kKB) / 2 : 1);
}

struct Params {
  __nv_bfloat16* kv;             // [num_pages][64][576]
  const int32_t* block_table;    // [B][max_pages]
  const int32_t* seq_lens;       // [B]
  const __nv_bfloat16* gain;     // [R] kv_rmsnorm gain
  float* part;                   // workspace [slices][T][576] fp32
  int32_t T, q_len, max_pages, num_pages, kblk, slices;   // kblk = M / 64
  float eps;
  double rope_base;
  uint64_t timeout_ns;
};

struct Cfg {
  static constexpr int kABytes = kM * kKB * 2;     // 16 KiB
  static constexpr int kBBytes = kN * kKB * 2;     // 8 KiB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kOffBar = kStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kCols = 64;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kM, kN, 0, 0);
};

__global__ void __launch_bounds__(128, 1)
cache_write_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const Params p) {
  using C = Cfg;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::kOffBar + 8u * i; };   // [0,S) full, [S,2S) empty, 2S done
  const uint32_t tmem_holder = sbase + C::kOffBar + 8u * (2 * kStages + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + 8 * (2 * kStages + 3));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kM, n0 = blockIdx.y * kN, slice = blockIdx.z;
  // this CTA's K blocks [kb0, kb1)
  const int kb0 = (int)((int64_t)p.kblk * slice / p.slices), kb1 = (int)((int64_t)p.kblk * (slice + 1) / p.slices);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(s), 1);
      ptx::mbar_init(bar(kStages + s), 1);
    }
    ptx::mbar_init(bar(2 * kStages), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_holder, C::kCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + C::kOffBar + 8 * (2 * kStages + 2));
  auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_bounded(b, parity, abort_flag, p.timeout_ns));
  };
  auto give_up = [&]() {
    if (lane == 0) {
      raise_status(kStatusTimeout);
      *abort_flag = 1;
    }
  };
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- loads
    const bool leader = ptx::elect_one();
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kStages, use = i / kStages;
      if (!wait_all(bar(kStages + s), (use & 1) ^ 1)) { give_up(); ok = false; break; }
      if (leader) {
        const uint32_t sa = sbase + s * C::kStageBytes, sb = sa + C::kABytes;
        ptx::mbar_arrive_expect_tx(bar(s), C::kStageBytes);
        ptx::tma_load_2d(sa, &tmA, bar(s), (kb0 + i) * kKB, m0);
        ptx::tma_load_2d(sb, &tmB, bar(s), (kb0 + i) * kKB, n0);
      }
    }
    for (int i = (nkb > kStages ? nkb - kStages : 0); i < nkb; ++i) wait_all(bar(i % kStages), (i / kStages) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const bool leader = ptx::elect_one();
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kStages, use = i / kStages;
      if (!wait_all(bar(s), use & 1)) { give_up(); ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t sa = sbase + s * C::kStageBytes, sb = sa + C::kABytes;
      const uint64_t dA = ptx::sdesc_sw128(sa, 16, 1024), dB = ptx::sdesc_sw128(sb, 16, 1024);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kKB / 16; ++kk)
          ptx::umma_f16_ss(tbase, dA + (uint64_t)((kk * 32) >> 4), dB + (uint64_t)((kk * 32) >> 4), C::kIdesc,
                           (i | kk) ? 1u : 0u);
        ptx::umma_commit(bar(kStages + s));
        if (i == nkb - 1) ptx::umma_commit(bar(2 * kStages));
      }
      __syncwarp();
    }
  }

  // ---------------------------------------------------------------- epilogue: the fp32 partial
  const bool done = ok && nkb > 0 && wait_all(bar(2 * kStages), 0);
  if (!done && nkb > 0) give_up();
  ptx::tc_fence_after();
  const int t = m0 + 32 * warp + lane;
  if (done) {
    float v[4][16];
#pragma unroll
    for (int q = 0; q < 4; ++q) ptx::tmem_ld_32x32b_x16(tbase + ((32u * warp) << 16) + 16 * q, v[q]);
    ptx::tmem_wait_ld();
    if (t < p.T) {
      float4* dst = reinterpret_cast<float4*>(p.part + ((int64_t)slice * p.T + t) * kRow + n0);
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[4 * q + j] = make_float4(v[q][4 * j], v[q][4 * j + 1], v[q][4 * j + 2], v[q][4 * j + 3]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, C::kCols);
  }
}

// One CTA of 256 threads per token. Thread i < 144 adds the slices of columns 4i..4i+3
// (all slices' loads in flight at once) while threads 224-255 compute the token's 32
// rotation angles (double precision: the position times the lowest frequency must keep
// its fraction of a turn) into shared memory; the latent part's sum of squares is
// reduced over the block; then threads < 128 write the normalised latent part, threads
// 128 + j (j < 32) turn the shared key's plane (512 + j, 544 + j), and, when q_rope is
// given, all threads turn the token's query rope planes (every head) in place.
constexpr int kFinishThreads = 256;
static_assert(kFinishThreads >= kR / 4 + kDr / 2 && kFinishThreads >= kRow / 4 + kDr / 2, "finish threads");
__global__ void __launch_bounds__(kFinishThreads)
cache_write_finish_kernel(const Params p, __nv_bfloat16* __restrict__ q_rope, int32_t H) {
  __shared__ float red[kFinishThreads / 32];
  __shared__ float key[kDr];
  __shared__ float cs[kDr / 2], sn[kDr / 2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = blockIdx.x;
  const int b = t / p.q_len, i = t % p.q_len;
  const int pos = p.seq_lens[b] - p.q_len + i;
  if (pos < 0) return;   // the same for every thread of the block
  const int32_t page = p.block_table[(int64_t)b * p.max_pages + pos / kPage];
  float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid < kRow / 4) {
    float4 v[kMaxSlices];
#pragma unroll
    for (int s = 0; s < kMaxSlices; ++s)
      if (s < p.slices)
        v[s] = __ldcs(reinterpret_cast<const float4*>(p.part + ((int64_t)s * p.T + t) * kRow) + tid);
#pragma unroll
    for (int s = 0; s < kMaxSlices; ++s)
      if (s < p.slices) {
        f.x += v[s].x;
        f.y += v[s].y;
        f.z += v[s].z;
        f.w += v[s].w;
      }
  } else if (tid >= kFinishThreads - kDr / 2) {
    const int j = tid - (kFinishThreads - kDr / 2);
    const double th = exp(-2.0 * (double)j / (double)kDr * log(p.rope_base));
    double s_, c_;
    sincos((double)pos * th, &s_, &c_);
    cs[j] = (float)c_;
    sn[j] = (float)s_;
  }
  float ss = tid < kR / 4 ? f.x * f.x + f.y * f.y + f.z * f.z + f.w * f.w : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  if (tid >= kR / 4 && tid < kRow / 4) {
    const int c = 4 * tid - kR;
    key[c] = f.x;
    key[c + 1] = f.y;
    key[c + 2] = f.z;
    key[c + 3] = f.w;
  }
  __syncthreads();
  if (q_rope) {
    // 8 threads per head, 4 planes each (8-byte accesses); a pass covers 32 heads x 4
    // groups, every load of a pass issued before any rotation
    constexpr int kPer = 4, kTph = (kDr / 2) / kPer, kHeadsPerGroup = kFinishThreads / kTph;
    const int j0 = (tid % kTph) * kPer;
    __nv_bfloat16* q = q_rope + (int64_t)t * H * kDr;
    for (int h0 = 0; h0 < H; h0 += 4 * kHeadsPerGroup) {
      uint2 a[4], c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int h = h0 + k * kHeadsPerGroup + tid / kTph;
        if (h < H) {
          const __nv_bfloat16* qh = q + (int64_t)h * kDr;
          a[k] = *reinterpret_cast<const uint2*>(qh + j0);
          c[k] = *reinterpret_cast<const uint2*>(qh + j0 + kDr / 2);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int h = h0 + k * kHeadsPerGroup + tid / kTph;
        if (h < H) {
          const __nv_bfloat162* x1 = reinterpret_cast<const __nv_bfloat162*>(&a[k]);
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&c[k]);
          uint2 ya, yc;
          __nv_bfloat162* y1 = reinterpret_cast<__nv_bfloat162*>(&ya);
          __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(&yc);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float2 u = __bfloat1622float2(x1[e]), w = __bfloat1622float2(x2[e]);
            const int j = j0 + 2 * e;
            y1[e] = __floats2bfloat162_rn(u.x * cs[j] - w.x * sn[j], u.y * cs[j + 1] - w.y * sn[j + 1]);
            y2[e] = __floats2bfloat162_rn(u.x * sn[j] + w.x * cs[j], u.y * sn[j + 1] + w.y * cs[j + 1]);
          }
          __nv_bfloat16* qh = q + (int64_t)h * kDr;
          *reinterpret_cast<uint2*>(qh + j0) = ya;
          *reinterpret_cast<uint2*>(qh + j0 + kDr / 2) = yc;
        }
      }
    }
  }
  if (page < 0 || page >= p.num_pages) {
    if (tid == 0) raise_status(kStatusBadPage);
    return;
  }
  __nv_bfloat16* row = p.kv + ((int64_t)page * kPage + pos % kPage) * kRow;
  if (tid < kR / 4) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kFinishThreads / 32; ++w) tot += red[w];
    const float inv = 1.f / sqrtf(tot / (float)kR + p.eps);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(p.gain) + 2 * tid;
    const float2 g0 = __bfloat1622float2(g2[0]), g1 = __bfloat1622float2(g2[1]);
    const __nv_bfloat162 a = __floats2bfloat162_rn(f.x * inv * g0.x, f.y * inv * g0.y);
    const __nv_bfloat162 c = __floats2bfloat162_rn(f.z * inv * g1.x, f.w * inv * g1.y);
    *reinterpret_cast<uint2*>(row + 4 * tid) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&c));
  } else if (tid < kR / 4 + kDr / 2) {
    const int j = tid - kR / 4;
    const float x1 = key[j], x2 = key[j + kDr / 2];
    row[kR + j] = __float2bfloat16_rn(x1 * cs[j] - x2 * sn[j]);
    row[kR + kDr / 2 + j] = __float2bfloat16_rn(x1 * sn[j] + x2 * cs[j]);
  }
}

}  // namespace cw
}  // namespace mla
