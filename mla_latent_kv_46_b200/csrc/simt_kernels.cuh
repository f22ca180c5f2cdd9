// simt_kernels.cuh -- CUDA-core kernels of every step, for any geometry and for
// fp32 as well as bf16 storage. The tensor-core kernels replace some of them
// where the geometry allows (see decode_tc.cuh, gemm_tc.cuh).
#pragma once

#include "common.cuh"

namespace mla {
namespace simt {

// ------------------------------------------------------------------ a2: cache append
// One warp per new row, 16-byte copies (rows whose byte size is a multiple of 16):
// kv[page][pos % ps][:] = new_ckr[b*q_len + i][:].
__global__ void __launch_bounds__(128) cache_append_vec_kernel(uint4* __restrict__ kv, const int32_t* __restrict__ block_table,
                                                               const int32_t* __restrict__ seq_lens,
                                                               const uint4* __restrict__ new_ckr, int32_t items,
                                                               int32_t q_len, int32_t max_pages, int32_t num_pages,
                                                               int32_t row_vec, int32_t page_size) {
  const int32_t item = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (item >= items) return;
  const int32_t b = item / q_len, i = item % q_len;
  // rows of up to 96 vectors (bf16 576-wide: 72) are read into registers before the
  // length and page lookups, so the row's load does not wait behind them
  constexpr int kHeld = 3;
  const uint4* src = new_ckr + (int64_t)item * row_vec;
  const bool held = row_vec <= 32 * kHeld;
  uint4 v[kHeld];
  if (held) {
#pragma unroll
    for (int k = 0; k < kHeld; ++k) {
      const int32_t e = lane + 32 * k;
      if (e < row_vec) v[k] = src[e];
    }
  }
  const int32_t pos = seq_lens[b] - q_len + i;
  if (pos < 0) return;
  const int32_t pidx = pos / page_size;
  if (pidx >= max_pages) {
    if (lane == 0) raise_status(kStatusBadPage);
    return;
  }
  const int32_t page = block_table[(int64_t)b * max_pages + pidx];
  if (page < 0 || page >= num_pages) {
    if (lane == 0) raise_status(kStatusBadPage);
    return;
  }
  uint4* dst = kv + ((int64_t)page * page_size + pos % page_size) * row_vec;
  if (held) {
#pragma unroll
    for (int k = 0; k < kHeld; ++k) {
      const int32_t e = lane + 32 * k;
      if (e < row_vec) dst[e] = v[k];
    }
    return;
  }
  for (int32_t e = lane; e < row_vec; e += 32) dst[e] = src[e];
}

// One block per new row, element copies (any row width).
template <typename T>
__global__ void cache_append_kernel(T* __restrict__ kv, const int32_t* __restrict__ block_table,
                                    const int32_t* __restrict__ seq_lens,
                                    const T* __restrict__ new_ckr, int32_t q_len, int32_t max_pages,
                                    int32_t num_pages, int32_t row, int32_t page_size) {
  const int32_t item = blockIdx.x;
  const int32_t b = item / q_len, i = item % q_len;
  const int32_t pos = seq_lens[b] - q_len + i;
  if (pos < 0) return;
  const int32_t pidx = pos / page_size;
  if (pidx >= max_pages) {
    if (threadIdx.x == 0) raise_status(kStatusBadPage);
    return;
  }
  const int32_t page = block_table[(int64_t)b * max_pages + pidx];
  if (page < 0 || page >= num_pages) {
    if (threadIdx.x == 0) raise_status(kStatusBadPage);
    return;
  }
  T* dst = kv + ((int64_t)page * page_size + pos % page_size) * row;
  const T* src = new_ckr + (int64_t)item * row;
  for (int32_t e = threadIdx.x; e < row; e += blockDim.x) dst[e] = src[e];
}

// ------------------------------------------------------------------ a1: absorb
// q_lat[t][h][r] = sum_n q_nope[t][h][n] * W_UK[h][n][r]
// grid (ceil(R/128), H, ceil(T/kTT)), block 128: thread = one r, kTT tokens.
constexpr int kTT = 8;
template <typename T>
__global__ void absorb_kernel(const T* __restrict__ qn, const T* __restrict__ w, T* __restrict__ ql,
                              int32_t T_, int32_t H, int32_t Dn, int32_t R) {
  extern __shared__ float sq[];  // [kTT][Dn]
  const int32_t h = blockIdx.y, t0 = blockIdx.z * kTT;
  const int32_t r = blockIdx.x * blockDim.x + threadIdx.x;
  for (int32_t e = threadIdx.x; e < kTT * Dn; e += blockDim.x) {
    const int32_t t = t0 + e / Dn, n = e % Dn;
    sq[e] = t < T_ ? to_f32(qn[((int64_t)t * H + h) * Dn + n]) : 0.f;
  }
  __syncthreads();
  if (r >= R) return;
  float acc[kTT];
#pragma unroll
  for (int k = 0; k < kTT; ++k) acc[k] = 0.f;
  const T* wp = w + (int64_t)h * Dn * R + r;
  for (int32_t n = 0; n < Dn; ++n) {
    const float wv = to_f32(wp[(int64_t)n * R]);
#pragma unroll
    for (int k = 0; k < kTT; ++k) acc[k] = fmaf(sq[k * Dn + n], wv, acc[k]);
  }
#pragma unroll
  for (int k = 0; k < kTT; ++k)
    if (t0 + k < T_) ql[((int64_t)(t0 + k) * H + h) * R + r] = from_f32<T>(acc[k]);
}

// ------------------------------------------------------------------ a7: output projection
// out[t][h][v] = sum_r W_UV[h][v][r] * o_lat[t][h][r]
// grid (H, ceil(T/kTT)), block 256: the kTT latent rows in shared memory, one warp per v.
template <typename T>
__global__ void outproj_kernel(const float* __restrict__ ol, const T* __restrict__ w, T* __restrict__ out,
                               int32_t T_, int32_t H, int32_t Dv, int32_t R) {
  extern __shared__ float so[];  // [kTT][R]
  const int32_t h = blockIdx.x, t0 = blockIdx.y * kTT;
  for (int32_t e = threadIdx.x; e < kTT * R; e += blockDim.x) {
    const int32_t t = t0 + e / R, r = e % R;
    so[e] = t < T_ ? ol[((int64_t)t * H + h) * R + r] : 0.f;
  }
  __syncthreads();
  const int32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarp = blockDim.x >> 5;
  for (int32_t v = warp; v < Dv; v += nwarp) {
    const T* wp = w + ((int64_t)h * Dv + v) * R;
    float acc[kTT];
#pragma unroll
    for (int k = 0; k < kTT; ++k) acc[k] = 0.f;
    for (int32_t r = lane; r < R; r += 32) {
      const float wv = to_f32(wp[r]);
#pragma unroll
      for (int k = 0; k < kTT; ++k) acc[k] = fmaf(wv, so[k * R + r], acc[k]);
    }
#pragma unroll
    for (int k = 0; k < kTT; ++k) {
      const float s = warp_sum(acc[k]);
      if (lane == 0 && t0 + k < T_) out[((int64_t)(t0 + k) * H + h) * Dv + v] = from_f32<T>(s);
    }
  }
}

// ------------------------------------------------------------------ a3-a5: decode attention
// grid (num_units, H), block 128. Each warp runs an online softmax over every
// 4th visible token of the unit; the four warp states are merged at the end.
struct DecodeSimtArgs {
  const int32_t* plan;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int32_t max_pages, num_pages, H, R, Dr, page_size;
  float scale;
  void* o_lat;        // fp32 [T][H][R]
  float* lse;
  float* o_part;
  float* lse_part;
};

template <typename T>
__global__ void decode_kernel(const T* __restrict__ q_lat, const T* __restrict__ q_rope,
                              const T* __restrict__ kv, DecodeSimtArgs a) {
  extern __shared__ float smem[];
  const int32_t row = a.R + a.Dr;
  float* qs = smem;                   // [row]
  float* os = qs + row;               // [4][R]
  float* ms = os + 4 * a.R;           // [4]
  float* ls = ms + 4;                 // [4]
  const PlanView plan{a.plan};
  const Unit u = plan.units()[blockIdx.x];
  const int32_t h = blockIdx.y;
  const int32_t q_len = plan.q_len();
  const int32_t L = a.seq_lens[u.b];
  const int32_t n = visible_tokens(L, q_len, u.item % q_len);
  const int32_t tb = u.page_begin * a.page_size;
  const int32_t te = min(u.page_end * a.page_size, n);
  const int32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int32_t e = threadIdx.x; e < row; e += blockDim.x)
    qs[e] = e < a.R ? to_f32(q_lat[((int64_t)u.item * a.H + h) * a.R + e])
                    : to_f32(q_rope[((int64_t)u.item * a.H + h) * a.Dr + (e - a.R)]);
  float* ow = os + warp * a.R;
  for (int32_t e = lane; e < a.R; e += 32) ow[e] = 0.f;
  __syncthreads();

  float m = -CUDART_INF_F, l = 0.f;
  for (int32_t t = tb + warp; t < te; t += 4) {
    const int32_t page = a.block_table[(int64_t)u.b * a.max_pages + t / a.page_size];
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0) raise_status(kStatusBadPage);
      continue;
    }
    const T* rp = kv + ((int64_t)page * a.page_size + t % a.page_size) * row;
    float part = 0.f;
    for (int32_t e = lane; e < row; e += 32) part = fmaf(qs[e], to_f32(rp[e]), part);
    const float x = warp_sum(part) * a.scale;
    const float m_new = fmaxf(m, x);
    const float corr = expf(m - m_new);  // 0 on the first token (m = -inf)
    const float p = expf(x - m_new);
    l = l * corr + p;
    for (int32_t e = lane; e < a.R; e += 32) ow[e] = fmaf(p, to_f32(rp[e]), ow[e] * corr);
    m = m_new;
  }
  if (lane == 0) {
    ms[warp] = m;
    ls[warp] = l;
  }
  __syncthreads();
  float M = fmaxf(fmaxf(ms[0], ms[1]), fmaxf(ms[2], ms[3]));
  float wgt[4], tot = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    wgt[k] = (M == -CUDART_INF_F) ? 0.f : expf(ms[k] - M);
    tot += wgt[k] * ls[k];
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  const float lse_v = tot > 0.f ? M + logf(tot) : -CUDART_INF_F;
  if (u.part < 0) {
    float* dst = static_cast<float*>(a.o_lat) + ((int64_t)u.item * a.H + h) * a.R;
    for (int32_t e = threadIdx.x; e < a.R; e += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) s = fmaf(wgt[k], os[k * a.R + e], s);
      dst[e] = s * inv;
    }
    if (threadIdx.x == 0 && a.lse) a.lse[(int64_t)u.item * a.H + h] = lse_v;
  } else {
    float* dst = a.o_part + ((int64_t)u.part * a.H + h) * a.R;
    for (int32_t e = threadIdx.x; e < a.R; e += blockDim.x) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) s = fmaf(wgt[k], os[k * a.R + e], s);
      dst[e] = s * inv;
    }
    if (threadIdx.x == 0) a.lse_part[(int64_t)u.part * a.H + h] = lse_v;
  }
}

// ------------------------------------------------------------------ a6: split-KV combine
// grid (num_items, H), block 128. Items computed by a single unit are skipped.
__global__ void combine_kernel(const int32_t* __restrict__ plan_w, const float* __restrict__ o_part,
                               const float* __restrict__ lse_part, float* __restrict__ o_lat,
                               float* __restrict__ lse, int32_t H, int32_t R) {
  const PlanView plan{plan_w};
  const int32_t item = blockIdx.x, h = blockIdx.y;
  const int32_t first = plan.item_parts()[2 * item], np = plan.item_parts()[2 * item + 1];
  if (np == 0) return;
  float M = -CUDART_INF_F;
  for (int32_t s = 0; s < np; ++s) M = fmaxf(M, lse_part[(int64_t)(first + s) * H + h]);
  float tot = 0.f;
  for (int32_t s = 0; s < np; ++s) {
    const float z = lse_part[(int64_t)(first + s) * H + h];
    tot += (M == -CUDART_INF_F) ? 0.f : expf(z - M);
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  for (int32_t e = threadIdx.x; e < R; e += blockDim.x) {
    float acc = 0.f;
    for (int32_t s = 0; s < np; ++s) {
      const float z = lse_part[(int64_t)(first + s) * H + h];
      const float wgt = (M == -CUDART_INF_F) ? 0.f : expf(z - M);
      if (wgt > 0.f) acc = fmaf(wgt, o_part[((int64_t)(first + s) * H + h) * R + e], acc);
    }
    o_lat[((int64_t)item * H + h) * R + e] = acc * inv;
  }
  if (threadIdx.x == 0 && lse) lse[(int64_t)item * H + h] = tot > 0.f ? M + logf(tot) : -CUDART_INF_F;
}

// Same merge, one warp per (item, head), rows of R <= 512 (R % 4 == 0) as float4:
// grid (num_items, ceil(H / 4)), block 128. One pass over the parts, two at a time, each
// part's lse loaded together with its row (a single round trip to memory per pair):
// the running maximum M and the sums are rescaled when a part raises M, as an online
// softmax does, so the result equals the max-first merge up to fp32 rounding.
__global__ void __launch_bounds__(128) combine_vec_kernel(const int32_t* __restrict__ plan_w,
                                                          const float* __restrict__ o_part,
                                                          const float* __restrict__ lse_part,
                                                          float* __restrict__ o_lat, float* __restrict__ lse,
                                                          int32_t H, int32_t R) {
  const PlanView plan{plan_w};
  const int32_t item = blockIdx.x;
  const int32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t h = blockIdx.y * 4 + warp;
  if (h >= H) return;
  const int32_t first = plan.item_parts()[2 * item], np = plan.item_parts()[2 * item + 1];
  if (np == 0) return;
  const int32_t nv = R / 4;
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  float M = -CUDART_INF_F, tot = 0.f;
  for (int32_t s = 0; s < np; s += 2) {
    const bool two = s + 1 < np;
    float z[2];
    float4 v[2][4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int32_t ps = first + s + (q && two ? 1 : 0);
      z[q] = (q && !two) ? -CUDART_INF_F : lse_part[(int64_t)ps * H + h];
      const float4* src = reinterpret_cast<const float4*>(o_part + ((int64_t)ps * H + h) * R);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int32_t i = lane + 32 * k;
        v[q][k] = i < nv ? __ldcs(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const float Mn = fmaxf(M, fmaxf(z[0], z[1]));
    if (Mn == -CUDART_INF_F) continue;   // no part so far saw a token
    const float r = expf(M - Mn);        // 0 while M is -inf
    const float w0 = expf(z[0] - Mn), w1 = expf(z[1] - Mn);
    tot = tot * r + (w0 + w1);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[k].x = fmaf(w1, v[1][k].x, fmaf(w0, v[0][k].x, acc[k].x * r));
      acc[k].y = fmaf(w1, v[1][k].y, fmaf(w0, v[0][k].y, acc[k].y * r));
      acc[k].z = fmaf(w1, v[1][k].z, fmaf(w0, v[0][k].z, acc[k].z * r));
      acc[k].w = fmaf(w1, v[1][k].w, fmaf(w0, v[0][k].w, acc[k].w * r));
    }
    M = Mn;
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  float* dst = o_lat + ((int64_t)item * H + h) * R;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int32_t i = lane + 32 * k;
    if (i < nv)
      *reinterpret_cast<float4*>(dst + 4 * i) =
          make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
  }
  if (lane == 0 && lse) lse[(int64_t)item * H + h] = tot > 0.f ? M + logf(tot) : -CUDART_INF_F;
}

// The same merge with one (item, head)'s parts spread over W warps: grid (num_items, H),
// block 32 W, rows of R <= 512 (R % 4 == 0). Warp w merges parts w, w + W, w + 2W, ...
// online, two per round trip, as combine_vec_kernel does, and the W running (maximum,
// sum, row) triples are then merged through shared memory. For plans that cut a few
// queries into many parts (long sequences spread over every slot), where one warp's serial
// pass over all of a query's parts would set the kernel's duration.
template <int W>
__global__ void __launch_bounds__(32 * W) combine_wide_kernel(const int32_t* __restrict__ plan_w,
                                                              const float* __restrict__ o_part,
                                                              const float* __restrict__ lse_part,
                                                              float* __restrict__ o_lat, float* __restrict__ lse,
                                                              int32_t H, int32_t R) {
  __shared__ float s_m[W], s_t[W];
  __shared__ float4 s_acc[W][128];
  const PlanView plan{plan_w};
  const int32_t item = blockIdx.x, h = blockIdx.y;
  const int32_t warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t first = plan.item_parts()[2 * item], np = plan.item_parts()[2 * item + 1];
  if (np == 0) return;   // the same for every thread of the block
  const int32_t nv = R / 4;
  float4 acc[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  float M = -CUDART_INF_F, tot = 0.f;
  for (int32_t s = warp; s < np; s += 2 * W) {
    const bool two = s + W < np;
    float z[2];
    float4 v[2][4];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int32_t ps = first + s + (q && two ? W : 0);
      z[q] = (q && !two) ? -CUDART_INF_F : lse_part[(int64_t)ps * H + h];
      const float4* src = reinterpret_cast<const float4*>(o_part + ((int64_t)ps * H + h) * R);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int32_t i = lane + 32 * k;
        v[q][k] = i < nv ? __ldcs(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    const float Mn = fmaxf(M, fmaxf(z[0], z[1]));
    if (Mn == -CUDART_INF_F) continue;   // no part so far saw a token
    const float r = expf(M - Mn);        // 0 while M is -inf
    const float w0 = expf(z[0] - Mn), w1 = expf(z[1] - Mn);
    tot = tot * r + (w0 + w1);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[k].x = fmaf(w1, v[1][k].x, fmaf(w0, v[0][k].x, acc[k].x * r));
      acc[k].y = fmaf(w1, v[1][k].y, fmaf(w0, v[0][k].y, acc[k].y * r));
      acc[k].z = fmaf(w1, v[1][k].z, fmaf(w0, v[0][k].z, acc[k].z * r));
      acc[k].w = fmaf(w1, v[1][k].w, fmaf(w0, v[0][k].w, acc[k].w * r));
    }
    M = Mn;
  }
  // merge the warps' triples: each row rescaled to the common maximum
  if (lane == 0) {
    s_m[warp] = M;
    s_t[warp] = tot;
  }
  __syncthreads();
  float Mx = -CUDART_INF_F;
#pragma unroll
  for (int w = 0; w < W; ++w) Mx = fmaxf(Mx, s_m[w]);
  const float f = M == -CUDART_INF_F ? 0.f : expf(M - Mx);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int32_t i = lane + 32 * k;
    if (i < nv) s_acc[warp][i] = make_float4(acc[k].x * f, acc[k].y * f, acc[k].z * f, acc[k].w * f);
  }
  __syncthreads();
  float T = 0.f;
#pragma unroll
  for (int w = 0; w < W; ++w) T += s_m[w] == -CUDART_INF_F ? 0.f : s_t[w] * expf(s_m[w] - Mx);
  const float inv = T > 0.f ? 1.f / T : 0.f;
  float* dst = o_lat + ((int64_t)item * H + h) * R;
  for (int32_t i = threadIdx.x; i < nv; i += 32 * W) {
    float4 a = s_acc[0][i];
#pragma unroll
    for (int w = 1; w < W; ++w) {
      const float4 b = s_acc[w][i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    *reinterpret_cast<float4*>(dst + 4 * i) = make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
  }
  if (threadIdx.x == 0 && lse) lse[(int64_t)item * H + h] = T > 0.f ? Mx + logf(T) : -CUDART_INF_F;
}

}  // namespace simt
}  // namespace mla
