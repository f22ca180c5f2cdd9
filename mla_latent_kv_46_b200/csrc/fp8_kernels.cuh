// fp8_kernels.cuh -- the 8-bit (E4M3) latent cache: writing rows and preparing queries.
//
// Cache format (the softved page "Introduction to MLA vs. KV Cache in Large Language
// Models", "Practical Implementation Tips for MLA in LLM Serving", advises quantising the
// cache; the format is this library's reading): every element of a cached row [c ; k_rope]
// is an E4M3 code (OCP 8-bit floating point: bias 7, three mantissa bits, subnormals, no
// infinities, largest finite 448), and each row has one power-of-two scale 2^k stored as
// the byte k + 127. k is the smallest integer in [-126, 7] with max |x| <= 448 * 2^k; the
// code of x is x * 2^-k rounded to nearest (ties to even, saturating at 448). Scaling by a
// power of two is exact, so the row dequantises to code * 2^k exactly.
//
// The decode kernel scores against the codes with 8-bit tensor-core MMAs. Its query must
// then be 8-bit too: each bf16 query row [q_lat ; q_rope] is multiplied by 2^e (e the
// largest with max |q| 2^e <= 448) and split into two E4M3 pieces, hi = round(q 2^e) and
// lo = round(q 2^e - hi). A bf16 value has 8 significant bits and each piece carries 4, so
// hi + lo equals q 2^e except where the remainder is finer than E4M3's subnormal step
// (2^-9, i.e. elements below 2^-17 of the row's largest): the two MMAs over the pieces
// give the bf16 query's scores times 2^e.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace mla {
namespace f8 {

constexpr int kRow = 576;               // R + Dr
constexpr int kRowChunks = kRow / 8;    // 8-element chunks of a row
constexpr int kKMin = -126, kKMax = 7;

// Two floats to E4M3 (nearest even, saturating): a in the low byte.
__device__ __forceinline__ uint32_t to_e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
// The values of two E4M3 codes (low byte first), exactly.
__device__ __forceinline__ float2 from_e4m3x2(uint32_t v) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)v, __NV_E4M3);
  return __half22float2(__half2(h));
}
__device__ __forceinline__ float pow2(int e) { return __int_as_float((127 + e) << 23); }   // e in [-126, 127]

// Eight bf16 values of a 16-byte chunk.
__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Warp-wide maximum of a non-negative float.
__device__ __forceinline__ float warp_max_abs(float a) {
  return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
}

// ------------------------------------------------------------------ cache rows
// One warp per row of `src` (bf16 [n][576]): its codes and scale byte. Dense mode
// (block_table == nullptr): row r goes to row r of codes/scales. Append mode: row
// item = b * q_len + i goes to position seq_lens[b] - q_len + i of sequence b, as
// mla_cache_append places rows (positions < 0 skipped, bad page ids reported).
__global__ void __launch_bounds__(256) quantise_rows_kernel(const __nv_bfloat16* __restrict__ src,
                                                            uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales, int64_t n,
                                                            const int32_t* __restrict__ block_table,
                                                            const int32_t* __restrict__ seq_lens, int32_t q_len,
                                                            int32_t max_pages, int32_t num_pages,
                                                            int32_t page_size) {
  const int64_t item = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (item >= n) return;
  int64_t drow = item;
  if (block_table) {
    const int32_t b = (int32_t)(item / q_len), i = (int32_t)(item % q_len);
    const int32_t pos = seq_lens[b] - q_len + i;
    if (pos < 0) return;
    const int32_t pidx = pos / page_size;
    const int32_t page = pidx < max_pages ? block_table[(int64_t)b * max_pages + pidx] : -1;
    if (page < 0 || page >= num_pages) {
      if (lane == 0) raise_status(kStatusBadPage);
      return;
    }
    drow = (int64_t)page * page_size + pos % page_size;
  }
  const uint4* s = reinterpret_cast<const uint4*>(src + item * kRow);
  float x[3][8];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int c = lane + 32 * r;
    if (c < kRowChunks) {
      unpack8(s[c], x[r]);
#pragma unroll
      for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(x[r][k]));
    }
  }
  amax = warp_max_abs(amax);
  int k = kKMin;
  if (amax > 0.f) {
    int E;
    const float f = frexpf(amax, &E);   // amax = f 2^E, f in [0.5, 1); 448 = 0.875 2^9
    k = min(max(f <= 0.875f ? E - 9 : E - 8, kKMin), kKMax);
  }
  const float inv = pow2(-k);
  uint8_t* d = codes + drow * kRow;
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int c = lane + 32 * r;
    if (c < kRowChunks) {
      uint2 o;
      o.x = to_e4m3x2(x[r][0] * inv, x[r][1] * inv) | (to_e4m3x2(x[r][2] * inv, x[r][3] * inv) << 16);
      o.y = to_e4m3x2(x[r][4] * inv, x[r][5] * inv) | (to_e4m3x2(x[r][6] * inv, x[r][7] * inv) << 16);
      *reinterpret_cast<uint2*>(d + 8 * c) = o;
    }
  }
  if (lane == 0) scales[drow] = (uint8_t)(k + 127);
}

// ------------------------------------------------------------------ the split query
// One warp per query row (t, h): q8[0][row] = hi, q8[1][row] = lo (576 codes each),
// q_scale[row] = 2^-e.
__global__ void __launch_bounds__(256) split_query_kernel(const __nv_bfloat16* __restrict__ q_lat,
                                                          const __nv_bfloat16* __restrict__ q_rope,
                                                          uint8_t* __restrict__ q8, float* __restrict__ q_scale,
                                                          int64_t rows) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float x[3][8];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int c = lane + 32 * r;
    if (c < kRowChunks) {
      const uint4 v = c < 64 ? reinterpret_cast<const uint4*>(q_lat + row * 512)[c]
                             : reinterpret_cast<const uint4*>(q_rope + row * 64)[c - 64];
      unpack8(v, x[r]);
#pragma unroll
      for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(x[r][k]));
    }
  }
  amax = warp_max_abs(amax);
  int e = 0;
  if (amax > 0.f) {
    int E;
    const float f = frexpf(amax, &E);
    e = min(max(f <= 0.875f ? 9 - E : 8 - E, -126), 126);
  }
  const float up = pow2(e);
  uint8_t* hi = q8 + row * kRow;
  uint8_t* lo = q8 + (rows + row) * kRow;
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int c = lane + 32 * r;
    if (c < kRowChunks) {
      uint32_t h[4], l[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float a = x[r][2 * i] * up, b = x[r][2 * i + 1] * up;
        h[i] = to_e4m3x2(a, b);
        const float2 hv = from_e4m3x2(h[i]);
        l[i] = to_e4m3x2(a - hv.x, b - hv.y);
      }
      *reinterpret_cast<uint2*>(hi + 8 * c) = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
      *reinterpret_cast<uint2*>(lo + 8 * c) = make_uint2(l[0] | (l[1] << 16), l[2] | (l[3] << 16));
    }
  }
  if (lane == 0) q_scale[row] = pow2(-e);
}

}  // namespace f8
}  // namespace mla
