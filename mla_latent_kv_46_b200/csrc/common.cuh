// common.cuh -- shared definitions of the MLA decode library's kernels and host
// code: the device status word, the split-plan layout and small numeric helpers.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

namespace mla {

// Device status word (one per device; read and cleared by mla_check_status).
enum : unsigned int { kStatusTimeout = 1u, kStatusBadPage = 2u };
__device__ unsigned int g_status;

__device__ __forceinline__ void raise_status(unsigned int bits) { atomicOr(&g_status, bits); }

// ------------------------------------------------------------------ split plan
// int32 words:
//   [0] magic  [1] B  [2] q_len  [3] num_units  [4] num_slots  [5] num_parts
//   [6] head_groups  [7] H  [8] page_size  [9..15] 0
//   units      @16                      kUnitWords words per unit (see Unit)
//   slot_begin @16 + kUnitWords*num_units      num_slots + 1 words (unit index)
//   item_parts @slot_begin + num_slots + 1     2 words per item {first_part, num_parts}
constexpr int32_t kPlanMagic = 0x4D4C4131;  // "MLA1"
constexpr int kPlanHeader = 16;
constexpr int kUnitWords = 8;

struct Unit {
  int32_t item;        // query token index b*q_len + i
  int32_t b;           // sequence
  int32_t page_begin;  // first page (within the sequence's page list)
  int32_t page_end;    // one past the last page
  int32_t part;        // partial-output index, or -1: the unit writes the final result
  int32_t slot;
  int32_t pad0, pad1;
};

struct PlanView {
  const int32_t* w;
  __host__ __device__ int32_t B() const { return w[1]; }
  __host__ __device__ int32_t q_len() const { return w[2]; }
  __host__ __device__ int32_t num_units() const { return w[3]; }
  __host__ __device__ int32_t num_slots() const { return w[4]; }
  __host__ __device__ int32_t num_parts() const { return w[5]; }
  __host__ __device__ int32_t head_groups() const { return w[6]; }
  __host__ __device__ const Unit* units() const {
    return reinterpret_cast<const Unit*>(w + kPlanHeader);
  }
  __host__ __device__ const int32_t* slot_begin() const {
    return w + kPlanHeader + kUnitWords * num_units();
  }
  __host__ __device__ const int32_t* item_parts() const { return slot_begin() + num_slots() + 1; }
};

// Tokens seen by query i of the newest q_len-token chunk of a sequence of L tokens.
__host__ __device__ __forceinline__ int32_t visible_tokens(int32_t L, int32_t q_len, int32_t i) {
  int32_t n = L - q_len + i + 1;
  return n > 0 ? n : 0;
}

// ------------------------------------------------------------------ element access
template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace mla
