// prefill.cuh -- non-absorbed MLA prefill attention (causal) on tcgen05.
//
// The GatedMLA forward ("Build per-head Q, K and V", "Observe logits, then compute causal
// attention" of the kimi-k3 docs): every position of a sequence is a query; head h's keys
// are [K_c,h ; k_rope] with K_c,h = C W_UK[h]^T (the shared rope key broadcast to every
// head) and its values V_h = C W_UV[h]^T; softmax of scale * q . k over the keys at or
// before the query's position, times V. The up-projections run first as one GEMM each
// (gemm_tc.cuh, over all heads at once) into bf16 K_c [N][H][128] and V [N][H][128];
// this kernel is the attention.
//
// One CTA per (128-query tile of a sequence, head), cta_group::1, 256 threads:
//   warp 0  TMA producer: the query tile once (q_nope 2 boxes + q_rope 1 box, 48 KiB),
//           then per 128-key tile j the keys (K_c 2 boxes + k_rope 1 box) and the values
//           (2 boxes of 64 value columns), two stages each
//   warp 1  TMEM allocation and the MMA issuer: S = Q K^T (M=128, N=128, K=192, 12 MMAs),
//           then O += P V (M=128, N=128, K=128 keys, 8 MMAs; P from TMEM as the A operand,
//           V MN-major from shared memory), in the order S(0), [S(1), PV(0)], [S(2), PV(1)] ...
//   warps 4-7 the softmax: thread r owns query row r (TMEM lane r): it reads its 128 scores,
//           masks keys after its position (diagonal tile), keeps a lazily moved reference
//           maximum (O rescaled in TMEM only when a tile's maximum exceeds it by 2^8),
//           writes P = 2^(x - m) as bf16 and the remainder P_lo = bf16(p - bf16(p)) into
//           TMEM, and at the end writes O / l as bf16.
// P_lo enters a second value MMA on tiles where some row has 16 max p > l (l its running
// sum): where one key can carry a large share of a row, one bf16 rounding of P moves the
// output by more than the bf16 tolerance (the decode kernels do the same).
// TMEM (512 columns): S [0,128), P [128,256) (two buffers of 64), P_lo [256,384), O [384,512).
// Every wait is bounded; a CTA that gives up raises the device status word.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace pf {

constexpr int kM = 128, kN = 128;          // queries, keys per tile
constexpr int kDn = 128, kDr = 64, kDv = 128, kRow = 576;
constexpr int kBox = 128 * 128;            // 128 rows x 64 bf16 (128 B), 128-byte swizzle
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr int kOffQ = 0;                                   // 3 boxes
constexpr int kOffK = kOffQ + 3 * kBox;                    // stage x 3 boxes
constexpr int kOffV = kOffK + kStages * 3 * kBox;          // stage x 2 boxes
constexpr int kOffBar = kOffV + kStages * 2 * kBox;
enum {
  B_Q_FULL = 0,
  B_K_FULL,                        // +stage
  B_K_EMPTY = B_K_FULL + kStages,  // +stage
  B_V_FULL = B_K_EMPTY + kStages,  // +stage
  B_V_EMPTY = B_V_FULL + kStages,  // +stage
  B_S_FULL = B_V_EMPTY + kStages,
  B_S_EMPTY,
  B_P_FULL,                        // +buffer: the four softmax warps wrote P (and P_lo)
  B_P_DONE = B_P_FULL + 2,         // +buffer: the value MMAs that read the buffer are done
  B_O_DONE = B_P_DONE + 2,
  kNumBars
};
constexpr int kOffFlag = kOffBar + kNumBars * 8;           // uint32[2][4]: P_lo wanted, per buffer and warp
constexpr int kOffTmem = kOffFlag + 2 * 4 * 4;
constexpr int kOffAbort = kOffTmem + 8;
constexpr int kSmemBytes = kOffAbort + 8 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

constexpr uint32_t kColS = 0, kColP = 128, kColPlo = 256, kColO = 384;
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 128, 0, 0);   // Q (K-major) x K^T (K-major)
constexpr uint32_t kIdescV = ptx::idesc_bf16_f32(128, 128, 0, 1);   // P (TMEM) x V (MN-major)
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr float kLoShare = 16.0f;

struct Params {
  const int32_t* cu_seqlens;   // [B + 1] token offsets of the packed sequences
  int32_t B, H, max_qtiles;
  float scale_log2;
  __nv_bfloat16* out;          // [N][H][Dv]
  uint64_t timeout_ns;
};

// The tile of CTA x: tiles are taken longest first (query tile qt sees qt + 1 key tiles):
// for qt = max_qtiles - 1 down to 0, every sequence with more than qt tiles in order.
__device__ __forceinline__ bool tile_of(const Params& p, int32_t x, int32_t& b, int32_t& qt) {
  int32_t k = 0;
  for (int32_t t = p.max_qtiles - 1; t >= 0; --t) {
    for (int32_t s = 0; s < p.B; ++s) {
      const int32_t L = p.cu_seqlens[s + 1] - p.cu_seqlens[s];
      if ((L + kM - 1) / kM > t) {
        if (k == x) {
          b = s;
          qt = t;
          return true;
        }
        ++k;
      }
    }
  }
  return false;
}

__global__ void __launch_bounds__(kThreads, 1)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tm_qn, const __grid_constant__ CUtensorMap tm_qr,
                    const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_kr,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  volatile uint32_t* lo_flag = reinterpret_cast<volatile uint32_t*>(smem + kOffFlag);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  int32_t b = 0, qt = 0;
  if (!tile_of(p, blockIdx.x, b, qt)) return;   // (the grid has exactly one CTA per tile)
  const int32_t start = p.cu_seqlens[b], L = p.cu_seqlens[b + 1] - start;
  const int32_t nk = qt + 1;                    // key tiles 0..qt
  const int32_t q0 = start + kM * qt;           // first query row of the tile (packed index)

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 8; ++i) lo_flag[i] = 0u;
    ptx::mbar_init(bar(B_Q_FULL), 1);
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(B_K_FULL + s), 1);
      ptx::mbar_init(bar(B_K_EMPTY + s), 1);
      ptx::mbar_init(bar(B_V_FULL + s), 1);
      ptx::mbar_init(bar(B_V_EMPTY + s), 1);
    }
    ptx::mbar_init(bar(B_S_FULL), 1);
    ptx::mbar_init(bar(B_S_EMPTY), 4);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(B_P_FULL + i), 4);
      ptx::mbar_init(bar(B_P_DONE + i), 1);
    }
    ptx::mbar_init(bar(B_O_DONE), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(sbase + kOffTmem, 512);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_qn);
    ptx::prefetch_tmap(&tm_qr);
    ptx::prefetch_tmap(&tm_kc);
    ptx::prefetch_tmap(&tm_kr);
    ptx::prefetch_tmap(&tm_v);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  auto fail = [&]() {
    raise_status(kStatusTimeout);
    *abort_flag = 1;
  };
  auto wait_all = [&](uint32_t bb, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_bounded(bb, parity, abort_flag, p.timeout_ns));
  };

  if (warp == 0) {
    // ================================================================ TMA producer
    const bool leader = ptx::elect_one();
    if (leader) {
      ptx::mbar_arrive_expect_tx(bar(B_Q_FULL), 3 * kBox);
      ptx::tma_load_2d(sbase + kOffQ, &tm_qn, bar(B_Q_FULL), h * kDn, q0);
      ptx::tma_load_2d(sbase + kOffQ + kBox, &tm_qn, bar(B_Q_FULL), h * kDn + 64, q0);
      ptx::tma_load_2d(sbase + kOffQ + 2 * kBox, &tm_qr, bar(B_Q_FULL), h * kDr, q0);
    }
    bool ok = true;
    for (int32_t j = 0; j < nk && ok; ++j) {
      const uint32_t s = j % kStages, ph = (j / kStages) & 1;
      const int32_t k0 = start + kN * j;
      if (!wait_all(bar(B_K_EMPTY + s), ph ^ 1)) { if (leader) fail(); ok = false; break; }
      if (leader) {
        const uint32_t dst = sbase + kOffK + s * 3 * kBox;
        ptx::mbar_arrive_expect_tx(bar(B_K_FULL + s), 3 * kBox);
        ptx::tma_load_2d(dst, &tm_kc, bar(B_K_FULL + s), h * kDn, k0);
        ptx::tma_load_2d(dst + kBox, &tm_kc, bar(B_K_FULL + s), h * kDn + 64, k0);
        ptx::tma_load_2d(dst + 2 * kBox, &tm_kr, bar(B_K_FULL + s), 512, k0);
      }
      if (!wait_all(bar(B_V_EMPTY + s), ph ^ 1)) { if (leader) fail(); ok = false; break; }
      if (leader) {
        const uint32_t dst = sbase + kOffV + s * 2 * kBox;
        ptx::mbar_arrive_expect_tx(bar(B_V_FULL + s), 2 * kBox);
        ptx::tma_load_2d(dst, &tm_v, bar(B_V_FULL + s), h * kDv, k0);
        ptx::tma_load_2d(dst + kBox, &tm_v, bar(B_V_FULL + s), h * kDv + 64, k0);
      }
    }
    // copies still in flight land before the CTA exits (bounded; abort-independent)
    for (int32_t j = (nk > kStages ? nk - kStages : 0); j < nk; ++j) {
      const uint32_t s = j % kStages, ph = (j / kStages) & 1;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster_timed(bar(B_K_FULL + s), ph, p.timeout_ns))) break;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster_timed(bar(B_V_FULL + s), ph, p.timeout_ns))) break;
    }
    __all_sync(0xffffffffu, ptx::mbar_wait_cluster_timed(bar(B_Q_FULL), 0, p.timeout_ns));
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    const bool leader = ptx::elect_one();
    bool ok = wait_all(bar(B_Q_FULL), 0);
    if (!ok && leader) fail();
    ptx::tc_fence_after();
    const uint64_t dq = ptx::sdesc_sw128(sbase + kOffQ, 16, 1024);
    auto issue_s = [&](int32_t j) -> bool {
      const uint32_t s = j % kStages, ph = (j / kStages) & 1;
      if (!wait_all(bar(B_K_FULL + s), ph)) return false;
      if (!wait_all(bar(B_S_EMPTY), (j & 1) ^ 1)) return false;   // the softmax read S(j - 1)
      ptx::tc_fence_after();
      if (leader) {
        const uint64_t dk = ptx::sdesc_sw128(sbase + kOffK + s * 3 * kBox, 16, 1024);
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_ss(tbase + kColS, dq + (uint64_t)((c * kBox + kk * 32) >> 4),
                             dk + (uint64_t)((c * kBox + kk * 32) >> 4), kIdescS, (c | kk) ? 1u : 0u);
        ptx::umma_commit(bar(B_K_EMPTY + s));
        ptx::umma_commit(bar(B_S_FULL));
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](int32_t i) -> bool {
      const uint32_t s = i % kStages, ph = (i / kStages) & 1, pb = i & 1;
      if (!wait_all(bar(B_P_FULL + pb), (i >> 1) & 1)) return false;
      if (!wait_all(bar(B_V_FULL + s), ph)) return false;
      const uint32_t want_lo = lo_flag[4 * pb] | lo_flag[4 * pb + 1] | lo_flag[4 * pb + 2] | lo_flag[4 * pb + 3];
      ptx::tc_fence_after();
      if (leader) {
        const uint32_t vb = sbase + kOffV + s * 2 * kBox;
#pragma unroll 1
        for (int part = 0; part < (want_lo ? 2 : 1); ++part) {
          const uint32_t ta = tbase + (part ? kColPlo : kColP) + 64u * pb;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            ptx::umma_f16_ts(tbase + kColO, ta + 8u * kk, ptx::sdesc_sw128(vb + kk * 2048, kBox, 1024), kIdescV,
                             (i | part | kk) ? 1u : 0u);
        }
        ptx::umma_commit(bar(B_V_EMPTY + s));
        ptx::umma_commit(bar(B_P_DONE + pb));
        if (i == nk - 1) ptx::umma_commit(bar(B_O_DONE));
      }
      __syncwarp();
      return true;
    };
    if (ok) ok = issue_s(0);
    for (int32_t j = 1; j < nk && ok; ++j) {
      ok = issue_s(j);
      if (ok) ok = issue_pv(j - 1);
    }
    if (ok) ok = issue_pv(nk - 1);
    if (!ok && leader) fail();
  } else if (warp >= 4) {
    // ================================================================ softmax and epilogue
    const int sw = warp - 4;
    const int r = 32 * sw + lane;                       // query row of the tile, TMEM lane
    const uint32_t lane_addr = (32u * sw) << 16;
    const int32_t qpos = kM * qt + r;                   // position in the sequence
    float m_ref = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    for (int32_t j = 0; j < nk && ok; ++j) {
      const uint32_t pb = j & 1;
      if (!wait_all(bar(B_S_FULL), j & 1)) { fail(); ok = false; break; }
      ptx::tc_fence_after();
      float x[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[32];
        ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColS + 32u * c, v);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) x[32 * c + t] = __uint_as_float(v[t]) * p.scale_log2;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_S_EMPTY));
      if (j == qt) {
        // diagonal tile: keys after the query's position are not seen
#pragma unroll
        for (int t = 0; t < 128; ++t) x[t] = (t <= r) ? x[t] : -CUDART_INF_F;
      }
      float mx = x[0];
#pragma unroll
      for (int t = 1; t < 128; ++t) mx = fmaxf(mx, x[t]);
      // a row whose tile maximum exceeds its reference by more than the threshold moves the
      // reference; O is rescaled for the whole warp when any of its rows moved (factor 1
      // for the others), so the warp's waits and TMEM accesses stay convergent
      const bool need = mx > m_ref + kRescaleThreshold;
      const float al = need ? ptx::ex2(m_ref - mx) : 1.f;   // (0 on the first tile: l and O are 0)
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // O holds the sums over tiles < j: rescale once the value MMAs of tile j - 1 are done
        if (!wait_all(bar(B_P_DONE + ((j - 1) & 1)), ((j - 1) >> 1) & 1)) { fail(); ok = false; break; }
        ptx::tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColO + 32u * c, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * al);
          ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColO + 32u * c, o);
        }
        ptx::tmem_wait_st();
      }
      l *= al;
      if (need) m_ref = mx;
      // P buffer pb was last read by the value MMAs of tile j - 2
      if (j >= 2 && !wait_all(bar(B_P_DONE + pb), ((j >> 1) & 1) ^ 1)) { fail(); ok = false; break; }
      ptx::tc_fence_after();
      float sum = 0.f, pmax = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t ph[32], pl[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a0 = ptx::ex2(x[64 * c + 2 * i] - m_ref);
          const float a1 = ptx::ex2(x[64 * c + 2 * i + 1] - m_ref);
          sum += a0 + a1;
          pmax = fmaxf(pmax, fmaxf(a0, a1));
          __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
          ph[i] = *reinterpret_cast<uint32_t*>(&h2);
          __nv_bfloat162 l2 =
              __floats2bfloat162_rn(a0 - __uint_as_float(ph[i] << 16), a1 - __uint_as_float(ph[i] & 0xFFFF0000u));
          pl[i] = *reinterpret_cast<uint32_t*>(&l2);
        }
        ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColP + 64u * pb + 32u * c, ph);
        ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColPlo + 64u * pb + 32u * c, pl);
      }
      l += sum;
      const bool want_lo = pmax * kLoShare > l;
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      const uint32_t any_lo = __any_sync(0xffffffffu, want_lo) ? 1u : 0u;
      __syncwarp();
      if (lane == 0) {
        lo_flag[4 * pb + sw] = any_lo;
        ptx::mbar_arrive(bar(B_P_FULL + pb));
      }
    }
    // O / l to the output once the last value MMAs are done
    if (ok && wait_all(bar(B_O_DONE), 0)) {
      ptx::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const bool valid = qpos < L;
      __nv_bfloat16* dst = p.out + ((int64_t)(q0 + r) * p.H + h) * kDv;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColO + 32u * c, o);
        ptx::tmem_wait_ld();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            w[i] = *reinterpret_cast<uint32_t*>(&b2);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
          for (int k = 0; k < 4; ++k) d4[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
    } else if (ok) {
      fail();
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, 512);
  }
}

}  // namespace pf
}  // namespace mla
