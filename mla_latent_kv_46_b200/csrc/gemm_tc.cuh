// gemm_tc.cuh -- the per-head projections of the decode step on sm_100a tensor cores.
//
//   absorb   q_lat[t][h][:] = q_nope[t][h][:] @ W_UK[h]     A [T x Dn] (K-major),
//            B = W_UK[h] [Dn x R]: K rows, N = R contiguous (MN-major)
//   outproj  out[t][h][:]   = o_lat[t][h][:] @ W_UV[h]^T    A [T x R] fp32 (K-major),
//            B = W_UV[h] [Dv x R]: N rows, K = R contiguous (K-major); proj_a32_kernel
//            below splits each fp32 A element into bf16 hi + lo
//
// One CTA computes a 128-row tile of tokens x N output columns (block blockIdx.z of the
// output row) for one head: TMA streams 64-wide K blocks of A and B into a ring of stages
// (128-byte swizzle), one elected lane issues tcgen05.mma (M=128, N <= 256 per
// instruction, fp32 accumulators in TMEM), and the four warps read the accumulators back
// with tcgen05.ld (warp w owns rows 32w..32w+31) and store bf16 rows. Both projections
// read their weights once per token tile; at decode sizes (T <= 128) they are bound by
// the weight bytes, so the absorb's 512 output columns are cut into blocks to spread the
// weight reads over more CTAs than there are heads.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace gemm {

constexpr int kM = 128;           // token rows per CTA
constexpr int kKB = 64;           // K elements per block (one 128-byte swizzle row)

struct Params {
  __nv_bfloat16* out;             // [T][H][n_total]
  int32_t T, H;
  int32_t n_total;                // output row width (N x gridDim.z)
  uint64_t timeout_ns;
};

// KBLK: K / 64. N: output width. B_MN: B stored with N contiguous (absorb) or K (outproj).
template <int KBLK, int N, bool B_MN, int STAGES>
struct Cfg {
  static constexpr int kABytes = kM * kKB * 2;                 // 16 KiB
  static constexpr int kBBytes = N * kKB * 2;                  // N rows or N cols x 64 K
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kOffBar = STAGES * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;      // barriers + alignment slack
  static constexpr int kNInstr = N > 256 ? 256 : N;            // N per MMA
  static_assert(N % 64 == 0, "the epilogue writes 64-column groups");
  static constexpr int kNHalves = N / kNInstr;
  static constexpr uint32_t kCols = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : (N <= 256 ? 256 : 512)));
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kM, kNInstr, 0, B_MN ? 1 : 0);
};

template <int KBLK, int N, bool B_MN, int STAGES>
__global__ void __launch_bounds__(128, 1)
proj_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Params p) {
  using C = Cfg<KBLK, N, B_MN, STAGES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  auto bar = [&](int i) { return sbase + C::kOffBar + 8u * i; };   // [0,S) full, [S,2S) empty, 2S done
  const uint32_t tmem_holder = sbase + C::kOffBar + 8u * (2 * STAGES + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + 8 * (2 * STAGES + 3));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, m0 = blockIdx.y * kM, n0 = blockIdx.z * N;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar(s), 1);
      ptx::mbar_init(bar(STAGES + s), 1);
    }
    ptx::mbar_init(bar(2 * STAGES), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(tmem_holder, C::kCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + C::kOffBar + 8 * (2 * STAGES + 2));
  auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_bounded(b, parity, abort_flag, p.timeout_ns));
  };
  bool ok = true;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    const bool leader = ptx::elect_one();
    for (int kb = 0; kb < KBLK; ++kb) {
      const int s = kb % STAGES, use = kb / STAGES;
      if (!wait_all(bar(STAGES + s), (use & 1) ^ 1)) {
        if (leader) { raise_status(kStatusTimeout); *abort_flag = 1; }
        ok = false;
        break;
      }
      if (leader) {
        const uint32_t sa = sbase + s * C::kStageBytes, sb = sa + C::kABytes;
        ptx::mbar_arrive_expect_tx(bar(s), C::kStageBytes);
        // A: rows m0.., columns of head h, K block kb
        ptx::tma_load_2d(sa, &tmA, bar(s), h * (KBLK * kKB) + kb * kKB, m0);
        if (B_MN) {
          // B block: 64 K rows (head h's rows kb*64..) x N columns, as N/64 boxes
#pragma unroll
          for (int j = 0; j < N / 64; ++j)
            ptx::tma_load_2d(sb + j * (64 * 128), &tmB, bar(s), n0 + 64 * j, h * (KBLK * kKB) + kb * kKB);
        } else {
          // B block: N rows (head h's rows) x 64 K columns
#pragma unroll
          for (int j = 0; j < N / 64; ++j)
            ptx::tma_load_2d(sb + j * (64 * 128), &tmB, bar(s), kb * kKB, h * p.n_total + n0 + 64 * j);
        }
      }
    }
    // Copies still in flight land in this CTA's shared memory: wait (bounded) for the
    // last ones before the CTA may exit (on the normal path they are long complete).
    for (int kb = (KBLK > STAGES ? KBLK - STAGES : 0); kb < KBLK; ++kb)
      wait_all(bar(kb % STAGES), (kb / STAGES) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const bool leader = ptx::elect_one();
    for (int kb = 0; kb < KBLK; ++kb) {
      const int s = kb % STAGES, use = kb / STAGES;
      if (!wait_all(bar(s), use & 1)) {
        if (leader) { raise_status(kStatusTimeout); *abort_flag = 1; }
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t sa = sbase + s * C::kStageBytes, sb = sa + C::kABytes;
      const uint64_t dA = ptx::sdesc_sw128(sa, 16, 1024);
      const uint64_t dB = B_MN ? ptx::sdesc_sw128(sb, 64 * 128, 1024) : ptx::sdesc_sw128(sb, 16, 1024);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kKB / 16; ++kk) {
#pragma unroll
          for (int nh = 0; nh < C::kNHalves; ++nh) {
            // MN-major B: N half nh starts kNInstr/64 boxes further; K step = 16 rows of 128 B.
            // K-major B: N half nh starts kNInstr rows further (8-row groups of 1024 B).
            const uint32_t boff = B_MN ? (nh * (C::kNInstr / 64) * (64 * 128) + kk * 2048)
                                       : (nh * (C::kNInstr / 8) * 1024 + kk * 32);
            ptx::umma_f16_ss(tbase + nh * C::kNInstr, dA + (uint64_t)((kk * 32) >> 4), dB + (uint64_t)(boff >> 4),
                             C::kIdesc, (kb | kk) ? 1u : 0u);
          }
        }
        ptx::umma_commit(bar(STAGES + s));
        if (kb == KBLK - 1) ptx::umma_commit(bar(2 * STAGES));
      }
      __syncwarp();
    }
  }

  // ---------------------------------------------------------------- epilogue (all warps)
  const bool done = ok && wait_all(bar(2 * STAGES), 0);
  if (!done && lane == 0) {
    raise_status(kStatusTimeout);
    *abort_flag = 1;
  }
  ptx::tc_fence_after();
  const int row = m0 + 32 * warp + lane;
  if (done) {
    // four 16-column TMEM loads in flight per wait, then 128 contiguous bytes of the row
#pragma unroll 1
    for (int c0 = 0; c0 < N; c0 += 64) {
      float v[4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q) ptx::tmem_ld_32x32b_x16(tbase + ((32u * warp) << 16) + c0 + 16 * q, v[q]);
      ptx::tmem_wait_ld();
      if (row < p.T) {
        uint4 pk[8];
        uint32_t* w = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[q][2 * j], v[q][2 * j + 1]);
            w[8 * q + j] = *reinterpret_cast<uint32_t*>(&b2);
          }
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)row * p.H + h) * p.n_total + n0 + c0);
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = pk[k];
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, C::kCols);
  }
}

// ----------------------------------------------------------------------------------
// Output projection with fp32 A: out[t][h][:] = o_lat[t][h][:] @ W_UV[h]^T with o_lat
// in fp32. The tensor cores take bf16 operands, so each fp32 element is split into
// hi = bf16(x) and lo = bf16(x - hi) (together ~16 significant bits) and the MMA runs
// twice per K step, hi and lo against the same weight tile. Per stage TMA brings the
// 128 x 64 fp32 block of A (two 32-column boxes, 128-byte swizzle: 128-byte rows) and
// the N x 64 weight block; warps 2-5 turn each A row (one per thread), in place, into its
// hi row (where the first box's row was) and its lo row (the second box's), in the K-major
// 128-byte-swizzled layout the MMA reads; warp 1 issues the MMAs; warp 0 the loads;
// warps 0-3 read the accumulators back (warp w reaches TMEM lanes 32w..32w+31).
constexpr int kA32Threads = 192;
template <int KBLK, int N, int STAGES>
struct CfgA32 {
  static constexpr int kABytes = kM * kKB * 4;                 // 32 KiB fp32, then hi | lo bf16
  static constexpr int kBBytes = N * kKB * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kOffBar = STAGES * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kCols = N <= 128 ? 128 : 256;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kM, N, 0, 0);
  static_assert(N == 128 || N == 256, "N per MMA");
};

template <int KBLK, int N, int STAGES>
__global__ void __launch_bounds__(kA32Threads, 1)
proj_a32_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Params p) {
  using C = CfgA32<KBLK, N, STAGES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  // [0,S) loads landed, [S,2S) A converted, [2S,3S) stage free, 3S all MMAs done
  auto bar = [&](int i) { return sbase + C::kOffBar + 8u * i; };
  const uint32_t tmem_holder = sbase + C::kOffBar + 8u * (3 * STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + 8 * (3 * STAGES + 2));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, m0 = blockIdx.y * kM, n0 = blockIdx.z * N;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(bar(s), 1);
      ptx::mbar_init(bar(STAGES + s), 4);
      ptx::mbar_init(bar(2 * STAGES + s), 1);
    }
    ptx::mbar_init(bar(3 * STAGES), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, C::kCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + C::kOffBar + 8 * (3 * STAGES + 1));
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
    for (int kb = 0; kb < KBLK; ++kb) {
      const int s = kb % STAGES, use = kb / STAGES;
      if (!wait_all(bar(2 * STAGES + s), (use & 1) ^ 1)) { give_up(); ok = false; break; }
      if (leader) {
        const uint32_t sa = sbase + s * C::kStageBytes, sb = sa + C::kABytes;
        ptx::mbar_arrive_expect_tx(bar(s), C::kStageBytes);
        // A: rows m0.., fp32 columns of head h, K block kb, as two 32-column boxes
        ptx::tma_load_2d(sa, &tmA, bar(s), h * (KBLK * kKB) + kb * kKB, m0);
        ptx::tma_load_2d(sa + C::kABytes / 2, &tmA, bar(s), h * (KBLK * kKB) + kb * kKB + 32, m0);
        // B: N rows (head h's rows) x 64 K columns
#pragma unroll
        for (int j = 0; j < N / 64; ++j)
          ptx::tma_load_2d(sb + j * (64 * 128), &tmB, bar(s), kb * kKB, h * p.n_total + n0 + 64 * j);
      }
    }
    // copies still in flight land in this CTA's shared memory: wait (bounded) for them
    for (int kb = (KBLK > STAGES ? KBLK - STAGES : 0); kb < KBLK; ++kb)
      wait_all(bar(kb % STAGES), (kb / STAGES) & 1);
  } else if (warp >= 2 && warp < 6) {
    // ---------------------------------------------------------------- fp32 -> bf16 hi, lo
    const int r = 32 * (warp - 2) + lane;   // this thread's row of A
    for (int kb = 0; kb < KBLK; ++kb) {
      const int s = kb % STAGES, use = kb / STAGES;
      if (!wait_all(bar(s), use & 1)) { give_up(); ok = false; break; }
      const uint32_t sa = sbase + s * C::kStageBytes;
      {
        const uint32_t row0 = sa + (uint32_t)r * 128u, row1 = row0 + C::kABytes / 2;
        float x[64];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t off = (uint32_t)((j ^ (r & 7)) << 4);   // 16-byte chunk j of the row
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(x[4 * j]), "=f"(x[4 * j + 1]), "=f"(x[4 * j + 2]), "=f"(x[4 * j + 3])
                       : "r"(row0 + off));
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(x[32 + 4 * j]), "=f"(x[32 + 4 * j + 1]), "=f"(x[32 + 4 * j + 2]),
                         "=f"(x[32 + 4 * j + 3])
                       : "r"(row1 + off));
        }
        // the row's 64 K elements as bf16: chunk j (elements 8j..8j+7) of the hi row over
        // the first box's row, of the lo row over the second's
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = x[8 * j + 2 * e], b = x[8 * j + 2 * e + 1];
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(a, b);
            const float2 hf = __bfloat1622float2(h2);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(a - hf.x, b - hf.y);
            hw[e] = *reinterpret_cast<const uint32_t*>(&h2);
            lw[e] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          const uint32_t off = (uint32_t)((j ^ (r & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row0 + off), "r"(hw[0]), "r"(hw[1]),
                       "r"(hw[2]), "r"(hw[3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row1 + off), "r"(lw[0]), "r"(lw[1]),
                       "r"(lw[2]), "r"(lw[3])
                       : "memory");
        }
      }
      ptx::fence_proxy_async_smem();   // the MMA reads these rows through the async proxy
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(STAGES + s));
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    const bool leader = ptx::elect_one();
    for (int kb = 0; kb < KBLK; ++kb) {
      const int s = kb % STAGES, use = kb / STAGES;
      if (!wait_all(bar(STAGES + s), use & 1)) { give_up(); ok = false; break; }
      ptx::tc_fence_after();
      const uint32_t sa = sbase + s * C::kStageBytes, sb = sa + C::kABytes;
      const uint64_t dH = ptx::sdesc_sw128(sa, 16, 1024), dL = ptx::sdesc_sw128(sa + C::kABytes / 2, 16, 1024);
      const uint64_t dB = ptx::sdesc_sw128(sb, 16, 1024);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < kKB / 16; ++kk) {
          const uint64_t k2 = (uint64_t)((kk * 32) >> 4);
          ptx::umma_f16_ss(tbase, dH + k2, dB + k2, C::kIdesc, (kb | kk) ? 1u : 0u);
          ptx::umma_f16_ss(tbase, dL + k2, dB + k2, C::kIdesc, 1u);
        }
        ptx::umma_commit(bar(2 * STAGES + s));
        if (kb == KBLK - 1) ptx::umma_commit(bar(3 * STAGES));
      }
      __syncwarp();
    }
  }

  // ---------------------------------------------------------------- epilogue (warps 0-3)
  const bool done = warp < 4 && ok && wait_all(bar(3 * STAGES), 0);
  if (warp < 4 && !done) give_up();
  ptx::tc_fence_after();
  const int row = m0 + 32 * warp + lane;
  if (done) {
    // four 16-column TMEM loads in flight per wait, then 128 contiguous bytes of the row
#pragma unroll 1
    for (int c0 = 0; c0 < N; c0 += 64) {
      float v[4][16];
#pragma unroll
      for (int q = 0; q < 4; ++q) ptx::tmem_ld_32x32b_x16(tbase + ((32u * warp) << 16) + c0 + 16 * q, v[q]);
      ptx::tmem_wait_ld();
      if (row < p.T) {
        uint4 pk[8];
        uint32_t* w = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[q][2 * j], v[q][2 * j + 1]);
            w[8 * q + j] = *reinterpret_cast<uint32_t*>(&b2);
          }
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)row * p.H + h) * p.n_total + n0 + c0);
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = pk[k];
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, C::kCols);
  }
}

}  // namespace gemm
}  // namespace mla
