// decode_pair.cuh -- MLA decode attention for 128 heads on a cluster of two CTAs.
//
// The two CTAs of a cluster serve the same slot of the split plan. CTA r loads, for
// every page, only its half of the latent columns (boxes 2r, 2r+1 and 4+2r, 5+2r;
// CTA 0 also the rope box), so the pair holds each page once. Per page:
//   partial scores  S_r[h][t] = sum over CTA r's columns of Q[h][k] KV[t][k], all 128
//                   heads: tcgen05.mma M=128 (heads) x N=64 (tokens), Q from TMEM
//   exchange        CTA r keeps the partial rows of its own 64 heads and stores the
//                   other 64 rows into the peer's shared memory (DSMEM); each CTA adds
//                   the peer's half and has the full scores of its own heads
//   softmax         fp32, one thread per own head (64 tokens in registers); P is split
//                   into bf16 P_hi + P_lo and written to both CTAs' P buffers
//   values          O^T[d][h] += sum_t C[t][d] P[h][t] over CTA r's 256 latent rows and
//                   all 128 heads: tcgen05.mma M=128 x N=128 x K=64 (2 tiles, x2 for P_lo)
// So each CTA streams half a page through its shared memory and its tensor cores
// read half the value operand of a single-CTA design, and every MMA has M=128.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM
// allocator, warps 4-7 query staging, exchange, softmax, epilogue. Warp w (4-7)
// owns TMEM lanes 32(w%4).., i.e. heads 32(w%4)..+31; it "owns" them (softmax,
// output, lse) when (w%4)/2 == r and "sends" them to the peer otherwise.
//
// TMEM (512 columns): [0,256) O^T, two 128-lane x 128-column fp32 tiles (CTA r's
// latent rows, one column per head); [256,384) the query rows' own latent half
// (A operand, lane = head, bf16 pairs per column); [384,512) two score buffers.
//
// Online softmax as in decode_tc.cuh (lazily moved per-head reference maximum,
// P = P_hi + P_lo). A moved reference rescales O^T columns in both CTAs: each CTA
// sends its heads' factors with P.
//
// Every wait is bounded; a CTA that gives up raises the device status word and the
// peer's waits on it run out the same way. Both CTAs meet in a cluster barrier
// before exiting, so no CTA writes into a peer that has left.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace pair {

constexpr int kHeads = 128, kOwn = 64;
constexpr int kPage = 64, kR = 512, kDr = 64, kRow = kR + kDr;
constexpr int kBox = 64 * 128;              // 64 rows x 64 bf16
constexpr int kSlots = 5;                   // 4 latent boxes (own half) + rope (CTA 0)
constexpr int kStageBytes = kSlots * kBox;  // 40 KiB
constexpr int kStages = 3;

constexpr int kOffKV = 0;
constexpr int kOffQr = kOffKV + kStages * kStageBytes;   // rope query rows, 128 x 64 bf16
constexpr int kOffPhi = kOffQr + 2 * kBox;               // P_hi [128 heads][64 tokens] bf16
constexpr int kOffPlo = kOffPhi + 2 * kBox;
constexpr int kOffX = kOffPlo + 2 * kBox;                // 2 x [64 tokens][64 own heads] fp32
constexpr int kXBytes = kPage * kOwn * 4;
constexpr int kOffBar = kOffX + 2 * kXBytes;             // 32 mbarriers
constexpr int kOffTmem = kOffBar + 32 * 8;
constexpr int kOffAbort = kOffTmem + 8;
constexpr int kOffNeed = kOffAbort + 8;                  // uint32[2]
constexpr int kOffAlpha = kOffNeed + 8;                  // float[2][128]
constexpr int kOffL = kOffAlpha + 2 * 128 * 4;           // float[128]
constexpr int kOffM = kOffL + 128 * 4;                   // float[128]
constexpr int kSmemUsed = kOffM + 128 * 4;
constexpr int kSmemBytes = kSmemUsed + 1024;

enum {
  B_KV_FULL = 0,    // +stage (3)
  B_KV_EMPTY = 3,   // +stage (3)
  B_S_FULL = 6,     // +buffer (2)
  B_S_EMPTY = 8,    // +buffer (2), 4 local softmax warps
  B_X_FULL = 10,    // +slot (2), the peer's 2 sender warps filled my slot
  B_X_EMPTY = 12,   // +slot (2), the peer's 2 owner warps emptied the slot I fill
  B_PEER_P = 14,    // the peer's 2 owner warps wrote their P rows and factors here
  B_GROUP = 15,     // the 4 local softmax warps
  B_P_FULL = 16,    // 4 local softmax warps: P complete (and O^T rescaled) for the MMA
  B_O_DONE = 17,    // value MMAs of a page done in both CTAs (2 multicast commits)
  B_Q_FULL = 18,    // query rows staged (4 warps, + the rope TMA on CTA 0)
  B_Q_EMPTY = 19,   // last score MMA of a unit done
  B_O_FREE = 20,    // 4 local warps have read O^T
  B_DRAIN = 21,
  B_LM = 22,        // the peer's 2 owner warps wrote their heads' l, m
  kNumBars = 23
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColQ = 256, kColS = 384;
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 64, 0, 0);    // Q (TMEM / K-major) x KV^T (K-major)
constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(128, 128, 1, 0);   // C^T (MN-major) x P^T (K-major)
constexpr float kRescaleThreshold = 8.0f;

using tc::Params;
using tc::UnitInfo;
using tc::load_unit;

// Optional event trace (-DMLA_TRACE): per CTA 1024 clock64 values, 8 regions of 128
// pages: 0 load issued, 1 score MMA issued, 2 value MMA issued, 3 scores read, 4 peer
// rows received, 5 previous value MMAs done (P may be written), 6 peer P received,
// 7 P complete for the MMA; slot 1023 kernel start. Regions 3-7: first owner warp.
#ifdef MLA_TRACE
#define PAIR_TRACE(region, page)                                                                   \
  do {                                                                                             \
    if (p.trace && (page) < 127)                                                                   \
      p.trace[(size_t)blockIdx.x * 1024 + 128 * (region) + (page)] = (unsigned long long)clock64(); \
  } while (0)
#else
#define PAIR_TRACE(region, page) \
  do {                           \
  } while (0)
#endif

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(256, 1)
decode_pair_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_qrope,
                   const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t rank = ptx::cluster_rank(), peer = rank ^ 1u;
  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  auto peer_addr = [&](uint32_t local) { return ptx::map_peer(local, peer); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  volatile uint32_t* need_w = reinterpret_cast<volatile uint32_t*>(smem + kOffNeed);
  volatile float* alpha_s = reinterpret_cast<volatile float*>(smem + kOffAlpha);
  volatile float* l_s = reinterpret_cast<volatile float*>(smem + kOffL);
  volatile float* m_s = reinterpret_cast<volatile float*>(smem + kOffM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PlanView plan{p.plan};
  const int slot = blockIdx.x >> 1;
  const int32_t u_begin = plan.slot_begin()[slot], u_end = plan.slot_begin()[slot + 1];
  const int32_t H = p.H;   // == 128

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(B_KV_FULL + s), 1);
      ptx::mbar_init(bar(B_KV_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(B_S_FULL + b), 1);
      ptx::mbar_init(bar(B_S_EMPTY + b), 4);
      ptx::mbar_init(bar(B_X_FULL + b), 2);
      ptx::mbar_init(bar(B_X_EMPTY + b), 2);
    }
    ptx::mbar_init(bar(B_PEER_P), 2);
    ptx::mbar_init(bar(B_GROUP), 4);
    ptx::mbar_init(bar(B_P_FULL), 4);
    ptx::mbar_init(bar(B_O_DONE), 2);
    ptx::mbar_init(bar(B_Q_FULL), rank == 0 ? 5 : 4);
    ptx::mbar_init(bar(B_Q_EMPTY), 1);
    ptx::mbar_init(bar(B_O_FREE), 4);
    ptx::mbar_init(bar(B_DRAIN), 1);
    ptx::mbar_init(bar(B_LM), 2);
    need_w[0] = 0xFFFFFFFFu;
    need_w[1] = 0xFFFFFFFFu;
    ptx::fence_mbar_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(sbase + kOffTmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_kv);
    ptx::prefetch_tmap(&tm_qrope);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // both CTAs' barriers exist before anyone arrives remotely
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && p.trace) p.trace[(size_t)blockIdx.x * 1024 + 1023] = (unsigned long long)clock64();
#endif

  auto fail = [&]() {
    raise_status(kStatusTimeout);
    *abort_flag = 1;
  };
  auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_bounded(b, parity, abort_flag, p.timeout_ns));
  };
  auto wait_all_cluster = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(b, parity, abort_flag, p.timeout_ns));
  };
  // latent boxes of this CTA, in stage-slot order (tile 0 = slots 0,1; tile 1 = slots 2,3)
  auto box_of_slot = [&](int s) -> int { return s < 2 ? (int)(2 * rank) + s : 4 + (int)(2 * rank) + (s - 2); };

  if (warp == 0) {
    // ================================================================ TMA producer
    const bool leader = ptx::elect_one();
    const uint64_t pol_stream = ptx::policy_evict_first();
    const uint32_t stage_tx = (rank == 0 ? 5 : 4) * kBox;
    uint32_t gpg = 0, nu = 0;
    bool ok = true;
    int32_t pf_ui = u_begin, pf_k = -1;
    UnitInfo pf_u = load_unit(p, plan, pf_ui);
    auto prefetch_next = [&]() {
      ++pf_k;
      while (pf_ui < u_end && pf_k >= pf_u.npg) {
        if (++pf_ui >= u_end) return;
        pf_u = load_unit(p, plan, pf_ui);
        pf_k = 0;
        if (pf_u.npg > 0 && leader && rank == 0) {
          const int64_t qrow = (int64_t)pf_u.item * H;
          ptx::prefetch_l2_bulk(p.q_lat + qrow * kR, kHeads * kR * 2);
          ptx::prefetch_l2_bulk(p.q_rope + qrow * kDr, kHeads * kDr * 2);
        }
      }
      if (pf_ui < u_end && rank == 0) {
        const int32_t page = p.block_table[(int64_t)pf_u.b * p.max_pages + pf_u.pb + pf_k];
        if (page >= 0 && page < p.num_pages && leader)
          ptx::prefetch_l2_bulk(p.kv + (int64_t)page * kPage * kRow, kPage * kRow * 2);
      }
    };
    for (int i = 0; i < kStages + 4; ++i) prefetch_next();
    for (int32_t ui = u_begin; ui < u_end && ok; ++ui) {
      const UnitInfo u = load_unit(p, plan, ui);
      if (u.npg == 0) continue;
      if (rank == 0) {
        // rope query rows of the unit's 128 heads (the previous unit's scores are done)
        if (!wait_all(bar(B_Q_EMPTY), (nu & 1) ^ 1)) {
          if (leader) fail();
          ok = false;
          break;
        }
        if (leader) {
          const int32_t qrow = u.item * H;
          ptx::mbar_arrive_expect_tx(bar(B_Q_FULL), 2 * kBox);
          ptx::tma_load_2d(sbase + kOffQr, &tm_qrope, bar(B_Q_FULL), 0, qrow);
          ptx::tma_load_2d(sbase + kOffQr + kBox, &tm_qrope, bar(B_Q_FULL), 0, qrow + 64);
        }
      }
      for (int32_t k = 0; k < u.npg; ++k, ++gpg) {
        const uint32_t st = gpg % kStages, ph = (gpg / kStages) & 1;
        if (!wait_all(bar(B_KV_EMPTY + st), ph ^ 1)) {
          if (leader) fail();
          ok = false;
          break;
        }
        int32_t page = p.block_table[(int64_t)u.b * p.max_pages + u.pb + k];
        if (page < 0 || page >= p.num_pages) {
          if (leader) raise_status(kStatusBadPage);
          page = p.num_pages;  // rows past the tensor: TMA fills zeros
        }
        if (leader) {
          const uint32_t dst = sbase + kOffKV + st * kStageBytes;
          PAIR_TRACE(0, gpg);
          ptx::mbar_arrive_expect_tx(bar(B_KV_FULL + st), stage_tx);
#pragma unroll
          for (int s = 0; s < 4; ++s)
            ptx::tma_load_2d_hint(dst + s * kBox, &tm_kv, bar(B_KV_FULL + st), 64 * box_of_slot(s), page * kPage,
                                  pol_stream);
          if (rank == 0)
            ptx::tma_load_2d_hint(dst + 4 * kBox, &tm_kv, bar(B_KV_FULL + st), 64 * 8, page * kPage, pol_stream);
        }
        prefetch_next();
      }
      ++nu;
    }
    for (uint32_t k = (gpg >= kStages ? gpg - kStages : 0); k < gpg; ++k)
      wait_all(bar(B_KV_FULL + k % kStages), (k / kStages) & 1);
    if (rank == 0 && nu > 0) wait_all(bar(B_Q_FULL), (nu - 1) & 1);
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    const bool leader = ptx::elect_one();
    const uint64_t dQr = ptx::sdesc_sw128(sbase + kOffQr, 16, 1024);
    const uint64_t dPhi = ptx::sdesc_sw128(sbase + kOffPhi, 16, 1024);
    const uint64_t dPlo = ptx::sdesc_sw128(sbase + kOffPlo, 16, 1024);
    bool ok = true;
    uint32_t gs = 0, nq = 0;
    int32_t sui = u_begin - 1, sk = 0;
    UnitInfo su{};
    auto advance = [&](int32_t& ui, int32_t& k, UnitInfo& u) -> bool {
      if (ui >= u_begin && ++k < u.npg) return true;
      while (++ui < u_end) {
        u = load_unit(p, plan, ui);
        k = 0;
        if (u.npg > 0) return true;
      }
      return false;
    };
    auto issue_s = [&]() -> bool {
      if (sk == 0 && !wait_all(bar(B_Q_FULL), nq & 1)) return false;
      const uint32_t st = gs % kStages, sb = gs & 1;
      if (!wait_all(bar(B_KV_FULL + st), (gs / kStages) & 1) || !wait_all(bar(B_S_EMPTY + sb), ((gs >> 1) & 1) ^ 1))
        return false;
      ptx::tc_fence_after();
      const uint64_t dK = ptx::sdesc_sw128(sbase + kOffKV + st * kStageBytes, 16, 1024);
      const uint32_t d_s = tbase + kColS + 64u * sb;
      const bool last = sk == su.npg - 1;
      if (leader) {
        PAIR_TRACE(1, gs);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_ts(d_s, tbase + kColQ + 32 * s + 8 * kk, dK + (uint64_t)((s * kBox + kk * 32) >> 4),
                             kIdescS, (s | kk) ? 1u : 0u);
        }
        if (rank == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_ss(d_s, dQr + (uint64_t)((kk * 32) >> 4), dK + (uint64_t)((4 * kBox + kk * 32) >> 4),
                             kIdescS, 1u);
        }
        ptx::umma_commit(bar(B_S_FULL + sb));
        if (last) ptx::umma_commit(bar(B_Q_EMPTY));
      }
      __syncwarp();
      if (last) ++nq;
      ++gs;
      return true;
    };
    auto issue_v = [&](uint32_t gp, bool first_of_unit, uint32_t nu) -> bool {
      if (!wait_all(bar(B_P_FULL), gp & 1)) return false;
      if (first_of_unit && nu > 0 && !wait_all(bar(B_O_FREE), (nu - 1) & 1)) return false;
      ptx::tc_fence_after();
      const uint32_t st = gp % kStages;
      const uint64_t dC = ptx::sdesc_sw128(sbase + kOffKV + st * kStageBytes, kBox, 1024);
      if (leader) {
        PAIR_TRACE(2, gp);
#pragma unroll
        for (int m = 0; m < 2; ++m) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = dC + (uint64_t)(((2 * m) * kBox + kk * 2048) >> 4);
            const uint64_t bo = (uint64_t)((kk * 32) >> 4);
            ptx::umma_f16_ss(tbase + kColO + 128 * m, ad, dPhi + bo, kIdescO, (first_of_unit && kk == 0) ? 0u : 1u);
            ptx::umma_f16_ss(tbase + kColO + 128 * m, ad, dPlo + bo, kIdescO, 1u);
          }
        }
        ptx::umma_commit(bar(B_KV_EMPTY + st));
        ptx::umma_commit_cluster(bar(B_O_DONE), 0x3);
      }
      __syncwarp();
      return true;
    };
    // order: S(0); then per page j: S(j+1) (unless j ends a unit), V(j); a unit's first
    // score MMA waits for its last value MMA, because the query rows are staged only
    // after that unit's softmax (three stages keep the next page's load in flight).
    bool s_more = advance(sui, sk, su);
    if (s_more) {
      if (!issue_s()) { if (leader) fail(); ok = false; }
      s_more = advance(sui, sk, su);
    }
    uint32_t gv = 0, nu = 0;
    for (int32_t ui = u_begin; ui < u_end && ok; ++ui) {
      const UnitInfo u = load_unit(p, plan, ui);
      if (u.npg == 0) continue;
      for (int32_t k = 0; k < u.npg && ok; ++k, ++gv) {
        const bool unit_end = k == u.npg - 1;
        if (!unit_end && s_more) {
          if (!issue_s()) { if (leader) fail(); ok = false; break; }
          s_more = advance(sui, sk, su);
        }
        if (!issue_v(gv, k == 0, nu)) { if (leader) fail(); ok = false; break; }
        if (unit_end && s_more) {
          if (!issue_s()) { if (leader) fail(); ok = false; break; }
          s_more = advance(sui, sk, su);
        }
      }
      ++nu;
    }
    if (leader) ptx::umma_commit(bar(B_DRAIN));
    __syncwarp();
    wait_all(bar(B_DRAIN), 0);
  } else if (warp >= 4) {
    // ================================================================ query staging, exchange, softmax, epilogue
    const int sub = warp & 3;
    const int h = 32 * sub + lane;                 // this thread's head (TMEM lane)
    const bool owner = (uint32_t)(sub >> 1) == rank;
    const int hl = h - 64 * (sub >> 1);            // index among the owning CTA's 64 heads
    const bool tracer = owner && (sub & 1) == 0 && lane == 0;
    const uint32_t lane_addr = (32u * sub) << 16;
    uint32_t gpg = 0, nu = 0, ngroup = 0;
    bool ok = true;
    auto group_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_GROUP));
      const bool done = ptx::mbar_wait_bounded(bar(B_GROUP), ngroup & 1, abort_flag, p.timeout_ns);
      ++ngroup;
      return __all_sync(0xffffffffu, done);
    };
    // Stage the query rows of a unit: own latent half of head h, 256 bf16 -> 128 columns.
    auto stage_q = [&](const UnitInfo& u, uint32_t unit_index) -> bool {
      if (!wait_all(bar(B_Q_EMPTY), (unit_index & 1) ^ 1)) return false;
      ptx::tc_fence_after();
      const uint4* src = reinterpret_cast<const uint4*>(p.q_lat + ((int64_t)u.item * H + h) * kR);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        // columns 32c..32c+31 = K pairs of latent dims: tile (c/2), dims 64*(c%2).. within it
        const int dim0 = (c < 2 ? 128 * (int)rank : 256 + 128 * (int)rank) + 64 * (c & 1);
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 v = __ldg(src + dim0 / 8 + i);
          w[4 * i + 0] = v.x;
          w[4 * i + 1] = v.y;
          w[4 * i + 2] = v.z;
          w[4 * i + 3] = v.w;
        }
        ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColQ + 32 * c, w);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_Q_FULL));
      return true;
    };
    // first non-empty unit's query rows
    {
      int32_t ui = u_begin;
      while (ui < u_end && load_unit(p, plan, ui).npg == 0) ++ui;
      if (ui < u_end && !stage_q(load_unit(p, plan, ui), 0)) { fail(); ok = false; }
    }
    for (int32_t ui = u_begin; ui < u_end && ok; ++ui) {
      const UnitInfo u = load_unit(p, plan, ui);
      const bool final_out = u.part < 0;
      const int64_t row0 = final_out ? (int64_t)u.item * H : (int64_t)u.part * H;
      if (u.npg == 0) {
        // No visible token: o = 0 (this CTA's latent half, all heads), lse = -inf (own heads).
        for (int e = threadIdx.x - 128; e < kHeads * 256; e += 128) {
          const int hh = e / 256, j = e % 256;
          const int d = (j < 128 ? 128 * (int)rank : 256 + 128 * (int)rank) + (j & 127);
          if (final_out)
            p.o_lat[(row0 + hh) * kR + d] = __float2bfloat16_rn(0.f);
          else
            p.o_part[(row0 + hh) * kR + d] = 0.f;
        }
        if (owner) {
          if (final_out) {
            if (p.lse) p.lse[row0 + h] = -CUDART_INF_F;
          } else {
            p.lse_part[row0 + h] = -CUDART_INF_F;
          }
        }
        continue;
      }
      float m_run = -CUDART_INF_F, l_run = 0.f;
      for (int32_t k = 0; k < u.npg; ++k, ++gpg) {
        const uint32_t sb = gpg & 1;
        if (!wait_all(bar(B_S_FULL + sb), (gpg >> 1) & 1)) { fail(); ok = false; break; }
        ptx::tc_fence_after();
        float v[64];
        ptx::tmem_ld_32x32b_x64(tbase + lane_addr + kColS + 64u * sb, v);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_S_EMPTY + sb));
        if (tracer) PAIR_TRACE(3, gpg);
        const uint32_t xslot = sbase + kOffX + sb * kXBytes;
        if (!owner) {
          // ------------------------------------------------ send the peer its heads' partial rows
          if (!wait_all_cluster(bar(B_X_EMPTY + sb), ((gpg >> 1) & 1) ^ 1)) { fail(); ok = false; break; }
          const uint32_t dst = peer_addr(xslot) + 4u * hl;
#pragma unroll
          for (int t = 0; t < kPage; ++t) ptx::st_cluster_b32(dst + 4u * kOwn * t, __float_as_uint(v[t]));
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive_cluster(peer_addr(bar(B_X_FULL + sb)));
        } else {
          // ------------------------------------------------ add the peer's half, softmax, P
          if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(bar(B_X_FULL + sb), (gpg >> 1) & 1,
                                                                        abort_flag, p.timeout_ns))) {
            fail();
            ok = false;
            break;
          }
          if (tracer) PAIR_TRACE(4, gpg);
          const volatile float* xs = reinterpret_cast<const volatile float*>(smem + kOffX + sb * kXBytes);
#pragma unroll
          for (int t = 0; t < kPage; ++t) v[t] += xs[kOwn * t + hl];
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive_cluster(peer_addr(bar(B_X_EMPTY + sb)));
          const int32_t tok0 = (u.pb + k) * kPage;
          float mx = -CUDART_INF_F;
#pragma unroll
          for (int t = 0; t < kPage; ++t) {
            v[t] = (tok0 + t < u.ntok) ? v[t] * p.scale_log2 : -CUDART_INF_F;
            mx = fmaxf(mx, v[t]);
          }
          const bool need = mx > m_run + kRescaleThreshold;
          const float mu = need ? mx : m_run;
          const float al = need ? exp2f(m_run - mu) : 1.f;
          const float z = (mu == -CUDART_INF_F) ? 0.f : mu;
          uint32_t ph[32], pl[32];
          float sum = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float a0 = exp2f(v[2 * i] - z), a1 = exp2f(v[2 * i + 1] - z);
            sum += a0 + a1;
            __nv_bfloat162 hi = __floats2bfloat162_rn(a0, a1);
            const float2 fh = __bfloat1622float2(hi);
            __nv_bfloat162 lo = __floats2bfloat162_rn(a0 - fh.x, a1 - fh.y);
            ph[i] = *reinterpret_cast<uint32_t*>(&hi);
            pl[i] = *reinterpret_cast<uint32_t*>(&lo);
          }
          l_run = l_run * al + sum;
          m_run = mu;
          const bool any = __any_sync(0xffffffffu, need);
          // both CTAs' value MMAs of the previous page are done: the P buffers are free
          if (gpg > 0 && !__all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(bar(B_O_DONE), (gpg - 1) & 1,
                                                                                 abort_flag, p.timeout_ns))) {
            fail();
            ok = false;
            break;
          }
          if (tracer) PAIR_TRACE(5, gpg);
          // row h of P_hi / P_lo: 64 tokens bf16 = 8 chunks of 16 B, 128-byte swizzle
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t base = sbase + (part ? kOffPlo : kOffPhi) + h * 128;
            const uint32_t* w = part ? pl : ph;
            const uint32_t pbase = peer_addr(base);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 q = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
              const uint32_t off = (uint32_t)((c ^ (h & 7)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + off), "r"(q.x), "r"(q.y),
                           "r"(q.z), "r"(q.w)
                           : "memory");
              ptx::st_cluster_v4(pbase + off, q);
            }
          }
          alpha_s[128 * sb + h] = al;
          ptx::st_cluster_b32(peer_addr(sbase + kOffAlpha + 4u * (128 * sb + h)), __float_as_uint(al));
          if (any && lane == 0) {
            need_w[sb] = gpg;
            ptx::st_cluster_b32(peer_addr(sbase + kOffNeed + 4u * sb), gpg);
          }
          ptx::fence_proxy_async_cluster();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive_cluster(peer_addr(bar(B_PEER_P)));
        }
        // ------------------------------------------------ P of all 128 heads is here; rescale if needed
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(bar(B_PEER_P), gpg & 1, abort_flag,
                                                                      p.timeout_ns))) {
          fail();
          ok = false;
          break;
        }
        if (tracer) PAIR_TRACE(6, gpg);
        if (!group_sync()) { fail(); ok = false; break; }
        const bool any_need = need_w[sb] == gpg;
        if (any_need && k > 0) {
          if (!owner && !__all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(bar(B_O_DONE), (gpg - 1) & 1,
                                                                                 abort_flag, p.timeout_ns))) {
            fail();
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 2; ++m) {
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
              const uint32_t ta = tbase + lane_addr + kColO + 128 * m + 16 * c;
              float o[16];
              ptx::tmem_ld_32x32b_x16(ta, o);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] *= alpha_s[128 * sb + 16 * c + j];
              ptx::tmem_st_32x32b_x16(ta, o);
            }
          }
          ptx::tmem_wait_st();
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_P_FULL));
        if (tracer) PAIR_TRACE(7, gpg);
      }
      if (!ok) break;

      // ---------------------------------------------------------------- next unit's query rows
      {
        int32_t nx = ui + 1;
        while (nx < u_end && load_unit(p, plan, nx).npg == 0) ++nx;
        if (nx < u_end && !stage_q(load_unit(p, plan, nx), nu + 1)) { fail(); ok = false; break; }
      }
      // ---------------------------------------------------------------- epilogue
      if (owner) {
        l_s[h] = l_run;
        m_s[h] = m_run;
        ptx::st_cluster_b32(peer_addr(sbase + kOffL + 4u * h), __float_as_uint(l_run));
        ptx::st_cluster_b32(peer_addr(sbase + kOffM + 4u * h), __float_as_uint(m_run));
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(peer_addr(bar(B_LM)));
      }
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(bar(B_LM), nu & 1, abort_flag, p.timeout_ns)) ||
          !__all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(bar(B_O_DONE), (gpg - 1) & 1, abort_flag,
                                                                    p.timeout_ns)) ||
          !group_sync()) {
        fail();
        ok = false;
        break;
      }
      ptx::tc_fence_after();
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {
        const int d = (m == 0 ? 128 * (int)rank : 256 + 128 * (int)rank) + 32 * sub + lane;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[16];
          ptx::tmem_ld_32x32b_x16(tbase + lane_addr + kColO + 128 * m + 16 * c, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int hh = 16 * c + j;
            const float l = l_s[hh];
            const float val = l > 0.f ? o[j] / l : 0.f;
            if (final_out)
              p.o_lat[(row0 + hh) * kR + d] = __float2bfloat16_rn(val);
            else
              p.o_part[(row0 + hh) * kR + d] = val;
          }
        }
      }
      if (owner) {
        const float l = l_run;
        const float z = l > 0.f ? (m_run + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
        if (final_out) {
          if (p.lse) p.lse[row0 + h] = z;
        } else {
          p.lse_part[row0 + h] = z;
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_O_FREE));
      ++nu;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, kTmemCols);
  }
  ptx::cluster_sync();   // the peer no longer writes here
}

}  // namespace pair
}  // namespace mla
