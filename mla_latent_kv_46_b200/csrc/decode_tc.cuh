// decode_tc.cuh -- MLA decode attention on the sm_100a tensor cores.
//
// One CTA serves one slot of the split plan for one group of 64 heads. For every
// unit (query token, page range) of its slot it streams the unit's 64-token pages
// through shared memory with TMA and runs, per page:
//   scores   S[h][t]   = sum_k Q[h][k] * KV[t][k]        k over the 576-wide row
//            tcgen05.mma M=64 (heads) x N=64 (tokens) x K=576, fp32 in TMEM
//   softmax  fp32 online softmax per head in registers (4 softmax warps); P goes
//            to the tensor cores as two bf16 terms, P = P_hi + P_lo
//   values   O^T[d][h] += sum_t C[t][d] * P[h][t]         d over the 512 latent dims
//            tcgen05.mma M=128 (latent) x N=64 (heads) x K=64 (tokens), 4 tiles, x2
// The page tile in shared memory is read twice: K-major as the B operand of the
// score MMA and MN-major (latent contiguous) as the A operand of the value MMA,
// so every cached byte crosses HBM once per head group. All heads of the group
// share each page: QK^T and P.C are dense contractions over the heads.
//
// Warp roles (256 threads): warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM
// allocator, warps 4-7 softmax and epilogue (warp w % 4 owns TMEM lanes 32(w%4)..).
//
// TMEM columns: [0,256) O^T, four 128-lane x 64-column fp32 tiles (latent rows
// 128m..128m+127, one column per head); [256,384) the two 64-column score buffers
// in the M=64 layout (rows 16j..16j+15 in lanes 32j..32j+15).
//
// The four softmax warps meet only on mbarriers (bounded waits), never on named
// barriers, so a warp that gives up on a timeout cannot strand the others.
//
// Online softmax keeps a per-head reference maximum and only moves it (and
// rescales O and the running sum) when a page's maximum exceeds it by more than
// 2^8 in linear scale; otherwise the stale reference keeps every P <= 256, well
// inside bf16 and fp32 range. The result divides by the running sum (fp32, of the
// unrounded P) at the end, so it does not depend on the reference.
//
// Why P is split: with P rounded once to bf16 (8 significant bits) the latent
// output of a query that attends to a few tokens of comparable weight can be off
// by ~1% of the spread of those tokens' latents, beyond 2e-3 + 1e-2|o|. With
// P = P_hi + P_lo the rounding error drops by 2^8 for one extra value MMA per
// K-step. P_lo lives in the page's rope box, idle between the score MMA and the
// next load into the stage, so shared memory use does not grow.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace tc {

constexpr int kHeads = 64;            // heads per CTA
constexpr int kPage = 64;             // tokens per page
constexpr int kR = 512, kDr = 64, kRow = kR + kDr;
constexpr int kBox = 64 * 128;        // one TMA box: 64 rows x 64 bf16 = 8 KiB
constexpr int kBoxes = kRow / 64;     // 9 boxes per 576-wide row block
constexpr int kTileBytes = kBoxes * kBox;   // 73,728: Q tile or one page
constexpr int kStages = 2;
constexpr int kPBytes = kHeads * kPage * 2;  // 8 KiB of bf16 probabilities

// shared memory map (offsets from a 1024-aligned base)
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kTileBytes;
constexpr int kOffP = kOffKV + kStages * kTileBytes;
constexpr int kOffBar = kOffP + kPBytes;            // 16 mbarriers
constexpr int kOffTmem = kOffBar + 16 * 8;
constexpr int kOffAbort = kOffTmem + 8;
constexpr int kOffNeed = kOffAbort + 8;             // uint32[2]
constexpr int kOffAlpha = kOffNeed + 8;             // float[2][64]
constexpr int kOffL = kOffAlpha + 512;              // float[64]
constexpr int kOffM = kOffL + 256;                  // float[64]
constexpr int kSmemUsed = kOffM + 256;
constexpr int kSmemBytes = kSmemUsed + 1024;        // slack for aligning the base

// barrier indices
enum {
  B_KV_FULL = 0,   // +stage
  B_KV_EMPTY = 2,  // +stage
  B_S_FULL = 4,    // +buffer
  B_S_EMPTY = 6,   // +buffer
  B_P_FULL = 8,
  B_O_DONE = 9,
  B_Q_FULL = 10,
  B_Q_EMPTY = 11,
  B_O_FREE = 12,
  B_DRAIN = 13,
  B_GROUP = 14,    // the four softmax warps
  kNumBars = 15
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;

constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(64, 64, 0, 0);    // Q (K-major) x KV^T (K-major)
constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(128, 64, 1, 0);   // C^T (MN-major) x P^T (K-major)

constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Params {
  const int32_t* plan;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int32_t max_pages;
  int32_t num_pages;
  int32_t H;
  float scale_log2;           // softmax scale * log2(e)
  float* o_lat;               // [T][H][512] final results (fp32)
  float* lse;                 // [T][H] (nullable)
  float* o_part;              // [parts][H][512]
  float* lse_part;            // [parts][H]
  const __nv_bfloat16* kv;    // cache base (for L2 prefetch)
  const __nv_bfloat16* q_lat;
  const __nv_bfloat16* q_rope;
  uint64_t timeout_ns;
  unsigned long long* trace;  // per-CTA event clocks, only in builds with MLA_TRACE
  int32_t drop_load;          // testing hook: CTA 0 skips the load of its page with this ordinal (-1: none)
  // 8-bit cache (SM-pair kernel only)
  const uint8_t* kv_scale = nullptr;   // [num_pages][64] biased exponents of the rows' scales
  const uint8_t* q8 = nullptr;         // [2][T*H][576] the query rows split into E4M3 high and low pieces
  const float* q_scale = nullptr;      // [T*H] 2^-e of each split row
};

// Optional event trace (build with -DMLA_TRACE): per CTA 1024 clock64 values;
// [0,250) producer load k issued, [256,506) score MMA k issued, [512,762) value
// MMA k issued, [768,890) softmax P(k) ready, [896,1018) scores of page k read
// from TMEM, [1023] kernel start.
#ifdef MLA_TRACE
#define MLA_TRACE_AT(slot)                                                       \
  do {                                                                           \
    if (p.trace && ((slot) & 255) < 250 && ((slot) < 768 || ((slot) & 127) < 122)) \
      p.trace[(size_t)blockIdx.x * 1024 + (slot)] = (unsigned long long)clock64(); \
  } while (0)
#else
#define MLA_TRACE_AT(slot) \
  do {                     \
  } while (0)
#endif

constexpr int kPrefetchPages = 4;     // pages the producer keeps requested into L2 ahead of its loads

struct UnitInfo {
  int32_t item, b, pb, npg, ntok, part;
};

__device__ __forceinline__ UnitInfo load_unit(const Params& p, const PlanView& plan, int32_t idx) {
  const Unit u = plan.units()[idx];
  UnitInfo r;
  r.item = u.item;
  r.b = u.b;
  r.part = u.part;
  const int32_t q_len = plan.q_len();
  r.ntok = visible_tokens(p.seq_lens[u.b], q_len, u.item % q_len);
  const int32_t last = (r.ntok + kPage - 1) / kPage;       // pages holding visible tokens
  const int32_t pe = min(u.page_end, min(last, p.max_pages));
  r.pb = u.page_begin;
  r.npg = max(0, pe - u.page_begin);
  return r;
}

__global__ void __launch_bounds__(256, 1)
decode_kernel(const __grid_constant__ CUtensorMap tm_qlat, const __grid_constant__ CUtensorMap tm_qrope,
              const __grid_constant__ CUtensorMap tm_kv, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t sQ = sbase + kOffQ, sKV = sbase + kOffKV, sP = sbase + kOffP;
  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  float* alpha_s = reinterpret_cast<float*>(smem + kOffAlpha);
  float* l_s = reinterpret_cast<float*>(smem + kOffL);
  float* m_s = reinterpret_cast<float*>(smem + kOffM);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PlanView plan{p.plan};
  const int G = plan.head_groups();
  const int slot = blockIdx.x / G, g = blockIdx.x % G;
  const int32_t u_begin = plan.slot_begin()[slot], u_end = plan.slot_begin()[slot + 1];
  const int32_t H = p.H;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    ptx::mbar_init(bar(B_KV_FULL + 0), 1);
    ptx::mbar_init(bar(B_KV_FULL + 1), 1);
    ptx::mbar_init(bar(B_KV_EMPTY + 0), 1);
    ptx::mbar_init(bar(B_KV_EMPTY + 1), 1);
    ptx::mbar_init(bar(B_S_FULL + 0), 1);
    ptx::mbar_init(bar(B_S_FULL + 1), 1);
    ptx::mbar_init(bar(B_S_EMPTY + 0), 4);
    ptx::mbar_init(bar(B_S_EMPTY + 1), 4);
    ptx::mbar_init(bar(B_P_FULL), 4);
    ptx::mbar_init(bar(B_O_DONE), 1);
    ptx::mbar_init(bar(B_Q_FULL), 1);
    ptx::mbar_init(bar(B_Q_EMPTY), 1);
    ptx::mbar_init(bar(B_O_FREE), 4);
    ptx::mbar_init(bar(B_DRAIN), 1);
    ptx::mbar_init(bar(B_GROUP), 4);
    reinterpret_cast<uint32_t*>(smem + kOffNeed)[0] = 0xFFFFFFFFu;
    reinterpret_cast<uint32_t*>(smem + kOffNeed)[1] = 0xFFFFFFFFu;
    ptx::fence_mbar_init();
  }
  if (warp == 2) {
    ptx::tmem_alloc(sbase + kOffTmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_qlat);
    ptx::prefetch_tmap(&tm_qrope);
    ptx::prefetch_tmap(&tm_kv);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  if (threadIdx.x == 0) {
#ifdef MLA_TRACE
    if (p.trace) p.trace[(size_t)blockIdx.x * 1024 + 1023] = (unsigned long long)clock64();
#endif
  }

  auto fail = [&]() {
    raise_status(kStatusTimeout);
    *abort_flag = 1;
  };
  // Bounded mbarrier wait whose outcome is the same for every lane of the warp.
  auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_bounded(b, parity, abort_flag, p.timeout_ns));
  };

  if (warp == 0) {
    // ================================================================ TMA producer
    // The whole warp walks the schedule; one elected lane issues the copies.
    // Loads run kStages pages ahead of the MMAs; an L2 prefetch cursor runs a further
    // kPrefetchPages ahead (across unit boundaries, with the next unit's query rows),
    // so the loads into shared memory mostly hit L2.
    const bool leader = ptx::elect_one();
    const uint64_t pol_stream = ptx::policy_evict_first();
    uint32_t gpg = 0, nu = 0;
    bool ok = true;
    int32_t pf_ui = u_begin, pf_k = -1;   // prefetch cursor: next page to request into L2
    UnitInfo pf_u = load_unit(p, plan, pf_ui);
    auto prefetch_next = [&]() {
      ++pf_k;
      while (pf_ui < u_end && pf_k >= pf_u.npg) {
        if (++pf_ui >= u_end) return;
        pf_u = load_unit(p, plan, pf_ui);
        pf_k = 0;
        if (pf_u.npg > 0 && leader) {
          const int64_t qrow = (int64_t)pf_u.item * H + g * kHeads;
          ptx::prefetch_l2_bulk(p.q_lat + qrow * kR, kHeads * kR * 2);
          ptx::prefetch_l2_bulk(p.q_rope + qrow * kDr, kHeads * kDr * 2);
        }
      }
      if (pf_ui < u_end) {
        const int32_t page = p.block_table[(int64_t)pf_u.b * p.max_pages + pf_u.pb + pf_k];
        if (page >= 0 && page < p.num_pages && leader)
          ptx::prefetch_l2_bulk(p.kv + (int64_t)page * kPage * kRow, kTileBytes);
      }
    };
    for (int i = 0; i < kStages + kPrefetchPages; ++i) prefetch_next();
    for (int32_t ui = u_begin; ui < u_end && ok; ++ui) {
      const UnitInfo u = load_unit(p, plan, ui);
      if (u.npg == 0) continue;
      if (!wait_all(bar(B_Q_EMPTY), (nu & 1) ^ 1)) {
        if (leader) fail();
        ok = false;
        break;
      }
      const int32_t qrow = u.item * H + g * kHeads;
      if (leader) {
        ptx::mbar_arrive_expect_tx(bar(B_Q_FULL), kTileBytes);
        for (int j = 0; j < 8; ++j) ptx::tma_load_2d(sQ + j * kBox, &tm_qlat, bar(B_Q_FULL), 64 * j, qrow);
        ptx::tma_load_2d(sQ + 8 * kBox, &tm_qrope, bar(B_Q_FULL), 0, qrow);
      }
      for (int32_t k = 0; k < u.npg; ++k, ++gpg) {
        const uint32_t st = gpg & 1, ph = (gpg >> 1) & 1;
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
        const uint32_t dst = sKV + st * kTileBytes;
        // (the testing hook leaves the page's barrier without its load, so that the
        // waits on it run out and the kernel reports a timeout)
        if (leader && !(blockIdx.x == 0 && (int32_t)gpg == p.drop_load)) {
          MLA_TRACE_AT(gpg);
          ptx::mbar_arrive_expect_tx(bar(B_KV_FULL + st), kTileBytes);
#pragma unroll
          for (int j = 0; j < kBoxes; ++j)
            ptx::tma_load_2d_hint(dst + j * kBox, &tm_kv, bar(B_KV_FULL + st), 64 * j, page * kPage,
                                  pol_stream);
        }
        prefetch_next();
      }
      ++nu;
    }
    // Loads still in flight land in this CTA's shared memory: wait for them
    // (bounded) before the CTA may exit.
    for (uint32_t k = (gpg >= 2 ? gpg - 2 : 0); k < gpg; ++k)
      wait_all(bar(B_KV_FULL + (k & 1)), (k >> 1) & 1);
    if (nu > 0) wait_all(bar(B_Q_FULL), (nu - 1) & 1);
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // The whole warp walks the schedule so the operand descriptors stay warp-uniform;
    // one elected lane issues the tcgen05 instructions and their commits.
    const bool leader = ptx::elect_one();
    // Base descriptors; a K step or box adds (byte offset >> 4) to the start-address field.
    const uint64_t dQ = ptx::sdesc_sw128(sQ, 16, 1024);
    const uint64_t dP = ptx::sdesc_sw128(sP, 16, 1024);
    // Issue order: S(0), then for every page j: V(j) as soon as its probabilities are
    // ready, then S(j+1). With two stages the load of page j+2 starts only when V(j)
    // has finished, so V(j) must not queue behind S(j+1), which waits for its own load.
    bool ok = true;
    auto gemm_o = [&](uint32_t gp, bool first_of_unit, uint32_t nu) -> bool {
      if (!wait_all(bar(B_P_FULL), gp & 1)) return false;
      if (first_of_unit && nu > 0 && !wait_all(bar(B_O_FREE), (nu - 1) & 1)) return false;
      ptx::tc_fence_after();
      const uint32_t st = gp & 1;
      const uint32_t kv = sKV + st * kTileBytes;
      // A = C^T, MN-major: latent rows 128m.. (boxes 2m, 2m+1), 16 tokens per K step
      const uint64_t dC = ptx::sdesc_sw128(kv, kBox, 1024);
      // B = P^T, K-major rows = heads: high part in the P buffer, remainder in the rope box
      const uint64_t dPlo = ptx::sdesc_sw128(kv + 8 * kBox, 16, 1024);
      if (leader) {
        MLA_TRACE_AT(512 + gp);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = dC + (uint64_t)(((2 * m) * kBox + kk * 2048) >> 4);
            ptx::umma_f16_ss(tbase + kColO + 64 * m, ad, dP + (uint64_t)((kk * 32) >> 4), kIdescO,
                             (first_of_unit && kk == 0) ? 0u : 1u);
            ptx::umma_f16_ss(tbase + kColO + 64 * m, ad, dPlo + (uint64_t)((kk * 32) >> 4), kIdescO, 1u);
          }
        }
        ptx::umma_commit(bar(B_KV_EMPTY + st));
        ptx::umma_commit(bar(B_O_DONE));
      }
      __syncwarp();
      return true;
    };
    // Score cursor: unit sui, page sk; gs = global index of the next score page; nq =
    // non-empty units whose last score MMA has been issued (query tiles consumed).
    uint32_t gs = 0, nq = 0;
    int32_t sui = u_begin - 1, sk = 0;
    UnitInfo su{};
    auto next_s = [&]() -> bool {
      if (sui >= u_begin && ++sk < su.npg) return true;
      while (++sui < u_end) {
        su = load_unit(p, plan, sui);
        sk = 0;
        if (su.npg > 0) return true;
      }
      return false;
    };
    auto issue_s = [&]() -> bool {
      if (sk == 0 && !wait_all(bar(B_Q_FULL), nq & 1)) return false;
      const uint32_t st = gs & 1, ph = (gs >> 1) & 1;
      if (!wait_all(bar(B_KV_FULL + st), ph) || !wait_all(bar(B_S_EMPTY + st), ph ^ 1)) return false;
      ptx::tc_fence_after();
      const uint64_t dK = ptx::sdesc_sw128(sKV + st * kTileBytes, 16, 1024);
      const uint32_t d_s = tbase + kColS + 64u * st;
      const bool last = sk == su.npg - 1;
      if (leader) {
        MLA_TRACE_AT(256 + gs);
#pragma unroll
        for (int j = 0; j < kBoxes; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t off = (uint64_t)((j * kBox + kk * 32) >> 4);
            ptx::umma_f16_ss(d_s, dQ + off, dK + off, kIdescS, (j | kk) ? 1u : 0u);
          }
        }
        ptx::umma_commit(bar(B_S_FULL + st));
        if (last) ptx::umma_commit(bar(B_Q_EMPTY));
      }
      __syncwarp();
      if (last) ++nq;
      ++gs;
      return true;
    };
    if (next_s() && !issue_s()) {
      if (leader) fail();
      ok = false;
    }
    uint32_t gv = 0, nu = 0;
    for (int32_t ui = u_begin; ui < u_end && ok; ++ui) {
      const UnitInfo u = load_unit(p, plan, ui);
      if (u.npg == 0) continue;
      for (int32_t k = 0; k < u.npg; ++k, ++gv) {
        if (!gemm_o(gv, k == 0, nu) || (next_s() && !issue_s())) {
          if (leader) fail();
          ok = false;
          break;
        }
      }
      ++nu;
    }
    // Let every MMA issued so far finish before TMEM can be released.
    if (leader) ptx::umma_commit(bar(B_DRAIN));
    __syncwarp();
    wait_all(bar(B_DRAIN), 0);
  } else if (warp >= 4) {
    // ================================================================ softmax + epilogue
    const int sub = warp & 3;          // TMEM sub-partition
    const int sm_tid = threadIdx.x - 128;
    const int r0 = lane >> 2, c2 = 2 * (lane & 3);
    const int ha = 16 * sub + r0, hb = ha + 8;   // heads (within the group) of this thread
    volatile uint32_t* need_w = reinterpret_cast<volatile uint32_t*>(smem + kOffNeed);
    uint32_t gpg = 0, nu = 0, ngroup = 0;
    bool ok = true;
    // Bounded meeting point of the four softmax warps.
    auto group_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_GROUP));
      const bool done = ptx::mbar_wait_bounded(bar(B_GROUP), ngroup & 1, abort_flag, p.timeout_ns);
      ++ngroup;
      return __all_sync(0xffffffffu, done);
    };
    for (int32_t ui = u_begin; ui < u_end && ok; ++ui) {
      const UnitInfo u = load_unit(p, plan, ui);
      const bool final_out = u.part < 0;
      if (u.npg == 0) {
        // No visible token: o = 0, lse = -inf.
        for (int e = sm_tid; e < kHeads * kR; e += 128) {
          const int h = e / kR, d = e % kR;
          if (final_out)
            p.o_lat[((int64_t)u.item * H + g * kHeads + h) * kR + d] = 0.f;
          else
            p.o_part[((int64_t)u.part * H + g * kHeads + h) * kR + d] = 0.f;
        }
        if (sm_tid < kHeads) {
          if (final_out) {
            if (p.lse) p.lse[(int64_t)u.item * H + g * kHeads + sm_tid] = -CUDART_INF_F;
          } else {
            p.lse_part[(int64_t)u.part * H + g * kHeads + sm_tid] = -CUDART_INF_F;
          }
        }
        continue;
      }
      float m_a = -CUDART_INF_F, m_b = -CUDART_INF_F, l_a = 0.f, l_b = 0.f;
      for (int32_t k = 0; k < u.npg; ++k, ++gpg) {
        const uint32_t st = gpg & 1, ph = (gpg >> 1) & 1;
        const bool got = ptx::mbar_wait_bounded(bar(B_S_FULL + st), ph, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, got)) { fail(); ok = false; break; }
        ptx::tc_fence_after();
        float v[32];
        ptx::tmem_ld_16x256b_x8(tbase + ((32u * sub) << 16) + kColS + 64u * st, v);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_S_EMPTY + st));
        if (warp == 4 && lane == 0 && gpg < 122) MLA_TRACE_AT(896 + gpg);

        // scale to log2 units, mask tokens past the visible end
        const int32_t tok0 = (u.pb + k) * kPage;
        float mx_a = -CUDART_INF_F, mx_b = -CUDART_INF_F;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const bool valid = tok0 + 8 * i + c2 + c < u.ntok;
            v[4 * i + c] = valid ? v[4 * i + c] * p.scale_log2 : -CUDART_INF_F;
            v[4 * i + 2 + c] = valid ? v[4 * i + 2 + c] * p.scale_log2 : -CUDART_INF_F;
            mx_a = fmaxf(mx_a, v[4 * i + c]);
            mx_b = fmaxf(mx_b, v[4 * i + 2 + c]);
          }
        }
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
        mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
        mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
        const bool need_a = mx_a > m_a + kRescaleThreshold;
        const bool need_b = mx_b > m_b + kRescaleThreshold;
        const float mu_a = need_a ? mx_a : m_a, mu_b = need_b ? mx_b : m_b;
        const float al_a = need_a ? ptx::ex2(m_a - mu_a) : 1.f;   // 0 when m was -inf
        const float al_b = need_b ? ptx::ex2(m_b - mu_b) : 1.f;
        float* alpha = alpha_s + 64 * st;
        if ((lane & 3) == 0) {
          alpha[ha] = al_a;
          alpha[hb] = al_b;
        }
        if (__any_sync(0xffffffffu, need_a || need_b) && lane == 0) need_w[st] = gpg;
        const float za = (mu_a == -CUDART_INF_F) ? 0.f : mu_a;
        const float zb = (mu_b == -CUDART_INF_F) ? 0.f : mu_b;
        // P split into a bf16 high part (the top 16 bits of p) and a bf16 remainder (the
        // top 16 bits of p - P_hi): the value MMA runs on both, so P enters the sum
        // within 2^-15 of p instead of 2^-8; integer operations only, no conversions.
        uint32_t pk[16], pl[16];
        float sa = 0.f, sb = 0.f;
        auto split = [](float x, float y, uint32_t& hi, uint32_t& lo) {
          const uint32_t ux = __float_as_uint(x), uy = __float_as_uint(y);
          hi = __byte_perm(ux, uy, 0x7632);
          const float rx = x - __uint_as_float(ux & 0xFFFF0000u), ry = y - __uint_as_float(uy & 0xFFFF0000u);
          lo = __byte_perm(__float_as_uint(rx), __float_as_uint(ry), 0x7632);
        };
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float a0 = ptx::ex2(v[4 * i] - za), a1 = ptx::ex2(v[4 * i + 1] - za);
          const float b0 = ptx::ex2(v[4 * i + 2] - zb), b1 = ptx::ex2(v[4 * i + 3] - zb);
          sa += a0 + a1;
          sb += b0 + b1;
          split(a0, a1, pk[2 * i], pl[2 * i]);
          split(b0, b1, pk[2 * i + 1], pl[2 * i + 1]);
        }
        l_a = l_a * al_a + sa;
        l_b = l_b * al_b + sb;
        m_a = mu_a;
        m_b = mu_b;

        // all alphas and the need word of this page are written
        if (!group_sync()) { fail(); ok = false; break; }
        const bool any_need = need_w[st] == gpg;
        // the previous value MMA must be done: it reads P and accumulates O
        const bool prev = gpg == 0 ||
                          ptx::mbar_wait_bounded(bar(B_O_DONE), (gpg - 1) & 1, abort_flag, p.timeout_ns);
        if (!__all_sync(0xffffffffu, prev)) { fail(); ok = false; break; }
        if (any_need && k > 0) {
          ptx::tc_fence_after();
#pragma unroll 1
          for (int m = 0; m < 4; ++m) {
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              const uint32_t ta = tbase + ((32u * sub) << 16) + kColO + 64 * m + 16 * c;
              float o[16];
              ptx::tmem_ld_32x32b_x16(ta, o);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j) o[j] *= alpha[16 * c + j];
              ptx::tmem_st_32x32b_x16(ta, o);
            }
          }
          ptx::tmem_wait_st();
        }
        // P[h][t] bf16, K-major rows of 64 tokens with the 128-byte swizzle. The high
        // part goes to the P buffer, the remainder to this stage's rope box, which the
        // score MMA has finished with and the next load into this stage waits for.
        const uint32_t sPlo = sKV + st * kTileBytes + 8 * kBox;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t oa = ha * 128 + (((i ^ (ha & 7)) << 4) | (c2 * 2));
          const uint32_t ob = hb * 128 + (((i ^ (hb & 7)) << 4) | (c2 * 2));
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + oa), "r"(pk[2 * i]) : "memory");
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sP + ob), "r"(pk[2 * i + 1]) : "memory");
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPlo + oa), "r"(pl[2 * i]) : "memory");
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(sPlo + ob), "r"(pl[2 * i + 1]) : "memory");
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_P_FULL));
        if (warp == 4 && lane == 0 && gpg < 122) MLA_TRACE_AT(768 + gpg);
      }
      if (!ok) break;

      // ---------------------------------------------------------------- epilogue
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
      l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
      if ((lane & 3) == 0) {
        l_s[ha] = l_a;
        l_s[hb] = l_b;
        m_s[ha] = m_a;
        m_s[hb] = m_b;
      }
      const bool last = ptx::mbar_wait_bounded(bar(B_O_DONE), (gpg - 1) & 1, abort_flag, p.timeout_ns);
      if (!__all_sync(0xffffffffu, last)) { fail(); ok = false; break; }
      if (!group_sync()) { fail(); ok = false; break; }
      ptx::tc_fence_after();
      const int64_t row0 = final_out ? ((int64_t)u.item * H + g * kHeads) : ((int64_t)u.part * H + g * kHeads);
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + 32 * sub + lane;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[16];
          ptx::tmem_ld_32x32b_x16(tbase + ((32u * sub) << 16) + kColO + 64 * m + 16 * c, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int h = 16 * c + j;
            const float l = l_s[h];
            const float val = l > 0.f ? o[j] / l : 0.f;
            if (final_out)
              p.o_lat[(row0 + h) * kR + d] = val;
            else
              p.o_part[(row0 + h) * kR + d] = val;
          }
        }
      }
      if (sm_tid < kHeads) {
        const float l = l_s[sm_tid];
        const float z = l > 0.f ? (m_s[sm_tid] + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
        if (final_out) {
          if (p.lse) p.lse[row0 + sm_tid] = z;
        } else {
          p.lse_part[row0 + sm_tid] = z;
        }
      }
      // O may be overwritten by the next unit once every warp has read it; l_s and
      // m_s are rewritten only after the next unit's first group_sync.
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
}

}  // namespace tc
}  // namespace mla
