// decode_pair.cuh -- MLA decode attention for 128 heads on a cluster of two CTAs.
//
// The two CTAs of a cluster serve the same slot of the split plan. CTA r loads, for
// every page, only its half of the cached columns: latent boxes 2r, 2r+1, 4+2r, 5+2r
// (128-byte swizzle) and rope dims 32r..32r+31 (64-byte swizzle), so the pair holds
// each page once. Per page:
//   partial scores  S_r[h][t] = sum over CTA r's columns of Q[h][k] KV[t][k], all 128
//                   rows: tcgen05.mma M=128 (rows) x N=64 (tokens); the latent part
//                   takes Q from TMEM, the rope part from shared memory
//   exchange        each CTA encodes its 128 x 64 partial scores as 16-bit codes with
//                   one scale per 32 values (see kXRunBytes), stages them in shared
//                   memory and bulk-copies them into the peer's single receive slot
//                   (DSMEM, 17-18 KiB each way, one run per softmax warp with its own
//                   pair of barriers, so softmax warp w of one CTA waits only for warp w
//                   of the other); each CTA adds its own exact partial and the peer's
//                   decoded one, so the two sums agree to 2^-16 of the largest partial
//                   in a thread's block
//   softmax         fp32, kTG threads per row (64 / kTG tokens each), in both CTAs; each CTA
//                   keeps its own reference maximum, P, l and m, so each output half is
//                   normalised consistently with the P it was summed with;
//                   P = P_hi + P_lo (two bf16 parts) is written to TMEM
//   values          O[h][d] += sum_t P[h][t] C[t][d] over CTA r's 256 latent columns:
//                   tcgen05.mma M=128 (rows) x N=256 x K=16, P from TMEM, C from the
//                   stage (N-major), 4 K-steps x 2 parts per page
// So each CTA streams half a page through its shared memory, every MMA has M=128 and
// the value MMA reads only C from shared memory.
//
// The softmax warps read page j's exchange slot, release it, post their part of page
// j's row maxima to the other warps of their lane quarter and issue page j+1's
// exchange, then combine the maxima and run page j's exponentials, so the copy and the
// other warps' skew overlap work; the MMA warp runs the score MMAs two pages ahead of the value MMAs (order S0 S1
// S2 V0 S3 V1 ...). Five stages of pages (the small exchange buffers buy the fifth).
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer (and TMEM allocator), then
// 4 x kTG softmax warps (query staging, exchange, softmax, epilogue): 8 warps of 32
// tokens per row by default (320 threads), or 16 warps of 16 with
// MLA_PAIR_TOKEN_GROUPS=4 (576 threads, 96 registers each). The per-page chain of a
// softmax warp is mostly fixed latency (TMEM loads and stores, barrier round trips,
// proxy fences), so halving its arithmetic with twice the warps does not shorten it,
// and the 96-register build spills: 16 warps measured slower.
//
// TMEM (512 columns, lane = row): [0,256) O, fp32, CTA r's latent columns in box
// order; [256,384) the query's own latent half (bf16 pairs); [384,448) S; [448,480)
// P_hi, [480,512) P_lo (bf16 pairs).
//
// Online softmax with a lazily moved per-row reference maximum (moved only when a
// page's maximum exceeds it by more than 2^8); a moved reference rescales that
// row's O.
//
// Every wait is bounded; a CTA that gives up raises the device status word and the
// peer's waits on it run out the same way. Both CTAs meet in a cluster barrier
// before exiting, so no CTA writes into a peer that has left.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace mla {
namespace pair {

constexpr int kHeads = 128;
constexpr int kPage = 64, kR = 512, kDr = 64, kRow = kR + kDr;
constexpr int kBox = 64 * 128;              // 64 rows x 64 bf16, 128-byte swizzle
constexpr int kRopeBox = 64 * 64;           // 64 rows x 32 bf16, 64-byte swizzle
constexpr int kStageBytes = 4 * kBox + kRopeBox;   // 36 KiB
constexpr int kStages = 5;
// Softmax warps: kTG per TMEM lane quarter, each thread one row and kTokT of a page's
// tokens (token group tg = tokens kTokT*tg ..).
#ifndef MLA_PAIR_TOKEN_GROUPS
#define MLA_PAIR_TOKEN_GROUPS 2
#endif
constexpr int kTG = MLA_PAIR_TOKEN_GROUPS;
static_assert(kTG == 2 || kTG == 4, "token groups");
constexpr int kTokT = kPage / kTG;            // tokens per softmax thread
constexpr int kSoftWarps = 4 * kTG;
// Exchanged partial scores, per softmax thread (one row, one token group: kTokT values v_t):
// 16-bit codes c_t = round(v_t * 32767 / a) + 32768 with a = max |v_t|, and the decode
// step a / 32767 (fp32), so every value is kept to within 2^-16 of its block's largest
// magnitude. Layout of the exchange buffer: per softmax warp one contiguous run (one
// bulk copy) of [chunk kXChunks][lane 32][16 B] codes followed by [lane 32] fp32 steps;
// a warp's 16-byte accesses to one chunk are 512 contiguous bytes.
constexpr int kXChunks = kTokT / 8;
constexpr int kXRunBytes = kXChunks * 512 + 32 * 4;   // 2176 (kTG 2) or 1152 (kTG 4)
constexpr int kXBytes = kSoftWarps * kXRunBytes;      // 17 or 18 KiB

constexpr int kOffKV = 0;
constexpr int kQrBufs = 1;                               // rope query half buffers
constexpr int kOffQr = kOffKV + kStages * kStageBytes;   // rope query half, 128 x 32 bf16
constexpr int kQrBytes = 2 * kRopeBox;
constexpr int kOffX = kOffQr + kQrBufs * kQrBytes;       // the peer's partial scores
constexpr int kOffXout = kOffX + kXBytes;                // mine, staged for the bulk copy
constexpr int kOffBar = kOffXout + kXBytes;              // 64 mbarriers
constexpr int kOffTmem = kOffBar + 64 * 8;
constexpr int kOffAbort = kOffTmem + 8;
constexpr int kSmemUsed = kOffAbort + 8;
// The kTG threads of a row exchange page maxima (and a unit's sums) through the rope box
// of the page's stage, idle once that page's score MMAs are done: float[kTG][128] at
// kOffPairMax (maxima) and kOffPairL (sums) within the stage.
constexpr int kOffPairMax = 4 * kBox, kOffPairL = kOffPairMax + kTG * 128 * 4;
static_assert(kOffPairL + kTG * 128 * 4 <= kStageBytes, "pair scratch in the rope box");
constexpr int kRoleWarps = 2;                            // warp 0 TMA producer, warp 1 MMA
constexpr int kThreads = 32 * (kRoleWarps + kSoftWarps);
constexpr int kSmemBytes = kSmemUsed + 1024;

enum {
  B_KV_FULL = 0,                // +stage
  B_KV_EMPTY = kStages,         // +stage
  B_S_FULL = 2 * kStages,       // score MMAs of a page done
  B_S_EMPTY,                    // the softmax warps read S
  B_X_FULL,                     // +softmax warp: the peer's run for this warp landed
                                // (1 local arrival + one run of tx bytes)
  B_X_EMPTY = B_X_FULL + kSoftWarps,   // +softmax warp: the peer's warp has read the run I
                                // fill (and so my copy of it has landed: my staging run is free)
  B_P_FULL = B_X_EMPTY + kSoftWarps,   // the softmax warps: P in TMEM (and O rescaled)
  B_O_DONE,                     // value MMAs of a page done
  B_QT_FULL,                    // query latent half staged in TMEM (the softmax warps)
  B_QT_EMPTY,                   // last score MMA of a unit done: the TMEM query columns are free
  B_O_FREE,                     // the softmax warps have read O
  B_DRAIN,
  B_ALL,                        // the softmax warps
  B_PAIR,                       // +lane quarter (4): the kTG softmax warps of a quarter
  B_QR_FULL = B_PAIR + 4,       // +buffer: rope query half landed (TMA)
  B_QR_EMPTY = B_QR_FULL + kQrBufs,   // +buffer: last score MMA of the unit that used it done
  kNumBars = B_QR_EMPTY + kQrBufs
};
static_assert(kNumBars <= 64, "barrier area");
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColQ = 256, kColS = 384, kColP = 448;
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 64, 0, 0);    // Q (K-major) x KV^T (K-major)
constexpr uint32_t kIdescV = ptx::idesc_bf16_f32(128, 256, 0, 1);   // P (TMEM) x C (N-major)
constexpr float kRescaleThreshold = 8.0f;

using tc::Params;

// A plan unit for this kernel: 128 rows = the heads of n (1 or 2) consecutive query
// tokens of sequence b (rows_per_token = H = 128 / n), over pages [pb, pb + npg).
struct PairUnit {
  int32_t item, b, pb, npg;
  int32_t n;           // query tokens
  int32_t ntok[2];     // tokens each sees (-1: absent)
  int32_t part[2];     // partial-output index of each, or -1: final result
};

__device__ __forceinline__ PairUnit load_punit(const Params& p, const PlanView& plan, int32_t idx) {
  const Unit u = plan.units()[idx];
  PairUnit r;
  r.item = u.item;
  r.b = u.b;
  r.pb = u.page_begin;
  r.n = u.pad1 > 1 ? 2 : 1;
  const int32_t q_len = plan.q_len(), L = p.seq_lens[u.b];
  r.ntok[0] = visible_tokens(L, q_len, u.item % q_len);
  r.ntok[1] = r.n > 1 ? visible_tokens(L, q_len, u.item % q_len + 1) : -1;
  r.part[0] = u.part;
  r.part[1] = r.n > 1 ? u.pad0 : -1;
  const int32_t last = (max(r.ntok[0], r.ntok[1]) + kPage - 1) / kPage;   // pages holding visible tokens
  const int32_t pe = min(u.page_end, min(last, p.max_pages));
  r.npg = max(0, pe - r.pb);
  return r;
}

// Optional event trace (-DMLA_TRACE): per CTA 1024 clock64 values, 8 regions of 128
// pages: 0 load issued, 1 score MMA issued, 2 value MMA issued, 3 scores complete,
// 4 the peer freed the exchange buffers, 5 peer rows received, 6 softmax computed,
// 7 previous value MMAs done (P written next); slot 1023 kernel start. Regions 3-7:
// warp 4.
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

// Walks the pages of a slot's non-empty units in order.
struct PageCursor {
  int32_t ui;        // unit index
  int32_t k;         // page within the unit
  uint32_t n;        // ordinal of the unit among the slot's non-empty units
  bool valid;
  PairUnit u;
};

__device__ __forceinline__ bool next_nonempty(const Params& p, const PlanView& plan, int32_t& ui, int32_t u_end,
                                              PairUnit& u) {
  while (++ui < u_end) {
    u = load_punit(p, plan, ui);
    if (u.npg > 0) return true;
  }
  return false;
}

__device__ __forceinline__ PageCursor first_page(const Params& p, const PlanView& plan, int32_t u_begin,
                                                 int32_t u_end) {
  PageCursor c;
  c.ui = u_begin - 1;
  c.k = 0;
  c.n = 0;
  c.valid = next_nonempty(p, plan, c.ui, u_end, c.u);
  return c;
}

__device__ __forceinline__ void advance(const Params& p, const PlanView& plan, int32_t u_end, PageCursor& c) {
  if (!c.valid) return;
  if (++c.k < c.u.npg) return;
  c.k = 0;
  ++c.n;
  c.valid = next_nonempty(p, plan, c.ui, u_end, c.u);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_pair_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_kv_rope,
                   const __grid_constant__ CUtensorMap tm_q_rope, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t rank = ptx::cluster_rank(), peer = rank ^ 1u;
  auto bar = [&](int i) { return sbase + kOffBar + 8u * i; };
  auto peer_addr = [&](uint32_t local) { return ptx::map_peer(local, peer); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PlanView plan{p.plan};
  const int slot = blockIdx.x >> 1;
  const int32_t u_begin = plan.slot_begin()[slot], u_end = plan.slot_begin()[slot + 1];
  const int32_t H = p.H;   // 128, or 64 with two query tokens per unit

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar(B_KV_FULL + s), 1);
      ptx::mbar_init(bar(B_KV_EMPTY + s), 1);
    }
    ptx::mbar_init(bar(B_S_FULL), 1);
    ptx::mbar_init(bar(B_S_EMPTY), kSoftWarps);
    for (int w = 0; w < kSoftWarps; ++w) {
      ptx::mbar_init(bar(B_X_FULL + w), 1);
      ptx::mbar_init(bar(B_X_EMPTY + w), 1);
    }
    ptx::mbar_init(bar(B_P_FULL), kSoftWarps);
    ptx::mbar_init(bar(B_O_DONE), 1);
    ptx::mbar_init(bar(B_QT_FULL), kSoftWarps);
    ptx::mbar_init(bar(B_QT_EMPTY), 1);
    for (int b = 0; b < kQrBufs; ++b) {
      ptx::mbar_init(bar(B_QR_FULL + b), 1);
      ptx::mbar_init(bar(B_QR_EMPTY + b), 1);
    }
    ptx::mbar_init(bar(B_O_FREE), kSoftWarps);
    ptx::mbar_init(bar(B_DRAIN), 1);
    ptx::mbar_init(bar(B_ALL), kSoftWarps);
    for (int q = 0; q < 4; ++q) ptx::mbar_init(bar(B_PAIR + q), kTG);
    ptx::fence_mbar_init();
    for (int w = 0; w < kSoftWarps; ++w) ptx::mbar_arrive_expect_tx(bar(B_X_FULL + w), kXRunBytes);   // page 0
  }
  if (warp == 1) {
    ptx::tmem_alloc(sbase + kOffTmem, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_kv);
    ptx::prefetch_tmap(&tm_kv_rope);
    ptx::prefetch_tmap(&tm_q_rope);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // both CTAs' barriers exist before anyone arrives or copies remotely
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
  // latent boxes of this CTA, in stage-slot order: slots 0-3 = latent columns
  // 128r..128r+127 and 256+128r..256+128r+127 (the O column order)
  auto box_of_slot = [&](int s) -> int { return s < 2 ? (int)(2 * rank) + s : 4 + (int)(2 * rank) + (s - 2); };

  if (warp == 0) {
    // ================================================================ TMA producer
    const bool leader = ptx::elect_one();
    // a page is read once per step when every unit has its own sequence (q_len = 1);
    // with several query tokens per sequence the sequence's other units read it again
    const uint64_t pol_stream = plan.q_len() > 1 ? ptx::policy_evict_last() : ptx::policy_evict_first();
    uint32_t gpg = 0, nq = 0;   // pages and rope-query halves loaded
    bool ok = true;
    // L2 prefetch cursor (CTA 0 prefetches whole pages a few pages ahead)
    PageCursor pf = first_page(p, plan, u_begin, u_end);
    auto prefetch_one = [&]() {
      if (!pf.valid) return;
      if (rank == 0 && leader) {
        if (pf.k == 0) {
          // the unit's 128 query rows, clipped to the tensor's T * H rows
          const int64_t qrow = (int64_t)pf.u.item * H;
          const int64_t rows = min((int64_t)kHeads, (int64_t)plan.B() * plan.q_len() * H - qrow);
          if (rows > 0) {
            ptx::prefetch_l2_bulk(p.q_lat + qrow * kR, (uint32_t)(rows * kR * 2));
            ptx::prefetch_l2_bulk(p.q_rope + qrow * kDr, (uint32_t)(rows * kDr * 2));
          }
        }
        const int32_t page = p.block_table[(int64_t)pf.u.b * p.max_pages + pf.u.pb + pf.k];
        if (page >= 0 && page < p.num_pages)
          ptx::prefetch_l2_bulk(p.kv + (int64_t)page * kPage * kRow, kPage * kRow * 2);
      }
      advance(p, plan, u_end, pf);
    };
    for (int i = 0; i < kStages + 4; ++i) prefetch_one();
    PageCursor c = first_page(p, plan, u_begin, u_end);
    while (c.valid && ok) {
      if (c.k == 0) {
        // this CTA's rope query half for the unit's 128 heads, into buffer n & 1 (free once
        // the unit two back has finished its scores: the page stream never waits for the
        // current unit's scores)
        const uint32_t qb = c.n % kQrBufs;
        if (!wait_all(bar(B_QR_EMPTY + qb), ((c.n / kQrBufs) & 1) ^ 1)) {
          if (leader) fail();
          ok = false;
          break;
        }
        if (leader) {
          const int32_t qrow = c.u.item * H;
          const uint32_t dst = sbase + kOffQr + qb * kQrBytes;
          ptx::mbar_arrive_expect_tx(bar(B_QR_FULL + qb), 2 * kRopeBox);
          ptx::tma_load_2d(dst, &tm_q_rope, bar(B_QR_FULL + qb), 32 * rank, qrow);
          ptx::tma_load_2d(dst + kRopeBox, &tm_q_rope, bar(B_QR_FULL + qb), 32 * rank, qrow + 64);
        }
        ++nq;
      }
      const uint32_t st = gpg % kStages, ph = (gpg / kStages) & 1;
      if (!wait_all(bar(B_KV_EMPTY + st), ph ^ 1)) {
        if (leader) fail();
        ok = false;
        break;
      }
      int32_t page = p.block_table[(int64_t)c.u.b * p.max_pages + c.u.pb + c.k];
      if (page < 0 || page >= p.num_pages) {
        if (leader) raise_status(kStatusBadPage);
        page = p.num_pages;  // rows past the tensor: TMA fills zeros
      }
      // (the testing hook leaves the page's barrier without its load: the waits on it run
      // out and the kernel reports a timeout)
      if (leader && !(blockIdx.x == 0 && (int32_t)gpg == p.drop_load)) {
        const uint32_t dst = sbase + kOffKV + st * kStageBytes;
        PAIR_TRACE(0, gpg);
        ptx::mbar_arrive_expect_tx(bar(B_KV_FULL + st), kStageBytes);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          ptx::tma_load_2d_hint(dst + s * kBox, &tm_kv, bar(B_KV_FULL + st), 64 * box_of_slot(s), page * kPage,
                                pol_stream);
        ptx::tma_load_2d_hint(dst + 4 * kBox, &tm_kv_rope, bar(B_KV_FULL + st), kR + 32 * rank, page * kPage,
                              pol_stream);
      }
      prefetch_one();
      advance(p, plan, u_end, c);
      ++gpg;
    }
    // copies still in flight land in this CTA's shared memory: wait (bounded) for them
    for (uint32_t k = (gpg >= kStages ? gpg - kStages : 0); k < gpg; ++k)
      wait_all(bar(B_KV_FULL + k % kStages), (k / kStages) & 1);
    for (uint32_t n = (nq >= kQrBufs ? nq - kQrBufs : 0); n < nq; ++n)
      wait_all(bar(B_QR_FULL + n % kQrBufs), (n / kQrBufs) & 1);
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    const bool leader = ptx::elect_one();

    bool ok = true;
    PageCursor sc = first_page(p, plan, u_begin, u_end);   // next score MMA
    PageCursor vc = sc;                                      // next value MMA
    uint32_t gs = 0, gv = 0;
    auto issue_s = [&]() -> bool {
      const uint32_t qb = sc.n % kQrBufs;
      if (sc.k == 0 &&
          (!wait_all(bar(B_QT_FULL), sc.n & 1) || !wait_all(bar(B_QR_FULL + qb), (sc.n / kQrBufs) & 1)))
        return false;
      const uint64_t dQr = ptx::sdesc_sw64(sbase + kOffQr + qb * kQrBytes, 512);
      const uint32_t st = gs % kStages;
      if (!wait_all(bar(B_KV_FULL + st), (gs / kStages) & 1) || !wait_all(bar(B_S_EMPTY), (gs & 1) ^ 1))
        return false;
      ptx::tc_fence_after();
      const uint32_t stage = sbase + kOffKV + st * kStageBytes;
      const uint64_t dK = ptx::sdesc_sw128(stage, 16, 1024);
      const uint64_t dKr = ptx::sdesc_sw64(stage + 4 * kBox, 512);
      const uint32_t d_s = tbase + kColS;
      const bool last = sc.k == sc.u.npg - 1;
      if (leader) {
        PAIR_TRACE(1, gs);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::umma_f16_ts(d_s, tbase + kColQ + 32 * s + 8 * kk, dK + (uint64_t)((s * kBox + kk * 32) >> 4),
                             kIdescS, (s | kk) ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          ptx::umma_f16_ss(d_s, dQr + (uint64_t)((kk * 32) >> 4), dKr + (uint64_t)((kk * 32) >> 4), kIdescS, 1u);
        ptx::umma_commit(bar(B_S_FULL));
        if (last) {
          ptx::umma_commit(bar(B_QT_EMPTY));
          ptx::umma_commit(bar(B_QR_EMPTY + qb));
        }
      }
      __syncwarp();
      advance(p, plan, u_end, sc);
      ++gs;
      return true;
    };
    auto issue_v = [&]() -> bool {
      if (!wait_all(bar(B_P_FULL), gv & 1)) return false;
      if (vc.k == 0 && vc.n > 0 && !wait_all(bar(B_O_FREE), (vc.n - 1) & 1)) return false;
      ptx::tc_fence_after();
      const uint32_t st = gv % kStages;
      const uint64_t dC = ptx::sdesc_sw128(sbase + kOffKV + st * kStageBytes, kBox, 1024);
      if (leader) {
        PAIR_TRACE(2, gv);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = dC + (uint64_t)((kk * 2048) >> 4);
          ptx::umma_f16_ts(tbase + kColO, tbase + kColP + 8 * kk, bd, kIdescV, (vc.k == 0 && kk == 0) ? 0u : 1u);
          ptx::umma_f16_ts(tbase + kColO, tbase + kColP + 32 + 8 * kk, bd, kIdescV, 1u);
        }
        // a unit's last page keeps its stage: the epilogue stages the unit's output there
        // and then frees it
        if (vc.k != vc.u.npg - 1) ptx::umma_commit(bar(B_KV_EMPTY + st));
        ptx::umma_commit(bar(B_O_DONE));
      }
      __syncwarp();
      advance(p, plan, u_end, vc);
      ++gv;
      return true;
    };
    // S(0), S(1), then per page j: S(j+2), V(j) -- the order in which the softmax
    // warps free the score buffer (exchange of page j+1 before P of page j)
    for (int i = 0; i < 2 && sc.valid && ok; ++i)
      if (!issue_s()) { if (leader) fail(); ok = false; }
    while (vc.valid && ok) {
      if (sc.valid && !issue_s()) { if (leader) fail(); ok = false; break; }
      if (!issue_v()) { if (leader) fail(); ok = false; break; }
    }
    if (leader) ptx::umma_commit(bar(B_DRAIN));
    __syncwarp();
    wait_all(bar(B_DRAIN), 0);
  } else if (warp >= kRoleWarps) {
    // ================================================================ query staging, exchange, softmax, epilogue
    // Softmax warp sw = warp - kRoleWarps serves TMEM lane quarter q = warp % 4 (the only
    // quarter a warp reaches), i.e. rows 32q..32q+31, and token group g = sw / 4 of every
    // page (tokens kTokT*g ..): the kTG threads of a row (same lane in the kTG warps of
    // the quarter) meet on the quarter's pair barrier to combine their maxima (and, in
    // the epilogue, their sums).
    const int sw = warp - kRoleWarps;
    const int sub = warp & 3, tg = sw >> 2;
    const int h = 32 * sub + lane;                 // this thread's head (TMEM lane)
    const bool tracer = sw == 0 && lane == 0;
    const uint32_t lane_addr = (32u * sub) << 16;
    // this warp's run in an exchange buffer (one bulk copy), this thread's first chunk
    // of codes and its decode step there (see kXRunBytes)
    const uint32_t x_run = (uint32_t)sw * kXRunBytes;
    const uint32_t x_lane = x_run + (uint32_t)lane * 16u;
    const uint32_t x_step = x_run + (uint32_t)kXChunks * 512u + (uint32_t)lane * 4u;
    const uint32_t xo_lane = sbase + kOffXout + x_lane;
    auto pair_slot = [&](uint32_t stage, int off) {
      return reinterpret_cast<volatile float*>(smem + kOffKV + stage * kStageBytes + off);
    };
    uint32_t n_pair = 0, n_all = 0;
    bool ok = true;
    auto bounded_sync = [&](uint32_t b, uint32_t& n) -> bool {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(b));
      const bool done = ptx::mbar_wait_bounded(bar(b), n & 1, abort_flag, p.timeout_ns);
      ++n;
      return __all_sync(0xffffffffu, done);
    };
    // the same in two halves, with other work between the arrival and the wait
    auto sync_arrive = [&](uint32_t b) {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(b));
    };
    auto sync_wait = [&](uint32_t b, uint32_t& n) -> bool {
      const bool done = ptx::mbar_wait_bounded(bar(b), n & 1, abort_flag, p.timeout_ns);
      ++n;
      return __all_sync(0xffffffffu, done);
    };

    // Row h belongs to query token tok_h of a unit (0 for H = 128), head h % H.
    const int tok_h = h / H;

    // Units without a visible token: o = 0 (this CTA's latent half), lse = -inf (CTA 0).
    for (int32_t ui = u_begin; ui < u_end; ++ui) {
      const PairUnit u = load_punit(p, plan, ui);
      if (u.npg > 0) continue;
      for (int e = threadIdx.x - 32 * kRoleWarps; e < u.n * H * 256; e += kThreads - 32 * kRoleWarps) {
        const int r = e / 256, j = e % 256, t = r / H;
        const int d = (j < 128 ? 128 * (int)rank : 256 + 128 * (int)rank) + (j & 127);
        const int32_t prt = t ? u.part[1] : u.part[0];
        if (prt < 0)
          p.o_lat[((int64_t)(u.item + t) * H + r % H) * kR + d] = __float2bfloat16_rn(0.f);
        else
          p.o_part[((int64_t)prt * H + r % H) * kR + d] = 0.f;
      }
      if (rank == 0 && tg == 0 && tok_h < u.n) {
        const int32_t prt = tok_h ? u.part[1] : u.part[0];
        if (prt < 0) {
          if (p.lse) p.lse[(int64_t)(u.item + tok_h) * H + h % H] = -CUDART_INF_F;
        } else {
          p.lse_part[(int64_t)prt * H + h % H] = -CUDART_INF_F;
        }
      }
    }

    // Stage a unit's query: this thread's 256 / kTG of row h's own 256 latent dims, box
    // slots 4g/kTG .. (slot s: dims 128r + 64s for s < 2, 256 + 128r + 64(s-2) above) ->
    // TMEM columns 32s.. of the query block.
    auto stage_q = [&](const PairUnit& u, uint32_t n) -> bool {
      if (!wait_all(bar(B_QT_EMPTY), (n & 1) ^ 1)) return false;
      ptx::tc_fence_after();
      // rows of a token the unit does not have stay zero (their scores are never used)
      const bool present = tok_h < u.n;
      // 32-byte loads (one sector each): the 32 lanes read 32 different rows, so each
      // load instruction costs a transaction per lane and wider loads halve them; one box
      // slot (32 words) per round, so that the staging holds few registers
#pragma unroll 1
      for (int s = (4 / kTG) * tg; s < (4 / kTG) * (tg + 1); ++s) {
        const int d0 = s < 2 ? 128 * (int)rank + 64 * s : 256 + 128 * (int)rank + 64 * (s - 2);
        const __nv_bfloat16* src = p.q_lat + ((int64_t)u.item * H + h) * kR + d0;
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t* d = &w[8 * i];
          if (present) {
            asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]),
                           "=r"(d[7])
                         : "l"(src + 16 * i));
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) d[k] = 0u;
          }
        }
        ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColQ + 32 * s, w);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_QT_FULL));
      return true;
    };
    // Exchange of global page g: move this thread's kTokT scores out of TMEM into `own`
    // (freeing the score buffer), encode them (see kXRunBytes), stage them and bulk-copy
    // this warp's run into the peer's slot.
    auto exchange = [&](uint32_t g, float (&own)[kTokT]) -> bool {
      if (!wait_all(bar(B_S_FULL), g & 1)) return false;
      if (tracer) PAIR_TRACE(3, g);
      ptx::tc_fence_after();
      {
        uint32_t r[kTokT];
        ptx::tmem_ld_cols<kTokT>(tbase + lane_addr + kColS + kTokT * tg, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < kTokT; ++t) own[t] = __uint_as_float(r[t]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_S_EMPTY));
      // the peer's warp has read page g-1 from its slot, so my copy of it has landed and
      // the staging run is free
      if (!wait_all_cluster(bar(B_X_EMPTY + sw), (g & 1) ^ 1)) return false;
      if (tracer) PAIR_TRACE(4, g);
      ptx::fence_proxy_async_smem();   // the previous copy's reads before these writes
      // codes: v * (32767 / a) rounded to an integer by adding 1.5 * 2^23 + 2^15 (the sum's
      // unit in the last place is 1), whose low 16 bits are then round(v * 32767 / a) + 32768
      float a = 0.f;
#pragma unroll
      for (int t = 0; t < kTokT; ++t) a = fmaxf(a, fabsf(own[t]));
      // (an approximate quotient: |v| * enc stays below 32767.5; smaller partials are sent as 0)
      const float enc = a > 1e-30f ? __fdividef(32767.f, a) : 0.f;
#pragma unroll
      for (int c = 0; c < kXChunks; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float lo = fmaf(own[8 * c + 2 * i], enc, 12615680.f);
          const float hi = fmaf(own[8 * c + 2 * i + 1], enc, 12615680.f);
          w[i] = __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x5410);
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(xo_lane + 512u * c), "r"(w[0]), "r"(w[1]),
                     "r"(w[2]), "r"(w[3])
                     : "memory");
      }
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(sbase + kOffXout + x_step), "f"(a * (1.f / 32767.f))
                   : "memory");
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0)
        ptx::bulk_copy_to_cluster(peer_addr(sbase + kOffX + x_run), sbase + kOffXout + x_run, (uint32_t)kXRunBytes,
                                  peer_addr(bar(B_X_FULL + sw)));
      return true;
    };
    // Once the score MMA of a unit's last page is done (its S was read), the query
    // columns are free: stage the next unit's query so that its first score MMA can go.
    auto stage_next_q = [&](const PageCursor& c) -> bool {
      if (c.k != c.u.npg - 1) return true;
      int32_t ui = c.ui;
      PairUnit nu;
      return !next_nonempty(p, plan, ui, u_end, nu) || stage_q(nu, c.n + 1);
    };
    // Epilogue of a unit, run after the next unit's first P (or after the last page of
    // the slot) once the unit's last value MMAs are done: O[h][:] / l to the output. This
    // thread holds O columns (256/kTG)g ..; the warps of token group g stage their rows
    // (kRowB bytes per row and round) in the g-th 128 x kRowB block of the unit's last
    // stage (released to the producer at the end), and a warp reads back only its own 32
    // rows, so that each warp store writes whole row segments.
    struct Pending {
      bool on;
      int32_t item, n, part0, part1;   // the unit's tokens and their partial-output indices
      uint32_t stage;                  // stage of the unit's last page
      float l, m;                      // this thread's part of l; the shared reference maximum
    } pend{false, 0, 0, -1, -1, 0u, 0.f, 0.f};
    auto epilogue = [&]() -> bool {
      // l = the token groups' sums, added in group order (the same value in each thread of a row)
      volatile float* ls = pair_slot(pend.stage, kOffPairL);
      ls[128 * tg + h] = pend.l;
      if (!bounded_sync(B_PAIR + sub, n_pair)) return false;
      float l = 0.f;
#pragma unroll
      for (int t = 0; t < kTG; ++t) l += ls[128 * t + h];
      ptx::tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      constexpr int kRowB = 256 / kTG;   // staged bytes per row and round
      constexpr int kCh = kRowB / 16;    // 16-byte chunks per staged row
      const uint32_t buf = sbase + kOffKV + pend.stage * kStageBytes + (uint32_t)tg * (128u * kRowB);
      // this warp's 32 rows all belong to token tok_h of the unit: its output rows
      const bool present = tok_h < pend.n;
      const int32_t prt = tok_h ? pend.part1 : pend.part0;
      const bool final_out = prt < 0;
      const int64_t row0 = (final_out ? (int64_t)(pend.item + tok_h) * H : (int64_t)prt * H) - tok_h * H;
      const int rounds = final_out ? 2 : 4;                  // (256/kTG) columns in kRowB-byte rows
      const int cols = final_out ? kRowB / 2 : kRowB / 4;    // O columns per round
#pragma unroll 1
      for (int c = 0; c < rounds; ++c) {
        const int col0 = (256 / kTG) * tg + cols * c;        // TMEM column of the round
        uint32_t w[kRowB / 4];
        if (final_out) {
          uint32_t o[kRowB / 64][32];
#pragma unroll
          for (int k = 0; k < kRowB / 64; ++k) ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColO + col0 + 32 * k, o[k]);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < kRowB / 64; ++k) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(o[k][2 * i]) * inv_l,
                                                        __uint_as_float(o[k][2 * i + 1]) * inv_l);
              w[16 * k + i] = *reinterpret_cast<uint32_t*>(&b2);
            }
          }
        } else {
          ptx::tmem_ld_cols<kRowB / 4>(tbase + lane_addr + kColO + col0, w);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < kRowB / 4; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * inv_l);
        }
        __syncwarp();   // this warp's previous round has been read back
#pragma unroll
        for (int j = 0; j < kCh; ++j)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + (uint32_t)h * kRowB +
                                                                       (uint32_t)((j ^ (h & (kCh - 1))) << 4)),
                       "r"(w[4 * j]), "r"(w[4 * j + 1]), "r"(w[4 * j + 2]), "r"(w[4 * j + 3])
                       : "memory");
        __syncwarp();
        const int d0 = (col0 < 128 ? 128 * (int)rank + col0 : 256 + 128 * (int)rank + (col0 - 128));
#pragma unroll
        for (int it = 0; it < kCh; ++it) {
          const int row = 32 * sub + (32 / kCh) * it + lane / kCh, j = lane % kCh;
          uint4 q;
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(q.x), "=r"(q.y), "=r"(q.z), "=r"(q.w)
                       : "r"(buf + (uint32_t)row * kRowB + (uint32_t)((j ^ (row & (kCh - 1))) << 4))
                       : "memory");
          if (!present) continue;
          if (final_out)
            *reinterpret_cast<uint4*>(p.o_lat + (row0 + row) * kR + d0 + 8 * j) = q;
          else
            *reinterpret_cast<uint4*>(p.o_part + (row0 + row) * kR + d0 + 4 * j) = q;
        }
      }
      if (rank == 0 && tg == 0 && present) {
        const float z = l > 0.f ? (pend.m + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
        if (final_out) {
          if (p.lse) p.lse[row0 + h] = z;
        } else {
          p.lse_part[row0 + h] = z;
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_O_FREE));
      // every warp has read the staged rows: the stage goes back to the producer
      if (!bounded_sync(B_ALL, n_all)) return false;
      if (sw == 0 && lane == 0) {
        ptx::fence_proxy_async_smem();   // the staged rows' reads before the next TMA load
        ptx::mbar_arrive(bar(B_KV_EMPTY + pend.stage));
      }
      pend.on = false;
      return true;
    };

    PageCursor cur = first_page(p, plan, u_begin, u_end);
    PageCursor ex = cur;
    uint32_t gpg = 0;
    float own[kTokT];   // this thread's partial scores for the page read next
    if (cur.valid) {
      if (!stage_q(cur.u, 0) || !exchange(0, own) || !stage_next_q(ex)) { fail(); ok = false; }
      advance(p, plan, u_end, ex);
    }
    float m_run = -CUDART_INF_F, l_run = 0.f;
    while (cur.valid && ok) {
      const PairUnit& u = cur.u;
      const int32_t ntok = tok_h ? u.ntok[1] : u.ntok[0];   // tokens this row sees (-1: no row)
      if (cur.k == 0) {
        m_run = -CUDART_INF_F;
        l_run = 0.f;
      }
      // ------------------------------------------------ full scores: mine + the peer's
      if (!wait_all(bar(B_X_FULL + sw), gpg & 1)) { fail(); ok = false; break; }
      if (tracer) PAIR_TRACE(5, gpg);
      float v[kTokT];
      {
        float step;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(step) : "r"(sbase + kOffX + x_step) : "memory");
#pragma unroll
        for (int c = 0; c < kXChunks; ++c) {
          uint32_t w[4];
          asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                       : "r"(sbase + kOffX + x_lane + 512u * c)
                       : "memory");
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            // a code under the exponent and leading bits of 1.5 * 2^23 is that float plus
            // the code; less the code's offset of 2^15 it is the peer's value / step
            const float lo = __uint_as_float(__byte_perm(w[i], 0x4B400000u, 0x7610)) - 12615680.f;
            const float hi = __uint_as_float(__byte_perm(w[i], 0x4B400000u, 0x7632)) - 12615680.f;
            v[8 * c + 2 * i] = fmaf(lo, step, own[8 * c + 2 * i]);
            v[8 * c + 2 * i + 1] = fmaf(hi, step, own[8 * c + 2 * i + 1]);
          }
        }
      }
      // ------------------------------------------------ this page's maximum and reference
      const int32_t tok0 = (u.pb + cur.k) * kPage + kTokT * tg;
      if (tok0 + kTokT > ntok) {
#pragma unroll
        for (int t = 0; t < kTokT; ++t) v[t] = (tok0 + t < ntok) ? v[t] : -CUDART_INF_F;
      }
      float mx;
      {
        float t8[kTokT / 8];
#pragma unroll
        for (int i = 0; i < kTokT / 8; ++i) {
          const float a = fmaxf(fmaxf(v[8 * i], v[8 * i + 1]), fmaxf(v[8 * i + 2], v[8 * i + 3]));
          const float b = fmaxf(fmaxf(v[8 * i + 4], v[8 * i + 5]), fmaxf(v[8 * i + 6], v[8 * i + 7]));
          t8[i] = fmaxf(a, b);
        }
        mx = t8[0];
#pragma unroll
        for (int i = 1; i < kTokT / 8; ++i) mx = fmaxf(mx, t8[i]);
      }
      // The vote depends on every lane's loaded values, so all of this warp's reads of
      // the slot are complete when lane 0 tells the peer that it may be overwritten.
      ptx::vote_any_ordered(mx > -CUDART_INF_F);
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar(B_X_FULL + sw), kXRunBytes);   // arm the run's next use
        ptx::mbar_arrive_cluster_relaxed(peer_addr(bar(B_X_EMPTY + sw)));
      }
      // this group's maximum to the quarter's other warps; theirs are read after the
      // exchange below
      volatile float* ms = pair_slot(gpg % kStages, kOffPairMax);
      ms[128 * tg + h] = mx;
      sync_arrive(B_PAIR + sub);
      // ------------------------------------------------ the next page's exchange (the slot is
      // free once both CTAs have read it), overlapping this page's exponentials; `own` is
      // dead once v holds the sums and takes the next page's partial scores
      const bool more = ex.valid;
      if (more && (!exchange(gpg + 1, own) || !stage_next_q(ex))) { fail(); ok = false; break; }
      // the row's maximum over the token groups
      if (!sync_wait(B_PAIR + sub, n_pair)) { fail(); ok = false; break; }
#pragma unroll
      for (int t = 0; t < kTG; ++t) mx = fmaxf(mx, ms[128 * t + h]);
      mx *= p.scale_log2;
      const bool need = mx > m_run + kRescaleThreshold;
      const bool any_need = __any_sync(0xffffffffu, need);
      if (more) advance(p, plan, u_end, ex);
      // ------------------------------------------------ softmax of row h, this thread's kTokT tokens
      const float mu = need ? mx : m_run;
      const float al = need ? ptx::ex2(m_run - mu) : 1.f;
      const float nz = (mu == -CUDART_INF_F) ? 0.f : -mu;
      uint32_t ph[kTokT / 2], pl[kTokT / 2];
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kTokT / 2; ++i) {
        const float a0 = ptx::ex2(fmaf(v[2 * i], p.scale_log2, nz));
        const float a1 = ptx::ex2(fmaf(v[2 * i + 1], p.scale_log2, nz));
        sum4[i & 3] += a0 + a1;
        // P_hi = the top 16 bits of p (bf16 truncation), P_lo = the top 16 bits of the
        // exact remainder: P_hi + P_lo is within 2^-15 of p, with integer and FMA-pipe
        // operations only (no conversions on the special-function pipe, which the
        // exponentials already load)
        const uint32_t u0 = __float_as_uint(a0), u1 = __float_as_uint(a1);
        ph[i] = __byte_perm(u0, u1, 0x7632);
        const float r0 = a0 - __uint_as_float(u0 & 0xFFFF0000u), r1 = a1 - __uint_as_float(u1 & 0xFFFF0000u);
        pl[i] = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x7632);
      }
      l_run = l_run * al + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      m_run = mu;
      if (tracer) PAIR_TRACE(6, gpg);
      // ------------------------------------------------ P to TMEM once the previous value MMAs are done
      if (gpg > 0 && !wait_all(bar(B_O_DONE), (gpg - 1) & 1)) { fail(); ok = false; break; }
      ptx::tc_fence_after();
      if (tracer) PAIR_TRACE(7, gpg);
      ptx::tmem_st_cols<kTokT / 2>(tbase + lane_addr + kColP + (kTokT / 2) * tg, ph);
      ptx::tmem_st_cols<kTokT / 2>(tbase + lane_addr + kColP + 32 + (kTokT / 2) * tg, pl);
      if (cur.k > 0 && any_need) {
        // a moved reference: O[h][:] *= 2^(m_old - m_new) (1 for rows that kept theirs);
        // this thread scales its 256 / kTG columns
#pragma unroll 1
        for (int c = 0; c < 8 / kTG; ++c) {
          uint32_t o[32];
          const uint32_t ta = tbase + lane_addr + kColO + (256 / kTG) * tg + 32 * c;
          ptx::tmem_ld_32x32b_x32(ta, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * al);
          ptx::tmem_st_32x32b_x32(ta, o);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::fence_proxy_async_smem();   // the rope box's use above before the stage's next load
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_P_FULL));
      // the previous unit's O; this unit's first value MMA also waits for it (O_FREE)
      if (pend.on && !epilogue()) { fail(); ok = false; break; }

      if (cur.k == u.npg - 1) {
        pend.on = true;
        pend.item = u.item;
        pend.n = u.n;
        pend.part0 = u.part[0];
        pend.part1 = u.part[1];
        pend.stage = gpg % kStages;
        pend.l = l_run;
        pend.m = m_run;
      }
      advance(p, plan, u_end, cur);
      ++gpg;
    }
    if (ok && pend.on && !(wait_all(bar(B_O_DONE), (gpg - 1) & 1) && epilogue())) fail();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, kTmemCols);
  }
  ptx::cluster_sync();   // the peer no longer writes here
}

}  // namespace pair
}  // namespace mla
