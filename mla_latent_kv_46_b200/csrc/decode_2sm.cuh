// decode_2sm.cuh -- MLA decode attention on a pair of SMs (tcgen05 cta_group::2).
//
// A cluster of two CTAs serves one slot of the split plan. The pair holds 128 query
// rows: CTA r owns rows 64r..64r+63, i.e. heads 64r.. of one query token for H=128,
// or the 64 heads of the unit's token r for H=64 (two consecutive query tokens of a
// sequence per unit; with one token, CTA 1's rows are idle). For every 64-token page
// of a unit the even CTA issues, for both CTAs at once:
//   scores  S = Q . KV^T         tcgen05.mma.cta_group::2 M=128 (rows) x N=64 (tokens)
//                                x K=576; CTA r brings its 64 query rows and the page's
//                                tokens 32r..32r+31 (all 576 columns), and receives its
//                                rows' scores for all 64 tokens
//   values  O^T += C^T . P^T     tcgen05.mma.cta_group::2 M=256 (latent) x N=128 (rows)
//                                x K=64, twice (latent 0-255, 256-511); CTA r brings the
//                                page's 64 tokens of its own 128 latent columns of each
//                                half (128r.. and 256+128r..) and its rows' P, and
//                                receives O^T for those latent columns and all 128 rows
// The tensor cores combine the two CTAs' operands. Each CTA holds complete scores for
// its own rows, so the softmax runs once per row, in the CTA that owns it; the value
// MMA runs at full rate (128 rows per SM), while the score MMA, with 64 rows per SM,
// runs at half rate. The price of splitting the work this way is that each CTA also
// stages its own latent half of the page's other 32 tokens (per page a CTA stages
// 36 + 32 KiB; the pair reads 72 KiB of HBM, the rest is a second read of lines the
// peer loads at the same time, served by L2), and that each CTA's O^T holds every row:
// the rows' rescale factors (per page) and 1 / l (per unit) go to both CTAs.
//
// TMEM (512 columns, both CTAs):
//   [0,256)   O^T: lane L of region lh (columns 128lh..) is latent 256lh + 128r + L, one
//             column per row of the pair (rows 0-63 the even CTA's, 64-127 the odd's)
//   [256,288) the score buffer (a pair MMA with M=128 holds row m of the CTA in lanes m
//             and 64+m): lane half h holds tokens 32h..32h+31
//   [288,512) the score MMA's A operand for latent columns 0-447 of the query (bf16
//             pairs, 32 columns per 64 dims), row m in lanes m and 64+m
// Shared memory: the query's latent columns 448-511 and rope (two 64-row boxes), three
// score-operand slots (the page's own 32 tokens x 576: nine 32-row boxes), two
// value-operand slots (64 tokens x own 256 latent: eight 32-row boxes), and two
// buffers of P as bf16 (K-major, 64 rows x 64 tokens) with its remainder P_lo, so that
// page g's P is written while page g-1's value MMAs read the other buffer.
//
// P enters the value MMA in bf16 (round to nearest). Where one token can carry a
// large share of a row's weight, one bf16 rounding of P moves the output by more than
// the bf16 tolerance, so the value MMA is issued a second time with P_lo = bf16(p -
// bf16(p)) on the pages where some row of the pair has max_t p_t > l / 16 (l the
// row's running sum so far, of which each thread knows its own half: a conservative
// test). Elsewhere the single rounding is well inside the tolerance.
//
// Online softmax with a lazily moved per-row reference maximum, moved only when a
// page's maximum exceeds it by more than 2^24 (p and the fp32 sums stay far inside
// their range below that); a moved reference rescales the row's column of O^T in both
// CTAs.
//
// Warp roles (256 threads per CTA): warp 0 loads the query's shared-memory part and
// the score operands, warp 2 the value operands, warp 1 allocates TMEM and (even CTA)
// issues the MMAs, warps 4-7 stage the query's TMEM part, run the softmax and the
// epilogue (warp w reaches TMEM lanes 32(w%4)..).
//
// Barriers that gate an MMA live in the even CTA: both CTAs' TMA loads count their
// bytes there, and the odd CTA's warps arrive there remotely: arrivals that only
// report finished TMEM reads are relaxed; P's arrival has CTA-scope release (the data
// is in the arriving CTA's own shared memory) and the odd CTA's P_lo requests travel
// as st.async words whose bytes complete on the same barrier. Rescale factors and 1 / l
// travel the same way to a barrier of the receiving CTA. MMA completion is committed
// to both CTAs. Every wait is bounded; a CTA that gives up raises the device status
// word and sets both CTAs' abort flags.
//
// 8-bit cache (template F8 = true; codes and per-token power-of-two scales, see
// fp8_kernels.cuh). The query arrives split into two E4M3 pieces per element (hi, lo)
// times 2^e per row. Scores: one tcgen05.mma.cta_group::2.kind::f8f6f4 with M = 256 per
// K step of 32 codes: each CTA's 128 A rows are its 64 rows' hi pieces (TMEM lanes 0-63)
// and lo pieces (lanes 64-127), so lane m holds hi . codes and lane 64 + m lo . codes of
// row m for all 64 tokens; the two softmax warps of those lanes swap one half of the
// columns through shared memory and add. The softmax scales column t by the token's 2^k
// and the row by 2^-e. Values: four more warps (one warpgroup) widen the page's codes of
// the CTA's 256 latent columns, times 2^k, to bf16 in the value slot (exact), so the value
// MMA and P are those of the bf16 cache. Warp 2 loads those codes and the page's 64
// scale bytes into a local ring; the converter publishes the page's scales to the softmax
// before it waits for a free value slot.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "decode_tc.cuh"

namespace mla {
namespace duo {

constexpr int kRows = 128;             // MMA rows of the pair
constexpr int kCtaRows = 64;           // rows per CTA
constexpr int kPage = 64, kR = 512, kDr = 64, kRow = kR + kDr;
constexpr int kChunks = kRow / 64;     // 64-column chunks of a row (8 latent + rope)
constexpr int kQTmemChunks = 7;        // query chunks held in TMEM (latent 0-447)
constexpr int kQSmemChunks = kChunks - kQTmemChunks;   // latent 448-511 and rope
constexpr int kBox32 = 32 * 128;       // 32 rows x 128 bytes, 128-byte swizzle
constexpr int kBox64 = 64 * 128;       // 64 rows x 128 bytes
constexpr int kPBytes = kCtaRows * kPage * 2;      // 8,192
constexpr int kSoftWarps = 4;
constexpr int kFirstSoftWarp = 4;
constexpr int kFirstConvWarp = 8;      // (8-bit cache) the warpgroup that widens value operands
constexpr int kConvWarps = 4;
// 8-bit cache: a row is 576 one-byte codes; TMA boxes are 128 codes wide, the fifth (at
// column 512) holds the 64 rope codes and 64 columns of zero fill
constexpr int kF8Boxes = 5;
constexpr int kF8Steps = kRow / 32;    // K steps of 32 codes per row (18)
constexpr int kF8QTmemSteps = 14;      // of which the query holds 0-13 (columns 0-447) in TMEM

// Shared-memory layout: F8 = false for the bf16 cache, true for the 8-bit cache.
template <bool F8>
struct Lay {
  static constexpr int kThreads = 32 * (F8 ? kFirstConvWarp + kConvWarps : kFirstSoftWarp + kSoftWarps);
  // the query's shared-memory part: bf16 latent 448-511 and rope (two 64-row boxes), or
  // (F8) the high and low E4M3 pieces of columns 448-575 (one 64-row box each)
  static constexpr int kQBytes = kQSmemChunks * kBox64;                  // 16,384
  static constexpr int kQKSlotBytes = (F8 ? kF8Boxes : kChunks) * kBox32;   // 20,480 / 36,864
  static constexpr int kQKSlots = 3;
  static constexpr int kPV8SlotBytes = 2 * kBox64;   // (F8) 64 tokens x the CTA's two 128-code latent blocks
  static constexpr int kPV8Slots = F8 ? 2 : 0;
  static constexpr int kPVSlotBytes = 8 * kBox32;    // 32,768
  static constexpr int kPVSlots = 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffQK = kOffQ + kQBytes;
  static constexpr int kOffPV8 = kOffQK + kQKSlots * kQKSlotBytes;
  static constexpr int kOffPV = kOffPV8 + kPV8Slots * kPV8SlotBytes;
  static constexpr int kOffP = kOffPV + kPVSlots * kPVSlotBytes;   // two buffers of P_hi then P_lo
  static constexpr int kOffXch = kOffP + 4 * kPBytes;               // (F8) float[128][32]: score halves exchanged
  static constexpr int kOffXs8 = kOffXch + (F8 ? 128 * 32 * 4 : 0);   // (F8) uint8[slot][64]: scale bytes per code slot
  static constexpr int kOffXsc = kOffXs8 + (F8 ? kPV8Slots * 64 : 0);  // (F8) float[4][64]: token scales
  static constexpr int kMaxBars = F8 ? 40 : 32;
  static constexpr int kOffBar = kOffXsc + (F8 ? 4 * 64 * 4 : 0);  // kMaxBars mbarriers
  static constexpr int kOffXmax = kOffBar + kMaxBars * 8;   // float[2][128]: row maxima of the lane halves
  static constexpr int kOffXl = kOffXmax + 2 * 128 * 4;     // float[128]: row sums of the lane halves
  static constexpr int kOffFlag = kOffXl + 128 * 4;         // uint32[4][8] (even CTA): P_lo wanted, per tile % 4
                                                            // and softmax warp (0-3 even CTA, 4-7 odd CTA)
  static constexpr int kOffXal = kOffFlag + 4 * 8 * 4;      // float[2][128]: the pair's rescale factors, per row
  static constexpr int kOffXflg = kOffXal + 2 * 128 * 4;    // uint32[2][4]: a moved reference among 32 rows
  static constexpr int kOffXinv = kOffXflg + 2 * 4 * 4;     // float[128]: the pair's 1 / l, per row
  static constexpr int kOffTmem = kOffXinv + 128 * 4;
  static constexpr int kOffAbort = kOffTmem + 8;
  static constexpr int kSmemUsed = kOffAbort + 8;
  static constexpr int kSmemBytes = kSmemUsed + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
  static_assert(kOffQK % 1024 == 0 && kOffPV8 % 1024 == 0 && kOffPV % 1024 == 0 && kOffP % 1024 == 0 &&
                    kOffXs8 % 16 == 0 &&
                    kQKSlotBytes % 1024 == 0,
                "swizzled buffers on 1 KiB boundaries");
};
constexpr int kThreads = Lay<false>::kThreads;
constexpr int kSmemBytes = Lay<false>::kSmemBytes;
constexpr int kThreadsF8 = Lay<true>::kThreads;
constexpr int kSmemBytesF8 = Lay<true>::kSmemBytes;

enum {
  B_QK_FULL = 0,                   // +slot (even CTA): score operands of both CTAs landed
  B_QK_EMPTY = B_QK_FULL + 3,      // +slot: score MMAs that read the slot done
  B_PV_FULL = B_QK_EMPTY + 3,      // +slot (even CTA): value operands landed
  B_PV_EMPTY = B_PV_FULL + 2,      // +slot: value MMAs that read the slot done
  B_Q_FULL = B_PV_EMPTY + 2,       // (even CTA) the unit's query in both CTAs: TMA bytes of the
                                   // shared-memory part, one arrival per softmax warp for TMEM
  B_Q_EMPTY,                       // last score MMA of a unit done
  B_S_FULL,                        // score MMAs done
  B_S_EMPTY,                       // (even CTA) both CTAs' softmax warps read S
  B_P_FULL,                        // (even CTA) P of both CTAs in shared memory, O rescaled
  B_O_DONE,                        // +P buffer: value MMAs that read the buffer done
  B_O_FREE = B_O_DONE + 2,                        // (even CTA) both CTAs' epilogues have read O
  B_PAIR,                          // +1: the two softmax warps of rows 0-31 / 32-63
  B_AL_FULL = B_PAIR + 2,          // +buffer: both CTAs' rescale factors of a page (local arrivals,
                                   // the peer's words as transaction bytes)
  B_LX_FULL = B_AL_FULL + 2,       // both CTAs' 1 / l of a unit (likewise)
  B_ALL4,                          // the four softmax warps (epilogue staging)
  B_DRAIN,
  B_PV8_FULL,                      // +slot (F8): this CTA's value codes landed
  B_PV8_EMPTY = B_PV8_FULL + 3,    // +slot (F8): this CTA's converter warps read them
  B_CV_FULL = B_PV8_EMPTY + 3,     // +page % 4 (F8): this CTA's token scales of the page written
  kNumBars = B_CV_FULL + 4
};
static_assert(kNumBars <= Lay<true>::kMaxBars && B_PV8_FULL <= Lay<false>::kMaxBars, "barrier area");
static_assert(Lay<true>::kQKSlots <= 3 && Lay<true>::kPVSlots <= 2 && Lay<true>::kPV8Slots <= 3, "barrier slots");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 256, kColQ = 288;
static_assert(kColQ + 32 * kQTmemChunks <= kTmemCols, "TMEM columns");
// (F8) scores of an M = 256 MMA: 64 columns; the query piece of each lane: 112 columns
constexpr uint32_t kColQ8 = kColS + 64;
static_assert(kColQ8 + 4 * kF8QTmemSteps * 2 <= kTmemCols, "TMEM columns (8-bit cache)");
constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(128, 64, 0, 0);    // Q (K-major) x KV^T (K-major)
constexpr uint32_t kIdescV = ptx::idesc_bf16_f32(256, 128, 1, 0);   // C^T (M-major) x P^T (K-major)
constexpr uint32_t kIdescS8 = ptx::idesc_e4m3_f32(256, 64, 0, 0);   // (F8) query pieces x codes, both K-major
// log2 units: p stays below 2^24, far inside the range of the bf16 P and of the fp32
// sums (at most 2^24 x 2^17 tokens x |c|), so the reference moves (and O is rescaled)
// only when a row's maximum jumps by that much, which almost never happens
constexpr float kRescaleThreshold = 24.0f;
constexpr uint32_t kAlBytes = 64 * 4 + 2 * 4;   // one CTA's rescale factors and votes
constexpr float kLoShare = 16.0f;           // P_lo wanted when 16 * max p > l

using tc::Params;

// A plan unit: the rows of n (1 or 2) consecutive query tokens of sequence b over
// pages [pb, pb + npg).
struct Unit2 {
  int32_t item, b, pb, npg, n;
  int32_t ntok[2];   // tokens each token sees (-1: absent)
  int32_t part[2];   // partial-output index of each token, or -1: final result
};

__device__ __forceinline__ Unit2 load_unit2(const Params& p, const PlanView& plan, int32_t idx) {
  const Unit u = plan.units()[idx];
  Unit2 r;
  r.item = u.item;
  r.b = u.b;
  r.pb = u.page_begin;
  r.n = u.pad1 > 1 ? 2 : 1;
  const int32_t q_len = plan.q_len(), L = p.seq_lens[u.b];
  r.ntok[0] = visible_tokens(L, q_len, u.item % q_len);
  r.ntok[1] = r.n > 1 ? visible_tokens(L, q_len, u.item % q_len + 1) : -1;
  r.part[0] = u.part;
  r.part[1] = r.n > 1 ? u.pad0 : -1;
  const int32_t last = (max(r.ntok[0], r.ntok[1]) + kPage - 1) / kPage;
  const int32_t pe = min(u.page_end, min(last, p.max_pages));
  r.npg = max(0, pe - r.pb);
  return r;
}

// Optional event trace (-DMLA_TRACE): per CTA 1024 clock64 values, 16 regions of 64
// tiles: 0 score operand load issued, 1 value operand load issued, 2 score operand
// landed (MMA warp), 3 score MMA issued, 4 P of both CTAs ready (MMA warp), 5 value
// MMA issued, 6 scores read (softmax warp 4), 7 P stored (softmax warp 4), 8 value
// operand landed (MMA warp), 9 query staged in TMEM (softmax warp 4, per unit), 10 and
// 11 epilogue start and end (softmax warp 4, per unit), 12 unit's query ready and 13
// the previous unit's O read (MMA warp, per unit), 14 epilogue: both CTAs' 1 / l
// received; slot 1020 the SM id, 1021 the global timer at start, 1022 clock at exit,
// 1023 at start.
#ifdef MLA_TRACE
#define DUO_TRACE(region, g)                                                                     \
  do {                                                                                           \
    if (p.trace && (g) < 60)                                                                     \
      p.trace[(size_t)blockIdx.x * 1024 + 64 * (region) + (g)] = (unsigned long long)clock64(); \
  } while (0)
#else
#define DUO_TRACE(region, g) \
  do {                       \
  } while (0)
#endif

// Walks the pages of a slot's non-empty units in order.
struct Cursor {
  int32_t ui, k;
  uint32_t n;   // ordinal of the unit among the slot's non-empty units
  bool valid;
  Unit2 u;
};

__device__ __forceinline__ bool next_unit(const Params& p, const PlanView& plan, int32_t& ui, int32_t u_end,
                                          Unit2& u) {
  while (++ui < u_end) {
    u = load_unit2(p, plan, ui);
    if (u.npg > 0) return true;
  }
  return false;
}

__device__ __forceinline__ Cursor first_page(const Params& p, const PlanView& plan, int32_t u_begin,
                                             int32_t u_end) {
  Cursor c;
  c.ui = u_begin - 1;
  c.k = 0;
  c.n = 0;
  c.valid = next_unit(p, plan, c.ui, u_end, c.u);
  return c;
}

__device__ __forceinline__ void advance(const Params& p, const PlanView& plan, int32_t u_end, Cursor& c) {
  if (!c.valid) return;
  if (++c.k < c.u.npg) return;
  c.k = 0;
  ++c.n;
  c.valid = next_unit(p, plan, c.ui, u_end, c.u);
}

__device__ __forceinline__ int32_t page_id(const Params& p, const Unit2& u, int32_t k, bool report) {
  int32_t page = p.block_table[(int64_t)u.b * p.max_pages + u.pb + k];
  if (page < 0 || page >= p.num_pages) {
    if (report) raise_status(kStatusBadPage);
    page = p.num_pages;   // rows past the tensor: the loads fill zeros
  }
  return page;
}

// F8 = false: bf16 cache; tm_kv: the cache in 32-row boxes, tm_q / tm_qr: q_lat / q_rope
// in 64-row boxes. F8 = true: 8-bit cache (codes and per-token scales, p.kv_scale);
// tm_kv: the codes in 32-row boxes of 128 codes, tm_q: the split query (p.q8) in 64-row
// boxes (high pieces), tm_ql: the same for the low pieces, tm_qr: the codes in 64-row
// boxes. tm_o / tm_op: fp32 output stores (final rows, partial rows).
template <bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Lay<F8>::kThreads, 1)
decode_2sm_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_qr, const __grid_constant__ CUtensorMap tm_o,
                  const __grid_constant__ CUtensorMap tm_op, const __grid_constant__ CUtensorMap tm_ql,
                  const Params p) {
  using L = Lay<F8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const uint32_t rank = ptx::cluster_rank();
  const bool even = rank == 0;
  auto bar = [&](int i) { return sbase + L::kOffBar + 8u * i; };
  auto lead = [&](uint32_t local) { return ptx::map_peer(local, 0); };   // the even CTA's copy
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kOffAbort);
  volatile uint32_t* lo_flag = reinterpret_cast<volatile uint32_t*>(smem + L::kOffFlag);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PlanView plan{p.plan};
  const int slot = blockIdx.x >> 1;
  const int32_t u_begin = plan.slot_begin()[slot], u_end = plan.slot_begin()[slot + 1];
  const int32_t H = p.H;   // 128, or 64 with up to two query tokens per unit
  const int64_t TH = (int64_t)plan.B() * plan.q_len() * H;   // query rows

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 32; ++i) lo_flag[i] = 0u;
    for (int s = 0; s < L::kQKSlots; ++s) {
      ptx::mbar_init(bar(B_QK_FULL + s), 1);
      ptx::mbar_init(bar(B_QK_EMPTY + s), 1);
    }
    for (int s = 0; s < L::kPVSlots; ++s) {
      // bf16: the TMA bytes; F8: every converter warp of both CTAs
      ptx::mbar_init(bar(B_PV_FULL + s), F8 ? 2 * kConvWarps : 1);
      ptx::mbar_init(bar(B_PV_EMPTY + s), 1);
    }
    if constexpr (F8) {
      for (int s = 0; s < L::kPV8Slots; ++s) {
        ptx::mbar_init(bar(B_PV8_FULL + s), 1);
        ptx::mbar_init(bar(B_PV8_EMPTY + s), kConvWarps);
      }
      for (int i = 0; i < 4; ++i) ptx::mbar_init(bar(B_CV_FULL + i), kConvWarps / 2);   // warps of block 0
    }
    ptx::mbar_init(bar(B_S_FULL), 1);
    ptx::mbar_init(bar(B_S_EMPTY), 2 * kSoftWarps);
    ptx::mbar_init(bar(B_Q_FULL), 1 + 2 * kSoftWarps);
    ptx::mbar_init(bar(B_Q_EMPTY), 1);
    ptx::mbar_init(bar(B_P_FULL), 2 * kSoftWarps);
    ptx::mbar_init(bar(B_O_DONE), 1);
    ptx::mbar_init(bar(B_O_DONE + 1), 1);
    ptx::mbar_init(bar(B_O_FREE), 2 * kSoftWarps);
    ptx::mbar_init(bar(B_PAIR), 2);
    ptx::mbar_init(bar(B_PAIR + 1), 2);
    ptx::mbar_init(bar(B_AL_FULL), 2);
    ptx::mbar_init(bar(B_AL_FULL + 1), 2);
    ptx::mbar_init(bar(B_LX_FULL), 2);
    ptx::mbar_init(bar(B_ALL4), kSoftWarps);
    ptx::mbar_init(bar(B_DRAIN), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(sbase + L::kOffTmem, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_kv);
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_qr);
    ptx::prefetch_tmap(&tm_o);
    ptx::prefetch_tmap(&tm_op);
    if (F8) ptx::prefetch_tmap(&tm_ql);
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // both CTAs' barriers exist before anyone arrives, loads or issues
  ptx::tc_fence_after();
  const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(smem + L::kOffTmem);
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && p.trace) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    unsigned long long* tr = p.trace + (size_t)blockIdx.x * 1024;
    tr[1020] = smid;
    tr[1021] = ptx::globaltimer_ns();
    tr[1023] = (unsigned long long)clock64();
  }
#endif

  auto fail = [&]() {
    raise_status(kStatusTimeout);
    *abort_flag = 1;
    ptx::st_cluster_u32(ptx::map_peer(sbase + L::kOffAbort, rank ^ 1u), 1u);
  };
  auto wait_all = [&](uint32_t b, uint32_t parity) -> bool {
    return __all_sync(0xffffffffu, ptx::mbar_wait_cluster_bounded(b, parity, abort_flag, p.timeout_ns));
  };

  if (warp == 0 || warp == 2) {
    // ================================================================ TMA producers
    // warp 0: each page's score operand (own 32 tokens x 576); warp 2: each page's value
    // operand (64 tokens x own 256 latent)
    const bool leader = ptx::elect_one();
    const bool qk = warp == 0;
    // F8: warp 2 loads this CTA's value codes for its own converters (local barriers)
    const int nslots = qk ? L::kQKSlots : (F8 ? L::kPV8Slots : L::kPVSlots);
    const int empty_bar = qk ? B_QK_EMPTY : (F8 ? B_PV8_EMPTY : B_PV_EMPTY);
    const int full_bar = qk ? B_QK_FULL : (F8 ? B_PV8_FULL : B_PV_FULL);
    Cursor c = first_page(p, plan, u_begin, u_end);
    uint32_t g = 0;
    bool ok = true;
    while (c.valid && ok) {
      const uint32_t s = g % nslots, ph = (g / nslots) & 1;
      if (!wait_all(bar(empty_bar + s), ph ^ 1)) { if (leader) fail(); ok = false; break; }
      const int32_t page = page_id(p, c.u, c.k, leader && qk);
      // (the testing hook leaves the page's barrier without the even CTA's load: the waits
      // on it run out and the kernel reports a timeout)
      const bool drop = qk && blockIdx.x == 0 && (int32_t)g == p.drop_load;
      if (leader) {
        if (qk) {
          // all nine boxes of the page at once (issued together, the page's rows are read
          // from DRAM together)
          DUO_TRACE(0, g);
          if (even) ptx::mbar_arrive_expect_tx(bar(B_QK_FULL + s), 2 * L::kQKSlotBytes);
          if (!drop) {
            const uint32_t dst = sbase + L::kOffQK + s * L::kQKSlotBytes;
            constexpr int nbox = F8 ? kF8Boxes : kChunks, wbox = F8 ? 128 : 64;
#pragma unroll 1
            for (int ch = 0; ch < nbox; ++ch)
              ptx::tma_load_2d_pair(dst + ch * kBox32, &tm_kv, lead(bar(B_QK_FULL + s)), wbox * ch,
                                    page * kPage + 32 * (int32_t)rank);
          }
        } else if constexpr (F8) {
          // the CTA's latent blocks 2hh + rank (128 codes each) of all 64 tokens, and the
          // page's 64 scale bytes (those of page 0 stand in for a page id outside the pool:
          // its codes read as zeros)
          DUO_TRACE(1, g);
          ptx::mbar_arrive_expect_tx(bar(B_PV8_FULL + s), L::kPV8SlotBytes + 64);
          const uint32_t dst = sbase + L::kOffPV8 + s * L::kPV8SlotBytes;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            ptx::tma_load_2d(dst + hh * kBox64, &tm_qr, bar(B_PV8_FULL + s), 128 * (2 * hh + (int)rank),
                             page * kPage);
          ptx::bulk_load_g2s(sbase + L::kOffXs8 + s * 64,
                             p.kv_scale + (int64_t)(page < p.num_pages ? page : 0) * kPage, 64, bar(B_PV8_FULL + s));
        } else {
          DUO_TRACE(1, g);
          if (even) ptx::mbar_arrive_expect_tx(bar(B_PV_FULL + s), 2 * L::kPVSlotBytes);
          const uint32_t dst = sbase + L::kOffPV + s * L::kPVSlotBytes;
          // box (hh, th, b) at ((hh * 2 + th) * 2 + b): latent block 4hh + 2r + b, tokens 32th..
#pragma unroll 1
          for (int i = 0; i < 8; ++i) {
            const int hh = i >> 2, th = (i >> 1) & 1, b = i & 1;
            ptx::tma_load_2d_pair(dst + i * kBox32, &tm_kv, lead(bar(B_PV_FULL + s)),
                                  64 * (4 * hh + 2 * (int)rank + b), page * kPage + 32 * th);
          }
        }
      }
      advance(p, plan, u_end, c);
      ++g;
    }
    // The even CTA's barriers count both CTAs' loads: before the pair exits, wait for the
    // phases armed last, so no copy is still landing in either CTA. These waits ignore the
    // abort flag (copies in flight land within microseconds) and stop at the wait bound;
    // after one runs out (a phase that cannot complete) the rest are skipped.
    if (even || (F8 && !qk)) {   // (F8: each CTA's value codes count on its own barriers)
      bool landed = true;
      for (uint32_t k = (g >= (uint32_t)nslots ? g - nslots : 0); k < g && landed; ++k)
        landed = __all_sync(0xffffffffu, ptx::mbar_wait_cluster_timed(bar(full_bar + k % nslots),
                                                                      (k / nslots) & 1, p.timeout_ns));
    }
  } else if (warp == 3) {
    // ================================================================ the query's shared-memory part
    // per unit (latent 448-511 and rope of the CTA's 64 rows), once the previous unit's
    // last score MMA is done; the even CTA also prefetches the next unit's query rows
    // into L2 for the softmax warps, which stage the TMEM part
    const bool leader = ptx::elect_one();
    int32_t ui = u_begin - 1;
    Unit2 u;
    uint32_t nq = 0;
    bool have = next_unit(p, plan, ui, u_end, u);
    while (have) {
      Unit2 nu;
      int32_t ni = ui;
      const bool more = next_unit(p, plan, ni, u_end, nu);
      if (even && leader && more) {
        const int64_t qrow = (int64_t)nu.item * H;
        const int64_t rows = min((int64_t)kRows, TH - qrow);
        if (rows > 0) {
          if constexpr (F8) {
            ptx::prefetch_l2_bulk(p.q8 + qrow * kRow, (uint32_t)(rows * kRow));
            ptx::prefetch_l2_bulk(p.q8 + (TH + qrow) * kRow, (uint32_t)(rows * kRow));
          } else {
            ptx::prefetch_l2_bulk(p.q_lat + qrow * kR, (uint32_t)(rows * kR * 2));
          }
        }
      }
      if (!wait_all(bar(B_Q_EMPTY), (nq & 1) ^ 1)) { if (leader) fail(); break; }
      if (leader) {
        if (even) ptx::mbar_arrive_expect_tx(bar(B_Q_FULL), 2 * L::kQBytes);
        const int32_t qrow = u.item * H + kCtaRows * (int32_t)rank;   // rows past the tensor read zeros
        if constexpr (F8) {
          // columns 448-575 of the high and the low pieces
          ptx::tma_load_2d_pair(sbase + L::kOffQ, &tm_q, lead(bar(B_Q_FULL)), 32 * kF8QTmemSteps, qrow);
          ptx::tma_load_2d_pair(sbase + L::kOffQ + kBox64, &tm_ql, lead(bar(B_Q_FULL)), 32 * kF8QTmemSteps, qrow);
        } else {
#pragma unroll 1
          for (int ch = 0; ch < kQSmemChunks - 1; ++ch)
            ptx::tma_load_2d_pair(sbase + L::kOffQ + ch * kBox64, &tm_q, lead(bar(B_Q_FULL)),
                                  64 * (kQTmemChunks + ch), qrow);
          ptx::tma_load_2d_pair(sbase + L::kOffQ + (kQSmemChunks - 1) * kBox64, &tm_qr, lead(bar(B_Q_FULL)), 0,
                                qrow);
        }
      }
      ++nq;
      ui = ni;
      u = nu;
      have = more;
    }
    if (even && nq > 0) wait_all(bar(B_Q_FULL), (nq - 1) & 1);
  } else if (warp == 1) {
    // ================================================================ MMA issuer (even CTA)
    if (even) {
      const bool leader = ptx::elect_one();
      bool ok = true;
      Cursor qc = first_page(p, plan, u_begin, u_end);   // next score MMA
      Cursor vc = qc;                                     // next value MMA
      uint32_t gq = 0, gv = 0;
      auto issue_s = [&]() -> bool {
        if (qc.k == 0 && !wait_all(bar(B_Q_FULL), qc.n & 1)) return false;
        if (qc.k == 0 && leader) DUO_TRACE(12, qc.n);
        const uint32_t s = gq % L::kQKSlots, ph = (gq / L::kQKSlots) & 1;
        if (!wait_all(bar(B_QK_FULL + s), ph)) return false;
        if (leader) DUO_TRACE(2, gq);
        if (!wait_all(bar(B_S_EMPTY), (gq & 1) ^ 1)) return false;   // both CTAs read S(gq - 1)
        ptx::tc_fence_after();
        const uint32_t kvs = sbase + L::kOffQK + s * L::kQKSlotBytes;
        const uint32_t d_s = tbase + kColS;
        if (leader) {
          DUO_TRACE(3, gq);
          if constexpr (F8) {
            // M = 256: each CTA's 128 A rows are its 64 query rows' high pieces (lanes
            // 0-63) and low pieces (lanes 64-127), so each SM runs a full 128-row MMA. K
            // steps of 32 codes: step j reads box j / 4 of the page at byte 32 (j % 4); the
            // query's steps 0-13 are in TMEM (column 8j), steps 14-17 in shared memory (the
            // high box's 64 rows, then the low box's)
#pragma unroll 1
            for (int j = 0; j < kF8Steps; ++j) {
              const uint64_t dk = ptx::sdesc_sw128(kvs + (j >> 2) * kBox32, 16, 1024) + (uint64_t)(2 * (j & 3));
              if (j < kF8QTmemSteps)
                ptx::umma_pair_ts_f8(d_s, tbase + kColQ8 + 8u * j, dk, kIdescS8, j ? 1u : 0u);
              else
                ptx::umma_pair_ss_f8(d_s, ptx::sdesc_sw128(sbase + L::kOffQ, 16, 1024) +
                                              (uint64_t)(2 * (j - kF8QTmemSteps)),
                                     dk, kIdescS8, 1u);
            }
          } else {
#pragma unroll 1
          for (int ch = 0; ch < kChunks; ++ch) {
            const uint64_t dk = ptx::sdesc_sw128(kvs + ch * kBox32, 16, 1024);
            if (ch < kQTmemChunks) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                ptx::umma_pair_ts(d_s, tbase + kColQ + 32u * ch + 8u * kk, dk + (uint64_t)(2 * kk), kIdescS,
                                  (ch | kk) ? 1u : 0u);
            } else {
              const uint64_t dq = ptx::sdesc_sw128(sbase + L::kOffQ + (ch - kQTmemChunks) * kBox64, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                ptx::umma_pair_ss(d_s, dq + (uint64_t)(2 * kk), dk + (uint64_t)(2 * kk), kIdescS, 1u);
            }
          }
          }
          ptx::umma_commit_pair(bar(B_QK_EMPTY + s), 3);
          ptx::umma_commit_pair(bar(B_S_FULL), 3);
          if (qc.k == qc.u.npg - 1) ptx::umma_commit_pair(bar(B_Q_EMPTY), 3);
        }
        __syncwarp();
        advance(p, plan, u_end, qc);
        ++gq;
        return true;
      };
      auto issue_v = [&]() -> bool {
        if (!wait_all(bar(B_P_FULL), gv & 1)) return false;
        if (leader) DUO_TRACE(4, gv);
        if (vc.k == 0 && vc.n > 0 && !wait_all(bar(B_O_FREE), (vc.n - 1) & 1)) return false;
        if (vc.k == 0 && leader) DUO_TRACE(13, vc.n);
        const uint32_t s = gv % L::kPVSlots, ph = (gv / L::kPVSlots) & 1;
        if (!wait_all(bar(B_PV_FULL + s), ph)) return false;
        if (leader) DUO_TRACE(8, gv);
        uint32_t want_lo = 0;
#pragma unroll
        for (int w = 0; w < 2 * kSoftWarps; ++w) want_lo |= lo_flag[8 * (gv & 3) + w];
        ptx::tc_fence_after();
        const uint32_t pvs = sbase + L::kOffPV + s * L::kPVSlotBytes;
        if (leader) {
          DUO_TRACE(5, gv);
#pragma unroll 1
          for (int part = 0; part < (want_lo ? 2 : 1); ++part) {
            const uint64_t dp = ptx::sdesc_sw128(sbase + L::kOffP + (2 * (gv & 1) + part) * kPBytes, 16, 1024);
#pragma unroll
            for (int lh = 0; lh < 2; ++lh) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                // O^T[latent][row] += C^T[latent][t] P^T[t][row], tokens 16kk..16kk+15: box
                // pair (lh, kk / 2) at rows 16 (kk % 2) holds this CTA's 128 latent rows
                const uint64_t dc =
                    ptx::sdesc_sw128(pvs + ((lh * 2 + (kk >> 1)) * 2) * kBox32 + (kk & 1) * 2048, kBox32, 1024);
                ptx::umma_pair_ss(tbase + kColO + 128u * lh, dc, dp + (uint64_t)(2 * kk), kIdescV,
                                  (part == 0 && vc.k == 0 && kk == 0) ? 0u : 1u);
              }
            }
          }
          ptx::umma_commit_pair(bar(B_PV_EMPTY + s), 3);
          ptx::umma_commit_pair(bar(B_O_DONE + (gv & 1)), 3);
        }
        __syncwarp();
        advance(p, plan, u_end, vc);
        ++gv;
        return true;
      };
      // S(0), then per page j: S(j+1), V(j)
      if (qc.valid && !issue_s()) { if (leader) fail(); ok = false; }
      while (vc.valid && ok) {
        if (qc.valid && !issue_s()) { if (leader) fail(); ok = false; break; }
        if (!issue_v()) { if (leader) fail(); ok = false; break; }
      }
      if (leader) ptx::umma_commit_pair(bar(B_DRAIN), 1);
      __syncwarp();
      wait_all(bar(B_DRAIN), 0);
    }
  } else if (F8 && warp >= kFirstConvWarp) {
    // ================================================================ (F8) value operands to bf16
    // Thread (t, hh) widens token t's 128 codes of latent block 2hh + rank into the bf16
    // value slot (the layout the bf16 cache's loads produce) times the token's scale 2^k:
    // a code's bits placed under a bf16 exponent field give the code's value times
    // 2^-120 (subnormal codes included), and one bf16 product by 2^(120+k) is exact. Rows
    // past the unit's visible tokens are written as zeros (P is zero there, and stale
    // codes must not turn into NaN). Thread t of the first block also publishes the
    // token's scale for the softmax warps (which apply it to the score column) as soon
    // as the page's codes and scale bytes land, before it waits for a free value slot.
    const int ct = (int)threadIdx.x - 32 * kFirstConvWarp;
    const int t = ct & 63, hh = ct >> 6;
    const int th = t >> 5, rr = t & 31;
    volatile float* xsc = reinterpret_cast<volatile float*>(smem + L::kOffXsc);
    Cursor c = first_page(p, plan, u_begin, u_end);
    uint32_t g = 0;
    while (c.valid) {
      constexpr uint32_t n8 = F8 ? L::kPV8Slots : 1;   // (the bf16 kernel has no such warps)
      const uint32_t s8 = g % n8, ph8 = (g / n8) & 1;
      const uint32_t sb = g & 1, phb = (g >> 1) & 1;
      const int32_t pos = (c.u.pb + c.k) * kPage + t;
      const bool valid = pos < max(c.u.ntok[0], c.u.ntok[1]);
      if (!wait_all(bar(B_PV8_FULL + s8), ph8)) { if (lane == 0) fail(); break; }
      uint32_t e = valid ? (uint32_t)smem[L::kOffXs8 + s8 * 64 + t] : 127u;
      e = min(max(e, 1u), 134u);   // 2^(120+k) must be a finite bf16
      // the page's token scales for the softmax warps first (ring of four: slot g % 4 was
      // read by the softmax of page g - 4, whose P the value MMAs of page g - 4 consumed
      // before this warp could convert page g - 2)
      if (hh == 0) {
        xsc[64 * (g & 3) + t] = valid ? __uint_as_float(e << 23) : 0.f;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(B_CV_FULL + (g & 3)));
      }
      if (!wait_all(bar(B_PV_EMPTY + sb), phb ^ 1)) { if (lane == 0) fail(); break; }
      const uint32_t src = sbase + L::kOffPV8 + s8 * L::kPV8SlotBytes + hh * kBox64 + t * 128;
      const uint32_t dst = sbase + L::kOffPV + sb * L::kPVSlotBytes + ((hh * 2 + th) * 2) * kBox32 + rr * 128;
      const uint32_t mul = ((e + 120u) << 7) * 0x00010001u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {   // codes 16j..16j+15 of the block
        uint32_t w[4];
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "r"(src + (uint32_t)((j ^ (t & 7)) << 4)));
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            // codes 4q + 2h2, 4q + 2h2 + 1 into the high bytes of the two 16-bit lanes
            const uint32_t x = __byte_perm(w[q], 0u, h2 ? 0x3424u : 0x1404u);
            const uint32_t y = ((x >> 4) & 0x07F007F0u) | (x & 0x80008000u);
            o[2 * q + h2] = valid ? ptx::mul_bf16x2(y, mul) : 0u;
          }
        }
        // bf16 elements 16j.. are 64-column block j / 4, 16-byte chunks 2 (j % 4) and 2 (j % 4) + 1
        const uint32_t row = dst + (uint32_t)((j >> 2) * kBox32);
        const int c0 = 2 * (j & 3);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (uint32_t)((c0 ^ (rr & 7)) << 4)),
                     "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + (uint32_t)(((c0 + 1) ^ (rr & 7)) << 4)),
                     "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                     : "memory");
      }
      ptx::fence_proxy_async_smem();   // the value MMAs read the slot through the async proxy
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(bar(B_PV8_EMPTY + s8));
        if (even) ptx::mbar_arrive(bar(B_PV_FULL + sb));
        else ptx::mbar_arrive_remote(lead(bar(B_PV_FULL + sb)));
      }
      advance(p, plan, u_end, c);
      ++g;
    }
  } else if (warp >= kFirstSoftWarp) {
    // ================================================================ query staging, softmax, epilogue
    const int sw = warp - kFirstSoftWarp;         // softmax warp 0-3
    const int q = warp & 3;                       // TMEM lane quarter
    const int L = 32 * q + lane;                  // this thread's TMEM lane
    // scores: row m of the CTA, tokens 32h..32h+31 of the page (h = lane half); O^T: latent
    // row 256lh + 128 rank + L of region lh, one column per row of the pair
    const int m = L & 63, half = L >> 6;
    const int prow = kCtaRows * (int)rank + m;    // this thread's score row among the pair's 128
    const uint32_t lane_addr = (32u * q) << 16;
    const int tok = H == kRows ? 0 : (int)rank;   // the unit's query token this CTA's rows belong to
    volatile float* xmax = reinterpret_cast<volatile float*>(smem + L::kOffXmax);
    volatile float* xl = reinterpret_cast<volatile float*>(smem + L::kOffXl);
    volatile float* xal = reinterpret_cast<volatile float*>(smem + L::kOffXal);
    volatile uint32_t* xflg = reinterpret_cast<volatile uint32_t*>(smem + L::kOffXflg);
    volatile float* xinv = reinterpret_cast<volatile float*>(smem + L::kOffXinv);
    auto peer = [&](uint32_t local) { return ptx::map_peer(local, rank ^ 1u); };
    uint32_t n_pair = 0, n_lx = 0, n_all4 = 0;
    bool ok = true;
    // the two warps of rows 32(q&1).. (lane halves 0 and 1) meet on B_PAIR + (q & 1)
    auto pair_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_PAIR + (q & 1)));
      const bool done = ptx::mbar_wait_bounded(bar(B_PAIR + (q & 1)), n_pair & 1, abort_flag, p.timeout_ns);
      ++n_pair;
      return __all_sync(0xffffffffu, done);
    };
    // the four softmax warps of this CTA
    auto all4_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(B_ALL4));
      const bool done = ptx::mbar_wait_bounded(bar(B_ALL4), n_all4 & 1, abort_flag, p.timeout_ns);
      ++n_all4;
      return __all_sync(0xffffffffu, done);
    };
    // arrivals on the even CTA's barriers that only report finished TMEM reads
    auto arrive_read = [&](int b) {
      if (even) ptx::mbar_arrive(bar(b));
      else ptx::mbar_arrive_cluster_relaxed(lead(bar(b)));
    };
    // query row of the pair's row n (H=64: rows 64.. are the unit's second token)
    auto qrow_of = [&](int32_t item, int n) -> int64_t { return (int64_t)item * H + n; };

    // Units without a visible token: o = 0, lse = -inf for this CTA's latent half of the
    // pair's rows (this thread: latent rows 128 rank + L and 256 + 128 rank + L).
    for (int32_t ui = u_begin; ui < u_end; ++ui) {
      const Unit2 u = load_unit2(p, plan, ui);
      if (u.npg > 0) continue;
      for (int n = 0; n < kRows; ++n) {
        const int tn = H == kRows ? 0 : n / kCtaRows;
        if (tn >= u.n) continue;
        const int64_t row = qrow_of(u.item, n);
        const int32_t prt = u.part[tn];
        for (int lh = 0; lh < 2; ++lh) {
          const int d = 256 * lh + 128 * (int)rank + L;
          if (prt < 0) p.o_lat[row * kR + d] = 0.f;
          else p.o_part[((int64_t)prt * H + row % H) * kR + d] = 0.f;
        }
      }
      if (half == 0 && tok < u.n) {
        const int64_t row = qrow_of(u.item, prow);
        const int32_t prt = u.part[tok];
        if (prt < 0) { if (p.lse) p.lse[row] = -CUDART_INF_F; }
        else p.lse_part[(int64_t)prt * H + row % H] = -CUDART_INF_F;
      }
    }

    // (F8) the staged query row's scale 2^-e (the split query holds the row times 2^e)
    float q_scale_next = 1.f;
    // The TMEM part of a unit's query (latent 0-447 of this thread's score row, both lane
    // halves hold it), once the previous unit's last score MMA is done.
    auto stage_q = [&](const Unit2& u, uint32_t n) -> bool {
      if (!wait_all(bar(B_Q_EMPTY), (n & 1) ^ 1)) return false;
      ptx::tc_fence_after();
      const int64_t row = qrow_of(u.item, prow);
      const bool inside = row < TH;   // rows past the query tensor (an absent token) stay zero
      if constexpr (F8) {
        // lane L holds piece L / 64 (high, low) of its row: codes 0-447 in columns 0-111
        q_scale_next = inside ? p.q_scale[row] : 0.f;
        const uint8_t* src8 = p.q8 + ((int64_t)half * TH + row) * kRow;
        uint32_t w[112];
#pragma unroll
        for (int i = 0; i < 14; ++i) {
          uint32_t* d = &w[8 * i];
          if (inside) {
            asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]),
                           "=r"(d[7])
                         : "l"(src8 + 32 * i));
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) d[k] = 0u;
          }
        }
#pragma unroll
        for (int c = 0; c < 3; ++c)
          ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColQ8 + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(&w[32 * c]));
        ptx::tmem_st_32x32b_x16u(tbase + lane_addr + kColQ8 + 96u, *reinterpret_cast<uint32_t(*)[16]>(&w[96]));
      } else {
      const __nv_bfloat16* src = p.q_lat + row * kR;
#pragma unroll 1
      for (int ch = 0; ch < kQTmemChunks; ch += 2) {
        uint32_t w[2][32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t* d = &w[h][8 * i];
            if (inside && ch + h < kQTmemChunks) {
              asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                           : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3]), "=r"(d[4]), "=r"(d[5]), "=r"(d[6]),
                             "=r"(d[7])
                           : "l"(src + 64 * (ch + h) + 16 * i));
            } else {
#pragma unroll
              for (int k = 0; k < 8; ++k) d[k] = 0u;
            }
          }
        }
        ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColQ + 32u * ch, w[0]);
        if (ch + 1 < kQTmemChunks) ptx::tmem_st_32x32b_x32(tbase + lane_addr + kColQ + 32u * (ch + 1), w[1]);
      }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (even) ptx::mbar_arrive(bar(B_Q_FULL));
        else ptx::mbar_arrive_cluster(lead(bar(B_Q_FULL)));
      }
      if (sw == 0 && lane == 0) DUO_TRACE(9, n);
      return true;
    };

    struct Pending {
      bool on;
      int32_t item, n, part0, part1;
      float l, m;
    } pend{false, 0, 0, -1, -1, 0.f, 0.f};
    // O^T[:, row] / l_row to the output, once the unit's last value MMAs are done: the row's
    // owner CTA adds its two threads' sums and publishes 1 / l to both CTAs; every thread
    // then writes its two latent rows for all of the pair's rows.
    uint32_t n_ep = 0;
    auto epilogue = [&](uint32_t g_last) -> bool {
      if (!wait_all(bar(B_O_DONE + (g_last & 1)), (g_last >> 1) & 1)) return false;
      ptx::tc_fence_after();
      if (sw == 0 && lane == 0) DUO_TRACE(10, n_ep);
      xl[L] = pend.l;
      if (!pair_sync()) return false;
      if (half == 0) {
        const float l = pend.l + xl[L ^ 64];   // half 0 + half 1
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        xinv[prow] = inv_l;
        const uint32_t xa = sbase + L::kOffXinv + 4u * prow;
        ptx::st_async_u32(peer(xa), __float_as_uint(inv_l), peer(bar(B_LX_FULL)));
        if (tok < pend.n) {
          const int64_t row = qrow_of(pend.item, prow);
          const int32_t prt = tok ? pend.part1 : pend.part0;
          const float z = l > 0.f ? (pend.m + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
          if (prt < 0) { if (p.lse) p.lse[row] = z; }
          else p.lse_part[(int64_t)prt * H + row % H] = z;
        }
        __syncwarp();
        if (lane == 0) {
          if (sw == 0) ptx::mbar_arrive_expect_tx(bar(B_LX_FULL), 4u * kCtaRows);   // the peer's words
          else ptx::mbar_arrive(bar(B_LX_FULL));
        }
      }
      const bool got = ptx::mbar_wait_cluster_bounded(bar(B_LX_FULL), n_lx & 1, abort_flag, p.timeout_ns);
      ++n_lx;
      if (!__all_sync(0xffffffffu, got)) return false;
      if (sw == 0 && lane == 0) DUO_TRACE(14, n_ep);
      // Each warp writes its own 32 latent columns (latent rows of its TMEM lane quarter)
      // of each 32-row chunk of O^T: scale by 1 / l, stage two 16-row fp32 blocks row-major
      // in the warp's two tiles in the idle P buffers, and hand each to a TMA store (final
      // rows to o_lat, partial rows to the workspace). The stores run in the background; a
      // tile is restaged once the store two blocks back has read it.
      const uint32_t tiles = sbase + L::kOffP + (uint32_t)sw * kPBytes;   // 2 x 4 KiB
      uint32_t nst = 0;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        const int lh = c >> 2, n0 = 32 * (c & 3);
        const int tn = H == kRows ? 0 : n0 / kCtaRows;   // the 32 rows' query token
        if (tn >= pend.n) continue;                       // (the same for every thread)
        const int32_t prt = tn ? pend.part1 : pend.part0;
        uint32_t o[32];
        ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColO + 32u * c, o);
        float inv[32];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(inv[4 * k]), "=f"(inv[4 * k + 1]), "=f"(inv[4 * k + 2]), "=f"(inv[4 * k + 3])
                       : "r"(sbase + L::kOffXinv + 4u * (n0 + 4 * k)));
        ptx::tmem_wait_ld();
        const int x = 256 * lh + 128 * (int)rank + 32 * q;   // this warp's latent columns
        const int64_t row0 = qrow_of(pend.item, n0);
        const CUtensorMap* map = prt < 0 ? &tm_o : &tm_op;
        const int64_t y0 = prt < 0 ? row0 : (int64_t)prt * H + row0 % H;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          if (nst >= 2 && lane == 0) ptx::bulk_wait_group_read<1>();   // the tile's previous store read it
          __syncwarp();
          const uint32_t tile = tiles + (nst & 1) * (uint32_t)kPBytes / 2;
#pragma unroll
          for (int j = 0; j < 16; ++j)
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(tile + (uint32_t)(j * 128 + 4 * lane)),
                         "f"(__uint_as_float(o[16 * hr + j]) * inv[16 * hr + j])
                         : "memory");
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(map, tile, x, (int32_t)(y0 + 16 * hr));
            ptx::bulk_commit_group();
          }
          ++nst;
        }
      }
      // O^T is read: the next unit's value MMAs may overwrite it
      ptx::tc_fence_before();
      __syncwarp();
      if (sw == 0 && lane == 0) DUO_TRACE(11, n_ep);
      ++n_ep;
      if (lane == 0) arrive_read(B_O_FREE);
      pend.on = false;
      // every warp's tiles are read before P is written into those buffers again
      if (lane == 0) ptx::bulk_wait_group_read<0>();
      if (!all4_sync()) return false;
      return true;
    };

    Cursor cur = first_page(p, plan, u_begin, u_end);
    if (cur.valid && !stage_q(cur.u, 0)) { fail(); ok = false; }
    uint32_t g = 0;
    float m_ref = -CUDART_INF_F, l_part = 0.f;
    float sl2 = p.scale_log2;   // the row's logit scale (log2 units)
    while (cur.valid && ok) {
      const Unit2& u = cur.u;
      if (cur.k == 0) {
        if (pend.on && !epilogue(g - 1)) { fail(); ok = false; break; }
        m_ref = -CUDART_INF_F;
        l_part = 0.f;
        if (F8) sl2 = p.scale_log2 * q_scale_next;
      }
      const int32_t ntok = tok < u.n ? max(u.ntok[tok], 0) : 0;
      // ------------------------------------------------ this thread's 32 scores
      if (!wait_all(bar(B_S_FULL), g & 1)) { fail(); ok = false; break; }
      ptx::tc_fence_after();
      if (sw == 0 && lane == 0) DUO_TRACE(6, g);
      float v[32];
      if constexpr (F8) {
        // lane L holds piece L / 64 of row m for all 64 tokens: keep tokens 32 half.. and
        // hand the other 32 to the partner lane L ^ 64 (the other piece of the same row)
        // through shared memory (16-byte chunks swizzled by the row), then add its half
        {
          uint32_t r[32];
          ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColS + 32u * (uint32_t)(half ^ 1), r);
          ptx::tmem_wait_ld();
          const uint32_t xr = sbase + L::kOffXch + 128u * (uint32_t)L;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(xr + (uint32_t)((k ^ (L & 7)) << 4)),
                         "r"(r[4 * k]), "r"(r[4 * k + 1]), "r"(r[4 * k + 2]), "r"(r[4 * k + 3])
                         : "memory");
        }
        {
          uint32_t r[32];
          ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColS + 32u * (uint32_t)half, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
        }
      } else {
        uint32_t r[32];
        ptx::tmem_ld_32x32b_x32(tbase + lane_addr + kColS, r);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r[t]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_read(B_S_EMPTY);
      if constexpr (F8) {
        if (!pair_sync()) { fail(); ok = false; break; }
        const uint32_t xr = sbase + L::kOffXch + 128u * (uint32_t)(L ^ 64);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float x0, x1, x2, x3;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(x0), "=f"(x1), "=f"(x2), "=f"(x3)
                       : "r"(xr + (uint32_t)((k ^ (L & 7)) << 4)));
          v[4 * k] += x0;
          v[4 * k + 1] += x1;
          v[4 * k + 2] += x2;
          v[4 * k + 3] += x3;
        }
      }
      // the unit's last score MMA is done: stage the next unit's query
      if (cur.k == u.npg - 1) {
        int32_t ui = cur.ui;
        Unit2 nu;
        if (next_unit(p, plan, ui, u_end, nu) && !stage_q(nu, cur.n + 1)) { fail(); ok = false; break; }
      }
      if constexpr (F8) {
        // score column t times the token's scale (the MMA summed the raw codes)
        if (!wait_all(bar(B_CV_FULL + (g & 3)), (g >> 2) & 1)) { fail(); ok = false; break; }
        const uint32_t xs = sbase + L::kOffXsc + 256u * (g & 3) + 128u * (uint32_t)half;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float w0, w1, w2, w3;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(w0), "=f"(w1), "=f"(w2), "=f"(w3)
                       : "r"(xs + 16u * k));
          v[4 * k] *= w0;
          v[4 * k + 1] *= w1;
          v[4 * k + 2] *= w2;
          v[4 * k + 3] *= w3;
        }
      }
      const int32_t tok0 = (u.pb + cur.k) * kPage + 32 * half;
      if (tok0 + 32 > ntok) {
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = (tok0 + t < ntok) ? v[t] : -CUDART_INF_F;
      }
      float mx;
      {
        float a[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          a[i] = fmaxf(fmaxf(fmaxf(v[8 * i], v[8 * i + 1]), fmaxf(v[8 * i + 2], v[8 * i + 3])),
                       fmaxf(fmaxf(v[8 * i + 4], v[8 * i + 5]), fmaxf(v[8 * i + 6], v[8 * i + 7])));
        mx = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
      }
      // ------------------------------------------------ the row's maximum over both lane halves
      xmax[128 * (g & 1) + L] = mx;
      if (!pair_sync()) { fail(); ok = false; break; }
      const float mrow = fmaxf(mx, xmax[128 * (g & 1) + (L ^ 64)]) * sl2;
      const bool need = mrow > m_ref + kRescaleThreshold;
      const float mu = need ? mrow : m_ref;
      const float al = need ? ptx::ex2(m_ref - mu) : 1.f;
      const float nz = (mu == -CUDART_INF_F) ? 0.f : -mu;
      // ------------------------------------------------ the rows' rescale factors to both CTAs
      // (each CTA's O^T holds every row of the pair); one thread per row sends its factor
      const uint32_t ab = g & 1;
      if (half == 0) {
        const uint32_t xa = sbase + L::kOffXal + 4u * (128 * ab + prow);
        xal[128 * ab + prow] = al;
        ptx::st_async_u32(peer(xa), __float_as_uint(al), peer(bar(B_AL_FULL + ab)));
        const uint32_t moved = __any_sync(0xffffffffu, need && cur.k > 0) ? 1u : 0u;
        if (lane == 0) {
          const uint32_t fi = 4 * ab + 2 * rank + (q & 1);
          xflg[fi] = moved;
          ptx::st_async_u32(peer(sbase + L::kOffXflg + 4u * fi), moved, peer(bar(B_AL_FULL + ab)));
        }
        __syncwarp();
        if (lane == 0) {
          if (sw == 0) ptx::mbar_arrive_expect_tx(bar(B_AL_FULL + ab), kAlBytes);   // the peer's words
          else ptx::mbar_arrive(bar(B_AL_FULL + ab));
        }
      }
      // ------------------------------------------------ p = 2^(x - m), its bf16 rounding and remainder
      uint32_t ph[16], pl[16];
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a0 = ptx::ex2(fmaf(v[2 * i], sl2, nz));
        const float a1 = ptx::ex2(fmaf(v[2 * i + 1], sl2, nz));
        sum4[i & 3] += a0 + a1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
        ph[i] = *reinterpret_cast<uint32_t*>(&h2);
        const float r0 = a0 - __uint_as_float(ph[i] << 16), r1 = a1 - __uint_as_float(ph[i] & 0xFFFF0000u);
        __nv_bfloat162 l2 = __floats2bfloat162_rn(r0, r1);
        pl[i] = *reinterpret_cast<uint32_t*>(&l2);
      }
      l_part = l_part * al + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      m_ref = mu;
      const float pmax = ptx::ex2(fmaf(mx, sl2, nz));
      const bool want_lo = pmax * kLoShare > l_part;
      // ------------------------------------------------ P to shared memory once the previous value MMAs are done
      // P buffer g % 2 was last read by the value MMAs of page g - 2
      if (g >= 2 && cur.k != 0 && !wait_all(bar(B_O_DONE + (g & 1)), ((g >> 1) & 1) ^ 1)) { fail(); ok = false; break; }
      if (!wait_all(bar(B_AL_FULL + ab), (g >> 1) & 1)) { fail(); ok = false; break; }
      ptx::tc_fence_after();
      if (xflg[4 * ab] | xflg[4 * ab + 1] | xflg[4 * ab + 2] | xflg[4 * ab + 3]) {
        // O^T is stable once page g - 1's value MMAs are done
        if (!wait_all(bar(B_O_DONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1)) { fail(); ok = false; break; }
        ptx::tc_fence_after();
        // a moved reference: O^T[:, row] *= 2^(m_old - m_new) for every row of the pair (1 for
        // rows that kept theirs); this thread scales its two latent rows
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          const uint32_t ta = tbase + lane_addr + kColO + 32u * c;
          ptx::tmem_ld_32x32b_x32(ta, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            o[j] = __float_as_uint(__uint_as_float(o[j]) * xal[128 * ab + 32 * (c & 3) + j]);
          ptx::tmem_st_32x32b_x32(ta, o);
        }
        ptx::tmem_wait_st();
      }
      {
        // row m, tokens 32h..32h+31 = 16-byte chunks 4h..4h+3 of the 128-byte row (128-byte swizzle)
        const uint32_t prow_s = sbase + L::kOffP + 2u * kPBytes * (g & 1) + (uint32_t)m * 128u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t off = (uint32_t)(((4 * half + i) ^ (m & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow_s + off), "r"(ph[4 * i]),
                       "r"(ph[4 * i + 1]), "r"(ph[4 * i + 2]), "r"(ph[4 * i + 3])
                       : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow_s + kPBytes + off), "r"(pl[4 * i]),
                       "r"(pl[4 * i + 1]), "r"(pl[4 * i + 2]), "r"(pl[4 * i + 3])
                       : "memory");
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      const uint32_t any_lo = __any_sync(0xffffffffu, want_lo) ? 1u : 0u;
      __syncwarp();   // every lane's P stores before lane 0's release
      if (sw == 0 && lane == 0) DUO_TRACE(7, g);
      if (lane == 0) {
        const uint32_t fa = sbase + L::kOffFlag + 4u * (8 * (g & 3) + 4 * rank + sw);
        if (even) {
          lo_flag[8 * (g & 3) + sw] = any_lo;
          if (sw == 0) ptx::mbar_arrive_expect_tx(bar(B_P_FULL), 4u * kSoftWarps);   // the odd CTA's words
          else ptx::mbar_arrive(bar(B_P_FULL));
        } else {
          ptx::st_async_u32(lead(fa), any_lo, lead(bar(B_P_FULL)));
          ptx::mbar_arrive_remote(lead(bar(B_P_FULL)));
        }
      }
      if (cur.k == u.npg - 1) {
        pend.on = true;
        pend.item = u.item;
        pend.n = u.n;
        pend.part0 = u.part[0];
        pend.part1 = u.part[1];
        pend.l = l_part;
        pend.m = m_ref;
      }
      advance(p, plan, u_end, cur);
      ++g;
    }
    if (ok && pend.on && !epilogue(g - 1)) fail();
    if (lane == 0) ptx::bulk_wait_group<0>();   // this warp's output stores are complete
  }

  ptx::tc_fence_before();
  __syncthreads();
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && p.trace) p.trace[(size_t)blockIdx.x * 1024 + 1022] = (unsigned long long)clock64();
#endif
  ptx::cluster_sync();   // the even CTA's MMAs, commits and loads for both CTAs are done
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tbase, kTmemCols);
  }
  ptx::cluster_sync();
}

}  // namespace duo
}  // namespace mla
