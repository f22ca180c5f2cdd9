/*
 * mla.h -- C ABI of the B200 (sm_100a) MLA decode library (libmla.so).
 *
 * Multi-head Latent Attention decode over a paged cache whose rows hold only a
 * latent c_t (kv_lora_rank R, 512) and one decoupled-RoPE key k_t (Dr, 64) shared
 * by every head: 576 elements, 1,152 bytes in bf16, per token per layer
 * (modeldna.ai "learn/mla", section "Under the hood" and its cache-size table).
 * Each head's content query is absorbed through W_UK into latent space, scored
 * against c_t, its rope query against k_t; the softmax scale is 1/sqrt(Dn + Dr)
 * (kimi-k3 docs "GatedMLA", section "Observe logits, then compute causal
 * attention"); the probabilities weight c_t itself and the R-wide result is
 * up-projected per head through W_UV, so per-head K/V are never materialised.
 *
 * One decode step on one CUDA stream:
 *   mla_cache_append   write the newest q_len rows of every sequence into its pages
 *   mla_absorb_q       q_lat = q_nope @ W_UK[h]                       (per head)
 *   mla_plan_splits    host: cut the work into balanced (sequence, page range) units
 *   mla_decode_attn    scores, online softmax and latent value sum per unit
 *   mla_combine        log-sum-exp merge of units that share a query
 *   mla_out_proj       out = W_UV[h] @ o_lat                          (per head)
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers unless the name ends in _host; all
 *    tensors are row-major and contiguous with the shapes given; the caller owns
 *    every buffer. The library never allocates device memory and never
 *    synchronises the stream (except mla_check_status, which says so).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous on it.
 *  - Arguments are validated before any launch. On error the call returns a
 *    negative mla_status, launches nothing, and mla_last_error() describes why.
 *  - dtype MLA_BF16: q_nope, q_rope, W_UK, W_UV, kv_cache, new_ckr, q_lat and out are
 *    bf16 (RN-even conversions); accumulation is fp32. MLA_F32: all fp32. The latent
 *    output o_lat, partial outputs and log-sum-exp values are fp32 for both dtypes
 *    (o_lat enters the output projection in full: with only a few visible tokens a
 *    bf16 o_lat alone would move `out` by more than a bf16 rounding).
 *  - A cache row is [c (R) ; k_rope (Dr)]; k_rope is stored already rotated.
 *    seq_lens[b] counts cached tokens of sequence b INCLUDING its q_len new ones.
 *    Query i (0 <= i < q_len) of sequence b sits at position seq_lens[b]-q_len+i
 *    and sees tokens t <= that position (causal within the chunk). A query that
 *    sees no token yields o_lat = 0, out = 0 and lse = -inf.
 *  - Token t of sequence b is row t % page_size of page block_table[b*max_pages +
 *    t / page_size] of kv_cache[num_pages][page_size][R+Dr].
 *  - Kernels bound every wait; a wait that runs out sets a device status word
 *    that mla_check_status() reports as MLA_ERR_TIMEOUT. A page id outside
 *    [0, num_pages) is skipped and reported as MLA_ERR_INVALID the same way.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 6

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID = -1,      /* bad argument (null pointer, size, layout, plan) */
  MLA_ERR_UNSUPPORTED = -2,  /* dims or policy the library has no kernel for */
  MLA_ERR_WORKSPACE = -3,    /* workspace / plan buffer too small */
  MLA_ERR_CUDA = -4,         /* a CUDA runtime or driver call failed */
  MLA_ERR_TIMEOUT = -5       /* a kernel wait ran out (reported by mla_check_status) */
} mla_status;

typedef enum { MLA_BF16 = 0, MLA_F32 = 1 } mla_dtype;

/* Geometry of one MLA layer. Validated like a KV-state ledger config (every
 * field a positive integer; datawhalechina "ARCH-MLA", section "Step 4"). */
typedef struct {
  int32_t H;          /* query heads */
  int32_t Dn;         /* per-head content query width (W_UK rows) */
  int32_t Dr;         /* shared rope key width */
  int32_t Dv;         /* per-head value width (W_UV rows) */
  int32_t R;          /* latent width, kv_lora_rank */
  int32_t page_size;  /* tokens per cache page */
  int32_t dtype;      /* mla_dtype */
} mla_dims;

/* Kernel selection for mla_decode_attn / mla_absorb_q / mla_out_proj.
 * AUTO: tensor-core (tcgen05) kernels where the dims allow (bf16, R=512, Dr=64,
 * page_size=64, H a multiple of 64, Dn=Dv=128), else the SIMT CUDA kernels.
 * SIMT: always the SIMT CUDA kernels. TCGEN05: tensor-core kernels or
 * MLA_ERR_UNSUPPORTED. There is no CPU path. */
typedef enum { MLA_POLICY_AUTO = 0, MLA_POLICY_SIMT = 1, MLA_POLICY_TCGEN05 = 2 } mla_policy;

/* Summary of a split plan (filled by mla_plan_splits). */
typedef struct {
  int32_t num_items;    /* B * q_len query tokens */
  int32_t num_units;    /* (query token, page range) work units */
  int32_t num_slots;    /* page-balanced groups of units; one CTA per slot and head group */
  int32_t num_parts;    /* units whose result is partial and needs mla_combine */
  int32_t head_groups;  /* heads are processed in groups of H / head_groups */
  int32_t plan_words;   /* int32 words of the plan buffer in use */
  int32_t max_pages;    /* block_table row length the plan's page ranges were cut for;
                           mla_decode_attn(_noalloc) rejects a call with another one */
} mla_plan_info;

int32_t mla_abi_version(void);

/* Thread-local description of the last error of this thread ("" if none). */
const char* mla_last_error(void);

/* Select the kernel policy for later calls (process-wide). */
mla_status mla_set_policy(int32_t policy);

/* Bound, in nanoseconds, on every wait inside a kernel (default 2e9). */
mla_status mla_set_wait_timeout_ns(uint64_t ns);

/* The split planner's estimate of what merging split queries (mla_combine) costs, in
 * pages of decode work (process-wide; applies to plans for the SM-pair kernel, H=64 and
 * H=128 on the tensor-core path). Negative (the default): mla_plan_splits cuts queries
 * wherever a slot fills up, balancing the slots as finely as one page. Zero or more: the
 * planner also lays every query out whole (no partial results, no merge) and takes that
 * layout when its heaviest slot is at most the cut layout's plus `pages`: e.g. 64
 * queries of 64 pages on 74 slots then run one query per slot (64 of the 74 busy)
 * instead of every query cut in two. The split of work between queries and the token
 * ranges they see are unchanged; only where the ranges are cut. MLA_ERR_INVALID for NaN.
 * The split-KV merge it trades against is the log-sum-exp merge of mla_combine. */
mla_status mla_set_plan_combine_cost(double pages);

/* TEST-ONLY hook for the failure path of the tensor-core decode kernels: while set
 * (ordinal >= 0), the first CTA of each mla_decode_attn launch skips the shared-memory
 * load of its page with that ordinal (0 = its first page), so the waits on that page
 * run out after the wait bound (mla_set_wait_timeout_ns), the kernel stops, and
 * mla_check_status then reports MLA_ERR_TIMEOUT; the outputs of that launch are
 * undefined. A negative ordinal switches the hook off (the default). Process-wide;
 * always returns MLA_OK. Nothing in the pages corresponds to it. Production code
 * never sets it: while it is set, mla_check_status returns MLA_ERR_INVALID even
 * when no kernel reported a problem, so a hook left on cannot go unnoticed. */
mla_status mla_debug_drop_page_load(int32_t ordinal);

/* Synchronises `stream`, then reads and clears the device status word of the
 * current device: MLA_OK, MLA_ERR_TIMEOUT (a bounded wait ran out) or
 * MLA_ERR_INVALID (a page id outside the pool was skipped, or the test-only
 * mla_debug_drop_page_load hook is still set; mla_last_error says which). */
mla_status mla_check_status(void* stream);

/* ---------------------------------------------------------------- a2: cache append
 * Writes new_ckr[b*q_len + i] to position seq_lens[b] - q_len + i of sequence b
 * ("MLA + KV cache (Tier 3 #5)" ticket, "Description" item 1: project only the
 * new token and keep earlier ones cached). Positions < 0 are skipped.
 *   kv_cache    [num_pages][page_size][R+Dr]   dtype, written
 *   block_table [B][max_pages] int32, seq_lens [B] int32 (device)
 *   new_ckr     [B*q_len][R+Dr]                dtype                              */
mla_status mla_cache_append(void* kv_cache, const int32_t* block_table, const int32_t* seq_lens,
                            const void* new_ckr, int32_t B, int32_t q_len, int32_t max_pages,
                            int32_t num_pages, mla_dims d, void* stream);

/* ---------------------------------------------------------------- cache-write prologue
 * The rows a step appends, computed from the new tokens' hidden states, then appended
 * as mla_cache_append does. For every new token t (token i of sequence
 * b, position pos = seq_lens[b] - q_len + i):
 *   f = W_DKV h_t                       (kimi-k3 docs "GatedMLA", "Projection geometry and
 *                                        stored weights": one down projection M -> R_kv + D_s
 *                                        to the compressed KV feature and the shared key)
 *   c = f[:R] / sqrt(mean(f[:R]^2) + eps) * kv_gain       (kv_rmsnorm on the feature)
 *   k = rope(f[R:], pos): dims i and i + Dr/2 turned by pos * rope_base^(-2i/Dr)
 *       (the shared key carries the position: modeldna "learn/mla", "Under the hood";
 *       the frequencies and the pairing are the usual reading, the pages fix neither)
 * and [c ; k] (bf16) is written to the token's row of its page. If q_rope is not NULL
 * its rows [B*q_len][H][Dr] (bf16) are turned in place by the same rule at the query
 * token's position. fp32 accumulation and normalisation; angles in double precision.
 *   hidden [B*q_len][M] bf16, W_DKV [R+Dr][M] bf16 (out x in), kv_gain [R] bf16; M a
 *   multiple of 64; dims bf16, R=512, Dr=64, page_size=64 (else MLA_ERR_UNSUPPORTED, as
 *   under the SIMT policy: the prologue has only a tensor-core kernel). Tokens with pos <
 *   0 are skipped; a page id outside the pool is skipped and reported by mla_check_status.
 *   workspace: >= mla_cache_write_workspace_size(B*q_len, M) bytes, 16-byte aligned: the
 *   down projection is split over K (fp32 partial sums there, added by the last kernel). */
size_t mla_cache_write_workspace_size(int32_t T, int32_t M);
mla_status mla_cache_write(const void* hidden, const void* W_DKV, const void* kv_gain, int32_t M,
                           void* kv_cache, const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                           int32_t q_len, int32_t max_pages, int32_t num_pages, void* q_rope, float eps,
                           float rope_base, void* workspace, size_t workspace_bytes, mla_dims d, void* stream);

/* ---------------------------------------------------------------- a1: absorb the query
 * q_lat[t][h][:] = q_nope[t][h][:] @ W_UK[h]  (modeldna "learn/mla", "Under the
 * hood": the key up-projection folds into the query; W_UK[h] is head h's slice
 * of the GatedMLA KV up-projection, "Projection geometry and stored weights").
 *   q_nope [T][H][Dn], W_UK [H][Dn][R]  ->  q_lat [T][H][R]          all dtype      */
mla_status mla_absorb_q(const void* q_nope, const void* W_UK, void* q_lat, int32_t T, mla_dims d,
                        void* stream);

/* ---------------------------------------------------------------- split planning (host)
 * The pages fix what a decode step computes, not how the work of a batch of
 * sequences is spread over the GPU. Splitting a query's cached tokens into ranges
 * and merging the ranges' results exactly by their log-sum-exp is the flash-decoding
 * reading of the softmax: softmax over a union of token sets equals the
 * lse-weighted mix of the softmaxes over each set (the merge identity written out
 * in mla_combine below). The plan, its workspace and the combine serve that split.
 * Upper bound, in int32 words, of the plan buffer for these sizes. */
size_t mla_plan_capacity(int32_t B, int32_t q_len, int32_t num_sms);

/* Cuts the decode work into units of whole pages and groups them into slots
 * of nearly equal page counts (num_sms / head_groups slots), so that one CTA per
 * slot and head group covers the GPU evenly; a query whose pages span several
 * units gets one partial output per unit, merged by mla_combine.
 *   seq_lens_host [B] int32 HOST; plan_host: HOST int32 buffer of `capacity`
 *   words, written; copy its first info->plan_words words to the device and pass
 *   that copy to mla_decode_attn and mla_combine. `info` (host) is written.     */
mla_status mla_plan_splits(const int32_t* seq_lens_host, int32_t B, int32_t q_len, int32_t max_pages,
                           mla_dims d, int32_t num_sms, int32_t* plan_host, size_t capacity,
                           mla_plan_info* info);

/* Bytes of workspace mla_decode_attn / mla_combine need for this plan: fp32
 * partials [num_parts][H][R] followed by fp32 lse [num_parts][H] (one partial
 * o_lat and lse per unit of a split query, the inputs of the merge identity
 * above). Returns 0 for a null info or invalid dims. */
size_t mla_workspace_size(const mla_plan_info* info, mla_dims d);

/* ---------------------------------------------------------------- a3-a5: decode attention
 * For every query token (b, i) and head h, over the visible tokens t:
 *   s_t = scale * ([q_lat ; q_rope] . [c_t ; k_t])     one (R+Dr)-long dot product
 *   p   = softmax_t(s),  o_lat = sum_t p_t c_t  (R wide),  lse = log sum_t exp(s_t)
 * (the absorbed form of the GatedMLA attention; scale = 1/sqrt(Dn+Dr) there).
 *   q_lat [B*q_len][H][R], q_rope [B*q_len][H][Dr], kv_cache as above (dtype)
 *   plan_dev: device copy of the mla_plan_splits buffer; info: its host summary
 *   o_lat [B*q_len][H][R] fp32 and lse [B*q_len][H] fp32 (lse may be NULL):
 *   written for queries whose work is one unit; others go to the workspace.
 *   workspace: >= mla_workspace_size bytes, 256-byte aligned (may be NULL when
 *   the plan has no parts).                                                       */
mla_status mla_decode_attn(const void* q_lat, const void* q_rope, const void* kv_cache,
                           const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                           int32_t q_len, int32_t max_pages, int32_t num_pages, float scale,
                           const int32_t* plan_dev, const mla_plan_info* info, void* o_lat,
                           float* lse, void* workspace, size_t workspace_bytes, mla_dims d,
                           void* stream);

/* ---------------------------------------------------------------- a6: split-KV combine
 * The exact merge of softmax results over disjoint token sets (the pages' attention,
 * GatedMLA "Observe logits, then compute causal attention", is one softmax over all
 * visible tokens; the merge restores it from the per-range results):
 * for each query whose work was split: m = max_s lse_s, w_s = exp(lse_s - m),
 * o_lat = sum_s w_s o_s / sum_s w_s, lse = m + log sum_s w_s (parts with
 * lse = -inf weigh 0). Writes o_lat (dtype) and lse (fp32, may be NULL) of those
 * queries only (both fp32). A no-op launch-free call when info->num_parts == 0.      */
mla_status mla_combine(const int32_t* plan_dev, const mla_plan_info* info, const void* workspace,
                       size_t workspace_bytes, void* o_lat, float* lse, mla_dims d, void* stream);

/* ---------------------------------------------------------------- a7: output up-projection
 * out[t][h][:] = W_UV[h] @ o_lat[t][h][:]  (the value up-projection folded into
 * the output side; GatedMLA "Output projection and optional gate" applies Wo and
 * the gate after this, outside this library).
 *   o_lat [T][H][R] fp32, W_UV [H][Dv][R] dtype  ->  out [T][H][Dv] dtype
 * (bf16 on the tensor cores: each fp32 o_lat element enters as bf16 hi + lo, two MMAs
 * per K step, so o_lat keeps ~16 significant bits; fp32 accumulation)              */
mla_status mla_out_proj(const void* o_lat, const void* W_UV, void* out, int32_t T, mla_dims d,
                        void* stream);

/* ---------------------------------------------------------------- 8-bit (E4M3) latent cache
 * The softved page "Introduction to MLA vs. KV Cache in Large Language Models" ("Practical
 * Implementation Tips for MLA in LLM Serving") advises quantising the latent cache to cut
 * its memory further; it fixes no format. This library's reading:
 *  - every element of a cached row [c ; k_rope] is one byte, an E4M3 code of the OCP 8-bit
 *    floating-point format (sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals,
 *    no infinities, 0x7F/0xFF NaN, largest finite 448): kv_codes [num_pages][64][576] uint8;
 *  - every row has one power-of-two scale 2^k shared by c and k_rope, stored as the byte
 *    k + 127: kv_scales [num_pages][64] uint8. k is the smallest integer in [-126, 7] with
 *    max_i |x_i| <= 448 * 2^k (a row beyond 448 * 2^7 keeps k = 7 and saturates);
 *  - code_i = x_i * 2^-k rounded to nearest, ties to even, saturating at +-448; the row
 *    stands for code_i * 2^k exactly. 577 bytes per token instead of 1,152.
 * Decoding attends over those exact values: mla_decode_attn_fp8 computes what
 * mla_decode_attn computes for a bf16 cache holding code * 2^k (which bf16 represents
 * exactly). Queries, o_lat, lse, plans, mla_combine and mla_out_proj are unchanged.
 * Geometry: bf16 rows, R=512, Dr=64, page_size=64 (else MLA_ERR_UNSUPPORTED).
 *
 * Quantises n dense bf16 rows [n][576] into codes [n][576] and scale bytes [n]
 * (rows 16-byte aligned, codes 8-byte aligned). Converts an existing bf16 pool. */
mla_status mla_quantize_rows_fp8(const void* rows, void* codes, void* scales, int64_t n, mla_dims d,
                                 void* stream);

/* mla_cache_append for the 8-bit cache: new_ckr[b*q_len + i] (bf16 [576], 16-byte
 * aligned) is quantised into position seq_lens[b] - q_len + i of sequence b (codes and
 * scale byte). Positions < 0 are skipped; a page id outside the pool is skipped and
 * reported by mla_check_status. */
mla_status mla_cache_append_fp8(void* kv_codes, void* kv_scales, const int32_t* block_table,
                                const int32_t* seq_lens, const void* new_ckr, int32_t B, int32_t q_len,
                                int32_t max_pages, int32_t num_pages, mla_dims d, void* stream);

/* Workspace of mla_decode_attn_fp8: the split partials exactly as mla_workspace_size lays
 * them out (so mla_combine takes the same buffer), then the query split into two E4M3
 * pieces per element ([2][T*H][576] bytes) and its per-row scales ([T*H] fp32). */
size_t mla_workspace_size_fp8(const mla_plan_info* info, mla_dims d);

/* a3-a5 over the 8-bit cache, for a plan made by mla_plan_splits with the same dims, q_len
 * and max_pages. Arguments as for mla_decode_attn, plus kv_scales (16-byte aligned); the workspace is
 * required (>= mla_workspace_size_fp8, 256-byte aligned). Two launches: the query split
 * (q_lat, q_rope -> workspace), then the SM-pair decode kernel, which scores against the
 * codes on the 8-bit tensor cores, applies each token's scale to its score column, and
 * widens the codes times the scale to bf16 for the value sum. H must be 64 or 128. */
mla_status mla_decode_attn_fp8(const void* q_lat, const void* q_rope, const void* kv_codes, const void* kv_scales,
                               const int32_t* block_table, const int32_t* seq_lens, int32_t B, int32_t q_len,
                               int32_t max_pages, int32_t num_pages, float scale, const int32_t* plan_dev,
                               const mla_plan_info* info, void* o_lat, float* lse, void* workspace,
                               size_t workspace_bytes, mla_dims d, void* stream);

/* ---------------------------------------------------------------- f4: non-absorbed prefill
 * The GatedMLA forward over whole sequences (kimi-k3 docs "GatedMLA": "Build per-head Q,
 * K and V" and "Observe logits, then compute causal attention"): every position of a
 * sequence is a query. For head h, K_h = [C W_UK[h]^T ; k_rope] (the shared rope key
 * broadcast to every head), V_h = C W_UV[h]^T, and
 *   out[t][h] = sum_{t' <= t} softmax_t'(scale * [q_nope ; q_rope][t][h] . K_h[t']) V_h[t'],
 * scale = 1/sqrt(Dn + Dr) as for the decode. The non-absorbed form is the cheaper one when
 * every position is a query: 2 (Dn + Dr + Dv) FLOP per head and (query, key) pair against
 * the absorbed form's 2 (R + Dr + R). The output gate and Wo that follow in GatedMLA are
 * plain projections outside this library.
 *   ckr        [N][R+Dr] bf16: the packed sequences' rows [c ; k_rope] (k_rope rotated)
 *   q_nope     [N][H][Dn], q_rope [N][H][Dr] bf16 (q_rope rotated)
 *   W_UK [H][Dn][R], W_UV [H][Dv][R] bf16
 *   cu_seqlens [B+1] int32 on the DEVICE and cu_seqlens_host the same on the HOST:
 *              sequence b is rows cu_seqlens[b] .. cu_seqlens[b+1]-1, cu_seqlens[0] = 0
 *   out        [N][H][Dv] bf16
 *   workspace  >= mla_prefill_workspace_size(N, d) bytes, 256-byte aligned: the per-head
 *              K_c and V in bf16 ([N][H][128] each), written by the first two launches
 * Three launches: two tensor-core GEMMs (the up-projections of every token for all heads),
 * then causal attention (tensor cores; 128 queries x one head per CTA). Dims: bf16, R=512,
 * Dr=64, Dn=Dv=128, even H (else MLA_ERR_UNSUPPORTED; no SIMT kernel). Precision: K_c, V
 * and P enter the MMAs in bf16 (P with its bf16 remainder where one key can dominate a
 * row), fp32 accumulation and softmax.                                                */
size_t mla_prefill_workspace_size(int32_t N, mla_dims d);
mla_status mla_prefill_attn(const void* ckr, const void* q_nope, const void* q_rope, const void* W_UK,
                            const void* W_UV, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int32_t B,
                            float scale, void* out, void* workspace, size_t workspace_bytes, mla_dims d,
                            void* stream);

/* ---------------------------------------------------------------- allocation-free decode
 * The pages describe no counterpart of this call; it exists for callers that cannot
 * allocate device memory: code inside another framework's fixed memory pool, or a
 * host environment with no allocator exposed.
 * It computes exactly what mla_decode_attn followed by mla_combine computes, final
 * o_lat and lse for every query, but keeps the partial outputs of split queries in
 * a scratch array that the library owns: a file-scope device array of 48 MiB
 * (50,331,648 bytes) that every GPU which loads libmla.so holds until the process
 * exits. The caller still allocates and passes all inputs, the plan and the
 * outputs. It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - A plan whose partials need more than 48 MiB (mla_workspace_size) is rejected
 *    with MLA_ERR_WORKSPACE before any launch: fewer num_sms or fewer splits, or
 *    mla_decode_attn with a caller workspace, serve those.
 *  - The first call in each CUDA context looks up the array's device address
 *    (cudaGetSymbolAddress) in that context. The address is kept per context (its
 *    driver context id), so a context that is destroyed and created again (for
 *    instance after cudaDeviceReset) gets a fresh lookup, never a stale address.
 *  - Every call on a device shares the one array, which keeps the last call's
 *    contents. Nothing in it has to start at zero: each partial is written before it
 *    is read in the same call. Calls that overlap on the GPU (concurrent streams)
 *    race on it; order them on one stream or with events.
 * Arguments as for mla_decode_attn, without the workspace. */
mla_status mla_decode_attn_noalloc(const void* q_lat, const void* q_rope, const void* kv_cache,
                                   const int32_t* block_table, const int32_t* seq_lens, int32_t B,
                                   int32_t q_len, int32_t max_pages, int32_t num_pages, float scale,
                                   const int32_t* plan_dev, const mla_plan_info* info, void* o_lat,
                                   float* lse, mla_dims d, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
