"""fp64 reference for MLA decode over a paged latent + shared-RoPE-key cache.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py): the library never imports this.

Notation (follows the GatedMLA docs' geometry, "Projection geometry and stored
weights", and the modeldna primer, "Under the hood"):
  R   kv_lora_rank, width of the cached latent c_t
  Dr  width of the shared decoupled-RoPE key k_t (one per token, not per head)
  Dn  per-head content ("nope") query/key width,  Dv  per-head value width
  W_UK[h] [Dn, R]  and  W_UV[h] [Dv, R]  are head h's slices of the KV up-projection
  R_kv -> H(D + D_v); a cache row is [c_t (R) ; k_t (Dr)], k_t already rotated.

Reference semantics (the non-absorbed definition):
  K_h,t = [W_UK[h] c_t ; k_t]     the shared key is broadcast to every head
  V_h,t =  W_UV[h] c_t
  s_h,t = scale * ([qn_h ; qr_h] . K_h,t),   scale = 1/sqrt(Dn + Dr)
  p     = softmax over the visible t,  o_h = sum_t p_h,t V_h,t
Visibility: query i of a q_len-token chunk of a sequence with L cached tokens
(the chunk included) is at absolute position L - q_len + i and sees t <= that.

All inputs are the storage values (bf16 bit patterns or float32) upcast exactly
to float64; all arithmetic is float64.
"""
from __future__ import annotations

import numpy as np


# ----------------------------------------------------------------------------- helpers

def to_f64(x: np.ndarray) -> np.ndarray:
    """Exact upcast of stored values: uint16 = bf16 bit patterns, else a float array."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def visible_len(L: int, q_len: int, i: int) -> int:
    """Tokens seen by query i of the newest q_len-token chunk (causal within the chunk)."""
    return max(0, int(L) - int(q_len) + int(i) + 1)


def gather_rows(kv_cache: np.ndarray, bt_row: np.ndarray, L: int, page_size: int) -> np.ndarray:
    """The first L cache rows of one sequence, in order, read through its page list.

    Position t lives in page bt_row[t // page_size], row t % page_size (paged KV
    pool as in the "MLA + KV cache" ticket, "Description")."""
    rows = [kv_cache[int(bt_row[t // page_size]), t % page_size] for t in range(int(L))]
    if not rows:
        return np.zeros((0, kv_cache.shape[-1]), dtype=np.float64)
    return to_f64(np.stack(rows))


# ----------------------------------------------------------------------------- reference semantics

def reconstruct_kv(C: np.ndarray, kr: np.ndarray, wuk_h: np.ndarray, wuv_h: np.ndarray):
    """Head h's keys and values from the cache (GatedMLA, "Build per-head Q, K and V").

    C [L, R], kr [L, Dr], wuk_h [Dn, R], wuv_h [Dv, R]
    -> K [L, Dn + Dr] = [C W_UK^T | kr]   (the same kr rows for every head)
       V [L, Dv]      =  C W_UV^T
    """
    K = np.concatenate([C @ wuk_h.T, kr], axis=1)
    V = C @ wuv_h.T
    return K, V


def softmax_attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """One query row against visible keys (GatedMLA, "Observe logits, then compute
    causal attention": softmax of scaled dot products, weights applied to V).

    Returns (o, p, lse); an empty key set gives o = 0 and lse = -inf."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1]), np.zeros(0), -np.inf
    s = scale * (K @ q)
    m = np.max(s)
    e = np.exp(s - m)
    l = np.sum(e)
    p = e / l
    return p @ V, p, m + np.log(l)


def decode_nonabsorbed(q_nope, q_rope, kv_cache, block_table, seq_lens, W_UK, W_UV, scale,
                       q_len=1, page_size=64, R=None, seqs=None, heads=None):
    """Reference decode: rebuild K, V per head, then plain softmax attention.

    q_nope [B*q_len, H, Dn], q_rope [B*q_len, H, Dr], kv_cache [P, page, R+Dr],
    block_table [B, max_pages], seq_lens [B], W_UK [H, Dn, R], W_UV [H, Dv, R].
    seqs / heads restrict the work to a sample (others stay NaN).

    Returns dict(out [T,H,Dv], o_lat [T,H,R], lse [T,H]) in float64, where o_lat =
    sum_t p_t c_t uses the same probabilities (a diagnostic of the latent output).
    """
    qn, qr = to_f64(q_nope), to_f64(q_rope)
    wuk, wuv = to_f64(W_UK), to_f64(W_UV)
    T, H, _ = qn.shape
    Dv = wuv.shape[1]
    R = wuk.shape[2] if R is None else R
    B = len(seq_lens)
    out = np.full((T, H, Dv), np.nan)
    o_lat = np.full((T, H, R), np.nan)
    lse = np.full((T, H), np.nan)
    seqs = range(B) if seqs is None else seqs
    heads = range(H) if heads is None else heads
    for b in seqs:
        L = int(seq_lens[b])
        rows = gather_rows(kv_cache, block_table[b], L, page_size)
        C, kr = rows[:, :R], rows[:, R:]
        for h in heads:
            K, V = reconstruct_kv(C, kr, wuk[h], wuv[h])
            for i in range(q_len):
                t = b * q_len + i
                n = visible_len(L, q_len, i)
                q = np.concatenate([qn[t, h], qr[t, h]])
                o, p, z = softmax_attend(q, K[:n], V[:n], scale)
                out[t, h] = o
                o_lat[t, h] = p @ C[:n] if n else 0.0
                lse[t, h] = z
    return dict(out=out, o_lat=o_lat, lse=lse)


def full_causal(C, kr, qn_all, qr_all, W_UK, W_UV, scale, heads=None, intermediates=None):
    """Full causal forward over one sequence, every position a query (the GatedMLA
    shape: per-head K = [K_c ; shared k], V, causal SDPA with scale over D + D_s).

    C [L,R], kr [L,Dr] (float64), qn_all [L,H,Dn], qr_all [L,H,Dr] (stored values).
    intermediates="kv_bf16" rounds the per-head content keys K_c = C W_UK^T and the
    values V = C W_UV^T to bf16, as a pipeline that stores its up-projections in bf16
    before the attention does; everything else stays float64.
    Returns out [L, H, Dv]."""
    qn, qr = to_f64(qn_all), to_f64(qr_all)
    wuk, wuv = to_f64(W_UK), to_f64(W_UV)
    L, H, _ = qn.shape
    out = np.full((L, H, wuv.shape[1]), np.nan)
    for h in (range(H) if heads is None else heads):
        K, V = reconstruct_kv(C, kr, wuk[h], wuv[h])
        if intermediates == "kv_bf16":
            K = np.concatenate([round_bf16(K[:, :wuk.shape[1]]), K[:, wuk.shape[1]:]], axis=1)
            V = round_bf16(V)
        Q = np.concatenate([qn[:, h], qr[:, h]], axis=1)
        S = scale * (Q @ K.T)
        S[np.triu_indices(L, k=1)] = -np.inf
        M = S.max(axis=1, keepdims=True)
        E = np.exp(S - M)
        out[:, h] = (E / E.sum(axis=1, keepdims=True)) @ V
    return out


# ----------------------------------------------------------------------------- absorbed form, per step
# The modeldna primer ("Under the hood") states the up-projections can be folded into
# the query and output projections so per-head K/V are never cached. Written out:
#   ql_h = W_UK[h]^T qn_h  (R-wide),  s_h,t = scale * ([ql_h ; qr_h] . [c_t ; k_t]),
#   ol_h = sum_t p_h,t c_t,  o_h = W_UV[h] ol_h.

def absorb_q(q_nope, W_UK):
    """ql[t,h,:] = qn[t,h,:] @ W_UK[h]:  [T,H,Dn] x [H,Dn,R] -> [T,H,R]."""
    return np.einsum("thn,hnr->thr", to_f64(q_nope), to_f64(W_UK))


def attend_latent(q_lat, q_rope, kv_cache, block_table, seq_lens, scale, q_len=1, page_size=64,
                  seqs=None, heads=None):
    """Attention in latent space: each head's [ql ; qr] scored against the cache row
    [c ; k] as stored; the probabilities weight c itself.

    Returns dict(o_lat [T,H,R], lse [T,H])."""
    ql, qr = to_f64(q_lat), to_f64(q_rope)
    T, H, R = ql.shape
    o_lat = np.full((T, H, R), np.nan)
    lse = np.full((T, H), np.nan)
    for b in (range(len(seq_lens)) if seqs is None else seqs):
        L = int(seq_lens[b])
        rows = gather_rows(kv_cache, block_table[b], L, page_size)
        C = rows[:, :R]
        for h in (range(H) if heads is None else heads):
            for i in range(q_len):
                t = b * q_len + i
                n = visible_len(L, q_len, i)
                q = np.concatenate([ql[t, h], qr[t, h]])
                o, _, z = softmax_attend(q, rows[:n], C[:n], scale)
                o_lat[t, h] = o
                lse[t, h] = z
    return dict(o_lat=o_lat, lse=lse)


def out_proj(o_lat, W_UV):
    """o[t,h,:] = W_UV[h] @ ol[t,h,:]:  [T,H,R] x [H,Dv,R] -> [T,H,Dv]."""
    return np.einsum("hvr,thr->thv", to_f64(W_UV), to_f64(o_lat))


def round_bf16(x):
    """Round to the nearest bf16 value (ties to even), via float32, as a kernel that
    computes in float32 and stores bf16 does. Returns float64."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def decode_absorbed(q_nope, q_rope, kv_cache, block_table, seq_lens, W_UK, W_UV, scale,
                    q_len=1, page_size=64, intermediates=None):
    """The absorbed pipeline in float64 (cross-check of the reference semantics).

    intermediates="bf16" rounds the two tensors a bf16 pipeline may store between its
    steps, the absorbed query ql and the latent output o_lat, to bf16;
    intermediates="q_lat" rounds only ql (a pipeline that keeps o_lat in fp32);
    everything else stays float64. This is the reference for an end-to-end check of
    such a pipeline on inputs where those roundings alone move the result by more
    than a per-step tolerance (queries that see only a few tokens)."""
    ident = lambda a: a  # noqa: E731
    rnd_q = round_bf16 if intermediates in ("bf16", "q_lat") else ident
    rnd_o = round_bf16 if intermediates == "bf16" else ident
    ql = rnd_q(absorb_q(q_nope, W_UK))
    a = attend_latent(ql, q_rope, kv_cache, block_table, seq_lens, scale, q_len, page_size)
    ol = np.where(np.isnan(a["o_lat"]), np.nan, rnd_o(np.nan_to_num(a["o_lat"])))
    return dict(out=out_proj(ol, W_UV), o_lat=ol, lse=a["lse"])


# ----------------------------------------------------------------------------- split-KV merge

def combine(o_parts, lse_parts):
    """Merge partial attentions over disjoint key sets.

    Part s holds o_s = sum_{t in S_s} p_t^(s) v_t (normalised within S_s) and
    lse_s = log sum_{t in S_s} exp(s_t). The attention over the union is
    sum_s w_s o_s / sum_s w_s with w_s = exp(lse_s - max lse), and its lse is
    max + log sum_s w_s. Parts with lse = -inf (no keys) get weight 0; if every
    part is empty the result is o = 0, lse = -inf.

    o_parts [S, ..., R], lse_parts [S, ...] -> (o [..., R], lse [...])."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe), 0.0)
    tot = np.sum(w, axis=0)
    num = np.sum(w[..., None] * np.nan_to_num(o_parts), axis=0)
    o = np.where(finite[..., None], num / np.where(tot > 0, tot, 1.0)[..., None], 0.0)
    lse = np.where(finite, m_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return o, lse


# ----------------------------------------------------------------------------- cache append

def cache_append(kv_cache, block_table, seq_lens, new_ckr, q_len, page_size=64):
    """Write the q_len newest rows of every sequence into its pages: row i of
    sequence b goes to position L_b - q_len + i (project only the new token and
    keep the rest cached: "MLA + KV cache" ticket, "Description", item 1).

    Returns a new cache array (the input is not modified)."""
    out = np.array(kv_cache, copy=True)
    for b, L in enumerate(seq_lens):
        for i in range(q_len):
            pos = int(L) - q_len + i
            if pos < 0:
                continue
            out[int(block_table[b][pos // page_size]), pos % page_size] = new_ckr[b * q_len + i]
    return out


# ----------------------------------------------------------------------------- cache-write prologue

def token_positions(seq_lens, q_len):
    """Absolute position of every new token, [B * q_len]: token i of sequence b (L_b
    cached tokens, its q_len new ones included) sits at L_b - q_len + i."""
    return np.array([int(L) - q_len + i for L in seq_lens for i in range(q_len)], dtype=np.int64)


def rope(x, pos, base=10000.0):
    """Rotary position embedding of the last axis (width d, even) at positions `pos`
    (broadcast over the leading axes): dims i and i + d/2 (i < d/2) form a plane turned
    by the angle pos * base^(-2i/d). The pages fix only that the shared key carries the
    position (modeldna primer, "Under the hood"); the frequencies (base 10000, exponent
    -2i/d) and this pairing are the usual reading, stated as such in the design notes."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    theta = base ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rms_norm(x, gain, eps):
    """RMSNorm of the last axis: x / sqrt(mean(x^2) + eps) * gain (the GatedMLA docs'
    kv_rmsnorm on the compressed KV feature, "Projection geometry and stored weights")."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * to_f64(gain)


def cache_write_rows(hidden, W_DKV, kv_gain, positions, R, eps=1e-6, rope_base=10000.0):
    """The rows a decode step appends to the cache, [T, R + Dr], float64.

    The down projection W_DKV maps each token's hidden state (width M) to the compressed
    KV feature (R) and the shared key (Dr) in one matrix, M -> R_kv + D_s (GatedMLA docs,
    "Projection geometry and stored weights"; W_DKV stored out x in as nn.Linear). The
    feature is normalised by kv_rmsnorm; the shared key is rotated by its token's
    position (rope above): [c ; k] is the cached row.
      hidden [T, M], W_DKV [R + Dr, M], kv_gain [R], positions [T]"""
    f = to_f64(hidden) @ to_f64(W_DKV).T
    c = rms_norm(f[:, :R], kv_gain, eps)
    k = rope(f[:, R:], positions, rope_base)
    return np.concatenate([c, k], axis=1)
