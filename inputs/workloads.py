"""Seeded synthetic inputs for MLA decode over a paged latent+RoPE cache.

This module draws random numbers, rounds them to the storage dtype and lays
them out (pages, block tables). It holds none of the attention arithmetic, so
both the CUDA path and the fp64 oracle can be fed from it.

Every array is a host numpy array. bf16 tensors are stored as ``uint16`` bit
patterns (round-to-nearest-even from float32); fp32 workloads use float32.

Shapes (the library's layout, row-major, contiguous):
  kv_cache    [num_pages, page_size, R + Dr]   row = [c (R) ; k_rope (Dr)]
  block_table [B, max_pages] int32             page ids, 0-padded past the end
  seq_lens    [B] int32                        cached tokens incl. the q_len new ones
  q_nope      [B*q_len, H, Dn]
  q_rope      [B*q_len, H, Dr]
  W_UK        [H, Dn, R]                       per-head key up-projection slice
  W_UV        [H, Dv, R]                       per-head value up-projection slice
  new_ckr     [B*q_len, R + Dr]                rows of the q_len newest tokens

Random streams are keyed by ``numpy.random.SeedSequence`` entropy tuples so a
single sequence's rows (or queries) can be regenerated on their own.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

PAGE_SIZE = 64


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    B: int
    H: int
    R: int
    Dr: int
    Dn: int
    Dv: int
    q_len: int
    dtype: str                 # "bf16" or "f32"
    seq_len: Optional[int]     # fixed length, or None for ragged
    ragged: Optional[tuple] = None   # (lo, hi) inclusive, uniform integers
    w_std: float = 0.0
    logit_noise_std: float = 0.0     # per-token logit offset std (0 = off)
    all_query_positions: bool = False  # also draw queries for every cached position
    page_size: int = PAGE_SIZE
    description: str = ""

    @property
    def scale(self) -> float:
        # softmax scale over the full query/key head width (nope + rope)
        return 1.0 / math.sqrt(self.Dn + self.Dr)

    @property
    def row(self) -> int:
        return self.R + self.Dr


WORKLOADS: Dict[str, WorkloadSpec] = {
    "tiny_fp32": WorkloadSpec(
        name="tiny_fp32", B=1, H=4, R=32, Dr=16, Dn=16, Dv=16, q_len=1, dtype="f32",
        seq_len=64, w_std=1.0 / math.sqrt(32),
        description="tiny fp32 decode, dense cache (one 64-token page), 64 cached tokens"),
    "kimi_h64_b64_l4096": WorkloadSpec(
        name="kimi_h64_b64_l4096", B=64, H=64, R=512, Dr=64, Dn=128, Dv=128, q_len=1,
        dtype="bf16", seq_len=4096, w_std=1.0 / math.sqrt(512),
        description="Kimi/GLM-scale decode, H=64, 64 sequences x 4096 tokens, paged"),
    "deepseek_h128_b128_ragged": WorkloadSpec(
        name="deepseek_h128_b128_ragged", B=128, H=128, R=512, Dr=64, Dn=128, Dv=128, q_len=1,
        dtype="bf16", seq_len=None, ragged=(512, 16384), w_std=1.0 / math.sqrt(512),
        description="DeepSeek head count, H=128, 128 sequences, lengths uniform in [512,16384]"),
    "longctx_h64_b4_l131072": WorkloadSpec(
        name="longctx_h64_b4_l131072", B=4, H=64, R=512, Dr=64, Dn=128, Dv=128, q_len=1,
        dtype="bf16", seq_len=131072, w_std=1.0 / math.sqrt(512), logit_noise_std=4.0,
        description="long-context split-KV decode, 4 x 131072 tokens, logit noise std 4"),
    "mtp2_h128_b64_ragged": WorkloadSpec(
        name="mtp2_h128_b64_ragged", B=64, H=128, R=512, Dr=64, Dn=128, Dv=128, q_len=2,
        dtype="bf16", seq_len=None, ragged=(512, 16384), w_std=1.0 / math.sqrt(512),
        description="two new tokens per sequence (multi-token decode), H=128, 64 sequences, "
                    "lengths uniform in [512,16384]"),
    "prefill_h64_b4_l4096": WorkloadSpec(
        name="prefill_h64_b4_l4096", B=4, H=64, R=512, Dr=64, Dn=128, Dv=128, q_len=4096,
        dtype="bf16", seq_len=4096, w_std=1.0 / math.sqrt(512), all_query_positions=True,
        description="non-absorbed prefill (every position a query, causal), H=64, 4 sequences x 4096"),
    "causal_chunk_h64_b8_2048p256": WorkloadSpec(
        name="causal_chunk_h64_b8_2048p256", B=8, H=64, R=512, Dr=64, Dn=128, Dv=128, q_len=256,
        dtype="bf16", seq_len=2048 + 256, w_std=1.0 / math.sqrt(512), all_query_positions=True,
        description="multi-token causal chunk: 2048 cached + 256 new tokens, H=64"),
}


def spec_with(base: str, **overrides) -> WorkloadSpec:
    """A copy of a named workload with some fields replaced (small parity cases)."""
    return dataclasses.replace(WORKLOADS[base], **overrides)


# ----------------------------------------------------------------------------- dtype helpers

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _store(spec: WorkloadSpec, x32: np.ndarray) -> np.ndarray:
    return f32_to_bf16_bits(x32) if spec.dtype == "bf16" else np.ascontiguousarray(x32, np.float32)


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, *key]))


# ----------------------------------------------------------------------------- pieces

def seq_lens_of(spec: WorkloadSpec, seed: int = 0) -> np.ndarray:
    if spec.ragged is not None:
        lo, hi = spec.ragged
        return _rng(seed, 1).integers(lo, hi, size=spec.B, endpoint=True).astype(np.int32)
    return np.full(spec.B, spec.seq_len, dtype=np.int32)


def weights_of(spec: WorkloadSpec, seed: int = 0):
    g = _rng(seed, 0)
    wuk = g.standard_normal((spec.H, spec.Dn, spec.R), dtype=np.float32) * np.float32(spec.w_std)
    wuv = g.standard_normal((spec.H, spec.Dv, spec.R), dtype=np.float32) * np.float32(spec.w_std)
    return _store(spec, wuk), _store(spec, wuv)


def sequence_rows(spec: WorkloadSpec, b: int, L: int, seed: int = 0) -> np.ndarray:
    """The [L, R+Dr] cache rows of sequence b, in storage dtype."""
    g = _rng(seed, 3, b)
    rows = g.standard_normal((L, spec.row), dtype=np.float32)
    if spec.logit_noise_std > 0.0:
        # Per-token logit offset realised in the data: k_rope[0] = n_t / scale and every
        # head's q_rope[0] = 1 (see queries_of), so each head's logit gains scale*k_rope[0].
        n = _rng(seed, 5, b).standard_normal(L, dtype=np.float32) * np.float32(spec.logit_noise_std)
        rows[:, spec.R] = n / np.float32(spec.scale)
    return _store(spec, rows)


def query_count(spec: WorkloadSpec, L: int) -> int:
    return L if spec.all_query_positions else spec.q_len


def queries_of(spec: WorkloadSpec, b: int, L: int, seed: int = 0):
    """(q_nope, q_rope) of sequence b: [n, H, Dn], [n, H, Dr].

    n = q_len for decode workloads (the newest q_len positions), or L when every
    position's query is drawn (the last q_len of them are the decode queries).
    """
    n = query_count(spec, L)
    g = _rng(seed, 4, b)
    qn = g.standard_normal((n, spec.H, spec.Dn), dtype=np.float32)
    qr = g.standard_normal((n, spec.H, spec.Dr), dtype=np.float32)
    if spec.logit_noise_std > 0.0:
        qr[:, :, 0] = 1.0
    return _store(spec, qn), _store(spec, qr)


def block_table_of(spec: WorkloadSpec, seq_lens: np.ndarray, seed: int = 0):
    """Random permutation of a shared page pool, cut into per-sequence page lists."""
    P = spec.page_size
    npages = [(int(L) + P - 1) // P for L in seq_lens]
    total = int(sum(npages))
    perm = _rng(seed, 2).permutation(total).astype(np.int32)
    max_pages = max(1, max(npages) if npages else 1)
    bt = np.zeros((len(seq_lens), max_pages), dtype=np.int32)
    off = 0
    for b, n in enumerate(npages):
        bt[b, :n] = perm[off:off + n]
        off += n
    return bt, total


def make(spec: WorkloadSpec | str, seed: int = 0, new_rows_in_cache: bool = True,
         seq_lens: Optional[Sequence[int]] = None) -> dict:
    """Build a whole workload.

    new_rows_in_cache: if False the q_len newest rows of every sequence are left zero
    in the pages (they arrive through ``new_ckr`` and the append call).
    seq_lens: override the workload's lengths (small parity cases, edge cases).
    """
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    lens = np.asarray(seq_lens, dtype=np.int32) if seq_lens is not None else seq_lens_of(spec, seed)
    B = len(lens)
    bt, num_pages = block_table_of(spec, lens, seed)
    num_pages = max(num_pages, 1)
    sdt = np.uint16 if spec.dtype == "bf16" else np.float32
    kv = np.zeros((num_pages, spec.page_size, spec.row), dtype=sdt)
    T = B * spec.q_len
    q_nope = np.zeros((T, spec.H, spec.Dn), dtype=sdt)
    q_rope = np.zeros((T, spec.H, spec.Dr), dtype=sdt)
    new_ckr = np.zeros((T, spec.row), dtype=sdt)
    all_q: List[tuple] = []
    P = spec.page_size
    for b in range(B):
        L = int(lens[b])
        rows = sequence_rows(spec, b, L, seed)
        n_store = L if new_rows_in_cache else max(0, L - spec.q_len)
        for p in range((n_store + P - 1) // P):
            lo, hi = p * P, min(n_store, (p + 1) * P)
            kv[bt[b, p], : hi - lo] = rows[lo:hi]
        qn, qr = queries_of(spec, b, L, seed)
        nq = qn.shape[0]
        take = min(spec.q_len, nq)
        q_nope[b * spec.q_len + spec.q_len - take: (b + 1) * spec.q_len] = qn[nq - take:]
        q_rope[b * spec.q_len + spec.q_len - take: (b + 1) * spec.q_len] = qr[nq - take:]
        k = min(spec.q_len, L)
        new_ckr[b * spec.q_len + spec.q_len - k: (b + 1) * spec.q_len] = rows[L - k:]
        if spec.all_query_positions:
            all_q.append((qn, qr))
    wuk, wuv = weights_of(spec, seed)
    out = dict(spec=spec, seed=seed, kv_cache=kv, block_table=bt, seq_lens=lens,
               q_nope=q_nope, q_rope=q_rope, W_UK=wuk, W_UV=wuv, new_ckr=new_ckr,
               num_pages=num_pages, scale=spec.scale)
    if spec.all_query_positions:
        out["all_queries"] = all_q
    return out


def cache_bytes(spec: WorkloadSpec, seq_lens: np.ndarray) -> int:
    """Algorithmic cache bytes of one decode pass: every valid cached row read once."""
    elem = 2 if spec.dtype == "bf16" else 4
    return int(np.sum(seq_lens, dtype=np.int64)) * spec.row * elem


def attention_pairs(spec: WorkloadSpec, seq_lens: np.ndarray) -> int:
    """(query, visible cached token) pairs; causal within a multi-token chunk."""
    total = 0
    for L in seq_lens:
        L = int(L)
        for i in range(spec.q_len):
            total += max(0, L - spec.q_len + i + 1)
    return total


def attention_flops(spec: WorkloadSpec, seq_lens: np.ndarray) -> int:
    """2*H*((R+Dr) + R) FLOP per (query, token) pair: scores over the 576-wide row,
    then the latent value sum over R."""
    return attention_pairs(spec, seq_lens) * 2 * spec.H * (spec.row + spec.R)


def latent_queries(spec: WorkloadSpec, T: int, seed: int = 0) -> np.ndarray:
    """Seeded stand-in for an absorbed query, [T, H, R] in storage dtype: entries
    N(0, 0.5^2), the spread W_UK^T q_nope has with q_nope ~ N(0,1), W_UK std 1/sqrt(R)
    and Dn = R/4 (the kernel-level decode tests feed it directly)."""
    g = _rng(seed, 6)
    return _store(spec, g.standard_normal((T, spec.H, spec.R), dtype=np.float32) * np.float32(0.5))


def prologue_inputs(spec: WorkloadSpec, T: int, M: int, seed: int = 0) -> dict:
    """Seeded inputs of the cache-write prologue in the workload's storage dtype: hidden
    states [T, M] ~ N(0, 1), the down projection W_DKV [R + Dr, M] ~ N(0, 1/M) (unit-scale
    outputs) and the latent norm's gain [R] ~ 1 + N(0, 0.1^2)."""
    g = _rng(seed, 8)
    hidden = g.standard_normal((T, M), dtype=np.float32)
    w = g.standard_normal((spec.R + spec.Dr, M), dtype=np.float32) * np.float32(1.0 / math.sqrt(M))
    gain = np.float32(1.0) + g.standard_normal(spec.R, dtype=np.float32) * np.float32(0.1)
    return dict(hidden=_store(spec, hidden), W_DKV=_store(spec, w), kv_gain=_store(spec, gain))


def latent_outputs(spec: WorkloadSpec, T: int, seed: int = 0, fp32: bool = False) -> np.ndarray:
    """Seeded stand-in for a latent attention output, [T, H, R]: entries N(0, 0.1^2),
    in the workload's storage dtype, or as float32 values when `fp32`."""
    g = _rng(seed, 7)
    x = g.standard_normal((T, spec.H, spec.R), dtype=np.float32) * np.float32(0.1)
    return x if fp32 else _store(spec, x)


def prefill_inputs(spec: WorkloadSpec, seq_lens: Optional[Sequence[int]] = None, seed: int = 0) -> dict:
    """Packed inputs of a prefill over whole sequences (every position a query): the rows
    [c ; k_rope] of all sequences back to back [N, R+Dr], their queries [N, H, Dn] and
    [N, H, Dr], cu_seqlens [B+1] and the weights, in storage dtype. The same per-sequence
    streams as the decode workloads' rows and queries."""
    lens = [int(x) for x in (seq_lens if seq_lens is not None else seq_lens_of(spec, seed))]
    s_all = dataclasses.replace(spec, all_query_positions=True)
    rows, qns, qrs = [], [], []
    for b, L in enumerate(lens):
        rows.append(sequence_rows(s_all, b, L, seed))
        qn, qr = queries_of(s_all, b, L, seed)
        qns.append(qn)
        qrs.append(qr)
    sdt = np.uint16 if spec.dtype == "bf16" else np.float32
    cat = lambda xs, shape: np.concatenate(xs) if xs else np.zeros(shape, sdt)  # noqa: E731
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    wuk, wuv = weights_of(spec, seed)
    return dict(spec=spec, seq_lens=np.asarray(lens, np.int32), cu_seqlens=cu,
                ckr=cat(rows, (0, spec.row)), q_nope=cat(qns, (0, spec.H, spec.Dn)),
                q_rope=cat(qrs, (0, spec.H, spec.Dr)), W_UK=wuk, W_UV=wuv, scale=spec.scale)


def prefill_flops(spec: WorkloadSpec, seq_lens) -> dict:
    """FLOPs of a non-absorbed prefill: the up-projections (2 R H (Dn + Dv) per token) and
    the causal attention (2 H (Dn + Dr + Dv) per (query, key) pair, key <= query)."""
    lens = np.asarray(seq_lens, dtype=np.int64)
    pairs = int(np.sum(lens * (lens + 1) // 2))
    up = int(lens.sum()) * 2 * spec.R * spec.H * (spec.Dn + spec.Dv)
    attn = pairs * 2 * spec.H * (spec.Dn + spec.Dr + spec.Dv)
    return dict(pairs=pairs, up=up, attention=attn)
