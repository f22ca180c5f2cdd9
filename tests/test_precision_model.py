"""Numerics model of the tcgen05 decode kernels' arithmetic choices (CPU, no GPU).

This replays, in NumPy, the page-wise algorithm the decode kernels run on a bf16 cache
and compares its latent output with the fp64 oracle at the bf16 output bound of the
parity tests (|err| <= 2e-3 + 1e-2 |ref|). It is a model of the kernels' rounding
points, not the kernels: the GPU parity tests check the kernels themselves. It pins two
design decisions recorded with the kernels:

* P enters the value sum as two bf16 terms (P_hi = the top 16 bits of p, P_lo = the top
  16 bits of p - P_hi). One bf16 rounding of P (8 significant bits) exceeds the bound
  on queries that attend to a few comparable tokens; the two terms stay well inside.
* In the 2-CTA kernel each CTA's half of every score reaches the other CTA as a 16-bit
  code with one fp32 step per 32 scores, kept to 2^-16 of the block's largest
  magnitude; that leaves the result where the exact fp32 sum puts it.

Modelled per page of 64 tokens (the kernels' order): fp32 partial scores over each
CTA's half of the 576 columns, their sum, the scale in log2 units, a reference maximum
moved only when a page's maximum exceeds it by more than 8 (log2 units) with O and l
rescaled then, p = 2^(x - m) in fp32, l summed from the fp32 p, O accumulated from the
(rounded) P in fp32, and o = O / l rounded to bf16. The method's definition (softmax of
the scaled scores, weighted sum of the latent rows) is the Primer page's "Under the
hood" absorbed form, which the oracle pins to the non-absorbed definition.
"""
import math

import numpy as np
import pytest

from mla_latent_kv_46_b200 import workloads as wl
from oracle import mla_oracle as orc

BOUND_ABS, BOUND_REL = 2e-3, 1e-2
# the columns each CTA of a cluster owns: latent 0-127 and 256-383 plus rope 0-31 (CTA 0)
COLS0 = np.r_[0:128, 256:384, 512:544]
COLS1 = np.r_[128:256, 384:512, 544:576]


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32)


def bf16_rn(x):
    return wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(f32(x)))


def trunc16(x):
    return (f32(x).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def block16(v):
    """Codes and decoded values of the 16-bit exchange, blocks of 32 along the last axis."""
    v = f32(v)
    codes = np.empty(v.shape, np.int64)
    out = np.empty(v.shape, np.float64)
    for b0 in range(0, v.shape[-1], 32):
        blk = v[..., b0:b0 + 32]
        a = np.abs(blk).max(-1, keepdims=True)
        enc = np.where(a > 1e-30, f32(32767.0 / np.maximum(a, 1e-30).astype(np.float64)), f32(0))
        c = np.rint(blk.astype(np.float64) * enc.astype(np.float64)).astype(np.int64)   # one rounding (FMA)
        step = f32(a * f32(1.0 / 32767.0))
        codes[..., b0:b0 + 32] = c
        out[..., b0:b0 + 32] = c * step.astype(np.float64)
    return codes, out


def page_wise_o_lat(q, rows, n, scale, p_mode, exchange):
    """One query's o_lat [H, 512] by the kernels' page-wise algorithm (see the module doc)."""
    H = q.shape[0]
    sl2 = f32(scale / math.log(2))
    m = np.full(H, -np.inf, np.float32)
    l = np.zeros(H, np.float32)
    O = np.zeros((H, 512), np.float32)
    for pg in range((n + 63) // 64):
        R = rows[pg * 64:pg * 64 + 64]
        s0 = f32(q[:, COLS0] @ R[:, COLS0].T)
        s1 = f32(q[:, COLS1] @ R[:, COLS1].T)
        s = f32(s0 + (block16(s1)[1] if exchange else s1))
        s[:, np.arange(pg * 64, pg * 64 + R.shape[0]) >= n] = -np.inf
        x = f32(s.astype(np.float64) * sl2)
        mx = x.max(1)
        need = mx > m + 8
        mu = np.where(need, mx, m)
        al = np.where(need, f32(np.exp2((m - mu).astype(np.float64))), f32(1))
        z = np.where(np.isneginf(mu), 0, mu)
        p = f32(np.exp2((x - z[:, None]).astype(np.float64)))
        if p_mode == "bf16":
            P = bf16_rn(p).astype(np.float64)
        else:
            hi = trunc16(p)
            P = hi.astype(np.float64) + trunc16(p - hi).astype(np.float64)
        l = f32(l * al + p.astype(np.float64).sum(1))
        O = f32(O * al[:, None] + P @ R[:, :512])
        m = mu
    return bf16_rn(O / np.maximum(l, 1e-30)[:, None]).astype(np.float64)


def worst_ratio(H, q_len, lens, noise, p_mode, exchange, seed=11):
    """Largest |model - oracle| / bound over every output element of the case."""
    spec = wl.WorkloadSpec(name="model", B=0, H=H, R=512, Dr=64, Dn=128, Dv=128, q_len=q_len, dtype="bf16",
                           seq_len=None, w_std=1 / math.sqrt(512), page_size=64, logit_noise_std=noise)
    w = wl.make(spec, seed=seed, seq_lens=lens)
    ql = wl.latent_queries(spec, len(lens) * q_len, seed=9)
    ref = orc.attend_latent(ql, w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"], w["scale"],
                            q_len=q_len)
    q = np.concatenate([orc.to_f64(ql), orc.to_f64(w["q_rope"])], -1)
    worst = 0.0
    for b, L in enumerate(lens):
        rows = orc.gather_rows(w["kv_cache"], w["block_table"][b], L, 64)
        for i in range(q_len):
            n = orc.visible_len(L, q_len, i)
            if n <= 0:
                continue
            t = b * q_len + i
            o = page_wise_o_lat(q[t], rows, n, w["scale"], p_mode, exchange)
            r = ref["o_lat"][t]
            worst = max(worst, float((np.abs(o - r) / (BOUND_ABS + BOUND_REL * np.abs(r))).max()))
    return worst


# (H, q_len, lengths, logit noise std): a chunk whose early queries see a few tokens, two
# long sequences with spread-out logits, and lengths around page boundaries
CASES = [(64, 5, [70, 5, 129], 0.0), (64, 1, [1000, 777], 4.0), (64, 1, [1, 63, 64, 65, 333], 0.0)]


def test_block16_exchange_keeps_each_value_within_2e_16_of_its_block():
    rng = np.random.default_rng(3)
    # magnitudes spread over six decades, a zero block and a block with one outlier
    v = rng.standard_normal((64, 128)) * 10.0 ** rng.uniform(-3, 3, (64, 1))
    v[5, :32] = 0.0
    v[7, 40] = 1e4
    codes, dec = block16(v)
    v32 = f32(v).astype(np.float64)
    assert np.abs(codes).max() <= 32767                  # + 32768 fits 16 bits without wrapping
    for b0 in range(0, 128, 32):
        a = np.abs(v32[:, b0:b0 + 32]).max(1, keepdims=True)
        err = np.abs(dec[:, b0:b0 + 32] - v32[:, b0:b0 + 32])
        # half a code step (a / 65534) plus the fp32 rounding of the step times the code
        assert np.all(err <= a * 2.0 ** -16 * 1.01 + 1e-300)
    assert np.all(dec[5, :32] == 0.0)


@pytest.mark.parametrize("case", CASES[:2])
def test_one_bf16_rounding_of_p_exceeds_the_bound(case):
    assert worst_ratio(*case, p_mode="bf16", exchange=False) > 1.0


@pytest.mark.parametrize("case", CASES)
def test_split_p_with_the_score_exchange_stays_well_inside_the_bound(case):
    assert worst_ratio(*case, p_mode="split", exchange=True) < 0.5
