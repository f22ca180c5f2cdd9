"""Numerics model of the tensor-core decode kernel's rounding points (CPU, no GPU).

This replays, in NumPy, the page-wise algorithm the SM-pair decode kernel runs on a
bf16 cache and compares its latent output with the fp64 oracle at the bf16 output
bound of the parity tests (|err| <= 2e-3 + 1e-2 |ref|). It is a model of the kernel's
rounding points, not the kernel: the GPU parity tests check the kernel itself. It pins
the one arithmetic decision the kernel makes for speed:

* P enters the value MMA in bf16, rounded to nearest. One rounding (8 significant
  bits) exceeds the bound on rows where one token carries a large share of the weight.
  So the kernel adds a second value MMA with the remainder P_lo = bf16(p - bf16(p)) on
  the pages where some row has 16 * max_t p_t > l, with l the running sum of the p
  that row's thread has summed so far (half of the row's tokens: the test only fires
  more often than one on the whole row would). With that rule the model stays under
  half the bound, and on long sequences the second MMA is needed on few pages.

Modelled per page of 64 tokens (the kernel's order): fp32 scores (one fp32 contraction
over the 576 columns), the scale in log2 units, a reference maximum moved only when a
page's maximum exceeds it by more than 24 (log2 units) with O and l rescaled then,
p = 2^(x - m) in fp32, l summed in fp32 from the unrounded p (two halves of 32 tokens
per row, added at the end), O accumulated from bf16(p) (+ P_lo on the pages the rule
picks) in fp32, and o = O / l kept in fp32 (the kernel's o_lat). The method's definition (softmax of the
scaled scores, weighted sum of the latent rows) is the Primer page's "Under the hood"
absorbed form, which the oracle pins to the non-absorbed definition.
"""
import math

import numpy as np
import pytest

from inputs import workloads as wl
from oracle import mla_oracle as orc

BOUND_ABS, BOUND_REL = 2e-3, 1e-2
LO_SHARE = 16.0
RESCALE = 24.0     # log2 units by which a page's maximum must pass the reference to move it


def f32(x):
    return np.asarray(x, np.float64).astype(np.float32)


def bf16_rn(x):
    return wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(f32(x)))


def page_wise_o_lat(q, rows, n, scale, p_lo, stats=None):
    """One query's o_lat [H, 512] by the kernel's page-wise algorithm (see the module doc).

    p_lo: "never" (one bf16 rounding of P), "rule" (the kernel's per-page rule) or
    "always"."""
    H = q.shape[0]
    sl2 = f32(scale / math.log(2))
    m = np.full(H, -np.inf, np.float32)
    l2 = np.zeros((H, 2), np.float32)       # the two lane halves' sums
    O = np.zeros((H, 512), np.float32)
    for pg in range((n + 63) // 64):
        R = rows[pg * 64:pg * 64 + 64]
        s = f32(q @ R.T)
        if s.shape[1] < 64:
            s = np.concatenate([s, np.full((H, 64 - s.shape[1]), -np.inf, np.float32)], 1)
            R = np.concatenate([R, np.zeros((64 - R.shape[0], R.shape[1]))], 0)
        s[:, np.arange(pg * 64, pg * 64 + 64) >= n] = -np.inf
        x = f32(s.astype(np.float64) * sl2)
        mx = x.max(1)
        need = mx > m + RESCALE
        mu = np.where(need, mx, m)
        al = np.where(need, f32(np.exp2((m - mu).astype(np.float64))), f32(1))
        z = np.where(np.isneginf(mu), 0, mu)
        p = f32(np.exp2((x - z[:, None]).astype(np.float64)))
        half_sums = p.reshape(H, 2, 32).astype(np.float64).sum(2)
        l2 = f32(l2 * al[:, None] + half_sums)
        hi = bf16_rn(p)
        lo = bf16_rn(p - hi)
        half_max = p.reshape(H, 2, 32).max(2)
        use_lo = {"never": False, "always": True}.get(p_lo, bool(np.any(half_max * LO_SHARE > l2)))
        if stats is not None:
            stats["pages"] += 1
            stats["lo"] += int(use_lo)
        P = hi.astype(np.float64) + (lo.astype(np.float64) if use_lo else 0.0)
        O = f32(O * al[:, None] + P @ R[:, :512])
        m = mu
    l = f32(l2[:, 0].astype(np.float64) + l2[:, 1])
    return f32(O / np.maximum(l, 1e-30)[:, None]).astype(np.float64)


def worst_ratio(H, q_len, lens, noise, p_lo, seed=11, stats=None):
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
            o = page_wise_o_lat(q[t], rows, n, w["scale"], p_lo, stats)
            r = ref["o_lat"][t]
            worst = max(worst, float((np.abs(o - r) / (BOUND_ABS + BOUND_REL * np.abs(r))).max()))
    return worst


# (H, q_len, lengths, logit noise std): a chunk whose early queries see a few tokens, two
# long sequences with spread-out logits, lengths around page boundaries, and a handful of
# very short 128-head queries
CASES = [(64, 5, [70, 5, 129], 0.0), (64, 1, [1000, 777], 4.0), (64, 1, [1, 63, 64, 65, 333], 0.0),
         (128, 1, [2, 3, 4, 5, 8, 17], 0.0)]


@pytest.mark.parametrize("case", [CASES[0], CASES[1], CASES[3]])
def test_one_bf16_rounding_of_p_exceeds_the_bound(case):
    assert worst_ratio(*case, p_lo="never") > 1.0


@pytest.mark.parametrize("case", CASES)
def test_p_lo_on_the_rule_pages_stays_well_inside_the_bound(case):
    assert worst_ratio(*case, p_lo="rule") < 0.5


def test_p_lo_is_rare_on_long_sequences():
    """A 3000-token 128-head query: the rule wants P_lo on its first pages only (the
    cost the kernel pays for the remainder is a small fraction of the value MMAs)."""
    stats = {"pages": 0, "lo": 0}
    r = worst_ratio(128, 1, [3000], 0.0, p_lo="rule", stats=stats)
    assert r < 0.5
    assert stats["lo"] <= 0.25 * stats["pages"], stats


# ----------------------------------------------------------------------------- prefill: stored up-projections

def _prefill_ratios(lens, H, heads, noise=0.0, seed=3):
    """Largest |out - definition| / bound per range of visible keys for a prefill that stores
    the per-head K_c = C W_UK^T and V = C W_UV^T in bf16 (everything else exact, output
    stored bf16): the part of the prefill's error its stored intermediates alone cause."""
    spec = wl.WorkloadSpec(name="prefill_model", B=0, H=H, R=512, Dr=64, Dn=128, Dv=128, q_len=1, dtype="bf16",
                           seq_len=None, w_std=1.0 / math.sqrt(512), all_query_positions=True,
                           logit_noise_std=noise)
    pin = wl.prefill_inputs(spec, lens, seed=seed)
    cu = pin["cu_seqlens"]
    worst = {}
    for b in range(len(lens)):
        a, e = int(cu[b]), int(cu[b + 1])
        rows = orc.to_f64(pin["ckr"][a:e])
        C, kr = rows[:, :512], rows[:, 512:]
        qn, qr = pin["q_nope"][a:e], pin["q_rope"][a:e]
        exact = orc.full_causal(C, kr, qn, qr, pin["W_UK"], pin["W_UV"], spec.scale, heads=heads)
        stored = orc.full_causal(C, kr, qn, qr, pin["W_UK"], pin["W_UV"], spec.scale, heads=heads,
                                 intermediates="kv_bf16")
        for h in heads:
            out = bf16_rn(stored[:, h])
            ratio = (np.abs(out - exact[:, h]) / (BOUND_ABS + BOUND_REL * np.abs(exact[:, h]))).max(axis=1)
            for lo, hi in [(2, 64), (65, 128), (129, 1 << 30)]:
                if e - a >= lo:
                    worst[(lo, hi)] = max(worst.get((lo, hi), 0.0), float(ratio[lo - 1:hi].max()))
    return worst


def test_prefill_short_rows_need_the_stored_intermediates_oracle():
    """The exemption the prefill's GPU tests make: with K_c and V stored in bf16, rows that
    see few keys leave the bound against the exact definition, rows past 128 keys stay
    inside it when the attention is spread, and with logit noise of std 4 (a few keys carry
    each row) long rows leave it too."""
    spread = _prefill_ratios([300, 700], 8, range(8))
    assert spread[(2, 64)] > 1.0              # short rows: stored values move single outputs past the bound
    assert spread[(129, 1 << 30)] < 0.9       # long spread rows: compared with the definition on the GPU
    peaked = _prefill_ratios([700], 4, range(4), noise=4.0, seed=5)
    assert peaked[(129, 1 << 30)] > 1.0       # peaked rows: held to the stored-intermediates oracle only
