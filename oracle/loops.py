"""Scalar pure-Python restatement of MLA decode, for tiny brute-force cases.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

It takes nested Python lists of floats (no numpy) and spells out every sum, so it
shares neither code nor library calls with mla_oracle. Semantics as in the GatedMLA
docs ("Build per-head Q, K and V"; "Observe logits, then compute causal attention"):
per head, keys are [W_UK c_t ; k_t] with the same k_t for every head, values W_UV c_t,
softmax of scale times the dot product over the full Dn + Dr width.
"""
from __future__ import annotations

import math


def decode_one(qn, qr, rows, wuk_h, wuv_h, scale, R):
    """One head, one query.

    qn [Dn], qr [Dr], rows [L][R+Dr] (visible cache rows), wuk_h [Dn][R], wuv_h [Dv][R].
    Returns (out [Dv], lse)."""
    Dn, Dv = len(wuk_h), len(wuv_h)
    if not rows:
        return [0.0] * Dv, float("-inf")
    scores = []
    values = []
    for row in rows:
        c = row[:R]
        k_rope = row[R:]
        s = 0.0
        for d in range(Dn):
            kd = 0.0
            for r in range(R):
                kd += wuk_h[d][r] * c[r]
            s += qn[d] * kd
        for d in range(len(k_rope)):
            s += qr[d] * k_rope[d]
        scores.append(s * scale)
        v = []
        for d in range(Dv):
            acc = 0.0
            for r in range(R):
                acc += wuv_h[d][r] * c[r]
            v.append(acc)
        values.append(v)
    mx = max(scores)
    weights = [math.exp(s - mx) for s in scores]
    total = 0.0
    for w in weights:
        total += w
    out = []
    for d in range(Dv):
        acc = 0.0
        for w, v in zip(weights, values):
            acc += w * v[d]
        out.append(acc / total)
    return out, mx + math.log(total)
