"""Pins of the E4M3 cache oracle (oracle/fp8.py) against things other than itself (CPU).

A library routine (torch's float8_e4m3fn conversions) for every code and for in-range
rounding including exact ties, an exhaustive nearest-code search for brute force, the
format's closed-form values, the scale rule's defining inequalities, exact round trips
of representable rows, and the link to the bf16 oracle: a dequantised cache is a cache
of bf16-representable values, so attention over it is the bf16 oracle's attention.
"""
import math

import numpy as np
import pytest
import torch

from inputs import workloads as wl
from oracle import fp8
from oracle import mla_oracle as orc

ALL_CODES = np.arange(256, dtype=np.uint8)


def torch_decode(codes):
    t = torch.from_numpy(np.asarray(codes, dtype=np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_round(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.float8_e4m3fn).to(torch.float64).numpy()


def finite_grid():
    v = torch_decode(ALL_CODES)
    return np.unique(v[np.isfinite(v)])


def test_decode_matches_torch_for_every_code():
    ours, ref = fp8.e4m3_decode(ALL_CODES), torch_decode(ALL_CODES)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.array_equal(np.signbit(ours[ok]), np.signbit(ref[ok]))   # 0x80 is -0
    assert np.sum(np.isnan(ours)) == 2                                   # 0x7F, 0xFF


def test_format_closed_forms():
    d = fp8.e4m3_decode
    assert d(0x7E) == 448.0 and d(0xFE) == -448.0          # 1.75 * 2^8
    assert d(0x08) == 2.0 ** -6                             # smallest normal
    assert d(0x01) == 2.0 ** -9 and d(0x07) == 7 * 2.0 ** -9
    assert d(0x38) == 1.0                                   # exponent field 7 = bias
    assert len(finite_grid()) == 253                        # 254 finite codes, +0 and -0 equal


def test_round_matches_torch_in_range_including_ties():
    g = np.random.default_rng(11)
    grid = finite_grid()
    pos = grid[grid > 0]
    mids = (pos[:-1] + pos[1:]) / 2.0                       # exact ties between neighbours
    rand = np.exp2(g.uniform(-13.0, math.log2(460.0), 20000)) * g.choice([-1.0, 1.0], 20000)
    x = np.concatenate([mids, -mids, rand, grid, [2.0 ** -10, 3 * 2.0 ** -10, 1.0625, 1.1875, 460.0]])
    assert np.array_equal(fp8.e4m3_round(x), torch_round(x))


def test_round_saturates_and_keeps_the_sign_of_zero():
    x = np.array([464.0, 470.0, 1e9, -1e30, -480.0, 2.0 ** -11, -(2.0 ** -11), 0.0, -0.0])
    r = fp8.e4m3_round(x)
    assert np.array_equal(r[:5], [448.0, 448.0, 448.0, -448.0, -448.0])
    assert np.all(r[5:] == 0.0)
    assert np.array_equal(np.signbit(r[5:]), [False, True, False, True])


def brute_round(x):
    """Nearest finite code by exhaustive search; a tie goes to the code with even
    mantissa; beyond the range the extreme code."""
    vals = fp8.e4m3_decode(ALL_CODES)
    out = []
    for xi in x:
        best = None
        for c in range(256):
            v = vals[c]
            if np.isnan(v) or (c & 0x80) != (0x80 if xi < 0 or (xi == 0 and math.copysign(1, xi) < 0) else 0):
                continue
            d = abs(v - xi)
            key = (d, (c & 1))                  # smaller distance, then even mantissa
            if best is None or key < best[0]:
                best = (key, v)
        out.append(best[1])
    return np.array(out)


def test_round_against_exhaustive_search():
    g = np.random.default_rng(12)
    grid = finite_grid()
    pos = grid[grid > 0]
    x = np.concatenate([g.uniform(-500, 500, 300), np.exp2(g.uniform(-12, 8.9, 300)),
                        (pos[:-1] + pos[1:])[::5] / 2.0, [2.0 ** -10, -3 * 2.0 ** -10, 700.0, -1e6]])
    assert np.array_equal(fp8.e4m3_round(x), brute_round(x))


def test_encode_inverts_decode():
    finite = ~np.isnan(fp8.e4m3_decode(ALL_CODES))
    codes = ALL_CODES[finite]
    assert np.array_equal(fp8.e4m3_encode(fp8.e4m3_decode(codes)), codes)
    with pytest.raises(ValueError):
        fp8.e4m3_encode(np.array([1.0 + 1.0 / 16.0]))          # between two codes


def test_scale_is_the_smallest_power_of_two_that_fits():
    g = np.random.default_rng(13)
    rows = g.standard_normal((400, 576)) * np.exp2(g.uniform(-30, 20, (400, 1)))
    rows[0] = 0.0
    rows[1, 5] = 448.0 * 2.0 ** -3                              # exactly on a boundary
    rows[2] *= 0.0
    rows[2, 0] = 1e9                                            # beyond 448 * 2^7: saturates
    k = fp8.row_scale_exponent(rows)
    amax = np.abs(rows).max(axis=1)
    assert np.all(k >= fp8.SCALE_K_MIN) and np.all(k <= fp8.SCALE_K_MAX)
    fits = amax <= np.ldexp(448.0, k)
    assert np.all(fits | (k == fp8.SCALE_K_MAX))
    smaller_fits = amax <= np.ldexp(448.0, k - 1)
    assert not np.any(smaller_fits & (k > fp8.SCALE_K_MIN))
    assert k[0] == fp8.SCALE_K_MIN and k[1] == -3 and k[2] == fp8.SCALE_K_MAX
    codes, sb = fp8.quantise_rows(rows[2:3])
    assert fp8.dequantise_rows(codes, sb)[0, 0] == 448.0 * 2.0 ** 7


def test_representable_rows_round_trip_exactly():
    g = np.random.default_rng(14)
    grid = finite_grid()
    for k in (-20, -6, 0, 5):
        v = g.choice(grid, (8, 576))
        v[:, 0] = g.choice(grid[(np.abs(grid) > 224.0)], 8)      # amax in (224, 448]
        rows = np.ldexp(v, k)
        codes, sb = fp8.quantise_rows(rows)
        assert np.all(sb == k + fp8.SCALE_BIAS)
        assert np.array_equal(fp8.dequantise_rows(codes, sb), rows)


def test_quantisation_error_is_at_most_half_a_step():
    g = np.random.default_rng(15)
    rows = g.standard_normal((64, 576))
    codes, sb = fp8.quantise_rows(rows)
    deq = fp8.dequantise_rows(codes, sb)
    s = np.ldexp(1.0, sb.astype(np.int64) - 127)[:, None]
    a = np.abs(rows)
    bound = np.where(a >= 2.0 ** -6 * s, a * 2.0 ** -4, 2.0 ** -10 * s)
    assert np.all(np.abs(deq - rows) <= bound)


def test_attention_over_a_dequantised_cache_is_bf16_attention_of_the_same_values():
    spec = wl.WorkloadSpec(name="small", B=2, H=4, R=64, Dr=16, Dn=32, Dv=24, q_len=1, dtype="bf16",
                           seq_len=None, w_std=1.0 / 8.0, page_size=16)
    w = wl.make(spec, seed=3, seq_lens=[40, 17])
    rows = orc.to_f64(w["kv_cache"])
    codes, sb = fp8.quantise_rows(rows)
    deq = fp8.dequantise_rows(codes, sb)
    # every dequantised value has at most four significant bits: it is a bf16 value
    bits = wl.f32_to_bf16_bits(deq.astype(np.float32))
    assert np.array_equal(orc.to_f64(bits), deq)
    args = (w["q_nope"], w["q_rope"])
    rest = (w["block_table"], w["seq_lens"], w["W_UK"], w["W_UV"], w["scale"])
    a = orc.decode_nonabsorbed(*args, deq, *rest, page_size=16)
    b = orc.decode_nonabsorbed(*args, bits, *rest, page_size=16)
    for key in ("out", "o_lat", "lse"):
        assert np.array_equal(a[key], b[key])


@pytest.mark.parametrize("mistake", ["ties_away", "bias_8", "no_saturation", "scale_off_by_one"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    """Each plausible slip in the E4M3 oracle fails at least one pin above."""
    if mistake == "ties_away":
        monkeypatch.setattr(fp8.np, "rint", lambda a: np.floor(a + 0.5))
        pins = [test_round_matches_torch_in_range_including_ties]
    elif mistake == "bias_8":
        real = fp8.e4m3_decode
        monkeypatch.setattr(fp8, "e4m3_decode", lambda c: real(c) / 2.0)
        pins = [test_decode_matches_torch_for_every_code, test_format_closed_forms]
    elif mistake == "no_saturation":
        monkeypatch.setattr(fp8, "E4M3_MAX", np.inf)
        pins = [test_round_saturates_and_keeps_the_sign_of_zero]
    else:
        real_k = fp8.row_scale_exponent
        monkeypatch.setattr(fp8, "row_scale_exponent", lambda r: np.minimum(real_k(r) + 1, fp8.SCALE_K_MAX))
        pins = [test_scale_is_the_smallest_power_of_two_that_fits, test_representable_rows_round_trip_exactly]
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError):
            caught += 1
    assert caught >= 1
