"""Pins of the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each oracle function is checked against something other than itself: the pages'
printed values (tests/golden/), closed forms, a library routine
(torch's scaled_dot_product_attention in float64), a scalar brute-force
restatement (oracle/loops.py), and invariants. The last block plants plausible
mistakes in the oracle and checks that some pin catches each of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from inputs import workloads as wl
from oracle import ledger, loops
from oracle import mla_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def small_bf16(B=3, H=4, R=64, Dr=16, Dn=32, Dv=24, q_len=1, lens=(70, 1, 129), page=16, **kw):
    spec = wl.WorkloadSpec(name="small", B=B, H=H, R=R, Dr=Dr, Dn=Dn, Dv=Dv, q_len=q_len,
                           dtype="bf16", seq_len=None, w_std=1.0 / math.sqrt(R), page_size=page, **kw)
    return wl.make(spec, seed=7, seq_lens=list(lens))


def tiny():
    return wl.make("tiny_fp32", seed=0)


def run_ref(w, **kw):
    s = w["spec"]
    return orc.decode_nonabsorbed(w["q_nope"], w["q_rope"], w["kv_cache"], w["block_table"],
                                  w["seq_lens"], w["W_UK"], w["W_UV"], w["scale"], q_len=s.q_len,
                                  page_size=s.page_size, **kw)


# ----------------------------------------------------------------------------- ledger (tutorial Step 4)

def test_ledger_matches_tutorial_printed_values():
    g = _golden("ledger_tutorial.json")
    cfg = g["config"]
    for mode, v in g["bytes_per_token"].items():
        assert ledger.cache_bytes_per_token(mode, cfg) == v
    rep = ledger.compare_attention_states(cfg)
    assert rep["ratio_vs_mha"] == g["ratio_vs_mha"]
    assert rep["most_compact"] == g["most_compact"]
    for bad in g["rejected_overrides"]:
        with pytest.raises(ValueError):
            ledger.validate_attention_state_config(dict(cfg, **bad))


@pytest.mark.parametrize("bad", [{"head_dim": 0}, {"rope_dim": -1}, {"latent_dim": 2.5}, {"dtype_bytes": True}])
def test_ledger_rejects_non_positive_integers(bad):
    cfg = _golden("ledger_tutorial.json")["config"]
    with pytest.raises(ValueError):
        ledger.validate_attention_state_config(dict(cfg, **bad))


def test_ledger_rejects_missing_field_and_unknown_mode():
    cfg = dict(_golden("ledger_tutorial.json")["config"])
    with pytest.raises(ValueError):
        ledger.cache_bytes_per_token("mqa", cfg)
    del cfg["rope_dim"]
    with pytest.raises(ValueError):
        ledger.validate_attention_state_config(cfg)


def test_primer_cache_size_table():
    g = _golden("primer_cache_table.json")
    cfg = g["config"]
    for mode, v in g["elements_per_token"].items():
        assert ledger.elements_per_token(mode, cfg) == v
    assert ledger.cache_bytes_per_token("mla", dict(cfg, dtype_bytes=2)) == g["bf16_bytes_mla"]
    mha, mla, gqa = (ledger.elements_per_token(m, cfg) for m in ("mha", "mla", "gqa"))
    assert round(mha / mla) == g["mha_over_mla_rounded"]
    assert mha // gqa == g["mha_over_gqa"]


def test_tutorial_cache_reduction():
    g = _golden("tutorial_reduction.json")
    rep = ledger.compare_attention_states(g["config"])
    for mode, red in g["reduction_vs_mha"].items():
        assert 1.0 - rep["ratio_vs_mha"][mode] == red


def test_workload_row_is_576_elements_1152_bytes():
    s = wl.WORKLOADS["kimi_h64_b64_l4096"]
    assert s.row == 576 and s.row * 2 == 1152


# ----------------------------------------------------------------------------- paging and append

def test_gather_rows_recovers_generated_sequences():
    w = small_bf16()
    s = w["spec"]
    for b, L in enumerate(w["seq_lens"]):
        want = orc.to_f64(wl.sequence_rows(s, b, int(L), seed=7))
        got = orc.gather_rows(w["kv_cache"], w["block_table"][b], int(L), s.page_size)
        np.testing.assert_array_equal(got, want)


def test_cache_append_writes_only_the_new_rows():
    w = small_bf16(q_len=3, lens=(70, 3, 129))
    s = w["spec"]
    empty = wl.make(s, seed=7, new_rows_in_cache=False, seq_lens=list(w["seq_lens"]))
    filled = orc.cache_append(empty["kv_cache"], w["block_table"], w["seq_lens"], w["new_ckr"], s.q_len,
                              s.page_size)
    np.testing.assert_array_equal(filled, w["kv_cache"])
    # the input cache is left as it was
    assert not np.array_equal(empty["kv_cache"], w["kv_cache"])


# ----------------------------------------------------------------------------- algebraic identity (primer)

@pytest.mark.parametrize("case", ["tiny", "paged_bf16", "chunk_bf16"])
def test_absorbed_equals_nonabsorbed(case):
    w = {"tiny": tiny, "paged_bf16": small_bf16,
         "chunk_bf16": lambda: small_bf16(q_len=5, lens=(37, 5, 64))}[case]()
    s = w["spec"]
    ref = run_ref(w)
    ab = orc.decode_absorbed(w["q_nope"], w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"],
                             w["W_UK"], w["W_UV"], w["scale"], q_len=s.q_len, page_size=s.page_size)
    for k in ("out", "o_lat", "lse"):
        np.testing.assert_allclose(ab[k], ref[k], rtol=0, atol=1e-10)


# ----------------------------------------------------------------------------- brute force (scalar loops)

def _loops_case(w):
    s = w["spec"]
    qn, qr = orc.to_f64(w["q_nope"]), orc.to_f64(w["q_rope"])
    wuk, wuv = orc.to_f64(w["W_UK"]), orc.to_f64(w["W_UV"])
    out = np.zeros((qn.shape[0], s.H, s.Dv))
    lse = np.zeros((qn.shape[0], s.H))
    for b, L in enumerate(w["seq_lens"]):
        L = int(L)
        rows = []
        for t in range(L):
            page = int(w["block_table"][b][t // s.page_size])
            rows.append([float(x) for x in orc.to_f64(w["kv_cache"][page, t % s.page_size])])
        for i in range(s.q_len):
            t = b * s.q_len + i
            n = L - s.q_len + i + 1
            for h in range(s.H):
                o, z = loops.decode_one(qn[t, h].tolist(), qr[t, h].tolist(), rows[:max(n, 0)],
                                        wuk[h].tolist(), wuv[h].tolist(), w["scale"], s.R)
                out[t, h] = o
                lse[t, h] = z
    return out, lse


@pytest.mark.parametrize("case", ["tiny", "chunk_bf16"])
def test_oracle_matches_scalar_brute_force(case):
    w = tiny() if case == "tiny" else small_bf16(B=2, H=2, R=16, Dr=8, Dn=8, Dv=8, q_len=3, lens=(11, 20),
                                                 page=4)
    ref = run_ref(w)
    out, lse = _loops_case(w)
    np.testing.assert_allclose(ref["out"], out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ref["lse"], lse, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- library special case (SDPA)

def test_full_causal_equals_torch_sdpa_fp64():
    """GatedMLA runs causal SDPA on per-head Q=[qn;qr], K=[K_c;shared k], V with the
    default scale over the full Q/K width; build those with torch and compare."""
    w = tiny()
    s = w["spec"]
    L = int(w["seq_lens"][0])
    rows = orc.to_f64(wl.sequence_rows(s, 0, L, seed=0))
    qn, qr = wl.queries_of(wl.spec_with("tiny_fp32", all_query_positions=True), 0, L, seed=0)
    ours = orc.full_causal(rows[:, :s.R], rows[:, s.R:], qn, qr, w["W_UK"], w["W_UV"], w["scale"])
    C = torch.tensor(rows[:, :s.R])                                  # [L, R]
    kr = torch.tensor(rows[:, s.R:])                                 # [L, Dr]
    wuk = torch.tensor(w["W_UK"], dtype=torch.float64)               # [H, Dn, R]
    wuv = torch.tensor(w["W_UV"], dtype=torch.float64)               # [H, Dv, R]
    Kc = torch.einsum("lr,hdr->hld", C, wuk)                         # [H, L, Dn]
    K = torch.cat([Kc, kr.unsqueeze(0).expand(s.H, L, s.Dr)], dim=-1)
    V = torch.einsum("lr,hdr->hld", C, wuv)
    Q = torch.cat([torch.tensor(qn, dtype=torch.float64), torch.tensor(qr, dtype=torch.float64)], -1)
    Q = Q.permute(1, 0, 2)                                           # [H, L, Dn+Dr]
    lib = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True)
    np.testing.assert_allclose(ours, lib.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    assert abs(w["scale"] - 1.0 / math.sqrt(Q.shape[-1])) < 1e-15


# ----------------------------------------------------------------------------- ticket acceptance

def test_incremental_decode_equals_full_causal_tiny():
    """'MLA + KV cache' ticket, acceptance: decode over the cache == full forward
    (atol 1e-5); here every prefix length 1..64 of the tiny fp32 workload."""
    s = wl.spec_with("tiny_fp32", all_query_positions=True)
    L = 64
    rows = wl.sequence_rows(s, 0, L, seed=0)
    qn, qr = wl.queries_of(s, 0, L, seed=0)
    wuk, wuv = wl.weights_of(s, seed=0)
    full = orc.full_causal(orc.to_f64(rows[:, :s.R]), orc.to_f64(rows[:, s.R:]), qn, qr, wuk, wuv, s.scale)
    kv = np.zeros((1, 64, s.row), np.float32)
    kv[0] = rows
    bt = np.zeros((1, 1), np.int32)
    for n in range(1, L + 1):
        dec = orc.decode_nonabsorbed(qn[n - 1:n], qr[n - 1:n], kv, bt, np.array([n]), wuk, wuv, s.scale)
        np.testing.assert_allclose(dec["out"][0], full[n - 1], rtol=0, atol=1e-5)
        np.testing.assert_allclose(dec["out"][0], full[n - 1], rtol=0, atol=1e-12)


def test_chunk_decode_equals_full_causal_tail():
    """A q_len-token causal chunk over the cache equals the last q_len rows of the full
    causal forward (the multi-token chunk workload's check, at a small size)."""
    spec = wl.WorkloadSpec(name="c", B=2, H=3, R=32, Dr=8, Dn=16, Dv=16, q_len=12, dtype="bf16",
                           seq_len=None, w_std=1 / math.sqrt(32), all_query_positions=True, page_size=8)
    w = wl.make(spec, seed=3, seq_lens=[40, 12])
    dec = run_ref(w)
    for b, L in enumerate(w["seq_lens"]):
        L = int(L)
        rows = orc.to_f64(wl.sequence_rows(spec, b, L, seed=3))
        qn, qr = w["all_queries"][b]
        full = orc.full_causal(rows[:, :spec.R], rows[:, spec.R:], qn, qr, w["W_UK"], w["W_UV"], w["scale"])
        np.testing.assert_allclose(dec["out"][b * 12:(b + 1) * 12], full[L - 12:], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- closed forms and invariants

def test_single_token_gives_w_uv_c0():
    w = small_bf16(lens=(1, 1, 1))
    ref = run_ref(w)
    s = w["spec"]
    for b in range(3):
        c0 = orc.to_f64(w["kv_cache"][w["block_table"][b][0], 0, :s.R])
        want = np.einsum("hvr,r->hv", orc.to_f64(w["W_UV"]), c0)
        np.testing.assert_allclose(ref["out"][b], want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(ref["o_lat"][b], np.broadcast_to(c0, (s.H, s.R)), rtol=0, atol=1e-15)


def test_equal_rows_give_w_uv_c_and_log_len_lse():
    w = small_bf16(lens=(50, 9, 129))
    s = w["spec"]
    row = w["kv_cache"][0, 0].copy()
    w["kv_cache"][:] = row
    ref = run_ref(w)
    c = orc.to_f64(row[:s.R])
    want = np.einsum("hvr,r->hv", orc.to_f64(w["W_UV"]), c)
    qn, qr = orc.to_f64(w["q_nope"]), orc.to_f64(w["q_rope"])
    wuk = orc.to_f64(w["W_UK"])
    for b, L in enumerate(w["seq_lens"]):
        np.testing.assert_allclose(ref["out"][b], want, rtol=0, atol=1e-12)
        s0 = w["scale"] * (np.einsum("hn,hnr,r->h", qn[b], wuk, c) + qr[b] @ orc.to_f64(row[s.R:]))
        np.testing.assert_allclose(ref["lse"][b], s0 + math.log(int(L)), rtol=0, atol=1e-10)


def test_zero_query_gives_uniform_mean():
    w = small_bf16()
    s = w["spec"]
    w["q_nope"][:] = 0
    w["q_rope"][:] = 0
    ref = run_ref(w)
    for b, L in enumerate(w["seq_lens"]):
        rows = orc.to_f64(wl.sequence_rows(s, b, int(L), seed=7))
        want = np.einsum("hvr,r->hv", orc.to_f64(w["W_UV"]), rows[:, :s.R].mean(axis=0))
        np.testing.assert_allclose(ref["out"][b], want, rtol=0, atol=1e-12)
        np.testing.assert_allclose(ref["lse"][b], math.log(int(L)), rtol=0, atol=1e-12)


def test_empty_sequence_gives_zero_and_minus_inf():
    w = small_bf16(lens=(0, 5, 0))
    ref = run_ref(w)
    for b in (0, 2):
        assert np.all(ref["out"][b] == 0) and np.all(ref["o_lat"][b] == 0)
        assert np.all(np.isneginf(ref["lse"][b]))
    assert np.all(np.isfinite(ref["out"][1]))


def test_head_permutation_equivariance():
    w = small_bf16()
    ref = run_ref(w)
    perm = np.array([2, 0, 3, 1])
    w2 = dict(w, q_nope=w["q_nope"][:, perm], q_rope=w["q_rope"][:, perm], W_UK=w["W_UK"][perm],
              W_UV=w["W_UV"][perm])
    ref2 = run_ref(w2)
    np.testing.assert_allclose(ref2["out"], ref["out"][:, perm], rtol=0, atol=1e-14)


def test_shared_rope_key_is_the_same_for_every_head():
    """With identical per-head queries and weights, all heads must agree: the rope
    key is one per token, broadcast (GatedMLA, 'Build per-head Q, K and V')."""
    w = small_bf16()
    for k in ("q_nope", "q_rope"):
        w[k][:] = w[k][:, :1]
    for k in ("W_UK", "W_UV"):
        w[k][:] = w[k][:1]
    ref = run_ref(w)
    np.testing.assert_array_equal(ref["out"], np.broadcast_to(ref["out"][:, :1], ref["out"].shape))


def test_rope_key_shift_moves_logits_by_q_dot_shift():
    """Adding a vector u to every cached rope key adds scale*(qr_h . u) to every
    logit of head h: the lse moves by exactly that and the output does not change."""
    w = small_bf16()
    s = w["spec"]
    kv = wl.bf16_bits_to_f32(w["kv_cache"]).copy()
    kv[:, :, s.R + 3] = np.round(kv[:, :, s.R + 3] * 2) / 2      # halves: shifts by 0.5 stay exact
    w["kv_cache"] = wl.f32_to_bf16_bits(kv)
    ref = run_ref(w)
    u = np.zeros(s.Dr, np.float32)
    u[3] = 0.5
    kv[:, :, s.R:] += u
    w2 = dict(w, kv_cache=wl.f32_to_bf16_bits(kv))
    # only exact if the shifted values stay representable: check it
    assert np.array_equal(wl.bf16_bits_to_f32(w2["kv_cache"])[:, :, s.R:], kv[:, :, s.R:])
    ref2 = run_ref(w2)
    shift = w["scale"] * (orc.to_f64(w["q_rope"]) @ u.astype(np.float64))
    np.testing.assert_allclose(ref2["lse"], ref["lse"] + shift, rtol=0, atol=1e-10)
    np.testing.assert_allclose(ref2["out"], ref["out"], rtol=0, atol=1e-10)


# ----------------------------------------------------------------------------- per-step pieces

def test_absorb_q_and_out_proj_match_explicit_sums():
    w = small_bf16(B=2, H=2, R=8, Dr=4, Dn=4, Dv=3, lens=(5, 6), page=4)
    qn, wuk, wuv = orc.to_f64(w["q_nope"]), orc.to_f64(w["W_UK"]), orc.to_f64(w["W_UV"])
    ql = orc.absorb_q(w["q_nope"], w["W_UK"])
    ol = np.arange(2 * 2 * 8, dtype=np.float64).reshape(2, 2, 8) / 7.0
    o = orc.out_proj(ol, w["W_UV"])
    for t in range(2):
        for h in range(2):
            for r in range(8):
                assert abs(ql[t, h, r] - sum(qn[t, h, n] * wuk[h, n, r] for n in range(4))) < 1e-14
            for v in range(3):
                assert abs(o[t, h, v] - sum(wuv[h, v, r] * ol[t, h, r] for r in range(8))) < 1e-13


def _split_parts(w, bounds):
    """Attend over each [lo, hi) token range of every sequence separately."""
    s = w["spec"]
    ql = orc.absorb_q(w["q_nope"], w["W_UK"])
    parts_o, parts_l = [], []
    for lo, hi in bounds:
        o = np.zeros((len(w["seq_lens"]), s.H, s.R))
        l = np.full((len(w["seq_lens"]), s.H), -np.inf)
        for b, L in enumerate(w["seq_lens"]):
            rows = orc.gather_rows(w["kv_cache"], w["block_table"][b], int(L), s.page_size)[lo:min(hi, int(L))]
            for h in range(s.H):
                q = np.concatenate([ql[b, h], orc.to_f64(w["q_rope"][b, h])])
                o[b, h], _, l[b, h] = orc.softmax_attend(q, rows, rows[:, :s.R], w["scale"])
        parts_o.append(o)
        parts_l.append(l)
    return np.stack(parts_o), np.stack(parts_l)


def test_combine_of_splits_equals_unsplit_attention():
    w = small_bf16(lens=(70, 1, 129))
    ref = run_ref(w)
    po, pl = _split_parts(w, [(0, 16), (16, 17), (17, 64), (64, 200)])
    o, lse = orc.combine(po, pl)
    np.testing.assert_allclose(o, ref["o_lat"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref["lse"], rtol=0, atol=1e-12)


def test_combine_closed_forms():
    a = np.array([[1.0, 2.0], [3.0, 4.0]])
    o, lse = orc.combine(a[:, None, :], np.array([[0.5], [0.5]]))
    np.testing.assert_allclose(o[0], [2.0, 3.0])           # equal weights: plain mean
    np.testing.assert_allclose(lse, [0.5 + math.log(2)])
    o, lse = orc.combine(a[:, None, :], np.array([[-np.inf], [1.0]]))
    np.testing.assert_allclose(o[0], [3.0, 4.0])           # empty part has no weight
    o, lse = orc.combine(a[:, None, :], np.array([[-np.inf], [-np.inf]]))
    assert np.all(o == 0) and np.isneginf(lse[0])


# ----------------------------------------------------------------------------- planted mistakes

def _pins_fail(monkeypatch, name, fake):
    monkeypatch.setattr(orc, name, fake)
    failures = 0
    for pin in (lambda: test_oracle_matches_scalar_brute_force("tiny"),
                test_full_causal_equals_torch_sdpa_fp64,
                lambda: test_absorbed_equals_nonabsorbed("paged_bf16"),
                test_single_token_gives_w_uv_c0,
                test_zero_query_gives_uniform_mean):
        try:
            pin()
        except AssertionError:
            failures += 1
    return failures


def test_planted_mistakes_are_caught(monkeypatch):
    good_kv, good_att = orc.reconstruct_kv, orc.softmax_attend

    def no_rope(C, kr, wuk_h, wuv_h):
        K, V = good_kv(C, kr, wuk_h, wuv_h)
        K[:, wuk_h.shape[0]:] = 0.0
        return K, V

    def wrong_scale(q, K, V, scale):
        return good_att(q, K, V, scale * math.sqrt(192.0 / 576.0))

    def values_from_keys(C, kr, wuk_h, wuv_h):
        K, V = good_kv(C, kr, wuk_h, wuv_h)
        return K, K[:, :V.shape[1]]

    def off_by_one_visibility(L, q_len, i):
        return max(0, int(L) - int(q_len) + int(i))

    for name, fake in (("reconstruct_kv", no_rope), ("softmax_attend", wrong_scale),
                       ("reconstruct_kv", values_from_keys), ("visible_len", off_by_one_visibility)):
        with monkeypatch.context() as m:
            assert _pins_fail(m, name, fake) >= 1, name


def test_round_bf16_nearest_even_and_identity_on_bf16_values():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -20, -2.5, 0.0])
    got = orc.round_bf16(x)
    np.testing.assert_array_equal(got, [1.0, 1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7, -2.5, 0.0])
    w = small_bf16()
    v = orc.to_f64(w["kv_cache"])
    np.testing.assert_array_equal(orc.round_bf16(v), v)


def test_bf16_intermediates_variant_stays_near_the_definition():
    """Rounding ql and o_lat to bf16 perturbs the exact result by at most a few bf16
    ulps of the output scale on long contexts (no rounding: identical)."""
    w = small_bf16(lens=(300, 257, 129))
    s = w["spec"]
    args = (w["q_nope"], w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"], w["W_UK"], w["W_UV"],
            w["scale"])
    ref = run_ref(w)
    exact = orc.decode_absorbed(*args, q_len=s.q_len, page_size=s.page_size)
    mixed = orc.decode_absorbed(*args, q_len=s.q_len, page_size=s.page_size, intermediates="bf16")
    np.testing.assert_allclose(exact["out"], ref["out"], rtol=0, atol=1e-10)
    d = np.abs(mixed["out"] - ref["out"])
    assert 0 < d.max() < 2e-3 + 1e-2 * np.abs(ref["out"]).max()
    np.testing.assert_array_equal(mixed["o_lat"], orc.round_bf16(mixed["o_lat"]))
    # only the query rounded: still within the bound at this length, o_lat off the bf16 grid
    qonly = orc.decode_absorbed(*args, q_len=s.q_len, page_size=s.page_size, intermediates="q_lat")
    dq = np.abs(qonly["out"] - ref["out"])
    assert 0 < dq.max() < 2e-3 + 1e-2 * np.abs(ref["out"]).max()
    assert np.any(qonly["o_lat"] != orc.round_bf16(qonly["o_lat"]))


def test_query_only_rounding_is_exact_when_the_query_is_on_the_bf16_grid():
    """With q_nope = 0 the absorbed query is 0, which bf16 holds exactly: rounding only the
    query then changes nothing, and the pipeline equals the non-absorbed definition."""
    w = small_bf16(lens=(70, 5, 129))
    s = w["spec"]
    qn = np.zeros_like(w["q_nope"])
    args = (qn, w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"], w["W_UK"], w["W_UV"], w["scale"])
    exact = orc.decode_nonabsorbed(*args, q_len=s.q_len, page_size=s.page_size)
    qonly = orc.decode_absorbed(*args, q_len=s.q_len, page_size=s.page_size, intermediates="q_lat")
    np.testing.assert_allclose(qonly["out"], exact["out"], rtol=0, atol=1e-10)
    np.testing.assert_allclose(qonly["lse"], exact["lse"], rtol=0, atol=1e-10)


# ----------------------------------------------------------------------------- cache-write prologue

def test_rope_equals_a_complex_rotation():
    """Rotate-half RoPE is multiplication of z_i = x_i + i x_{i+d/2} by exp(i pos theta_i),
    theta_i = base^(-2i/d): checked through numpy's complex arithmetic (another route to
    the same numbers); for d = 2 the plane turns by exactly pos radians."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 64))
    pos = np.array([0, 1, 7, 4096, 131071])
    theta = 10000.0 ** (-2.0 * np.arange(32) / 64)
    z = (x[:, :32] + 1j * x[:, 32:]) * np.exp(1j * pos[:, None] * theta)
    np.testing.assert_allclose(orc.rope(x, pos), np.concatenate([z.real, z.imag], 1), rtol=0, atol=1e-12)
    v = np.array([[0.6, -0.8]])
    for p in (1, 2, 3.5):
        np.testing.assert_allclose(orc.rope(v, np.array([p]))[0],
                                   [0.6 * np.cos(p) + 0.8 * np.sin(p), 0.6 * np.sin(p) - 0.8 * np.cos(p)],
                                   rtol=0, atol=1e-15)


def test_rope_scores_depend_only_on_the_position_difference():
    """The decoupled key's purpose: rope(q, m) . rope(k, n) is a function of m - n."""
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for m, n in [(5, 2), (100, 0), (70000, 65000)]:
        ref = orc.rope(q, np.array(m)) @ orc.rope(k, np.array(n))
        for s in (1, 17, 1000):
            got = orc.rope(q, np.array(m + s)) @ orc.rope(k, np.array(n + s))
            assert abs(got - ref) < 1e-9 * (1 + abs(ref))


def test_rope_composes_keeps_norms_and_is_the_identity_at_zero():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 64))
    a, b = np.array([3, 10, 512, 9000]), np.array([1, 6, 100, 31])
    np.testing.assert_allclose(orc.rope(orc.rope(x, a), b), orc.rope(x, a + b), rtol=0, atol=1e-10)
    np.testing.assert_allclose(np.linalg.norm(orc.rope(x, a), axis=1), np.linalg.norm(x, axis=1), rtol=1e-14)
    np.testing.assert_array_equal(orc.rope(x, np.zeros(4)), x)


def test_rms_norm_matches_torch_and_has_unit_rms():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((6, 512)) * np.array([[1e-3], [1.0], [30.0], [2.0], [0.5], [7.0]])
    gain = rng.standard_normal(512)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (512,), weight=torch.from_numpy(gain), eps=1e-6)
    np.testing.assert_allclose(orc.rms_norm(x, gain, 1e-6), ref.numpy(), rtol=1e-12, atol=1e-12)
    unit = orc.rms_norm(x[1:], np.ones(512), 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(unit ** 2, axis=1)), 1.0, rtol=1e-12)


def test_cache_write_rows_against_scalar_loops():
    """Brute force on a tiny case: the projection, the norm of the latent part and the
    rotation of the shared key written out one element at a time."""
    rng = np.random.default_rng(7)
    T, M, R, Dr = 3, 8, 6, 4
    hidden, W = rng.standard_normal((T, M)), rng.standard_normal((R + Dr, M))
    gain, pos, eps = rng.standard_normal(R), np.array([0, 3, 11]), 1e-6
    got = orc.cache_write_rows(hidden, W, gain, pos, R, eps=eps, rope_base=10000.0)
    for t in range(T):
        f = [sum(hidden[t][m] * W[j][m] for m in range(M)) for j in range(R + Dr)]
        ms = sum(f[j] * f[j] for j in range(R)) / R
        for j in range(R):
            assert abs(got[t][j] - f[j] / math.sqrt(ms + eps) * gain[j]) < 1e-12
        for i in range(Dr // 2):
            th = 10000.0 ** (-2.0 * i / Dr) * pos[t]
            a, b = f[R + i], f[R + Dr // 2 + i]
            assert abs(got[t][R + i] - (a * math.cos(th) - b * math.sin(th))) < 1e-12
            assert abs(got[t][R + Dr // 2 + i] - (a * math.sin(th) + b * math.cos(th))) < 1e-12


def test_token_positions_follow_the_append_convention():
    np.testing.assert_array_equal(orc.token_positions([5, 2, 9], 2), [3, 4, 0, 1, 7, 8])


def test_stored_up_projection_variant_is_exact_on_the_bf16_grid_and_close_otherwise():
    """full_causal(intermediates="kv_bf16") rounds only K_c = C W_UK^T and V = C W_UV^T.
    With weights that pick single latent columns times powers of two, K_c and V are bf16
    values already and the variant equals the definition; with the workload's weights it
    stays within the bf16 rounding of those two products."""
    g = np.random.default_rng(31)
    L, H, R, Dr, Dn, Dv = 37, 3, 32, 8, 8, 8
    C = orc.to_f64(wl.f32_to_bf16_bits(g.standard_normal((L, R)).astype(np.float32)))
    kr = orc.to_f64(wl.f32_to_bf16_bits(g.standard_normal((L, Dr)).astype(np.float32)))
    qn = wl.f32_to_bf16_bits(g.standard_normal((L, H, Dn)).astype(np.float32))
    qr = wl.f32_to_bf16_bits(g.standard_normal((L, H, Dr)).astype(np.float32))
    pick = np.zeros((H, Dn, R))
    for h in range(H):
        for d in range(Dn):
            pick[h, d, g.integers(R)] = 2.0 ** int(g.integers(-3, 3))
    exact = orc.full_causal(C, kr, qn, qr, pick, pick, 0.25)
    var = orc.full_causal(C, kr, qn, qr, pick, pick, 0.25, intermediates="kv_bf16")
    np.testing.assert_array_equal(var, exact)
    W = g.standard_normal((H, Dn, R)) / np.sqrt(R)
    exact = orc.full_causal(C, kr, qn, qr, W, W, 0.25)
    var = orc.full_causal(C, kr, qn, qr, W, W, 0.25, intermediates="kv_bf16")
    assert not np.array_equal(var, exact)
    assert np.max(np.abs(var - exact)) < 0.05 * np.max(np.abs(exact))
