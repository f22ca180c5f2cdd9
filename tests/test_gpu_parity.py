"""GPU parity: every libmla.so kernel against the fp64 oracle on the same seeded inputs.

Tolerances (from the arithmetic, as the benchmark spec of this path sets them):
bf16 storage with fp32 accumulation: |got - ref| <= 2e-3 + 1e-2 |ref| elementwise;
fp32 storage: |got - ref| <= 1e-5. Cache append is bit-exact.

Small cases span several pages and a ragged tail and include empty sequences; both
kernel policies (SIMT CUDA cores, tcgen05 tensor cores) run where the geometry allows.
The full-size workloads run in the launch configuration the benchmark times and every
(query, head) output is checked: against the fp64 absorbed pipeline for the decode
workloads (plus a non-absorbed sample holding the longest sequence), against the full
causal forward for the multi-token chunk.
"""
import math

import numpy as np
import pytest
import torch

import mla_latent_kv_46_b200 as mla
from mla_latent_kv_46_b200 import decoder as dec
from inputs import workloads as wl
from oracle import mla_oracle as orc

pytestmark = pytest.mark.gpu

POLICIES = {"simt": mla.MLA_POLICY_SIMT, "tcgen05": mla.MLA_POLICY_TCGEN05}


@pytest.fixture(autouse=True)
def _policy_reset():
    yield
    mla.mla_set_policy(mla.MLA_POLICY_AUTO)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got, ref, fp32, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    ninf_r, ninf_g = np.isneginf(ref), np.isneginf(got)
    assert np.array_equal(ninf_r, ninf_g), f"{what}: -inf pattern differs"
    m = ~ninf_r
    err = np.abs(got[m] - ref[m])
    bound = 1e-5 if fp32 else 2e-3 + 1e-2 * np.abs(ref[m])
    bad = err > bound
    assert not np.any(np.isnan(got[m])), f"{what}: NaN in output"
    assert not np.any(bad), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; max err "
                             f"{err.max():.3e}, worst ratio {(err / bound).max():.2f}")


def small_spec(H=64, q_len=1, R=512, Dr=64, Dn=128, Dv=128, dtype="bf16", page=64, noise=0.0):
    return wl.WorkloadSpec(name=f"small_h{H}_q{q_len}", B=0, H=H, R=R, Dr=Dr, Dn=Dn, Dv=Dv, q_len=q_len,
                           dtype=dtype, seq_len=None, w_std=1.0 / math.sqrt(R), page_size=page,
                           logit_noise_std=noise)


# lengths: single token, one short of a page, exact page, one over, several pages
# with a ragged tail, and an empty sequence
SMALL_LENS = [1, 63, 64, 65, 333, 0]


def make_case(spec, lens, seed=11, sms=None):
    w = wl.make(spec, seed=seed, seq_lens=lens)
    step = dec.DecodeStep(w, sms=sms)
    return w, step


def run_policy(policy):
    mla.mla_set_policy(POLICIES[policy])


# ----------------------------------------------------------------------------- a2: cache append

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_cache_append_bit_exact(dtype):
    spec = small_spec(H=64, q_len=3, dtype=dtype) if dtype == "bf16" else \
        small_spec(H=4, q_len=3, R=32, Dr=16, Dn=16, Dv=16, dtype="f32")
    lens = [3, 70, 130, 64]
    full = wl.make(spec, seed=5, seq_lens=lens)
    empty = wl.make(spec, seed=5, seq_lens=lens, new_rows_in_cache=False)
    step = dec.DecodeStep(empty)
    step.append()
    torch.cuda.synchronize()
    mla.mla_check_status()
    got = step.kv.view(torch.int16).cpu().numpy().view(np.uint16) if dtype == "bf16" else step.kv.cpu().numpy()
    want = orc.cache_append(empty["kv_cache"], empty["block_table"], empty["seq_lens"], empty["new_ckr"],
                            spec.q_len, spec.page_size)
    assert np.array_equal(got, want)
    assert np.array_equal(want, full["kv_cache"])


# ----------------------------------------------------------------------------- a1 / a7

# (tokens: up to 64 rows the tensor-core absorption cuts each head's 512 columns into four
# blocks, above that into two; 300 rows: three 128-row tiles with a ragged tail)
PROJ_CASES = [("bf16_h64", "simt"), ("bf16_h64", "tcgen05"), ("bf16_h128", "simt"), ("bf16_h128", "tcgen05"),
              ("bf16_h64_t300", "tcgen05"), ("bf16_h64_t64", "tcgen05"), ("bf16_h128_t65", "tcgen05"),
              ("bf16_h64_t1", "tcgen05"), ("f32_tiny", "simt")]


def proj_case(case):
    if case == "f32_tiny":
        return wl.make("tiny_fp32")
    H = 128 if case.startswith("bf16_h128") else 64
    n = int(case.rsplit("_t", 1)[1]) if "_t" in case else 37
    return wl.make(small_spec(H=H), seed=3, seq_lens=[5] * n)


@pytest.mark.parametrize("case,policy", PROJ_CASES)
def test_absorb_q_matches_oracle(case, policy):
    w = proj_case(case)
    step = dec.DecodeStep(w)
    run_policy(policy)
    step.absorb()
    torch.cuda.synchronize()
    ref = orc.absorb_q(w["q_nope"], w["W_UK"])
    assert_close(host(step.q_lat), ref, w["spec"].dtype == "f32", "q_lat")


@pytest.mark.parametrize("case,policy", PROJ_CASES)
def test_out_proj_matches_oracle(case, policy):
    w = proj_case(case)
    spec = w["spec"]
    step = dec.DecodeStep(w)
    ol = wl.latent_outputs(spec, step.T, seed=4, fp32=True)   # o_lat is fp32 for every dtype
    step.o_lat.copy_(torch.from_numpy(ol).to(step.device))
    run_policy(policy)
    step.project()
    torch.cuda.synchronize()
    ref = orc.out_proj(ol, w["W_UV"])
    got = host(step.out)
    assert_close(got, ref, spec.dtype == "f32", "out")
    if spec.dtype == "bf16":
        # o_lat enters in full: only the bf16 store of `out` rounds (half a bf16 ulp, 2^-9
        # relative); o_lat cut to bf16 first would add ~1e-3 absolute here (512 terms of
        # |w| ~ 0.04 times |o| ~ 0.1 with 2^-9 relative errors)
        err = np.abs(got - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2e-5), float((err - 2.0 ** -8 * np.abs(ref)).max())


# ----------------------------------------------------------------------------- a3-a6: attention (+ combine)

def attention_case(policy, H, q_len, lens, sms, noise=0.0):
    run_policy(policy)
    spec = small_spec(H=H, q_len=q_len, noise=noise)
    w, step = make_case(spec, lens, sms=sms)
    ql = wl.latent_queries(spec, step.T, seed=9)
    step.q_lat.copy_(dec.to_torch(ql, step.device))
    step.attend()
    step.combine()
    torch.cuda.synchronize()
    mla.mla_check_status()
    ref = orc.attend_latent(ql, w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"], w["scale"],
                            q_len=q_len, page_size=spec.page_size)
    assert_close(host(step.o_lat), ref["o_lat"], False, "o_lat")
    assert_close(host(step.lse), ref["lse"], False, "lse")
    return step


@pytest.mark.parametrize("policy", ["simt", "tcgen05"])
@pytest.mark.parametrize("H", [64, 128])
@pytest.mark.parametrize("sms", [148, 9])
def test_decode_attention_matches_oracle(policy, H, sms):
    # with few slots a 2000-token sequence is cut between slots: partial outputs + combine
    step = attention_case(policy, H, 1, SMALL_LENS + ([2000] if sms == 9 else []), sms)
    if sms == 9:
        assert step.info.num_parts > 0   # the combine ran


@pytest.mark.parametrize("policy,H,lens,sms,warps", [
    ("tcgen05", 64, [9000, 40], 148, 8),
    ("tcgen05", 64, [3000, 40], 30, 4),
    ("tcgen05", 128, [9000, 40, 700], 148, 8),
    ("simt", 64, [3000, 40, 0], 30, 8),
])
def test_many_parts_per_query_combine_matches_oracle(policy, H, lens, sms, warps):
    """A few long queries cut into many parts: the combine spreads one (query, head)'s
    parts over 4 or 8 warps (chosen from parts per query) and merges the warps' partial
    sums; the short queries are single-unit items it skips."""
    step = attention_case(policy, H, 1, lens, sms)
    per_item = step.info.num_parts // step.info.num_items
    assert (8 if per_item >= 8 else 4 if per_item >= 3 else 1) == warps


@pytest.mark.parametrize("policy", ["simt", "tcgen05"])
def test_causal_chunk_attention_matches_oracle(policy):
    attention_case(policy, 64, 5, [70, 5, 129], 6)


@pytest.mark.parametrize("sms", [148, 9])
@pytest.mark.parametrize("q_len", [2, 4])
def test_paired_token_attention_matches_oracle(q_len, sms):
    """64 heads, several new tokens: the tensor-core path serves two consecutive tokens
    of a sequence per 2-CTA cluster (128 rows); the two tokens see different lengths,
    page ranges are cut between slots, and one sequence is shorter than a page."""
    step = attention_case("tcgen05", 64, q_len, [300, 64, q_len, 1000, 130], sms)
    assert step.info.head_groups == 2
    if sms == 9:
        assert step.info.num_parts > 0


@pytest.mark.parametrize("sms", [148, 20])
@pytest.mark.parametrize("q_len", [2, 4])
def test_multi_token_128_heads_attention_matches_oracle(q_len, sms):
    """128 heads, several new tokens per sequence: each token's units sit on a slot block
    of their own with the same page ranges as the other tokens' (the kernel clips a
    unit to the pages its token sees), so some units of the earlier tokens are empty."""
    step = attention_case("tcgen05", 128, q_len, [300, 65, q_len, 1000, 130, 129], sms)
    assert step.info.head_groups == 2
    if sms == 20:
        assert step.info.num_parts > 0


@pytest.mark.parametrize("policy", ["simt", "tcgen05"])
def test_attention_with_large_logit_offsets(policy):
    """Per-token logit noise of std 4 (the long-context workload's stress): the
    reference maximum moves several times inside a unit."""
    attention_case(policy, 64, 1, [1000, 777], 3, noise=4.0)


def test_decode_fp32_tiny_matches_oracle():
    w = wl.make("tiny_fp32")
    spec = w["spec"]
    step = dec.DecodeStep(w)
    ql = wl.latent_queries(spec, step.T, seed=9)
    step.q_lat.copy_(dec.to_torch(ql, step.device))
    step.attend()
    step.combine()
    torch.cuda.synchronize()
    ref = orc.attend_latent(ql, w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"], w["scale"])
    assert_close(host(step.o_lat), ref["o_lat"], True, "o_lat")
    assert_close(host(step.lse), ref["lse"], True, "lse")


def test_tcgen05_policy_rejects_unsupported_dims():
    mla.mla_set_policy(mla.MLA_POLICY_TCGEN05)
    w = wl.make(small_spec(H=32), seed=1, seq_lens=[10, 20])
    step = dec.DecodeStep(w)
    with pytest.raises(mla.MlaError) as e:
        step.attend()
    assert e.value.status == mla._binding.MLA_ERR_UNSUPPORTED


# ----------------------------------------------------------------------------- whole step vs the definition

@pytest.mark.parametrize("policy", ["simt", "tcgen05"])
@pytest.mark.parametrize("H,q_len,lens,sms", [(64, 1, SMALL_LENS, 148), (128, 1, SMALL_LENS, 7),
                                              (64, 4, [200, 4, 65], 9)])
def test_whole_step_matches_oracle(policy, H, q_len, lens, sms):
    """append -> absorb -> attention (policy under test) -> combine -> projection.

    Against the oracle of the same pipeline (the absorbed query stored in bf16, all else
    fp64; o_lat stays fp32) at the bf16 tolerance everywhere, and against the exact
    non-absorbed definition on every query that sees at least 17 tokens. (With only a
    few visible tokens of comparable weight the bf16 store of the absorbed query alone
    moves `out` by more than the tolerance.)"""
    spec = small_spec(H=H, q_len=q_len)
    empty = wl.make(spec, seed=21, seq_lens=lens, new_rows_in_cache=False)
    full = wl.make(spec, seed=21, seq_lens=lens)
    step = dec.DecodeStep(empty, sms=sms)
    step.append()
    step.absorb()
    run_policy(policy)
    step.replan(step.seq_lens_host)   # the split plan depends on the kernel policy
    step.attend()
    step.combine()
    mla.mla_set_policy(mla.MLA_POLICY_AUTO)
    step.project()
    torch.cuda.synchronize()
    mla.mla_check_status()
    args = (full["q_nope"], full["q_rope"], full["kv_cache"], full["block_table"], full["seq_lens"],
            full["W_UK"], full["W_UV"], full["scale"])
    mixed = orc.decode_absorbed(*args, q_len=q_len, page_size=spec.page_size, intermediates="q_lat")
    out, lse = host(step.out), host(step.lse)
    assert_close(out, mixed["out"], False, "out vs bf16-query pipeline oracle")
    assert_close(lse, mixed["lse"], False, "lse vs bf16-query pipeline oracle")
    exact = orc.decode_nonabsorbed(*args, q_len=q_len, page_size=spec.page_size)
    vis = np.array([max(0, L - q_len + i + 1) for L in lens for i in range(q_len)])
    seen = vis >= 17
    assert seen.any()
    assert_close(out[seen], exact["out"][seen], False, "out vs definition")


@pytest.mark.parametrize("H", [64, 128])
def test_pipelined_end_to_end_steps_match_device_step(H):
    """The pipelined end-to-end runner (host inputs, copies overlapping the neighbouring
    steps' kernels, two buffer sets) returns, step after step, exactly the output of the
    device-resident step."""
    spec = small_spec(H=H)
    w = wl.make(spec, seed=5, seq_lens=[900, 65, 1, 640, 2000])
    step = dec.DecodeStep(w, sms=9)
    step.run()
    torch.cuda.synchronize()
    want = step.out.view(torch.int16).cpu().clone()
    hostin = dec.HostInputs(step, w)
    pipe = dec.PipelinedE2E(step, hostin)
    for k in range(5):
        ev = pipe.enqueue()
        if k >= 1:
            prev = pipe.outs[(k - 1) & 1]
            pipe.out_read[(k - 1) & 1].synchronize()
            assert torch.equal(prev, want), f"step {k - 1}"
    ev.synchronize()
    mla.mla_check_status()
    assert torch.equal(pipe.outs[4 & 1], want)


def test_whole_step_tiny_fp32_matches_definition():
    w = wl.make("tiny_fp32")
    step = dec.DecodeStep(w)
    step.run()
    torch.cuda.synchronize()
    ref = orc.decode_nonabsorbed(w["q_nope"], w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"],
                                 w["W_UK"], w["W_UV"], w["scale"])
    assert_close(host(step.out), ref["out"], True, "out")


def test_incremental_gpu_decode_equals_full_causal_tiny():
    """Decode at every prefix 1..64 of the tiny fp32 sequence equals the oracle's full
    causal forward (the ticket's incremental-vs-full acceptance, atol 1e-5)."""
    s = wl.spec_with("tiny_fp32", all_query_positions=True)
    rows = wl.sequence_rows(s, 0, 64, seed=0)
    qn, qr = wl.queries_of(s, 0, 64, seed=0)
    wuk, wuv = wl.weights_of(s, seed=0)
    full = orc.full_causal(orc.to_f64(rows[:, :s.R]), orc.to_f64(rows[:, s.R:]), qn, qr, wuk, wuv, s.scale)
    for n in (1, 2, 17, 63, 64):
        w = dict(spec=wl.spec_with("tiny_fp32"), kv_cache=np.zeros((1, 64, s.row), np.float32),
                 block_table=np.zeros((1, 1), np.int32), seq_lens=np.array([n], np.int32), q_nope=qn[n - 1:n],
                 q_rope=qr[n - 1:n], W_UK=wuk, W_UV=wuv, new_ckr=rows[n - 1:n], num_pages=1, scale=s.scale)
        w["kv_cache"][0, :n] = rows[:n]
        step = dec.DecodeStep(w)
        step.run(append=False)
        torch.cuda.synchronize()
        assert_close(host(step.out)[0], full[n - 1], True, f"prefix {n}")


# ----------------------------------------------------------------------------- full-size workloads, every output

FULL = ["kimi_h64_b64_l4096", "deepseek_h128_b128_ragged", "longctx_h64_b4_l131072",
        "causal_chunk_h64_b8_2048p256", "mtp2_h128_b64_ragged"]


def _full_step(name):
    """The whole step (append included) at full size, in the launch configuration the
    benchmark times; returns the workload (cache as after the append) and host outputs."""
    spec = wl.WORKLOADS[name]
    w = wl.make(spec, seed=0, new_rows_in_cache=False)
    step = dec.DecodeStep(w)
    step.run(append=True)
    torch.cuda.synchronize()
    mla.mla_check_status()
    out, lse, o_lat = host(step.out), host(step.lse), host(step.o_lat)
    del step
    torch.cuda.empty_cache()
    return wl.make(spec, seed=0), out, lse, o_lat


@pytest.mark.parametrize("name", FULL[:3] + FULL[4:])
def test_full_size_workload_every_output(name):
    """Every (query, head) of the workload against the fp64 absorbed pipeline with the
    absorbed query rounded to bf16 as the kernels store it (o_lat stays fp32): out, lse
    and o_lat, elementwise at the bf16 bound. That oracle is pinned to the non-absorbed definition
    (tests/test_oracle.py); here the definition itself is checked too, on a sample that
    always holds the longest sequence (for the long-context workload: 131,072 tokens
    with per-token logit noise of std 4)."""
    spec = wl.WORKLOADS[name]
    full, out, lse, o_lat = _full_step(name)
    args = (full["q_nope"], full["q_rope"], full["kv_cache"], full["block_table"], full["seq_lens"],
            full["W_UK"], full["W_UV"], full["scale"])
    mixed = orc.decode_absorbed(*args, q_len=spec.q_len, page_size=spec.page_size, intermediates="q_lat")
    assert_close(out, mixed["out"], False, f"{name} out, every query and head")
    assert_close(lse, mixed["lse"], False, f"{name} lse, every query and head")
    assert_close(o_lat, mixed["o_lat"], False, f"{name} o_lat, every query and head")
    lens = np.asarray(full["seq_lens"])
    rng = np.random.default_rng(123)
    seqs = sorted({int(np.argmax(lens))} | set(rng.choice(len(lens), size=min(2, len(lens)),
                                                          replace=False).tolist()))
    heads = sorted(rng.choice(spec.H, size=2, replace=False).tolist())
    ref = orc.decode_nonabsorbed(*args, q_len=spec.q_len, page_size=spec.page_size, seqs=seqs, heads=heads)
    for b in seqs:
        for h in heads:
            assert_close(out[b, h], ref["out"][b, h], False, f"{name} out vs definition b={b} h={h}")
            assert_close(lse[b, h], ref["lse"][b, h], False, f"{name} lse vs definition b={b} h={h}")


def test_full_size_causal_chunk_every_output():
    """All 8 sequences x 64 heads x 256 new tokens of the multi-token causal chunk
    against the oracle's full causal forward over all 2304 positions (the definition:
    rebuilt per-head K and V, causal softmax), the last 256 rows of each."""
    name = FULL[3]
    spec = wl.WORKLOADS[name]
    full, out, lse, o_lat = _full_step(name)
    for b in range(len(full["seq_lens"])):
        L = int(full["seq_lens"][b])
        rows = orc.to_f64(wl.sequence_rows(spec, b, L, seed=0))
        qn, qr = full["all_queries"][b]
        ref = orc.full_causal(rows[:, :spec.R], rows[:, spec.R:], qn, qr, full["W_UK"], full["W_UV"],
                              full["scale"])
        got = out[b * spec.q_len:(b + 1) * spec.q_len]
        assert_close(got, ref[L - spec.q_len:], False, f"{name} b={b}, every new token and head")
    assert np.all(np.isfinite(lse))


# ----------------------------------------------------------------------------- failure reporting

@pytest.mark.parametrize("H,q_len", [(64, 1), (128, 1), (64, 2)])
def test_bad_page_id_is_reported_not_faulted(H, q_len):
    """A block-table entry outside the pool is skipped (the tile reads as zeros) and
    reported through the status word; the single-CTA kernel (64 heads), the cluster
    kernel (128 heads) and the cluster kernel with paired query tokens."""
    w = wl.make(small_spec(H=H, q_len=q_len), seed=2, seq_lens=[130, 64])
    w["block_table"][1, 0] = 10_000          # outside the pool
    step = dec.DecodeStep(w)
    step.run(append=False)
    torch.cuda.synchronize()
    with pytest.raises(mla.MlaError) as e:
        mla.mla_check_status()
    assert e.value.status == mla._binding.MLA_ERR_INVALID
    mla.mla_check_status()                   # cleared


@pytest.mark.parametrize("H,q_len", [(64, 1), (128, 1), (64, 2)])
def test_dropped_page_load_times_out_and_context_stays_usable(H, q_len):
    """Fault injection without a GPU fault: the first CTA skips one page load (testing
    hook), its waits run out after a short bound, the kernel stops and the status word
    reports MLA_ERR_TIMEOUT; afterwards the same context decodes correctly."""
    spec = small_spec(H=H, q_len=q_len)
    lens = [700, 300, 129]
    w = wl.make(spec, seed=4, seq_lens=lens)
    step = dec.DecodeStep(w, sms=4)
    ql = wl.latent_queries(spec, step.T, seed=9)
    step.q_lat.copy_(dec.to_torch(ql, step.device))
    mla.mla_set_wait_timeout_ns(20_000_000)       # 20 ms
    mla.mla_debug_drop_page_load(2)
    try:
        step.attend()
        torch.cuda.synchronize()
        with pytest.raises(mla.MlaError) as e:
            mla.mla_check_status()
        assert e.value.status == mla._binding.MLA_ERR_TIMEOUT
    finally:
        mla.mla_debug_drop_page_load(-1)
        mla.mla_set_wait_timeout_ns(2_000_000_000)
    mla.mla_check_status()                         # cleared
    step.attend()
    step.combine()
    torch.cuda.synchronize()
    mla.mla_check_status()
    ref = orc.attend_latent(ql, w["q_rope"], w["kv_cache"], w["block_table"], w["seq_lens"], w["scale"],
                            q_len=q_len, page_size=spec.page_size)
    assert_close(host(step.o_lat), ref["o_lat"], False, "o_lat after the injected timeout")


def test_check_status_reports_a_test_hook_left_set():
    """The drop-page hook is test-only: while it is set, mla_check_status fails even
    though no kernel reported anything, and passes again once it is switched off."""
    mla.mla_check_status()
    mla.mla_debug_drop_page_load(0)
    try:
        with pytest.raises(mla.MlaError) as e:
            mla.mla_check_status()
        assert e.value.status == mla._binding.MLA_ERR_INVALID
        assert "mla_debug_drop_page_load" in mla.mla_last_error()
    finally:
        mla.mla_debug_drop_page_load(-1)
    mla.mla_check_status()


@pytest.mark.parametrize("name", ["deepseek_h128_b128_ragged", "causal_chunk_h64_b8_2048p256"])
def test_decode_is_deterministic(name):
    """Two runs of the same step give bitwise equal outputs (no atomics, fixed order)."""
    spec = wl.WORKLOADS[name]
    lens = wl.seq_lens_of(spec, 0)[:16]
    w = wl.make(spec, seed=0, seq_lens=lens)
    step = dec.DecodeStep(w)
    outs = []
    for _ in range(2):
        step.run(append=True)
        torch.cuda.synchronize()
        outs.append((step.out.clone(), step.lse.clone()))
    mla.mla_check_status()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


# ----------------------------------------------------------------------------- cache-write prologue

def _cache_write_case(lens, q_len, M, seed=31, with_q=True):
    spec = small_spec(H=128, q_len=q_len)
    w = wl.make(spec, seed=seed, seq_lens=lens, new_rows_in_cache=False)
    step = dec.DecodeStep(w)
    T = step.T
    pin = wl.prologue_inputs(spec, T, M, seed=seed)
    hidden, W, gain = (dec.to_torch(pin[k], step.device) for k in ("hidden", "W_DKV", "kv_gain"))
    before = step.kv.view(torch.int16).cpu().numpy()      # bit patterns
    q0 = host(step.q_rope)
    ws_bytes = mla.mla_cache_write_workspace_size(T, M)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=step.device)
    mla.mla_cache_write(hidden, W, gain, M, step.kv, step.block_table, step.seq_lens, step.B, q_len, step.max_pages,
                        step.num_pages, step.q_rope if with_q else None, 1e-6, 10000.0, ws, ws_bytes, step.dims)
    torch.cuda.synchronize()
    mla.mla_check_status()
    pos = orc.token_positions(lens, q_len)
    rows = orc.cache_write_rows(pin["hidden"], pin["W_DKV"], pin["kv_gain"], pos, spec.R, eps=1e-6)
    after = step.kv.view(torch.int16).cpu().numpy()
    bt = np.asarray(w["block_table"])
    written = np.zeros(after.shape[:2], bool)
    for t, p in enumerate(pos):
        if p < 0:
            continue
        b = t // q_len
        pg, r = int(bt[b][p // 64]), p % 64
        written[pg, r] = True
        got = orc.to_f64(after[pg, r].view(np.uint16))
        assert_close(got, rows[t], False, f"cache row of token {t} (position {p})")
    np.testing.assert_array_equal(after[~written], before[~written])   # nothing else touched
    if with_q:
        qr = orc.rope(q0, pos[:, None])
        assert_close(host(step.q_rope), qr, False, "q_rope turned in place")
    return rows


@pytest.mark.parametrize("q_len,lens", [(1, [70, 5, 129, 1]), (2, [70, 2, 129]), (4, [300, 4, 65])])
def test_cache_write_matches_oracle(q_len, lens):
    """Down projection, kv_rmsnorm of the latent, rotary shared key, append: the rows the
    prologue writes against the oracle's, at the bf16 bound, and every other cache row
    unchanged; the query's rope part turned in place."""
    _cache_write_case(lens, q_len, M=1024)


def test_cache_write_at_model_width_and_long_positions():
    """Hidden width 7168 (112 K blocks) and positions up to 131071, where the lowest
    frequency's angle is large: every written row against the oracle."""
    _cache_write_case([131072, 4096, 70000, 1], 1, M=7168)
