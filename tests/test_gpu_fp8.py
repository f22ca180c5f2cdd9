"""GPU parity of the 8-bit (E4M3) cache path against the fp64 oracle (oracle/fp8.py).

Quantisation (bulk rows and the append) is compared bit for bit: codes and scale bytes.
Attention over the 8-bit cache is compared with the oracle's attention over the exact
dequantised values (code * 2^k in float64) at the bf16 bound 2e-3 + 1e-2 |ref|: the
kernel scores the codes with the query split into two E4M3 pieces (exact for bf16
queries up to elements below 2^-17 of the row's largest) and sums values widened to bf16
exactly, so its arithmetic matches the bf16 path's on the same values. Every cache the
kernel reads here was quantised by the oracle, never by the library.
"""
import math

import numpy as np
import pytest
import torch

import mla_latent_kv_46_b200 as mla
from mla_latent_kv_46_b200 import decoder as dec
from inputs import workloads as wl
from oracle import fp8
from oracle import mla_oracle as orc

from test_gpu_parity import SMALL_LENS, assert_close, host, small_spec

pytestmark = pytest.mark.gpu


def quantised(w, chunk=32768):
    """The workload with its cache pool quantised by the oracle: kv_codes, kv_scales and
    the dequantised pool the oracle attends over (float32, which holds code * 2^k exactly),
    worked in chunks of rows."""
    P, ps, row = w["kv_cache"].shape
    flat = w["kv_cache"].reshape(P * ps, row)
    codes = np.empty((P * ps, row), np.uint8)
    scales = np.empty(P * ps, np.uint8)
    deq = np.empty((P * ps, row), np.float32)
    for a in range(0, P * ps, chunk):
        c, s = fp8.quantise_rows(orc.to_f64(flat[a:a + chunk]))
        codes[a:a + chunk], scales[a:a + chunk] = c, s
        deq[a:a + chunk] = fp8.dequantise_rows(c, s)
    return dict(w, kv_codes=codes.reshape(P, ps, row), kv_scales=scales.reshape(P, ps),
                kv_deq=deq.reshape(P, ps, row))


def edge_rows():
    """bf16 rows that exercise the rounding: exact ties after scaling, saturation at the
    top scale, subnormal codes, a zero row, tiny (bf16-subnormal) and huge rows."""
    rows = []
    for k in (-9, 0, 3):
        r = np.zeros(576, np.float32)
        r[0] = 448.0 * 2.0 ** k                           # the row's scale is exactly 2^k
        ties = np.array([1.0625, 1.1875, 3 * 2.0 ** -10, 2.0 ** -10, -5 * 2.0 ** -10, 17.0, 19.0, 200.0])
        r[1:1 + len(ties)] = ties * 2.0 ** k
        r[20:40] = np.linspace(-3, 3, 20) * 2.0 ** (k - 12)  # subnormal codes
        rows.append(r)
    rows.append(np.zeros(576, np.float32))
    big = np.full(576, 3.0e4, np.float32)
    big[0] = 1e9                                          # beyond 448 * 2^7: k = 7, saturates
    rows.append(big)
    rows.append(np.full(576, 1e-39, np.float32))          # subnormal in bf16
    rows.append(-np.linspace(1e-3, 2.0, 576).astype(np.float32))
    return wl.f32_to_bf16_bits(np.stack(rows))


def test_quantize_rows_bit_exact():
    g = np.random.default_rng(21)
    rnd = wl.f32_to_bf16_bits((g.standard_normal((500, 576)) * np.exp2(g.uniform(-20, 12, (500, 1))))
                              .astype(np.float32))
    rows = np.concatenate([edge_rows(), rnd])
    n = rows.shape[0]
    d = mla.dims_of(small_spec(H=64))
    src = dec.to_torch(rows, "cuda")
    codes = torch.full((n, 576), 0x55, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(n, dtype=torch.uint8, device="cuda")
    mla.mla_quantize_rows_fp8(src, codes, scales, n, d)
    torch.cuda.synchronize()
    want_c, want_s = fp8.quantise_rows(orc.to_f64(rows))
    assert np.array_equal(scales.cpu().numpy(), want_s)
    got_c = codes.cpu().numpy()
    bad = np.argwhere(got_c != want_c)
    assert bad.size == 0, (f"{len(bad)} codes differ; first at {bad[:3].tolist()}: got "
                           f"{got_c[tuple(bad[0])]:#04x} want {want_c[tuple(bad[0])]:#04x}")


def test_cache_append_fp8_bit_exact():
    spec = small_spec(H=64, q_len=3)
    lens = [3, 70, 130, 64, 2]
    empty = wl.make(spec, seed=5, seq_lens=lens, new_rows_in_cache=False)
    step = dec.DecodeStep(dict(empty, kv_codes=np.zeros(empty["kv_cache"].shape, np.uint8),
                               kv_scales=np.zeros(empty["kv_cache"].shape[:2], np.uint8)), cache="fp8")
    step.append()
    torch.cuda.synchronize()
    mla.mla_check_status()
    P, ps, row = empty["kv_cache"].shape
    placed = orc.cache_append(np.zeros_like(empty["kv_cache"]), empty["block_table"], empty["seq_lens"],
                              empty["new_ckr"], spec.q_len, spec.page_size)
    written = np.zeros((P, ps), bool)
    for b, L in enumerate(lens):
        for i in range(spec.q_len):
            pos = L - spec.q_len + i
            if pos >= 0:
                written[empty["block_table"][b, pos // ps], pos % ps] = True
    want_c, want_s = fp8.quantise_rows(orc.to_f64(placed).reshape(P * ps, row))
    want_c = np.where(written.reshape(-1, 1), want_c, 0).reshape(P, ps, row)
    want_s = np.where(written.reshape(-1), want_s, 0).reshape(P, ps)
    assert np.array_equal(step.kv_scales.cpu().numpy(), want_s)
    assert np.array_equal(step.kv_codes.cpu().numpy(), want_c)


def fp8_attention_case(H, q_len, lens, sms, noise=0.0):
    spec = small_spec(H=H, q_len=q_len, noise=noise)
    w = quantised(wl.make(spec, seed=11, seq_lens=lens))
    step = dec.DecodeStep(w, sms=sms, cache="fp8")
    ql = wl.latent_queries(spec, step.T, seed=9)
    step.q_lat.copy_(dec.to_torch(ql, step.device))
    step.attend()
    step.combine()
    torch.cuda.synchronize()
    mla.mla_check_status()
    ref = orc.attend_latent(ql, w["q_rope"], w["kv_deq"], w["block_table"], w["seq_lens"], w["scale"],
                            q_len=q_len, page_size=spec.page_size)
    assert_close(host(step.o_lat), ref["o_lat"], False, "o_lat (8-bit cache)")
    assert_close(host(step.lse), ref["lse"], False, "lse (8-bit cache)")
    return step


@pytest.mark.parametrize("H", [64, 128])
@pytest.mark.parametrize("sms", [148, 9])
def test_fp8_decode_matches_oracle(H, sms):
    step = fp8_attention_case(H, 1, SMALL_LENS + ([2000] if sms == 9 else []), sms)
    if sms == 9:
        assert step.info.num_parts > 0


@pytest.mark.parametrize("H,q_len", [(64, 2), (64, 5), (128, 2)])
def test_fp8_decode_several_tokens_matches_oracle(H, q_len):
    step = fp8_attention_case(H, q_len, [300, 64, q_len, 1000, 130], 20)
    assert step.info.head_groups == 2


def test_fp8_decode_large_logit_offsets():
    fp8_attention_case(64, 1, [1000, 777], 3, noise=4.0)


def test_fp8_and_bf16_paths_agree_on_representable_caches():
    """A bf16 cache whose values are exactly code * 2^k: both decode paths attend over the
    same numbers, so their outputs agree to the bf16 bound."""
    spec = small_spec(H=128)
    w = quantised(wl.make(spec, seed=4, seq_lens=[500, 64, 1]))
    wb = dict(w, kv_cache=wl.f32_to_bf16_bits(w["kv_deq"].astype(np.float32)))
    ql = dec.to_torch(wl.latent_queries(spec, 3, seed=2), "cuda")
    outs = []
    for step in (dec.DecodeStep(w, cache="fp8"), dec.DecodeStep(wb)):
        step.q_lat.copy_(ql)
        step.attend()
        step.combine()
        torch.cuda.synchronize()
        outs.append((host(step.o_lat), host(step.lse)))
    assert_close(outs[0][0], outs[1][0], False, "o_lat fp8 vs bf16")
    assert_close(outs[0][1], outs[1][1], False, "lse fp8 vs bf16")


@pytest.mark.parametrize("name", ["kimi_h64_b64_l4096", "deepseek_h128_b128_ragged"])
def test_full_size_fp8_every_output(name):
    """The whole step at full size on the 8-bit cache (the new rows appended by
    mla_cache_append_fp8, every other row quantised by the oracle), every (query, head):
    out, lse and o_lat against the fp64 absorbed pipeline over the dequantised cache."""
    spec = wl.WORKLOADS[name]
    full = quantised(wl.make(spec, seed=0))
    # the new rows' slots start out wrong (code 448, the largest scale): the append must
    # overwrite them
    codes, scales = full["kv_codes"].copy(), full["kv_scales"].copy()
    for b, L in enumerate(full["seq_lens"]):
        for i in range(spec.q_len):
            pos = int(L) - spec.q_len + i
            page = full["block_table"][b, pos // spec.page_size]
            codes[page, pos % spec.page_size] = 0x7E
            scales[page, pos % spec.page_size] = 134
    step = dec.DecodeStep(dict(full, kv_codes=codes, kv_scales=scales), cache="fp8")
    step.run(append=True)
    torch.cuda.synchronize()
    mla.mla_check_status()
    assert np.array_equal(step.kv_codes.cpu().numpy(), full["kv_codes"])
    assert np.array_equal(step.kv_scales.cpu().numpy(), full["kv_scales"])
    out, lse, o_lat = host(step.out), host(step.lse), host(step.o_lat)
    del step
    torch.cuda.empty_cache()
    args = (full["q_nope"], full["q_rope"], full["kv_deq"], full["block_table"], full["seq_lens"],
            full["W_UK"], full["W_UV"], full["scale"])
    ref = orc.decode_absorbed(*args, q_len=spec.q_len, page_size=spec.page_size, intermediates="q_lat")
    assert_close(out, ref["out"], False, f"{name} out (8-bit cache)")
    assert_close(lse, ref["lse"], False, f"{name} lse (8-bit cache)")
    assert_close(o_lat, ref["o_lat"], False, f"{name} o_lat (8-bit cache)")


@pytest.mark.parametrize("H,q_len", [(128, 1), (64, 2)])
def test_fp8_bad_page_id_is_reported_not_faulted(H, q_len):
    """A block-table entry outside the pool: the 8-bit kernel's loads read zeros there (the
    scale bytes of page 0 stand in), the status word reports it, the next check passes."""
    spec = small_spec(H=H, q_len=q_len)
    w = quantised(wl.make(spec, seed=2, seq_lens=[130, 64]))
    w["block_table"][1, 0] = 10_000
    step = dec.DecodeStep(w, cache="fp8")
    step.q_lat.copy_(dec.to_torch(wl.latent_queries(spec, step.T, seed=1), step.device))
    step.attend()
    step.combine()
    torch.cuda.synchronize()
    with pytest.raises(mla.MlaError) as e:
        mla.mla_check_status()
    assert e.value.status == mla._binding.MLA_ERR_INVALID
    mla.mla_check_status()


def test_fp8_dropped_page_load_times_out_and_context_stays_usable():
    """The testing hook skips one score-operand load of the first CTA: the MMA issuer's
    wait runs out, every role of both CTAs (converters included) leaves through the abort
    flag, the status word reports MLA_ERR_TIMEOUT, and the same context then decodes the
    8-bit cache correctly."""
    spec = small_spec(H=128)
    w = quantised(wl.make(spec, seed=4, seq_lens=[700, 300, 129]))
    step = dec.DecodeStep(w, sms=4, cache="fp8")
    ql = wl.latent_queries(spec, step.T, seed=9)
    step.q_lat.copy_(dec.to_torch(ql, step.device))
    mla.mla_set_wait_timeout_ns(20_000_000)
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
    mla.mla_check_status()
    step.attend()
    step.combine()
    torch.cuda.synchronize()
    mla.mla_check_status()
    ref = orc.attend_latent(ql, w["q_rope"], w["kv_deq"], w["block_table"], w["seq_lens"], w["scale"],
                            q_len=1, page_size=spec.page_size)
    assert_close(host(step.o_lat), ref["o_lat"], False, "o_lat (8-bit cache) after the injected timeout")
