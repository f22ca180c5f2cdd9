"""Host-side checks of the C ABI (CPU only): symbols, planning, validation.

Nothing here launches a kernel: every call below either is host-only
(mla_plan_*, mla_workspace_size) or must fail validation before any launch.
"""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import mla_latent_kv_46_b200 as mla
from inputs import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(mla.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(mla.EXPORTS) == names


def test_abi_version_and_error_text():
    assert mla.mla_abi_version() == 6
    with pytest.raises(mla.MlaError) as e:
        mla.mla_set_policy(7)
    assert e.value.status == mla._binding.MLA_ERR_INVALID
    assert "policy" in mla.mla_last_error()


def parse_plan(plan):
    B, q_len, nu, ns, nparts, G, H, ps = (int(x) for x in plan[1:9])
    assert plan[0] == 0x4D4C4131
    units = plan[16:16 + 8 * nu].reshape(nu, 8)
    sb = plan[16 + 8 * nu:16 + 8 * nu + ns + 1]
    ip = plan[16 + 8 * nu + ns + 1:].reshape(-1, 2)
    return dict(B=B, q_len=q_len, units=units, slot_begin=sb, item_parts=ip, num_parts=nparts, G=G, H=H, ps=ps)


def dims(H=64, R=512, Dr=64, ps=64, dtype=mla.MLA_BF16):
    return mla.Dims(H, 128, Dr, 128, R, ps, dtype)


@pytest.mark.parametrize("q_len", [1, 3])
@pytest.mark.parametrize("sms", [1, 7, 148])
@pytest.mark.parametrize("H", [64, 128, 16])
def test_plan_covers_every_visible_page_once(q_len, sms, H):
    check_plan_covers(q_len, sms, H)


@pytest.fixture
def combine_cost():
    """Sets the planner's combine cost for one test and restores the default (off)."""
    def set_cost(pages):
        mla.mla_set_plan_combine_cost(pages)
    yield set_cost
    mla.mla_set_plan_combine_cost(-1.0)


@pytest.mark.parametrize("cost", [0.0, 6.5, 1e9])
@pytest.mark.parametrize("q_len", [1, 3])
@pytest.mark.parametrize("sms", [7, 148])
@pytest.mark.parametrize("H", [64, 128])
def test_plan_with_a_combine_cost_still_covers_every_visible_page_once(H, sms, q_len, cost, combine_cost):
    combine_cost(cost)
    check_plan_covers(q_len, sms, H)


def check_plan_covers(q_len, sms, H):
    rng = np.random.default_rng(q_len * 1000 + sms + H)
    lens = rng.integers(0, 700, size=9).astype(np.int32)
    lens[0] = 0
    lens[1] = max(lens[1], q_len)
    max_pages = 12
    d = dims(H=H)
    plan, info = mla.mla_plan_splits(lens, len(lens), q_len, max_pages, d, sms)
    p = parse_plan(plan)
    # SM pairs (2-CTA clusters) for 128 and 64 heads, with two consecutive tokens per
    # unit for 64 heads and several query tokens; otherwise one CTA per 64 heads
    pair = H in (64, 128)
    G = 2 if pair else (H // 64 if H % 64 == 0 else 1)
    per_unit = 128 // H if pair and q_len >= 2 else 1
    assert p["G"] == info.head_groups == G
    assert plan[9] == per_unit
    assert info.num_slots <= max(1, sms // G)
    cover = {}
    for (item, b, pb, pe, part, slot, part2, n) in p["units"]:
        assert item // q_len == b and 1 <= n <= per_unit and (item % q_len) % per_unit == 0
        for j in range(n):
            # a later token of the group may see more pages than an earlier one
            L = int(lens[b]); i = item % q_len + j
            npg = math.ceil(max(0, L - q_len + i + 1) / 64)
            assert item + j < len(lens) * q_len and (item + j) // q_len == b
            cover.setdefault(item + j, []).append((pb, min(pe, max(npg, pb)), part if j == 0 else part2, slot))
    slots = p["units"][:, 5]
    assert np.all(np.diff(slots) >= 0)
    for s in range(info.num_slots):
        assert np.all(slots[p["slot_begin"][s]:p["slot_begin"][s + 1]] == s)
    parts_seen = set()
    for item in range(len(lens) * q_len):
        b, i = divmod(item, q_len)
        n = max(0, int(lens[b]) - q_len + i + 1)
        npg = math.ceil(n / 64)
        segs = sorted(cover[item])
        got = []
        for pb, pe, part, slot in segs:
            got.extend(range(pb, pe))
        assert got == list(range(npg)), (item, segs)
        first, cnt = p["item_parts"][item]
        if len(segs) > 1:
            assert cnt == len(segs)
            assert sorted(s[2] for s in segs) == list(range(first, first + cnt))
            parts_seen.update(s[2] for s in segs)
        else:
            assert cnt == 0 and segs[0][2] == -1
    assert parts_seen == set(range(info.num_parts))


UNIT_COST = 7.5   # pages of work the SM-pair kernel spends per unit beyond its pages


def slot_loads(plan, info):
    p = parse_plan(plan)
    pages = np.zeros(info.num_slots, np.int64)
    units = np.zeros(info.num_slots, np.int64)
    for u in p["units"]:
        pages[u[5]] += u[3] - u[2]
        units[u[5]] += u[3] > u[2]
    return pages, units


@pytest.mark.parametrize("lens", [np.full(64, 4096, np.int32),
                                  np.random.default_rng(0).integers(512, 16385, 128).astype(np.int32)])
def test_plan_balances_pages_and_units_over_pair_slots(lens):
    """SM-pair plans (H=64/128): one slot per pair of SMs, and every slot's work, its
    pages plus a fixed cost per unit, within one unit's cost (and a page) of an equal share."""
    H = 64 if lens[0] == 4096 else 128
    plan, info = mla.mla_plan_splits(lens, len(lens), 1, 256, dims(H=H), 148)
    pages, units = slot_loads(plan, info)
    total = int(np.sum((lens + 63) // 64))
    assert pages.sum() == total
    assert info.num_slots == 74
    groups = len(lens)
    share = (total + UNIT_COST * (groups + 74 - 1)) / 74
    work = pages + UNIT_COST * units
    assert work.max() <= share + UNIT_COST + 1, (work.max(), share)


def heaviest_slot(plan, info):
    pages, units = slot_loads(plan, info)
    return float((pages + UNIT_COST * units).max())


def test_combine_cost_keeps_equal_queries_whole_when_the_merge_costs_more_than_it_saves(combine_cost):
    """64 queries of 64 pages on 74 pair slots: cut, every query is split in two (slots
    of ~68.3 pages of work, 128 partial results to merge); whole, one query per slot (71.5:
    its 64 pages plus one unit's cost) on 64 slots. The whole layout is taken exactly when
    its heaviest slot is at most the cut one's plus the combine cost."""
    lens = np.full(64, 4096, np.int32)
    d = dims(H=64)
    plan_cut, info_cut = mla.mla_plan_splits(lens, 64, 1, 64, d, 148)
    assert info_cut.num_parts == 128
    cut = heaviest_slot(plan_cut, info_cut)
    whole = 64 + UNIT_COST
    assert cut < whole
    combine_cost(whole - cut - 0.01)
    plan, info = mla.mla_plan_splits(lens, 64, 1, 64, d, 148)
    assert np.array_equal(plan, plan_cut)
    combine_cost(whole - cut + 0.01)
    plan, info = mla.mla_plan_splits(lens, 64, 1, 64, d, 148)
    assert info.num_parts == 0 and info.num_slots == 64 and info.num_units == 64
    p = parse_plan(plan)
    for s_, u in enumerate(p["units"]):
        assert (u[0], u[2], u[3], u[4], u[5]) == (s_, 0, 64, -1, s_)
    assert np.all(p["item_parts"] == [-1, 0])
    assert heaviest_slot(plan, info) == whole


def test_combine_cost_keeps_cutting_where_whole_queries_load_a_slot_far_more(combine_cost):
    """128 ragged queries (512..16384 tokens) on 74 slots: keeping them whole leaves a
    slot with a 256-page query and more; the cut layout stays, byte for byte."""
    lens = np.random.default_rng(0).integers(512, 16385, 128).astype(np.int32)
    d = dims(H=128)
    plan0, info0 = mla.mla_plan_splits(lens, 128, 1, 256, d, 148)
    combine_cost(12.0)
    plan, info = mla.mla_plan_splits(lens, 128, 1, 256, d, 148)
    assert info0.num_parts > 0 and np.array_equal(plan, plan0)


@pytest.mark.parametrize("q_len", [2, 4])
def test_combine_cost_whole_queries_keep_the_token_blocks_of_128_heads(q_len, combine_cost):
    """With the merge priced out, every token of the 128-head multi-token layout still
    gets the same layout on its own slot block, now one whole sequence per unit."""
    combine_cost(1e9)
    lens = np.random.default_rng(1).integers(512, 16385, 64).astype(np.int32)
    max_pages = int((lens.max() + 63) // 64)
    plan, info = mla.mla_plan_splits(lens, len(lens), q_len, max_pages, dims(H=128), 148)
    p = parse_plan(plan)
    ns = 74 // q_len
    assert info.num_parts == 0 and info.num_units == q_len * len(lens)
    blocks = [[] for _ in range(q_len)]
    for u in p["units"]:
        k = u[0] % q_len
        assert k * ns <= u[5] < (k + 1) * ns and u[2] == 0 and u[3] == (lens[u[1]] + 63) // 64
        blocks[k].append((u[1], u[5] - k * ns))
    for k in range(1, q_len):
        assert blocks[k] == blocks[0]


def test_combine_cost_rejects_nan_and_is_off_by_default(combine_cost):
    with pytest.raises(mla.MlaError):
        mla.mla_set_plan_combine_cost(float("nan"))
    lens = np.full(64, 4096, np.int32)
    plan, info = mla.mla_plan_splits(lens, 64, 1, 64, dims(H=64), 148)
    assert info.num_parts == 128


@pytest.mark.parametrize("q_len", [2, 4])
def test_plan_puts_each_token_of_128_heads_on_its_own_aligned_slot_block(q_len):
    """128 heads, q_len tokens per sequence (one token per SM-pair unit): the last token's
    pages are laid out on 74 // q_len slots and every token gets the same layout on a
    block of its own, so a sequence's tokens read the same pages on slot j of every block
    (and each token's units, clipped to its pages by the kernel, cover them in order)."""
    lens = np.random.default_rng(1).integers(512, 16385, 64).astype(np.int32)
    max_pages = int((lens.max() + 63) // 64)
    plan, info = mla.mla_plan_splits(lens, len(lens), q_len, max_pages, dims(H=128), 148)
    p = parse_plan(plan)
    ns = 74 // q_len
    assert info.num_slots == q_len * ns
    blocks = [[] for _ in range(q_len)]
    for u in p["units"]:
        k = u[0] % q_len
        assert k * ns <= u[5] < (k + 1) * ns
        blocks[k].append((u[1], u[2], u[3], u[5] - k * ns))
    for k in range(1, q_len):
        assert blocks[k] == blocks[0]
    last = (lens + 63) // 64
    for b in range(len(lens)):
        segs = sorted((pb, pe) for bb, pb, pe, _ in blocks[0] if bb == b)
        assert segs[0][0] == 0 and segs[-1][1] == last[b]
        assert all(segs[i][1] == segs[i + 1][0] for i in range(len(segs) - 1))


@pytest.mark.parametrize("case", ["null", "dims", "eps", "base", "M", "workspace"])
def test_cache_write_rejects_bad_arguments_before_launch(case):
    d = dims(H=128)
    args = dict(hidden=16, W_DKV=16, kv_gain=16, M=1024, kv_cache=16, block_table=16, seq_lens=16, B=2, q_len=1,
                max_pages=4, num_pages=8, q_rope=None, eps=1e-6, rope_base=10000.0, workspace=16,
                workspace_bytes=1 << 30, dims=d)
    if case == "null":
        args["hidden"] = None
    elif case == "dims":
        args["dims"] = dims(H=128, R=256)
    elif case == "eps":
        args["eps"] = float("nan")
    elif case == "base":
        args["rope_base"] = 1.0
    elif case == "M":
        args["M"] = 100
    else:
        args["workspace_bytes"] = mla.mla_cache_write_workspace_size(2, 1024) - 1
    with pytest.raises(mla.MlaError) as e:
        mla.mla_cache_write(**args, stream=0)
    assert e.value.status in (mla._binding.MLA_ERR_INVALID, mla._binding.MLA_ERR_UNSUPPORTED,
                              mla._binding.MLA_ERR_WORKSPACE)


def test_cache_write_workspace_holds_one_fp32_row_per_token_and_k_slice():
    assert mla.mla_cache_write_workspace_size(128, 7168) == 16 * 128 * 576 * 4
    assert mla.mla_cache_write_workspace_size(5, 1024) == 8 * 5 * 576 * 4
    assert mla.mla_cache_write_workspace_size(5, 100) == 0


def test_plan_balances_pages_for_the_single_cta_kernel():
    """Other head counts (one CTA per 64 heads) are planned on pages alone: slots differ
    by at most one page."""
    lens = np.full(64, 4096, np.int32)
    plan, info = mla.mla_plan_splits(lens, 64, 1, 64, dims(H=192), 148)
    pages, _ = slot_loads(plan, info)
    assert pages.sum() == 64 * 64
    assert info.num_slots == 148 // 3
    assert pages.max() - pages.min() <= 1


def test_plan_rejects_too_long_sequences_and_small_buffers():
    with pytest.raises(mla.MlaError) as e:
        mla.mla_plan_splits(np.array([65], np.int32), 1, 1, 1, dims(), 148)
    assert e.value.status == mla._binding.MLA_ERR_INVALID
    info = mla.PlanInfo()
    buf = np.zeros(4, np.int32)
    st = mla._binding._lib.mla_plan_splits(np.array([5], np.int32).ctypes.data, 1, 1, 1, dims(), 148,
                                           buf.ctypes.data, 4, ctypes.byref(info))
    assert st == mla._binding.MLA_ERR_WORKSPACE


def test_workspace_size_formula():
    info = mla.PlanInfo(num_items=4, num_units=6, num_slots=3, num_parts=5, head_groups=1, plan_words=0)
    d = dims(H=16, R=32)
    o = 5 * 16 * 32 * 4
    assert mla.mla_workspace_size(info, d) == (o + 255) // 256 * 256 + 5 * 16 * 4


@pytest.mark.parametrize("call", ["absorb", "out_proj", "append", "decode", "combine", "dims"])
def test_invalid_arguments_fail_before_launch(call):
    d = dims()
    info = mla.PlanInfo(num_items=1, num_units=1, num_slots=1, num_parts=1, head_groups=1, plan_words=30)
    with pytest.raises(mla.MlaError) as e:
        if call == "absorb":
            mla.mla_absorb_q(None, None, None, 4, d, stream=0)
        elif call == "out_proj":
            mla.mla_out_proj(None, 16, 16, 4, d, stream=0)
        elif call == "append":
            mla.mla_cache_append(16, 16, None, 16, 1, 1, 1, 1, d, stream=0)
        elif call == "decode":   # plan made for 2 query tokens, call has 1
            info.num_items = 2
            mla.mla_decode_attn(16, 16, 16, 16, 16, 1, 1, 1, 1, 0.1, 16, info, 16, None, None, 0, d, stream=0)
        elif call == "combine":  # parts but no workspace
            mla.mla_combine(16, info, None, 0, 16, None, d, stream=0)
        else:
            mla.mla_absorb_q(16, 16, 16, 4, mla.Dims(64, 0, 64, 128, 512, 64, 0), stream=0)
    assert e.value.status in (mla._binding.MLA_ERR_INVALID, mla._binding.MLA_ERR_WORKSPACE)


def test_generator_streams_are_independent_of_batch_subset():
    spec = wl.WORKLOADS["deepseek_h128_b128_ragged"]
    lens = wl.seq_lens_of(spec)
    assert lens.min() >= 512 and lens.max() <= 16384 and len(lens) == 128
    a = wl.sequence_rows(wl.spec_with("kimi_h64_b64_l4096"), 5, 100)
    b = wl.sequence_rows(wl.spec_with("kimi_h64_b64_l4096"), 5, 100)
    assert np.array_equal(a, b) and a.dtype == np.uint16


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.1415926], np.float32)
    got = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(x))
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1.0 + 2 ** -6 and got[3] == -2.5
    assert abs(got[4] - 3.140625) < 1e-7


def test_noalloc_rejects_plans_beyond_its_scratch():
    """1000 partial outputs of 64 heads x 512 fp32 need 131 MB, over the 48 MiB the
    allocation-free entry point holds: refused on the host, before any launch."""
    info = mla.PlanInfo(num_items=1, num_units=1000, num_slots=1, num_parts=1000, head_groups=2, plan_words=0,
                        max_pages=1)
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_attn_noalloc(16, 16, 16, 16, 16, 1, 1, 1, 1, 0.1, 16, info, 16, None, dims(), stream=0)
    assert e.value.status == mla._binding.MLA_ERR_WORKSPACE
    assert "48" in mla.mla_last_error() or "50331648" in mla.mla_last_error()


def test_plan_records_max_pages_and_decode_rejects_another():
    """The plan's page ranges index block_table rows of the max_pages it was cut for;
    a decode call with a shorter (or longer) row is refused on the host before any
    launch, so the kernels never index past a row."""
    d = dims(H=128)
    lens = np.array([700, 64, 1], np.int32)
    plan, info = mla.mla_plan_splits(lens, 3, 1, 12, d, 148)
    assert info.max_pages == 12
    for mp in (11, 13):
        with pytest.raises(mla.MlaError) as e:
            mla.mla_decode_attn(16, 16, 16, 16, 16, 3, 1, mp, 100, 0.1, 16, info, 16, None, None, 0, d,
                                stream=0)
        assert e.value.status == mla._binding.MLA_ERR_INVALID
        assert "max_pages" in mla.mla_last_error()
        with pytest.raises(mla.MlaError) as e:
            mla.mla_decode_attn_noalloc(16, 16, 16, 16, 16, 3, 1, mp, 100, 0.1, 16, info, 16, None, d, stream=0)
        assert "max_pages" in mla.mla_last_error()


@pytest.mark.parametrize("case", ["null", "dims_R", "dims_f32", "H", "workspace", "align"])
def test_fp8_decode_rejects_bad_arguments_before_launch(case):
    d = dims(H=128)
    lens = np.array([100, 7], np.int32)
    plan, info = mla.mla_plan_splits(lens, 2, 1, 4, d, 148)
    args = dict(q_lat=256, q_rope=256, kv_codes=256, kv_scales=256, block_table=256, seq_lens=256, B=2, q_len=1,
                max_pages=4, num_pages=8, scale=0.07, plan_dev=256, info=info, o_lat=256, lse=None, workspace=256,
                workspace_bytes=1 << 30, dims=d)
    if case == "null":
        args["kv_scales"] = None
    elif case == "dims_R":
        args["dims"] = dims(H=128, R=256)
    elif case == "dims_f32":
        args["dims"] = dims(H=128, dtype=mla.MLA_F32)
    elif case == "H":
        args["dims"] = dims(H=192)
    elif case == "workspace":
        args["workspace_bytes"] = mla.mla_workspace_size_fp8(info, d) - 1
    else:
        args["workspace"] = 256 + 16
    with pytest.raises(mla.MlaError) as e:
        mla.mla_decode_attn_fp8(**args, stream=0)
    assert e.value.status in (mla._binding.MLA_ERR_INVALID, mla._binding.MLA_ERR_UNSUPPORTED,
                              mla._binding.MLA_ERR_WORKSPACE)


def test_fp8_workspace_is_the_partials_then_the_split_query():
    d = dims(H=128)
    info = mla.PlanInfo(num_items=4, num_units=6, num_slots=3, num_parts=5, head_groups=2, plan_words=0)
    parts = mla.mla_workspace_size(info, d)
    rows = 4 * 128
    up = lambda x: (x + 255) // 256 * 256
    assert mla.mla_workspace_size_fp8(info, d) == up(parts) + up(2 * rows * 576) + rows * 4
    info0 = mla.PlanInfo(num_items=4, num_units=4, num_slots=4, num_parts=0, head_groups=2, plan_words=0)
    assert mla.mla_workspace_size_fp8(info0, d) == up(2 * rows * 576) + rows * 4


@pytest.mark.parametrize("case", ["null", "dims", "count", "align"])
def test_fp8_quantize_and_append_reject_bad_arguments(case):
    d = dims(H=128)
    if case == "null":
        call = lambda: mla.mla_quantize_rows_fp8(None, 256, 256, 4, d, stream=0)
    elif case == "dims":
        call = lambda: mla.mla_cache_append_fp8(256, 256, 256, 256, 256, 2, 1, 4, 8, dims(H=128, Dr=32), stream=0)
    elif case == "count":
        call = lambda: mla.mla_quantize_rows_fp8(256, 256, 256, -1, d, stream=0)
    else:
        call = lambda: mla.mla_cache_append_fp8(256, 256, 256, 256, 256 + 8, 2, 1, 4, 8, d, stream=0)
    with pytest.raises(mla.MlaError) as e:
        call()
    assert e.value.status in (mla._binding.MLA_ERR_INVALID, mla._binding.MLA_ERR_UNSUPPORTED)


@pytest.mark.parametrize("case", ["dims", "odd_heads", "decreasing", "first", "workspace", "null"])
def test_prefill_rejects_bad_arguments_before_launch(case):
    d = dims(H=8)
    cu = np.array([0, 100, 300], np.int32)
    args = dict(ckr=256, q_nope=256, q_rope=256, W_UK=256, W_UV=256, cu_seqlens=256, cu_seqlens_host=cu, B=2,
                scale=0.07, out=256, workspace=256, workspace_bytes=1 << 30, dims=d)
    if case == "dims":
        args["dims"] = mla.Dims(8, 128, 64, 64, 512, 64, mla.MLA_BF16)   # Dv = 64
    elif case == "odd_heads":
        args["dims"] = dims(H=7)
    elif case == "decreasing":
        args["cu_seqlens_host"] = np.array([0, 100, 50], np.int32)
    elif case == "first":
        args["cu_seqlens_host"] = np.array([4, 100, 300], np.int32)
    elif case == "workspace":
        args["workspace_bytes"] = mla.mla_prefill_workspace_size(300, d) - 1
    else:
        args["q_rope"] = None
    with pytest.raises(mla.MlaError) as e:
        mla.mla_prefill_attn(**args, stream=0)
    assert e.value.status in (mla._binding.MLA_ERR_INVALID, mla._binding.MLA_ERR_UNSUPPORTED,
                              mla._binding.MLA_ERR_WORKSPACE)


def test_prefill_workspace_holds_bf16_keys_and_values_of_every_head():
    d = dims(H=64)
    assert mla.mla_prefill_workspace_size(16384, d) == 2 * 16384 * 64 * 128 * 2
    assert mla.mla_prefill_workspace_size(3, dims(H=2)) == 2 * ((3 * 2 * 128 * 2 + 255) // 256 * 256)
    assert mla.mla_prefill_workspace_size(100, mla.Dims(8, 64, 64, 128, 512, 64, mla.MLA_BF16)) == 0   # Dn = 64
