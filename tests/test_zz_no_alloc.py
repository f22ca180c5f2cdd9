"""The allocation-free decode entry point (mla_decode_attn_noalloc).

Some callers cannot allocate device memory: code that runs while a CUDA graph is
being captured, code that must live inside another framework's fixed memory pool,
or hosts that expose no allocator to this library. For them the library offers a
decode call that keeps its split-KV partial outputs in a scratch array the library
owns instead of a caller workspace. Its results must equal those of the ordinary
entry points (mla_decode_attn followed by mla_combine) on the same inputs, on two
calls in a row (the scratch keeps the previous call's contents). This file sorts
last on purpose so that a run that stops at the first failure has run every other
test first; it also passes on its own in a fresh process.
"""
import math

import numpy as np
import pytest
import torch

import mla_latent_kv_46_b200 as mla
from mla_latent_kv_46_b200 import decoder as dec
from inputs import workloads as wl

pytestmark = pytest.mark.gpu


def _close(got, ref):
    got, ref = got.double().cpu().numpy(), ref.double().cpu().numpy()
    assert np.array_equal(np.isneginf(got), np.isneginf(ref))
    m = ~np.isneginf(ref)
    assert np.all(np.abs(got[m] - ref[m]) <= 2e-3 + 1e-2 * np.abs(ref[m]))


@pytest.mark.parametrize("H,policy", [(64, mla.MLA_POLICY_AUTO), (128, mla.MLA_POLICY_AUTO),
                                      (64, mla.MLA_POLICY_SIMT)])
def test_noalloc_decode_matches_workspace_decode_twice(H, policy):
    mla.mla_set_policy(policy)
    try:
        spec = wl.WorkloadSpec(name="noalloc", B=0, H=H, R=512, Dr=64, Dn=128, Dv=128, q_len=1, dtype="bf16",
                               seq_len=None, w_std=1.0 / math.sqrt(512))
        w = wl.make(spec, seed=31, seq_lens=[333, 65, 1000, 0, 64])
        step = dec.DecodeStep(w, sms=9)          # few slots: most queries are split
        assert step.info.num_parts > 0
        step.q_lat.copy_(dec.to_torch(wl.latent_queries(spec, step.T, seed=31), step.device))
        step.attend()
        step.combine()
        torch.cuda.synchronize()
        ref_o, ref_l = step.o_lat.clone(), step.lse.clone()
        for _ in range(2):
            o = torch.full_like(step.o_lat, float("nan"))
            lse = torch.full_like(step.lse, float("nan"))
            mla.mla_decode_attn_noalloc(step.q_lat, step.q_rope, step.kv, step.block_table, step.seq_lens, step.B,
                                        step.q_len, step.max_pages, step.num_pages, step.scale, step.plan,
                                        step.info, o, lse, step.dims)
            torch.cuda.synchronize()
            mla.mla_check_status()
            _close(o, ref_o)
            _close(lse, ref_l)
    finally:
        mla.mla_set_policy(mla.MLA_POLICY_AUTO)
