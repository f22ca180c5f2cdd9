"""One MLA decode step through the C ABI, with the buffers it needs.

`DecodeStep` owns the device tensors of one workload (cache, weights, queries,
outputs, plan, workspace) and issues the library calls of a step in order:
cache append, absorb, decode attention, combine, output projection. Torch is
used for device memory and streams only; every step runs in libmla.so kernels.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _binding as mla


def to_torch(a: np.ndarray, device) -> torch.Tensor:
    """Host array (uint16 = bf16 bits, float32, int32) -> device tensor, same bytes."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def num_sms(device=None) -> int:
    return torch.cuda.get_device_properties(device or torch.cuda.current_device()).multi_processor_count


class DecodeStep:
    def __init__(self, w: dict, device="cuda:0", sms: int | None = None):
        spec = w["spec"]
        self.spec = spec
        self.device = torch.device(device)
        self.dims = mla.dims_of(spec)
        self.B = int(len(w["seq_lens"]))
        self.q_len = spec.q_len
        self.T = self.B * self.q_len
        self.max_pages = int(w["block_table"].shape[1])
        self.num_pages = int(w["num_pages"])
        self.scale = float(w["scale"])
        self.sms = sms or num_sms(self.device)
        self.seq_lens_host = np.ascontiguousarray(w["seq_lens"], dtype=np.int32)
        d = self.device
        self.kv = to_torch(w["kv_cache"], d)
        self.block_table = to_torch(w["block_table"], d)
        self.seq_lens = to_torch(self.seq_lens_host, d)
        self.q_nope = to_torch(w["q_nope"], d)
        self.q_rope = to_torch(w["q_rope"], d)
        self.W_UK = to_torch(w["W_UK"], d)
        self.W_UV = to_torch(w["W_UV"], d)
        self.new_ckr = to_torch(w["new_ckr"], d)
        dt = self.q_nope.dtype
        H, R, Dv = spec.H, spec.R, spec.Dv
        self.q_lat = torch.empty((self.T, H, R), dtype=dt, device=d)
        self.o_lat = torch.empty((self.T, H, R), dtype=dt, device=d)
        self.lse = torch.empty((self.T, H), dtype=torch.float32, device=d)
        self.out = torch.empty((self.T, H, Dv), dtype=dt, device=d)
        self.replan(self.seq_lens_host)

    def replan(self, seq_lens_host: np.ndarray, stream=None):
        plan, info = mla.mla_plan_splits(seq_lens_host, self.B, self.q_len, self.max_pages, self.dims, self.sms)
        self.plan_host = plan
        self.info = info
        cap = mla.mla_plan_capacity(self.B, self.q_len, self.sms)
        self.plan = torch.zeros(cap, dtype=torch.int32, device=self.device)
        self.plan[:info.plan_words].copy_(torch.from_numpy(plan))
        self.ws_bytes = mla.mla_workspace_size(info, self.dims)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=self.device)

    # ---------------------------------------------------------------- individual calls
    def append(self, stream=None):
        mla.mla_cache_append(self.kv, self.block_table, self.seq_lens, self.new_ckr, self.B, self.q_len,
                             self.max_pages, self.num_pages, self.dims, stream)

    def absorb(self, stream=None):
        mla.mla_absorb_q(self.q_nope, self.W_UK, self.q_lat, self.T, self.dims, stream)

    def attend(self, stream=None):
        mla.mla_decode_attn(self.q_lat, self.q_rope, self.kv, self.block_table, self.seq_lens, self.B, self.q_len,
                            self.max_pages, self.num_pages, self.scale, self.plan, self.info, self.o_lat, self.lse,
                            self.workspace, self.ws_bytes, self.dims, stream)

    def combine(self, stream=None):
        mla.mla_combine(self.plan, self.info, self.workspace, self.ws_bytes, self.o_lat, self.lse, self.dims,
                        stream)

    def project(self, stream=None):
        mla.mla_out_proj(self.o_lat, self.W_UV, self.out, self.T, self.dims, stream)

    def run(self, append=True, stream=None):
        """The whole step on device-resident inputs: a2, a1, a3-a5, a6, a7."""
        if append:
            self.append(stream)
        self.absorb(stream)
        self.attend(stream)
        self.combine(stream)
        self.project(stream)

    def launches_per_step(self, append=True) -> int:
        return int(append) + 3 + int(self.info.num_parts > 0)


class HostInputs:
    """Pinned host copies of one step's per-step inputs and its result."""

    def __init__(self, step: DecodeStep, w: dict):
        def pin(a):
            t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16
                                 else np.ascontiguousarray(a))
            return t.pin_memory()
        self.q_nope = pin(w["q_nope"])
        self.q_rope = pin(w["q_rope"])
        self.new_ckr = pin(w["new_ckr"])
        self.block_table = pin(w["block_table"])
        self.seq_lens_np = np.ascontiguousarray(w["seq_lens"], dtype=np.int32)
        self.seq_lens = pin(self.seq_lens_np)
        self.plan = torch.empty(mla.mla_plan_capacity(step.B, step.q_len, step.sms), dtype=torch.int32).pin_memory()
        self.plan_copied = None
        self.out = torch.empty(step.out.shape, dtype=torch.int16 if step.out.dtype == torch.bfloat16
                               else step.out.dtype).pin_memory()

    def h2d_bytes(self, step: DecodeStep) -> int:
        return sum(t.numel() * t.element_size() for t in (self.q_nope, self.q_rope, self.new_ckr,
                                                           self.block_table, self.seq_lens)) + \
            step.info.plan_words * 4

    def d2h_bytes(self) -> int:
        return self.out.numel() * self.out.element_size()


def run_e2e(step: DecodeStep, host: HostInputs, stream=None):
    """One step through the public calls with host inputs: plan on the host, copy the
    step's inputs in, run every kernel, copy the output back (async on `stream`)."""
    s = stream or torch.cuda.current_stream()
    plan, info = mla.mla_plan_splits(host.seq_lens_np, step.B, step.q_len, step.max_pages, step.dims, step.sms)
    if host.plan_copied is not None:
        host.plan_copied.synchronize()   # the previous step's copy has read the pinned plan
    host.plan[:info.plan_words].copy_(torch.from_numpy(plan))
    with torch.cuda.stream(s):
        step.q_nope.view(torch.int16 if step.q_nope.dtype == torch.bfloat16 else step.q_nope.dtype).copy_(
            host.q_nope, non_blocking=True)
        step.q_rope.view(torch.int16 if step.q_rope.dtype == torch.bfloat16 else step.q_rope.dtype).copy_(
            host.q_rope, non_blocking=True)
        step.new_ckr.view(torch.int16 if step.new_ckr.dtype == torch.bfloat16 else step.new_ckr.dtype).copy_(
            host.new_ckr, non_blocking=True)
        step.block_table.copy_(host.block_table, non_blocking=True)
        step.seq_lens.copy_(host.seq_lens, non_blocking=True)
        step.plan[:info.plan_words].copy_(host.plan[:info.plan_words], non_blocking=True)
        if host.plan_copied is None:
            host.plan_copied = torch.cuda.Event()
        host.plan_copied.record(s)
        step.info = info
        step.run(stream=s)
        host.out.copy_(step.out.view(host.out.dtype), non_blocking=True)
