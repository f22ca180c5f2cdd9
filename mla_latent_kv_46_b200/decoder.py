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
    """cache="fp8": the cache is held as E4M3 codes and per-token scale bytes (the 8-bit
    cache calls); the codes come from w["kv_codes"] / w["kv_scales"] when given, else
    the workload's bf16 rows are quantised on the device by mla_quantize_rows_fp8."""

    def __init__(self, w: dict, device="cuda:0", sms: int | None = None, cache: str = "bf16"):
        spec = w["spec"]
        self.spec = spec
        self.fp8 = cache == "fp8"
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
        if self.fp8:
            P, ps = self.num_pages, spec.page_size
            if "kv_codes" in w:
                self.kv_codes = to_torch(w["kv_codes"], d)
                self.kv_scales = to_torch(w["kv_scales"], d)
            else:
                rows = to_torch(w["kv_cache"], d)
                self.kv_codes = torch.empty((P, ps, spec.row), dtype=torch.uint8, device=d)
                self.kv_scales = torch.empty((P, ps), dtype=torch.uint8, device=d)
                mla.mla_quantize_rows_fp8(rows, self.kv_codes, self.kv_scales, P * ps, self.dims)
                torch.cuda.synchronize(d)
                del rows
            self.kv = None
        else:
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
        self.o_lat = torch.empty((self.T, H, R), dtype=torch.float32, device=d)   # fp32 for every dtype
        self.lse = torch.empty((self.T, H), dtype=torch.float32, device=d)
        self.out = torch.empty((self.T, H, Dv), dtype=dt, device=d)
        # the cache append and the query absorption are independent: the append runs on
        # this side stream beside the absorption, and the decode waits for both
        self.side = torch.cuda.Stream(device=d)
        self.replan(self.seq_lens_host)

    def replan(self, seq_lens_host: np.ndarray, stream=None):
        plan, info = mla.mla_plan_splits(seq_lens_host, self.B, self.q_len, self.max_pages, self.dims, self.sms)
        self.plan_host = plan
        self.info = info
        cap = mla.mla_plan_capacity(self.B, self.q_len, self.sms)
        self.plan = torch.zeros(cap, dtype=torch.int32, device=self.device)
        self.plan[:info.plan_words].copy_(torch.from_numpy(plan))
        self.ws_bytes = (mla.mla_workspace_size_fp8 if self.fp8 else mla.mla_workspace_size)(info, self.dims)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=self.device)

    # ---------------------------------------------------------------- individual calls
    def append(self, stream=None):
        if self.fp8:
            mla.mla_cache_append_fp8(self.kv_codes, self.kv_scales, self.block_table, self.seq_lens, self.new_ckr,
                                     self.B, self.q_len, self.max_pages, self.num_pages, self.dims, stream)
            return
        mla.mla_cache_append(self.kv, self.block_table, self.seq_lens, self.new_ckr, self.B, self.q_len,
                             self.max_pages, self.num_pages, self.dims, stream)

    def absorb(self, stream=None):
        mla.mla_absorb_q(self.q_nope, self.W_UK, self.q_lat, self.T, self.dims, stream)

    def attend(self, stream=None):
        if self.fp8:
            mla.mla_decode_attn_fp8(self.q_lat, self.q_rope, self.kv_codes, self.kv_scales, self.block_table,
                                    self.seq_lens, self.B, self.q_len, self.max_pages, self.num_pages, self.scale,
                                    self.plan, self.info, self.o_lat, self.lse, self.workspace, self.ws_bytes,
                                    self.dims, stream)
            return
        mla.mla_decode_attn(self.q_lat, self.q_rope, self.kv, self.block_table, self.seq_lens, self.B, self.q_len,
                            self.max_pages, self.num_pages, self.scale, self.plan, self.info, self.o_lat, self.lse,
                            self.workspace, self.ws_bytes, self.dims, stream)

    def combine(self, stream=None):
        mla.mla_combine(self.plan, self.info, self.workspace, self.ws_bytes, self.o_lat, self.lse, self.dims,
                        stream)

    def project(self, stream=None):
        mla.mla_out_proj(self.o_lat, self.W_UV, self.out, self.T, self.dims, stream)

    def append_and_absorb(self, stream=None):
        """a2 on the side stream beside a1 on `stream`; `stream` then waits for both."""
        s = stream or torch.cuda.current_stream(self.device)
        self.side.wait_stream(s)               # the step's inputs are in place
        self.append(self.side)
        self.absorb(s)
        s.wait_stream(self.side)

    def run(self, append=True, stream=None):
        """The whole step on device-resident inputs: a2 (beside a1), a1, a3-a5, a6, a7."""
        if append:
            self.append_and_absorb(stream)
        else:
            self.absorb(stream)
        self.attend(stream)
        self.combine(stream)
        self.project(stream)

    def sibling(self) -> "DecodeStep":
        """A second set of per-step buffers (queries, new rows, block table, lengths,
        plan, workspace, intermediates, output) sharing this step's cache and weights."""
        t = object.__new__(DecodeStep)
        t.__dict__.update(self.__dict__)
        for name in ("block_table", "seq_lens", "q_nope", "q_rope", "new_ckr", "q_lat", "o_lat", "lse", "out",
                     "plan", "workspace"):
            setattr(t, name, torch.empty_like(getattr(self, name)))
        t.plan.copy_(self.plan)
        return t

    def launches_per_step(self, append=True) -> int:
        # (the 8-bit cache's decode is two launches: the query split, then attention)
        return int(append) + 3 + int(self.info.num_parts > 0) + int(self.fp8)


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


class PipelinedE2E:
    """Consecutive end-to-end steps through the public calls, with host inputs, where
    step k+1's host-to-device copies and step k-1's device-to-host copy overlap step
    k's kernels: two sets of per-step device buffers, one stream for copies in and one
    for copies out beside the compute stream, and events for every hand-over. The host plans step k+1 while the device
    runs step k, and waits for step k-1's result before it enqueues step k+1 (it
    consumes results one step behind).
    """

    def __init__(self, step: DecodeStep, host: HostInputs, stream=None):
        self.sets = [step, step.sibling()]
        self.host = host
        self.comp = stream or torch.cuda.current_stream()
        self.copy = torch.cuda.Stream(device=step.device)      # host -> device
        self.copy_out = torch.cuda.Stream(device=step.device)  # device -> host
        self.plans = [torch.empty_like(host.plan).pin_memory() for _ in range(2)]
        self.outs = [host.out, torch.empty_like(host.out).pin_memory()]
        self.inputs_free = [None, None]   # compute of the set's previous step done
        self.out_read = [None, None]      # device-to-host copy of the set's previous step done
        self.k = 0

    def enqueue(self):
        """Plan and enqueue the next step; returns the event of its result on the host."""
        i = self.k & 1
        st, host = self.sets[i], self.host
        if self.k >= 2:
            self.out_read[i].synchronize()   # the host has the result of step k-2: consume it
        plan, info = mla.mla_plan_splits(host.seq_lens_np, st.B, st.q_len, st.max_pages, st.dims, st.sms)
        self.plans[i][:info.plan_words].copy_(torch.from_numpy(plan))
        ready = torch.cuda.Event()
        with torch.cuda.stream(self.copy):
            if self.inputs_free[i] is not None:
                self.copy.wait_event(self.inputs_free[i])
            for dst, src in ((st.q_nope, host.q_nope), (st.q_rope, host.q_rope), (st.new_ckr, host.new_ckr)):
                dst.view(torch.int16 if dst.dtype == torch.bfloat16 else dst.dtype).copy_(src, non_blocking=True)
            st.block_table.copy_(host.block_table, non_blocking=True)
            st.seq_lens.copy_(host.seq_lens, non_blocking=True)
            st.plan[:info.plan_words].copy_(self.plans[i][:info.plan_words], non_blocking=True)
            ready.record(self.copy)
        st.info = info
        done = torch.cuda.Event()
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(ready)
            if self.out_read[i] is not None:
                self.comp.wait_event(self.out_read[i])   # the output buffer was read back
            st.run(stream=self.comp)
            done.record(self.comp)
        self.inputs_free[i] = done
        out_read = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.copy_out):
            self.copy_out.wait_event(done)
            self.outs[i].copy_(st.out.view(self.outs[i].dtype), non_blocking=True)
            out_read.record(self.copy_out)
        self.out_read[i] = out_read
        self.k += 1
        return out_read
