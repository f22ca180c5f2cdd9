#!/usr/bin/env python
"""Benchmark of one MLA decode step over a paged latent + RoPE cache on B200.

A step is the whole hot path on one batch: cache append of the new rows, query
absorption through W_UK, decode attention (tcgen05), split-KV combine and the W_UV
output projection, all in libmla.so kernels. The metric is cache bytes read per
second (every visible cached row of 1,152 bytes counted once per step), with the
step's FLOPs and the decode kernel's roofline fraction beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

N > 1 runs under torchrun, one process per GPU; every rank decodes its own batch
of the workload (sequences are independent: no collective on the data path) and
rank 0 prints the JSON line, timed as the max over ranks.
`--impl reference` times the fp64 CPU oracle (the only other implementation of
this computation) on the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode: cache GB/s and TFLOP/s, fraction of B200 roofline"
DEFAULT_WORKLOAD = "deepseek_h128_b128_ragged"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 512 << 20
L2_BYTES = 126 << 20          # B200 L2
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def decode_kernel_of(H, q_len):
    """(source file, kernel name) of the tensor-core decode kernel used for H heads and
    q_len query tokens per sequence (the library's default policy)."""
    if H in (64, 128):
        return "decode_2sm.cuh", "mla_decode_attn (tcgen05 cta_group::2 decode_2sm_kernel, SM pairs)"
    return "decode_tc.cuh", "mla_decode_attn (tcgen05 decode_kernel)"


def traffic_record(workload, H, q_len):
    """DRAM bytes per launch of the decode kernel from a committed ncu summary, valid
    only while the kernel source is unchanged (its sha256 is recorded there)."""
    src_name, _ = decode_kernel_of(H, q_len)
    src = os.path.join(ROOT, "mla_latent_kv_46_b200", "csrc", src_name)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    path = os.path.join(ROOT, "profiles", f"ncu_decode_attn_{workload}.md")
    if not os.path.exists(path):
        return None, sha
    text = open(path).read()
    m_sha = re.search(re.escape(src_name) + r" sha256\[:16\]:\s*([0-9a-f]{16})", text)
    m_tr = re.search(r"traffic per full launch \(bytes\):\s*([0-9]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != sha:
        return None, sha
    return int(m_tr.group(1)), sha


# ----------------------------------------------------------------------------- clocks (NVML poller)

class ClockSampler:
    """Polls SM clock and throttle reasons of one GPU every few ms while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hh)
                u = u.decode() if isinstance(u, bytes) else u
                if uuid in u:
                    h = hh
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvml unavailable"}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        reasons = sorted(name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "sm_mhz_min": min(mhz)}


# ----------------------------------------------------------------------------- reference arm (oracle, CPU)

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(spec, w, budget_s=20.0, max_seqs=None, absorbed=False):
    """Time the oracle (the non-absorbed fp64 definition, or its absorbed fp64 form) on
    whole sequences of the workload, shortest first, until about budget_s of CPU work.
    Returns (bytes, seconds, desc)."""
    from oracle import mla_oracle as orc
    run = orc.decode_absorbed if absorbed else orc.decode_nonabsorbed
    lens = w["seq_lens"]
    order = np.argsort(lens, kind="stable")
    done_bytes, spent, seqs = 0, 0.0, []
    for b in order:
        b = int(b)
        t0 = time.perf_counter()
        sl = slice(b * spec.q_len, (b + 1) * spec.q_len)
        run(w["q_nope"][sl], w["q_rope"][sl], w["kv_cache"], w["block_table"][b:b + 1], w["seq_lens"][b:b + 1],
            w["W_UK"], w["W_UV"], w["scale"], q_len=spec.q_len, page_size=spec.page_size)
        spent += time.perf_counter() - t0
        seqs.append(b)
        done_bytes += int(lens[b]) * spec.row * (2 if spec.dtype == "bf16" else 4)
        if spent >= budget_s or (max_seqs and len(seqs) >= max_seqs):
            break
    form = "absorbed" if absorbed else "non-absorbed"
    desc = (f"oracle (fp64 numpy, {form}) on {len(seqs)} of {len(lens)} sequences "
            f"(shortest first, {int(sum(int(lens[b]) for b in seqs))} tokens, all {spec.H} heads)")
    return done_bytes, spent, desc


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from inputs import workloads as wl
    spec = wl.WORKLOADS[args.workload]
    w = wl.make(spec, seed=0)
    per_step_budget = 4.0
    for _ in range(args.warmup):
        oracle_sample(spec, w, budget_s=per_step_budget, max_seqs=1)
    tot_b, tot_t, desc = 0, 0.0, ""
    for _ in range(args.steps):
        b, t, desc = oracle_sample(spec, w, budget_s=per_step_budget, max_seqs=1)
        tot_b += b
        tot_t += t
    value = tot_b / tot_t / 1e9
    cores = cpu_threads()
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(spec, w, args),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": f"per step: {desc}"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def reduce_over_ranks(world, device, sums=(), maxes=()):
    """Sums and maxima of per-rank numbers over all ranks of the default process group, in
    float64 on `device` (identity on one rank). Every rank makes the same calls in the same
    order: one all-reduce for the sums, one for the maxima."""
    sums, maxes = [float(x) for x in sums], [float(x) for x in maxes]
    if world == 1:
        return sums, maxes
    import torch
    import torch.distributed as dist
    out = []
    for vals, op in ((sums, dist.ReduceOp.SUM), (maxes, dist.ReduceOp.MAX)):
        if vals:
            t = torch.tensor(vals, dtype=torch.float64, device=device)
            dist.all_reduce(t, op=op)
            vals = t.cpu().tolist()
        out.append(vals)
    return out[0], out[1]


def wl_cache_bytes(spec, lens, fp8=False):
    """Algorithmic cache bytes of one pass: every valid row once; the 8-bit cache reads
    R + Dr codes and one scale byte per token."""
    if fp8:
        return int(np.sum(lens, dtype=np.int64)) * (spec.R + spec.Dr + 1)
    elem = 2 if spec.dtype == "bf16" else 4
    return int(np.sum(lens, dtype=np.int64)) * (spec.R + spec.Dr) * elem


def time_cache_write(step, spec, stream, M=7168, reps=20):
    """The cache-write prologue (mla_cache_write: down projection of the step's new tokens'
    hidden states, width M = 7168 as in DeepSeek-scale models, kv_rmsnorm, rotary shared
    key, append; the query's rope part turned in place) timed on its own, outside the
    step: CUDA events around each call on the launching stream. It rewrites the rows the
    step's append wrote. None where the dims have no prologue kernel."""
    import torch
    import mla_latent_kv_46_b200 as mla
    from mla_latent_kv_46_b200 import decoder as dec
    from inputs import workloads as wl
    if spec.dtype != "bf16" or spec.R != 512 or spec.Dr != 64 or spec.page_size != 64:
        return None
    pin = wl.prologue_inputs(spec, step.T, M, seed=3)
    hidden, W, gain = (dec.to_torch(pin[k], step.device) for k in ("hidden", "W_DKV", "kv_gain"))

    ws_bytes = mla.mla_cache_write_workspace_size(step.T, M)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=step.device)

    def call():
        mla.mla_cache_write(hidden, W, gain, M, step.kv, step.block_table, step.seq_lens, step.B, step.q_len,
                            step.max_pages, step.num_pages, step.q_rope, 1e-6, 10000.0, ws, ws_bytes, step.dims,
                            stream)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    mla.mla_check_status()
    ms = statistics.median(ts)
    wbytes = (spec.R + spec.Dr) * M * 2
    abytes = step.T * M * 2
    return {"ms": ms, "hidden_width": M, "tokens": step.T, "weight_bytes": wbytes,
            "gb_per_s": (wbytes + abytes) / (ms / 1e3) / 1e9, "launches": 2,
            "kernels": "cache_write_gemm_kernel (split-K down projection), cache_write_finish_kernel (norm, "
                       "rotations, append)"}


def timing_blocks(steps, max_blocks=4):
    """Sizes of the blocks the timed steps are cut into (each followed by as many steps
    with every kernel bracketed): at most `max_blocks`, sizes differing by at most one,
    summing to `steps`."""
    n = max(1, min(max_blocks, steps))
    return [steps // n + (1 if i < steps % n else 0) for i in range(n)]


def needs_flush(cache_bytes):
    """Inputs larger than twice the L2 evict it on their own: every step streams the whole
    cache through L2, so nothing a step reads is still resident at the next one. Smaller
    workloads get a 512 MiB write between timed steps instead."""
    return cache_bytes <= 2 * L2_BYTES


def l2_method(cache_bytes):
    if needs_flush(cache_bytes):
        return f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write, outside the timed events)"
    return (f"inputs larger than L2: each step streams the {cache_bytes / 1e9:.2f} GB cache through the "
            f"{L2_BYTES >> 20} MiB L2, evicting the previous step's data; no flush")


def workload_config(spec, w, args, job_tokens=None):
    """The line's `config`: rank 0's batch, plus the whole job's when several ranks run
    (rank r decodes the batch generated with seed r)."""
    lens = w["seq_lens"]
    seed = "seed 0" if args.gpus == 1 else "seed = rank of each replica"
    cfg = {"workload": spec.name, "B": int(len(lens)), "H": spec.H, "kv_lora_rank": spec.R, "rope_dim": spec.Dr,
           "D_nope": spec.Dn, "D_v": spec.Dv, "q_len": spec.q_len, "page_size": spec.page_size,
           "seq_lens": (f"uniform in [{spec.ragged[0]},{spec.ragged[1]}], {seed}" if spec.ragged
                        else f"{spec.seq_len} each"),
           "cached_tokens": int(np.sum(lens, dtype=np.int64)),
           "l2": l2_method(wl_cache_bytes(spec, lens, getattr(args, "cache", "bf16") == "fp8")),
           "parallelism": f"replicas x{args.gpus} (independent sequences per GPU)"}
    if args.gpus > 1:
        cfg["global_batch"] = int(len(lens)) * args.gpus
        if job_tokens is not None:
            cfg["cached_tokens_all_ranks"] = int(job_tokens)
    if getattr(args, "cache", "bf16") == "fp8":
        cfg["cache"] = ("E4M3 codes (576 per token) + one power-of-two scale byte per token, 577 bytes per "
                        "token; the bf16 rows of the workload quantised once on the device before timing")
    if getattr(args, "seqs", 0):
        cfg["subset"] = f"first {args.seqs} sequences only (profiling run, not a bench line)"
    return cfg


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import __graft_entry__
    __graft_entry__.build()
    import mla_latent_kv_46_b200 as mla
    from mla_latent_kv_46_b200 import decoder as dec
    from inputs import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    spec = wl.WORKLOADS[args.workload]
    if args.seqs:
        # profiling knob: the first N sequences of the workload only (not a bench line)
        w = wl.make(spec, seed=rank, seq_lens=wl.seq_lens_of(spec, rank)[:args.seqs])
    else:
        w = wl.make(spec, seed=rank)
    fp8 = args.cache == "fp8"
    step = dec.DecodeStep(w, device=dev, cache=args.cache)
    mla.mla_set_policy(mla.MLA_POLICY_AUTO)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---------------------------------------------------------------- device-resident timing
    # The timed steps carry no events between their kernels (an event recorded between two
    # kernels stalls the stream ~3-4 us): one pair of events around each block of steps,
    # or around each step where an L2 flush runs between steps (outside the events). Each
    # timed block is followed by as many untimed steps that bracket every kernel with
    # events, for the per-kernel split and the decode kernel's duration (the roofline):
    # the two kinds alternate in four blocks, so both see the same clocks when the power
    # cap lowers them as the run goes on. The append runs on a side stream beside the
    # absorption (DecodeStep.run), so those two share one interval.
    names = ["append+absorb", "attend", "combine", "project"]
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    mla.mla_check_status()
    flush_each = needs_flush(wl_cache_bytes(spec, w["seq_lens"], fp8))
    blocks = timing_blocks(args.steps)
    nblk = len(blocks)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps if flush_each else nblk)]
    barrier()
    with ClockSampler(dev.index) as clk:
        k = 0
        for bi, nb in enumerate(blocks):
            if flush_each:
                for j in range(k, k + nb):
                    b0, b1 = bounds[j]
                    flush.fill_(j & 0xFF)      # evict the cache from L2 (outside the timed events)
                    b0.record(stream)
                    step.run(stream=stream)
                    b1.record(stream)
            else:
                bounds[bi][0].record(stream)
                for _ in range(nb):
                    step.run(stream=stream)
                bounds[bi][1].record(stream)
            # the same number of steps with every kernel bracketed (not part of the timed steps)
            for j in range(k, k + nb):
                if flush_each:
                    flush.fill_(j & 0xFF)
                e = ev[j]
                e[0].record(stream)
                step.append_and_absorb(stream)
                e[1].record(stream)
                step.attend(stream)
                e[2].record(stream)
                step.combine(stream)
                e[3].record(stream)
                step.project(stream)
                e[4].record(stream)
            k += nb
        barrier()
    step_total_ms = float(sum(b0.elapsed_time(b1) for b0, b1 in bounds))
    mla.mla_check_status()
    per_kernel = {n: 0.0 for n in names}
    attend_ms = []
    split_ms = []
    for e in ev:
        for i, n in enumerate(names):
            per_kernel[n] += e[i].elapsed_time(e[i + 1])
        attend_ms.append(e[1].elapsed_time(e[2]))
        split_ms.append(e[0].elapsed_time(e[-1]))
    # this rank's batch; the job's work is the sum over ranks (each rank decodes its own
    # ragged batch) and its time the slowest rank's
    cache_bytes = wl_cache_bytes(spec, w["seq_lens"], fp8)
    flops = wl.attention_flops(spec, w["seq_lens"])
    tokens = int(np.sum(w["seq_lens"], dtype=np.int64))
    (job_bytes, job_flops, job_tokens), (total_ms_max,) = reduce_over_ranks(
        world, dev, (cache_bytes, flops, tokens), (step_total_ms,))
    ms_per_step = total_ms_max / args.steps
    value = job_bytes * args.steps / (total_ms_max / 1e3) / 1e9

    # ---------------------------------------------------------------- roofline of the decode kernel
    peaks, peak_src = load_peaks()
    attn_ms = per_kernel["attend"] / args.steps
    t_hbm = cache_bytes / (peaks["hbm_gbs"] * 1e9)
    # (the 8-bit cache too: its query enters the score MMAs as two E4M3 pieces, two 8-bit
    # MMAs per K step at twice the rate, the tensor time of one bf16 MMA)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    traffic, sha = traffic_record(spec.name + ("_fp8" if fp8 else ""), spec.H, spec.q_len)
    if args.seqs:
        traffic = None   # the committed figure is for the whole workload
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": cache_bytes / (attn_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / (attn_ms / 1e3) / 1e12, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    src_name, roof["kernel"] = decode_kernel_of(spec.H, spec.q_len)
    roof["algorithmic_bytes_per_launch"] = cache_bytes
    roof["algorithmic_flops_per_launch"] = flops
    roof["roofline_ms"] = 1e3 * max(t_hbm, t_tc)
    roof["frac_of_roofline_time"] = 1e3 * max(t_hbm, t_tc) / attn_ms
    roof["tflops"] = flops / (attn_ms / 1e3) / 1e12
    # the same against the spec sheet (~8 TB/s HBM3e, 2.25 PFLOP/s dense bf16)
    t_spec = max(cache_bytes / SPEC_PEAKS["hbm_gbs"] / 1e9, flops / SPEC_PEAKS["bf16_tflops"] / 1e12)
    roof["frac_vs_spec"] = 1e3 * t_spec / attn_ms
    roof["spec_peaks"] = dict(SPEC_PEAKS)
    roof["attend_ms_median"] = float(np.median(attend_ms))
    roof["attend_ms_min"] = float(np.min(attend_ms))
    roof["source_sha256_16"] = f"{src_name} {sha}"

    # ---------------------------------------------------------------- end to end through the public API
    if args.device_only:
        # profiling aid: the device-resident steps only (no end-to-end section)
        e2e = None
        if rank == 0:
            print(json.dumps({"device_only": True, "ms_per_step": ms_per_step, "roofline": roof,
                              "per_kernel_ms": {n: v / args.steps for n, v in per_kernel.items()},
                              "split_pass_ms_per_step": float(np.mean(split_ms))}), flush=True)
        del flush
        return 0
    hostin = dec.HostInputs(step, w)
    e2e_steps = args.steps
    barrier()
    if cache_bytes > 2 * L2_BYTES:
        # steps back to back, each one's copies overlapping its neighbours' kernels; the
        # cache is larger than L2, so no flush is needed between them
        pipe = dec.PipelinedE2E(step, hostin, stream)
        for _ in range(max(3, args.warmup)):
            pipe.enqueue()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(pipe.copy)
        last = None
        for _ in range(e2e_steps):
            last = pipe.enqueue()
        last.synchronize()            # the last step's result is on the host
        e2e_ms = e0.elapsed_time(last)
        e2e_mode = "pipelined: step k+1's copies in and step k-1's copy out overlap step k"
    else:
        for _ in range(max(3, args.warmup)):
            dec.run_e2e(step, hostin, stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_ms = 0.0
        for k in range(e2e_steps):
            flush.fill_(k & 0xFF)
            e0.record(stream)
            dec.run_e2e(step, hostin, stream)
            e1.record(stream)
            e1.synchronize()          # the step's result is on the host
            e2e_ms += e0.elapsed_time(e1)
        e2e_mode = "one step at a time, L2 flushed before each"
    barrier()
    mla.mla_check_status()
    _, (e2e_ms,) = reduce_over_ranks(world, dev, (), (e2e_ms,))
    e2e = {"value": job_bytes * e2e_steps / (e2e_ms / 1e3) / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": hostin.h2d_bytes(step), "d2h_bytes_per_step": hostin.d2h_bytes(),
           "ms_per_step": e2e_ms / e2e_steps, "mode": e2e_mode}

    prologue = None if fp8 else time_cache_write(step, spec, stream)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            b, t, desc = oracle_sample(spec, w, budget_s=args.cpu_budget)
            cpu = {"value": b / t / 1e9, "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
                   "sample": desc, "seconds": t}
            # the absorbed fp64 form as a second, more algorithm-matched host baseline
            b2, t2, desc2 = oracle_sample(spec, w, budget_s=min(5.0, args.cpu_budget), absorbed=True)
            cpu["absorbed_form"] = {"value": b2 / t2 / 1e9, "unit": "GB/s", "sample": desc2, "seconds": t2}
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "e4m3 cache, bf16 queries" if fp8 else "bf16", "data": "synthetic",
                "config": workload_config(spec, w, argparse.Namespace(gpus=world, seqs=args.seqs, cache=args.cache),
                                          job_tokens),
                "tflops": job_flops * args.steps / (total_ms_max / 1e3) / 1e12,
                "per_kernel_ms": {n: per_kernel[n] / args.steps for n in names},
                "split_pass_ms_per_step": float(np.mean(split_ms)),
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "cache_write": prologue,
                "gpu_launches": step.launches_per_step() * args.steps,
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    del flush
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- prefill workloads

PREFILL_METRIC = "MLA prefill (non-absorbed, causal): TFLOP/s and fraction of the B200 bf16 tensor roofline"


def prefill_oracle_sample(spec, pin, budget_s):
    """The oracle's full causal forward on whole (sequence, head) pairs in order, until
    about budget_s of CPU work. Returns (flops, seconds, desc)."""
    from oracle import mla_oracle as orc
    cu = pin["cu_seqlens"]
    flops, spent, n = 0, 0.0, 0
    for b in range(len(pin["seq_lens"])):
        a, e = int(cu[b]), int(cu[b + 1])
        rows = orc.to_f64(pin["ckr"][a:e])
        for h in range(spec.H):
            t0 = time.perf_counter()
            orc.full_causal(rows[:, :spec.R], rows[:, spec.R:], pin["q_nope"][a:e], pin["q_rope"][a:e],
                            pin["W_UK"], pin["W_UV"], spec.scale, heads=[h])
            spent += time.perf_counter() - t0
            L = e - a
            flops += 2 * spec.R * (spec.Dn + spec.Dv) * L + L * (L + 1) // 2 * 2 * (spec.Dn + spec.Dr + spec.Dv)
            n += 1
            if spent >= budget_s:
                return flops, spent, f"oracle (fp64 numpy full causal forward) on {n} (sequence, head) pairs"
    return flops, spent, f"oracle (fp64 numpy full causal forward) on {n} (sequence, head) pairs"


def run_prefill(args):
    """A step is one mla_prefill_attn call over the workload's packed sequences: the two
    up-projection GEMMs and the causal attention, inputs resident in HBM."""
    import torch
    import __graft_entry__
    __graft_entry__.build()
    import mla_latent_kv_46_b200 as mla
    from mla_latent_kv_46_b200 import decoder as dec
    from inputs import workloads as wl

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    spec = wl.WORKLOADS[args.workload]
    pin = wl.prefill_inputs(spec, seed=0)
    d = mla.dims_of(spec)
    N, B = int(pin["cu_seqlens"][-1]), len(pin["seq_lens"])
    t = {k: dec.to_torch(pin[k], dev) for k in ("ckr", "q_nope", "q_rope", "W_UK", "W_UV", "cu_seqlens")}
    out = torch.empty((N, spec.H, spec.Dv), dtype=torch.bfloat16, device=dev)
    ws_bytes = mla.mla_prefill_workspace_size(N, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call(q_nope=t["q_nope"], q_rope=t["q_rope"], ckr=t["ckr"]):
        mla.mla_prefill_attn(ckr, q_nope, q_rope, t["W_UK"], t["W_UV"], t["cu_seqlens"], pin["cu_seqlens"], B,
                             spec.scale, out, ws, ws_bytes, d, stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    mla.mla_check_status()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        for e0, e1 in ev:
            e0.record(stream)
            call()
            e1.record(stream)
        torch.cuda.synchronize()
    mla.mla_check_status()
    ms = [a.elapsed_time(b) for a, b in ev]
    ms_per_step = float(np.mean(ms))
    fl = wl.prefill_flops(spec, pin["seq_lens"])
    total = fl["up"] + fl["attention"]
    peaks, peak_src = load_peaks()
    achieved = total / (ms_per_step / 1e3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": achieved / peaks["bf16_tflops"], "traffic": None,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback",
            "kernel": "mla_prefill_attn (tcgen05 up-projection GEMMs + causal attention), the whole call",
            "algorithmic_flops_per_launch": total, "flops_up_projection": fl["up"],
            "flops_attention": fl["attention"], "roofline_ms": 1e3 * total / (peaks["bf16_tflops"] * 1e12),
            "frac_vs_spec": total / (ms_per_step / 1e3) / 1e12 / SPEC_PEAKS["bf16_tflops"]}
    # end to end: the step's queries and rows from pinned host memory, the output back
    host_in = {k: torch.from_numpy(np.ascontiguousarray(pin[k]).view(np.int16)).pin_memory()
               for k in ("ckr", "q_nope", "q_rope")}
    host_out = torch.empty((N, spec.H, spec.Dv), dtype=torch.int16).pin_memory()
    e2e_ms = 0.0
    for k in range(args.steps + 3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for name in ("ckr", "q_nope", "q_rope"):
            t[name].view(torch.int16).copy_(host_in[name], non_blocking=True)
        call()
        host_out.copy_(out.view(torch.int16), non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        if k >= 3:
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms /= args.steps
    h2d = sum(x.numel() * x.element_size() for x in host_in.values())
    cpu = None
    if not args.no_cpu_baseline:
        f, sec, desc = prefill_oracle_sample(spec, pin, args.cpu_budget)
        cpu = {"value": f / sec / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle", "sample": desc,
               "seconds": sec}
    lens = pin["seq_lens"]
    line = {"metric": PREFILL_METRIC, "value": achieved, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": spec.name, "B": B, "H": spec.H, "kv_lora_rank": spec.R, "rope_dim": spec.Dr,
                       "D_nope": spec.Dn, "D_v": spec.Dv, "seq_lens": f"{int(lens[0])} each" if len(set(lens)) == 1
                       else "ragged", "tokens": N,
                       "l2": "inputs larger than L2 (the queries alone are "
                             f"{N * spec.H * (spec.Dn + spec.Dr) * 2 / 1e6:.0f} MB); no flush"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": total / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": host_out.numel() * 2, "ms_per_step": e2e_ms,
                    "mode": "one step at a time: rows and queries in, output out"},
            "gpu_launches": 3 * args.steps, "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


def run_prefill_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    from inputs import workloads as wl
    spec = wl.WORKLOADS[args.workload]
    pin = wl.prefill_inputs(spec, seed=0)
    for _ in range(args.warmup):
        prefill_oracle_sample(spec, pin, 1.0)
    tot_f, tot_t, desc = 0, 0.0, ""
    for _ in range(args.steps):
        f, sec, desc = prefill_oracle_sample(spec, pin, 4.0)
        tot_f += f
        tot_t += sec
    value = tot_f / tot_t / 1e12
    line = {"metric": PREFILL_METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "B": spec.B, "H": spec.H},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"per step: {desc}"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="cache format: bf16 rows, or E4M3 codes with per-token scales")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--device-only", action="store_true",
                    help="profiling only: time the device-resident steps, skip the end-to-end section")
    ap.add_argument("--seqs", type=int, default=0,
                    help="profiling only: run the first N sequences of the workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    prefill = args.workload.startswith("prefill")
    if args.impl == "reference":
        return run_prefill_reference(args) if prefill else run_reference(args)
    return run_prefill(args) if prefill else run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
