"""Replica path of bench.py with two ranks on the CPU (gloo): every rank decodes its own
batch, and the line's throughput is the sum of the ranks' work over the slowest rank's
time. These are the host-side steps of `bench.py --gpus N` (no GPU, no kernel)."""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp

WORLD = 2
WORKLOAD = "deepseek_h128_b128_ragged"


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from inputs import workloads as wl

        spec = wl.WORKLOADS[WORKLOAD]
        lens = wl.seq_lens_of(spec, rank)            # the batch bench.py gives rank r: seed r
        local = (wl.cache_bytes(spec, lens), wl.attention_flops(spec, lens), int(lens.sum()))
        local_ms = 100.0 + 25.0 * rank               # a slower second rank
        sums, maxes = bench.reduce_over_ranks(WORLD, torch.device("cpu"), local, (local_ms,))
        # the same collectives again with only maxima, as the end-to-end leg does
        _, (e2e_max,) = bench.reduce_over_ranks(WORLD, torch.device("cpu"), (), (local_ms * 2,))
        cfg = bench.workload_config(spec, {"seq_lens": lens}, type("A", (), {"gpus": WORLD, "seqs": 0})(),
                                    job_tokens=sums[2])
        out.put((rank, local, local_ms, sums, maxes, e2e_max, cfg))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(WORLD):
            r = out.get(timeout=180)
            res[r[0]] = r
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    return res


def test_ranks_decode_different_batches(ranks):
    assert ranks[0][1] != ranks[1][1]


def test_job_work_is_the_sum_and_time_the_max_over_ranks(ranks):
    want_sums = [float(ranks[0][1][i] + ranks[1][1][i]) for i in range(3)]
    for r in range(WORLD):
        _, _, _, sums, maxes, e2e_max, _ = ranks[r]
        assert sums == want_sums                      # every rank sees the job's totals
        assert maxes == [max(ranks[0][2], ranks[1][2])]
        assert e2e_max == 2 * max(ranks[0][2], ranks[1][2])


def test_line_throughput_counts_every_rank(ranks):
    steps = 7
    job_bytes, _, _ = ranks[0][3]
    (t_max,) = ranks[0][4]
    value = job_bytes * steps / (t_max / 1e3) / 1e9
    # rank 0's bytes times the world size would misstate a job whose ranks hold ragged batches
    wrong = WORLD * ranks[0][1][0] * steps / (t_max / 1e3) / 1e9
    assert value != pytest.approx(wrong, rel=1e-6)
    assert value == pytest.approx(sum(ranks[r][1][0] for r in range(WORLD)) * steps / (t_max / 1e3) / 1e9)


def test_config_describes_the_whole_job(ranks):
    cfg = ranks[0][6]
    assert cfg["global_batch"] == WORLD * cfg["B"]
    assert cfg["cached_tokens_all_ranks"] == ranks[0][1][2] + ranks[1][1][2]
    assert "seed = rank" in cfg["seq_lens"]
    assert cfg["parallelism"].startswith(f"replicas x{WORLD}")
