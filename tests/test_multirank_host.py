"""The N > 1 path of bench.py on the CPU: world-size-2 `gloo` process groups.

The layer has no exchange step, so `bench.py --gpus N` runs N independent
replicas (one batch per rank per step); the only collective steps are the
barrier and the maximum of the ranks' device times, and the whole-job
throughput is all ranks' tokens over the slowest rank's time.  These tests run
that host logic with two processes and no GPU, and check that the reference
arm runs on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import numpy as np
import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # this rank's device ms for the timed steps, e2e and graph legs
        mine = torch.tensor([100.0 + 7.0 * rank, 80.0 - 5.0 * rank, 0.0], dtype=torch.float64)
        out = bench.max_over_ranks(mine.clone(), world)
        q.put((rank, out.tolist(), bench.whole_job_tokens_per_s(world, 32, 50, float(out[0]))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(2):
            rank, vals, tps = q.get(timeout=120)
            got[rank] = (vals, tps)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    # every rank sees the element-wise maximum: timed 107 ms (rank 1), e2e 80 ms (rank 0)
    for rank in (0, 1):
        vals, tps = got[rank]
        assert vals == [107.0, 80.0, 0.0]
        assert tps == pytest.approx(2 * 32 * 50 / 0.107)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    import torch
    v = torch.tensor([3.0, 4.0])
    assert bench.max_over_ranks(v, 1) is v
    assert bench.whole_job_tokens_per_s(1, 8, 10, 40.0) == pytest.approx(2000.0)


def test_replicas_get_distinct_batches():
    wl = synth.workload("olmoe_like")
    a = synth.make_tokens(wl, 8, stream=0)
    b = synth.make_tokens(wl, 8, stream=1)
    assert a.shape == b.shape and not np.array_equal(a, b)
    assert np.array_equal(a, synth.make_tokens(wl, 8, stream=0))


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_runs_on_rank_zero_only(rank):
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--gpus", "2", "--workload", "tiny",
           "--tokens", "4", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    if rank == 0:
        assert len(lines) == 1
        d = json.loads(lines[0])
        assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle"
        assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    else:
        assert lines == []
