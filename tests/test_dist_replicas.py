"""The N > 1 path of bench.py on CPU: two gloo ranks.

The layer needs no exchange between GPUs, so `bench.py --gpus N` runs one
independent replica per rank (weak scaling).  What crosses ranks is host
plumbing only, and that is what these tests run:
- the step time is the slowest rank's (max over ranks), and every rank
  gets the same value;
- the whole-job throughput is world x per-rank work / that time;
- replicas draw distinct seeded inputs (rank-dependent seed offsets);
- the reference arm (the oracle) runs on rank 0 only; other ranks exit
  without output.
"""
import contextlib
import datetime
import hashlib
import io
import os
import socket
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from mixed_precision_weight_b200 import synth
        ms = [3.0, 5.0, 4.0, 2.0][rank]
        slow = bench.max_over_ranks(ms, world, "cpu")
        value = bench.job_throughput(world, 2.0e9, slow, 1e9)
        # the replica's own seeded input, as the workloads draw it
        wl = synth.WORKLOADS["tiny"]
        w = wl.weight(seed_offset=100 * rank)
        digest = hashlib.sha256(w.float().numpy().tobytes()).hexdigest()
        # the reference arm: rank > 0 returns at once and prints nothing
        out = io.StringIO()
        if rank > 0:
            with contextlib.redirect_stdout(out):
                ret = bench.run_reference(types.SimpleNamespace(steps=1, warmup=0), world, rank)
            ref_silent = ret is None and out.getvalue() == ""
        else:
            ref_silent = True
        dist.barrier()
        q.put((rank, slow, value, digest, ref_silent))
    finally:
        dist.destroy_process_group()


def _run(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


@pytest.mark.parametrize("world", [2])
def test_replicas_time_throughput_and_seeds(world):
    res = _run(world)
    slowest = max([3.0, 5.0, 4.0, 2.0][:world])
    for rank, slow, value, _, ref_silent in res:
        assert slow == slowest                       # every rank holds the max
        assert value == pytest.approx(world * 2.0e9 / (slowest * 1e-3) / 1e9)
        assert ref_silent
    digests = {d for _, _, _, d, _ in res}
    assert len(digests) == world                     # distinct inputs per replica


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_throughput(1, 17.6e6, 0.01, 1e9) == pytest.approx(1760.0)
