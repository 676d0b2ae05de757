"""The multi-rank plumbing of bench.py on CPU: two gloo ranks agree on the
max of their per-rank times, and the whole-job throughput is computed from
that max (weak scaling: every rank runs its own replica)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 2.0 + rank * 1.5          # rank 1 is the slow one
        m = bench.reduce_max(local_ms)
        dist.barrier()
        out[rank] = (m, bench.aggregate_throughput(8192, world, m))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_aggregate():
    ctx = mp.get_context("spawn")
    world, port = 2, _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    for r in range(world):
        m, v = res[r]
        assert m == pytest.approx(3.5)
        assert v == pytest.approx(2 * 8192 / 3.5e-3)


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(1.25) == 1.25
    assert bench.aggregate_throughput(100, 1, 2.0) == pytest.approx(50000.0)


def test_cpu_backward_baseline_runs_on_a_small_sample():
    """The backward's CPU baseline (the fp64 oracle on a bounded sample) runs
    on the host and reports tokens/s of all heads."""
    sys.path.insert(0, ROOT)
    import bench
    from linear_attention_recurrence_gdr2_b200 import inputs as gen
    inp = gen.make_inputs(2, 40, 4, 16, 16, "bf16", seed=3, init_std=0.1)
    d_o, _ = gen.cotangents(inp)
    r = bench.cpu_backward_baseline(inp, d_o, "tiny", tokens=32, heads=2)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s" and r["value"] > 0
    assert "first 32 tokens, 2 of 4 heads" in r["sample"]


def test_cpu_backward_baseline_stays_in_the_first_packed_sequence():
    sys.path.insert(0, ROOT)
    import bench
    from linear_attention_recurrence_gdr2_b200 import inputs as gen
    inp = gen.make_inputs(1, 0, 2, 16, 16, "fp32", seed=4, init_std=0.1, lengths=[20, 50])
    d_o, _ = gen.cotangents(inp)
    r = bench.cpu_backward_baseline(inp, d_o, "tiny packed", tokens=512, heads=1)
    assert "first 20 tokens" in r["sample"]
