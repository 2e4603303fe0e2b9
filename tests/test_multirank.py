"""World-size-2 gloo checks of bench.py's multi-rank logic on CPU: every rank draws its own
independent problem (weak scaling, no data-path collective) and the step time is the max
over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from block_sparse_attention_42_b200 import inputs
        w = inputs.Workload("mr", 1, 2, 1, 256, 64, 64, "bf16", 0.25, "stem", 5)
        d = inputs.make_inputs(w, device="cpu", seed_offset=rank)
        digest = float(d["q"].float().sum())
        mx = bench.reduce_max(10.0 + rank, world, "cpu")
        val = bench.whole_job_tflops(1e12, world, 1000.0)
        q.put((rank, digest, mx, val))
    finally:
        dist.destroy_process_group()


def test_two_ranks_independent_problems_and_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, d0, m0, v0), (r1, d1, m1, v1) = res
    assert d0 != d1                      # each rank has its own problem
    assert m0 == m1 == 11.0              # max over ranks, identical on every rank
    assert v0 == v1 == pytest.approx(2.0)  # 2 ranks x 1 TFLOP in 1 s
