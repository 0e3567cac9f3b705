"""Host logic of bench.py: byte accounting of the grouped layer and the
multi-rank timing (barrier, max over ranks, whole-job aggregate) on two gloo
ranks on the CPU."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import workloads


def _group(d_in, d_outs, seed=0):
    rng = np.random.default_rng(seed)
    x = workloads.draw_vector(rng, d_in, "laplace")
    th = {0.5: workloads.quantile_threshold(x, 0.5)}
    return [workloads.Projection(f"p{i}", workloads.draw_weight(rng, d_in, d, 0.02), x, th)
            for i, d in enumerate(d_outs)]


def test_group_bytes_counts_shared_input_once():
    g = _group(64, (16, 8, 24))
    nnz = bench.kept_count(g[0], 0.5)
    assert nnz == int((np.abs(g[0].x.astype(np.float64)) >= g[0].thresholds[0.5]).sum())
    # kept rows of the three weights (2 bytes each), x once, the three y's
    assert bench.group_bytes(g, nnz) == nnz * 2 * 48 + 2 * 64 + 2 * 48
    assert bench.layer_bytes([g, g[:1]], 0.5) == (bench.group_bytes(g, nnz)
                                                  + bench.group_bytes(g[:1], nnz))


def test_layer_groups_follow_the_decoder_wiring():
    names = [n for n, _, _ in workloads.LLAMA2_7B_PROJECTIONS]
    assert sorted(sum(map(list, bench.GROUPS), [])) == sorted(names)
    for g in bench.GROUPS:
        shapes = {d_in for n, d_in, _ in workloads.LLAMA2_7B_PROJECTIONS if n in g}
        assert len(shapes) == 1          # one shared input per launch


def test_aggregate_uses_the_slowest_rank():
    v, slow = bench.aggregate(100.0, [0.5, 2.0, 1.0], 3)
    assert slow == 2.0 and v == pytest.approx(150.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        secs = [0.25, 1.75][rank]
        bench.barrier(world)
        slow = bench.max_over_ranks(secs, world)
        units = 10.0
        value = units * world / slow
        out.put((rank, slow, value))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, slow, value in got:
        assert slow == 1.75                        # every rank sees the slowest time
        assert value == pytest.approx(20.0 / 1.75)  # all ranks' units over it


def test_warmup_is_at_least_three_steps(monkeypatch):
    for given, run in (("0", 3), ("1", 3), ("3", 3), ("7", 7)):
        monkeypatch.setattr("sys.argv", ["bench.py", "--steps", "5", "--warmup", given])
        args = bench.parse()
        assert args.warmup == run and args.steps == 5
