"""The N > 1 path of the benchmark on CPU: two gloo ranks, each an
independent replica of the same seeded workload (no data-path collective),
combined by the max-over-ranks timing rule; each rank replays its replica's
requests on its own host allocator and all ranks must agree."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _replica_digest(plan):
    """SHA-256 of the block tables, slots and copy-on-write pairs the
    library's host allocator gives this workload's requests."""
    import hashlib

    import numpy as np

    import paged_kv_cache_351_b200 as pa
    from workloads import AddOp, ForkOp

    w = plan.workload
    alloc = pa.Allocator(plan.num_blocks, w.block_size, plan.free_order)
    h = hashlib.sha256()
    for op in list(plan.setup_ops) + list(plan.step_ops):
        if isinstance(op, AddOp):
            alloc.add(op.seq)
        elif isinstance(op, ForkOp):
            alloc.fork(op.parent, op.child)
        else:
            slots, cows = alloc.append(op.seq, op.n)
            h.update(np.asarray(slots, dtype=np.int64).tobytes())
            h.update(np.asarray(cows, dtype=np.int64).tobytes())
    tables, lens = alloc.block_tables(list(plan.batch), plan.max_blocks_per_seq)
    h.update(np.asarray(tables, dtype=np.int32).tobytes())
    h.update(np.asarray(lens, dtype=np.int32).tobytes())
    return h.hexdigest()


def _worker(rank, world, port, q):
    import bench
    from workloads import make_plan

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        plan = make_plan("llama7b_bs64")
        nbytes = bench.step_bytes(plan)
        # each replica holds the same workload: identical bytes per step
        t = torch.tensor([float(nbytes["step"])], dtype=torch.float64)
        lo, hi = t.clone(), t.clone()
        dist.all_reduce(lo, op=dist.ReduceOp.MIN)
        dist.all_reduce(hi, op=dist.ReduceOp.MAX)
        mx = bench.max_over_ranks([1.0 + rank, 10.0 - rank], "cpu", world)
        val = bench.aggregate_value(nbytes["step"], mx[0], world)
        # each rank replays its replica's requests on its own host allocator
        # (the library's C++ allocator): the block tables, slots and memory
        # report must come out identical on every rank
        forks = make_plan("parallel_sampling_13b")  # forks and copy-on-write
        rep = (bench.allocator_report(plan), bench.allocator_report(forks))
        digest = (_replica_digest(plan), _replica_digest(forks))
        gathered = [None] * world
        dist.all_gather_object(gathered, (rep, digest))
        q.put((rank, float(lo), float(hi), mx, val, nbytes["step"], gathered))
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, lo, hi, mx, val, nb, gathered in res:
        assert lo == hi == nb
        assert mx == [2.0, 10.0]  # max over ranks of each value
        assert val == pytest.approx(nb * world / 2.0e-3 / 1e9)
        assert len(gathered) == world
        assert all(g == gathered[0] for g in gathered)
        assert gathered[0][0][0]["blocks_used"] > 0
        assert gathered[0][0][1]["cow_copies"] > 0


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks([3.0, 4.0], "cpu", 1) == [3.0, 4.0]
    assert bench.aggregate_value(1e9, 1.0, 1) == pytest.approx(1000.0)
