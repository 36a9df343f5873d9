"""Host logic of the multi-GPU bench path on CPU: world_size 2 over gloo.

The boundary shards by independent decode batches (replicas); the only
cross-rank steps are the barrier around the timed region and the max over
ranks of the device time. These run here as two gloo processes."""

import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        elapsed = [3.0, 5.0][rank]  # rank 1 is the slower one
        ms = bench.max_over_ranks(elapsed, world)
        q.put((rank, ms, bench.aggregate_us_per_boundary(ms, 1000, world)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, us in got:
        assert ms == 5.0                    # every rank sees the slowest rank's time
        assert us == 5.0 * 1000 / (1000 * 2)  # units of both ranks over that time


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


# ---------------------------------------------------------------- TP partial table (host logic)

def _tp_worker(rank, world, port, q, bad_shape):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mhc_residual_stream_b200 import tp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        handle = bytes([rank]) * 72                     # stands in for an exported IPC handle
        shape = (4, 64 + (64 if bad_shape and rank == 1 else 0))
        try:
            gathered = tp.exchange(handle, shape)
        except ValueError:
            q.put((rank, "shape mismatch"))
            return
        imported = []

        def fake_import(h):                               # maps a peer's handle to a fake address
            imported.append(h[0])
            return 0x10000 * (h[0] + 1)

        table, mapped = tp.partial_table(rank, 0xABC0, gathered, fake_import)
        q.put((rank, table, mapped, imported))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bad_shape", [False, True])
def test_tp_partial_table_gloo(bad_shape):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, q, bad_shape)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted((q.get(timeout=5) for _ in range(world)), key=lambda t: t[0])
    if bad_shape:
        assert all(g[1] == "shape mismatch" for g in got)  # every rank refuses, none maps anything
        return
    for rank, table, mapped, imported in got:
        # rank order; this rank's own buffer in its slot; every peer mapped once
        assert table == [0xABC0 if r == rank else 0x10000 * (r + 1) for r in range(world)]
        assert sorted(imported) == [r for r in range(world) if r != rank]
        assert mapped == [0x10000 * (r + 1) for r in range(world) if r != rank]
