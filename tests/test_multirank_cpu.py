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


# ---------------------------------------------------------------- failure detection on the host

def _hb_worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mhc_residual_stream_b200 import tp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    hb = tp.Heartbeat(rank, world)
    try:
        for t in range(3):
            if t > 0:
                hb.require(t - 1, timeout_s=10.0)
            if rank == world - 1 and t == 2:
                q.put((rank, "left", None))  # this rank stops between rounds
                return
            hb.beat(t)
        try:
            hb.require(2, timeout_s=1.0)
            q.put((rank, "all reached", None))
        except tp.PeerLost as e:
            q.put((rank, "lost", (e.ranks, e.round)))
        # the survivors end together (rank 0 hosts the store): a count on the store
        import time
        store = dist.distributed_c10d._get_default_store()
        store.add("mhc/test/done", 1)
        deadline = time.monotonic() + 30
        while store.add("mhc/test/done", 0) < world - 1 and time.monotonic() < deadline:
            time.sleep(0.01)
    finally:
        dist.destroy_process_group()


def test_heartbeat_names_a_rank_that_stopped():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_hb_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[world - 1][1] == "left"
    for rank, what, info in got[:world - 1]:
        assert what == "lost" and info == ([world - 1], 2), (rank, what, info)


def _late_worker(rank, world, port, q):
    import datetime
    import time

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mhc_residual_stream_b200 import tp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=3))
    try:
        if rank == 1:
            time.sleep(8)  # never joins the handle exchange
            q.put((rank, "absent", 0.0))
            return
        t0 = time.monotonic()
        try:
            tp.exchange(bytes(72), (4, 64))
            q.put((rank, "no error", time.monotonic() - t0))
        except Exception as e:  # the group's timeout ends the collective with an error
            q.put((rank, type(e).__name__, time.monotonic() - t0))
    finally:
        dist.destroy_process_group()


def test_exchange_errors_when_a_rank_never_joins():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_late_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
    rank0 = got[0]
    assert rank0[1] != "no error" and rank0[2] < 30.0, rank0


# ---------------------------------------------------------------- mailbox rounds (host logic)

def test_peer_mailbox_round_checks_and_reset(monkeypatch):
    # one gloo rank in this process; the library calls are replaced by recorders,
    # so only the host bookkeeping runs
    import torch
    import torch.distributed as dist
    from mhc_residual_stream_b200 import mhc as M
    from mhc_residual_stream_b200 import tp
    calls = []
    monkeypatch.setattr(M, "new_mailbox", lambda W, R, H, device=None: torch.zeros(64, dtype=torch.uint8))
    monkeypatch.setattr(M, "ipc_export", lambda t: bytes(72))
    monkeypatch.setattr(M, "mhc_mailbox_publish", lambda x, rank, r, ptrs, mr, stream=None: calls.append(("pub", r)))
    monkeypatch.setattr(M, "mhc_boundary_collect", lambda mb, W, mr, r, *a, **k: calls.append(("col", r)))
    monkeypatch.setattr(M, "mhc_mailbox_init", lambda mb, stream=None: calls.append(("init",)))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        hb = tp.Heartbeat(0, 1)
        box = tp.PeerMailbox(4, 64, heartbeat=hb)
        x, args = torch.zeros(4, 64), (torch.zeros(4, 4, 64),) + (None,) * 7
        box.publish(x, 0)
        box.publish(x, 1)
        with pytest.raises(RuntimeError):
            box.publish(x, 2)          # rounds 0 and 1 both uncollected: the mailbox holds two
        with pytest.raises(RuntimeError):
            box.collect(1, *args)      # round 0 first
        box.collect(0, *args)
        box.publish(x, 2)
        with pytest.raises(RuntimeError):
            box.publish(x, 4)          # round 3 skipped
        box.collect(1, *args)
        with pytest.raises(RuntimeError):
            box.collect(2, torch.zeros(3, 4, 64), *args[1:])  # 4 rows published, 3 collected
        box.collect(2, *args)
        with pytest.raises(RuntimeError):
            box.collect(3, *args)      # not published by this rank
        assert hb.reached() == [2]
        box.reset()                    # an aborted step: rounds restart at 0
        assert hb.epoch == 1 and hb.reached() == [-1]
        box.publish(x, 0)
        assert calls == [("pub", 0), ("pub", 1), ("col", 0), ("pub", 2), ("col", 1), ("col", 2), ("init",),
                         ("pub", 0)]
    finally:
        dist.destroy_process_group()
