"""Tensor-parallel boundary: every rank of a TP group sums all ranks' partials
itself, reading the peers' buffers with plain loads over NVLink.

On the pages the sublayers' outputs are TP partials and the boundary's fused
kernel does the all-reduce ([boundary] Boundaries.post_only:
tensor_model_parallel_all_reduce then mhc_post; [all_reduce]
BoundaryAllReduce.__call__, through a multicast mailbox). Here each rank
exports its partial buffer once (CUDA IPC), maps every peer's, and passes the
table of the group's buffers, in rank order, to mhc_boundary_post_pre_ptrs:
one launch per rank reads the R x H partial of every rank and computes the
whole boundary for every row (the result is the same on every rank, as after
an all-reduce). Ordering is the caller's: the group's partials must be
complete before the boundaries read them and must not be overwritten until all
have read them (``barrier`` below is the plain host form of both). Nothing
here uses multicast.

PeerMailbox is the publish/collect form ([all_reduce] publish_target /
mark_published): producers store their rows, negative zero cleared, into every
rank's mailbox, whose unwritten elements hold negative zero; each rank's
boundary re-reads its own mailbox's elements until they are written, so the
group needs no barrier between a sublayer and the boundary.
"""

from __future__ import annotations

import time
from typing import List, Optional

import torch
import torch.distributed as dist

from . import mhc as M


def exchange(handle: bytes, shape, group=None) -> List:
    """Every rank's (handle, shape), in rank order; the shapes must agree."""
    gathered: List = [None] * dist.get_world_size(group)
    dist.all_gather_object(gathered, (handle, tuple(shape)), group=group)
    for _, sh in gathered:
        if tuple(sh) != tuple(shape):
            raise ValueError(f"partial shapes differ across the group: {sh} vs {tuple(shape)}")
    return gathered


def partial_table(rank: int, local_ptr: int, gathered: List, import_fn):
    """Device addresses of the group's partials in rank order: this rank's own
    buffer, the peers' mapped through import_fn. Returns (table, imported)."""
    table, imported = [], []
    for r, (h, _) in enumerate(gathered):
        if r == rank:
            table.append(int(local_ptr))
        else:
            a = import_fn(h)
            imported.append(a)
            table.append(a)
    return table, imported


class PeerLost(RuntimeError):
    """Peers of the group that did not reach a round in time (host-side check)."""

    def __init__(self, ranks, round_):
        super().__init__(f"ranks {sorted(ranks)} did not reach round {round_}")
        self.ranks = sorted(ranks)
        self.round = round_


class Heartbeat:
    """Host-side liveness of a group through a c10d store (the process group's by
    default): each rank posts the last round it reached, and before work that
    reads peers' memory a rank checks, with a time limit, that every peer has
    reached a given round, raising PeerLost otherwise. A rank that died or left
    is thus noticed on the host before the next launch instead of by a device
    wait running out; nothing here touches the GPU."""

    def __init__(self, rank: int, world: int, store=None, prefix: str = "mhc/heartbeat"):
        self.store = store if store is not None else dist.distributed_c10d._get_default_store()
        self.rank, self.world, self.prefix = rank, world, prefix
        self.epoch = 0  # advanced by every rank together when rounds restart

    def _key(self, r: int) -> str:
        return f"{self.prefix}/{self.epoch}/{r}"

    def next_epoch(self):
        """Rounds restart at 0 (every rank calls this at the same point)."""
        self.epoch += 1

    def beat(self, round_: int):
        """This rank has reached `round_`."""
        self.store.set(self._key(self.rank), str(int(round_)))

    def reached(self) -> List[int]:
        """The last round every rank posted (-1 where none yet)."""
        out = []
        for r in range(self.world):
            k = self._key(r)
            out.append(int(self.store.get(k).decode()) if self.store.check([k]) else -1)
        return out

    def require(self, round_: int, timeout_s: float = 5.0, poll_s: float = 0.01):
        """Wait until every peer has reached `round_`; PeerLost after `timeout_s`."""
        deadline = time.monotonic() + timeout_s
        while True:
            seen = self.reached()
            missing = [r for r in range(self.world) if r != self.rank and seen[r] < round_]
            if not missing:
                return
            if time.monotonic() >= deadline:
                raise PeerLost(missing, round_)
            time.sleep(poll_s)


class PeerPartials:
    """The group's partial buffers [R, H] bf16, one per rank, mapped on every rank."""

    def __init__(self, local: torch.Tensor, group: Optional[dist.ProcessGroup] = None):
        if not local.is_cuda or local.dtype != torch.bfloat16 or local.dim() != 2 or not local.is_contiguous():
            raise ValueError("the local partial must be a contiguous bf16 [R, H] CUDA tensor")
        self.local = local
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        gathered = exchange(M.ipc_export(local), tuple(local.shape), group)
        self.ptrs, self._imported = partial_table(self.rank, local.data_ptr(), gathered, M.ipc_import)

    def barrier(self):
        """Host-side ordering of the group: all work queued on this device so far
        is complete and every rank has reached this point."""
        torch.cuda.current_stream(self.local.device).synchronize()
        dist.barrier(group=self.group)

    def close(self):
        for a in self._imported:
            M.ipc_release(a)
        self._imported = []
        self.ptrs = []

    def boundary(self, residual, post, comb, pre, norm_weight, norm_eps, coeffs, residual_out, **kw):
        """mhc_boundary_post_pre over the group's partials (all ranks, rank order)."""
        M.mhc_boundary_post_pre_ptrs(self.ptrs, residual, post, comb, pre, norm_weight, norm_eps, coeffs,
                                     residual_out, **kw)


def _sync(device):
    """Wait for the work queued on `device` (nothing to wait for off the GPU)."""
    if torch.device(device).type == "cuda":
        torch.cuda.current_stream(device).synchronize()


class PeerMailbox:
    """Publish/collect over the group: each rank's mailbox lives in its own memory
    and is mapped by every other rank; producers store their rows into every
    mailbox, and each rank's boundary reads the slots of its own mailbox as they
    fill (an element is written once it is not negative zero), so no host barrier
    sits between the sublayer and the boundary.

    Rounds are checked on the host before anything is launched ([all_reduce]
    mark_published / reset keep the same kind of state): this rank publishes
    rounds 0, 1, 2, ... in order, at most one round ahead of its collects, and
    collects only a round it has published, in order, over as many rows as it
    published in that round (slots past the rows a collect reads would keep
    their values, and a later round of the same parity would take them for
    fresh ones). `reset` drops what an aborted step left behind, on every rank
    of the group together."""

    def __init__(self, max_rows: int, hidden: int, group: Optional[dist.ProcessGroup] = None, device=None,
                 heartbeat: Optional[Heartbeat] = None):
        self.group = group
        self.heartbeat = heartbeat
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.max_rows = max_rows
        self.local = M.new_mailbox(self.world, max_rows, hidden, device)
        _sync(self.local.device)  # initialised before anyone maps it
        gathered = exchange(M.ipc_export(self.local), tuple(self.local.shape), group)
        self.ptrs, self._imported = partial_table(self.rank, self.local.data_ptr(), gathered, M.ipc_import)
        self.published = -1  # the last round this rank published
        self.collected = -1  # the last round this rank collected
        self.rows = {}  # round -> rows this rank published in it (the rounds not yet collected)

    def publish(self, x: torch.Tensor, round_: int, stream=None):
        """This rank's contribution of round `round_` into every rank's mailbox.
        With a heartbeat: every peer must have reached the previous round (its
        mailbox is still served), then this rank posts this one."""
        if round_ != self.published + 1:
            raise RuntimeError(f"round {round_} published out of order (last published {self.published})")
        if round_ > self.collected + 2:
            raise RuntimeError(f"round {round_} published while round {self.collected + 1} is still uncollected "
                               "(a mailbox holds two rounds)")
        if self.heartbeat is not None and round_ > 0:
            self.heartbeat.require(round_ - 1)
        M.mhc_mailbox_publish(x, self.rank, round_, self.ptrs, self.max_rows, stream)
        self.published = round_
        self.rows[round_] = int(x.shape[0])
        if self.heartbeat is not None:
            self.heartbeat.beat(round_)

    def collect(self, round_: int, residual, post, comb, pre, norm_weight, norm_eps, coeffs, residual_out, **kw):
        """This rank's boundary of round `round_` over the group's contributions."""
        if round_ != self.collected + 1 or round_ > self.published:
            raise RuntimeError(f"round {round_} collected out of order (last collected {self.collected}, "
                               f"last published {self.published})")
        if int(residual.shape[0]) != self.rows[round_]:
            raise RuntimeError(f"round {round_} collected over {int(residual.shape[0])} rows, "
                               f"published over {self.rows[round_]}")
        M.mhc_boundary_collect(self.local, self.world, self.max_rows, round_, residual, post, comb, pre, norm_weight,
                               norm_eps, coeffs, residual_out, **kw)
        self.collected = round_
        del self.rows[round_]

    def reset(self, stream=None):
        """Drop the rounds an aborted step left published but uncollected: every
        rank of the group calls this together; afterwards rounds restart at 0.
        The group first finishes the work it has queued (no producer may still
        be storing into a mailbox), then each rank re-initialises its own."""
        _sync(self.local.device)
        dist.barrier(group=self.group)
        M.mhc_mailbox_init(self.local, stream)
        _sync(self.local.device)
        dist.barrier(group=self.group)
        self.published = self.collected = -1
        self.rows = {}
        if self.heartbeat is not None:
            self.heartbeat.next_epoch()

    def close(self):
        for a in self._imported:
            M.ipc_release(a)
        self._imported = []
        self.ptrs = []
