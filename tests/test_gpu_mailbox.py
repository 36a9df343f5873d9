"""The publish/collect mailbox of the tensor-parallel boundary on one GPU.

* One process plays every producer and every consumer of a group on one stream:
  each round every producer publishes, then every consumer collects. Each
  collect must give bitwise the results of the strided entry over the same
  partials (the same sum order), over four rounds, so both parities are used
  twice and the flow control of round t + 2 sees round t consumed; the row
  count varies from round to round below the mailbox's capacity.
* The mailbox words: after round t the consumed word of parity t & 1 reads
  t + 1, and every slot element of both parities is back to negative zero.
* A published negative zero arrives as positive zero.
* A collect of a round nobody published runs out of its (shortened) wait,
  records MHC_ERR_DEVICE_TIMEOUT in the workspace and leaves the round
  unconsumed, so that the producer of the round two later runs out of its own
  wait and reports it too; after a reset the rounds go through. A publish two rounds ahead of
  a consumer runs out of its wait, writes nothing and records the timeout in the
  producer's own mailbox. Both are waits on words that nothing writes.
* Two processes on the same GPU form a gloo group of 2 and exchange mailboxes
  through CUDA IPC (PeerMailbox, with a host heartbeat). Each round both
  publish, a host barrier follows, then both collect: every wait is satisfied
  when its kernel starts, so no kernel waits on another that runs at the same
  time. After three rounds the group resets and replays round 0, which must
  give bitwise the first round 0.
"""

import datetime
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from mhc_residual_stream_b200 import mhc as M
from mhc_residual_stream_b200 import synthetic as S

from _parity import DEV, alloc_outputs, assert_bf16_close, check_tail, f64, gpu_post_pre, oracle_post_pre, to_dev

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = 256  # status word at byte 0, consumed words at bytes 8 and 12, then the slots
NEG_ZERO = 0x8000


def _consumed(mb: torch.Tensor):
    words = mb[:HEADER].cpu().view(torch.int32).numpy().view(np.uint32)
    return words[2:4].copy()


def _slots(mb: torch.Tensor, W: int, M_: int, H: int) -> np.ndarray:
    """The slot elements' bit patterns, [2][W][M][H] uint16."""
    return mb[HEADER:].cpu().view(torch.int16).numpy().view(np.uint16).reshape(2, W, M_, H).copy()


def _collect(mb, W, M_, t, d, g, packed=False):
    R, n, H = g["residual"].shape
    out = alloc_outputs(R, n, H)
    ws = M.new_workspace(R, H, n, DEV)
    M.mhc_boundary_collect(mb, W, M_, t, g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"],
                           d["norm_eps"], M.Coeffs.from_weights(d["coeff"], DEV, packed=packed),
                           out["residual_out"], layer_input=out["layer_input"],
                           mxfp8=(out["q_data"], out["q_scale"], True), post_out=out["post"], comb_out=out["comb"],
                           pre_out=out["pre"], workspace=ws)
    return out, ws


def _round_trip(mbs, W, M_, t, d, packed=False):
    """Every producer publishes d's partials as round t, every consumer collects;
    each consumer's results, compared bitwise with the strided entry."""
    g = to_dev({k: d[k] for k in ("residual", "post", "comb", "pre", "norm_weight")})
    xs = [d["partials"][u].to(DEV).contiguous() for u in range(W)]
    ptrs = [m.data_ptr() for m in mbs]
    for u in range(W):
        M.mhc_mailbox_publish(xs[u], u, t, ptrs, M_)
    outs = [_collect(mbs[c], W, M_, t, d, g, packed) for c in range(W)]
    torch.cuda.synchronize()
    ref = gpu_post_pre(d, packed=packed)
    for c, (out, ws) in enumerate(outs):
        assert M.mhc_get_device_status(ws) == M.OK, (t, c)
        for k, v in out.items():
            assert torch.equal(v.cpu(), ref[k]), (t, c, k)


@pytest.mark.parametrize("M_,H,n,W,packed,rows", [(32, 7168, 4, 2, True, (32, 32, 32, 32)),
                                                  (8, 192, 2, 3, False, (7, 3, 8, 1)),
                                                  (128, 512, 4, 16, False, (128, 5, 77, 128)),
                                                  (1, 64, 1, 1, False, (1, 1, 1, 1))])
def test_rounds_match_strided_bitwise(M_, H, n, W, packed, rows):
    from mhc_residual_stream_b200 import build
    build.build()
    mbs = [M.new_mailbox(W, M_, H, DEV) for _ in range(W)]
    torch.cuda.synchronize()
    for c in range(W):
        assert (_slots(mbs[c], W, M_, H) == NEG_ZERO).all() and (_consumed(mbs[c]) == 0).all()
    for t, R in enumerate(rows):
        d = S.draw_boundary(R, H, n=n, partials=W, seed=7100 + 10 * t + W)
        _round_trip(mbs, W, M_, t, d, packed)
        for c in range(W):
            assert M.mhc_get_device_status(mbs[c]) == M.OK  # no producer timed out
            done = _consumed(mbs[c])
            assert done[t & 1] == t + 1 and (t == 0 or done[(t - 1) & 1] == t), (t, c, done)
            assert (_slots(mbs[c], W, M_, H) == NEG_ZERO).all(), (t, c)  # every read element re-marked


def test_published_negative_zero_arrives_as_positive_zero():
    R, H, n, W = 4, 128, 2, 2
    d = S.draw_boundary(R, H, n=n, partials=W, seed=7150)
    mbs = [M.new_mailbox(W, R, H, DEV) for _ in range(W)]
    x = d["partials"][0].clone()
    x[1, 5] = -0.0
    x[2, :] = -0.0
    # publish only producer 0; then inspect consumer 1's slot before anyone collects
    M.mhc_mailbox_publish(x.to(DEV), 0, 0, [m.data_ptr() for m in mbs], R)
    torch.cuda.synchronize()
    slot = _slots(mbs[1], W, R, H)[0, 0]
    want = x.view(torch.int16).numpy().view(np.uint16).copy()
    want[want == NEG_ZERO] = 0
    assert np.array_equal(slot, want)
    assert (_slots(mbs[1], W, R, H)[0, 1] == NEG_ZERO).all()  # producer 1's slot untouched
    # the round completes as the strided entry on the cleared partials
    M.mhc_mailbox_publish(d["partials"][1].to(DEV).contiguous(), 1, 0, [m.data_ptr() for m in mbs], R)
    d["partials"][0] = torch.from_numpy(want.view(np.int16)).view(torch.bfloat16)
    g = to_dev({k: d[k] for k in ("residual", "post", "comb", "pre", "norm_weight")})
    outs = [_collect(mbs[c], W, R, 0, d, g) for c in range(W)]
    torch.cuda.synchronize()
    ref = gpu_post_pre(d)
    for out, ws in outs:
        assert M.mhc_get_device_status(ws) == M.OK
        for k, v in out.items():
            assert torch.equal(v.cpu(), ref[k]), k


def test_collect_of_unpublished_round_times_out_and_recovers():
    R, H, n, W = 4, 256, 4, 2
    d = S.draw_boundary(R, H, n=n, partials=W, seed=7201)
    g = to_dev({k: d[k] for k in ("residual", "post", "comb", "pre", "norm_weight")})
    mbs = [M.new_mailbox(W, R, H, DEV) for _ in range(W)]
    old = M.mhc_debug_set_wait(20_000_000, 0)  # 20 ms
    try:
        outs = [_collect(mbs[c], W, R, 0, d, g) for c in range(W)]
        for out, ws in outs:
            assert M.mhc_get_device_status(ws) == M.DEVICE_TIMEOUT
    finally:
        M.mhc_debug_set_wait(old, 0)
    for c, (out, ws) in enumerate(outs):
        assert M.mhc_get_device_status(ws) == M.OK  # reading cleared it
        # the collect gave up: round 0 stays unconsumed and its slots stay marked
        assert _consumed(mbs[c])[0] == 0 and (_slots(mbs[c], W, R, H) == NEG_ZERO).all()
    # round 1 (the other parity) goes through as usual
    _round_trip(mbs, W, R, 1, d)
    # a producer of round 2 (parity 0 again) finds round 0 unconsumed: its wait runs
    # out, it writes nothing and reports the timeout in its own mailbox
    before = [m.clone() for m in mbs]
    old = M.mhc_debug_set_wait(20_000_000, 0)
    try:
        M.mhc_mailbox_publish(d["partials"][0].to(DEV).contiguous(), 0, 2, [m.data_ptr() for m in mbs], R)
        torch.cuda.synchronize()
    finally:
        M.mhc_debug_set_wait(old, 0)
    assert M.mhc_get_device_status(mbs[0]) == M.DEVICE_TIMEOUT
    for m, b in zip(mbs, before):
        assert torch.equal(m, b)
    # after a reset of every mailbox the rounds start again from 0
    for m in mbs:
        M.mhc_mailbox_init(m)
    for t in (0, 1, 2):
        _round_trip(mbs, W, R, t, d)


def test_publish_ahead_of_consumer_times_out_and_writes_nothing():
    R, H, W = 3, 128, 2
    mbs = [M.new_mailbox(W, R, H, DEV) for _ in range(W)]
    fresh = [m.clone() for m in mbs]
    x = torch.randn(R, H, device=DEV).to(torch.bfloat16)
    old = M.mhc_debug_set_wait(20_000_000, 0)
    try:
        M.mhc_mailbox_publish(x, 0, 2, [m.data_ptr() for m in mbs], R)  # nobody consumed round 0
        torch.cuda.synchronize()
    finally:
        M.mhc_debug_set_wait(old, 0)
    assert M.mhc_get_device_status(mbs[0]) == M.DEVICE_TIMEOUT  # the producer's own mailbox
    assert M.mhc_get_device_status(mbs[1]) == M.OK
    for m, f in zip(mbs, fresh):
        assert torch.equal(m, f)  # no slot or consumed word written
    # once round 0 is consumed (here: published and collected), round 2 goes through
    d = S.draw_boundary(R, H, n=1, partials=W, seed=7301)
    d["partials"][0] = x.cpu()
    for t in (0, 2):
        _round_trip(mbs, W, R, t, d)
    assert M.mhc_get_device_status(mbs[0]) == M.OK


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


ROUNDS = 3


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mhc_residual_stream_b200 import mhc as M
    from mhc_residual_stream_b200 import synthetic as S
    from mhc_residual_stream_b200.tp import Heartbeat, PeerMailbox
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    box = None
    try:
        torch.cuda.set_device(0)
        R, H, n = 16, 7168, 4
        hb = Heartbeat(rank, world)  # each publish first requires the peer's previous round
        box = PeerMailbox(R, H, device="cuda:0", heartbeat=hb)  # capacity R
        for step in range(ROUNDS + 1):
            if step == ROUNDS:
                box.reset()  # as after an aborted step: rounds restart at 0
            t = step % ROUNDS
            d = S.draw_boundary(R, H, n=n, partials=world, seed=7400 + t)  # the same draw on both ranks
            x = d["partials"][rank].to("cuda:0").contiguous()  # this rank's sublayer output
            box.publish(x, t)
            torch.cuda.synchronize()
            dist.barrier()  # every rank's rows of round t are in every mailbox
            g = {k: d[k].to("cuda:0") for k in ("residual", "post", "comb", "pre", "norm_weight")}
            res_out = torch.empty_like(g["residual"])
            li = torch.empty(R, H, dtype=torch.bfloat16, device="cuda:0")
            post, comb, pre = (torch.empty(R, n, device="cuda:0"), torch.empty(R, n, n, device="cuda:0"),
                               torch.empty(R, n, device="cuda:0"))
            ws = M.new_workspace(R, H, n, "cuda:0")
            box.collect(t, g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"], d["norm_eps"],
                        M.Coeffs.from_weights(d["coeff"], "cuda:0"), res_out, layer_input=li, post_out=post,
                        comb_out=comb, pre_out=pre, workspace=ws)
            torch.cuda.synchronize()
            st, pst = M.mhc_get_device_status(ws), M.mhc_get_device_status(box.local)
            dist.barrier()  # round t consumed everywhere before anyone publishes round t + 1
            q.put((rank, step, st, pst, {k: v.cpu() for k, v in dict(residual_out=res_out, layer_input=li,
                                                                      post=post, comb=comb, pre=pre).items()}))
        hb.require(0, timeout_s=10.0)  # every rank published round 0 again
    finally:
        if box is not None:
            box.close()      # unmap the peer's mailbox ...
            dist.barrier()   # ... on every rank before any rank frees its own
        dist.destroy_process_group()


def test_two_processes_publish_and_collect_through_ipc():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in range(2 * (ROUNDS + 1))]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    by_round = {}
    for rank, t, st, pst, res in got:
        assert st == M.OK and pst == M.OK, (rank, t, st, pst)
        by_round.setdefault(t, {})[rank] = res
    for t in range(ROUNDS):
        d = S.draw_boundary(16, 7168, n=4, partials=2, seed=7400 + t)
        orc = oracle_post_pre(d, mxfp8=False)
        for rank, res in sorted(by_round[t].items()):
            assert_bf16_close(f64(res["residual_out"]), orc["residual"], f"round {t} rank {rank} streams")
            check_tail(d, dict(res), orc, mxfp8=False, what=f"round {t} rank {rank}")
        for k in by_round[t][0]:  # both ranks computed the same boundary
            assert torch.equal(by_round[t][0][k], by_round[t][1][k]), (t, k)
    for rank in range(2):  # round 0 after the reset: bitwise the first round 0
        for k, v in by_round[ROUNDS][rank].items():
            assert torch.equal(v, by_round[0][rank][k]), (rank, k)
