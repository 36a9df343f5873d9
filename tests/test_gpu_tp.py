"""The tensor-parallel boundary's partial table on one GPU.

* The table entry over P separately allocated buffers gives bitwise the
  results of the strided entry over the same values.
* Two processes on the same GPU form a gloo group of 2; each exports its
  partial through CUDA IPC, maps the other's (PeerPartials), and runs the
  boundary over the table of both: each must match the oracle on the sum of
  the two partials. The processes order their accesses with host barriers
  only; no kernel waits on another.
"""

import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

from mhc_residual_stream_b200 import mhc as M
from mhc_residual_stream_b200 import synthetic as S

from _parity import DEV, alloc_outputs, assert_bf16_close, check_tail, f64, gpu_post_pre, oracle_post_pre, to_dev

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# up to 16 rows and 8 partials the strided entry brings the rows in by tensor-map
# copies, the table entry always by per-lane loads: both must give the same bits
@pytest.mark.parametrize("R,H,n,P", [(32, 7168, 4, 8), (16, 7168, 4, 8), (1, 7168, 4, 8), (5, 192, 2, 3),
                                     (7, 64, 1, 16), (128, 512, 4, 11)])
def test_partial_table_matches_strided_bitwise(R, H, n, P):
    from mhc_residual_stream_b200 import build
    build.build()
    d = S.draw_boundary(R, H, n=n, partials=P, seed=6100 + R + P)
    ref = gpu_post_pre(d)
    g = to_dev({k: d[k] for k in ("residual", "post", "comb", "pre", "norm_weight")})
    bufs = [d["partials"][u].to(DEV).clone() for u in range(P)]  # separate allocations
    out = alloc_outputs(R, n, H)
    ws = M.new_workspace(R, H, n, DEV)
    M.mhc_boundary_post_pre_ptrs([b.data_ptr() for b in bufs], g["residual"], g["post"], g["comb"], g["pre"],
                                 g["norm_weight"], d["norm_eps"], M.Coeffs.from_weights(d["coeff"], DEV),
                                 out["residual_out"], layer_input=out["layer_input"],
                                 mxfp8=(out["q_data"], out["q_scale"], True), post_out=out["post"],
                                 comb_out=out["comb"], pre_out=out["pre"], workspace=ws)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    for k, v in out.items():
        assert torch.equal(v.cpu(), ref[k]), k


def _random_table_cases(count=8, seed=20261207):
    import numpy as np
    rng = np.random.default_rng(seed)
    return [(int(rng.choice([1, 2, 4, 9, 16, 17, 32, 64, 100, 128])), 64 * int(rng.integers(1, 149)),
             int(rng.choice([1, 2, 4])), int(rng.integers(1, 17))) for _ in range(count)]


@pytest.mark.parametrize("R,H,n,P", _random_table_cases())
def test_partial_table_random_shapes(R, H, n, P):
    test_partial_table_matches_strided_bitwise(R, H, n, P)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from mhc_residual_stream_b200 import mhc as M
    from mhc_residual_stream_b200 import synthetic as S
    from mhc_residual_stream_b200.tp import PeerPartials
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    peers = None
    try:
        torch.cuda.set_device(0)
        R, H, n = 16, 7168, 4
        d = S.draw_boundary(R, H, n=n, partials=world, seed=6200)  # the same draw on both ranks
        local = d["partials"][rank].to("cuda:0").contiguous()      # this rank's sublayer output
        peers = PeerPartials(local)
        g = {k: d[k].to("cuda:0") for k in ("residual", "post", "comb", "pre", "norm_weight")}
        res_out = torch.empty_like(g["residual"])
        li = torch.empty(R, H, dtype=torch.bfloat16, device="cuda:0")
        post, comb, pre = (torch.empty(R, n, device="cuda:0"), torch.empty(R, n, n, device="cuda:0"),
                           torch.empty(R, n, device="cuda:0"))
        ws = M.new_workspace(R, H, n, "cuda:0")
        peers.barrier()  # every rank's partial is written
        peers.boundary(g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"], d["norm_eps"],
                       M.Coeffs.from_weights(d["coeff"], "cuda:0"), res_out, layer_input=li, post_out=post,
                       comb_out=comb, pre_out=pre, workspace=ws)
        torch.cuda.synchronize()
        st = M.mhc_get_device_status(ws)
        peers.barrier()  # no rank frees or rewrites its partial before the others have read it
        q.put((rank, st, peers.ptrs[rank] == local.data_ptr(),
               {k: v.cpu() for k, v in dict(residual_out=res_out, layer_input=li, post=post, comb=comb,
                                            pre=pre).items()}))
        peers.barrier()
    finally:
        if peers is not None:
            peers.close()      # unmap the peer's buffer ...
            dist.barrier()     # ... on every rank before any rank frees its own
        dist.destroy_process_group()


def test_two_processes_share_partials_through_ipc():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    d = S.draw_boundary(16, 7168, n=4, partials=2, seed=6200)
    orc = oracle_post_pre(d, mxfp8=False)
    outs = {}
    for rank, st, own_slot, res in sorted(got, key=lambda t: t[0]):
        assert st == M.OK and own_slot
        assert_bf16_close(f64(res["residual_out"]), orc["residual"], f"rank {rank} streams")
        res = dict(res)
        check_tail(d, res, orc, mxfp8=False, what=f"rank {rank}")
        outs[rank] = res
    for k in outs[0]:  # both ranks computed the same boundary
        assert torch.equal(outs[0][k], outs[1][k]), k
