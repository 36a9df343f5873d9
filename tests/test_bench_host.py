"""Host-side arithmetic of the benchmark (no GPU): the algorithmic byte count the
roofline divides by, the rotation that keeps inputs out of L2, and the staging
buffers of the end-to-end measurement; on a GPU, that the end-to-end loop
downloads what the boundary computes."""

import types

import pytest
import torch

import bench


def test_algorithmic_bytes_of_the_headline_workload():
    """Rows 32, H 7168, n 4, P 8, MXFP8 with swizzled scales, coefficients: every
    tensor the boundary must read or write, once, tallied from its shape."""
    R, H, n, P = 32, 7168, 4, 8
    C = 2 * n + n * n
    tensors = {
        "partials": (P * R * H, 2),
        "residual in": (R * n * H, 2),
        "residual out": (R * n * H, 2),
        "post, comb, pre in": (R * C, 4),
        "norm weight": (H, 2),
        "layer input": (R * H, 2),
        "fn": (n * H * C, 4),
        "scale": (3, 4),
        "base": (C, 4),
        "post, comb, pre out": (R * C, 4),
        "mxfp8 data": (R * H, 1),
        "mxfp8 scales (128 padded rows x 224 block columns)": (128 * 224, 1),
    }
    total = sum(count * size for count, size in tensors.values())
    assert total == 10_829_932
    assert bench.boundary_bytes(R) == total


def test_rotating_sets_exceed_twice_l2():
    for R in (1, 2, 4, 8, 16, 32, 64, 128):
        assert bench.sets_for(R) * bench.boundary_bytes(R) > 2 * bench.L2_BYTES


def test_end_to_end_staging_views_are_aligned_and_disjoint():
    like = types.SimpleNamespace(
        partials=torch.zeros(8, 3, 64, dtype=torch.bfloat16),
        residual=torch.zeros(3, 4, 64, dtype=torch.bfloat16),
        post=torch.zeros(3, 4), comb=torch.zeros(3, 4, 4), pre=torch.zeros(3, 4))
    keys = bench.E2E_INPUTS
    nbytes = bench._arena_bytes(like, keys)
    buf = torch.zeros(nbytes + 256, dtype=torch.uint8)
    base = (-buf.data_ptr()) % 256
    buf = buf[base:base + nbytes]  # a 256-byte aligned buffer, as device allocations are
    views = bench._arena_views(like, keys, buf)
    spans = []
    for k in keys:
        v, t = views[k], getattr(like, k)
        assert v.shape == t.shape and v.dtype == t.dtype
        assert v.data_ptr() % 256 == 0
        spans.append((v.data_ptr(), v.data_ptr() + v.numel() * v.element_size()))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert spans[-1][1] <= buf.data_ptr() + nbytes
    for i, k in enumerate(keys):  # each view writes its own bytes only
        views[k].fill_(i + 1)
    for i, k in enumerate(keys):
        assert torch.all(views[k] == i + 1)


@pytest.mark.gpu
def test_end_to_end_steps_download_the_boundary_outputs():
    """The end-to-end loop (uploads, boundaries and downloads on three streams,
    two device slots) hands back bitwise the outputs of a direct call."""
    from mhc_residual_stream_b200 import mhc as M
    dev = torch.device("cuda", 0)
    b = bench.BoundarySet(4, 4242, dev)
    ws = M.new_workspace(4, bench.HIDDEN, bench.HC, dev)
    _, nin, nout, got = bench.e2e_time(b, ws, 5, dev)
    assert nin == bench._arena_bytes(b, bench.E2E_INPUTS) and nout == bench._arena_bytes(b, bench.E2E_OUTPUTS)
    b.launch(ws)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    for k in bench.E2E_OUTPUTS:
        assert torch.equal(got[k], getattr(b, k).cpu()), k
