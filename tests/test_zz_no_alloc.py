"""The boundary entry point that allocates nothing (mhc_boundary_post_pre_noalloc).

Callers that cannot allocate device memory (a plugin inside a runtime that owns
all device memory, code running during CUDA-graph capture, allocation-free
serving loops) use this entry point: its scratch is a fixed array inside the
library instead of a caller workspace. It must give the results of
mhc_boundary_post_pre with a workspace, call after call, at the tolerances the
parity tests use. This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from mhc_residual_stream_b200 import mhc as M
from mhc_residual_stream_b200 import synthetic as S

from _parity import (DEV, alloc_outputs, assert_bf16_close, assert_bf16_ulp, check_tail, f64, gpu_post_pre,
                     oracle_post_pre, stream_terms, to_dev)


def _noalloc(d):
    g = to_dev({k: d[k] for k in ("partials", "residual", "post", "comb", "pre", "norm_weight")})
    R, n, H = g["residual"].shape
    out = alloc_outputs(R, n, H)
    M.mhc_boundary_post_pre_noalloc(
        g["partials"], g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"], d["norm_eps"],
        M.Coeffs.from_weights(d["coeff"], DEV), out["residual_out"], layer_input=out["layer_input"],
        mxfp8=(out["q_data"], out["q_scale"], True), post_out=out["post"], comb_out=out["comb"],
        pre_out=out["pre"])
    torch.cuda.synchronize()
    return {k: v.cpu() for k, v in out.items()}


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    from mhc_residual_stream_b200 import build
    build.build()
    M.lib()
    # two calls in a row on different inputs: the second must not see the first's scratch
    for seed, R in ((2032, 32), (2033, 5)):
        d = S.draw_boundary(R, 7168, n=4, partials=8, seed=seed)
        got = _noalloc(d)
        ref = gpu_post_pre(d)
        what = f"no-alloc rows {R}"
        assert_bf16_close(f64(got["residual_out"]), f64(ref["residual_out"]), what + " streams")
        assert_bf16_close(f64(got["layer_input"]), f64(ref["layer_input"]), what + " layer input")
        assert np.array_equal(got["q_data"].numpy(), ref["q_data"].numpy()), what + " mxfp8 data"
        assert np.array_equal(got["q_scale"].numpy(), ref["q_scale"].numpy()), what + " mxfp8 scales"
        for k in ("post", "comb", "pre"):
            assert np.max(np.abs(f64(got[k]) - f64(ref[k]))) <= 1e-5, what + " " + k


@pytest.mark.gpu
@pytest.mark.parametrize("R", [32, 128])
def test_noalloc_matches_the_oracle_at_full_size(R):
    # rows 32 and 128 (the largest the scratch holds), H 7168, n 4, P 8: the streams
    # and the layer input within the bf16 bounds, MXFP8 data and E8M0 scales
    # bit-exact, the coefficients within 1e-5 of the oracle fed the GPU's streams
    from mhc_residual_stream_b200 import build
    build.build()
    M.lib()
    d = S.draw_boundary(R, 7168, n=4, partials=8, seed=7100 + R)
    got = _noalloc(d)
    orc = oracle_post_pre(d)
    what = f"no-alloc rows {R}"
    assert_bf16_close(f64(got["residual_out"]), orc["residual"], what + " streams")
    assert_bf16_ulp(f64(got["residual_out"]), orc["residual"], what + " streams (ulp)",
                    terms=stream_terms(f64(d["partials"]), f64(d["residual"]), f64(d["post"]), f64(d["comb"])))
    check_tail(d, got, orc, what=what)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from mhc_residual_stream_b200 import build
    build.build()
    L = M.lib()
    a = ctypes.c_void_p(0x10000)
    # host-side size check, before any CUDA call: rows 64, hidden 9472 needs more
    # scratch than the fixed array (sized for hidden 7168) holds
    st = L.mhc_boundary_post_pre_noalloc(a, 8, 64 * 9472, a, a, a, a, a, 1e-6, None, a, None, a, None, None, None,
                                         None, 64, 9472, 4, None)
    assert st == M.WORKSPACE
