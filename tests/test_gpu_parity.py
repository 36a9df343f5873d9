"""GPU parity of the CUDA mHC boundary against the CPU oracle (needs a B200).

Every case draws seeded inputs (mhc_residual_stream_b200.synthetic), runs the
C-ABI entry point through the binding and compares with the oracle at the
tolerances stated in tests/_parity.py. Sizes span several column blocks and
ragged row counts; the decode workloads (rows 32 and 128 at H=7168, MoE rows
64 with top_k 8) are compared element by element at full size.
"""

import numpy as np
import pytest
import torch

import oracle as O
from mhc_residual_stream_b200 import mhc as M
from mhc_residual_stream_b200 import synthetic as S

from _parity import (DEV, alloc_outputs, assert_bf16_close, assert_bf16_ulp, assert_coeffs_close, check_tail,
                     coeff_np, f64, gpu_post_pre, oracle_post_pre, stream_terms, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from mhc_residual_stream_b200 import build
    build.build()
    M.lib()
    yield


# ---------------------------------------------------------------- partial-sum boundary

def _case(R, H, n, P, seed, swizzled=True, mxfp8=True, coeff=True, affine=True, fn_std=0.01, part_std=0.05,
          packed=False):
    d = S.draw_boundary(R, H, n=n, partials=P, seed=seed, fn_std=fn_std, affine=affine, part_std=part_std)
    gpu = gpu_post_pre(d, mxfp8=mxfp8, swizzled=swizzled, coeff=coeff, packed=packed)
    orc = oracle_post_pre(d, mxfp8=mxfp8, swizzled=swizzled, coeff=coeff)
    what = f"R={R} H={H} n={n} P={P}"
    assert_bf16_close(f64(gpu["residual_out"]), orc["residual"], what + " residual")
    assert_bf16_ulp(f64(gpu["residual_out"]), orc["residual"], what + " residual (ulp)",
                    terms=stream_terms(f64(d["partials"]), f64(d["residual"]), f64(d["post"]), f64(d["comb"])))
    check_tail(d, gpu, orc, mxfp8=mxfp8, swizzled=swizzled, coeff=coeff, what=what)
    if coeff:  # end to end as well, at the looser level a bf16 flip allows
        for name in ("post", "comb", "pre"):
            assert np.max(np.abs(f64(gpu[name]) - orc[name])) < 2e-3, name
    return d, gpu, orc


def test_tiny_attention_boundary():
    # rows 4, H 256, n 4, P 2, fn N(0, 0.02), scale 1, base 0
    _case(4, 256, 4, 2, seed=1004, affine=False, fn_std=0.02)


def test_decode_attention_boundary_rows32_full_size():
    # rows 32, H 7168, n 4, P 8, MXFP8 layer input with swizzled scales
    _case(32, 7168, 4, 8, seed=2032)


@pytest.mark.parametrize("R,H,n,P,swz", [
    (1, 7168, 4, 8, True), (2, 7168, 4, 8, False), (3, 256, 4, 1, True), (5, 192, 4, 3, True),
    (13, 320, 2, 16, False), (7, 64, 1, 2, True), (33, 1024, 4, 8, True), (64, 7168, 4, 8, True),
    (128, 7168, 4, 8, True), (128, 128, 2, 5, False), (100, 9472, 4, 4, True),
])
def test_boundary_shapes(R, H, n, P, swz):
    _case(R, H, n, P, seed=7000 + R * 7 + n, swizzled=swz)


def _random_cases(count=40, seed=20261203):
    """Seeded draws over the supported shape space: rows 1-128, H = 64 x 1-148
    column blocks, n in {1, 2, 4}, 1-16 partials, both scale layouts, with and
    without MXFP8 and coefficients, fp32 or packed fn, small or unit partials."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(count):
        R = int(rng.choice([1, 2, 3, 4, 5, 8, 15, 16, 17, 31, 32, 33, 47, 48, 63, 64, 65, 96, 127, 128]))
        G = int(rng.integers(1, 149))
        cases.append((R, 64 * G, int(rng.choice([1, 2, 4])), int(rng.integers(1, 17)), bool(rng.integers(2)),
                      bool(rng.integers(4) > 0), bool(rng.integers(4) > 0), bool(rng.integers(2)),
                      float(rng.choice([0.05, 1.0])), 9000 + i))
    return cases


@pytest.mark.parametrize("R,H,n,P,swz,mxfp8,coeff,packed,part_std,seed", _random_cases())
def test_boundary_random_shapes(R, H, n, P, swz, mxfp8, coeff, packed, part_std, seed):
    _case(R, H, n, P, seed=seed, swizzled=swz, mxfp8=mxfp8, coeff=coeff, packed=packed and coeff,
          part_std=part_std)


def test_boundary_without_mxfp8_and_without_coefficients():
    _case(9, 512, 4, 8, seed=11, mxfp8=False, coeff=False)
    _case(9, 512, 4, 8, seed=12, mxfp8=False, coeff=True)


def test_residual_only_matches_full_streams_bitwise():
    d = S.draw_boundary(32, 7168, n=4, partials=8, seed=2132)
    full = gpu_post_pre(d)
    ronly = gpu_post_pre(d, residual_only=True)
    assert torch.equal(full["residual_out"], ronly["residual_out"])
    orc = oracle_post_pre(d, residual_only=True)
    assert_bf16_close(f64(ronly["residual_out"]), orc["residual"], "residual-only")
    # the dedicated entry point agrees bit for bit
    g = to_dev(d)
    out = torch.empty_like(g["residual"])
    M.mhc_boundary_residual_only(g["partials"], g["residual"], g["post"], g["comb"], out)
    torch.cuda.synchronize()
    assert torch.equal(out.cpu(), ronly["residual_out"])


def test_in_place_residual_and_strided_partials():
    d = S.draw_boundary(17, 1024, n=4, partials=4, seed=99)
    ref = gpu_post_pre(d)
    # partials as slices of a larger buffer: stride between partials != R*H
    big = torch.zeros(4, 17 * 1024 + 64, dtype=torch.bfloat16, device=DEV)
    view = big[:, : 17 * 1024].view(4, 17, 1024)
    view.copy_(d["partials"].to(DEV))
    assert view.stride(0) == 17 * 1024 + 64
    got = gpu_post_pre(d, in_place=True, partials=view)
    for k in ref:
        assert torch.equal(ref[k], got[k]), k


def test_bitwise_deterministic():
    d = S.draw_boundary(32, 7168, n=4, partials=8, seed=5)
    a = gpu_post_pre(d)
    b = gpu_post_pre(d)
    for k in a:
        assert torch.equal(a[k], b[k]), k


def test_zero_partials_and_identity_mixes():
    d = S.draw_boundary(8, 256, n=4, partials=2, seed=3)
    d["partials"].zero_()
    d["comb"] = torch.eye(4).expand(8, 4, 4).contiguous()
    gpu = gpu_post_pre(d)
    assert torch.equal(gpu["residual_out"], d["residual"])


def test_sinkhorn_iteration_counts_and_eps():
    for iters, eps in ((0, 1e-6), (1, 0.0), (50, 1e-3)):
        d = S.draw_boundary(6, 256, n=4, partials=2, seed=40 + iters)
        d["coeff"].sinkhorn_iters = iters
        d["coeff"].sinkhorn_eps = eps
        gpu = gpu_post_pre(d)
        post, comb, pre = O.mhc_coefficients(f64(gpu["residual_out"]), **coeff_np(d["coeff"]))
        assert_coeffs_close(gpu, post, comb, pre, f"iters={iters}")


def _extreme_comb(n, row1, seed):
    # one dominant comb entry (+30) and comb row 1 shifted by `row1`; 50 iterations
    d = S.draw_boundary(6, 256, n=n, partials=2, seed=seed)
    c = d["coeff"]
    base = c.base.clone()
    c0 = 2 * n
    base[c0 + 0] = 30.0
    base[c0 + 1 * n: c0 + 2 * n] = row1
    c.base = base
    c.sinkhorn_iters = 50
    return d, c


@pytest.mark.parametrize("n", [4, 2])
def test_sinkhorn_wide_comb_logits(n):
    # exp(L - max L) down to ~e^-75, still a normal fp32 number: the small row's
    # sums are far below eps, so the iterations grow it back to a full row
    d, c = _extreme_comb(n, -40.0, 4100 + n)
    gpu = gpu_post_pre(d)
    post, comb, pre = O.mhc_coefficients(f64(gpu["residual_out"]), **coeff_np(c))
    assert_coeffs_close(gpu, post, comb, pre, f"wide comb logits, n={n}")


@pytest.mark.parametrize("n", [4, 2])
def test_sinkhorn_comb_logits_at_the_supported_spread(n):
    # the contract (mhc_coeff_args): parity holds while every comb logit of a row's
    # matrix lies within 80 of the largest (exp(L - max L) >= e^-80, a normal
    # float). fn is scaled down so that the logits are base to within ~0.05:
    # comb[0][0] at 30 and row 1 at 30 - 79.5, 50 iterations
    d = S.draw_boundary(6, 256, n=n, partials=2, seed=4300 + n, fn_std=1e-4)
    c = d["coeff"]
    base = c.base.clone()
    c0 = 2 * n
    base[c0:] = 0.0
    base[c0 + 0] = 30.0
    base[c0 + 1 * n: c0 + 2 * n] = 30.0 - 79.5
    c.base = base
    c.sinkhorn_iters = 50
    gpu = gpu_post_pre(d)
    post, comb, pre = O.mhc_coefficients(f64(gpu["residual_out"]), **coeff_np(c))
    assert np.isfinite(f64(gpu["comb"])).all()
    assert_coeffs_close(gpu, post, comb, pre, f"comb logit spread 79.5, n={n}")


@pytest.mark.parametrize("n", [4, 2])
def test_sinkhorn_underflowing_comb_row_stays_finite(n):
    # comb row 1 ~280 below the largest logit: its exp(L - max L) is exactly zero
    # in fp32 (float64 keeps ~1e-122 and grows it back into a full row: outside
    # what fp32 represents). The row must come out as zeros, nothing as NaN.
    d, c = _extreme_comb(n, -250.0, 4200 + n)
    gpu = gpu_post_pre(d)
    cb = f64(gpu["comb"])
    assert np.isfinite(cb).all()
    assert (cb[:, 1, :] == 0.0).all()
    assert (cb >= 0.0).all() and (cb <= 1.0 + 1e-6).all()


# ---------------------------------------------------------------- MoE finalize

def _moe_gpu(d, pre=True, mxfp8=False, coeff=True, ws=None, check_status=True, packed=False):
    g = to_dev(d)
    R, n, H = g["residual"].shape
    out = alloc_outputs(R, n, H, mxfp8, True, coeff)
    ws = ws if ws is not None else M.new_workspace(R, H, n, DEV)
    M.mhc_boundary_moe_finalize(
        g["gemm2_permuted"], g["expert_weights"], g["expanded_idx_to_permuted_idx"], g["shared_output"],
        g["residual"], g["post"], g["comb"], g["pre"] if pre else None, g["norm_weight"] if pre else None,
        d["norm_eps"], M.Coeffs.from_weights(d["coeff"], DEV, packed=packed) if (coeff and pre) else None,
        out["residual_out"],
        layer_input=out["layer_input"] if pre else None,
        mxfp8=(out["q_data"], out["q_scale"], True) if mxfp8 else None,
        post_out=out.get("post"), comb_out=out.get("comb"), pre_out=out.get("pre"), workspace=ws)
    torch.cuda.synchronize()
    st = M.mhc_get_device_status(ws)
    if check_status:
        assert st == M.OK, M.STATUS_NAMES[st]
    return {k: v.cpu() for k, v in out.items()}, st


def _moe_oracle(d, pre=True, mxfp8=False, coeff=True):
    f = {k: f64(v) for k, v in d.items() if isinstance(v, torch.Tensor)}
    moe = {k: f[k] for k in ("gemm2_permuted", "expert_weights", "shared_output")}
    moe["expanded_idx_to_permuted_idx"] = d["expanded_idx_to_permuted_idx"].numpy().astype(np.int64)
    return O.boundary(moe=moe, residual=f["residual"], post=f["post"], comb=f["comb"],
                      pre=f["pre"] if pre else None, norm_weight=f["norm_weight"], norm_eps=d["norm_eps"],
                      coeff=coeff_np(d["coeff"]) if coeff else None, mxfp8=mxfp8)


def _moe_terms(d):
    """Magnitude sums of the new streams' terms with x = shared + sum_t w g (MoE front)."""
    g = f64(d["gemm2_permuted"])
    w = f64(d["expert_weights"])
    idx = d["expanded_idx_to_permuted_idx"].numpy().astype(np.int64)
    R, k = w.shape
    xa = np.abs(f64(d["shared_output"]))
    for r in range(R):
        for t in range(k):
            e = idx[r * k + t]
            if 0 <= e < g.shape[0]:
                xa[r] += abs(w[r, t]) * np.abs(g[e])
    return stream_terms(xa[None], f64(d["residual"]), f64(d["post"]), f64(d["comb"]))


def test_moe_boundary_rows64_full_size():
    d = S.draw_moe(64, 7168, n=4, top_k=8, seed=3064)
    gpu, _ = _moe_gpu(d)
    orc = _moe_oracle(d)
    assert_bf16_ulp(f64(gpu["residual_out"]), orc["residual"], "moe rows 64 residual (ulp)", terms=_moe_terms(d))
    assert_bf16_close(f64(gpu["residual_out"]), orc["residual"], "moe residual")
    check_tail(d, gpu, orc, mxfp8=False, what="moe")


@pytest.mark.parametrize("R,H,k,extra", [(1, 256, 1, 0), (5, 192, 16, 7), (32, 7168, 8, 100), (128, 512, 8, 3)])
def test_moe_shapes_with_mxfp8(R, H, k, extra):
    d = S.draw_moe(R, H, n=4, top_k=k, seed=R * 31 + k, extra_permuted=extra)
    gpu, _ = _moe_gpu(d, mxfp8=True)
    orc = _moe_oracle(d, mxfp8=True)
    assert_bf16_close(f64(gpu["residual_out"]), orc["residual"], "moe residual")
    assert_bf16_ulp(f64(gpu["residual_out"]), orc["residual"], f"moe R={R} H={H} k={k} residual (ulp)",
                    terms=_moe_terms(d))
    check_tail(d, gpu, orc, mxfp8=True, what="moe")


def _random_moe_cases(count=16, seed=20261204):
    """Seeded draws of MoE-finalize boundaries: rows 1-128, H = 64 x 1-148, n in
    {1, 2, 4}, top_k 1-16, 0-64 permuted rows beyond rows x top_k, with and
    without MXFP8, fp32 or packed fn."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(count):
        R = int(rng.choice([1, 2, 3, 7, 8, 16, 31, 32, 33, 64, 65, 100, 128]))
        cases.append((R, 64 * int(rng.integers(1, 149)), int(rng.choice([1, 2, 4])), int(rng.integers(1, 17)),
                      int(rng.integers(0, 65)), bool(rng.integers(2)), bool(rng.integers(2)), 9500 + i))
    return cases


@pytest.mark.parametrize("R,H,n,k,extra,mxfp8,packed,seed", _random_moe_cases())
def test_moe_random_shapes(R, H, n, k, extra, mxfp8, packed, seed):
    d = S.draw_moe(R, H, n=n, top_k=k, seed=seed, extra_permuted=extra)
    gpu, _ = _moe_gpu(d, mxfp8=mxfp8, packed=packed)
    orc = _moe_oracle(d, mxfp8=mxfp8)
    what = f"moe R={R} H={H} n={n} k={k}"
    assert_bf16_close(f64(gpu["residual_out"]), orc["residual"], what + " residual")
    assert_bf16_ulp(f64(gpu["residual_out"]), orc["residual"], what + " residual (ulp)", terms=_moe_terms(d))
    check_tail(d, gpu, orc, mxfp8=mxfp8, what=what)


def test_moe_gather_indexing_bit_exact():
    # row-coded permuted rows, one-hot weights, zero shared output and residual,
    # comb = I, post = 1: the new streams must equal the selected rows exactly
    R, H, k, n = 12, 256, 8, 4
    d = S.draw_moe(R, H, n=n, top_k=k, seed=77, extra_permuted=9)
    num = d["gemm2_permuted"].shape[0]
    code = torch.arange(num, dtype=torch.float32)[:, None] + torch.arange(H, dtype=torch.float32)[None, :] / 512
    d["gemm2_permuted"] = code.to(torch.bfloat16)
    sel = torch.randint(0, k, (R,), generator=S.gen(78))
    w = torch.zeros(R, k)
    w[torch.arange(R), sel] = 1.0
    d["expert_weights"] = w
    d["shared_output"].zero_()
    d["residual"].zero_()
    d["comb"] = torch.eye(n).expand(R, n, n).contiguous()
    d["post"] = torch.ones(R, n)
    gpu, _ = _moe_gpu(d, pre=False)
    idx = d["expanded_idx_to_permuted_idx"].long()
    for r in range(R):
        want = d["gemm2_permuted"][idx[r * k + sel[r]]]
        for i in range(n):
            assert torch.equal(gpu["residual_out"][r, i], want)


def test_moe_negative_and_out_of_range_indices():
    d = S.draw_moe(6, 256, n=4, top_k=4, seed=55)
    d["expanded_idx_to_permuted_idx"][3] = -1
    gpu, st = _moe_gpu(d)
    orc = _moe_oracle(d)
    assert st == M.OK
    assert_bf16_close(f64(gpu["residual_out"]), orc["residual"], "moe with index -1")
    d["expanded_idx_to_permuted_idx"][5] = d["gemm2_permuted"].shape[0]  # one past the end
    _, st = _moe_gpu(d, check_status=False)
    assert st == M.DEVICE_INDEX


def test_moe_residual_only():
    d = S.draw_moe(16, 1024, n=4, top_k=8, seed=66)
    gpu, _ = _moe_gpu(d, pre=False)
    orc = _moe_oracle(d, pre=False)
    assert_bf16_close(f64(gpu["residual_out"]), orc["residual"], "moe residual-only")
    full, _ = _moe_gpu(d)
    assert torch.equal(full["residual_out"], gpu["residual_out"])


# ---------------------------------------------------------------- coefficients entry / first layer

def test_coeffs_on_given_streams():
    d = S.draw_boundary(24, 7168, n=4, partials=1, seed=808)
    g = to_dev(d)
    R, n, H = g["residual"].shape
    out = alloc_outputs(R, n, H, False, True, True)
    ws = M.new_workspace(R, H, n, DEV)
    M.mhc_coeffs(M.Coeffs.from_weights(d["coeff"], DEV), out["post"], out["comb"], out["pre"],
                 residual=g["residual"], pre_mix=g["pre"], norm_weight=g["norm_weight"], norm_eps=d["norm_eps"],
                 layer_input=out["layer_input"], workspace=ws)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    res = f64(d["residual"])
    o = O.coeffs_entry(residual=res, pre_mix=f64(d["pre"]), norm_weight=f64(d["norm_weight"]),
                       norm_eps=d["norm_eps"], coeff=coeff_np(d["coeff"]))
    assert_coeffs_close({k: out[k].cpu() for k in ("post", "comb", "pre")}, o["post"], o["comb"], o["pre"], "coeffs")
    assert_bf16_close(f64(out["layer_input"]), o["layer_input"], "coeffs layer input")
    # without a layer input: coefficients only, identical
    out2 = alloc_outputs(R, n, H, False, True, True)
    M.mhc_coeffs(M.Coeffs.from_weights(d["coeff"], DEV), out2["post"], out2["comb"], out2["pre"],
                 residual=g["residual"], workspace=ws)
    torch.cuda.synchronize()
    for k in ("post", "comb", "pre"):
        assert torch.equal(out[k], out2[k]), k


@pytest.mark.parametrize("R", [1, 2, 4, 8, 16, 32, 64, 128])
def test_first_layer_broadcast(R):
    d = S.draw_first_layer(R, 7168, n=4, seed=4000 + R)
    x = d["x"].to(DEV)
    n, H = 4, 7168
    out = alloc_outputs(R, n, H, False, True, True)
    ws = M.new_workspace(R, H, n, DEV)
    M.mhc_coeffs(M.Coeffs.from_weights(d["coeff"], DEV), out["post"], out["comb"], out["pre"], x=x,
                 residual_out=out["residual_out"], norm_weight=d["norm_weight"].to(DEV), norm_eps=d["norm_eps"],
                 layer_input=out["layer_input"], workspace=ws)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    # every stream is x bit for bit; identity pre-mix selects stream 0
    assert torch.equal(out["residual_out"].cpu(), d["x"][:, None, :].expand(R, n, H))
    o = O.coeffs_entry(x=f64(d["x"]), hc_mult=n, norm_weight=f64(d["norm_weight"]), norm_eps=d["norm_eps"],
                       coeff=coeff_np(d["coeff"]))
    assert_bf16_close(f64(out["layer_input"]), o["layer_input"], "first-layer layer input")
    assert_coeffs_close({k: out[k].cpu() for k in ("post", "comb", "pre")}, o["post"], o["comb"], o["pre"],
                        "first-layer coefficients")


def _random_entry_cases(count, seed):
    rng = np.random.default_rng(seed)
    return [(int(rng.choice([1, 2, 3, 5, 8, 16, 17, 32, 33, 48, 64, 97, 128])), 64 * int(rng.integers(1, 149)),
             int(rng.choice([1, 2, 4])), bool(rng.integers(2)), 9700 + i) for i in range(count)]


@pytest.mark.parametrize("R,H,n,with_layer,seed", _random_entry_cases(10, 20261205))
def test_first_layer_broadcast_random_shapes(R, H, n, with_layer, seed):
    """Seeded draws of the first-layer entry: streams bitwise x, identity pre-mix."""
    d = S.draw_first_layer(R, H, n=n, seed=seed)
    out = alloc_outputs(R, n, H, False, True, True)
    ws = M.new_workspace(R, H, n, DEV)
    M.mhc_coeffs(M.Coeffs.from_weights(d["coeff"], DEV), out["post"], out["comb"], out["pre"], x=d["x"].to(DEV),
                 residual_out=out["residual_out"], norm_weight=d["norm_weight"].to(DEV) if with_layer else None,
                 norm_eps=d["norm_eps"], layer_input=out["layer_input"] if with_layer else None, workspace=ws)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    assert torch.equal(out["residual_out"].cpu(), d["x"][:, None, :].expand(R, n, H))
    o = O.coeffs_entry(x=f64(d["x"]), hc_mult=n, norm_weight=f64(d["norm_weight"]), norm_eps=d["norm_eps"],
                       coeff=coeff_np(d["coeff"]))
    if with_layer:
        assert_bf16_close(f64(out["layer_input"]), o["layer_input"], f"broadcast R={R} H={H} n={n} layer input")
    assert_coeffs_close({k: out[k].cpu() for k in ("post", "comb", "pre")}, o["post"], o["comb"], o["pre"],
                        f"broadcast R={R} H={H} n={n} coefficients")


@pytest.mark.parametrize("R,H,n,with_layer,seed", _random_entry_cases(10, 20261206))
def test_coeffs_on_given_streams_random_shapes(R, H, n, with_layer, seed):
    """Seeded draws of the coefficients entry on given streams (Engram-entry form)."""
    d = S.draw_boundary(R, H, n=n, partials=1, seed=seed)
    g = to_dev(d)
    out = alloc_outputs(R, n, H, False, True, True)
    ws = M.new_workspace(R, H, n, DEV)
    M.mhc_coeffs(M.Coeffs.from_weights(d["coeff"], DEV), out["post"], out["comb"], out["pre"],
                 residual=g["residual"], pre_mix=g["pre"] if with_layer else None,
                 norm_weight=g["norm_weight"] if with_layer else None, norm_eps=d["norm_eps"],
                 layer_input=out["layer_input"] if with_layer else None, workspace=ws)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    o = O.coeffs_entry(residual=f64(d["residual"]), pre_mix=f64(d["pre"]), norm_weight=f64(d["norm_weight"]),
                       norm_eps=d["norm_eps"], coeff=coeff_np(d["coeff"]))
    what = f"coeffs R={R} H={H} n={n}"
    assert_coeffs_close({k: out[k].cpu() for k in ("post", "comb", "pre")}, o["post"], o["comb"], o["pre"], what)
    if with_layer:
        assert_bf16_close(f64(out["layer_input"]), o["layer_input"], what + " layer input")


# ---------------------------------------------------------------- standalone MXFP8

def _mxfp8_inputs(R, H, seed):
    g = S.gen(seed)
    y = torch.randn(R, H, generator=g) * torch.exp(torch.randn(R, H, generator=g) * 3)
    y = y * torch.exp2(torch.randint(-40, 40, (R, H // 32, 1), generator=g).float()).repeat_interleave(32, 1)[:, :, 0]
    y = y.to(torch.bfloat16)
    y[0, :32] = 0.0                                 # zero block
    y[0, 32:64] = -0.0
    if H >= 128:
        y[0, 64:96] = torch.tensor(448.0)           # amax exactly 448
        y[0, 96:128] = torch.tensor(2.0 ** -130)    # bf16 subnormals
    return y


@pytest.mark.parametrize("R,H,swz", [(1, 32, True), (3, 96, False), (37, 7168, True), (130, 192, True),
                                     (200, 4096, False)])
def test_mxfp8_quantize_rows_bit_exact(R, H, swz):
    y = _mxfp8_inputs(R, H, seed=R + H)
    data = torch.empty(R, H, dtype=torch.uint8, device=DEV)
    scale = torch.full((M.mhc_mxfp8_scale_bytes(R, H, swz),), 0xCD, dtype=torch.uint8, device=DEV)
    M.mxfp8_quantize_rows(y.to(DEV), data, scale, swz)
    torch.cuda.synchronize()
    od, osc = O.mxfp8_quantize(f64(y))
    assert np.array_equal(data.cpu().numpy(), od)
    want = O.swizzle_scales_128x4(osc) if swz else osc.reshape(-1)
    assert np.array_equal(scale.cpu().numpy(), want)


def test_mxfp8_nonfinite_block():
    y = torch.randn(2, 64).to(torch.bfloat16)
    y[1, 40] = float("inf")
    y[0, 3] = float("nan")
    data = torch.empty(2, 64, dtype=torch.uint8, device=DEV)
    scale = torch.empty(4, dtype=torch.uint8, device=DEV)
    M.mxfp8_quantize_rows(y.to(DEV), data, scale, False)
    torch.cuda.synchronize()
    od, osc = O.mxfp8_quantize(f64(y))
    assert np.array_equal(data.cpu().numpy(), od)
    assert np.array_equal(scale.cpu().numpy(), osc.reshape(-1))


# ---------------------------------------------------------------- aux stream mean

@pytest.mark.parametrize("R,H,n", [(32, 7168, 4), (5, 192, 2), (3, 64, 1), (128, 512, 4)])
def test_aux_stream_mean_on_every_front(R, H, n):
    d = S.draw_boundary(R, H, n=n, partials=4, seed=5100 + R + n)
    g = to_dev({k: d[k] for k in ("partials", "residual", "post", "comb", "pre", "norm_weight")})
    orc = oracle_post_pre(d, mxfp8=False, coeff=False)
    o_aux = O.stream_mean(orc["residual"])
    runs = {}
    # full boundary (no coefficients), the residual-only form, and the no-workspace entry
    out, aux = alloc_outputs(R, n, H, False, True, False), torch.empty(R, H, dtype=torch.bfloat16, device=DEV)
    M.mhc_boundary_post_pre(g["partials"], g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"],
                            d["norm_eps"], None, out["residual_out"], layer_input=out["layer_input"],
                            workspace=M.new_workspace(R, H, n, DEV), aux=aux)
    runs["post_pre"] = (out["residual_out"], aux)
    res2, aux2 = torch.empty_like(g["residual"]), torch.empty(R, H, dtype=torch.bfloat16, device=DEV)
    M.mhc_boundary_residual_only(g["partials"], g["residual"], g["post"], g["comb"], res2, aux=aux2)
    runs["residual_only"] = (res2, aux2)
    if R <= 128 and H <= 7168 and n <= 4:
        out3, aux3 = alloc_outputs(R, n, H, False, True, True), torch.empty(R, H, dtype=torch.bfloat16, device=DEV)
        M.mhc_boundary_post_pre_noalloc(g["partials"], g["residual"], g["post"], g["comb"], g["pre"],
                                        g["norm_weight"], d["norm_eps"], M.Coeffs.from_weights(d["coeff"], DEV),
                                        out3["residual_out"], layer_input=out3["layer_input"], post_out=out3["post"],
                                        comb_out=out3["comb"], pre_out=out3["pre"], aux=aux3)
        runs["noalloc"] = (out3["residual_out"], aux3)
    torch.cuda.synchronize()
    for name, (res, ax) in runs.items():
        g_res = f64(res.cpu())
        # stage-wise exact: the mean of the streams the GPU wrote, rounded once
        assert np.array_equal(f64(ax.cpu()), O.stream_mean(g_res)), name
        assert_bf16_close(f64(ax.cpu()), o_aux, name + " aux (end to end)")


def test_aux_stream_mean_moe_front_and_null_aux_writes_nothing():
    d = S.draw_moe(16, 7168, n=4, top_k=8, seed=5216)
    g = to_dev(d)
    out = alloc_outputs(16, 4, 7168, False, True, True)
    aux = torch.empty(16, 7168, dtype=torch.bfloat16, device=DEV)
    ws = M.new_workspace(16, 7168, 4, DEV)
    M.mhc_boundary_moe_finalize(
        g["gemm2_permuted"], g["expert_weights"], g["expanded_idx_to_permuted_idx"], g["shared_output"],
        g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"], d["norm_eps"],
        M.Coeffs.from_weights(d["coeff"], DEV), out["residual_out"], layer_input=out["layer_input"],
        post_out=out["post"], comb_out=out["comb"], pre_out=out["pre"], workspace=ws, aux=aux)
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(ws) == M.OK
    assert np.array_equal(f64(aux.cpu()), O.stream_mean(f64(out["residual_out"].cpu())))
    # the same call without aux gives the same streams, layer input and coefficients
    b, _ = _moe_gpu(d)
    for k in ("residual_out", "layer_input", "post", "comb", "pre"):
        assert torch.equal(out[k].cpu(), b[k]), k


# ---------------------------------------------------------------- packed projection weights

@pytest.mark.parametrize("R,H,n,P", [(1, 7168, 4, 8), (5, 192, 4, 3), (13, 320, 2, 16), (7, 64, 1, 2),
                                     (32, 7168, 4, 8), (128, 7168, 4, 8), (100, 9472, 4, 4)])
def test_packed_projection_matches_fn_bitwise(R, H, n, P):
    # fn packed once into bf16 terms gives the same bits as the in-kernel split,
    # and so the oracle's results at the parity tolerances
    d = S.draw_boundary(R, H, n=n, partials=P, seed=4100 + R + n)
    a = gpu_post_pre(d)
    b = gpu_post_pre(d, packed=True)
    for k in a:
        assert torch.equal(a[k], b[k]), f"R={R} H={H} n={n}: {k} differs with packed fn"
    if R <= 32:
        orc = oracle_post_pre(d)
        assert_bf16_close(f64(b["residual_out"]), orc["residual"], "packed residual")
        check_tail(d, b, orc, what=f"packed R={R} H={H} n={n}")


def test_packed_projection_moe_and_coeffs_entry():
    d = S.draw_moe(32, 7168, n=4, top_k=8, seed=4232)
    a, _ = _moe_gpu(d, mxfp8=True)
    b, _ = _moe_gpu(d, mxfp8=True, packed=True)
    for k in a:
        assert torch.equal(a[k], b[k]), f"moe: {k} differs with packed fn"
    d = S.draw_boundary(24, 7168, n=4, partials=1, seed=4824)
    g = to_dev(d)
    outs = []
    for packed in (False, True):
        cw = M.Coeffs.from_weights(d["coeff"], DEV, packed=packed)
        if packed:
            cw.fn = None  # the packed form alone is enough
        out = alloc_outputs(24, 4, 7168, False, True, True)
        ws = M.new_workspace(24, 7168, 4, DEV)
        M.mhc_coeffs(cw, out["post"], out["comb"], out["pre"], residual=g["residual"], pre_mix=g["pre"],
                     norm_weight=g["norm_weight"], norm_eps=d["norm_eps"], layer_input=out["layer_input"],
                     workspace=ws)
        torch.cuda.synchronize()
        assert M.mhc_get_device_status(ws) == M.OK
        outs.append({k: out[k].cpu() for k in ("post", "comb", "pre", "layer_input")})
    for k in outs[0]:
        assert torch.equal(outs[0][k], outs[1][k]), f"coeffs entry: {k} differs with packed fn"


@pytest.mark.parametrize("n", [1, 4])
def test_packed_layout_holds_the_three_bf16_terms(n):
    # element (t, c, k) of block g is term t of fn[(k/64)*H + 64g + k%64][c]; terms add back to fn
    H = 128
    C = 2 * n + n * n
    fn = torch.randn(n * H, C, dtype=torch.float32) * 0.02
    pk = M.mhc_projection_pack(fn.to(DEV), H, n)
    torch.cuda.synchronize()
    KS, CP8 = n * 64 + 8, ((C + 7) // 8) * 8
    t = pk.cpu().view(torch.bfloat16).view(H // 64, 3, CP8, KS).to(torch.float64)
    for g in range(H // 64):
        for k in [k for k in (0, 5, 63, 64, 200, n * 64 - 1) if k < n * 64]:
            row = (k // 64) * H + 64 * g + k % 64
            s = t[g, 0, :C, k] + t[g, 1, :C, k] + t[g, 2, :C, k]
            assert torch.allclose(s, fn[row].double(), rtol=2 ** -22, atol=0), (g, k)
            hi = fn[row].to(torch.bfloat16).double()
            assert torch.equal(t[g, 0, :C, k], hi), (g, k)
    for pad in (t[:, :, C:, :], t[:, :, :, n * 64:]):  # padding columns and gaps are zero
        assert pad.numel() == 0 or float(pad.abs().max()) == 0.0


# ---------------------------------------------------------------- bounded waits

def test_weight_copy_wait_times_out_and_recovers():
    # the wait on the fn slice's TMA copies expects one 16-byte unit that never
    # comes: it must give up after its budget and record the timeout, and the
    # next boundary must be correct
    d = S.draw_boundary(4, 256, n=4, partials=2, seed=9)
    ws = M.new_workspace(4, 256, 4, DEV)
    old = M.mhc_debug_set_wait(20_000_000, 1)  # 20 ms
    try:
        g = to_dev(d)
        out = alloc_outputs(4, 4, 256)
        M.mhc_boundary_post_pre(g["partials"], g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"],
                                d["norm_eps"], M.Coeffs.from_weights(d["coeff"], DEV), out["residual_out"],
                                layer_input=out["layer_input"], post_out=out["post"], comb_out=out["comb"],
                                pre_out=out["pre"], workspace=ws)
        assert M.mhc_get_device_status(ws) == M.DEVICE_TIMEOUT
    finally:
        M.mhc_debug_set_wait(old, 0)
    assert M.mhc_get_device_status(ws) == M.OK  # reading cleared it
    gpu = gpu_post_pre(d, ws=ws)
    orc = oracle_post_pre(d)
    check_tail(d, gpu, orc, what="after recovery")


def test_packed_weight_copy_wait_times_out_and_recovers():
    # the same with packed fn, whose copy is waited for only before the projection
    d = S.draw_boundary(4, 256, n=4, partials=2, seed=19)
    ws = M.new_workspace(4, 256, 4, DEV)
    old = M.mhc_debug_set_wait(20_000_000, 1)  # 20 ms
    try:
        g = to_dev(d)
        out = alloc_outputs(4, 4, 256)
        M.mhc_boundary_post_pre(g["partials"], g["residual"], g["post"], g["comb"], g["pre"], g["norm_weight"],
                                d["norm_eps"], M.Coeffs.from_weights(d["coeff"], DEV, packed=True),
                                out["residual_out"], layer_input=out["layer_input"], post_out=out["post"],
                                comb_out=out["comb"], pre_out=out["pre"], workspace=ws)
        assert M.mhc_get_device_status(ws) == M.DEVICE_TIMEOUT
    finally:
        M.mhc_debug_set_wait(old, 0)
    assert M.mhc_get_device_status(ws) == M.OK
    gpu = gpu_post_pre(d, ws=ws, packed=True)
    orc = oracle_post_pre(d)
    check_tail(d, gpu, orc, what="packed, after recovery")
