"""Helpers of the GPU parity tests: run the CUDA library and the CPU oracle on
the same seeded inputs and compare.

Tolerances (written here, used by every parity test):
  * bf16 outputs, one rounding from the oracle's inputs (the streams; the layer
    input from the GPU's streams): where the result is not much smaller than
    its terms (|o| >= 2^-6 of the sum of the terms' magnitudes), the GPU's bf16
    value is the oracle's bf16 rounding of the exact result or an adjacent bf16
    value (at most one bf16 ulp apart: the fp32 result and the float64 one
    straddle a rounding point), and such 1-ulp flips are rare (at most 1 in 500
    elements; their count is reported at the end of the run). Where terms
    cancel, fp32 arithmetic carries an absolute error of order 2^-24 times the
    terms' magnitudes, which can exceed one ulp of the small result: there the
    bound is 2^-16 times that magnitude plus one ulp;
  * bf16 outputs end to end (the layer input from the oracle's own streams,
    which may differ from the GPU's by those flips): |g - o| <= 1e-2 |o| +
    1e-2 rms(o_row), the second term keeping near-zero entries from dominating;
  * fp32 coefficients: 1e-5 absolute, checked stage-wise: the oracle's
    coefficient step is evaluated on the bf16 streams the GPU wrote (a single
    1-ulp bf16 flip of a stream element moves a logit by ~|fn| * ulp, above 1e-5,
    so end to end the bar cannot be met by any implementation);
  * MXFP8: bit-exact scale and data bytes when the oracle quantises the GPU's
    bf16 layer input;
  * finalize gather indexing: bit-exact (row-coded inputs, one-hot weights).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle as O
from mhc_residual_stream_b200 import mhc as M

BF16_REL = 1e-2
COEFF_ABS = 1e-5
MAX_FLIP_FRAC = 2e-3
DEV = "cuda:0"
FLIPS = []  # (what, 1-ulp flips, elements) of every ulp check of the run


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def coeff_np(cw) -> dict:
    return {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in cw.as_dict().items()}


def assert_bf16_close(g: np.ndarray, o: np.ndarray, what: str):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    rows = o.reshape(o.shape[0], -1)
    rms = np.sqrt(np.mean(rows * rows, axis=1))
    rms = rms.reshape((-1,) + (1,) * (o.ndim - 1))
    err = np.abs(g - o)
    bound = BF16_REL * np.abs(o) + BF16_REL * rms
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, worst {np.max(err - bound):.3g}"


def bf16_ordinal(x) -> np.ndarray:
    """Position of each bf16 value on the number line: adjacent bf16 values are
    one apart (+0 and -0 share 0). x holds values that are bf16-exact."""
    b = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    b = b.astype(np.int32)
    mag = b & 0x7FFF
    return np.where(b < 0, -mag, mag)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (2^-133 below the normal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -126)))
    return np.ldexp(1.0, (e - 7).astype(np.int64))


def assert_bf16_ulp(g: np.ndarray, o_rounded: np.ndarray, what: str, terms=None) -> int:
    """g (bf16 values) against the oracle's bf16 rounding of the same quantity.
    `terms` (same shape, optional) is the sum of the magnitudes of the terms the
    value adds up; elements with |o| >= 2^-6 terms (or all, without it) must be at
    most one bf16 ulp apart, with 1-ulp flips in at most MAX_FLIP_FRAC of them;
    the others within 2^-16 terms + one ulp. Returns the number of flips."""
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o_rounded, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    assert np.isfinite(g).all(), what + ": non-finite values"
    well = np.ones(o.shape, dtype=bool) if terms is None else np.abs(o) >= np.ldexp(np.asarray(terms), -6)
    d = np.abs(bf16_ordinal(g) - bf16_ordinal(o))
    dw = d[well]
    flips = int((dw == 1).sum())
    FLIPS.append((what, flips, dw.size))
    assert dw.size == 0 or dw.max() <= 1, \
        f"{what}: {int((dw > 1).sum())} elements more than one bf16 ulp off (worst {int(dw.max())})"
    assert flips <= MAX_FLIP_FRAC * max(dw.size, 1), f"{what}: {flips} of {dw.size} elements one ulp off"
    if terms is not None and (~well).any():
        t = np.asarray(terms)[~well]
        err = np.abs(g[~well] - o[~well])
        bound = np.ldexp(t, -16) + bf16_ulp(o[~well])
        assert (err <= bound).all(), f"{what}: {int((err > bound).sum())} cancelling elements beyond 2^-16 terms + ulp"
    return flips


def stream_terms(partials, residual, post, comb):
    """Per new-stream element, the sum of the magnitudes of its terms:
    sum_j |comb[j][i] res[j]| + |post[i]| sum_p |partial_p| (float64)."""
    res = np.abs(np.asarray(residual, dtype=np.float64))
    xa = np.sum(np.abs(np.asarray(partials, dtype=np.float64)), axis=0)
    return np.einsum("rji,rjh->rih", np.abs(np.asarray(comb, dtype=np.float64)), res) + \
        np.abs(np.asarray(post, dtype=np.float64))[:, :, None] * xa[:, None, :]


def collapse_terms(streams, pre):
    """Per collapse element, sum_j |pre[j] new[j]| (float64)."""
    return np.einsum("rj,rjh->rh", np.abs(np.asarray(pre, dtype=np.float64)),
                     np.abs(np.asarray(streams, dtype=np.float64)))


def assert_coeffs_close(g: dict, o_post, o_comb, o_pre, what: str):
    for name, ov in (("post", o_post), ("comb", o_comb), ("pre", o_pre)):
        gv = f64(g[name])
        err = np.max(np.abs(gv - ov)) if gv.size else 0.0
        assert err <= COEFF_ABS, f"{what}: {name} max |err| {err:.3g} > {COEFF_ABS}"


def to_dev(d: dict) -> dict:
    return {k: (v.to(DEV).contiguous() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def alloc_outputs(R, n, H, mxfp8=True, swizzled=True, coeff=True):
    out = {
        "residual_out": torch.empty(R, n, H, dtype=torch.bfloat16, device=DEV),
        "layer_input": torch.empty(R, H, dtype=torch.bfloat16, device=DEV),
    }
    if mxfp8:
        out["q_data"] = torch.empty(R, H, dtype=torch.uint8, device=DEV)
        out["q_scale"] = torch.full((M.mhc_mxfp8_scale_bytes(R, H, swizzled),), 0xAB, dtype=torch.uint8,
                                    device=DEV)
    if coeff:
        out["post"] = torch.empty(R, n, dtype=torch.float32, device=DEV)
        out["comb"] = torch.empty(R, n, n, dtype=torch.float32, device=DEV)
        out["pre"] = torch.empty(R, n, dtype=torch.float32, device=DEV)
    return out


def gpu_post_pre(d: dict, *, mxfp8=True, swizzled=True, coeff=True, residual_only=False, ws=None,
                 in_place=False, partials=None, packed=False):
    """Run mhc_boundary_post_pre on the inputs of synthetic.draw_boundary; CPU results."""
    g = to_dev({k: d[k] for k in ("partials", "residual", "post", "comb", "pre", "norm_weight")})
    R, n, H = g["residual"].shape
    if partials is not None:
        g["partials"] = partials
    out = alloc_outputs(R, n, H, mxfp8 and not residual_only, swizzled, coeff and not residual_only)
    if in_place:
        out["residual_out"] = g["residual"]
    if ws is None:
        ws = M.new_workspace(R, H, n, DEV)
    cw = None if (not coeff or residual_only) else M.Coeffs.from_weights(d["coeff"], DEV, packed=packed)
    M.mhc_boundary_post_pre(
        g["partials"], g["residual"], g["post"], g["comb"], None if residual_only else g["pre"],
        None if residual_only else g["norm_weight"], d["norm_eps"], cw, out["residual_out"],
        layer_input=None if residual_only else out["layer_input"],
        mxfp8=(out["q_data"], out["q_scale"], swizzled) if (mxfp8 and not residual_only) else None,
        post_out=out.get("post"), comb_out=out.get("comb"), pre_out=out.get("pre"), workspace=ws)
    torch.cuda.synchronize()
    st = M.mhc_get_device_status(ws)
    assert st == M.OK, M.STATUS_NAMES[st]
    res = {k: v.cpu() for k, v in out.items()}
    if residual_only:
        res = {"residual_out": res["residual_out"]}
    return res


def oracle_post_pre(d: dict, *, mxfp8=True, swizzled=True, coeff=True, residual_only=False):
    f = {k: f64(d[k]) for k in ("partials", "residual", "post", "comb", "pre", "norm_weight")}
    return O.boundary(partials=f["partials"], residual=f["residual"], post=f["post"], comb=f["comb"],
                      pre=None if residual_only else f["pre"], norm_weight=f["norm_weight"],
                      norm_eps=d["norm_eps"], coeff=coeff_np(d["coeff"]) if coeff else None,
                      mxfp8=mxfp8, swizzled=swizzled)


def check_tail(d: dict, gpu: dict, orc: dict, *, mxfp8=True, swizzled=True, coeff=True, what=""):
    """Stage-wise and end-to-end checks of everything after the new streams."""
    g_res = f64(gpu["residual_out"])
    assert_bf16_close(f64(gpu["layer_input"]), orc["layer_input"], what + " layer_input (end to end)")
    # stage-wise: the oracle's collapse + RMSNorm of the GPU's streams
    li_stage = O.rms_norm(O.collapse(g_res, f64(d["pre"])), f64(d["norm_weight"]), d["norm_eps"])
    g_li = f64(gpu["layer_input"])
    assert_bf16_close(g_li, li_stage, what + " layer_input (stage-wise)")
    c_abs = collapse_terms(g_res, f64(d["pre"]))
    c = O.collapse(g_res, f64(d["pre"]))
    # y = c * inv * w: the terms' magnitude scales with |y / c| wherever c is not tiny
    scale = np.abs(li_stage) / np.maximum(np.abs(c), 1e-30)
    assert_bf16_ulp(g_li, li_stage, what + " layer_input (stage-wise, ulp)", terms=c_abs * scale)
    if mxfp8:
        data, sc = O.mxfp8_quantize(g_li)
        want_scale = O.swizzle_scales_128x4(sc) if swizzled else sc.reshape(-1)
        assert np.array_equal(gpu["q_data"].numpy(), data), what + " mxfp8 data not bit-exact"
        assert np.array_equal(gpu["q_scale"].numpy().reshape(-1), want_scale), what + " mxfp8 scale not bit-exact"
    if coeff:
        post, comb, pre = O.mhc_coefficients(g_res, **coeff_np(d["coeff"]))
        assert_coeffs_close(gpu, post, comb, pre, what + " coefficients (stage-wise)")
