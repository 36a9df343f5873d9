"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something other than its own formula:
a library routine (torch's float conversions), a closed form, a hand-derived
golden value under tests/golden/, an invariant the mathematics fixes, or an
independent brute-force evaluation. A plausible mistake in the oracle (a
dropped term, a wrong sign, a swapped index, a transposed operand) fails one
of them.
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from mhc_residual_stream_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append(line.split())
    return out


def _all_bf16_finite_positive():
    bits = np.arange(0x0001, 0x7F80, dtype=np.uint32)  # +subnormals .. +max finite
    return (bits << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- bf16

def test_bf16_round_matches_torch_on_random_float32():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(f.astype(np.float64))
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_bf16_round_ties_and_signs():
    one = 1.0
    assert O.bf16_round(np.array([one + 2**-8]))[0] == 1.0  # tie -> even
    assert O.bf16_round(np.array([one + 3 * 2**-8]))[0] == one + 2**-6
    assert np.signbit(O.bf16_round(np.array([-0.0]))[0])
    assert O.bf16_round(np.array([2.0**-134]))[0] == 0.0  # tie with 0 -> 0
    assert O.bf16_round(np.array([3 * 2.0**-134]))[0] == 2.0**-132


# ---------------------------------------------------------------- E4M3

def test_e4m3_exhaustive_vs_torch_in_range():
    mags = _all_bf16_finite_positive()
    mags = mags[mags <= 448.0]
    vals = np.concatenate([mags, -mags, [0.0, -0.0]])
    ref = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(vals)
    assert np.array_equal(got, ref)


def test_e4m3_golden_codes():
    for v, code, *_ in _rows("e4m3_codes.txt"):
        assert int(O.e4m3_encode(np.array([float(v)]))[0]) == int(code, 16), v


def test_e4m3_decode_inverts_encode_and_error_bound():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    assert np.array_equal(O.e4m3_encode(vals), codes)
    mags = _all_bf16_finite_positive()
    mags = mags[(mags >= 2.0**-6) & (mags <= 448.0)]
    deq = O.e4m3_decode(O.e4m3_encode(mags))
    assert np.max(np.abs(deq - mags) / mags) <= 2.0**-4


# ---------------------------------------------------------------- E8M0 / MXFP8

def test_e8m0_defining_inequality_and_minimality():
    a = _all_bf16_finite_positive()
    e = O.e8m0_exponent(a)
    assert np.all(a <= 448.0 * np.ldexp(1.0, e))
    not_clamped = e > -127
    assert np.all(a[not_clamped] > 448.0 * np.ldexp(1.0, e[not_clamped] - 1))


def test_e8m0_golden():
    for amax, byte, *_ in _rows("e8m0_cases.txt"):
        assert int(O.e8m0_exponent(np.array([float(amax)]))[0]) + 127 == int(byte), amax


def test_mxfp8_golden_block():
    rows = _rows("mxfp8_block.txt")
    scale_byte = int(rows[0][0])
    y = np.zeros((1, 32))
    want = np.zeros(32, dtype=np.uint8)
    for idx, val, code in rows[1:]:
        y[0, int(idx)] = float(val)
        want[int(idx)] = int(code, 16)
    assert np.array_equal(O.bf16_round(y), y)
    data, sc = O.mxfp8_quantize(y)
    assert int(sc[0, 0]) == scale_byte
    assert np.array_equal(data[0], want)


def _bf16_block_data(rng, R, H, spread=3.0):
    y = rng.standard_normal((R, H)) * np.exp(rng.standard_normal((R, H)) * spread)
    return O.bf16_round(y)


def test_mxfp8_power_of_two_equivariance():
    rng = np.random.default_rng(2)
    y = _bf16_block_data(rng, 6, 256)
    d0, s0 = O.mxfp8_quantize(y)
    for s in (-9, -1, 1, 5):
        d1, s1 = O.mxfp8_quantize(y * 2.0**s)
        assert np.array_equal(d1, d0)
        assert np.array_equal(s1.astype(int), s0.astype(int) + s)


def test_mxfp8_scaled_amax_range_and_dequant_error():
    rng = np.random.default_rng(3)
    y = _bf16_block_data(rng, 8, 512)
    d, s = O.mxfp8_quantize(y)
    e = s.astype(np.int64) - 127
    amax = np.max(np.abs(y.reshape(8, 16, 32)), axis=2)
    ratio = amax / np.ldexp(1.0, e)
    assert np.all((ratio > 224.0) & (ratio <= 448.0))
    deq = O.mxfp8_dequantize(d, s)
    step = np.repeat(np.ldexp(1.0, e - 10), 32, axis=1)  # half the subnormal spacing
    assert np.all(np.abs(deq - y) <= np.maximum(2.0**-4 * np.abs(y), step))


def test_mxfp8_zero_and_nonfinite_blocks():
    y = np.zeros((1, 64))
    y[0, 40] = np.nan
    d, s = O.mxfp8_quantize(y)
    assert s[0, 0] == 0 and np.all(d[0, :32] == 0)
    assert s[0, 1] == 0xFF and np.all(d[0, 32:] == 0x7F)


def _swizzle_by_reshape(scale):
    """The 128x4 layout built a second way: pad, then view the scale matrix as
    [row tiles, 4 row groups, 32 rows, col tiles, 4 cols] and reorder to
    [row tiles, col tiles, 32 rows, 4 row groups, 4 cols]."""
    R, Sc = scale.shape
    Rp, Sp = -(-R // 128) * 128, -(-Sc // 4) * 4
    pad = np.zeros((Rp, Sp), dtype=np.uint8)
    pad[:R, :Sc] = scale
    t = pad.reshape(Rp // 128, 4, 32, Sp // 4, 4)
    return t.transpose(0, 3, 2, 1, 4).reshape(-1)


@pytest.mark.parametrize("R,Sc", [(1, 8), (5, 6), (128, 224), (130, 10)])
def test_swizzle_matches_independent_construction(R, Sc):
    rng = np.random.default_rng(R * 1000 + Sc)
    sc = rng.integers(1, 255, size=(R, Sc), dtype=np.uint8)
    got = O.swizzle_scales_128x4(sc)
    assert got.size == O.scale_bytes_swizzled(R, Sc * 32)
    assert np.array_equal(got, _swizzle_by_reshape(sc))


def test_swizzle_golden_offsets():
    for rows, scols, r, c, off in _rows("swizzle_128x4_offsets.txt"):
        rows, scols, r, c, off = map(int, (rows, scols, r, c, off))
        sc = np.zeros((rows, scols), dtype=np.uint8)
        sc[r, c] = 7
        out = O.swizzle_scales_128x4(sc)
        assert np.flatnonzero(out).tolist() == [off]


# ---------------------------------------------------------------- Sinkhorn

def test_sinkhorn_2x2_closed_form():
    for a, b, c, d, p in _rows("sinkhorn_2x2.txt"):
        L = np.log(np.array([[float(a), float(b)], [float(c), float(d)]]))
        M = O.sinkhorn(L, 200, 0.0)
        want = np.array([[float(p), 1 - float(p)], [1 - float(p), float(p)]])
        assert np.max(np.abs(M - want)) < 1e-12


def test_sinkhorn_sums_equivariance_and_shift():
    rng = np.random.default_rng(4)
    for n in (2, 3, 4, 6):
        L = rng.standard_normal((n, n)) * 1.5
        M = O.sinkhorn(L, 20, 1e-6)
        assert np.all(np.abs(M.sum(axis=0) - 1.0) < 1e-5)  # ends on the column step
        M0 = O.sinkhorn(L, 20, 0.0)
        assert np.all(np.abs(M0.sum(axis=0) - 1.0) < 1e-14)
        Minf = O.sinkhorn(L, 500, 0.0)
        assert np.all(np.abs(Minf.sum(axis=1) - 1.0) < 1e-10)
        pr, pc = rng.permutation(n), rng.permutation(n)
        Mp = O.sinkhorn(L[pr][:, pc], 20, 1e-6)
        assert np.allclose(Mp, M[pr][:, pc], rtol=0, atol=1e-15)
        assert np.allclose(O.sinkhorn(L + 3.25, 20, 1e-6), M, rtol=0, atol=1e-15)


def test_sinkhorn_uniform_and_zero_iterations():
    M = O.sinkhorn(np.zeros((4, 4)), 20, 0.0)
    assert np.allclose(M, 0.25, atol=1e-15)
    L = np.array([[0.0, 1.0], [2.0, 0.5]])
    assert np.allclose(O.sinkhorn(L, 0, 1e-6), np.exp(L - 2.0))


# ---------------------------------------------------------------- post-mix / finalize

def _small_boundary(seed=5, R=3, n=4, H=64, P=3):
    d = S.draw_boundary(R, H, n=n, partials=P, seed=seed)
    f = {k: (v.to(torch.float64).numpy() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    return d, f


def test_post_mix_identity_comb_zero_post_is_bitwise_residual():
    _, f = _small_boundary()
    R, n, H = f["residual"].shape
    comb = np.broadcast_to(np.eye(n), (R, n, n))
    out = O.post_mix(f["residual"], O.partial_sum(f["partials"]), np.zeros((R, n)), comb)
    assert np.array_equal(out, f["residual"])


def test_post_mix_adds_x_to_one_stream_only():
    _, f = _small_boundary()
    R, n, H = f["residual"].shape
    x = O.partial_sum(f["partials"])
    comb = np.broadcast_to(np.eye(n), (R, n, n))
    post = np.zeros((R, n))
    post[:, 2] = 1.0
    out = O.post_mix(f["residual"], x, post, comb)
    for i in range(n):
        want = O.bf16_round(f["residual"][:, i] + x) if i == 2 else f["residual"][:, i]
        assert np.array_equal(out[:, i], want)


def test_post_mix_direction_of_comb():
    # comb[r, j, i] carries stream j into stream i: a permutation moves streams.
    _, f = _small_boundary()
    R, n, H = f["residual"].shape
    perm = np.array([1, 2, 3, 0])
    comb = np.zeros((R, n, n))
    comb[:, np.arange(n), perm] = 1.0  # stream j -> stream perm[j]
    out = O.post_mix(f["residual"], np.zeros((R, H)), np.zeros((R, n)), comb)
    for j in range(n):
        assert np.array_equal(out[:, perm[j]], f["residual"][:, j])


def test_partial_sum_single_partial_passthrough():
    _, f = _small_boundary(P=1)
    assert np.array_equal(O.partial_sum(f["partials"]), f["partials"][0])


def test_moe_finalize_one_hot_row_coded():
    R, k, H, n = 4, 3, 32, 2
    num = R * k + 5
    g = np.zeros((num, H))
    for p in range(num):
        g[p] = O.bf16_round((p + 1) * 1.0 + np.arange(H) / 64.0)
    rng = np.random.default_rng(6)
    idx = rng.permutation(num)[: R * k]
    w = np.zeros((R, k))
    sel = rng.integers(0, k, size=R)
    w[np.arange(R), sel] = 1.0
    x = O.moe_finalize(g, w, idx, np.zeros((R, H)))
    for r in range(R):
        assert np.array_equal(x[r], g[idx[r * k + sel[r]]])
    idx2 = idx.copy()
    idx2[0 * k + sel[0]] = -1
    x2 = O.moe_finalize(g, w, idx2, np.zeros((R, H)))
    assert np.all(x2[0] == 0.0)
    idx3 = idx.copy()
    idx3[1] = num
    with pytest.raises(ValueError):
        O.moe_finalize(g, w, idx3, np.zeros((R, H)))


def test_moe_finalize_weighted_row_coded():
    # slot weights 1/2, 1/4, 1/8 (exact in binary) on row-coded expert rows
    # g[p][h] = (p + 1) + h/64 and shared[r][h] = r/2: each output row is
    # shared + (4 (a+1) + 2 (b+1) + (c+1) + 7 h/64) / 8 for the selected rows a, b, c,
    # so a weight squared, a weight on the wrong slot or a slot dropped changes it
    R, k, H = 5, 3, 16
    num = R * k + 4
    h = np.arange(H)
    g = np.stack([(p + 1) + h / 64.0 for p in range(num)])
    shared = np.stack([np.full(H, r / 2.0) for r in range(R)])
    idx = np.random.default_rng(9).permutation(num)[: R * k]
    w = np.tile(np.array([0.5, 0.25, 0.125]), (R, 1))
    x = O.moe_finalize(g, w, idx, shared)
    for r in range(R):
        a, b, c = idx[r * k], idx[r * k + 1], idx[r * k + 2]
        want = r / 2.0 + (4 * (a + 1) + 2 * (b + 1) + (c + 1) + 7 * h / 64.0) / 8.0
        assert np.array_equal(x[r], want), r


# ---------------------------------------------------------------- collapse / norm / first layer

def test_rms_norm_constant_row():
    H = 128
    w = O.bf16_round(1.0 + np.random.default_rng(7).standard_normal(H) * 0.1)
    c = np.full((2, H), -3.0)
    c[1] = 0.75
    y = O.rms_norm(c, w, 1e-12)
    assert np.array_equal(y[0], O.bf16_round(-w))
    assert np.array_equal(y[1], O.bf16_round(w))


def test_first_layer_broadcast_identity_pre_and_fold():
    d = S.draw_first_layer(3, 64, n=4, seed=8)
    x = d["x"].double().numpy()
    w = d["norm_weight"].double().numpy()
    coeff = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v)
             for k, v in d["coeff"].as_dict().items()}
    out = O.coeffs_entry(x=x, hc_mult=4, norm_weight=w, norm_eps=1e-6, coeff=coeff)
    for j in range(4):
        assert np.array_equal(out["residual"][:, j], x)
    e0 = np.zeros((3, 4))
    e0[:, 0] = 1.0
    assert np.array_equal(O.collapse(out["residual"], e0), x)
    assert np.array_equal(out["layer_input"], O.rms_norm(x, w, 1e-6))
    # fold identity: the broadcast's coefficients equal x projected by the folded fn
    n, H = 4, 64
    fn = coeff["fn"]
    folded = fn.reshape(n, H, -1).sum(axis=0)
    inv = 1.0 / np.sqrt(np.mean(x * x, axis=1) + coeff["rms_eps"])
    logits = coeff["scale"][O.logit_groups(n)] * inv[:, None] * (x @ folded) + coeff["base"]
    pre = 1.0 / (1.0 + np.exp(-logits[:, :n])) + coeff["pre_eps"]
    post = coeff["post_alpha"] / (1.0 + np.exp(-logits[:, n:2 * n]))
    assert np.allclose(out["pre"], pre, rtol=0, atol=1e-12)
    assert np.allclose(out["post"], post, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- aux stream mean / final head

def test_stream_mean_hand_values_and_special_cases():
    # hand-computed: means of bf16-exact values, rounded once to bf16
    st = np.array([[[1.0, 3.0, -2.0], [2.0, 5.0, 2.0], [4.0, 0.5, -1.0], [5.0, 0.5, 1.0]]])  # [1, 4, 3]
    assert np.array_equal(O.stream_mean(st)[0], np.array([3.0, 2.25, 0.0]))
    # 1 + 2^-8 is not a bf16 value: the mean of (1, 1, 1, 1 + 2^-6) = 1 + 2^-8 rounds to even, 1.0
    st2 = np.array([[[1.0], [1.0], [1.0], [1.0 + 2.0 ** -6]]])
    assert O.stream_mean(st2)[0, 0] == 1.0
    # mean 1 + 3 * 2^-9 is 0.75 ulp above 1 (a bf16 ulp there is 2^-7): rounds up to 1 + 2^-7
    st3 = np.array([[[1.0 + 2.0 ** -7], [1.0 + 2.0 ** -7], [1.0 + 2.0 ** -7], [1.0]]])
    assert O.stream_mean(st3)[0, 0] == 1.0 + 2.0 ** -7
    # n identical streams: the mean is the stream; n = 1: the identity
    x = O.bf16_round(np.random.default_rng(11).standard_normal((3, 40)))
    assert np.array_equal(O.stream_mean(np.repeat(x[:, None, :], 4, axis=1)), x)
    assert np.array_equal(O.stream_mean(x[:, None, :]), x)


def test_final_head_is_the_norm_of_one_stream_for_a_one_hot_pre():
    rng = np.random.default_rng(12)
    st = O.bf16_round(rng.standard_normal((2, 4, 64)))
    w = O.bf16_round(1.0 + rng.standard_normal(64) * 0.1)
    for j in range(4):
        pre = np.zeros((2, 4))
        pre[:, j] = 1.0
        assert np.array_equal(O.final_head(st, pre, w, 1e-6), O.rms_norm(st[:, j], w, 1e-6))
    # a constant row collapses to sign * weight (see the RMSNorm pin)
    st2 = np.full((1, 4, 64), 0.5)
    pre = np.full((1, 4), 0.25)
    assert np.array_equal(O.final_head(st2, pre, w, 1e-12)[0], O.bf16_round(w))


def test_residual_only_streams_equal_full_path():
    d, f = _small_boundary(R=4, H=96, P=2)
    coeff = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v)
             for k, v in d["coeff"].as_dict().items()}
    full = O.boundary(partials=f["partials"], residual=f["residual"], post=f["post"],
                      comb=f["comb"], pre=f["pre"], norm_weight=f["norm_weight"],
                      norm_eps=1e-6, coeff=coeff, mxfp8=True)
    ronly = O.boundary(partials=f["partials"], residual=f["residual"], post=f["post"],
                       comb=f["comb"])
    assert np.array_equal(full["residual"], ronly["residual"])
    assert set(ronly) == {"residual"}


# ---------------------------------------------------------------- coefficients

def _coeff(n, H, seed, rms_eps=1e-6):
    g = S.gen(seed)
    cw = S.draw_coeff_weights(g, H, n, 0.02, affine=True)
    d = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in cw.as_dict().items()}
    d["rms_eps"] = rms_eps
    return d


def test_coefficients_closed_form_when_fn_column_is_the_row():
    n, H, R = 4, 32, 1
    rng = np.random.default_rng(9)
    v = O.bf16_round(rng.standard_normal((R, n, H)))
    c = _coeff(n, H, 10)
    fn = np.zeros((n * H, 2 * n + n * n))
    fn[:, 1] = v.reshape(-1)  # pre logit 1
    c["fn"] = fn
    post, comb, pre = O.mhc_coefficients(v, **c)
    ms = np.mean(v * v)
    logit = c["scale"][0] * np.sum(v * v) / math.sqrt(ms + c["rms_eps"]) + c["base"][1]
    assert abs(pre[0, 1] - (1.0 / (1.0 + math.exp(-logit)) + c["pre_eps"])) < 1e-12


def test_coefficients_invariant_under_power_of_two_scaling():
    n, H, R = 4, 48, 3
    rng = np.random.default_rng(11)
    v = O.bf16_round(rng.standard_normal((R, n, H)))
    c = _coeff(n, H, 12, rms_eps=0.0)
    a = O.mhc_coefficients(v, **c)
    for s in (-5, 3):
        b = O.mhc_coefficients(v * 2.0**s, **c)
        for x, y in zip(a, b):
            assert np.allclose(x, y, rtol=0, atol=1e-12)


def test_coefficient_groups_touch_only_their_output():
    n, H, R = 4, 16, 2
    rng = np.random.default_rng(13)
    v = O.bf16_round(rng.standard_normal((R, n, H)))
    c = _coeff(n, H, 14)
    c["fn"] = np.zeros((n * H, 2 * n + n * n))
    c["base"] = np.zeros(2 * n + n * n)
    post0, comb0, pre0 = O.mhc_coefficients(v, **c)
    # zero logits: pre = 1/2 + eps, post = alpha/2, comb uniform
    assert np.allclose(pre0, 0.5 + c["pre_eps"], atol=1e-15)
    assert np.allclose(post0, c["post_alpha"] / 2, atol=1e-15)
    assert np.allclose(comb0, 1.0 / n, atol=1e-5)
    for col, what in ((2, "pre"), (n + 1, "post"), (2 * n + 1 * n + 3, "comb")):
        cc = dict(c)
        cc["base"] = c["base"].copy()
        cc["base"][col] = 1.0
        post1, comb1, pre1 = O.mhc_coefficients(v, **cc)
        moved = {"pre": not np.allclose(pre1, pre0), "post": not np.allclose(post1, post0),
                 "comb": not np.allclose(comb1, comb0)}
        assert moved == {k: k == what for k in moved}
        if what == "pre":
            assert not np.allclose(pre1[:, 2], pre0[:, 2]) and np.allclose(np.delete(pre1, 2, 1), np.delete(pre0, 2, 1))
        if what == "post":
            assert not np.allclose(post1[:, 1], post0[:, 1]) and np.allclose(np.delete(post1, 1, 1), np.delete(post0, 1, 1))
        if what == "comb":
            # raising logit (j=1, i=3) raises comb[1, 3] above the rest of its row
            assert np.all(comb1[:, 1, 3] > comb0[:, 1, 3])
    # the scale of a group multiplies only that group's projection
    c["fn"] = rng.standard_normal((n * H, 2 * n + n * n)) * 0.05
    base = O.mhc_coefficients(v, **c)
    cc = dict(c)
    cc["scale"] = c["scale"].copy()
    cc["scale"][1] *= 2.0
    moved = O.mhc_coefficients(v, **cc)
    assert np.allclose(moved[2], base[2]) and np.allclose(moved[1], base[1])
    assert not np.allclose(moved[0], base[0])


# ---------------------------------------------------------------- brute force n=2 and n=3, H=8

def _bf16_exact(x: float) -> float:
    """bf16 rounding by exact rational arithmetic (independent of numpy)."""
    if x == 0.0:
        return x
    m, e = math.frexp(abs(x))
    q = max(e - 1, -126)
    ulp = Fraction(2) ** (q - 7)
    k = round(Fraction(abs(x)) / ulp)  # Fraction rounding: half to even
    return math.copysign(float(k * ulp), x)


@pytest.mark.parametrize("n", [2, 3])
def test_brute_force_small_matches_oracle(n):
    # n=3 as well: every 2x2 doubly stochastic matrix is symmetric, so n=2
    # alone cannot tell comb[j, i] from comb[i, j].
    H, R, P = 8, 3, 2
    d = S.draw_boundary(R, H, n=n, partials=P, seed=15, fn_std=0.2)
    t = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    cw = {k: (v.double().numpy() if isinstance(v, torch.Tensor) else v) for k, v in d["coeff"].as_dict().items()}
    part, res, post, comb, pre, w = t["partials"], t["residual"], t["post"], t["comb"], t["pre"], t["norm_weight"]
    eps = 1e-6
    out = O.boundary(partials=part, residual=res, post=post, comb=comb, pre=pre,
                     norm_weight=w, norm_eps=eps, coeff=cw)
    C = 2 * n + n * n
    for r in range(R):
        new = [[0.0] * H for _ in range(n)]
        for h in range(H):
            x = 0.0
            for p in range(P):
                x += float(part[p, r, h])
            for i in range(n):
                acc = float(post[r, i]) * x
                for j in range(n):
                    acc += float(comb[r, j, i]) * float(res[r, j, h])
                new[i][h] = _bf16_exact(acc)
        for i in range(n):
            for h in range(H):
                assert new[i][h] == out["residual"][r, i, h]
        csq, cs = 0.0, []
        for h in range(H):
            c = sum(float(pre[r, j]) * new[j][h] for j in range(n))
            cs.append(c)
            csq += c * c
        inv = 1.0 / math.sqrt(csq / H + eps)
        for h in range(H):
            assert abs(_bf16_exact(cs[h] * inv * float(w[h])) - out["layer_input"][r, h]) <= 1e-12
        vsq = sum(new[i][h] ** 2 for i in range(n) for h in range(H))
        invv = 1.0 / math.sqrt(vsq / (n * H) + cw["rms_eps"])
        logits = []
        for c in range(C):
            dot = sum(new[i][h] * float(cw["fn"][i * H + h, c]) for i in range(n) for h in range(H))
            grp = 0 if c < n else (1 if c < 2 * n else 2)
            logits.append(float(cw["scale"][grp]) * invv * dot + float(cw["base"][c]))
        for i in range(n):
            assert abs(1 / (1 + math.exp(-logits[i])) + cw["pre_eps"] - out["pre"][r, i]) < 1e-12
            assert abs(cw["post_alpha"] / (1 + math.exp(-logits[n + i])) - out["post"][r, i]) < 1e-12
        M = [[logits[2 * n + j * n + i] for i in range(n)] for j in range(n)]
        mx = max(max(row) for row in M)
        M = [[math.exp(v - mx) for v in row] for row in M]
        for _ in range(cw["sinkhorn_iters"]):
            for j in range(n):
                s = sum(M[j]) + cw["sinkhorn_eps"]
                M[j] = [v / s for v in M[j]]
            for i in range(n):
                s = sum(M[j][i] for j in range(n)) + cw["sinkhorn_eps"]
                for j in range(n):
                    M[j][i] /= s
        for j in range(n):
            for i in range(n):
                assert abs(M[j][i] - out["comb"][r, j, i]) < 1e-12
