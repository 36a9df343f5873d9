"""Float64 CPU oracle of the mHC boundary (test infrastructure only).

Sources. The three pages this follows are the vLLM API pages
``...specialized_decode.boundary.boundary`` (cited below as [boundary]),
``...specialized_decode.boundary.all_reduce`` ([all_reduce]) and
``...specialized_decode.runtime.decode`` ([decode]). They fix the dataflow,
argument lists, dtypes and variants of the boundary, but they call the mHC
kernels (``AllReduceMHC``, ``mhc_pre_delayed_overlap``, ``mhc_post_tilelang``)
without printing their arithmetic. The arithmetic below is the plain reading of
the mHC post and pre steps those calls name; every place where the pages leave a
choice open is marked READING and listed with its alternatives in the design
notes of the repository.

Notation: R rows (tokens), n = hc_mult streams, H hidden, K = n*H,
C = 2n + n^2 logits, P partial buffers, k = top_k.

Representation: every bf16 tensor is passed in and returned as a float64 array
holding bf16-exact values. Every rounding to bf16 is explicit (``bf16_round``).
Byte outputs (E4M3 data, E8M0 scales) are uint8 arrays.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_round",
    "e4m3_encode",
    "e4m3_decode",
    "e8m0_exponent",
    "mxfp8_quantize",
    "mxfp8_dequantize",
    "scale_bytes_swizzled",
    "swizzle_scales_128x4",
    "sigmoid",
    "sinkhorn",
    "partial_sum",
    "moe_finalize",
    "post_mix",
    "collapse",
    "rms_norm",
    "logit_groups",
    "mhc_coefficients",
    "stream_mean",
    "final_head",
    "boundary",
    "coeffs_entry",
]

# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------


def bf16_round(x):
    """Round float64 values to the nearest bfloat16, ties to even.

    bfloat16 keeps 8 significant bits and the float32 exponent range
    (normal binades 2^-126 .. 2^127, subnormal spacing 2^-133). A value with
    leading binade q is rounded on the grid of spacing 2^(q-7); ``np.rint``
    rounds the exact quotient to the nearest integer with ties to even, which
    is ties-to-even on the last significand bit. Values that round to 2^128
    or beyond become infinities. NaN stays NaN.

    Pinned in the tests against torch's float32 -> bfloat16 conversion
    (a library routine) on float32-exact inputs.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    fin = np.isfinite(x)
    xf = x[fin]
    _, e = np.frexp(np.abs(xf))  # |x| = m * 2^e, m in [0.5, 1)
    q = np.maximum(e - 1, -126)  # leading binade, clamped to the subnormal floor
    ulp = np.ldexp(1.0, q - 7)
    r = np.rint(xf / ulp) * ulp
    r = np.where(np.abs(r) >= 2.0**128, np.copysign(np.inf, xf), r)
    out[fin] = r
    return out


_E4M3_MAX = 448.0  # 1.75 * 2^8: exponent field 15, mantissa 6 (mantissa 7 is NaN)


def e4m3_encode(v):
    """Encode float64 values as E4M3 (OCP 'fn' variant) bytes, RNE, satfinite.

    Format: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normal
    values (1 + m/8) * 2^(E-7) for E in 1..15 except E=15, m=7 which is NaN;
    subnormals m * 2^-9; no infinities; max finite 448.

    Rounding: to the nearest representable value with ties to even mantissa
    (``np.rint`` on the exact quotient by the spacing), then magnitudes above
    448 saturate to 448 ("satfinite"). Signs are kept, including -0 -> 0x80.
    NaN encodes as 0x7F.

    Pinned in the tests: every finite bfloat16 magnitude up to 448 against
    torch's float32 -> float8_e4m3fn cast (a library routine); hand-derived
    codes in tests/golden/e4m3_codes.txt.
    """
    v = np.asarray(v, dtype=np.float64)
    nan = np.isnan(v)
    sign = np.signbit(v).astype(np.uint8)
    a = np.where(nan, 0.0, np.abs(v))
    a = np.minimum(a, 2.0 * _E4M3_MAX)  # keeps the arithmetic finite; saturates below
    _, e = np.frexp(a)
    q = np.maximum(e - 1, -6)  # binade; below 2^-6 the spacing is the subnormal 2^-9
    spacing = np.ldexp(1.0, q - 3)
    r = np.rint(a / spacing) * spacing
    r = np.minimum(r, _E4M3_MAX)
    # value -> (exponent field, mantissa field)
    _, e2 = np.frexp(r)
    qr = e2 - 1
    is_sub = (r < 2.0**-6)
    exp_field = np.where(is_sub, 0, qr + 7)
    mant = np.where(is_sub, r / 2.0**-9, (r / np.ldexp(1.0, qr) - 1.0) * 8.0)
    mant = np.where(r == 0.0, 0.0, mant)
    exp_field = np.where(r == 0.0, 0, exp_field)
    code = (sign << 7) | (exp_field.astype(np.uint8) << 3) | mant.astype(np.uint8)
    code = np.where(nan, np.uint8(0x7F), code).astype(np.uint8)
    return code


def e4m3_decode(code):
    """Value of E4M3 bytes (OCP 'fn' variant), as float64; 0x7F/0xFF are NaN."""
    code = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(code & 0x80, -1.0, 1.0)
    ef = (code >> 3) & 0xF
    m = code & 0x7
    val = np.where(ef == 0, m * 2.0**-9, (1.0 + m / 8.0) * np.ldexp(1.0, ef - 7))
    val = np.where((ef == 15) & (m == 7), np.nan, val)
    return s * val


def e8m0_exponent(amax):
    """The block exponent e of an MXFP8 block with largest magnitude ``amax``.

    READING (parity unpinned as a convention): e is the smallest integer with
    amax <= 448 * 2^e, so that no element of the block saturates. Written with
    amax = m * 2^q, m in [1, 2): e = q - 8 when m <= 1.75, else e = q - 7.
    Clamped to [-127, 127]. The OCP MX rule floor(log2 amax) - 8 is the
    documented alternative. A zero amax gives -127 (scale byte 0).

    Pinned in the tests by the defining inequality and minimality on
    exhaustive bfloat16 magnitudes, and by hand-derived golden values.
    """
    amax = np.asarray(amax, dtype=np.float64)
    m, e = np.frexp(amax)  # amax = m * 2^e, m in [0.5, 1)
    mant = 2.0 * m  # in [1, 2)
    q = e - 1
    ex = np.where(mant <= 1.75, q - 8, q - 7)
    ex = np.where(amax == 0.0, -127, ex)
    return np.clip(ex, -127, 127).astype(np.int64)


def mxfp8_quantize(y):
    """MXFP8 of a bf16-valued [R, H] array: (data uint8 [R, H], scale uint8 [R, H/32]).

    Blocks are 32 consecutive elements of a row. Per block: e = e8m0_exponent
    of the block's largest magnitude, scale byte e + 127, data
    e4m3_encode(y * 2^-e) (the scaling by a power of two is exact).
    A block holding a NaN or an infinity is out of contract; it is encoded as
    scale byte 0xFF and data 0x7F (NaN) throughout.

    [boundary: empty_quantized_layer_input] fixes the container: E4M3 data of
    shape [T, H] and a uint8 scale buffer; the block size 32 and the E8M0
    scale are the MXFP8 format's.
    """
    y = np.asarray(y, dtype=np.float64)
    R, H = y.shape
    assert H % 32 == 0
    blocks = y.reshape(R, H // 32, 32)
    finite = np.all(np.isfinite(blocks), axis=2)
    amax = np.max(np.abs(np.where(np.isfinite(blocks), blocks, 0.0)), axis=2)
    ex = e8m0_exponent(amax)
    scaled = blocks * np.ldexp(1.0, -ex)[:, :, None]
    data = e4m3_encode(scaled)
    data = np.where(finite[:, :, None], data, np.uint8(0x7F)).astype(np.uint8)
    scale = np.where(finite, ex + 127, 0xFF).astype(np.uint8)
    return data.reshape(R, H), scale


def mxfp8_dequantize(data, scale):
    """Inverse map of ``mxfp8_quantize``: float64 [R, H] from bytes and linear scales."""
    data = np.asarray(data, dtype=np.uint8)
    R, H = data.shape
    ex = np.asarray(scale, dtype=np.int64) - 127
    vals = e4m3_decode(data).reshape(R, H // 32, 32)
    return (vals * np.ldexp(1.0, ex)[:, :, None]).reshape(R, H)


def scale_bytes_swizzled(rows, hidden):
    """Bytes of the swizzled 128x4 scale buffer for a [rows, hidden] MXFP8 tensor:
    rows rounded up to 128 times hidden/32 rounded up to 4."""
    sc = hidden // 32
    return ((rows + 127) // 128 * 128) * ((sc + 3) // 4 * 4)


def swizzle_scales_128x4(scale):
    """Place linear [R, H/32] scale bytes in the swizzled 128x4 layout.

    [boundary: empty_quantized_layer_input] names the layout ("FlashInfer's
    swizzled 128x4 scales") without drawing it. READING: the public block
    scaling-factor layout of NVIDIA's block-scaled GEMMs. The [R, H/32] scale
    matrix is padded to a multiple of 128 rows and 4 columns and cut into
    128x4 tiles of 512 bytes, laid out tile row by tile row. Inside a tile,
    row r and column c sit at byte (r % 32) * 16 + (r // 32) * 4 + c. Padding
    bytes are 0.

    Pinned in the tests against an independent construction of the same
    layout by reshape and transpose, and by hand-placed golden offsets.
    """
    scale = np.asarray(scale, dtype=np.uint8)
    R, S = scale.shape
    rows_p = (R + 127) // 128 * 128
    cols_p = (S + 3) // 4 * 4
    out = np.zeros(rows_p * cols_p, dtype=np.uint8)
    col_tiles = cols_p // 4
    for r in range(R):
        for c in range(S):
            tile = (r // 128) * col_tiles + (c // 4)
            rr, cc = r % 128, c % 4
            out[tile * 512 + (rr % 32) * 16 + (rr // 32) * 4 + cc] = scale[r, c]
    return out


# --------------------------------------------------------------------------
# Coefficients: RMS-normalised projection, sigmoid, Sinkhorn
# --------------------------------------------------------------------------


def sigmoid(x):
    """Logistic function 1 / (1 + e^-x) in float64."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def sinkhorn(logits, iters, eps):
    """Doubly stochastic matrix from an [n, n] logit matrix L (indexed [j, i]).

    [boundary: Boundaries.sublayer] passes ``hc_sinkhorn_iters`` and a second
    ``hc_eps`` to the coefficient kernel; the pages print no more.
    READING (parity unpinned as to the eps placement and step order):
        M = exp(L - max L)        (the shift cancels in the first row step)
        repeat iters times:
            each row j of M divided by (its sum over i) + eps
            each column i of M divided by (its sum over j) + eps
    Ending on the column step makes the column sums sum_j M[j, i], which the
    post-mix weights stream j into stream i with, equal to 1 - O(eps).

    Pinned in the tests by the 2x2 closed form of Sinkhorn scaling, column
    sums, convergence of row sums, and permutation equivariance.
    """
    L = np.asarray(logits, dtype=np.float64)
    M = np.exp(L - np.max(L))
    for _ in range(int(iters)):
        M = M / (M.sum(axis=1, keepdims=True) + eps)
        M = M / (M.sum(axis=0, keepdims=True) + eps)
    return M


def logit_groups(n):
    """Scale group of each of the 2n + n^2 logits: 0 for pre, 1 for post, 2 for comb.

    READING (parity unpinned as a convention): the fn columns are ordered
    [pre 0..n-1 | post n..2n-1 | comb 2n..2n+n^2-1], and comb column
    2n + j*n + i is comb[j, i] (stream j into stream i).
    """
    return np.array([0] * n + [1] * n + [2] * (n * n), dtype=np.int64)


def mhc_coefficients(streams, fn, scale, base, rms_eps, pre_eps, sinkhorn_eps,
                     post_alpha, sinkhorn_iters):
    """Next coefficients (post [R, n], comb [R, n, n], pre [R, n]) from bf16 streams.

    [boundary: Boundaries.sublayer, Boundaries._pre] call the coefficient
    kernel as (residual, fn, scale, base, rms_norm_eps, hc_eps, hc_eps,
    hc_post_alpha, hc_sinkhorn_iters) and receive (post, comb, layer_input,
    next_pre). READING of the arithmetic:
      v      = the streams of a row flattened to K = n*H values, k = j*H + h
      inv    = 1 / sqrt(mean_k v_k^2 + rms_norm_eps)       (no weight)
      l_c    = scale[group(c)] * inv * sum_k v_k fn[k, c] + base[c]
      pre'   = sigmoid(l_pre) + hc_eps (first)
      post'  = hc_post_alpha * sigmoid(l_post)
      comb'  = sinkhorn(l_comb as [j, i], hc_sinkhorn_iters, hc_eps (second))
    Normalising after the projection is the same number as projecting the
    normalised streams.

    Pinned in the tests by: the closed form when a column of fn equals a row's
    own streams; invariance under scaling the streams by 2^s (with zero eps);
    the first-layer fold identity; brute force at n=2, H=8; the group order
    by columns that touch only one output.
    """
    s = np.asarray(streams, dtype=np.float64)
    R, n, H = s.shape
    v = s.reshape(R, n * H)
    fn = np.asarray(fn, dtype=np.float64)
    assert fn.shape == (n * H, 2 * n + n * n)
    inv = 1.0 / np.sqrt(np.mean(v * v, axis=1) + rms_eps)
    dots = v @ fn
    g = logit_groups(n)
    sc = np.asarray(scale, dtype=np.float64)[g]
    logits = sc[None, :] * inv[:, None] * dots + np.asarray(base, dtype=np.float64)[None, :]
    pre = sigmoid(logits[:, :n]) + pre_eps
    post = post_alpha * sigmoid(logits[:, n:2 * n])
    comb = np.stack([sinkhorn(logits[r, 2 * n:].reshape(n, n), sinkhorn_iters, sinkhorn_eps)
                     for r in range(R)]) if R else np.zeros((0, n, n))
    return post, comb, pre


# --------------------------------------------------------------------------
# The boundary: reduce, post-mix, collapse, RMSNorm
# --------------------------------------------------------------------------


def partial_sum(partials):
    """x[r, h] = sum over p of partials[p, r, h], in float64.

    On the pages every sublayer ends in TP-partial outputs that the boundary
    all-reduces ([boundary] module text; [boundary: Boundaries.post_only]
    calls tensor_model_parallel_all_reduce). On one GPU the P partials are
    local buffers and the reduction is this sum. Pinned by the zero-partials
    and one-partial cases of the post-mix tests.
    """
    return np.sum(np.asarray(partials, dtype=np.float64), axis=0)


def moe_finalize(gemm2_permuted, expert_weights, expanded_idx_to_permuted_idx,
                 shared_output):
    """x[r] = shared_output[r] + sum_t expert_weights[r, t] * gemm2_permuted[e2p[r*k + t]].

    [all_reduce: BoundaryAllReduce.finalize] and [boundary: Boundaries._reduce]
    pass (gemm2_permuted, expert_weights, expanded_idx_to_permuted_idx,
    shared_output) for an unfinalized MoE output.
    READING (parity unpinned as to the index convention): the expanded index
    of (row r, slot t) is r*top_k + t, matching expert_weights [R, top_k]; an
    index below zero contributes nothing. An index at or above the number of
    permuted rows is an error.

    Pinned in the tests by one-hot weights on row-coded inputs, which must
    reproduce the selected permuted row exactly.
    """
    g = np.asarray(gemm2_permuted, dtype=np.float64)
    w = np.asarray(expert_weights, dtype=np.float64)
    idx = np.asarray(expanded_idx_to_permuted_idx, dtype=np.int64)
    sh = np.asarray(shared_output, dtype=np.float64)
    R, k = w.shape
    assert idx.shape == (R * k,)
    if np.any(idx >= g.shape[0]):
        raise ValueError("expanded_idx_to_permuted_idx points past gemm2_permuted")
    x = sh.copy()
    for r in range(R):
        for t in range(k):
            p = idx[r * k + t]
            if p >= 0:
                x[r] += w[r, t] * g[p]
    return x


def post_mix(residual, x, post, comb):
    """mHC post: new[r, i, h] = bf16(sum_j comb[r, j, i] res[r, j, h] + post[r, i] x[r, h]).

    [boundary: BoundaryState] carries post and comb of the sublayer that
    produced the pending output; [boundary: Boundaries.post_only] applies them
    as mhc_post(x, residual, post, comb). READING: x stays float64 (not
    rounded to bf16 first); the new streams are rounded to bf16 once.

    Pinned in the tests: comb = I, post = 0 returns the streams bit for bit;
    comb = I, post = e_i adds x to stream i only; zero x leaves the comb mix.
    """
    res = np.asarray(residual, dtype=np.float64)
    comb = np.asarray(comb, dtype=np.float64)
    post = np.asarray(post, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    mixed = np.einsum("rji,rjh->rih", comb, res) + post[:, :, None] * x[:, None, :]
    return bf16_round(mixed)


def collapse(streams, pre):
    """c[r, h] = sum_j pre[r, j] streams[r, j, h] in float64.

    [boundary: Boundaries.sublayer] collapses with state.pre, the pre-mix
    carried from the previous boundary ([boundary: BoundaryState], "the
    pre-mix the next collapse uses"), not with the pre computed at this one.
    """
    return np.einsum("rj,rjh->rh", np.asarray(pre, dtype=np.float64),
                     np.asarray(streams, dtype=np.float64))


def rms_norm(c, weight, eps):
    """y[r, h] = bf16(c[r, h] / sqrt(mean_h c[r, h]^2 + eps) * weight[h]).

    The layer input of [boundary: Boundaries.sublayer] (attn_norm or
    ffn_norm). READING: one rounding to bf16, after the weight.
    Pinned in the tests: a constant row gives sign(c) * weight up to eps.
    """
    c = np.asarray(c, dtype=np.float64)
    inv = 1.0 / np.sqrt(np.mean(c * c, axis=1) + eps)
    return bf16_round(c * inv[:, None] * np.asarray(weight, dtype=np.float64)[None, :])


def stream_mean(streams):
    """aux[r, h] = bf16(mean over j of streams[r, j, h]).

    The hidden state a boundary keeps for the layers that capture it
    ([boundary: Boundaries.sublayer] with capture_aux: the mean over dim 1 of
    the new streams; [decode: SpecializedDecode.run] the same after the last
    post_only). READING: the exact mean rounded once to bf16 (torch reduces
    bf16 in fp32 and rounds the result once; for n <= 4 bf16 inputs the fp32
    sum is exact unless the inputs span more than 16 binades).
    """
    return bf16_round(np.mean(np.asarray(streams, dtype=np.float64), axis=1))


def final_head(streams, pre, norm_weight, norm_eps):
    """The decode step's hidden state after the last layer ([decode:
    SpecializedDecode._head]): the final norm of hc_collapse(streams, pre),
    with the pre carried from the last boundary that computed one."""
    return rms_norm(collapse(streams, pre), norm_weight, norm_eps)


def boundary(*, residual, post, comb, partials=None, moe=None, pre=None,
             norm_weight=None, norm_eps=0.0, coeff=None, mxfp8=False,
             swizzled=True, aux=False):
    """One boundary: reduce pending, post-mix, and with ``pre`` the layer input
    and (with ``coeff``) the next coefficients.

    ``partials`` [P, R, H] (the all-reduce front) or ``moe`` = dict(
    gemm2_permuted, expert_weights, expanded_idx_to_permuted_idx,
    shared_output) (the finalize front) — exactly one.
    ``pre`` None is the residual-only variant ([boundary: Boundaries._reduce]:
    no pre, no norm); it returns the streams only.
    ``coeff`` = dict(fn, scale, base, rms_eps, pre_eps, sinkhorn_eps,
    post_alpha, sinkhorn_iters) or None.

    ``aux`` also returns 'aux', the stream mean of the new streams.

    Returns a dict with 'residual' and, with pre: 'layer_input', and with
    mxfp8: 'mxfp8_data', 'mxfp8_scale' (swizzled or linear bytes), and with
    coeff: 'post', 'comb', 'pre'.
    """
    assert (partials is None) != (moe is None)
    if partials is not None:
        x = partial_sum(partials)
    else:
        x = moe_finalize(moe["gemm2_permuted"], moe["expert_weights"],
                         moe["expanded_idx_to_permuted_idx"], moe["shared_output"])
    new = post_mix(residual, x, post, comb)
    out = {"residual": new}
    if aux:
        out["aux"] = stream_mean(new)
    if pre is None:
        return out
    y = rms_norm(collapse(new, pre), norm_weight, norm_eps)
    out["layer_input"] = y
    if mxfp8:
        data, sc = mxfp8_quantize(y)
        out["mxfp8_data"] = data
        out["mxfp8_scale"] = swizzle_scales_128x4(sc) if swizzled else sc
    if coeff is not None:
        out["post"], out["comb"], out["pre"] = mhc_coefficients(new, **coeff)
    return out


def coeffs_entry(*, residual=None, x=None, hc_mult=None, pre_mix=None,
                 norm_weight=None, norm_eps=0.0, layer_input=True, coeff):
    """The stock mHC pre without a reduction ([boundary: Boundaries._pre]).

    Either ``residual`` [R, n, H] (with ``pre_mix`` [R, n] for the layer
    input), or the first layer's ``x`` [R, H] ([boundary: Boundaries.first]):
    the embedding broadcast to the n streams, whose identity pre-mix selects
    stream 0, so the layer input is the RMSNorm of x itself.

    Returns a dict with 'residual' (the broadcast streams for x), 'post',
    'comb', 'pre' and, with layer_input, 'layer_input'.
    """
    assert (residual is None) != (x is None)
    out = {}
    if x is not None:
        assert pre_mix is None
        x = np.asarray(x, dtype=np.float64)
        streams = np.repeat(x[:, None, :], hc_mult, axis=1)
        out["residual"] = streams
        if layer_input:
            out["layer_input"] = rms_norm(x, norm_weight, norm_eps)
    else:
        streams = np.asarray(residual, dtype=np.float64)
        if layer_input:
            out["layer_input"] = rms_norm(collapse(streams, pre_mix), norm_weight, norm_eps)
    out["post"], out["comb"], out["pre"] = mhc_coefficients(streams, **coeff)
    return out
