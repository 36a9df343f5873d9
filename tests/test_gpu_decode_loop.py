"""GPU parity of the decode step's layer loop: 61 layers, 123 chained boundaries
(first-layer broadcast, MoE finalize + MXFP8 attention entries, partial-sum FFN
entries, the final finalize fused with the head), each checked against the
oracle on the inputs the GPU actually fed it (stage-wise), with the stream means
of the captured layers, plus a CUDA-graph replay of the whole step that must
equal the eager run bit for bit."""

import numpy as np
import pytest
import torch

import oracle as O
from mhc_residual_stream_b200 import mhc as M
from mhc_residual_stream_b200.decode import DecodeLoop

from _parity import assert_bf16_close, assert_coeffs_close, f64

pytestmark = pytest.mark.gpu


def _coeff_np(c: M.Coeffs):
    return dict(fn=f64(c.fn), scale=f64(c.scale), base=f64(c.base), rms_eps=c.rms_eps, pre_eps=c.pre_eps,
                sinkhorn_eps=c.sinkhorn_eps, post_alpha=c.post_alpha, sinkhorn_iters=c.sinkhorn_iters)


def test_decode_loop_every_boundary_stage_wise():
    _check_loop(DecodeLoop(rows=4, layers=61, device="cuda:0"), 123)


def test_decode_loop_with_engram_entries_stage_wise():
    # Engram layers: streams only (with the captured mean), then the coefficients
    # and layer input of the injected streams with the carried pre
    _check_loop(DecodeLoop(rows=8, layers=8, device="cuda:0", engram_layers=(2, 5), aux_layers=(2, 5, 8)), 19)


def _check_loop(loop, n_steps):
    assert len(loop.steps) == n_steps
    for st in loop.steps:
        a = st.src
        inp = {k: f64(getattr(loop, k)[a]) for k in ("res", "post", "comb", "pre")} if st.kind != "first" else {}
        loop.run_step(st)
        torch.cuda.synchronize()
        assert M.mhc_get_device_status(loop.workspace) == M.OK
        b = st.dst
        g_res = f64(loop.res[b])
        what = f"{st.kind} layer {st.layer}"
        if st.kind == "engram":  # stage-wise on the injected streams the GPU held
            o = O.coeffs_entry(residual=g_res, pre_mix=inp["pre"], norm_weight=f64(st.weights.norm_weight),
                               norm_eps=1e-6, coeff=_coeff_np(st.weights.coeffs))
            assert_bf16_close(f64(loop.layer_input), o["layer_input"], what + " layer input")
            assert_coeffs_close({"post": loop.post[b].cpu(), "comb": loop.comb[b].cpu(), "pre": loop.pre[b].cpu()},
                                o["post"], o["comb"], o["pre"], what)
            continue
        if st.kind == "first":
            x = f64(loop.x)
            o = O.coeffs_entry(x=x, hc_mult=4, norm_weight=f64(st.weights.norm_weight), norm_eps=1e-6,
                               coeff=_coeff_np(st.weights.coeffs))
            assert np.array_equal(g_res, o["residual"])
            assert_bf16_close(f64(loop.layer_input), o["layer_input"], what)
            assert_coeffs_close({"post": loop.post[b].cpu(), "comb": loop.comb[b].cpu(), "pre": loop.pre[b].cpu()},
                                o["post"], o["comb"], o["pre"], what)
            continue
        pd = st.pending
        final = st.kind == "final"
        kw = dict(residual=inp["res"], post=inp["post"], comb=inp["comb"])
        if pd.kind == "partials":
            kw["partials"] = f64(pd.partials)
        else:
            kw["moe"] = dict(gemm2_permuted=f64(pd.gemm2_permuted), expert_weights=f64(pd.expert_weights),
                             expanded_idx_to_permuted_idx=pd.e2p.cpu().numpy().astype(np.int64),
                             shared_output=f64(pd.shared_output))
        if st.kind != "post_only":
            nw = f64(loop.final_norm) if final else f64(st.weights.norm_weight)
            kw.update(pre=inp["pre"], norm_weight=nw, norm_eps=1e-6, mxfp8=st.mxfp8)
        o = O.boundary(**kw)
        assert_bf16_close(g_res, o["residual"], what + " streams")
        aux = loop.aux_of(st)
        if aux is not None:  # the stream mean of the streams the GPU wrote: exact
            assert np.array_equal(f64(aux), O.stream_mean(g_res)), what + " aux"
        if st.kind == "post_only":
            continue
        if final:  # the step's hidden state: final norm of the collapse with the carried pre
            g_h = f64(loop.hidden_out)
            assert_bf16_close(g_h, o["layer_input"], what + " hidden (end to end)")
            assert_bf16_close(g_h, O.final_head(g_res, inp["pre"], nw, 1e-6), what + " hidden (stage-wise)")
            continue
        g_li = f64(loop.layer_input)
        assert_bf16_close(g_li, o["layer_input"], what + " layer input")
        if st.mxfp8:
            data, sc = O.mxfp8_quantize(g_li)
            assert np.array_equal(loop.q_data.cpu().numpy(), data), what
            assert np.array_equal(loop.q_scale.cpu().numpy(), O.swizzle_scales_128x4(sc)), what
        post, comb, pre = O.mhc_coefficients(g_res, **_coeff_np(st.weights.coeffs))
        assert_coeffs_close({"post": loop.post[b].cpu(), "comb": loop.comb[b].cpu(), "pre": loop.pre[b].cpu()},
                            post, comb, pre, what)


def test_decode_loop_graph_replay_equals_eager():
    loop = DecodeLoop(rows=32, layers=61, device="cuda:0")
    loop.run()
    torch.cuda.synchronize()
    eager = loop.streams().clone()
    eager_pre = loop.pre[loop.steps[-2].dst].clone()
    eager_hidden = loop.hidden_out.clone()
    eager_aux = {k: v.clone() for k, v in loop.aux.items()}
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        loop.run()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        loop.run()
    g.replay()
    torch.cuda.synchronize()
    assert M.mhc_get_device_status(loop.workspace) == M.OK
    assert torch.equal(loop.streams(), eager)
    assert torch.equal(loop.pre[loop.steps[-2].dst], eager_pre)
    assert torch.equal(loop.hidden_out, eager_hidden)
    for k, v in eager_aux.items():
        assert torch.equal(loop.aux[k], v), k
