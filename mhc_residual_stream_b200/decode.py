"""The boundaries of one decode step's layer loop, on the CUDA library.

Mirrors the layer loop of vllm ...specialized_decode.runtime.decode,
SpecializedDecode.run, with the sublayers (attention, MoE) replaced by seeded
synthetic outputs: per layer the attention entry (the first layer's broadcast,
else the finalize of the previous MoE output with an MXFP8 layer input), the
attention's TP-partial output, the FFN entry (the partial sum, bf16 layer
input) and the MoE's unfinalized output; after the last layer the finalize
that, fused with the step's head (SpecializedDecode._head: the final norm of the
streams collapsed with the carried pre), gives the step's hidden state. Layers
in `aux_layers` keep the mean of their new streams (capture_aux), the end layer
after the last finalize. The streams and the post / comb / pre mixes chain from
boundary to boundary as in BoundaryState.

Every boundary has its own seeded fn, scale, base and norm_weight, so the
weights a step reads exceed the L2 cache and come from HBM.
"""

from __future__ import annotations

from contextlib import nullcontext as _nullcontext
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import torch

from . import mhc as M
from . import synthetic as S


@dataclass
class BoundaryWeights:
    coeffs: M.Coeffs
    norm_weight: torch.Tensor


@dataclass
class Pending:
    kind: str  # "partials", "moe" or "engram" (the injection's stand-in: a delta added to the streams)
    partials: Optional[torch.Tensor] = None
    gemm2_permuted: Optional[torch.Tensor] = None
    expert_weights: Optional[torch.Tensor] = None
    e2p: Optional[torch.Tensor] = None
    shared_output: Optional[torch.Tensor] = None
    delta: Optional[torch.Tensor] = None


@dataclass
class Step:
    """One boundary of the schedule."""
    kind: str            # "first", "attn", "ffn", "post_only", "engram", "final"
    layer: int
    weights: Optional[BoundaryWeights]
    pending: Optional[Pending]
    mxfp8: bool
    src: int = 0         # state slot read
    dst: int = 0         # state slot written


@dataclass
class DecodeLoop:
    rows: int
    hidden: int = 7168
    hc_mult: int = 4
    layers: int = 61
    partials: int = 8
    top_k: int = 8
    seed: int = 5000
    device: str = "cuda"
    pack_fn: bool = True  # fn packed once at weight load (mhc_projection_pack)
    # layers whose hidden state (the stream mean) is kept; `layers` itself is the
    # end layer, captured after the last finalize. None: layers 2, L/2, L-3 and L.
    aux_layers: Optional[Tuple[int, ...]] = None
    # layers whose attention entry goes through an Engram injection ([decode]
    # SpecializedDecode.run: post_only, the injection, then Boundaries.pre on
    # the injected streams); the injection is a seeded delta (it needs weights)
    engram_layers: Tuple[int, ...] = ()
    steps: List[Step] = field(default_factory=list)

    def __post_init__(self):
        R, H, n, dev = self.rows, self.hidden, self.hc_mult, self.device
        s0 = self.seed
        first = S.draw_first_layer(R, H, n=n, seed=s0)
        self.x = first["x"].to(dev)
        # state slots: streams and mixes, ping-pong between boundaries
        self.res = [torch.empty(R, n, H, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.post = [torch.empty(R, n, dtype=torch.float32, device=dev) for _ in range(2)]
        self.comb = [torch.empty(R, n, n, dtype=torch.float32, device=dev) for _ in range(2)]
        self.pre = [torch.empty(R, n, dtype=torch.float32, device=dev) for _ in range(2)]
        self.layer_input = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
        self.q_data = torch.empty(R, H, dtype=torch.uint8, device=dev)
        self.q_scale = torch.empty(M.mhc_mxfp8_scale_bytes(R, H, True), dtype=torch.uint8, device=dev)
        self.workspace = M.new_workspace(R, H, n, dev)
        if self.aux_layers is None:
            self.aux_layers = tuple(sorted({l for l in (2, self.layers // 2, self.layers - 3, self.layers)
                                            if 1 <= l <= self.layers}))
        self.aux: Dict[int, torch.Tensor] = {l: torch.empty(R, H, dtype=torch.bfloat16, device=dev)
                                             for l in self.aux_layers}
        self.hidden_out = torch.empty(R, H, dtype=torch.bfloat16, device=dev)  # the step's output
        g = S.gen(s0 + 7)
        self.final_norm = (1.0 + torch.randn(H, generator=g) * 0.1).to(torch.bfloat16).to(dev)

        def weights(seed):
            g = S.gen(seed)
            cw = S.draw_coeff_weights(g, H, n, 0.01, affine=True)
            nw = (1.0 + torch.randn(H, generator=g) * 0.1).to(torch.bfloat16)
            return BoundaryWeights(M.Coeffs.from_weights(cw, dev, packed=self.pack_fn), nw.to(dev))

        def attn_pending(seed):
            g = S.gen(seed)
            p = (torch.randn(self.partials, R, H, generator=g) * 0.05).to(torch.bfloat16)
            return Pending("partials", partials=p.to(dev))

        def moe_pending(seed):
            d = S.draw_moe(R, H, n=n, top_k=self.top_k, seed=seed)
            return Pending("moe", gemm2_permuted=d["gemm2_permuted"].to(dev),
                           expert_weights=d["expert_weights"].to(dev),
                           e2p=d["expanded_idx_to_permuted_idx"].to(dev),
                           shared_output=d["shared_output"].to(dev))

        def engram_delta(seed):
            g = S.gen(seed)
            return Pending("engram", delta=(torch.randn(R, n, H, generator=g) * 0.05).to(torch.bfloat16).to(dev))

        steps = []
        slot = 0
        prev_moe = None
        for layer in range(self.layers):
            base = s0 + 10 * (layer + 1)
            if layer == 0:
                steps.append(Step("first", 0, weights(base + 1), None, False, src=0, dst=0))
            elif layer in self.engram_layers:
                # streams only, then the coefficients and layer input of the injected streams
                steps.append(Step("post_only", layer, None, prev_moe, False, src=slot, dst=1 - slot))
                steps.append(Step("engram", layer, weights(base + 1), engram_delta(base + 5), False,
                                  src=slot, dst=1 - slot))
                slot = 1 - slot
            else:
                steps.append(Step("attn", layer, weights(base + 1), prev_moe, True, src=slot, dst=1 - slot))
                slot = 1 - slot
            attn_out = attn_pending(base + 2)
            steps.append(Step("ffn", layer, weights(base + 3), attn_out, False, src=slot, dst=1 - slot))
            slot = 1 - slot
            prev_moe = moe_pending(base + 4)
        steps.append(Step("final", self.layers, None, prev_moe, False, src=slot, dst=1 - slot))
        self.steps = steps
        self.final_slot = 1 - slot

    # ------------------------------------------------------------------ running

    def run_step(self, st: Step, stream=None):
        ws = self.workspace
        if st.kind == "first":
            M.mhc_coeffs(st.weights.coeffs, self.post[st.dst], self.comb[st.dst], self.pre[st.dst], x=self.x,
                         residual_out=self.res[st.dst], norm_weight=st.weights.norm_weight, norm_eps=1e-6,
                         layer_input=self.layer_input, workspace=ws, stream=stream)
            return
        a, b = st.src, st.dst
        aux = self.aux_of(st)
        q = (self.q_data, self.q_scale, True) if st.mxfp8 else None
        if st.kind == "post_only":  # the finalize into the streams, no layer input
            pd = st.pending
            M.mhc_boundary_moe_finalize(
                pd.gemm2_permuted, pd.expert_weights, pd.e2p, pd.shared_output, self.res[a], self.post[a],
                self.comb[a], None, None, 0.0, None, self.res[b], workspace=ws, stream=stream, aux=aux)
            return
        if st.kind == "engram":  # injected = streams + delta (stand-in), then mhc pre with the carried pre
            with torch.cuda.stream(stream) if stream is not None else _nullcontext():
                self.res[b].add_(st.pending.delta)
            M.mhc_coeffs(st.weights.coeffs, self.post[b], self.comb[b], self.pre[b], residual=self.res[b],
                         pre_mix=self.pre[a], norm_weight=st.weights.norm_weight, norm_eps=1e-6,
                         layer_input=self.layer_input, workspace=ws, stream=stream)
            return
        if st.kind == "final":  # the last finalize fused with the head: no coefficients
            pd = st.pending
            M.mhc_boundary_moe_finalize(
                pd.gemm2_permuted, pd.expert_weights, pd.e2p, pd.shared_output, self.res[a], self.post[a],
                self.comb[a], self.pre[a], self.final_norm, 1e-6, None, self.res[b], layer_input=self.hidden_out,
                workspace=ws, stream=stream, aux=aux)
            return
        w = st.weights
        if st.pending.kind == "partials":
            M.mhc_boundary_post_pre(st.pending.partials, self.res[a], self.post[a], self.comb[a], self.pre[a],
                                    w.norm_weight, 1e-6, w.coeffs, self.res[b], layer_input=self.layer_input,
                                    mxfp8=q, post_out=self.post[b], comb_out=self.comb[b], pre_out=self.pre[b],
                                    workspace=ws, stream=stream, aux=aux)
        else:
            pd = st.pending
            M.mhc_boundary_moe_finalize(
                pd.gemm2_permuted, pd.expert_weights, pd.e2p, pd.shared_output, self.res[a], self.post[a],
                self.comb[a], self.pre[a], w.norm_weight, 1e-6, w.coeffs, self.res[b],
                layer_input=self.layer_input, mxfp8=q, post_out=self.post[b], comb_out=self.comb[b],
                pre_out=self.pre[b], workspace=ws, stream=stream, aux=aux)

    def aux_of(self, st: Step) -> Optional[torch.Tensor]:
        """The aux buffer a boundary writes: the attention entry of a captured layer
        (its new streams, [boundary] Boundaries.sublayer with capture_aux; for an
        Engram layer the streams before the injection) or the final finalize for
        the end layer."""
        if st.kind in ("attn", "post_only", "final") and st.layer in self.aux:
            return self.aux[st.layer]
        return None

    def run(self, stream=None):
        """Enqueue every boundary of the step on `stream` (no host synchronisation)."""
        for st in self.steps:
            self.run_step(st, stream)

    def streams(self) -> torch.Tensor:
        """The residual streams after the final boundary."""
        return self.res[self.final_slot]

    def algorithmic_bytes(self) -> int:
        """Bytes each boundary must move (inputs read once, outputs written once), summed."""
        R, H, n = self.rows, self.hidden, self.hc_mult
        C = 2 * n + n * n
        total = 0
        for st in self.steps:
            b = 0
            fn_b = n * H * C * 4 + (3 + C) * 4
            mix_in = R * (2 * n + n * n) * 4
            coeff_out = R * (2 * n + n * n) * 4
            if st.kind == "first":
                b = R * H * 2 + R * n * H * 2 + R * H * 2 + fn_b + H * 2 + coeff_out
            elif st.kind == "engram":  # the injection's add is the stand-in's, not counted
                b = R * n * H * 2 + R * n * 4 + fn_b + H * 2 + R * H * 2 + coeff_out
            elif st.kind == "post_only":
                b = (R * self.top_k + R) * H * 2 + R * self.top_k * 8 + 2 * R * n * H * 2 + R * (n + n * n) * 4
                if self.aux_of(st) is not None:
                    b += R * H * 2
            else:
                if st.pending.kind == "partials":
                    b += self.partials * R * H * 2
                else:
                    b += (R * self.top_k + R) * H * 2 + R * self.top_k * 8
                b += 2 * R * n * H * 2 + mix_in
                b += R * H * 2 + H * 2  # layer input (the hidden state at the end) and its norm weight
                if st.kind != "final":
                    b += fn_b + coeff_out
                    if st.mxfp8:
                        b += R * H + M.mhc_mxfp8_scale_bytes(R, H, True)
                if self.aux_of(st) is not None:
                    b += R * H * 2
            total += b
        return total
