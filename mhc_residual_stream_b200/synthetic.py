"""Seeded synthetic inputs for the mHC boundary, shared by tests and benchmarks.

This module draws random tensors only. It holds none of the boundary's
arithmetic: no post-mix, collapse, normalisation, projection, sigmoid of
logits, Sinkhorn or quantisation. Both the CUDA path and the CPU oracle are
fed the exact bytes made here (bf16 tensors are drawn in float32, then cast).

Distributions follow the decode workloads the boundary is measured on:
  * partials ~ N(0, 0.05) bf16, residual streams ~ N(0, 1) bf16;
  * post = logistic(N(0, 1)) via torch.sigmoid, pre = logistic(N(0, 1)) + 1e-6;
  * comb: a random doubly stochastic n x n matrix per row, drawn as a convex
    combination of random permutation matrices with Dirichlet(1) weights
    (Birkhoff). It stands in for the Sinkhorn output of normal logits, which
    this module cannot compute without holding the method's arithmetic;
  * fn ~ N(0, sigma) fp32 [n*H, 2n+n^2]; scale and base either 1 and 0 or
    drawn (scale ~ U(0.5, 1.5), base ~ N(0, 0.1));
  * norm_weight = 1 + N(0, 0.1) bf16;
  * MoE: gemm2_permuted ~ N(0, 0.05) bf16, expert_weights = softmax(N(0, 1))
    per row, expanded_idx_to_permuted_idx a random permutation of 0..R*k-1,
    shared_output ~ N(0, 0.05) bf16.
Seeds are 1000 * config + rows unless given.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

__all__ = ["CoeffWeights", "draw_coeff_weights", "draw_boundary", "draw_moe",
           "draw_first_layer", "draw_comb", "gen"]


def gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal(g, shape, std, dtype=torch.bfloat16):
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(dtype)


def draw_comb(g, rows: int, n: int, terms: int = 6) -> torch.Tensor:
    """[rows, n, n] fp32 doubly stochastic: a Dirichlet(1) mix of ``terms``
    random permutation matrices per row."""
    comb = torch.zeros(rows, n, n, dtype=torch.float64)
    for r in range(rows):
        w = -torch.log(torch.rand(terms, generator=g, dtype=torch.float64).clamp_min(1e-300))
        w = w / w.sum()
        for m in range(terms):
            perm = torch.randperm(n, generator=g)
            comb[r, torch.arange(n), perm] += w[m]
    return comb.to(torch.float32)


@dataclass
class CoeffWeights:
    fn: torch.Tensor      # [n*H, 2n+n^2] fp32
    scale: torch.Tensor   # [3] fp32
    base: torch.Tensor    # [2n+n^2] fp32
    rms_eps: float = 1e-6
    pre_eps: float = 1e-6
    sinkhorn_eps: float = 1e-6
    post_alpha: float = 2.0
    sinkhorn_iters: int = 20

    def as_dict(self):
        return dict(fn=self.fn, scale=self.scale, base=self.base, rms_eps=self.rms_eps,
                    pre_eps=self.pre_eps, sinkhorn_eps=self.sinkhorn_eps,
                    post_alpha=self.post_alpha, sinkhorn_iters=self.sinkhorn_iters)


def draw_coeff_weights(g, hidden: int, n: int, fn_std: float, affine: bool = True,
                       iters: int = 20) -> CoeffWeights:
    C = 2 * n + n * n
    fn = torch.randn(n * hidden, C, generator=g, dtype=torch.float32) * fn_std
    if affine:
        scale = 0.5 + torch.rand(3, generator=g, dtype=torch.float32)
        base = torch.randn(C, generator=g, dtype=torch.float32) * 0.1
    else:
        scale = torch.ones(3, dtype=torch.float32)
        base = torch.zeros(C, dtype=torch.float32)
    return CoeffWeights(fn=fn, scale=scale, base=base, sinkhorn_iters=iters)


def _mixes(g, rows, n):
    post = torch.sigmoid(torch.randn(rows, n, generator=g, dtype=torch.float32))
    comb = draw_comb(g, rows, n)
    pre = torch.sigmoid(torch.randn(rows, n, generator=g, dtype=torch.float32)) + 1e-6
    return post, comb, pre


def draw_boundary(rows: int, hidden: int, n: int = 4, partials: int = 8, seed: int = 0,
                  fn_std: float = 0.01, affine: bool = True, part_std: float = 0.05):
    """Inputs of a partial-sum boundary: dict of CPU tensors."""
    g = gen(seed)
    d = {}
    d["partials"] = _normal(g, (partials, rows, hidden), part_std)
    d["residual"] = _normal(g, (rows, n, hidden), 1.0)
    d["post"], d["comb"], d["pre"] = _mixes(g, rows, n)
    d["norm_weight"] = (1.0 + torch.randn(hidden, generator=g) * 0.1).to(torch.bfloat16)
    d["norm_eps"] = 1e-6
    d["coeff"] = draw_coeff_weights(g, hidden, n, fn_std, affine)
    return d


def draw_moe(rows: int, hidden: int, n: int = 4, top_k: int = 8, seed: int = 0,
             fn_std: float = 0.01, affine: bool = True, extra_permuted: int = 0):
    """Inputs of a MoE-finalize boundary: dict of CPU tensors."""
    g = gen(seed)
    d = {}
    num_perm = rows * top_k + extra_permuted
    d["gemm2_permuted"] = _normal(g, (num_perm, hidden), 0.05)
    d["expert_weights"] = torch.softmax(
        torch.randn(rows, top_k, generator=g, dtype=torch.float32), dim=1)
    d["expanded_idx_to_permuted_idx"] = torch.randperm(num_perm, generator=g)[: rows * top_k].to(torch.int32)
    d["shared_output"] = _normal(g, (rows, hidden), 0.05)
    d["residual"] = _normal(g, (rows, n, hidden), 1.0)
    d["post"], d["comb"], d["pre"] = _mixes(g, rows, n)
    d["norm_weight"] = (1.0 + torch.randn(hidden, generator=g) * 0.1).to(torch.bfloat16)
    d["norm_eps"] = 1e-6
    d["coeff"] = draw_coeff_weights(g, hidden, n, fn_std, affine)
    return d


def draw_first_layer(rows: int, hidden: int, n: int = 4, seed: int = 0, fn_std: float = 0.01,
                     affine: bool = True):
    """Inputs of the first layer's attention entry: the embedding x [rows, hidden]."""
    g = gen(seed)
    d = {}
    d["x"] = _normal(g, (rows, hidden), 1.0)
    d["norm_weight"] = (1.0 + torch.randn(hidden, generator=g) * 0.1).to(torch.bfloat16)
    d["norm_eps"] = 1e-6
    d["coeff"] = draw_coeff_weights(g, hidden, n, fn_std, affine)
    return d
