"""Seeded synthetic inputs for the expert-layer numerics path.

This module holds input generation only: no quantisation, rounding, GEMM or
routing-permutation arithmetic of the method.  Both the CUDA path and the CPU
oracle receive the bytes it produces.  All draws use explicit torch
Generators, so a (seed, device) pair always gives the same bytes.

Workloads (sizes from the configurations the library is measured on; the
shapes echo the model on the Hermes page "Thinking Machines' Inkling 2 Small
Trains a 594B Model in 68 Hours", section "594B weights, 17B at work": each
token uses 8 of 384 experts):

  tiny_layer     4 experts, top-2 of 256 tokens (uniform distinct choice),
                 d_model 256, d_ff 512, SiLU (no gate); x ~ N(0,1) with 0.1%
                 of entries x50; weights N(0, 0.02); upstream grad N(0,1)
  quant_stream   bf16 [16384, 4096], Student-t (nu=4) times a per-row scale
                 10^U(-3,3)
  fwd_gemm       64 experts, top-8 of 16384 tokens (131072 routed rows),
                 Zipf(1.1) loads, d_model 4096, d_ff 1536 (W1 4096->3072 gate+up,
                 W2 1536->4096); x ~ N(0,1); weights N(0,0.02)
  bwd_gemm       fwd_gemm shapes; upstream grads dY2 [M,4096], dH1 [M,3072]
                 ~ N(0, 1e-3), drawn independently
  moe_layer      384 experts, top-8 of 32768 tokens (262144 routed rows),
                 Zipf(1.2) loads with 8 experts forced empty, d_model 4096,
                 d_ff 1024, SwiGLU; x ~ t(nu=3); weights N(0,0.02); upstream
                 grad N(0,1)

Routing: Gumbel-top-k without replacement over log-weights, weights
proportional to rank^-s for a seeded permutation of the experts (forced-empty
experts get weight 0).  Student-t draws use z / sqrt(chi2_nu / nu) with chi2_nu
a sum of nu squared normals.
"""
from __future__ import annotations

import math

import torch

CONFIGS = {
    "tiny_layer": dict(T=256, k=2, E=4, D=256, F=512, gated=False, routing="uniform", zipf=0.0, n_empty=0,
                       x_dist="normal_outliers", w_std=0.02, grad_std=1.0, seed=1000),
    "quant_stream": dict(rows=16384, cols=4096, x_dist="t4_rowscale", seed=1001, sr_seed=0),
    "fwd_gemm": dict(T=16384, k=8, E=64, D=4096, F=1536, gated=True, routing="zipf", zipf=1.1, n_empty=0,
                     x_dist="normal", w_std=0.02, seed=1002),
    "bwd_gemm": dict(T=16384, k=8, E=64, D=4096, F=1536, gated=True, routing="zipf", zipf=1.1, n_empty=0,
                     x_dist="normal", w_std=0.02, grad_std=1e-3, seed=1003),
    "moe_layer": dict(T=32768, k=8, E=384, D=4096, F=1024, gated=True, routing="zipf", zipf=1.2, n_empty=8,
                      x_dist="t3", w_std=0.02, grad_std=1.0, seed=1004),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def routing(T: int, k: int, E: int, kind: str, zipf: float, n_empty: int, seed: int) -> torch.Tensor:
    """Top-k expert ids [T, k] int32 (distinct per token), generated on the CPU."""
    g = _gen(seed, "cpu")
    if kind == "uniform":
        logw = torch.zeros(E, dtype=torch.float64)
    else:
        perm = torch.randperm(E, generator=g)
        ranks = torch.empty(E, dtype=torch.float64)
        ranks[perm] = torch.arange(1, E + 1, dtype=torch.float64)
        logw = -zipf * torch.log(ranks)
        if n_empty:
            empty = torch.randperm(E, generator=g)[:n_empty]
            logw[empty] = -math.inf
    u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_(1e-300, 1.0)
    gumbel = -torch.log(-torch.log(u))
    scores = logw[None, :] + gumbel
    ids = torch.topk(scores, k, dim=1).indices
    return ids.to(torch.int32).contiguous()


def _student_t(shape, nu: int, g: torch.Generator, device) -> torch.Tensor:
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        chi2 += torch.randn(shape, generator=g, device=device, dtype=torch.float32) ** 2
    return z / torch.sqrt(chi2 / nu)


def activations(rows: int, cols: int, dist: str, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [rows, cols]."""
    g = _gen(seed, device)
    if dist == "normal":
        x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
    elif dist == "normal_outliers":
        x = torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32)
        n_out = int(round(0.001 * rows * cols))
        idx = torch.randperm(rows * cols, generator=g, device=device)[:n_out]
        x.view(-1)[idx] *= 50.0
    elif dist == "t3":
        x = torch.empty(rows, cols, device=device, dtype=torch.float32)
        step = max(1, (1 << 26) // cols)
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            x[r0:r1] = _student_t((r1 - r0, cols), 3, g, device)
    elif dist == "t4_rowscale":
        x = torch.empty(rows, cols, device=device, dtype=torch.float32)
        step = max(1, (1 << 26) // cols)
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            x[r0:r1] = _student_t((r1 - r0, cols), 4, g, device)
        scale = torch.pow(10.0, torch.rand(rows, 1, generator=g, device=device, dtype=torch.float32) * 6.0 - 3.0)
        x *= scale
    else:
        raise ValueError(dist)
    return x.to(torch.bfloat16)


def weights(E: int, N: int, K: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    """bf16 expert weight stack [E, N, K] ~ N(0, std), one expert at a time."""
    g = _gen(seed, device)
    w = torch.empty(E, N, K, device=device, dtype=torch.bfloat16)
    for e in range(E):
        w[e] = (torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)
    return w


def gradient(rows: int, cols: int, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randn(rows, cols, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def layer_inputs(name: str, device="cpu", with_weights: bool = True) -> dict:
    """All inputs of one expert-layer workload: x [T, D], topk ids [T, k] (CPU),
    combine weights [T, k] (1/k), W1 [E, 2F or F, D], W2 [E, D, F], dout [T, D]."""
    c = CONFIGS[name]
    T, k, E, D, F = c["T"], c["k"], c["E"], c["D"], c["F"]
    s = c["seed"]
    out = dict(cfg=c, name=name)
    out["topk"] = routing(T, k, E, c["routing"], c["zipf"], c["n_empty"], s)
    out["w_comb"] = torch.full((T, k), 1.0 / k, dtype=torch.float32)
    out["x"] = activations(T, D, c["x_dist"], s + 1, device)
    if with_weights:
        n1 = 2 * F if c["gated"] else F
        out["w1"] = weights(E, n1, D, c["w_std"], s + 2, device)
        out["w2"] = weights(E, D, F, c["w_std"], s + 3, device)
    if "grad_std" in c:
        out["dout"] = gradient(T, D, c["grad_std"], s + 4, device)
    return out


def max_routed_rows(T: int, k: int, E: int, align: int = 128) -> int:
    """Capacity for the expert-major row buffer: every expert padded to a
    multiple of `align` adds at most align-1 rows."""
    cap = T * k + E * (align - 1)
    return (cap + align - 1) // align * align
