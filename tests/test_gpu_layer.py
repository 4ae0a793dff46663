"""Layer-level parity: the tiny 4-expert layer (top-2 of 256 tokens, d_model
256, d_ff 512, SiLU) forward and backward through ExpertLayer on the GPU,
against the oracle running its own full chain from the same seeded inputs.

Stages whose inputs agree bit for bit (routing, NVFP4 dispatch, weight
quantisation, weight requantisation, the saved-token requantisation, combine
gradient and its MXFP8 quantisation) must agree bit for bit.  GEMM outputs are
bf16: the GPU rounds an fp32 sum, the oracle an fp64 sum, so an element may
differ by one bf16 rounding, and downstream stages inherit rare code flips
(a changed row maximum moves a whole row's scales).  For those stages the bar
is: >= 99% identical codes and a relative Frobenius error below 2e-2 -- far
below what a wrong expert, transpose or scale layout gives (O(1)).
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from fp8_moe_numerics_b200.layer import ExpertLayer
from tests.layouts import mma_to_rowmajor

pytestmark = pytest.mark.gpu


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(u):
    return oracle.bf16_to_f32(u).astype(np.float64)


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def pad(a, rows):
    out = np.zeros((rows,) + a.shape[1:], a.dtype)
    out[:a.shape[0]] = a
    return out


def test_tiny_layer_forward_backward_against_oracle(cuda):
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    E, T, k, D, F = c["E"], c["T"], c["k"], c["D"], c["F"]
    seed = 99
    L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(), inp["w2"].cuda(),
                    inp["dout"].cuda(), gated=False, seed=seed, wgrad_dtype=torch.float32)
    L.step()
    api.sync_status()
    M = L.M_cap

    # ---------------- oracle chain (its own bytes end to end)
    x, w1, w2, dout = u16(inp["x"]), u16(inp["w1"]).reshape(E * F, D), u16(inp["w2"]).reshape(E * D, F), u16(inp["dout"])
    w = inp["w_comb"].numpy()
    seg, src, pos = oracle.route(inp["topk"].numpy(), E)
    Mp = int(seg[-1])
    xq = oracle.nvfp4_quantize(x)
    xp = oracle.gather_nvfp4_rows(*xq, src)
    w1q = oracle.nvfp4_quantize(w1, group_rows=F)
    w2q = oracle.nvfp4_quantize(w2, group_rows=D)
    h1 = oracle.f64_to_bf16(oracle.grouped_gemm_nvfp4(*xp, *w1q, seg, F))
    a = oracle.swiglu_fwd(h1, gated=False)
    aq = oracle.nvfp4_quantize(a)
    y2 = oracle.f64_to_bf16(oracle.grouped_gemm_nvfp4(*aq, *w2q, seg, D))
    out = oracle.combine(y2, pos, w)
    dy2 = oracle.dispatch_grad(dout, pos, w, Mp)
    dy2_r = oracle.mxfp8_quantize_rows(dy2)
    dy2_c = oracle.mxfp8_quantize_cols(pad(dy2, M))
    w2t = oracle.mxfp8_requant_transpose_sr(*w2q, D, seed, 1, 16)
    da = oracle.f64_to_bf16(oracle.grouped_gemm_mxfp8_dgrad(*dy2_r, *w2t, seg))
    at = oracle.mxfp8_requant_transpose_sr(pad(aq[0], M), pad(aq[1], M), pad(aq[2], M), 1, seed, 2, 16)
    dw2 = oracle.grouped_gemm_mxfp8_wgrad(*dy2_c, *at, seg)
    dh1 = oracle.swiglu_bwd(h1, da, gated=False)
    dh1_r = oracle.mxfp8_quantize_rows(dh1)
    dh1_c = oracle.mxfp8_quantize_cols(pad(dh1, M))
    w1t = oracle.mxfp8_requant_transpose_sr(*w1q, F, seed, 3, 16)
    dxp = oracle.f64_to_bf16(oracle.grouped_gemm_mxfp8_dgrad(*dh1_r, *w1t, seg))
    xt = oracle.mxfp8_requant_transpose_sr(pad(xp[0], M), pad(xp[1], M), pad(xp[2], M), 1, seed, 4, 16)
    dw1 = oracle.grouped_gemm_mxfp8_wgrad(*dh1_c, *xt, seg)
    dx = oracle.combine(dxp, pos, np.ones_like(w))

    g = lambda t: t.detach().cpu().numpy()
    # ---------------- bit-exact stages
    assert np.array_equal(g(L.seg), seg) and np.array_equal(g(L.pos), pos)
    assert np.array_equal(g(L.xp[0])[:Mp], xp[0])
    assert np.array_equal(mma_to_rowmajor(g(L.xp[1]), M, D // 16)[:Mp], xp[1])
    assert np.array_equal(g(L.w1q[0]), w1q[0]) and np.array_equal(g(L.w2q[0]), w2q[0])
    assert np.array_equal(mma_to_rowmajor(g(L.w1q[1]), E * F, D // 16), w1q[1])
    assert np.array_equal(g(L.w1t[0]), w1t[0]) and np.array_equal(g(L.w2t[0]), w2t[0])
    assert np.array_equal(mma_to_rowmajor(g(L.w2t[1]), F, E * D // 32), w2t[1])
    assert np.array_equal(g(L.xt[0])[:, :Mp], xt[0][:, :Mp])
    assert np.array_equal(u16(L.dy2)[:Mp], dy2)
    assert np.array_equal(g(L.dy2q[0])[:Mp], dy2_r[0])
    assert np.array_equal(g(L.dy2q[2])[:, :Mp], dy2_c[0][:, :Mp])

    # ---------------- GEMM1 output: one bf16 rounding apart
    gh1 = f64(u16(L.h1)[:Mp])
    rh1 = f64(h1)
    assert np.all(np.abs(gh1 - rh1) <= 2.0 ** -7 * np.abs(rh1) + 1e-6 * np.abs(rh1).max())

    # ---------------- downstream stages: rare code flips only
    assert np.mean(g(L.aq[0])[:Mp] == aq[0]) >= 0.99
    assert np.mean(g(L.at[0])[:, :Mp] == at[0][:, :Mp]) >= 0.99
    for got, ref in ((f64(u16(L.out)), f64(out)), (f64(u16(L.da)[:Mp]), f64(da)), (g(L.dw2).astype(np.float64), dw2),
                     (f64(u16(L.dxp)[:Mp]), f64(dxp)), (g(L.dw1).astype(np.float64), dw1), (f64(u16(L.dx)), f64(dx))):
        assert rel(got, ref) < 2e-2


def test_host_stream_steps_matches_plain_step(cuda):
    # three steps with inputs from pinned host memory and outputs read back,
    # neighbouring steps' copies overlapping: the same bytes as one plain step
    from fp8_moe_numerics_b200.layer import host_stream_steps
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(), inp["w2"].cuda(),
                    inp["dout"].cuda(), gated=False, seed=5)
    own = {n: t.data_ptr() for n, t in L.io().items()}
    L.step()
    ref_out, ref_dx = L.out.cpu(), L.dx.cpu()
    host_in = {n: inp[n].pin_memory() for n in ("x", "topk", "w_comb", "dout")}
    host_out = {n: torch.zeros_like(getattr(L, n), device="cpu").pin_memory() for n in ("out", "dx")}
    host_stream_steps(L, host_in, host_out, 3)
    torch.cuda.synchronize()
    api.sync_status()
    assert torch.equal(host_out["out"], ref_out) and torch.equal(host_out["dx"], ref_dx)
    assert {n: t.data_ptr() for n, t in L.io().items()} == own
