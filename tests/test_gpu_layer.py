"""Layer-level parity, stage by stage: the tiny 4-expert layer (top-2 of 256
tokens, d_model 256, d_ff 512, SiLU) forward and backward through ExpertLayer
on the GPU, each stage checked against the oracle applied to the bytes the GPU
produced for that stage's inputs (so no stage inherits an earlier stage's
rounding differences):
  - routing, quantisers, gather, requantisations, combine gradient and its
    MXFP8 forms: bit-exact;
  - each GEMM: re-run in fp32 output on the layer's operands, relative
    Frobenius error <= 1e-4 against the oracle's fp64 product, and the layer's
    bf16 output equal to the round-to-nearest-even bf16 of that fp32 output
    (fp32 weight gradients are compared directly);
  - SiLU / SwiGLU and their backward, combine and un-permute: within one bf16
    rounding (plus the fp32 accumulation error of a k-term sum) of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from fp8_moe_numerics_b200.layer import ExpertLayer
from tests.layouts import mma_to_rowmajor

pytestmark = pytest.mark.gpu

TOL_FRO = 1e-4


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


def bf16_rne(x32: np.ndarray) -> np.ndarray:
    return oracle.f32_to_bf16(np.asarray(x32, dtype=np.float32))


def within_one_bf16(got_u16, ref_u16, slack=None):
    g, r = f64(got_u16), f64(ref_u16)
    tol = 2.0 ** -7 * np.abs(r)
    if slack is not None:
        tol = tol + slack
    return bool(np.all(np.abs(g - r) <= tol))


def test_tiny_layer_forward_backward_stagewise(cuda):
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    E, T, k, D, F = c["E"], c["T"], c["k"], c["D"], c["F"]
    seed, R = 99, 16
    L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(), inp["w2"].cuda(),
                    inp["dout"].cuda(), gated=False, seed=seed, wgrad_dtype=torch.float32, rbits=R)
    L.step()
    api.sync_status()
    M, seg = L.M_cap, L.seg
    g = lambda t: t.detach().cpu().numpy()
    w = inp["w_comb"].numpy()

    # ---------------- routing, token and weight quantisation, dispatch: bit-exact
    seg_o, src_o, pos_o = oracle.route(inp["topk"].numpy(), E)
    Mp = int(seg_o[-1])
    assert np.array_equal(g(seg), seg_o) and np.array_equal(g(L.pos), pos_o)
    s_gpu = g(L.src)
    assert np.array_equal(np.where(s_gpu[:Mp] >= 0, s_gpu[:Mp] // k, -1), src_o) and np.all(s_gpu[Mp:] == -1)
    xq = oracle.nvfp4_quantize(u16(inp["x"]))
    assert np.array_equal(g(L.xq[0]), xq[0]) and np.array_equal(g(L.xq[1]).reshape(T, D // 16), xq[1])
    xp = oracle.gather_nvfp4_rows(*xq, src_o)
    xp_g = (g(L.xp[0]), mma_to_rowmajor(g(L.xp[1]), M, D // 16), g(L.xp[2]))
    assert np.array_equal(xp_g[0][:Mp], xp[0]) and np.array_equal(xp_g[1][:Mp], xp[1])
    assert np.array_equal(xp_g[2][:Mp].view(np.uint32), xp[2].view(np.uint32))
    w1q = oracle.nvfp4_quantize(u16(inp["w1"]).reshape(E * F, D), group_rows=F)
    w2q = oracle.nvfp4_quantize(u16(inp["w2"]).reshape(E * D, F), group_rows=D)
    for got, ref, rows, cols in ((L.w1q, w1q, E * F, D), (L.w2q, w2q, E * D, F)):
        assert np.array_equal(g(got[0]), ref[0]) and np.array_equal(mma_to_rowmajor(g(got[1]), rows, cols // 16), ref[1])
        assert np.array_equal(g(got[2]).view(np.uint32), ref[2].view(np.uint32))

    def gemm_stage(layer_out, run32, ref64, rows=None):
        o32 = g(run32())
        api.sync_status()
        sl = slice(0, rows) if rows is not None else slice(None)
        assert rel(o32[sl].astype(np.float64), ref64[sl]) <= TOL_FRO
        if layer_out.dtype == torch.bfloat16:
            assert np.array_equal(u16(layer_out)[sl], bf16_rne(o32[sl]))
        else:
            assert np.array_equal(g(layer_out)[sl], o32[sl])

    # ---------------- GEMM1
    gemm_stage(L.h1, lambda: api.grouped_gemm_nvfp4(L.xp, L.w1q, seg, E, F, D, out_dtype=torch.float32),
               oracle.grouped_gemm_nvfp4(*xp_g, *w1q, seg_o, F), Mp)
    h1 = u16(L.h1)[:Mp]
    # ---------------- SiLU + NVFP4 (fused kernel) on the GPU's h1
    a_g = api.swiglu_fwd(L.h1, F, False, L.rows_valid)
    api.sync_status()
    assert within_one_bf16(u16(a_g)[:Mp], oracle.swiglu_fwd(h1, gated=False))
    aq = oracle.nvfp4_quantize(u16(a_g)[:Mp])
    aq_g = (g(L.aq[0]), mma_to_rowmajor(g(L.aq[1]), M, F // 16), g(L.aq[2]))
    assert np.array_equal(aq_g[0][:Mp], aq[0]) and np.array_equal(aq_g[1][:Mp], aq[1])
    assert np.array_equal(aq_g[2][:Mp].view(np.uint32), aq[2].view(np.uint32))
    # ---------------- GEMM2, combine
    gemm_stage(L.y2, lambda: api.grouped_gemm_nvfp4(L.aq, L.w2q, seg, E, D, F, out_dtype=torch.float32),
               oracle.grouped_gemm_nvfp4(*aq_g, *w2q, seg_o, D), Mp)
    y2 = u16(L.y2)[:Mp]
    acc = oracle.combine(oracle.f32_to_bf16(np.abs(f64(y2)).astype(np.float32)), pos_o, w)
    assert within_one_bf16(u16(L.out), oracle.combine(y2, pos_o, w), slack=2.0 ** -20 * f64(acc))

    # ---------------- backward: combine gradient and its MXFP8 forms (one fused kernel), bit-exact
    dy2 = oracle.dispatch_grad(u16(inp["dout"]), pos_o, w, Mp)
    dy2_g = np.zeros((M, D), np.uint16)
    dy2_g[:Mp] = dy2
    r_o, c_o = oracle.mxfp8_quantize_rows(dy2_g[:Mp]), oracle.mxfp8_quantize_cols(dy2_g)
    dy2r = (g(L.dy2q[0]), mma_to_rowmajor(g(L.dy2q[1]), M, D // 32))
    dy2c = (g(L.dy2q[2]), mma_to_rowmajor(g(L.dy2q[3]), D, M // 32))
    assert np.array_equal(dy2r[0][:Mp], r_o[0]) and np.array_equal(dy2r[1][:Mp], r_o[1])
    assert np.array_equal(dy2c[0][:, :Mp], c_o[0][:, :Mp]) and np.array_equal(dy2c[1][:, :Mp // 32], c_o[1][:, :Mp // 32])
    # requantisations of the saved operands (R = 16), bit-exact on the GPU's own NVFP4 bytes
    w2t = oracle.mxfp8_requant_transpose_sr(*w2q, D, seed, 1, R)
    at = oracle.mxfp8_requant_transpose_sr(*(pad(a[:Mp], M) for a in aq_g), 1, seed, 2, R)
    w1t = oracle.mxfp8_requant_transpose_sr(*w1q, F, seed, 3, R)
    xt = oracle.mxfp8_requant_transpose_sr(*(pad(a[:Mp], M) for a in xp_g), 1, seed, 4, R)
    for got, ref, rows, cols, n in ((L.w2t, w2t, F, E * D, E * D), (L.at, at, F, M, Mp), (L.w1t, w1t, D, E * F, E * F),
                                    (L.xt, xt, D, M, Mp)):
        assert np.array_equal(g(got[0])[:, :n], ref[0][:, :n])
        assert np.array_equal(mma_to_rowmajor(g(got[1]), rows, cols // 32)[:, :n // 32], ref[1][:, :n // 32])
    # ---------------- dgrad2, wgrad2
    gemm_stage(L.da, lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, L.dy2q[0], L.dy2q[1], *L.w2t, seg, E, M, F, D,
                                                    out_dtype=torch.float32),
               oracle.grouped_gemm_mxfp8_dgrad(*dy2r, *w2t, seg_o), Mp)
    gemm_stage(L.dw2, lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, L.dy2q[2], L.dy2q[3], *L.at, seg, E, M, D, F,
                                                     out_dtype=torch.float32),
               oracle.grouped_gemm_mxfp8_wgrad(*dy2c, *at, seg_o))
    # ---------------- SiLU backward on the GPU's h1 and da, its MXFP8 forms
    da = u16(L.da)[:Mp]
    assert within_one_bf16(u16(L.dh1)[:Mp], oracle.swiglu_bwd(h1, da, gated=False))
    dh1_g = u16(L.dh1)
    r_o, c_o = oracle.mxfp8_quantize_rows(dh1_g[:Mp]), oracle.mxfp8_quantize_cols(dh1_g)
    dh1r = (g(L.dh1q[0]), mma_to_rowmajor(g(L.dh1q[1]), M, F // 32))
    dh1c = (g(L.dh1q[2]), mma_to_rowmajor(g(L.dh1q[3]), F, M // 32))
    assert np.array_equal(dh1r[0][:Mp], r_o[0]) and np.array_equal(dh1r[1][:Mp], r_o[1])
    assert np.array_equal(dh1c[0][:, :Mp], c_o[0][:, :Mp])
    # ---------------- dgrad1, wgrad1, un-permute
    gemm_stage(L.dxp, lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, L.dh1q[0], L.dh1q[1], *L.w1t, seg, E, M, D,
                                                     F, out_dtype=torch.float32),
               oracle.grouped_gemm_mxfp8_dgrad(*dh1r, *w1t, seg_o), Mp)
    gemm_stage(L.dw1, lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, L.dh1q[2], L.dh1q[3], *L.xt, seg, E, M, F, D,
                                                     out_dtype=torch.float32),
               oracle.grouped_gemm_mxfp8_wgrad(*dh1c, *xt, seg_o))
    dxp = u16(L.dxp)[:Mp]
    ones = np.ones_like(w)
    acc = oracle.combine(oracle.f32_to_bf16(np.abs(f64(dxp)).astype(np.float32)), pos_o, ones)
    assert within_one_bf16(u16(L.dx), oracle.combine(dxp, pos_o, ones), slack=2.0 ** -20 * f64(acc))


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
