"""Stage-wise parity on the 64-expert layer and the spec GEMM bar at
full size.

Workloads (fp8_moe_numerics_b200.workloads):
  fwd_gemm   64 experts, top-8 of 16384 tokens (131072 routed rows), Zipf(1.1),
             d_model 4096, W1 4096 -> 3072 (gate + up, SwiGLU), W2 1536 -> 4096
  bwd_gemm   the same shapes; the saved NVFP4 tensors of a forward pass, upstream
             gradients dY2 [M, 4096] and dH1 [M, 3072] ~ N(0, 1e-3) drawn
             independently
  moe_layer  384 experts, top-8 of 32768 tokens, Zipf(1.2) with 8 empty
             experts, d_model 4096, d_ff 1024 SwiGLU, t(3) tokens

Each stage is checked on the bytes the GPU produced for its inputs (the oracle
consumes the previous GPU stage), so every stage has its own bar:
  - routing, gather, quantisers and requantisations: bit-exact;
  - grouped GEMMs in fp32 output: relative Frobenius error <= 1e-4 against the
    oracle's fp64 product, over every row and column of a seeded subset of
    experts (the largest, the smallest, the last non-empty one, one under 128
    rows where the routing has one, and seeded others);
  - a GEMM's bf16 output: the bf16 rounding (to nearest even) of its fp32
    output, bit for bit;
  - SwiGLU: within one bf16 rounding of the oracle (the device uses its fast
    exponential); the fused SwiGLU + NVFP4 quantiser then equals the oracle's
    quantisation of the GPU's own SwiGLU output, bit for bit.
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
R_BITS = 16


def np_(t):
    return t.detach().cpu().numpy()


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def rel_fro(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def sf_block(buf, R: int, S: int, r0: int, r1: int, s0: int = 0, s1=None) -> np.ndarray:
    """Row-major scales [r1-r0, s1-s0] of an [R, S] scale array held in the MMA
    layout on the device (gathered there, so only the block is copied)."""
    s1 = S if s1 is None else s1
    r = np.arange(r0, r1, dtype=np.int64)[:, None]
    s = np.arange(s0, s1, dtype=np.int64)[None, :]
    off = ((r // 128) * (S // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4
    return np_(buf.reshape(-1)[torch.from_numpy(off).to(buf.device)])


def bf16_of_f32(t: torch.Tensor) -> torch.Tensor:
    """fp32 -> bf16 bits by round-to-nearest-even, on the GPU (finite values)."""
    b = t.contiguous().view(torch.int32)
    r = b + 0x7FFF + ((b >> 16) & 1)
    return (r >> 16).to(torch.int16)


def assert_bf16_rounding(got_bf16: torch.Tensor, ref_f32: torch.Tensor, what: str, chunk: int = 1 << 26):
    """got_bf16 equals the round-to-nearest-even bf16 of ref_f32, bit for bit
    (compared in chunks to bound the temporaries)."""
    g = got_bf16.reshape(-1).view(torch.int16)
    r = ref_f32.reshape(-1)
    assert g.numel() == r.numel(), what
    for i in range(0, g.numel(), chunk):
        assert torch.equal(g[i:i + chunk], bf16_of_f32(r[i:i + chunk])), (what, i)


def expert_subset(counts, n_random=2, seed=0):
    counts = np.asarray(counts)
    nz = np.flatnonzero(counts)
    pick = {int(np.argmax(counts)), int(nz[np.argmin(counts[nz])]), int(nz[-1])}
    small = nz[counts[nz] < 128]
    if small.size:
        pick.add(int(small[0]))
    rng = np.random.default_rng(seed)
    rest = sorted(set(nz.tolist()) - pick)
    pick |= set(int(e) for e in rng.choice(rest, size=min(n_random, len(rest)), replace=False))
    return sorted(pick)


def nv4_rows(q, R: int, K: int, r0: int, r1: int):
    """Rows r0..r1-1 of an NVFP4 tensor on the device (MMA-layout scales) ->
    host (codes, row-major scales, per-row outer scales)."""
    return np_(q[0][r0:r1]), sf_block(q[1], R, K // 16, r0, r1), np_(q[2][r0:r1])


def check_nvfp4_gemm(run32, A, B, seg, N, K, experts, what):
    """run32(): the GEMM with fp32 output [M_cap, N] on the device; A = the
    row buffer (per-row outer), B = the weight stack [E*N, K] (per-expert outer)."""
    out = run32()
    api.sync_status()
    M = A[0].shape[0]
    for e in experts:
        r0, r1 = int(seg[e]), int(seg[e + 1])
        if r1 == r0:
            continue
        a = nv4_rows(A, M, K, r0, r1)
        b = np_(B[0][e * N:(e + 1) * N]), sf_block(B[1], B[0].shape[0], K // 16, e * N, (e + 1) * N)
        ref = oracle.grouped_gemm_nvfp4(*a, *b, np_(B[2][e:e + 1]), np.array([0, r1 - r0]), N)
        err = rel_fro(np_(out[r0:r1]).astype(np.float64), ref)
        assert err <= TOL_FRO, (what, e, r1 - r0, err)
    return out


def check_dgrad(run32, A, Bt, seg, Kc, experts, what):
    """A: MXFP8 rows (codes [M, Kc], e8m0); Bt: the requantised transposed
    weights (codes [Nout, E*Kc], e8m0), all on the device."""
    out = run32()
    api.sync_status()
    M, Nout = A[0].shape[0], Bt[0].shape[0]
    Sb = Bt[0].shape[1] // 32
    for e in experts:
        r0, r1 = int(seg[e]), int(seg[e + 1])
        if r1 == r0:
            continue
        a = np_(A[0][r0:r1]), sf_block(A[1], M, Kc // 32, r0, r1)
        b = (np_(Bt[0][:, e * Kc:(e + 1) * Kc]), sf_block(Bt[1], Nout, Sb, 0, Nout, e * Kc // 32, (e + 1) * Kc // 32))
        ref = oracle.grouped_gemm_mxfp8_dgrad(*a, *b, np.array([0, r1 - r0]))
        err = rel_fro(np_(out[r0:r1]).astype(np.float64), ref)
        assert err <= TOL_FRO, (what, e, r1 - r0, err)
    return out


def check_wgrad(run32, At, Bt, seg, experts, what):
    """At [Nw, M], Bt [Kw, M] on the device, MXFP8 along the tokens; out [E, Nw, Kw]."""
    out = run32()
    api.sync_status()
    Nw, M = At[0].shape
    Kw = Bt[0].shape[0]
    for e in experts:
        t0, t1 = int(seg[e]), int(seg[e + 1])
        if t1 == t0:
            assert bool(torch.all(out[e] == 0)), (what, e)
            continue
        a = np_(At[0][:, t0:t1]), sf_block(At[1], Nw, M // 32, 0, Nw, t0 // 32, t1 // 32)
        b = np_(Bt[0][:, t0:t1]), sf_block(Bt[1], Kw, M // 32, 0, Kw, t0 // 32, t1 // 32)
        ref = oracle.grouped_gemm_mxfp8_wgrad(*a, *b, np.array([0, t1 - t0]))[0]
        err = rel_fro(np_(out[e]).astype(np.float64), ref)
        assert err <= TOL_FRO, (what, e, t1 - t0, err)
    return out


def nvfp4_host(q, rows, cols):
    """(codes, MMA-layout sf, outer) device tensors -> whole host arrays, row-major scales."""
    return np_(q[0]), mma_to_rowmajor(np_(q[1]), rows, cols // 16), np_(q[2])


def mx_host(codes, e8, rows, cols):
    return np_(codes), mma_to_rowmajor(np_(e8), rows, cols // 32)


def forward_stagewise(name, expert_seed):
    """Route, quantise, gather, quantise the weights, GEMM1, SwiGLU + quantise,
    GEMM2 on the GPU; every stage against the oracle on the GPU's inputs.
    Returns the GPU tensors the backward consumes."""
    inp = workloads.layer_inputs(name, device="cuda")
    c = inp["cfg"]
    T, k, E, D, F = c["T"], c["k"], c["E"], c["D"], c["F"]
    N1 = 2 * F
    topk = inp["topk"]
    seg, src, pos = api.moe_route(topk.cuda(), E)
    xq = api.nvfp4_quantize(inp["x"], 1, api.MX_SF_ROWMAJOR)
    xp = api.nvfp4_gather_rows(*xq, src, k, D)
    w1q = api.nvfp4_quantize(inp["w1"].view(E * N1, D), N1, api.MX_SF_MMA)
    w2q = api.nvfp4_quantize(inp["w2"].view(E * D, F), D, api.MX_SF_MMA)
    api.sync_status()
    M = src.shape[0]

    # routing and the token quantisation, whole
    seg_o, src_o, pos_o = oracle.route(topk.numpy(), E)
    Mp = int(seg_o[-1])
    assert np.array_equal(np_(seg), seg_o) and np.array_equal(np_(pos), pos_o)
    s_gpu = np_(src)
    assert np.all(s_gpu[Mp:] == -1)
    assert np.array_equal(np.where(s_gpu[:Mp] >= 0, s_gpu[:Mp] // k, -1), src_o)     # assignment t*k+j -> token t
    counts = np.bincount(topk.numpy().ravel(), minlength=E)
    experts = expert_subset(counts, seed=expert_seed)
    xq_o = oracle.nvfp4_quantize(u16(inp["x"]))
    assert np.array_equal(np_(xq[0]), xq_o[0])
    assert np.array_equal(np_(xq[1]).reshape(T, D // 16), xq_o[1])
    assert np.array_equal(np_(xq[2]).view(np.uint32), xq_o[2].view(np.uint32))
    # the NVFP4 dispatch, whole
    xp_h = nvfp4_host(xp, M, D)
    xp_o = oracle.gather_nvfp4_rows(*xq_o, src_o)
    assert np.array_equal(xp_h[0][:Mp], xp_o[0]) and np.array_equal(xp_h[1][:Mp], xp_o[1])
    assert np.array_equal(xp_h[2][:Mp].view(np.uint32), xp_o[2].view(np.uint32))
    del xq_o, xp_o
    # expert weights, whole experts of the subset (an expert's quantisation reads only its own matrix)
    for e in experts:
        for wq, n, kk, w in ((w1q, N1, D, inp["w1"]), (w2q, D, F, inp["w2"])):
            ref = oracle.nvfp4_quantize(u16(w[e]), group_rows=n)
            got = nv4_rows(wq, E * n, kk, e * n, (e + 1) * n)
            assert np.array_equal(got[0], ref[0]), ("weight codes", e)
            assert np.array_equal(got[1], ref[1]), ("weight scales", e)
            assert np_(wq[2][e:e + 1]).view(np.uint32)[0] == ref[2].view(np.uint32)[0], ("outer", e)

    # GEMM1: fp32 against fp64 over whole experts; the bf16 form is its rounding
    h1 = api.grouped_gemm_nvfp4(xp, w1q, seg, E, N1, D)
    h1_32 = check_nvfp4_gemm(lambda: api.grouped_gemm_nvfp4(xp, w1q, seg, E, N1, D, out_dtype=torch.float32),
                             xp, w1q, seg_o, N1, D, experts, "gemm1")
    assert_bf16_rounding(h1[:Mp], h1_32[:Mp], "gemm1 bf16")
    del h1_32
    # SwiGLU on the GPU's h1: within one bf16 rounding; the fused quantiser = oracle quantise of the GPU's a
    rows_valid = seg[E:E + 1]
    a = api.swiglu_fwd(h1, F, True, rows_valid)
    aq = api.swiglu_nvfp4_quantize(h1, F, True, rows_valid, api.MX_SF_MMA)
    api.sync_status()
    a_ref = oracle.bf16_to_f32(oracle.swiglu_fwd(u16(h1)[:Mp], gated=True)).astype(np.float64)
    a_got = oracle.bf16_to_f32(u16(a)[:Mp]).astype(np.float64)
    assert np.all(np.abs(a_got - a_ref) <= 2.0 ** -7 * np.abs(a_ref))     # at most one bf16 step apart
    del a_ref, a_got
    aq_h = nvfp4_host(aq, M, F)
    aq_o = oracle.nvfp4_quantize(u16(a)[:Mp])
    assert np.array_equal(aq_h[0][:Mp], aq_o[0]) and np.array_equal(aq_h[1][:Mp], aq_o[1])
    assert np.array_equal(aq_h[2][:Mp].view(np.uint32), aq_o[2].view(np.uint32))
    del aq_o, a
    # GEMM2
    y2 = api.grouped_gemm_nvfp4(aq, w2q, seg, E, D, F)
    y2_32 = check_nvfp4_gemm(lambda: api.grouped_gemm_nvfp4(aq, w2q, seg, E, D, F, out_dtype=torch.float32),
                             aq, w2q, seg_o, D, F, experts, "gemm2")
    assert_bf16_rounding(y2[:Mp], y2_32[:Mp], "gemm2 bf16")
    del y2_32, y2
    return dict(seg=seg, src=src, xp=xp, w1q=w1q, w2q=w2q, aq=aq, seg_o=seg_o, Mp=Mp, M=M, experts=experts,
                xp_h=xp_h, aq_h=aq_h)


def test_fwd_gemm_config_stagewise(cuda):
    forward_stagewise("fwd_gemm", expert_seed=2)


def test_bwd_gemm_config_stagewise(cuda):
    f = forward_stagewise("bwd_gemm", expert_seed=3)
    c = workloads.CONFIGS["bwd_gemm"]
    E, D, F = c["E"], c["D"], c["F"]
    N1 = 2 * F
    seg, seg_o, M, Mp, experts = f["seg"], f["seg_o"], f["M"], f["Mp"], f["experts"]
    rows_valid = seg[E:E + 1]
    valid = (f["src"] >= 0)[:, None]
    # upstream gradients, drawn independently; rows that hold no routed token are zero, as in the layer
    dy2 = torch.where(valid, workloads.gradient(M, D, c["grad_std"], c["seed"] + 5, "cuda"), 0).to(torch.bfloat16)
    dh1 = torch.where(valid, workloads.gradient(M, N1, c["grad_std"], c["seed"] + 6, "cuda"), 0).to(torch.bfloat16)
    seed = 77
    # MXFP8 of the gradients, row- and column-wise (RNE), whole
    dy2q = api.mxfp8_quantize(dy2, rows_valid=rows_valid)
    dh1q = api.mxfp8_quantize(dh1, rows_valid=rows_valid)
    api.sync_status()
    for name, g, q, cols in (("dy2", dy2, dy2q, D), ("dh1", dh1, dh1q, N1)):
        gh = u16(g)
        r_o, c_o = oracle.mxfp8_quantize_rows(gh[:Mp]), oracle.mxfp8_quantize_cols(gh)
        r_h, c_h = mx_host(q[0], q[1], M, cols), mx_host(q[2], q[3], cols, M)
        assert np.array_equal(r_h[0][:Mp], r_o[0]) and np.array_equal(r_h[1][:Mp], r_o[1]), name
        assert np.array_equal(c_h[0][:, :Mp], c_o[0][:, :Mp]), name
        assert np.array_equal(c_h[1][:, :Mp // 32], c_o[1][:, :Mp // 32]), name
        del gh, r_o, c_o, r_h, c_h
    # requantisation of the saved NVFP4 tensors (dequantise, transpose, MXFP8 with SR), whole
    w2t = api.mxfp8_requant_transpose_sr(*f["w2q"], E * D, F, D, api.MX_SF_MMA, None, seed, 1, R_BITS)
    at = api.mxfp8_requant_transpose_sr(*f["aq"], M, F, 1, api.MX_SF_MMA, rows_valid, seed, 2, R_BITS)
    w1t = api.mxfp8_requant_transpose_sr(*f["w1q"], E * N1, D, N1, api.MX_SF_MMA, None, seed, 3, R_BITS)
    xt = api.mxfp8_requant_transpose_sr(*f["xp"], M, D, 1, api.MX_SF_MMA, rows_valid, seed, 4, R_BITS)
    api.sync_status()
    for name, g, q, group, stream, rows, cols in (
            ("w2t", w2t, f["w2q"], D, 1, E * D, F), ("at", at, f["aq_h"], 1, 2, M, F),
            ("w1t", w1t, f["w1q"], N1, 3, E * N1, D), ("xt", xt, f["xp_h"], 1, 4, M, D)):
        src_h = q if isinstance(q, tuple) and isinstance(q[0], np.ndarray) else nvfp4_host(q, rows, cols)
        ref = oracle.mxfp8_requant_transpose_sr(*src_h, group, seed, stream, R_BITS)
        h = mx_host(g[0], g[1], cols, rows)
        n = Mp if group == 1 else rows                   # token buffers: the routed rows
        assert np.array_equal(h[0][:, :n], ref[0][:, :n]), name
        assert np.array_equal(h[1][:, :n // 32], ref[1][:, :n // 32]), name
        del src_h, ref, h
    # dgrad / wgrad in fp32 over whole experts
    check_dgrad(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, dy2q[0], dy2q[1], *w2t, seg, E, M, F, D,
                                               out_dtype=torch.float32), dy2q[:2], w2t, seg_o, D, experts, "dgrad2")
    check_wgrad(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, dy2q[2], dy2q[3], *at, seg, E, M, D, F,
                                               out_dtype=torch.float32), dy2q[2:], at, seg_o, experts, "wgrad2")
    check_dgrad(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, dh1q[0], dh1q[1], *w1t, seg, E, M, D, N1,
                                               out_dtype=torch.float32), dh1q[:2], w1t, seg_o, N1, experts, "dgrad1")
    check_wgrad(lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, dh1q[2], dh1q[3], *xt, seg, E, M, N1, D,
                                               out_dtype=torch.float32), dh1q[2:], xt, seg_o, experts, "wgrad1")


def test_moe_layer_step_gemms_full_experts(cuda):
    """The 384-expert layer, one forward + backward step through ExpertLayer
    (R = 16): every GEMM re-run in fp32 on the layer's own operands and checked
    over whole experts of the subset against fp64, and the layer's bf16 GEMM
    outputs equal to the rounding of those fp32 outputs."""
    inp = workloads.layer_inputs("moe_layer", device="cuda")
    c = inp["cfg"]
    E, D, F = c["E"], c["D"], c["F"]
    N1 = 2 * F
    L = ExpertLayer(inp["x"], inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"], inp["w2"], inp["dout"],
                    gated=True, seed=c["seed"], rbits=R_BITS)
    L.step()
    api.sync_status()
    M, seg = L.M_cap, L.seg
    seg_o = np_(seg)
    Mp = int(seg_o[-1])
    counts = np.bincount(inp["topk"].numpy().ravel(), minlength=E)
    assert np.array_equal(np.diff(seg_o), (counts + 127) // 128 * 128)
    experts = expert_subset(counts, n_random=2, seed=4)
    empty = np.flatnonzero(counts == 0)
    assert empty.size                                           # the workload has empty experts
    experts.append(int(empty[0]))                               # and one of them is checked
    gemms = (
        ("gemm1", L.h1, lambda: check_nvfp4_gemm(
            lambda: api.grouped_gemm_nvfp4(L.xp, L.w1q, seg, E, N1, D, out_dtype=torch.float32),
            L.xp, L.w1q, seg_o, N1, D, experts, "gemm1")),
        ("gemm2", L.y2, lambda: check_nvfp4_gemm(
            lambda: api.grouped_gemm_nvfp4(L.aq, L.w2q, seg, E, D, F, out_dtype=torch.float32),
            L.aq, L.w2q, seg_o, D, F, experts, "gemm2")),
        ("dgrad2", L.da, lambda: check_dgrad(
            lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, L.dy2q[0], L.dy2q[1], *L.w2t, seg, E, M, F, D,
                                           out_dtype=torch.float32), L.dy2q[:2], L.w2t, seg_o, D, experts, "dgrad2")),
        ("dgrad1", L.dxp, lambda: check_dgrad(
            lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, L.dh1q[0], L.dh1q[1], *L.w1t, seg, E, M, D, N1,
                                           out_dtype=torch.float32), L.dh1q[:2], L.w1t, seg_o, N1, experts, "dgrad1")),
        ("wgrad2", L.dw2, lambda: check_wgrad(
            lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, L.dy2q[2], L.dy2q[3], *L.at, seg, E, M, D, F,
                                           out_dtype=torch.float32), L.dy2q[2:], L.at, seg_o, experts, "wgrad2")),
        ("wgrad1", L.dw1, lambda: check_wgrad(
            lambda: api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, L.dh1q[2], L.dh1q[3], *L.xt, seg, E, M, N1, D,
                                           out_dtype=torch.float32), L.dh1q[2:], L.xt, seg_o, experts, "wgrad1")),
    )
    for name, layer_out, check in gemms:
        o32 = check()
        n = None if name.startswith("wgrad") else Mp
        assert_bf16_rounding(layer_out[:n], o32[:n], name)
        del o32
