"""GPU parity of the NVFP4-backward entry points and the 16x16 shared-scale
quantiser (csrc/nvfp4_bwd.cu) against the oracle.

Bar: bit-exact codes, scales and outer scales; both sides take every
rounding decision in fp32 in the same order, and the stochastic rounding
draws the same Philox integers.  The NVFP4 dgrad (the forward grouped GEMM
with the requantised W_e^T stack as B) within the forward GEMM's relative
Frobenius bound of the oracle's fp64 product.

Their index arithmetic is also replayed on the CPU
(tests/test_nvfp4_bwd_indexing.py).
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api
from tests.layouts import mma_to_rowmajor
from tests.test_gpu_gemm import dev, rel_fro

pytestmark = pytest.mark.gpu


def to_dev_bf16(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_input(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(3, (rows, cols)) * 10.0 ** rng.uniform(-3, 3, (rows, 1))
    x[rows // 2] = 0.0                                           # a zero row
    x[1, 5] = -0.0
    return oracle.f32_to_bf16(x.astype(np.float32))


def host(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("rows,cols,group_rows,layout", [(128, 256, 1, api.MX_SF_MMA), (256, 512, 128, api.MX_SF_MMA),
                                                         (48, 96, 16, api.MX_SF_ROWMAJOR)])
@pytest.mark.parametrize("rbits", [8, 16, 32])
def test_nvfp4_quantize_sr_bit_exact(cuda, rows, cols, group_rows, layout, rbits):
    x = bf16_input(rows, cols, rows + cols + rbits)
    seed, stream = 1234, 5
    c, sf, o = api.nvfp4_quantize_sr(to_dev_bf16(x), group_rows, api.MX_ROUND_SR, seed, stream, rbits, layout)
    api.sync_status()
    rc, rsf, ro = oracle.nvfp4_quantize_f32(oracle.bf16_to_f32(x), group_rows, True, seed, stream, rbits)
    sf_h = mma_to_rowmajor(host(sf), rows, cols // 16) if layout == api.MX_SF_MMA else host(sf).reshape(rows, -1)
    assert np.array_equal(host(o), ro)
    assert np.array_equal(sf_h, rsf)
    assert np.array_equal(host(c), rc)


def edge_input(rows, cols, seed):
    """Blocks that reach the rounding's special cases: the block maximum and
    values down to bf16 subnormals (scaled values below fp32's normal range),
    signed zeros, values on the E2M1 grid of their block (k/6 of the maximum),
    values just above 6 after scaling (the block scale rounded down), and
    saturating blocks."""
    rng = np.random.default_rng(seed)
    x = np.zeros((rows, cols), np.float64)
    for r in range(rows):
        for b in range(cols // 16):
            kind = (r + b) % 5
            big = 10.0 ** rng.uniform(-2, 3)
            v = rng.standard_normal(16) * big
            if kind == 0:                                        # tiny neighbours of a large maximum
                v[1:] = np.ldexp(rng.uniform(1, 2, 15), rng.integers(-133, -110, 15))
            elif kind == 1:                                      # grid points of the block
                v = big * np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6] * 2) / 6 * rng.choice([-1, 1], 16)
            elif kind == 2:                                      # signed zeros with one nonzero
                v[:] = -0.0
                v[7] = big
            elif kind == 3:                                      # a maximum whose scale rounds down
                v[0] = big * 1.0624
                v[1:] = big * rng.uniform(0.9, 1.0, 15)
            v[0] = abs(v[0]) if kind != 2 else v[0]
            x[r, 16 * b:16 * b + 16] = v
    return oracle.f32_to_bf16(x.astype(np.float32))


@pytest.mark.parametrize("rbits", [8, 16, 32])
def test_nvfp4_quantize_sr_edge_values_bit_exact(cuda, rbits):
    rows, cols = 256, 256
    x = edge_input(rows, cols, 40 + rbits)
    seed, stream = 77, 3
    c, sf, o = api.nvfp4_quantize_sr(to_dev_bf16(x), 1, api.MX_ROUND_SR, seed, stream, rbits, api.MX_SF_MMA)
    api.sync_status()
    rc, rsf, ro = oracle.nvfp4_quantize_f32(oracle.bf16_to_f32(x), 1, True, seed, stream, rbits)
    assert np.array_equal(host(o), ro)
    assert np.array_equal(mma_to_rowmajor(host(sf), rows, cols // 16), rsf)
    assert np.array_equal(host(c), rc)


def test_nvfp4_quantize_sr_rne_equals_the_forward_quantiser(cuda):
    x = to_dev_bf16(bf16_input(256, 256, 3))
    a = api.nvfp4_quantize_sr(x, 1, api.MX_ROUND_RNE)
    b = api.nvfp4_quantize(x, 1, api.MX_SF_MMA)
    api.sync_status()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("rows,cols,rbits", [(256, 128, 16), (384, 256, 8), (128, 128, 32)])
def test_requant_transpose_activations_bit_exact(cuda, rows, cols, rbits):
    q = oracle.nvfp4_quantize(bf16_input(rows, cols, rows * cols))
    from tests.layouts import rowmajor_to_mma
    seed, stream = 77, 9
    oc, osf, oo = api.nvfp4_requant_transpose_sr(dev(q[0]), dev(rowmajor_to_mma(q[1])), dev(q[2]), rows, cols, 1,
                                                 api.MX_SF_MMA, 1, False, api.MX_ROUND_SR, seed, stream, rbits,
                                                 api.MX_SF_MMA)
    api.sync_status()
    rc, rsf, ro = oracle.nvfp4_requant_transpose_sr(*q, 1, seed, stream, rbits)
    assert np.array_equal(host(oo), ro)
    assert np.array_equal(mma_to_rowmajor(host(osf), cols, rows // 16), rsf)
    assert np.array_equal(host(oc), rc)


def test_requant_transpose_expert_weights_bit_exact(cuda):
    E, N, K = 3, 128, 256
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((E * N, K)) * np.repeat([1.0, 30.0, 0.01], N)[:, None]).astype(np.float32)
    q = oracle.nvfp4_quantize(oracle.f32_to_bf16(w), group_rows=N)
    from tests.layouts import rowmajor_to_mma
    seed, stream = 5, 6
    oc, osf, oo = api.nvfp4_requant_transpose_sr(dev(q[0]), dev(rowmajor_to_mma(q[1])), dev(q[2]), E * N, K, N,
                                                 api.MX_SF_MMA, E, True, api.MX_ROUND_SR, seed, stream, 16,
                                                 api.MX_SF_MMA)
    api.sync_status()
    rc, rsf, ro = oracle.nvfp4_requant_transpose_experts_sr(*q, E, seed, stream, 16)
    assert np.array_equal(host(oo), ro)
    assert np.array_equal(mma_to_rowmajor(host(osf), E * K, N // 16), rsf)
    assert np.array_equal(host(oc), rc)


@pytest.mark.parametrize("rows,cols,group_rows", [(64, 48, 32), (256, 512, 256), (16, 16, 16)])
def test_tile16_bit_exact(cuda, rows, cols, group_rows):
    x = bf16_input(rows, cols, 11 + rows)
    c, sf, o = api.nvfp4_quantize_tile16(to_dev_bf16(x), group_rows)
    api.sync_status()
    rc, rsf, ro = oracle.nvfp4_quantize_tile16(oracle.bf16_to_f32(x), group_rows)
    assert np.array_equal(host(o), ro) and np.array_equal(host(sf), rsf) and np.array_equal(host(c), rc)


def test_nvfp4_dgrad_through_the_forward_gemm(cuda):
    # dX = dY W_e per expert, with dY quantised by SR and B the requantised
    # stack of W_e^T: the forward grouped GEMM with output width K
    from tests.layouts import rowmajor_to_mma
    E, N, K, M = 2, 256, 256, 256
    seg = np.array([0, 128, 256], dtype=np.int64)
    rng = np.random.default_rng(12)
    w = oracle.nvfp4_quantize(oracle.f32_to_bf16((rng.standard_normal((E * N, K)) * 0.02).astype(np.float32)), N)
    dy = oracle.f32_to_bf16(rng.standard_normal((M, N)).astype(np.float32))
    wt = api.nvfp4_requant_transpose_sr(dev(w[0]), dev(rowmajor_to_mma(w[1])), dev(w[2]), E * N, K, N,
                                        api.MX_SF_MMA, E, True, api.MX_ROUND_SR, 2, 5, 16, api.MX_SF_MMA)
    dq = api.nvfp4_quantize_sr(to_dev_bf16(dy), 1, api.MX_ROUND_SR, 3, 6, 16, api.MX_SF_MMA)
    dx = api.grouped_gemm_nvfp4(dq, wt, dev(seg), E, K, N, out_dtype=torch.float32)
    api.sync_status()
    rwt = oracle.nvfp4_requant_transpose_experts_sr(*w, E, 2, 5, 16)
    rdq = oracle.nvfp4_quantize_f32(oracle.bf16_to_f32(dy), 1, True, 3, 6, 16)
    ref = oracle.grouped_gemm_nvfp4(*rdq, *rwt, seg, K)
    assert rel_fro(host(dx).astype(np.float64), ref) <= 1e-4


def _segments(counts):
    seg = np.zeros(len(counts) + 1, dtype=np.int64)
    seg[1:] = np.cumsum([(c + 127) // 128 * 128 for c in counts])
    return seg


@pytest.mark.parametrize("per_row", [True, False])
def test_transpose_segments_from_bf16_bit_exact(cuda, per_row):
    seg = _segments([200, 0, 90, 300])
    M, C = int(seg[-1]) + 128, 128                                # one block of padding rows
    x = bf16_input(M, C, 21)
    oc, osf, oo = api.nvfp4_quantize_transpose_segments(to_dev_bf16(x), dev(seg), len(seg) - 1, per_row,
                                                        api.MX_ROUND_SR, 8, 9, 16, api.MX_SF_MMA)
    api.sync_status()
    rc, rsf, ro = oracle.nvfp4_quantize_transpose_segments(oracle.bf16_to_f32(x), seg, per_row, True, 8, 9, 16)
    assert np.array_equal(host(oo), ro.reshape(-1))
    assert np.array_equal(mma_to_rowmajor(host(osf), C, M // 16), rsf)
    assert np.array_equal(host(oc), rc)


def test_requant_transpose_segments_bit_exact(cuda):
    from tests.layouts import rowmajor_to_mma
    seg = _segments([130, 60, 0, 250])
    M, C = int(seg[-1]), 256
    q = oracle.nvfp4_quantize(bf16_input(M, C, 22))
    oc, osf, oo = api.nvfp4_requant_transpose_segments(dev(q[0]), dev(rowmajor_to_mma(q[1])), dev(q[2]), M, C,
                                                       dev(seg), len(seg) - 1, False, 1, api.MX_SF_MMA,
                                                       api.MX_ROUND_SR, 10, 11, 8, api.MX_SF_MMA)
    api.sync_status()
    xh = oracle.nvfp4_dequantize(*q)
    rc, rsf, ro = oracle.nvfp4_quantize_transpose_segments(xh, seg, False, True, 10, 11, 8)
    assert np.array_equal(host(oo), ro)
    assert np.array_equal(mma_to_rowmajor(host(osf), C, M // 16), rsf)
    assert np.array_equal(host(oc), rc)


@pytest.mark.parametrize("Nw,Kw,counts", [(256, 256, [300, 0, 200, 512]), (128, 384, [100, 40])])
def test_nvfp4_wgrad_gemm(cuda, Nw, Kw, counts):
    # operands from the oracle (segments at multiples of 256 tokens), the GEMM on the GPU
    from tests.layouts import rowmajor_to_mma
    seg = np.zeros(len(counts) + 1, dtype=np.int64)
    seg[1:] = np.cumsum([(c + 255) // 256 * 256 for c in counts])
    E, M = len(counts), int(seg[-1])
    rng = np.random.default_rng(Nw + Kw)
    dy = (rng.standard_normal((M, Nw)) * 10.0 ** rng.uniform(-2, 2, (M, 1))).astype(np.float32)
    x = rng.standard_t(3, (M, Kw)).astype(np.float32)
    a = oracle.nvfp4_quantize_transpose_segments(dy, seg, True, True, 3, 4, 16)
    b = oracle.nvfp4_quantize_transpose_segments(x, seg, False, True, 3, 5, 16)
    A = (dev(a[0]), dev(rowmajor_to_mma(a[1])), dev(a[2].reshape(-1)))
    B = (dev(b[0]), dev(rowmajor_to_mma(b[1])), dev(b[2]))
    out = api.grouped_gemm_nvfp4_wgrad(A, B, dev(seg), E, Nw, Kw, out_dtype=torch.float32)
    api.sync_status()
    ref = oracle.grouped_gemm_nvfp4_wgrad(*a, *b, seg)
    got = host(out).astype(np.float64)
    for e in range(E):
        if seg[e + 1] == seg[e]:
            assert np.all(got[e] == 0)
        else:
            assert rel_fro(got[e], ref[e]) <= 1e-4


def test_tiny_layer_nvfp4_backward_against_oracle(cuda):
    # the tiny layer with backward="nvfp4" against the oracle's own chain:
    # routing padded to 256 rows, Philox streams 11-18 as the layer uses them
    from fp8_moe_numerics_b200 import workloads
    from fp8_moe_numerics_b200.layer import ExpertLayer
    from tests.test_gpu_layer import f64, pad, rel, u16
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    E, D, F = c["E"], c["D"], c["F"]
    seed, R = 99, 16
    L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(), inp["w2"].cuda(),
                    inp["dout"].cuda(), gated=False, seed=seed, wgrad_dtype=torch.float32, backward="nvfp4")
    L.step()
    api.sync_status()
    M = L.M_cap
    g = lambda t: t.cpu().numpy()

    x, dout = u16(inp["x"]), u16(inp["dout"])
    w1, w2 = u16(inp["w1"]).reshape(E * F, D), u16(inp["w2"]).reshape(E * D, F)
    w = inp["w_comb"].numpy()
    seg, src, pos = oracle.route(inp["topk"].numpy(), E, 256)
    Mp = int(seg[-1])
    xp = oracle.gather_nvfp4_rows(*oracle.nvfp4_quantize(x), src)
    w1q = oracle.nvfp4_quantize(w1, group_rows=F)
    w2q = oracle.nvfp4_quantize(w2, group_rows=D)
    h1 = oracle.f64_to_bf16(oracle.grouped_gemm_nvfp4(*xp, *w1q, seg, F))
    aq = oracle.nvfp4_quantize(oracle.swiglu_fwd(h1, gated=False))
    dy2 = oracle.dispatch_grad(dout, pos, w, Mp)
    f32 = lambda u, rows: oracle.bf16_to_f32(pad(u, rows))
    deq = lambda q: oracle.nvfp4_dequantize(pad(q[0], M), pad(q[1], M), pad(q[2], M))
    dy2n = oracle.nvfp4_quantize_f32(f32(dy2, M), 1, True, seed, 11, R)
    w2tn = oracle.nvfp4_requant_transpose_experts_sr(*w2q, E, seed, 12, R)
    da = oracle.f64_to_bf16(oracle.grouped_gemm_nvfp4(*dy2n, *w2tn, seg, F)[:Mp])
    dy2tn = oracle.nvfp4_quantize_transpose_segments(f32(dy2, M), seg, True, True, seed, 13, R)
    atn = oracle.nvfp4_quantize_transpose_segments(deq(aq), seg, False, True, seed, 14, R)
    dw2 = oracle.grouped_gemm_nvfp4_wgrad(*dy2tn, *atn, seg)
    dh1 = oracle.swiglu_bwd(h1, da, gated=False)
    dh1n = oracle.nvfp4_quantize_f32(f32(dh1, M), 1, True, seed, 15, R)
    w1tn = oracle.nvfp4_requant_transpose_experts_sr(*w1q, E, seed, 16, R)
    dxp = oracle.f64_to_bf16(oracle.grouped_gemm_nvfp4(*dh1n, *w1tn, seg, D)[:Mp])
    dh1tn = oracle.nvfp4_quantize_transpose_segments(f32(dh1, M), seg, True, True, seed, 17, R)
    xtn = oracle.nvfp4_quantize_transpose_segments(deq(xp), seg, False, True, seed, 18, R)
    dw1 = oracle.grouped_gemm_nvfp4_wgrad(*dh1tn, *xtn, seg)
    dx = oracle.combine(dxp, pos, np.ones_like(w))

    # operands built from bit-exact inputs: bit for bit
    assert np.array_equal(g(L.seg), seg)
    for got, ref, rows, cols in ((L.w2tn, w2tn, E * F, D), (L.w1tn, w1tn, E * D, F), (L.dy2n, dy2n, M, D),
                                 (L.dy2tn, dy2tn, D, M)):
        assert np.array_equal(g(got[0]), ref[0])
        assert np.array_equal(mma_to_rowmajor(g(got[1]), rows, cols // 16), ref[1])
        assert np.array_equal(g(got[2]), ref[2].reshape(-1))
    # after a GEMM output (fp32 vs fp64 sums, one bf16 rounding): rare code flips only
    assert np.mean(g(L.atn[0]) == atn[0]) >= 0.99 and np.mean(g(L.dh1n[0]) == dh1n[0]) >= 0.99
    for got, ref in ((f64(u16(L.da)[:Mp]), f64(da)), (g(L.dw2).astype(np.float64), dw2),
                     (f64(u16(L.dxp)[:Mp]), f64(dxp)), (g(L.dw1).astype(np.float64), dw1), (f64(u16(L.dx)), f64(dx))):
        assert rel(got, ref) < 2e-2
