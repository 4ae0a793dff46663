"""GPU parity of the combine path in S2F6: the 32-d random Hadamard rotation
with block-scaled S2F6 quantisation (standalone and as the NVFP4 GEMM's
epilogue) and the combine that reads it, against the CPU oracle.

Bar:
- hadamard_s2f6_quantize: codes and exponents bit-exact (both sides rotate
  the same fp32 values with the same butterflies).
- grouped_gemm_nvfp4_s2f6: the epilogue rotates the GPU's fp32 GEMM output,
  which differs from the oracle's fp64 product rounded to fp32 in its last
  bits, so a code may differ by one where the oracle's scaled value is within
  rounding distance of a half-integer, and an exponent may differ where the
  block amax sits on a power-of-two boundary; everything else is equal.  The
  decoded rows must also meet the quantisation error bound against the fp64
  product.
- moe_combine_s2f6: within one bf16 rounding of the oracle's fp64 value, plus
  the fp32 accumulation error bounded by the block's magnitude.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from tests.layouts import rowmajor_to_mma
from tests.test_gpu_gemm import dev, pad_rows, routed_rows

pytestmark = pytest.mark.gpu


def to_dev_bf16(u16):
    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def heavy_rows(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(3, (rows, cols)) * 10.0 ** rng.uniform(-3, 3, (rows, 1))
    x[rows // 3, cols // 5] = 3e4                                  # an outlier
    x[rows // 2] = 0                                               # a zero row
    if rows > 4:
        x[3, :32] = 1e-39                                          # a block of subnormal-range values
        x[4, 32:64] = 5e36                                         # large: the rotation's sums stay finite
    if rows > 4 and cols >= 96:
        x[4, 64:96] = 0
        x[4, 70] = 3.3895e38                                       # one-hot near the bf16 top: e clamps at 127
    return oracle.f32_to_bf16(x.astype(np.float32))


@pytest.mark.parametrize("rows,cols", [(256, 4096), (7, 96), (130, 1024), (64, 32)])
def test_hadamard_s2f6_quantize_bit_exact(cuda, rows, cols):
    x = heavy_rows(rows, cols, rows + cols)
    seed, stream = 12345 + rows, 3
    c_ref, e_ref = oracle.s2f6_quantize_hadamard(oracle.bf16_to_f32(x), seed, stream)
    c, e = api.hadamard_s2f6_quantize(to_dev_bf16(x), seed, stream)
    api.sync_status()
    assert np.array_equal(e.cpu().numpy(), e_ref)
    assert np.array_equal(c.cpu().numpy(), c_ref)


def test_hadamard_s2f6_quantize_empty(cuda):
    c, e = api.hadamard_s2f6_quantize(torch.empty(0, 64, dtype=torch.bfloat16, device="cuda"), 1, 2)
    api.sync_status()
    assert c.shape == (0, 64) and e.shape == (0, 2)


@pytest.mark.parametrize("E,N,K,counts", [(4, 256, 256, [128, 0, 256, 300]), (3, 512, 512, [100, 300, 7]),
                                          (2, 384, 256, [130, 50]), (2, 256, 2048, [200, 70]),
                                          (2, 4352, 256, [130, 50]),       # wider than the sign table
                                          # 1 or 3 row tiles per expert, 4 column tiles: 800 leftover tiles,
                                          # enough for the tail kernel's S2F6 form on 148 SMs
                                          (200, 1024, 256, [60 + 200 * (i % 2) for i in range(200)])])
def test_grouped_gemm_nvfp4_s2f6_epilogue(cuda, E, N, K, counts):
    x, seg = routed_rows(counts, K, seed=E * 100 + N + K, nu=4)
    M_pad = int(seg[-1])
    M_cap = M_pad + 128
    a = oracle.nvfp4_quantize(x)
    w = workloads.weights(E, N, K, 0.02, seed=N + K + 1).reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    b = oracle.nvfp4_quantize(w, group_rows=N)
    ref = oracle.grouped_gemm_nvfp4(*a, *b, seg, N)                # fp64 [M_pad, N]
    seed, stream = 99, 7
    c_ref, e_ref = oracle.s2f6_quantize_hadamard(ref.astype(np.float32), seed, stream)
    A = (dev(pad_rows(a[0], M_cap)), dev(rowmajor_to_mma(pad_rows(a[1], M_cap))), dev(pad_rows(a[2], M_cap)))
    B = (dev(b[0]), dev(rowmajor_to_mma(b[1])), dev(b[2]))
    codes = torch.full((M_cap, N), 77, dtype=torch.int8, device="cuda")
    e8 = torch.full((M_cap, N // 32), 201, dtype=torch.uint8, device="cuda")
    api.grouped_gemm_nvfp4_s2f6(A, B, dev(seg), E, N, K, seed, stream, out=(codes, e8))
    api.sync_status()
    c, e = codes.cpu().numpy(), e8.cpu().numpy()
    assert np.all(c[M_pad:] == 77) and np.all(e[M_pad:] == 201)   # rows past the routed rows untouched
    c, e = c[:M_pad], e[:M_pad]
    # exponents: equal except where the oracle's block amax is within 1e-5 of
    # either end of its exponent's range ((127/64) 2^(e-1), (127/64) 2^e]
    zr = oracle.fwht32_f32((ref.astype(np.float32) * oracle.hadamard_signs(seed, stream, N).astype(np.float32))
                           .reshape(M_pad, N // 32, 32))
    amax = np.abs(zr).max(-1).astype(np.float64)
    ratio = amax / np.ldexp(127 / 64, e_ref.astype(np.int64) - 127)
    edge = (np.abs(ratio - 1.0) < 1e-5) | (np.abs(ratio - 0.5) < 0.5e-5)
    assert np.all((e == e_ref) | edge)
    same_e = np.repeat(e == e_ref, 32, axis=1)
    dc = np.abs(c.astype(np.int64) - c_ref.astype(np.int64))
    assert np.all(dc[same_e] <= 1)
    assert np.mean(dc[same_e] != 0) < 0.01
    # decoded rows against the fp64 product: half a code step per rotated coordinate
    xh = oracle.s2f6_dequantize_hadamard(c, e, seed, stream)
    err = np.linalg.norm((xh - ref).reshape(M_pad, N // 32, 32), axis=-1)
    nrm = np.linalg.norm(ref.reshape(M_pad, N // 32, 32), axis=-1)
    assert np.all(err <= np.ldexp(1.0, e.astype(np.int64) - 127 - 7) + 1e-4 * nrm)


def test_combine_s2f6_within_one_rounding(cuda):
    T, k, E, D = 300, 4, 16, 512
    ids = workloads.routing(T, k, E, "zipf", 1.1, 0, seed=5)
    seg, src, pos = oracle.route(ids.numpy(), E)
    M = int(seg[-1])
    rng = np.random.default_rng(6)
    y = (rng.standard_t(4, (M, D)) * 10.0 ** rng.uniform(-2, 2, (M, 1))).astype(np.float32)
    seed, stream = 4, 11
    c, e = oracle.s2f6_quantize_hadamard(y, seed, stream)
    w = rng.uniform(0.05, 1.0, (T, k)).astype(np.float32)
    ref = oracle.combine_s2f6(c, e, pos, w, seed, stream)
    got = api.moe_combine_s2f6(dev(c), dev(e), dev(pos), dev(w), seed, stream).cpu().view(torch.int16).numpy()
    api.sync_status()
    g = oracle.bf16_to_f32(got.view(np.uint16)).astype(np.float64)
    r = oracle.bf16_to_f32(ref).astype(np.float64)
    # per (token, block): sum_j |w_j| * max|zhat_j| bounds every fp32 partial sum
    zmax = np.abs(c.astype(np.float64)).reshape(M, D // 32, 32).max(-1) * np.ldexp(1.0, e.astype(np.int64) - 133)
    S = np.einsum("tj,tjb->tb", w.astype(np.float64), zmax[pos])
    tol = np.abs(r) * 2.0 ** -7 + np.repeat(S, 32, axis=1) * 2.0 ** -18
    assert np.all(np.abs(g - r) <= tol)
    # NULL weights: all ones
    ref1 = oracle.combine_s2f6(c, e, pos, np.ones((T, k), np.float32), seed, stream)
    got1 = api.moe_combine_s2f6(dev(c), dev(e), dev(pos), None, seed, stream).cpu().view(torch.int16).numpy()
    r1 = oracle.bf16_to_f32(ref1).astype(np.float64)
    g1 = oracle.bf16_to_f32(got1.view(np.uint16)).astype(np.float64)
    S1 = np.einsum("tjb->tb", zmax[pos])
    assert np.all(np.abs(g1 - r1) <= np.abs(r1) * 2.0 ** -7 + np.repeat(S1, 32, axis=1) * 2.0 ** -18)


def test_layer_with_s2f6_combine_stays_within_the_format_error(cuda):
    # the same layer with the combine in bf16 and in S2F6: the two outputs
    # differ by the S2F6 quantisation only (about 1% of the rows' scale for
    # 7-bit codes of the rotated blocks), and the backward is unchanged
    from fp8_moe_numerics_b200.layer import ExpertLayer
    inp = workloads.layer_inputs("tiny_layer", device="cpu")
    c = inp["cfg"]
    outs, dxs = [], []
    for mode in ("bf16", "s2f6"):
        L = ExpertLayer(inp["x"].cuda(), inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"].cuda(),
                        inp["w2"].cuda(), inp["dout"].cuda(), gated=c["gated"], seed=3, combine=mode)
        L.step()
        api.sync_status()
        outs.append(L.out.float().cpu().numpy().astype(np.float64))
        dxs.append(L.dx.float().cpu().numpy())
    rel = np.linalg.norm(outs[1] - outs[0]) / np.linalg.norm(outs[0])
    assert 0 < rel < 0.03
    assert np.array_equal(dxs[0], dxs[1])
