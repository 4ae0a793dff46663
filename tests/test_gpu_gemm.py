"""GPU parity of the tcgen05 block-scaled grouped GEMMs against the oracle's
fp64 product of the same dequantised operands, through the C ABI.

Bar (fp32 output): relative Frobenius error <= 1e-4 over all routed rows;
bf16 output: each element within one bf16 rounding of the fp64 value (plus
the fp32 accumulation error).  Integer-exact inputs must match bit for bit.
Operands are produced by the oracle from seeded inputs and converted to the
MMA scale layout by the tests.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from tests.layouts import rowmajor_to_mma

pytestmark = pytest.mark.gpu

TOL_FRO = 1e-4


def rel_fro(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def seg_from_counts(counts):
    padded = [(c + 127) // 128 * 128 for c in counts]
    return np.concatenate([[0], np.cumsum(padded)]).astype(np.int64)


def routed_rows(counts, cols, seed, scale=1.0, nu=None):
    """bf16 [M_pad, cols] with each expert's true rows random and its padding rows zero."""
    seg = seg_from_counts(counts)
    rng = np.random.default_rng(seed)
    x = np.zeros((int(seg[-1]), cols), np.float32)
    for e, c in enumerate(counts):
        v = rng.standard_t(nu, (c, cols)) if nu else rng.standard_normal((c, cols))
        x[seg[e]:seg[e] + c] = v * scale * 10.0 ** rng.uniform(-1, 1, (c, 1))
    return oracle.f32_to_bf16(x), seg


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def pad_rows(a, rows):
    out = np.zeros((rows,) + a.shape[1:], a.dtype)
    out[:a.shape[0]] = a
    return out


NVFP4_CASES = [
    (4, 256, 256, [128, 0, 256, 300]),        # empty expert, ragged tail
    (3, 512, 512, [100, 300, 7]),
    (2, 384, 256, [130, 50]),                 # N % 256 != 0: 128-wide tiles
    (5, 256, 1024, [1, 129, 0, 0, 260]),
    (2, 256, 4096, [200, 70]),                # long K
    (3, 256, 256, [1, 7, 100]),               # one row tile per expert: half pairs only
    (3, 512, 256, [256, 0, 512]),             # even tile counts
    # 1 or 3 row tiles per expert, 4 column tiles: 800 leftover tiles, enough for the tail kernel on 148 SMs
    (200, 1024, 256, [60 + 200 * (i % 2) for i in range(200)]),
]


@pytest.mark.parametrize("E,N,K,counts", NVFP4_CASES)
def test_grouped_gemm_nvfp4_fp32_and_bf16(cuda, E, N, K, counts):
    x, seg = routed_rows(counts, K, seed=E * 1000 + N + K, nu=4)
    M_pad = int(seg[-1])
    M_cap = M_pad + 128
    a = oracle.nvfp4_quantize(x)
    w = workloads.weights(E, N, K, 0.02, seed=N + K).reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    b = oracle.nvfp4_quantize(w, group_rows=N)
    ref = oracle.grouped_gemm_nvfp4(*a, *b, seg, N)
    A = (dev(pad_rows(a[0], M_cap)), dev(rowmajor_to_mma(pad_rows(a[1], M_cap))), dev(pad_rows(a[2], M_cap)))
    B = (dev(b[0]), dev(rowmajor_to_mma(b[1])), dev(b[2]))
    dseg = dev(seg)
    out = torch.full((M_cap, N), float("nan"), dtype=torch.float32, device="cuda")
    api.grouped_gemm_nvfp4(A, B, dseg, E, N, K, out=out)
    api.sync_status()
    got = out.cpu().numpy()
    assert np.all(np.isnan(got[M_pad:]))                 # rows past the routed rows untouched
    assert np.all(np.isfinite(got[:M_pad]))
    assert rel_fro(got[:M_pad].astype(np.float64), ref) <= TOL_FRO
    outb = api.grouped_gemm_nvfp4(A, B, dseg, E, N, K, out_dtype=torch.bfloat16)
    gb = outb.float().cpu().numpy()[:M_pad].astype(np.float64)
    assert np.all(np.abs(gb - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max())


def test_grouped_gemm_nvfp4_integer_exact(cuda):
    # codes +-1 or +-2, block scales 1 or 2, outer scales 1: every product and
    # partial sum is a small integer, so the fp32 result is exact
    E, N, K = 2, 256, 512
    counts = [128, 256]
    seg = seg_from_counts(counts)
    M = int(seg[-1])
    rng = np.random.default_rng(0)
    code_vals = np.array([0x2, 0xA, 0x4, 0xC], np.uint8)                 # 1, -1, 2, -2
    ac = (code_vals[rng.integers(0, 4, (M, K))]).astype(np.uint8)
    bc = (code_vals[rng.integers(0, 4, (E * N, K))]).astype(np.uint8)
    pack = lambda c: (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
    asf = np.where(rng.random((M, K // 16)) < 0.5, 0x38, 0x40).astype(np.uint8)   # 1.0 / 2.0
    bsf = np.where(rng.random((E * N, K // 16)) < 0.5, 0x38, 0x40).astype(np.uint8)
    ao = np.ones(M, np.float32)
    bo = np.ones(E, np.float32)
    ref = oracle.grouped_gemm_nvfp4(pack(ac), asf, ao, pack(bc), bsf, bo, seg, N)
    out = api.grouped_gemm_nvfp4((dev(pack(ac)), dev(rowmajor_to_mma(asf)), dev(ao)),
                                 (dev(pack(bc)), dev(rowmajor_to_mma(bsf)), dev(bo)), dev(seg), E, N, K,
                                 out_dtype=torch.float32)
    assert np.array_equal(out.cpu().numpy().astype(np.float64), ref)


MX_CASES = [
    (3, 256, 256, [128, 0, 300]),
    (2, 384, 128, [50, 260]),                 # N % 256 != 0
    (4, 512, 512, [1, 0, 129, 256]),
    (3, 256, 256, [1, 7, 100]),               # half pairs only
    (3, 256, 256, [256, 0, 512]),             # full pairs only
    (200, 1024, 128, [60 + 200 * (i % 2) for i in range(200)]),  # the tail kernel (800 leftover tiles)
]


@pytest.mark.parametrize("E,Nout,Kc,counts", MX_CASES)
def test_grouped_gemm_mxfp8_dgrad(cuda, E, Nout, Kc, counts):
    # dX = dY . W: A = dY [M, Kc] row-wise MXFP8, B = requantised W^T [Nout, E*Kc]
    dy, seg = routed_rows(counts, Kc, seed=E + Nout + Kc)
    M_pad = int(seg[-1])
    M_cap = M_pad + 128
    ac, ae = oracle.mxfp8_quantize_rows(dy)
    w = workloads.weights(E, Kc, Nout, 0.02, seed=Kc).reshape(E * Kc, Nout).view(torch.int16).numpy().view(np.uint16)
    wq = oracle.nvfp4_quantize(w, group_rows=Kc)
    bc, be = oracle.mxfp8_requant_transpose_sr(*wq, Kc, seed=1, stream=2)
    ref = oracle.grouped_gemm_mxfp8_dgrad(ac, ae, bc, be, seg)
    out = torch.full((M_cap, Nout), float("nan"), dtype=torch.float32, device="cuda")
    api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, dev(pad_rows(ac, M_cap)), dev(rowmajor_to_mma(pad_rows(ae, M_cap))),
                           dev(bc), dev(rowmajor_to_mma(be)), dev(seg), E, M_cap, Nout, Kc, out=out)
    api.sync_status()
    got = out.cpu().numpy()
    assert np.all(np.isnan(got[M_pad:]))
    assert rel_fro(got[:M_pad].astype(np.float64), ref) <= TOL_FRO
    outb = api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, dev(pad_rows(ac, M_cap)), dev(rowmajor_to_mma(pad_rows(ae, M_cap))),
                                  dev(bc), dev(rowmajor_to_mma(be)), dev(seg), E, M_cap, Nout, Kc,
                                  out_dtype=torch.bfloat16)
    gb = outb.float().cpu().numpy()[:M_pad].astype(np.float64)
    assert np.all(np.abs(gb - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max())


@pytest.mark.parametrize("E,N,K,counts", [(3, 256, 512, [100, 0, 300]), (2, 512, 256, [130, 50])])
def test_mxfp8_forward_gemm_with_weights_as_rows(cuda, E, N, K, counts):
    # the MXFP8 forward baseline: X [M, K] and W [E, N, K] both row-wise MXFP8
    # (RNE, quantised on the GPU), W laid out [N, E*K] for the row GEMM
    x, seg = routed_rows(counts, K, seed=3 * E + N + K, nu=4)
    M_pad = int(seg[-1])
    M_cap = M_pad + 128
    w = workloads.weights(E, N, K, 0.02, seed=N + 2 * K)
    wp = w.permute(1, 0, 2).reshape(N, E * K).contiguous()
    ac, ae = oracle.mxfp8_quantize_rows(pad_rows(x, M_cap))
    bc, be = oracle.mxfp8_quantize_rows(wp.view(torch.int16).numpy().view(np.uint16))
    ref = oracle.grouped_gemm_mxfp8_dgrad(ac[:M_pad], ae[:M_pad], bc, be, seg)
    ga = api.mxfp8_quantize(dev(pad_rows(x, M_cap).view(np.int16)).view(torch.bfloat16), col=False)
    gb = api.mxfp8_quantize(wp.cuda(), col=False)
    assert np.array_equal(ga[0].cpu().numpy(), ac) and np.array_equal(gb[0].cpu().numpy(), bc)
    out = api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, ga[0], ga[1], gb[0], gb[1], dev(seg), E, M_cap, N, K,
                                 out_dtype=torch.float32)
    api.sync_status()
    assert rel_fro(out.cpu().numpy()[:M_pad].astype(np.float64), ref) <= TOL_FRO


@pytest.mark.parametrize("E,Nw,Kw,counts", [(3, 256, 256, [128, 0, 300]), (2, 128, 384, [60, 200]),
                                            (4, 256, 512, [0, 129, 1, 256])])
def test_grouped_gemm_mxfp8_wgrad(cuda, E, Nw, Kw, counts):
    # dW_e = dY_e^T . X_e: A = dY^T [Nw, M] (column-wise MXFP8), B = X^T [Kw, M] (requantised)
    dy, seg = routed_rows(counts, Nw, seed=7 * E + Nw)
    x, _ = routed_rows(counts, Kw, seed=5 * E + Kw, nu=3)
    M_pad = int(seg[-1])
    M_cap = M_pad + 128
    ac, ae = oracle.mxfp8_quantize_cols(pad_rows(dy, M_cap))
    xq = oracle.nvfp4_quantize(pad_rows(x, M_cap))
    bc, be = oracle.mxfp8_requant_transpose_sr(*xq, 1, seed=3, stream=4)
    ref = oracle.grouped_gemm_mxfp8_wgrad(ac, ae, bc, be, seg)
    out = torch.full((E, Nw, Kw), float("nan"), dtype=torch.float32, device="cuda")
    api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, dev(ac), dev(rowmajor_to_mma(ae)), dev(bc), dev(rowmajor_to_mma(be)),
                           dev(seg), E, M_cap, Nw, Kw, out=out)
    api.sync_status()
    got = out.cpu().numpy().astype(np.float64)
    for e in range(E):
        if seg[e + 1] == seg[e]:
            assert np.all(got[e] == 0)                    # empty expert -> zeros
    assert rel_fro(got, ref) <= TOL_FRO
    outb = api.grouped_gemm_mxfp8(api.MX_GEMM_WGRAD, dev(ac), dev(rowmajor_to_mma(ae)), dev(bc), dev(rowmajor_to_mma(be)),
                                  dev(seg), E, M_cap, Nw, Kw, out_dtype=torch.bfloat16)
    gb = outb.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gb - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max())
