"""Grouped GEMMs on seeded random routings, against the oracle.

A fixed list of shapes drawn once from a seeded generator: expert counts from
1 to 300, per-expert row counts with empty experts and ragged tails, output
widths with and without 256-wide tiles, and loads on either side of the
row-mode schedule's decision (a CTA-pair kernel with half pairs, or full
pairs plus the single-CTA tail kernel for the leftover row tiles).  Every
case: fp32 output within relative Frobenius 1e-4 of the oracle's fp64 product
of the same operands, over all routed rows; rows past the routed rows keep
the output buffer's NaN fill.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from tests.layouts import rowmajor_to_mma
from tests.test_gpu_gemm import TOL_FRO, dev, pad_rows, rel_fro, routed_rows

pytestmark = pytest.mark.gpu


def _cases(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        E = int(rng.choice([1, 3, 17, 64, 150, 300]))
        # loads: mostly 1-3 row tiles, some empty experts, a few large ones
        counts = rng.integers(0, 3 * 128, E)
        counts[rng.random(E) < 0.15] = 0
        counts[rng.random(E) < 0.05] += int(rng.integers(400, 1200))
        N = int(rng.choice([128, 256, 384, 1024] if E <= 64 else [256, 1024]))
        out.append((i, E, N, [int(c) for c in counts]))
    return out


def _tail_taken(counts, N, sms=148):
    # the row-mode schedule's decision on a 148-SM B200 (for the case ids only)
    tiles = np.array([(c + 127) // 128 for c in counts])
    return N % 256 == 0 and int(np.sum(tiles % 2)) * (N // 256) >= 4 * sms


NV_CASES = _cases(8, seed=11)
MX_CASES = _cases(8, seed=12)


@pytest.mark.parametrize("i,E,N,counts", NV_CASES,
                         ids=[f"nv{i}-E{E}-N{N}-{'tail' if _tail_taken(c, N) else 'pairs'}" for i, E, N, c in NV_CASES])
def test_grouped_gemm_nvfp4_random_routing(cuda, i, E, N, counts):
    K = 256
    x, seg = routed_rows(counts, K, seed=100 + i, nu=4)
    M_pad = int(seg[-1])
    M_cap = M_pad + 256
    a = oracle.nvfp4_quantize(x)
    w = workloads.weights(E, N, K, 0.02, seed=200 + i).reshape(E * N, K).view(torch.int16).numpy().view(np.uint16)
    b = oracle.nvfp4_quantize(w, group_rows=N)
    ref = oracle.grouped_gemm_nvfp4(*a, *b, seg, N)
    A = (dev(pad_rows(a[0], M_cap)), dev(rowmajor_to_mma(pad_rows(a[1], M_cap))), dev(pad_rows(a[2], M_cap)))
    B = (dev(b[0]), dev(rowmajor_to_mma(b[1])), dev(b[2]))
    out = torch.full((M_cap, N), float("nan"), dtype=torch.float32, device="cuda")
    api.grouped_gemm_nvfp4(A, B, dev(seg), E, N, K, out=out)
    api.sync_status()
    got = out.cpu().numpy()
    assert np.all(np.isnan(got[M_pad:]))
    assert np.all(np.isfinite(got[:M_pad]))
    assert rel_fro(got[:M_pad].astype(np.float64), ref) <= TOL_FRO


@pytest.mark.parametrize("i,E,N,counts", MX_CASES,
                         ids=[f"mx{i}-E{E}-N{N}-{'tail' if _tail_taken(c, N) else 'pairs'}" for i, E, N, c in MX_CASES])
def test_grouped_gemm_mxfp8_dgrad_random_routing(cuda, i, E, N, counts):
    Kc = 128
    dy, seg = routed_rows(counts, Kc, seed=300 + i)
    M_pad = int(seg[-1])
    M_cap = M_pad + 256
    ac, ae = oracle.mxfp8_quantize_rows(dy)
    w = workloads.weights(E, Kc, N, 0.02, seed=400 + i).reshape(E * Kc, N).view(torch.int16).numpy().view(np.uint16)
    wq = oracle.nvfp4_quantize(w, group_rows=Kc)
    bc, be = oracle.mxfp8_requant_transpose_sr(*wq, Kc, seed=1, stream=2)
    ref = oracle.grouped_gemm_mxfp8_dgrad(ac, ae, bc, be, seg)
    out = torch.full((M_cap, N), float("nan"), dtype=torch.float32, device="cuda")
    api.grouped_gemm_mxfp8(api.MX_GEMM_DGRAD, dev(pad_rows(ac, M_cap)), dev(rowmajor_to_mma(pad_rows(ae, M_cap))),
                           dev(bc), dev(rowmajor_to_mma(be)), dev(seg), E, M_cap, N, Kc, out=out)
    api.sync_status()
    got = out.cpu().numpy()
    assert np.all(np.isnan(got[M_pad:]))
    assert np.all(np.isfinite(got[:M_pad]))
    assert rel_fro(got[:M_pad].astype(np.float64), ref) <= TOL_FRO
