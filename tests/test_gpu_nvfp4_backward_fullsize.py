"""The NVFP4 backward of the 384-expert layer at full size, stage by stage.

One forward + backward step of ExpertLayer(backward="nvfp4") on the
benchmark's layer, then each stage checked on the GPU's own bytes of the
stage before it, where the oracle can reproduce the stage's random integers:
prefixes of each output (the Philox index of an element is its linear output
index, so an output prefix is the oracle's whole output of the input
prefix).

- the SR quantisers of dY2 and dH1: their first 256 rows, bit-exact;
- the per-expert requantisations of W2 and W1 to the stacks of W_e^T: the
  first two experts, bit-exact;
- the segment-wise transposes dY2^T and dH1^T (one outer scale per segment
  and row): their first 64 rows, bit-exact;
- the NVFP4 dgrad of the second GEMM on sampled outputs, and its wgrad for
  the first non-empty expert, against fp64 sums of the decoded operands.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_moe_numerics_b200 import api, workloads
from fp8_moe_numerics_b200.layer import ExpertLayer
from tests.test_gpu_fullsize import MOE, _close_bf16, mma_rows, np_, u16

pytestmark = pytest.mark.gpu


def _nv_rows(q, rows, cols):
    """Codes, row-major scales and outer scales of `rows` of an NVFP4 triple with MMA scales."""
    r = np.asarray(rows, dtype=np.int64)
    return np_(q[0][torch.from_numpy(r).cuda()]), mma_rows(np_(q[1]), r, cols // 16), np_(q[2])


def test_moe_layer_nvfp4_backward_full_size(cuda):
    T, k, E, D, F = MOE["T"], MOE["k"], MOE["E"], MOE["D"], MOE["F"]
    N1 = 2 * F
    inp = workloads.layer_inputs("moe_layer", device="cuda")
    L = ExpertLayer(inp["x"], inp["topk"].cuda(), inp["w_comb"].cuda(), inp["w1"], inp["w2"], inp["dout"],
                    gated=True, seed=2024, backward="nvfp4")
    L.step()
    api.sync_status()
    seed, R, M = L.seed, L.rbits, L.M_cap
    seg = np_(L.seg)

    # the SR quantisers (per-row outer scales), first 256 rows of dY2 (stream 11) and dH1 (stream 15)
    for name, g, q, cols, stream in (("dy2", L.dy2, L.dy2n, D, 11), ("dh1", L.dh1, L.dh1n, N1, 15)):
        rows = np.arange(256)
        ref = oracle.nvfp4_quantize_f32(oracle.bf16_to_f32(u16(g[:256])), 1, True, seed, stream, R)
        got = _nv_rows(q, rows, cols)
        assert np.array_equal(got[0], ref[0]), name
        assert np.array_equal(got[1], ref[1]), name
        assert np.array_equal(got[2][:256].view(np.uint32), ref[2].view(np.uint32)), name

    # the per-expert requantisations to the stacks of W_e^T, experts 0 and 1 (W2: stream 12, W1: stream 16)
    for name, wq, wt, n_rows, cols, stream in (("w2", L.w2q, L.w2tn, D, F, 12), ("w1", L.w1q, L.w1tn, N1, D, 16)):
        src = _nv_rows(wq, np.arange(2 * n_rows), cols)
        ref = oracle.nvfp4_requant_transpose_experts_sr(src[0], src[1], src[2][:2], 2, seed, stream, R)
        got = _nv_rows(wt, np.arange(2 * cols), n_rows)
        assert np.array_equal(got[0], ref[0]), name
        assert np.array_equal(got[1], ref[1]), name
        assert np.array_equal(got[2][:2].view(np.uint32), ref[2].view(np.uint32)), name

    # the segment-wise transposes with one outer scale per (segment, row): first 64 rows of dY2^T (stream 13)
    # and dH1^T (stream 17), from the GPU's bf16 gradients
    for name, g, q, cols, stream in (("dy2t", L.dy2, L.dy2tn, D, 13), ("dh1t", L.dh1, L.dh1tn, N1, 17)):
        x = oracle.bf16_to_f32(u16(g[:, :64]))
        ref = oracle.nvfp4_quantize_transpose_segments(x, seg, True, True, seed, stream, R)
        got = _nv_rows(q, np.arange(64), M)
        assert np.array_equal(got[0], ref[0]), name
        assert np.array_equal(got[1], ref[1]), name
        outer = np_(q[2]).reshape(E, cols)[:, :64]
        assert np.array_equal(outer.view(np.uint32), ref[2].view(np.uint32)), name

    # the NVFP4 dgrad of GEMM2 (dA = dY2 W2 through the forward GEMM, B = the stack of W2_e^T): sampled outputs
    rng = np.random.default_rng(5)
    rows = rng.integers(0, int(seg[E]), 256)
    cols = rng.integers(0, F, 256)
    ex = np.searchsorted(seg, rows, side="right") - 1
    a = _nv_rows(L.dy2n, rows, D)
    b = _nv_rows(L.w2tn, ex * F + cols, D)
    ref = (np.sum(oracle.nvfp4_block_values(a[0], a[1]) * oracle.nvfp4_block_values(b[0], b[1]), axis=1) *
           a[2][rows].astype(np.float64) * b[2][ex].astype(np.float64))
    got = oracle.bf16_to_f32(u16(L.da[torch.from_numpy(rows).cuda(), torch.from_numpy(cols).cuda()])).astype(np.float64)
    assert _close_bf16(got, ref)

    # the NVFP4 wgrad of GEMM2 for the first non-empty expert: dW2_e = dY2_e^T A_e over its token segment
    e = int(np.argmax(np.diff(seg) > 0))
    t0, t1 = int(seg[e]), int(seg[e + 1])

    def seg_cols(q, n_rows):
        # the expert's token columns of a transposed operand [n_rows, M]: codes sliced on the device
        codes = np_(q[0][:, t0 // 2:t1 // 2])
        sf = mma_rows(np_(q[1]), np.arange(n_rows), M // 16)[:, t0 // 16:t1 // 16]
        return codes, sf, np_(q[2])

    A = seg_cols(L.dy2tn, D)                                   # dY2^T, outer [E, D]
    B = seg_cols(L.atn, F)                                     # a^T, outer [E]
    seg_e = np.array([0, t1 - t0], dtype=np.int64)
    ref = oracle.grouped_gemm_nvfp4_wgrad(A[0], A[1], A[2].reshape(E, D)[e:e + 1], B[0], B[1], B[2][e:e + 1],
                                          seg_e)[0]
    got = oracle.bf16_to_f32(u16(L.dw2[e])).astype(np.float64)
    assert _close_bf16(got, ref)
