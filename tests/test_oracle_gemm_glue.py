"""Pins for the oracle's fp64 grouped GEMMs and the expert-layer glue.

GEMMs are checked against brute-force Python loops over operands decoded by
ml_dtypes (an independent decoder), against plain matmuls in special cases,
and on empty experts.  The routing permutation is checked against a sort,
SiLU against torch, combine against loops.
"""
import ml_dtypes
import numpy as np
import torch


def _q_nvfp4(orc, rows, cols, seed, group_rows=1):
    rng = np.random.default_rng(seed)
    x = orc.f32_to_bf16((rng.standard_normal((rows, cols)) * 10.0 ** rng.uniform(-2, 2, (rows, 1))).astype(np.float32))
    return orc.nvfp4_quantize(x, group_rows=group_rows)


def _decode_nvfp4_ml(codes, sf):
    lo = (codes & 15).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (codes >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    q = np.empty((codes.shape[0], codes.shape[1] * 2))
    q[:, 0::2], q[:, 1::2] = lo, hi
    s = sf.view(ml_dtypes.float8_e4m3fn).astype(np.float64).repeat(16, axis=1)
    return q * s


def _decode_mxfp8_ml(codes, e8):
    return codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64) * \
        e8.view(ml_dtypes.float8_e8m0fnu).astype(np.float64).repeat(32, axis=1)


def test_grouped_gemm_nvfp4_brute_force(orc):
    E, N, K = 3, 8, 32
    seg = np.array([0, 4, 4, 10], dtype=np.int64)          # expert 1 empty
    a = _q_nvfp4(orc, 12, K, 1)
    b = _q_nvfp4(orc, E * N, K, 2, group_rows=N)
    C = orc.grouped_gemm_nvfp4(*a, *b, seg, N)
    A = _decode_nvfp4_ml(a[0], a[1])
    B = _decode_nvfp4_ml(b[0], b[1])
    for r in range(12):
        owner = [i for i in range(E) if seg[i] <= r < seg[i + 1]]
        for n in range(N):
            if not owner:
                assert C[r, n] == 0.0
                continue
            e = owner[0]
            acc = 0.0
            for kk in range(K):
                acc += A[r, kk] * B[e * N + n, kk]
            ref = acc * float(a[2][r]) * float(b[2][e])
            assert abs(C[r, n] - ref) <= 1e-12 * max(1.0, abs(ref))
    s = orc.grouped_gemm_nvfp4_sampled(*a, *b, seg, N, [0, 5, 11, 9], [1, 7, 0, 3])
    assert np.allclose(s, C[[0, 5, 11, 9], [1, 7, 0, 3]], rtol=1e-13, atol=0)


def test_grouped_gemm_nvfp4_single_expert_is_plain_matmul(orc):
    N, K, M = 16, 64, 8
    a = _q_nvfp4(orc, M, K, 3)
    b = _q_nvfp4(orc, N, K, 4, group_rows=N)
    C = orc.grouped_gemm_nvfp4(*a, *b, np.array([0, M]), N)
    Ad = orc.nvfp4_dequantize(*a).astype(np.float64)
    Bd = orc.nvfp4_dequantize(*b, group_rows=N).astype(np.float64)
    assert np.allclose(C, Ad @ Bd.T, rtol=1e-6, atol=1e-30)


def test_grouped_gemm_mxfp8_dgrad_and_wgrad_brute_force(orc):
    rng = np.random.default_rng(5)
    E, Kc, Nout = 2, 32, 8
    seg = np.array([0, 0, 64], dtype=np.int64)             # expert 0 empty
    M = 64
    a_c, a_e = orc.mxfp8_quantize_rows(orc.f32_to_bf16(rng.standard_normal((M, Kc)).astype(np.float32)))
    b_c, b_e = orc.mxfp8_quantize_rows(orc.f32_to_bf16(rng.standard_normal((Nout, E * Kc)).astype(np.float32)))
    C = orc.grouped_gemm_mxfp8_dgrad(a_c, a_e, b_c, b_e, seg)
    A, B = _decode_mxfp8_ml(a_c, a_e), _decode_mxfp8_ml(b_c, b_e)
    for r in range(M):
        for n in range(Nout):
            ref = sum(A[r, k] * B[n, 1 * Kc + k] for k in range(Kc))
            assert abs(C[r, n] - ref) <= 1e-12 * max(1, abs(ref))
    # WGRAD: A [Nw, M], B [Kw, M]
    Nw, Kw = 4, 6
    wa_c, wa_e = orc.mxfp8_quantize_cols(orc.f32_to_bf16(rng.standard_normal((M, Nw)).astype(np.float32)))
    wb_c, wb_e = orc.mxfp8_quantize_cols(orc.f32_to_bf16(rng.standard_normal((M, Kw)).astype(np.float32)))
    W = orc.grouped_gemm_mxfp8_wgrad(wa_c, wa_e, wb_c, wb_e, seg)
    assert np.all(W[0] == 0)                               # empty expert -> zeros
    WA, WB = _decode_mxfp8_ml(wa_c, wa_e), _decode_mxfp8_ml(wb_c, wb_e)
    for n in range(Nw):
        for k in range(Kw):
            ref = sum(WA[n, t] * WB[k, t] for t in range(64))
            assert abs(W[1, n, k] - ref) <= 1e-12 * max(1, abs(ref))


def test_grouped_gemm_mxfp8_experts_past_the_first_segment(orc):
    # two non-empty experts around an empty one, the later one 1000x larger:
    # each expert's operands and scales sit at its own token or column offset
    rng = np.random.default_rng(15)
    E, Kc, Nout, Nw, Kw = 3, 64, 8, 4, 6
    seg = np.array([0, 64, 64, 160], dtype=np.int64)
    M = 160
    mag = np.where(np.arange(M) >= 64, 1000.0, 1.0)[:, None]
    a_c, a_e = orc.mxfp8_quantize_rows(orc.f32_to_bf16((rng.standard_normal((M, Kc)) * mag).astype(np.float32)))
    bw = rng.standard_normal((Nout, E * Kc)) * np.repeat([1.0, 7.0, 1000.0], Kc)[None, :]
    b_c, b_e = orc.mxfp8_quantize_rows(orc.f32_to_bf16(bw.astype(np.float32)))
    C = orc.grouped_gemm_mxfp8_dgrad(a_c, a_e, b_c, b_e, seg)
    A, B = _decode_mxfp8_ml(a_c, a_e), _decode_mxfp8_ml(b_c, b_e)
    for r in range(M):
        e = 0 if r < 64 else 2
        for n in range(Nout):
            ref = sum(A[r, k] * B[n, e * Kc + k] for k in range(Kc))
            assert abs(C[r, n] - ref) <= 1e-12 * max(1, abs(ref))
    wa_c, wa_e = orc.mxfp8_quantize_cols(orc.f32_to_bf16((rng.standard_normal((M, Nw)) * mag).astype(np.float32)))
    wb_c, wb_e = orc.mxfp8_quantize_cols(orc.f32_to_bf16(rng.standard_normal((M, Kw)).astype(np.float32)))
    W = orc.grouped_gemm_mxfp8_wgrad(wa_c, wa_e, wb_c, wb_e, seg)
    assert np.all(W[1] == 0)
    WA, WB = _decode_mxfp8_ml(wa_c, wa_e), _decode_mxfp8_ml(wb_c, wb_e)
    for e, (t0, t1) in ((0, (0, 64)), (2, (64, 160))):
        for n in range(Nw):
            for k in range(Kw):
                ref = sum(WA[n, t] * WB[k, t] for t in range(t0, t1))
                assert abs(W[e, n, k] - ref) <= 1e-12 * max(1, abs(ref))


def test_gather_puts_each_token_at_its_routed_rows(orc):
    # after routing, row pos[t, j] of the gathered tensor is token t's
    # quantised row, bit for bit (codes, block scales, outer scale) and so
    # decodes to the same values; every other row is a zero padding row
    rng = np.random.default_rng(17)
    T, k, E, cols = 40, 3, 5, 64
    topk = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    seg, src, pos = orc.route(topk, E)
    codes, sf, outer = _q_nvfp4(orc, T, cols, 18)
    gc, gsf, go = orc.gather_nvfp4_rows(codes, sf, outer, src)
    assert gc.shape == (int(seg[-1]), cols // 2) and gsf.shape == (int(seg[-1]), cols // 16)
    used = np.zeros(int(seg[-1]), bool)
    for t in range(T):
        for j in range(k):
            p = int(pos[t, j])
            used[p] = True
            assert np.array_equal(gc[p], codes[t]) and np.array_equal(gsf[p], sf[t]) and go[p] == outer[t]
    assert np.all(gc[~used] == 0) and np.all(gsf[~used] == 0) and np.all(go[~used] == 0)
    deq = orc.nvfp4_dequantize(gc, gsf, go)
    assert np.array_equal(deq[pos.reshape(-1)], orc.nvfp4_dequantize(codes, sf, outer)[np.repeat(np.arange(T), k)])


def test_integer_exact_gemm_case(orc):
    # Power-of-two scales and small integer products: the fp64 sum is exact.
    E, N, K, M = 1, 4, 64, 4
    codes = np.full((M, K // 2), 0x22, np.uint8)           # all elements 1.0
    sf = np.full((M, K // 16), 0x38, np.uint8)             # 1.0
    outer = np.ones(M, np.float32)
    C = orc.grouped_gemm_nvfp4(codes, sf, outer, codes[:N], sf[:N], np.ones(1, np.float32),
                               np.array([0, M]), N)
    assert np.all(C == K)


def test_route_matches_stable_sort(orc):
    rng = np.random.default_rng(6)
    T, k, E = 50, 3, 7
    ids = np.stack([rng.choice([0, 1, 2, 3, 5, 6], k, replace=False) for _ in range(T)]).astype(np.int32)
    seg, src, pos = orc.route(ids, E, align=8)
    counts = np.bincount(ids.ravel(), minlength=E)
    assert counts[4] == 0 and seg[5] == seg[4]             # empty expert: empty segment
    pad = (counts + 7) // 8 * 8
    assert np.array_equal(np.diff(seg), pad)
    flat_t = np.repeat(np.arange(T), k)
    flat_e = ids.ravel()
    order = np.lexsort((flat_t, flat_e))                   # by expert, then token
    for e in range(E):
        toks = flat_t[order][flat_e[order] == e]
        assert np.array_equal(src[seg[e]:seg[e] + len(toks)], toks)
        assert np.all(src[seg[e] + len(toks):seg[e + 1]] == -1)
    for t in range(T):
        for j in range(k):
            p = pos[t, j]
            assert src[p] == t and seg[ids[t, j]] <= p < seg[ids[t, j] + 1]


def test_silu_swiglu_against_torch(orc):
    rng = np.random.default_rng(7)
    h = orc.f32_to_bf16(rng.standard_normal((5, 16)).astype(np.float32) * 4)
    hf = torch.from_numpy(orc.bf16_to_f32(h).astype(np.float64))
    a = orc.bf16_to_f32(orc.swiglu_fwd(h, gated=True)).astype(np.float64)
    ref = torch.nn.functional.silu(hf[:, :8]) * hf[:, 8:]
    assert np.allclose(a, ref.numpy(), rtol=2 ** -8, atol=0)
    a2 = orc.bf16_to_f32(orc.swiglu_fwd(h, gated=False)).astype(np.float64)
    assert np.allclose(a2, torch.nn.functional.silu(hf).numpy(), rtol=2 ** -8, atol=0)
    # backward: autograd of the same expression
    da = orc.f32_to_bf16(rng.standard_normal((5, 8)).astype(np.float32))
    daf = torch.from_numpy(orc.bf16_to_f32(da).astype(np.float64))
    hv = hf.clone().requires_grad_(True)
    (torch.nn.functional.silu(hv[:, :8]) * hv[:, 8:] * daf).sum().backward()
    dh = orc.bf16_to_f32(orc.swiglu_bwd(h, da, gated=True)).astype(np.float64)
    assert np.allclose(dh, hv.grad.numpy(), rtol=2 ** -8, atol=1e-30)
    # ungated backward: autograd of silu(h)
    da1 = orc.f32_to_bf16(rng.standard_normal((5, 16)).astype(np.float32))
    hv1 = hf.clone().requires_grad_(True)
    (torch.nn.functional.silu(hv1) * torch.from_numpy(orc.bf16_to_f32(da1).astype(np.float64))).sum().backward()
    dh1 = orc.bf16_to_f32(orc.swiglu_bwd(h, da1, gated=False)).astype(np.float64)
    assert np.allclose(dh1, hv1.grad.numpy(), rtol=2 ** -8, atol=1e-30)
    assert orc.bf16_to_f32(orc.swiglu_fwd(orc.f32_to_bf16(np.zeros((1, 2), np.float32)), True))[0, 0] == 0


def test_f64_to_bf16_single_rounding(orc):
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -8 + 2 ** -30, -2.5, 0.0], np.float64)
    got = orc.bf16_to_f32(orc.f64_to_bf16(x))
    assert list(got) == [1.0, 1.0 + 2 ** -6, 1.0 + 2 ** -7, -2.5, 0.0]


def test_combine_and_dispatch_grad_loops(orc):
    rng = np.random.default_rng(8)
    T, k, E = 6, 2, 3
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    seg, src, pos = orc.route(ids, E, align=4)
    M = int(seg[-1])
    y = orc.f32_to_bf16(rng.standard_normal((M, 8)).astype(np.float32))
    w = np.full((T, k), 0.5, np.float32)
    out = orc.bf16_to_f32(orc.combine(y, pos, w))
    yf = orc.bf16_to_f32(y).astype(np.float64)
    for t in range(T):
        ref = sum(0.5 * yf[pos[t, j]] for j in range(k))
        assert np.allclose(out[t], ref, rtol=2 ** -8)
    d = orc.f32_to_bf16(rng.standard_normal((T, 8)).astype(np.float32))
    dy = orc.bf16_to_f32(orc.dispatch_grad(d, pos, w, M))
    df = orc.bf16_to_f32(d)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(dy[pos[t, j]], (0.5 * df[t]).astype(np.float32))
    assert np.all(dy[src < 0] == 0)
