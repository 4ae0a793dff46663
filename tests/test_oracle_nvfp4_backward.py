"""Pins of the oracle for NVFP4 in the backward pass and the 16x16 tile scale.

[ai-primer §NVFP4 forward, MXFP8 backward]: four-bit arithmetic in the
backward pass is the lab's stated future work.  [ai-primer §Stochastic
rounding across transposes]: quantising the two orientations of a tensor
independently changes the represented values; a scale shared by each 16x16
tile avoids that but lets one large value force the tile's others to zero;
after regrouping, a represented 4.5 becomes 4 with probability 0.75 and 6 with
0.25, keeping its expectation.

Each pin checks the oracle against something other than itself: the pinned
forward quantiser, ml_dtypes' independent E2M1/E4M3 decoding, brute-force
neighbours on the E2M1 grid, the pages' regrouping example on a tensor whose
every value is exactly representable, expectations over many random streams,
brute-force GEMM sums, and the pages' outlier statement.
"""
import ml_dtypes
import numpy as np
import pytest

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e2m1_values(codes):
    """Element values (code units) of packed E2M1 codes, decoded by ml_dtypes."""
    lo = (codes & 15).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (codes >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def _e4m3(sf):
    return np.asarray(sf, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def _rand_bf16_values(orc, rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_t(4, (rows, cols)) * 10.0 ** rng.uniform(-2, 2, (rows, 1))).astype(np.float32)
    return orc.bf16_to_f32(orc.f32_to_bf16(x))


def test_fp32_quantiser_without_sr_equals_the_forward_quantiser(orc):
    x = _rand_bf16_values(orc, 64, 128, 1)
    for g in (1, 32):
        a = orc.nvfp4_quantize(orc.f32_to_bf16(x), group_rows=g)
        b = orc.nvfp4_quantize_f32(x, group_rows=g)
        for u, v in zip(a, b):
            assert np.array_equal(u, v)


def test_sr_keeps_the_scales_and_picks_a_grid_neighbour(orc):
    x = _rand_bf16_values(orc, 32, 128, 2)
    c0, sf0, o0 = orc.nvfp4_quantize_f32(x)
    c1, sf1, o1 = orc.nvfp4_quantize_f32(x, sr=True, seed=5, stream=9, R=16)
    assert np.array_equal(sf0, sf1) and np.array_equal(o0, o1)
    # y = x / (sf s) in fp32 as the quantiser forms it; each SR code is one of
    # the two E2M1 magnitudes around |y| (|y| itself when it is on the grid)
    den = (np.repeat(_e4m3(sf1), 16, axis=1).astype(np.float32) * o1[:, None]).astype(np.float32)
    ok = den > 0
    y = np.zeros_like(x)
    y[ok] = x[ok] * (np.float32(1.0) / den[ok])
    got = np.abs(_e2m1_values(c1))
    ay = np.minimum(np.abs(y.astype(np.float64)), 6.0)
    lo = np.array([E2M1_GRID[E2M1_GRID <= v].max() for v in ay.reshape(-1)]).reshape(ay.shape)
    hi = np.array([E2M1_GRID[E2M1_GRID >= v].min() for v in ay.reshape(-1)]).reshape(ay.shape)
    assert np.all((got == lo) | (got == hi))
    assert np.all(got[lo == hi] == lo[lo == hi])
    assert np.all(np.signbit(_e2m1_values(c1)[got > 0]) == np.signbit(x[got > 0]))
    assert 0 < np.mean(got != np.abs(_e2m1_values(c0))) < 0.5


def _worked_example_row():
    # s = 10.5 / 2688 = 2^-8; block 1 holds 6 (scale 256, so sf s = 1) and 4.5
    x = np.zeros((1, 32), np.float32)
    x[0, 0] = 10.5
    x[0, 16], x[0, 17] = 6.0, 4.5
    return x


def test_worked_example_4_5_in_the_quantiser(orc):
    # [ai-primer §Stochastic rounding across transposes]: 4.5 -> 4 (p = 0.75) or 6 (p = 0.25)
    x = _worked_example_row()
    c, sf, o = orc.nvfp4_quantize_f32(x)
    assert o[0] == 2.0 ** -8 and _e4m3(sf)[0, 1] == 256.0
    assert _e2m1_values(c)[0, 17] == 4.0                      # nearest even: always down
    n = 4000
    v = np.array([_e2m1_values(orc.nvfp4_quantize_f32(x, sr=True, seed=7, stream=s, R=8)[0])[0, 17]
                  for s in range(n)])
    assert set(np.unique(v)) == {4.0, 6.0}
    p6 = np.mean(v == 6.0)
    assert abs(p6 - 0.25) < 4 * np.sqrt(0.25 * 0.75 / n)
    assert abs(v.mean() - 4.5) < 4 * 2 * np.sqrt(0.25 * 0.75 / n)


def _regroup_tensor():
    """Forward [32, 32] whose every value is exactly representable per token:
    row 0 = 4.5 (code 3 under block scale 384), 9 and 10.5; row 1 = 6 and 10.5;
    row 16 = 10.5.  Its column 0, the transpose's row 0, is [4.5, 6, 0.., 10.5, 0..]."""
    x = np.zeros((32, 32), np.float32)
    x[0, 0], x[0, 1], x[0, 16] = 4.5, 9.0, 10.5
    x[1, 0], x[1, 16] = 6.0, 10.5
    x[16, 0] = 10.5
    return x


def test_regrouping_example_across_the_transpose(orc):
    # the pages' illustration at the requantisation: a represented 4.5 lands
    # between 4 and 6 on the transposed grid and keeps its expectation
    x = _regroup_tensor()
    q = orc.nvfp4_quantize(orc.f32_to_bf16(x))
    assert np.array_equal(orc.nvfp4_dequantize(*q), x)       # every value represented exactly
    assert _e2m1_values(q[0])[0, 0] == 3.0 and _e4m3(q[1])[0, 0] == 384.0
    c, sf, o = orc.nvfp4_requant_transpose_sr(*q, 1, seed=3, stream=0, sr=False)
    assert o[0] == 2.0 ** -8 and _e4m3(sf)[0, 0] == 256.0 and _e2m1_values(c)[0, 0] == 4.0   # RNE: biased down
    n = 4000
    v = np.array([orc.nvfp4_dequantize(*orc.nvfp4_requant_transpose_sr(*q, 1, seed=3, stream=s, R=8))[0, 0]
                  for s in range(n)])
    assert set(np.unique(v)) == {4.0, 6.0}
    assert abs(np.mean(v == 6.0) - 0.25) < 4 * np.sqrt(0.25 * 0.75 / n)


def test_requantisation_is_unbiased_over_streams(orc):
    rows, cols = 32, 48
    q = orc.nvfp4_quantize(orc.f32_to_bf16(_rand_bf16_values(orc, rows, cols, 4)))
    xt = orc.nvfp4_dequantize(*q).T.astype(np.float64)          # the transposed forward values
    S = 600
    acc = np.zeros((cols, rows))
    for s in range(S):
        c, sf, o = orc.nvfp4_requant_transpose_sr(*q, 1, seed=11, stream=s, R=16)
        acc += orc.nvfp4_dequantize(c, sf, o).astype(np.float64)
    _, sf, o = orc.nvfp4_requant_transpose_sr(*q, 1, seed=11, stream=0, R=16)   # scales do not depend on the stream
    den = np.repeat(_e4m3(sf), 16, axis=1) * o.astype(np.float64)[:, None]
    ay = np.abs(xt) / np.where(den > 0, den, 1)
    step = np.where(ay < 2, 0.5, np.where(ay < 4, 1.0, 2.0)) * den           # E2M1 spacing at each value
    # a block scale rounded down can leave the block's largest value a little
    # past 6 code units; the format saturates there, so its expectation is 6
    assert np.any(ay > 6)
    want = np.sign(xt) * np.minimum(ay, 6.0) * den
    # mean of S draws within 5 standard deviations (<= step/2 each) plus the
    # 2^-R bias of the discrete rule and the fp32 rounding of each decoded value
    tol = 5 * step / (2 * np.sqrt(S)) + step * 2.0 ** -16 + np.abs(xt) * 2.0 ** -22
    assert np.all(np.abs(acc / S - want) <= tol)


def test_expert_weight_requant_is_per_expert(orc):
    E, N, K = 3, 32, 64
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((E, N, K)) * np.array([1.0, 50.0, 0.01])[:, None, None]).astype(np.float32)
    q = orc.nvfp4_quantize(orc.f32_to_bf16(w.reshape(E * N, K)), group_rows=N)
    wd = orc.nvfp4_dequantize(*q, group_rows=N).reshape(E, N, K)
    c, sf, o = orc.nvfp4_requant_transpose_experts_sr(*q, E, seed=1, stream=2, sr=False)
    assert c.shape == (E * K, N // 2) and o.shape == (E,)
    for e in range(E):
        assert o[e] == np.float32(np.abs(wd[e]).max()) / np.float32(2688.0)
        one = orc.nvfp4_quantize_f32(np.ascontiguousarray(wd[e].T), K)
        assert np.array_equal(c[e * K:(e + 1) * K], one[0]) and np.array_equal(sf[e * K:(e + 1) * K], one[1])
    # the requantised stack decodes to each W_e^T within NVFP4's block error
    back = orc.nvfp4_dequantize(c, sf, o, group_rows=K).reshape(E, K, N).astype(np.float64)
    for e in range(E):
        ref = wd[e].T.astype(np.float64)
        blk = np.abs(ref).reshape(K, N // 16, 16).max(-1, keepdims=True)
        assert np.all(np.abs(back[e] - ref).reshape(K, N // 16, 16) <= blk / 4 + 1e-30)


def test_segment_transpose_with_one_segment_is_the_row_quantiser(orc):
    # one segment over all tokens: per (segment, row) is the per-row quantiser
    # of the transpose, per segment the per-tensor one, random indices included
    x = _rand_bf16_values(orc, 64, 48, 13)
    seg = np.array([0, 64])
    for per_row, g in ((True, 1), (False, 48)):
        c, sf, o = orc.nvfp4_quantize_transpose_segments(x, seg, per_row, True, 4, 7, 16)
        rc, rsf, ro = orc.nvfp4_quantize_f32(np.ascontiguousarray(x.T), g, True, 4, 7, 16)
        assert np.array_equal(c, rc) and np.array_equal(sf, rsf) and np.array_equal(o.reshape(-1), ro)


def test_segment_outer_scales_closed_form_and_padding(orc):
    rng = np.random.default_rng(14)
    M, C = 160, 32
    seg = np.array([0, 64, 64, 128])                             # expert 1 empty; rows 128.. are padding
    x = (rng.standard_normal((M, C)) * np.where(np.arange(M) < 64, 1.0, 40.0)[:, None]).astype(np.float32)
    a, sa, oa = orc.nvfp4_quantize_transpose_segments(x, seg, True, sr=False)
    b, sb, ob = orc.nvfp4_quantize_transpose_segments(x, seg, False, sr=False)
    assert oa.shape == (3, C) and ob.shape == (3,)
    for e, (t0, t1) in ((0, (0, 64)), (2, (64, 128))):
        assert np.array_equal(oa[e], np.abs(x[t0:t1]).max(axis=0).astype(np.float32) / np.float32(2688.0))
        assert ob[e] == np.float32(np.abs(x[t0:t1]).max()) / np.float32(2688.0)
    assert np.all(oa[1] == 0) and ob[1] == 0
    for codes, sf in ((a, sa), (b, sb)):
        assert np.all(codes[:, 128 // 2:] == 0) and np.all(sf[:, 128 // 16:] == 0)
    # decoded values within NVFP4's block error of the transposed input
    for codes, sf, outer_of in ((a, sa, lambda e: oa[e][:, None]), (b, sb, lambda e: ob[e])):
        v = _e2m1_values(codes) * np.repeat(_e4m3(sf), 16, axis=1)
        for e, (t0, t1) in ((0, (0, 64)), (2, (64, 128))):
            got = v[:, t0:t1] * outer_of(e)
            ref = x[t0:t1].T.astype(np.float64)
            blk = np.abs(ref).reshape(C, -1, 16).max(-1, keepdims=True)
            assert np.all(np.abs(got - ref).reshape(C, -1, 16) <= blk / 4 + 1e-30)


def test_nvfp4_wgrad_brute_force(orc):
    rng = np.random.default_rng(8)
    E, Nw, Kw = 3, 4, 5
    seg = np.array([0, 64, 64, 160], dtype=np.int64)            # expert 1 empty
    M = 160
    mag = np.where(np.arange(M) >= 64, 300.0, 1.0)[:, None]
    dy = (rng.standard_normal((M, Nw)) * mag).astype(np.float32)
    x = (rng.standard_normal((M, Kw)) * mag[::-1]).astype(np.float32)
    a = orc.nvfp4_quantize_transpose_segments(dy, seg, True, True, 1, 2, 16)     # dY^T, per (segment, row)
    b = orc.nvfp4_quantize_transpose_segments(x, seg, False, True, 1, 3, 16)     # X^T, per segment
    C = orc.grouped_gemm_nvfp4_wgrad(*a, *b, seg)
    A = _e2m1_values(a[0]) * np.repeat(_e4m3(a[1]), 16, axis=1)
    B = _e2m1_values(b[0]) * np.repeat(_e4m3(b[1]), 16, axis=1)
    assert np.all(C[1] == 0)
    for e, (t0, t1) in ((0, (0, 64)), (2, (64, 160))):
        for n in range(Nw):
            for k in range(Kw):
                ref = float(a[2][e, n]) * float(b[2][e]) * sum(A[n, t] * B[k, t] for t in range(t0, t1))
                assert abs(C[e, n, k] - ref) <= 1e-12 * max(1e-30, abs(ref))
    # and close to the unquantised product (SR noise over 64-96 tokens)
    for e, (t0, t1) in ((0, (0, 64)), (2, (64, 160))):
        exact = dy[t0:t1].T.astype(np.float64) @ x[t0:t1].astype(np.float64)
        assert np.linalg.norm(C[e] - exact) <= 0.2 * np.linalg.norm(exact)


def test_nvfp4_dgrad_is_the_forward_gemm_with_transposed_weights(orc):
    rng = np.random.default_rng(9)
    E, N, K, M = 2, 32, 64, 256
    seg = np.array([0, 128, 256], dtype=np.int64)
    w = orc.nvfp4_quantize(orc.f32_to_bf16((rng.standard_normal((E * N, K)) * 0.02).astype(np.float32)), N)
    wt = orc.nvfp4_requant_transpose_experts_sr(*w, E, seed=2, stream=5)
    dy = orc.nvfp4_quantize_f32(rng.standard_normal((M, N)).astype(np.float32), 1, True, 3, 6, 16)
    dx = orc.grouped_gemm_nvfp4(*dy, *wt, seg, K)             # [M, K]
    Dy = _e2m1_values(dy[0]) * np.repeat(_e4m3(dy[1]), 16, axis=1) * dy[2].astype(np.float64)[:, None]
    Wt = (_e2m1_values(wt[0]) * np.repeat(_e4m3(wt[1]), 16, axis=1)).reshape(E, K, N) \
        * wt[2].astype(np.float64)[:, None, None]
    for r in (0, 77, 128, 255):
        e = 0 if r < 128 else 1
        for k in (0, 13, 63):
            ref = sum(Dy[r, n] * Wt[e, k, n] for n in range(N))
            assert abs(dx[r, k] - ref) <= 1e-12 * max(1e-30, abs(ref))


def test_tile16_outlier_forces_the_rest_of_its_tile_to_zero(orc):
    # the pages' reason for rejecting the 16x16 shared scale
    rng = np.random.default_rng(10)
    x = rng.uniform(0.5, 1.0, (16, 16)).astype(np.float32)
    x[3, 7] = 4096.0
    c, sf, o = orc.nvfp4_quantize_tile16(x, group_rows=16)
    v = _e2m1_values(c)
    assert v[3, 7] == 6.0 and np.count_nonzero(v) == 1
    # 1x16 blocks under the same outer scale keep every row without the outlier
    cb, sfb, ob = orc.nvfp4_quantize_f32(x, group_rows=16)
    deq = orc.nvfp4_dequantize(cb, sfb, ob, 16)
    others = np.arange(16) != 3
    assert np.all(deq[others] != 0)
    assert np.all(np.abs(deq[others] - x[others]) <= 0.25 * x[others].max(axis=1, keepdims=True))


def test_tile16_codes_are_the_same_in_both_orientations(orc):
    x = _rand_bf16_values(orc, 64, 48, 12)
    c, sf, o = orc.nvfp4_quantize_tile16(x, group_rows=64)
    ct, sft = orc.nvfp4_tile16_transpose(c, sf)
    c2, sf2, o2 = orc.nvfp4_quantize_tile16(np.ascontiguousarray(x.T), group_rows=48)
    assert np.array_equal(ct, c2) and np.array_equal(sft, sf2) and o[0] == o2[0]
    d = orc.nvfp4_tile16_dequantize(c, sf, o, 64)
    assert np.array_equal(orc.nvfp4_tile16_dequantize(c2, sf2, o2, 48), d.T)
    # 1x16 blocks: the two orientations represent some values differently
    a = orc.nvfp4_dequantize(*orc.nvfp4_quantize_f32(x, group_rows=64), group_rows=64)
    b = orc.nvfp4_dequantize(*orc.nvfp4_quantize_f32(np.ascontiguousarray(x.T), group_rows=48), group_rows=48)
    assert np.any(a != b.T)


def test_tile16_constant_tiles_closed_form(orc):
    # a constant tile of value v under outer scale s = gmax / 2688 gets the
    # E4M3 scale of v / (6 s) and codes of magnitude 6 (the grid top)
    x = np.repeat(np.repeat(np.array([[3.0, -0.75], [0.0, 12.0]], np.float32), 16, 0), 16, 1)
    c, sf, o = orc.nvfp4_quantize_tile16(x, group_rows=32)
    assert o[0] == np.float32(12.0) / np.float32(2688.0)
    v = _e2m1_values(c)
    assert np.all(np.abs(v[:16, :16]) == 6) and np.all(v[:16, 16:] == -6) and np.all(v[16:, :16] == 0)
    assert sf[1, 0] == 0 and _e4m3(sf)[1, 1] == 448.0
    d = orc.nvfp4_tile16_dequantize(c, sf, o, 32)
    assert np.allclose(d, x, rtol=2 ** -3, atol=0)
