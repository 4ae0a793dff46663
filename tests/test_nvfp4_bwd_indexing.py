"""Index arithmetic of the NVFP4-backward kernels (csrc/nvfp4_bwd.cu), checked
on the CPU before they run on a GPU.

Each kernel's launch grid and thread-to-element mapping is replayed here (the
formulas restated from the kernel source) over several shapes, scale layouts
and expert splits: every global read stays inside its buffer, every output
byte is written by exactly one thread, and every atomic target lies inside
the scale array.
"""
import numpy as np
import pytest

T = 256                                   # threads per block


def sf_offset(r, s, S, mma):
    """Scale byte of row r, block column s of an [R, S] scale array (MMA: 512-byte
    atoms of 128 rows x 4 columns)."""
    if not mma:
        return r * S + s
    return (((r >> 7) * (S >> 2) + (s >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (s & 3)


def _threads(items):
    grid = (items + T - 1) // T
    g = np.arange(grid * T, dtype=np.int64)
    return g[g < items]


def _exactly_once(starts, width, size):
    """Byte ranges [start, start + width) tile [0, size) with no overlap."""
    starts = np.sort(np.asarray(starts, np.int64))
    assert starts.min() >= 0 and starts.max() + width <= size
    assert len(starts) * width == size and np.all(np.diff(starts) == width)


def _group_amax_replay(rows, cols, group_rows, in_mma, block_rows, target_of_block, n_targets):
    """group_amax_nvfp4_kernel: block = 128 rows (skipped when target_of_block
    gives None), thread t = row r0 + t % 128, 64-value chunks k = t / 128,
    t / 128 + 2, ...: 32 code bytes and the 4 scale bytes of blocks 4k .. 4k + 3."""
    S = cols // 16
    t = np.arange(T)
    for r0 in block_rows:
        tg = target_of_block(r0)
        if tg is None:
            continue
        assert 0 <= tg < n_targets
        r = r0 + (t & 127)
        assert r.max() < rows and (r // group_rows).max() < rows // group_rows
        for k in range(cols // 64):
            rr = r[(t >> 7) == (k & 1)]
            co = rr * (cols // 2) + 32 * k
            assert co.min() >= 0 and (co + 32).max() <= rows * cols // 2 and np.all(co % 16 == 0)
            so = np.array([sf_offset(int(a), 4 * k, S, in_mma) for a in rr])
            assert so.min() >= 0 and (so + 4).max() <= rows * S and np.all(so % 4 == 0)
            # the 4 scale bytes of a chunk are blocks 4k .. 4k + 3 of the row, in order
            for a in rr[::37]:
                base = sf_offset(int(a), 4 * k, S, in_mma)
                assert [sf_offset(int(a), 4 * k + i, S, in_mma) for i in range(4)] == [base + i for i in range(4)]


def _requant_tile_replay(rows, cols, group_rows, in_mma, out_mma, live_of_tile, out_row_base, out_cols, n_out_rows,
                         bf16=False):
    """requant_nvfp4_tile_kernel: grid (cols / 64, rows / 128), 8 warps.
    Phase 1: lane (rho, b) of warp w loads rows r0 + 16w + 8g + rho (g = 0, 1):
    8 code bytes at column c0 + 16b, the row's 4 scale bytes of the tile.
    Phase 2: lane (m, jj, q) of warp w takes tile column c = 16 (m / 2) + 2w + m % 2
    and, for it = 0, 1, input rows 16j .. with j = 4 it + 2q + jj: 8 output code
    bytes at L0 / 2 (L0 = o * out_cols + n0 + 16j), and lane jj = q = 0 one scale
    word at block n0 / 16 + 4 it of output row o.  A bf16 source (bf16=True)
    loads in phase 1 16 bytes per lane instead: unit n of warp w is row
    r0 + 16w + 8 (n / 2) + rho, columns c0 + 16b + 8 (n % 2) .. + 7."""
    S = cols // 16
    codes_out, sf_words, L_all = [], [], []
    lane = np.arange(32)
    for by in range(rows // 128):
        r0 = by * 128
        live = live_of_tile(r0)
        n0, o_base = out_row_base(r0)
        for bx in range(cols // 64):
            c0 = bx * 64
            for w in range(8):
                if live and bf16:
                    rho, b = lane >> 2, lane & 3
                    seen = []
                    for n in range(4):
                        r = r0 + 16 * w + 8 * (n >> 1) + rho
                        xi = r * cols + c0 + 16 * b + 8 * (n & 1)
                        assert xi.min() >= 0 and (xi + 8).max() <= rows * cols and np.all(xi % 8 == 0)
                        seen.extend(xi.tolist())
                    # the warp's 16 rows x 64 columns, each element loaded once
                    rel = np.array(seen) - (r0 + 16 * w) * cols - c0
                    _exactly_once(rel // cols * 64 + rel % cols, 8, 16 * 64)
                elif live:
                    rho, b = lane >> 2, lane & 3
                    for g in range(2):
                        r = r0 + 16 * w + 8 * g + rho
                        co = r * (cols // 2) + c0 // 2 + 8 * b
                        assert co.min() >= 0 and (co + 8).max() <= rows * cols // 2 and np.all(co % 8 == 0)
                        so = np.array([sf_offset(int(a), c0 // 16, S, in_mma) for a in r])
                        assert so.min() >= 0 and (so + 4).max() <= rows * S
                        # the row's four scale bytes of the tile are consecutive
                        assert all(sf_offset(int(a), c0 // 16 + i, S, in_mma) == sf_offset(int(a), c0 // 16, S, in_mma)
                                   + i for a in r[:4] for i in range(4))
                        assert (r // group_rows).max() < rows // group_rows
                m, jj, q = lane & 7, (lane >> 3) & 1, lane >> 4
                c = 16 * (m >> 1) + 2 * w + (m & 1)
                o = o_base + c0 + c
                assert o.max() < n_out_rows
                for it in range(2):
                    j = 4 * it + 2 * q + jj
                    L0 = o * out_cols + n0 + 16 * j
                    codes_out.extend((L0 // 2).tolist())
                    L_all.append(L0)
                    lead = (jj == 0) & (q == 0)
                    nb = out_cols // 16
                    for a in o[lead]:
                        base = sf_offset(int(a), n0 // 16 + 4 * it, nb, out_mma)
                        assert base % 4 == 0
                        assert [sf_offset(int(a), n0 // 16 + 4 * it + i, nb, out_mma) for i in range(4)] == \
                            [base + i for i in range(4)]
                        sf_words.append(base)
                    # the word's bytes come from lanes ^ 8 and ^ 16 of the same output row, byte 2q + jj
                    for l in range(32):
                        assert c[l ^ 8] == c[l] and c[l ^ 16] == c[l]
    n_out = n_out_rows * out_cols
    _exactly_once(codes_out, 8, n_out // 2)
    _exactly_once(sf_words, 4, n_out // 16)
    L = np.concatenate(L_all)[:, None] + np.arange(16)[None, :]
    assert np.array_equal(np.sort(L.reshape(-1)), np.arange(n_out))


@pytest.mark.parametrize("rows,cols,group_rows,mma", [(128, 64, 1, True), (256, 128, 128, True), (48, 32, 16, False),
                                                      (16, 16, 1, False)])
def test_quantize_sr_kernel_indexing(rows, cols, group_rows, mma):
    assert cols % 16 == 0 and rows % group_rows == 0 and (not mma or (rows % 128 == 0 and cols % 64 == 0))
    # group_outer_kernel: block g reads uint4 words i < group_rows * cols / 8 of its group
    n = group_rows * cols // 8
    last = (rows // group_rows - 1) * group_rows * cols * 2 + (n - 1) * 16 + 16
    assert last <= rows * cols * 2 and (group_rows * cols) % 8 == 0
    # nvfp4_quantize_sr_kernel: one thread per 16-value block
    S = cols // 16
    item = _threads(rows * S)
    r, b = item // S, item % S
    x_start = (r * cols + b * 16) * 2
    assert x_start.min() >= 0 and x_start.max() + 32 <= rows * cols * 2 and np.all(x_start % 16 == 0)
    assert np.all(r // group_rows < rows // group_rows)
    _exactly_once((r * cols + b * 16) // 2, 8, rows * cols // 2)
    _exactly_once([sf_offset(int(a), int(c), S, mma) for a, c in zip(r, b)], 1, rows * S)


@pytest.mark.parametrize("rows,cols,group_rows,experts,per_expert,in_mma,out_mma", [
    (256, 128, 1, 1, 0, True, True),            # activations: one outer scale per output row
    (512, 128, 128, 4, 1, True, True),          # weight stack [E*N, K]: per-expert outer scale
    (384, 64, 1, 3, 1, False, False),
    (256, 192, 256, 1, 1, True, False),
])
def test_requant_kernels_indexing(rows, cols, group_rows, experts, per_expert, in_mma, out_mma):
    rpe = rows // experts
    # the shapes the entry point accepts
    assert rpe % 128 == 0 and cols % 64 == 0 and rows % group_rows == 0
    assert not in_mma or rows % 128 == 0
    assert not out_mma or ((experts * cols) % 128 == 0 and rpe % 64 == 0)
    assert per_expert or experts == 1
    S_in = cols // 16
    n_outer = experts if per_expert else experts * cols
    assert rows // 128 <= 65535
    for r0 in range(0, rows, 128):
        assert (r0 + 127) // rpe == r0 // rpe                 # a block never straddles two experts
    if per_expert:
        # pass 1, one outer scale per expert: group_amax_nvfp4_kernel, grid rows / 128
        _group_amax_replay(rows, cols, group_rows, in_mma, range(0, rows, 128), lambda r0: r0 // rpe, n_outer)
    else:
        # pass 1, one outer scale per output row (experts == 1): requant_amax_kernel, grid (cols / 64, rows / 128);
        # thread (cl = t % 64, rg = t / 64) reads 32 rows of one column, target the column
        for r0 in range(0, rows, 128):
            for bx in range(cols // 64):
                t = np.arange(T)
                cl, rg = t & 63, t >> 6
                c = bx * 64 + cl
                rr = r0 + rg[:, None] * 32 + np.arange(32)[None, :]
                assert rr.max() < rows and c.max() < cols
                assert ((rr * cols + c[:, None]) // 2).max() < rows * cols // 2
                offs = [sf_offset(int(a), int(cc) // 16, S_in, in_mma) for a, cc in zip(rr.reshape(-1),
                                                                                        np.repeat(c, 32))]
                assert min(offs) >= 0 and max(offs) < rows * S_in
                assert c.max() < n_outer
    # pass 2: the tile kernel; output row o = e * cols + c, its rpe columns the expert's rows
    _requant_tile_replay(rows, cols, group_rows, in_mma, out_mma, lambda r0: True,
                         lambda r0: (r0 - (r0 // rpe) * rpe, (r0 // rpe) * cols), rpe, experts * cols)


@pytest.mark.parametrize("rows,cols,group_rows", [(64, 48, 32), (16, 16, 16), (128, 256, 128)])
def test_tile16_kernel_indexing(rows, cols, group_rows):
    ntc = cols // 16
    warps = rows // 16 * ntc
    gid = _threads(warps * 32)
    tile, lane = gid >> 5, gid & 31
    assert np.all(tile < warps)
    tr, tc = tile // ntc, tile % ntc
    r, c0 = tr * 16 + (lane >> 1), tc * 16 + 8 * (lane & 1)
    x_start = (r * cols + c0) * 2
    assert x_start.max() + 16 <= rows * cols * 2 and np.all(x_start % 16 == 0)
    assert np.all((tr * 16) // group_rows < rows // group_rows)
    _exactly_once((r * cols + c0) // 2, 4, rows * cols // 2)
    lead = lane == 0
    _exactly_once(tr[lead] * ntc + tc[lead], 1, rows // 16 * ntc)
    # every warp's lanes belong to one tile (the warp leaves or stays whole)
    assert np.all(np.diff(tile.reshape(-1, 32), axis=1) == 0)


def _find_expert(seg, E, t):
    lo, hi = 0, E                                # seg[lo] <= t < seg[hi]
    while hi - lo > 1:
        mid = (lo + hi) >> 1
        if seg[mid] <= t:
            lo = mid
        else:
            hi = mid
    return lo


@pytest.mark.parametrize("M,C,seg,per_row,out_mma,in_mma,group_rows", [
    (512, 128, [0, 128, 128, 384], True, True, True, 1),          # an empty expert, 128 padding rows
    (384, 64, [0, 384], False, False, False, 1),
    (640, 256, [0, 0, 256, 256, 512, 512], True, True, True, 128),
])
def test_segment_kernels_indexing(M, C, seg, per_row, out_mma, in_mma, group_rows):
    seg = np.array(seg)
    E = len(seg) - 1
    # the shapes the entry points accept; segments as moe_route writes them
    assert M % 128 == 0 and C % 64 == 0 and (not out_mma or C % 128 == 0) and M % group_rows == 0
    assert np.all(seg % 128 == 0) and seg[-1] <= M and np.all(np.diff(seg) >= 0)
    end = seg[E]
    n_outer = E * C if per_row else E
    # pass 1 of the bf16 source: segment_amax_bf16_kernel, grid (C / 64, M / 128); thread (k = t % 8,
    # g = t / 8) loads 16 bytes of rows r0 + 4g .. r0 + 4g + 3 at column c0 + 8k
    t = np.arange(T)
    k8, g8 = t & 7, t >> 3
    assert np.all(k8 == (t ^ 8) & 7) and np.all(k8 == (t ^ 16) & 7)   # the lanes a shuffle combines
    for r0 in range(0, min(M, end), 128):
        lo = _find_expert(seg, E, r0)
        for bx in range(C // 64):
            xi = ((r0 + 4 * g8[:, None] + np.arange(4)[None, :]) * C + bx * 64 + 8 * k8[:, None]).reshape(-1)
            assert xi.min() >= 0 and (xi + 8).max() <= M * C and np.all(xi % 8 == 0)
            _exactly_once(np.sort((xi // C - r0) * 64 + xi % C - bx * 64), 8, 128 * 64)
            tg = lo * C + bx * 64 + np.arange(64) if per_row else np.array([lo])
            assert tg.min() >= 0 and tg.max() < n_outer
    # pass 1 of the NVFP4 source with per-row outer scales: segment_amax_kernel, grid (C / 64, M / 128);
    # blocks at or past seg[E] leave before any barrier
    for by in range(M // 128):
        r0 = by * 128
        if r0 >= end:
            continue
        lo = _find_expert(seg, E, r0)
        assert seg[lo] <= r0 and r0 + 127 < seg[lo + 1]              # the tile lies in one segment
        for bx in range(C // 64):
            c = bx * 64 + np.arange(64)
            rows = r0 + np.arange(128)
            assert rows.max() < M and c.max() < C
            assert ((rows[:, None] * C + c[None, :]) // 2).max() < M * C // 2       # NVFP4 source bytes
            assert (rows[:, None] * C + c[None, :]).max() < M * C                    # bf16 source elements
            offs = [sf_offset(int(r), int(cc) // 16, C // 16, in_mma) for r in rows[::31] for cc in c[::15]]
            assert max(offs) < M * (C // 16) and (rows // group_rows).max() < M // group_rows
            tg = lo * C + c if per_row else np.array([lo])
            assert tg.min() >= 0 and tg.max() < n_outer
    # pass 1 of the NVFP4 source with per-segment outer scales: group_amax_nvfp4_kernel over the live blocks
    if not per_row:
        _group_amax_replay(M, C, group_rows, in_mma, range(0, M, 128),
                           lambda r0: None if r0 >= end else _find_expert(seg, E, r0), n_outer)
    # pass 2: the tile kernel, output row c, its M columns the tokens; tiles past seg[E] only write zeros
    for r0 in range(0, M, 128):
        if r0 < end:
            lo = _find_expert(seg, E, r0)
            assert (lo * C + C - 1 if per_row else lo) < n_outer
    _requant_tile_replay(M, C, group_rows, in_mma, out_mma, lambda r0: r0 < end, lambda r0: (r0, 0), M, C)
    # pass 2 of the bf16 source: the same tile kernel with bf16 loads
    _requant_tile_replay(M, C, 1, in_mma, out_mma, lambda r0: r0 < end, lambda r0: (r0, 0), M, C, bf16=True)


@pytest.mark.parametrize("M,N,K,seg,pair", [
    (1280, 256, 256, [0, 512, 512, 768, 1280], True),
    (512, 128, 384, [0, 256, 512], False),
    (1280, 512, 1024, [0, 512, 512, 768, 1280], True),    # more k-tiles than n-tiles: n varies fastest
    (1280, 1024, 256, [0, 256, 1280], True),              # more n-tiles: k varies fastest
])
def test_nvfp4_wgrad_tile_mapping(M, N, K, seg, pair):
    # csrc/gemm.cu make_tile, WGRAD branch with NVFP4 operands: A [N, M] and B
    # [K, M] codes (M/2 bytes per row), scale atoms of 128 rows x 64 tokens
    seg = np.array(seg)
    assert np.all(seg % 256 == 0) and seg[-1] <= M and M % 256 == 0
    kBM, kStage = 128, 128
    kBN = 256 if pair else 128
    rows = 2 * kBM if pair else kBM
    groups = M // 64                                             # sfa_groups = sfb_groups
    atoms_a, atoms_b = (N // 128) * groups, (K // 128) * groups
    E = len(seg) - 1
    nt_n, nt_k = N // rows, K // kBN
    seen = set()
    for idx in range(E * nt_n * nt_k):
        e = idx // (nt_n * nt_k)
        rem = idx % (nt_n * nt_k)
        # the dimension with fewer tiles varies fastest
        tn, tk = (rem % nt_n, rem // nt_n) if nt_k >= nt_n else (rem // nt_k, rem % nt_k)
        assert (e, tn, tk) not in seen and 0 <= tn < nt_n and 0 <= tk < nt_k
        seen.add((e, tn, tk))
        s0, s1 = seg[e], seg[e + 1]
        for rank in ((0, 1) if pair else (0,)):
            a_y = tn * rows + rank * kBM
            col0 = tk * kBN
            b_y = col0 + (rank * kBN // 2 if pair else 0)
            k_tiles, k0 = (s1 - s0) // (2 * kStage), s0 // 2
            sfa0 = a_y // kBM * groups + s0 // 64
            sfb0 = col0 // kBM * groups + s0 // 64
            assert a_y + kBM <= N and b_y + (kBN // 2 if pair else kBN) <= K
            for kt in range(k_tiles):
                kx = k0 + kt * kStage
                assert kx % 16 == 0 and kx + kStage <= M // 2          # TMA x aligned and inside the row
                assert sfa0 + kt * 4 + 4 <= atoms_a
                for h in range(kBN // 128):
                    assert sfb0 + h * groups + kt * 4 + 4 <= atoms_b
            # the stages cover the segment's tokens exactly
            assert k_tiles * 256 == s1 - s0


# The same replays over shapes drawn at random within what the entry points
# accept: expert counts, empty experts, padding rows, layouts, group sizes.
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=30, deadline=None)
@given(st.data())
def test_segment_kernels_indexing_random_shapes(data):
    E = data.draw(st.integers(1, 5))
    seg = np.concatenate([[0], np.cumsum([data.draw(st.integers(0, 3)) * 128 for _ in range(E)])])
    M = max(128, int(seg[-1]) + data.draw(st.integers(0, 2)) * 128)
    C = data.draw(st.sampled_from([64, 128, 192, 256]))
    out_mma = C % 128 == 0 and data.draw(st.booleans())
    group_rows = data.draw(st.sampled_from([g for g in (1, 64, 128) if M % g == 0]))
    test_segment_kernels_indexing(M, C, list(seg), data.draw(st.booleans()), out_mma,
                                  data.draw(st.booleans()), group_rows)


@settings(max_examples=30, deadline=None)
@given(st.data())
def test_requant_kernels_indexing_random_shapes(data):
    per_expert = data.draw(st.booleans())
    experts = data.draw(st.integers(1, 4)) if per_expert else 1
    rpe = data.draw(st.integers(1, 3)) * 128
    rows = experts * rpe
    cols = data.draw(st.sampled_from([64, 128, 192, 256]))
    out_mma = (experts * cols) % 128 == 0 and data.draw(st.booleans())
    group_rows = data.draw(st.sampled_from([g for g in (1, 128, rpe) if rows % g == 0]))
    test_requant_kernels_indexing(rows, cols, group_rows, experts, int(per_expert), data.draw(st.booleans()),
                                  out_mma)


@settings(max_examples=30, deadline=None)
@given(st.data())
def test_quantize_and_tile_indexing_random_shapes(data):
    rows = data.draw(st.integers(1, 6)) * 128
    cols = data.draw(st.sampled_from([64, 128, 192, 320]))
    test_quantize_sr_kernel_indexing(rows, cols, data.draw(st.sampled_from([1, 16, 128])), cols % 64 == 0)
    trows, tcols = data.draw(st.integers(1, 8)) * 16, data.draw(st.integers(1, 8)) * 16
    test_tile16_kernel_indexing(trows, tcols, data.draw(st.sampled_from([g for g in (16, 32, trows)
                                                                          if trows % g == 0 and g % 16 == 0])))
