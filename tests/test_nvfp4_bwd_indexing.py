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
    # pass 1: grid (cols / 64, rows / 128); thread (cl = t % 64, rg = t / 64) reads 32 rows of one column
    n_outer = experts if per_expert else experts * cols
    for by in range(rows // 128):
        r0 = by * 128
        e = r0 // rpe
        assert (r0 + 127) // rpe == e                         # a block never straddles two experts
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
            targets = np.full(1, e) if per_expert else e * cols + c[:64]
            assert targets.min() >= 0 and targets.max() < n_outer
    # pass 2: one thread per output block of 16; item -> (c fastest, then block b, then expert e)
    nb = rpe // 16
    item = _threads(experts * nb * cols)
    c = item % cols
    b = (item // cols) % nb
    e = item // cols // nb
    o = e * cols + c
    rr = e[:, None] * rpe + b[:, None] * 16 + np.arange(16)[None, :]
    assert rr.max() < rows
    assert np.all((per_expert and e.max() < experts) or o.max() < experts * cols)
    _exactly_once((o * rpe + b * 16) // 2, 8, experts * cols * rpe // 2)
    _exactly_once([sf_offset(int(a), int(bb), nb, out_mma) for a, bb in zip(o, b)], 1, experts * cols * nb)
    # the random index of each element is its linear output index, each used once
    L = (o * rpe + b * 16)[:, None] + np.arange(16)[None, :]
    assert np.array_equal(np.sort(L.reshape(-1)), np.arange(experts * cols * rpe))


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
    # pass 1: grid (C / 64, M / 128); blocks at or past seg[E] leave before any barrier
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
    # pass 2: one thread per output block of 16 tokens, c fastest
    nb = M // 16
    item = _threads(nb * C)
    c, b = item % C, item // C
    t0 = b * 16
    assert (t0 + 15).max() < M
    for tt in np.unique(t0[t0 < end]):
        lo = _find_expert(seg, E, int(tt))
        assert seg[lo] <= tt < seg[lo + 1]
    _exactly_once((c * M + t0) // 2, 8, C * M // 2)
    _exactly_once([sf_offset(int(a), int(bb), nb, out_mma) for a, bb in zip(c, b)], 1, C * nb)
    L = (c * M + t0)[:, None] + np.arange(16)[None, :]
    assert np.array_equal(np.sort(L.reshape(-1)), np.arange(C * M))


@pytest.mark.parametrize("M,N,K,seg,pair", [
    (1280, 256, 256, [0, 512, 512, 768, 1280], True),
    (512, 128, 384, [0, 256, 512], False),
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
    for idx in range(E * (N // rows) * (K // kBN)):
        e = idx // ((N // rows) * (K // kBN))
        rem = idx % ((N // rows) * (K // kBN))
        tn, tk = rem // (K // kBN), rem % (K // kBN)
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
