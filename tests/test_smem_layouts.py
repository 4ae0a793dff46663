"""Shared-memory layouts of the transpose kernels, checked on the CPU.

The requantisation and the MXFP8 quantiser transpose their tiles through
shared memory with XOR swizzles (csrc/quant.cu: tsw for the fp32 tile of the
register-prefetch MXFP8 kernel, rq_swz for the f16 tile of the requantisation, t2_word for the bf16
pair tile of the TMA-fed MXFP8 kernel; the TMA tiles use the hardware's
128-byte swizzle).  The swizzle functions are restated here and every warp
access pattern of the kernels is replayed to check that each layout is a
bijection and that no access has a bank conflict: 32 lanes of 4-byte
accesses hit 32 distinct banks; a 16-byte access is served per quarter warp,
whose 8 lanes must hit 8 distinct 16-byte bank groups.
"""
import numpy as np

TR, TC = 128, 64                     # tile rows x columns


def tsw(c, r):
    rs = (r & ~12) | ((((r >> 2) & 3) ^ ((r >> 5) & 3)) << 2)
    return c * TR + (rs ^ ((c >> 5) << 4))


def t2_word(cp, r):
    rr = r ^ ((cp >> 4) << 4)
    rr ^= ((rr >> 5) & 3) << 2
    return cp * TR + rr


def sw128(row, chunk):               # byte offset of 16-byte chunk `chunk` of a 128-byte TMA row
    return row * 128 + ((chunk ^ (row & 7)) << 4)


def _words_conflict_free(words):
    return len({w % 32 for w in words}) == len(words)


def _quads_conflict_free(byte_addrs):
    for q in range(0, 32, 8):        # one quarter warp at a time
        if len({(a // 16) % 8 for a in byte_addrs[q:q + 8]}) != 8:
            return False
    return True


def test_fp32_tile_swizzle_is_a_bijection():
    assert sorted(tsw(c, r) for c in range(TC) for r in range(TR)) == list(range(TC * TR))


def test_fp32_tile_phase1_scalar_stores_conflict_free():
    # thread t writes row t/2, columns 32(t%2) + 2i and + 2i + 1 (one store each)
    for warp in range(8):
        for i in range(16):
            for off in (0, 1):
                lanes = range(32)
                words = [tsw(32 * (l & 1) + 2 * i + off, (32 * warp + l) >> 1) for l in lanes]
                assert _words_conflict_free(words), (warp, i, off)


def test_fp32_tile_phase2_vector_loads_conflict_free():
    # thread (c = 32 it + 4 warp + lane/8, g = lane % 8) reads rows 16g + 4j .. +3 of column c
    for it in range(2):
        for warp in range(8):
            for j in range(4):
                addrs = []
                for lane in range(32):
                    c, g = it * 32 + warp * 4 + (lane >> 3), lane & 7
                    w = tsw(c, 16 * g + 4 * j)
                    assert w % 4 == 0 and all(tsw(c, 16 * g + 4 * j + m) == w + m for m in range(4))
                    addrs.append(4 * w)
                assert _quads_conflict_free(addrs), (it, warp, j)


def test_pair_tile_swizzle_is_a_bijection():
    assert sorted(t2_word(cp, r) for cp in range(TC // 2) for r in range(TR)) == list(range(TC // 2 * TR))


def test_pair_tile_phase1_stores_conflict_free():
    # thread t (row t/2, half t%2) stores word j of its row half at (16 half + j, row)
    for warp in range(8):
        for j in range(16):
            words = [t2_word(16 * (l & 1) + j, (32 * warp + l) >> 1) for l in range(32)]
            assert _words_conflict_free(words), (warp, j)


def test_pair_tile_phase2_vector_loads_conflict_free():
    # thread (cp = t/8, g = t%8) reads rows 16g + 4k .. +3 of column pair cp
    for warp in range(8):
        for k in range(4):
            addrs = []
            for lane in range(32):
                t = 32 * warp + lane
                cp, g = t >> 3, t & 7
                w = t2_word(cp, 16 * g + 4 * k)
                assert w % 4 == 0 and all(t2_word(cp, 16 * g + 4 * k + m) == w + m for m in range(4))
                addrs.append(4 * w)
            assert _quads_conflict_free(addrs), (warp, k)


def test_tma_tile_row_reads_conflict_free():
    # TMA-fed MXFP8 kernel, phase 1: thread (row t/2, half t%2) reads chunks 4 half + i of its row
    for warp in range(8):
        for i in range(4):
            addrs = [sw128((32 * warp + l) >> 1, 4 * (l & 1) + i) for l in range(32)]
            assert _quads_conflict_free(addrs), (warp, i)
    # and the swizzle is a bijection over the 128 x 128-byte tile
    assert sorted(sw128(r, c) for r in range(TR) for c in range(8)) == list(range(0, TR * 128, 16))


def test_pair_tile_holds_each_row_pair_once():
    # every (column pair, row) word is written by exactly one phase-1 thread
    seen = np.zeros(TC // 2 * TR, np.int64)
    for t in range(256):
        for j in range(16):
            seen[t2_word(16 * (t & 1) + j, t >> 1)] += 1
    assert np.all(seen == 1)


# ---------------------------------------------------------------------------
# The R = 16 requantisation's f16 tile (requant16_tile_kernel): f16 [64 cols][128 rows],
# 256 bytes per column, 16-byte chunks (8 rows) XOR-swizzled by rq_swz(c).
# ---------------------------------------------------------------------------

def rq_swz(c):
    return ((c >> 4) & 3) | ((c & 1) << 2)


def rq_chunk_addr(c, k):            # byte address of chunk k (rows 8k..8k+7) of column c
    return c * 256 + ((k ^ rq_swz(c)) << 4)


def test_f16_tile_chunks_are_a_bijection():
    addrs = sorted(rq_chunk_addr(c, k) for c in range(TC) for k in range(TR // 8))
    assert addrs == list(range(0, TC * TR * 2, 16))


def _stmatrix_rows(warp, n):
    """Stored rows of stmatrix call n of `warp`: for lane 8j + m, (matrix j, tile column, chunk)."""
    out = []
    for lane in range(32):
        j, m = lane >> 3, lane & 7
        g, kap = n >> 1, 4 * (n & 1) + j
        out.append((j, 16 * (m >> 1) + 2 * kap + (m & 1), 2 * warp + g))
    return out


def test_f16_tile_stmatrix_writes_every_value_once_in_its_place():
    # fragment: lane (rho, b) holds, for matrix (g, kappa), tile row 16 warp + 8 g + rho and tile columns
    # 2 beta, 2 beta + 1 with beta = 8 b + kappa (its code byte); stored row m of the transposed matrix is
    # fragment column m = 2b + delta, i.e. tile column 16 b + 2 kappa + delta, values = the 8 fragment rows
    seen = {}
    for warp in range(8):
        for n in range(4):
            g = n >> 1
            for j, c, k in _stmatrix_rows(warp, n):
                kap = 4 * (n & 1) + j
                b, delta = (c - 2 * kap) // 16, (c - 2 * kap) % 16
                assert delta in (0, 1) and 0 <= b < 4          # column c is in lane b's code bytes
                assert 2 * (8 * b + kap) + delta == c
                rows = [16 * warp + 8 * g + rho for rho in range(8)]
                for i, r in enumerate(rows):
                    a = rq_chunk_addr(c, k) + 2 * i
                    assert r // 8 == k and r % 8 == i              # row r sits at position r % 8 of chunk r / 8
                    assert a not in seen
                    seen[a] = (c, r)
    assert len(seen) == TC * TR


def test_f16_tile_stmatrix_conflict_free():
    # each 8x8 matrix is 8 stored rows of 16 bytes; its 8 row addresses must hit 8 distinct bank groups
    for warp in range(8):
        for n in range(4):
            rows = _stmatrix_rows(warp, n)
            for j in range(4):
                addrs = [rq_chunk_addr(c, k) for jj, c, k in rows if jj == j]
                assert len({(a // 16) % 8 for a in addrs}) == 8, (warp, n, j)


def test_f16_tile_phase2_loads_conflict_free_and_cover_the_tile():
    # lane (m = lane % 8, jj = lane / 8 % 2, q = lane / 16) of warp w, pass it: column c = 16 (m / 2) + 2 w + m % 2,
    # rows 16 j .. 16 j + 15 with j = 2 (2 it + q) + jj, read as chunks 2j and 2j + 1
    covered = set()
    for warp in range(8):
        for it in range(2):
            for half in range(2):
                addrs = []
                for lane in range(32):
                    m, jj, q = lane & 7, (lane >> 3) & 1, lane >> 4
                    c = 16 * (m >> 1) + 2 * warp + (m & 1)
                    j = 2 * (2 * it + q) + jj
                    addrs.append(rq_chunk_addr(c, 2 * j + half))
                    covered.add((c, 2 * j + half))
                    # the 32-row E8M0 block of this lane is completed by lane ^ 8
                    m2, jj2, q2 = (lane ^ 8) & 7, ((lane ^ 8) >> 3) & 1, (lane ^ 8) >> 4
                    assert (m2, q2) == (m, q) and jj2 != jj
                assert _quads_conflict_free(addrs), (warp, it, half)
    assert len(covered) == TC * TR // 8
