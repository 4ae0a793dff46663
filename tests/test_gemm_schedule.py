"""The ROWS-mode tile schedule of the grouped GEMMs, replayed on the CPU.

csrc/gemm.cu runs a ROWS call with 256-wide column tiles as two kernels.
When the experts with an odd tile count give at least tail_min_items leftover
tiles (times the column tiles), the pair kernel takes each expert's full row
pairs (floor(tiles_e / 2)) and the tail kernel (single CTAs, 128 x 256 tiles)
the leftover tiles; otherwise the pair kernel takes ceil(tiles_e / 2) pairs,
the last one possibly half empty (its CTA 1 recomputes CTA 0's rows and
stores nothing), and the tail kernel nothing.  Other shapes walk the 128-row
tiles with single CTAs.  The replay follows the kernels' decision, prefix
scan, item decoding and coordinates, and checks that every routed row tile
and column tile is stored exactly once, with every TMA box and scale-atom
range inside its tensor.
"""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

kBM, kStage, kMaxPairExperts = 128, 128, 768


def split_decision(seg, N, tail_min_items):
    tiles = np.diff(seg) // kBM
    return int(np.sum(tiles & 1)) * (N // 256) >= tail_min_items


def row_prefix(seg, tail, split=True):
    tiles = np.diff(seg) // kBM
    if split:
        per = (tiles & 1) if tail else tiles // 2
    else:
        per = 0 * tiles if tail else (tiles + 1) // 2
    return np.concatenate([[0], np.cumsum(per)]).astype(np.int64)


def last_expert_at_or_below(pfx, E, mt):
    lo, hi = 0, E                        # the kernel's binary search: last e with pfx[e] <= mt
    while hi - lo > 1:
        mid = (lo + hi) >> 1
        if pfx[mid] <= mt:
            lo = mid
        else:
            hi = mid
    return lo


def find_expert(seg, E, row):
    lo, hi = 0, E
    while hi - lo > 1:
        mid = (lo + hi) >> 1
        if seg[mid] <= row:
            lo = mid
        else:
            hi = mid
    return lo


def rows_items(seg, N, K, kind, kBN, pair, tail, tail_min_items):
    """Every CTA of every item of one kernel (expert, rows, columns, K stages, store), and the item count."""
    E = len(seg) - 1
    K_bytes = K // 2 if kind == "nvfp4" else K
    pfx = row_prefix(seg, tail, split_decision(seg, N, tail_min_items)) if (pair or tail) else None
    n_tiles = N // kBN
    total = (pfx[E] if (pair or tail) else seg[E] // kBM) * n_tiles
    out = []
    for idx in range(int(total)):
        mt, nt = divmod(idx, n_tiles)
        if pair or tail:
            e = last_expert_at_or_below(pfx, E, mt)
            base = seg[e] + (mt - pfx[e]) * 2 * kBM if pair else seg[e + 1] - kBM
        else:
            base = mt * kBM
            e = find_expert(seg, E, base)
        for rank in ((0, 1) if pair else (0,)):
            store = not pair or rank == 0 or base + kBM < seg[e + 1]
            a_row = base + rank * kBM if store else base
            col0 = nt * kBN
            out.append(dict(e=e, row0=base + rank * kBM, col0=col0, a_y=a_row, rank=rank, store=store,
                            k_tiles=K_bytes // kStage))
    return out, total


def check_rows_schedule(seg, M_cap, N, K, kind, tail_min_items):
    """The whole call: the pair + tail kernels when N % 256 == 0, else the 128-wide single kernel."""
    E = len(seg) - 1
    wide = N % 256 == 0 and E <= kMaxPairExperts
    kernels = [(256, True, False), (256, False, True)] if wide else [(128, False, False)]
    covered = np.zeros((M_cap // kBM, N // 128), np.int64)
    sfa_groups = K // 64 if kind == "nvfp4" else K // 128
    atoms_per_stage = 4 if kind == "nvfp4" else 1
    for kBN, pair, tail in kernels:
        items, total = rows_items(seg, N, K, kind, kBN, pair, tail, tail_min_items)
        if tail:                                                 # the host's grid bound for the tail kernel
            assert total <= min(E, M_cap // kBM) * (N // 256)
        for it in items:
            e, a_y, col0 = it["e"], it["a_y"], it["col0"]
            # this CTA's 128 rows belong to expert e and lie inside A
            assert seg[e] <= a_y and a_y + kBM <= seg[e + 1] and a_y + kBM <= M_cap
            # B rows: NVFP4 weight stack [E*N, K], the CTA's share of the kBN rows; MXFP8 DGRAD B [N, E*K]
            share = kBN // 2 if pair else kBN
            b_y = (e * N if kind == "nvfp4" else 0) + col0 + (it["rank"] * share if pair else 0)
            b_rows = E * N if kind == "nvfp4" else N
            assert b_y + share <= b_rows
            # TMA boxes: A one 128-row box; B boxes of 128 rows (pair: one, tail: two)
            assert share % 128 == 0
            # scale atoms of every stage inside their arrays
            sfa_atoms = M_cap // 128 * sfa_groups
            sfb_groups = sfa_groups if kind == "nvfp4" else E * K // 128
            sfb_atoms = (E * N if kind == "nvfp4" else N) // 128 * sfb_groups
            sfa0 = a_y // kBM * sfa_groups
            b_first = e * N + col0 if kind == "nvfp4" else col0
            sfb0 = b_first // kBM * sfb_groups + (0 if kind == "nvfp4" else e * K // 128)
            for kt in range(it["k_tiles"]):
                assert sfa0 + kt * atoms_per_stage + atoms_per_stage <= sfa_atoms
                for h in range(kBN // 128):
                    assert sfb0 + h * sfb_groups + kt * atoms_per_stage + atoms_per_stage <= sfb_atoms
            if it["store"]:
                assert it["row0"] == a_y
                covered[a_y // kBM, col0 // 128:(col0 + kBN) // 128] += 1
            else:                                                # half pair: rows past the expert, not stored
                assert it["rank"] == 1 and it["row0"] >= seg[e + 1]
    # every routed row tile (below seg[E]) computed exactly once, nothing past it
    routed = int(seg[E]) // kBM
    assert np.all(covered[:routed] == 1)
    assert np.all(covered[routed:] == 0)


def seg_from_tiles(tiles):
    return np.concatenate([[0], np.cumsum(np.asarray(tiles, np.int64) * kBM)])


@pytest.mark.parametrize("tiles", [
    [1, 0, 2, 3],            # odd, empty, even, odd
    [1, 1, 1],               # no pairs: the tail kernel does everything
    [2, 0, 4],               # no tails: the tail kernel has no item
    [0, 0, 0],               # nothing routed
    [7],
])
@pytest.mark.parametrize("kind", ["nvfp4", "mxfp8"])
@pytest.mark.parametrize("N", [256, 512, 384])
@pytest.mark.parametrize("tail_min_items", [0, 1, 10 ** 9])    # split always / when any / never
def test_rows_schedule_small(tiles, kind, N, tail_min_items):
    seg = seg_from_tiles(tiles)
    M_cap = max(128, int(seg[-1]) + 256)
    check_rows_schedule(seg, M_cap, N, 512, kind, tail_min_items)


def test_rows_schedule_384_expert_layer_counts():
    # 384 experts with Zipf-like loads: the pair kernel runs floor(t/2) pairs per expert, the tail one tile
    # per odd expert; together they cover sum(t) row tiles, and no pair is half empty
    rng = np.random.default_rng(0)
    counts = np.minimum((rng.zipf(1.2, 384) * 40), 30000)
    tiles = (counts + 127) // 128
    seg = seg_from_tiles(tiles)
    pairs, tails = row_prefix(seg, False), row_prefix(seg, True)
    assert 2 * pairs[-1] + tails[-1] == tiles.sum()
    assert tails[-1] == int(np.sum(tiles % 2))
    assert split_decision(seg, 2048, 4 * 148)                   # GEMM1 of such a layer splits on 148 SMs
    check_rows_schedule(seg, int(seg[-1]) + 128, 256, 256, "nvfp4", 4 * 148)


def test_rows_schedule_decision_matches_gpu_test_shapes():
    # tests/test_gpu_gemm.py's many-expert cases must take the split on a B200 (148 SMs), the small ones not
    alt = [60 + 200 * (i % 2) for i in range(200)]
    seg = np.concatenate([[0], np.cumsum([(c + 127) // 128 * 128 for c in alt])])
    assert split_decision(seg, 1024, 4 * 148)
    assert not split_decision(seg_from_tiles([1, 0, 2, 3]), 4096, 4 * 148)


@settings(max_examples=40, deadline=None)
@given(st.data())
def test_rows_schedule_random_shapes(data):
    E = data.draw(st.integers(1, 12))
    tiles = [data.draw(st.integers(0, 5)) for _ in range(E)]
    seg = seg_from_tiles(tiles)
    M_cap = max(128, int(seg[-1]) + data.draw(st.integers(0, 3)) * 128)
    N = data.draw(st.sampled_from([128, 256, 384, 512]))
    K = data.draw(st.sampled_from([256, 512, 1024]))
    check_rows_schedule(seg, M_cap, N, K, data.draw(st.sampled_from(["nvfp4", "mxfp8"])),
                        data.draw(st.sampled_from([0, 3, 8, 10 ** 9])))
