"""The expert-parallel exchange (fp8_moe_numerics_b200/expert_parallel.py) on
CPU ranks.

[ai-primer §Quantized NVLink and BBBK]: tokens travel to the GPU holding their
expert in NVFP4 and return for the combine.  Here two and three gloo ranks
exchange synthetic expert-major row buffers whose every byte names its source
rank and row, so each received row can be traced: after dispatch every local
expert's rows are the rows each source routed to it, sources in rank order,
rows in their source order; combine returns every row to the row it left
from.  The regrouping kernel (moe_permute_row_groups) is replaced by a torch
indexing emulation in this CPU test; its GPU form is checked against the same
emulation in tests/test_gpu_quant.py.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from fp8_moe_numerics_b200 import expert_parallel as ep  # noqa: E402


def permute_emulation(x, table, group_bytes):
    """Output group g = input group table[g] (zeros for -1), by torch indexing."""
    xg = x.reshape(-1, group_bytes)
    out = torch.zeros(table.numel(), group_bytes, dtype=torch.uint8)
    ok = table >= 0
    out[ok] = xg[table[ok].long()]
    return out.reshape(-1)


def _seg_for(rank, E, seed):
    rng = np.random.default_rng(seed + 17 * rank)
    groups = rng.integers(0, 4, E)
    groups[rng.integers(0, E)] = 0                      # an empty expert
    seg = np.zeros(E + 1, np.int64)
    seg[1:] = np.cumsum(groups) * 128
    return seg


def _buffers(rank, M_cap):
    """Three arrays of one row buffer whose bytes name (rank, row): codes-like
    [M_cap, 16] u8, a scale-like flat array of 4 bytes per row, and one float
    per row."""
    r = torch.arange(M_cap, dtype=torch.int64)
    codes = ((r[:, None] * 16 + torch.arange(16)[None, :] + 101 * rank) % 251).to(torch.uint8)
    sf = ((r[:, None] * 4 + torch.arange(4)[None, :] + 53 * rank) % 241).to(torch.uint8).reshape(-1)
    outer = (rank * 1e6 + r).to(torch.float32)
    return [codes.contiguous(), sf.contiguous(), outer.contiguous()]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, E, seed, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        segs = [_seg_for(r, E, seed) for r in range(world)]
        M_caps = [int(s[-1]) + 256 for s in segs]           # capacity past the routed rows
        mine = _buffers(rank, M_caps[rank])
        local, local_seg, plan = ep.dispatch(mine, M_caps[rank], torch.from_numpy(segs[rank]), world, rank,
                                             permute=permute_emulation)
        E_loc = E // world
        # expected: for local expert e, the rows each source routed to expert rank*E_loc + e, sources in order
        want = [[] for _ in range(3)]
        want_seg = [0]
        for e in range(E_loc):
            g = rank * E_loc + e
            for s in range(world):
                a, b = int(segs[s][g]), int(segs[s][g + 1])
                src = _buffers(s, M_caps[s])
                want[0].append(src[0][a:b])
                want[1].append(src[1][a * 4:b * 4])
                want[2].append(src[2][a:b])
            want_seg.append(want_seg[-1] + sum(int(segs[s][g + 1] - segs[s][g]) for s in range(world)))
        assert np.array_equal(local_seg.numpy(), np.array(want_seg))
        for got, w, row_bytes in zip(local, want, (16, 4, 4)):
            w = torch.cat([x.reshape(-1).view(torch.uint8) for x in w]) if w else torch.empty(0, dtype=torch.uint8)
            assert torch.equal(got, w)
        # combine: the expert rows return to the rows they left from
        back = [torch.full_like(a, 0) for a in mine]
        ep.combine(local, plan, back, M_caps[rank], permute=permute_emulation)
        n = int(segs[rank][-1])
        assert torch.equal(back[0][:n], mine[0][:n])
        assert torch.equal(back[1][:n * 4], mine[1][:n * 4])
        assert torch.equal(back[2][:n], mine[2][:n])
        assert torch.all(back[0][n:] == 0)                   # rows past the routing are not written
        out.put((rank, plan.send_total, plan.recv_total))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E", [(2, 8), (3, 6)])
def test_dispatch_and_combine_over_gloo_ranks(world, E):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, E, 5, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(out.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every group sent is received exactly once
    assert sum(g[1] for g in got) == sum(g[2] for g in got)


def test_plan_regroups_by_expert_then_source():
    seg = np.array([0, 128, 384, 384, 512], np.int64)       # 4 experts: 1, 2, 0, 1 groups
    recv = np.array([[1, 2], [3, 0], [0, 1]])               # 3 sources x 2 local experts
    plan = ep.make_plan(seg, world=2, rank=0, recv_counts=np.array([[1, 2], [3, 0]]))
    assert plan.send_groups == [3, 1] and plan.recv_groups == [3, 3]
    assert np.array_equal(plan.local_seg, np.array([0, 4, 6]) * 128)
    # received: src0 (e0: g0 | e1: g1 g2), src1 (e0: g3 g4 g5); expert-major: e0 <- g0 g3 g4 g5, e1 <- g1 g2
    assert plan.to_expert_major.tolist() == [0, 3, 4, 5, 1, 2]
    assert plan.to_source_major[plan.to_expert_major].tolist() == list(range(6))
    plan3 = ep.make_plan(np.array([0, 0, 128, 256, 256, 256, 384]), world=3, rank=1, recv_counts=recv)
    assert plan3.recv_groups == [3, 3, 1] and plan3.local_seg.tolist() == [0, 4 * 128, 7 * 128]
    assert plan3.to_expert_major.tolist() == [0, 3, 4, 5, 1, 2, 6]


def test_plan_rejects_unaligned_segments_and_uneven_experts():
    with pytest.raises(ValueError):
        ep.make_plan(np.array([0, 100, 228]), 2, 0, np.zeros((2, 1)))
    with pytest.raises(ValueError):
        ep.make_plan(np.array([0, 128, 256, 384]), 2, 0, np.zeros((2, 1)))
