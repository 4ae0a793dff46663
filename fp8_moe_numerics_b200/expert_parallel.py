"""Expert-parallel exchange of quantised token rows.

[ai-primer] "Inkling 2 Small uses four-bit training...", §Quantized NVLink and
BBBK: tokens are sent to the GPUs holding their experts in NVFP4, and the
expert outputs come back for the combine (there, rotated and in S2F6).  This
module moves those rows between ranks; every byte it moves was produced by the
library's kernels, and the only arithmetic here is the bookkeeping of offsets.

Layout.  With W ranks and E experts, rank d holds experts [d E/W, (d+1) E/W).
Each rank routes its own tokens over all E experts (moe_route), quantises and
gathers them into its expert-major NVFP4 row buffer, whose expert segments are
padded to 128 rows.  The rows bound for rank d are then one contiguous range,
[seg[d E/W], seg[(d+1) E/W]), of every array of that buffer: codes, scales in
the MMA layout (whose 512-byte atoms cover 128 rows) and outer scales.  So a
rank's send buffer is the prefix [0, seg[E]) of each array, split by
destination, and nothing is packed.

dispatch: the per-(destination, expert) group counts go through one
all-to-all (the data all-to-all needs its split sizes on the host, so the
counts are read back once), each array through one all_to_all_single, and
moe_permute_row_groups turns the received (source, expert) order into
(expert, source) order, with the local segment offsets of the expert GEMMs.

combine: the inverse.  The expert rank regroups its output rows (bf16 rows, or
S2F6 codes and exponents) by source, sends them back, and they land in each
source's own expert-major buffer at the rows of its routing, where moe_combine
or moe_combine_s2f6 reads them through pos.

Collectives go through torch.distributed (NCCL between GPUs).  No load here
reads another GPU's memory directly.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

GROUP_ROWS = 128                                        # the padding unit of an expert segment


@dataclass
class ExchangePlan:
    """Offsets of one dispatch / combine, in 128-row groups.

    send_groups[d]   groups this rank sends to rank d (its rows for d's experts)
    recv_groups[s]   groups this rank receives from rank s
    recv_counts      [W, E_loc]: groups from source s for local expert e
    local_seg        [E_loc + 1] row offsets of the local experts in the
                     expert-major receive buffer
    to_expert_major  int32 [total groups]: output group g (expert-major) takes
                     received group to_expert_major[g] (source-major)
    to_source_major  the inverse permutation
    """
    world: int
    rank: int
    experts: int
    experts_local: int
    send_groups: list
    recv_groups: list
    recv_counts: np.ndarray
    local_seg: np.ndarray
    to_expert_major: np.ndarray
    to_source_major: np.ndarray

    @property
    def send_total(self) -> int:
        return int(sum(self.send_groups))

    @property
    def recv_total(self) -> int:
        return int(sum(self.recv_groups))


def group_counts(seg_host: np.ndarray) -> np.ndarray:
    """Groups of 128 rows per expert from the segment offsets of moe_route."""
    seg = np.asarray(seg_host, dtype=np.int64)
    sizes = np.diff(seg)
    if seg[0] != 0 or np.any(sizes < 0) or np.any(sizes % GROUP_ROWS):
        raise ValueError("segment offsets must start at 0 and grow by multiples of 128 rows")
    return sizes // GROUP_ROWS


def make_plan(seg_host: np.ndarray, world: int, rank: int, recv_counts: np.ndarray) -> ExchangePlan:
    """The plan of this rank from its own segment offsets [E+1] and the
    per-(source, local expert) group counts [W, E_loc] it receives (what rank s
    sends here: its group counts of this rank's experts)."""
    per_expert = group_counts(seg_host)
    E = per_expert.size
    if E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    E_loc = E // world
    send = per_expert.reshape(world, E_loc)
    recv = np.asarray(recv_counts, dtype=np.int64).reshape(world, E_loc)
    # received buffer: by source, then by local expert
    in_first = np.zeros((world, E_loc), dtype=np.int64)
    flat = recv.reshape(-1)
    in_first.reshape(-1)[1:] = np.cumsum(flat)[:-1]
    # local expert-major buffer: by local expert, then by source
    order = recv.T.reshape(-1)                             # (e, s) order
    out_first = np.zeros(E_loc * world, dtype=np.int64)
    out_first[1:] = np.cumsum(order)[:-1]
    total = int(flat.sum())
    to_em = np.empty(total, dtype=np.int32)
    for e in range(E_loc):
        for s in range(world):
            n = int(recv[s, e])
            o = int(out_first[e * world + s])
            to_em[o:o + n] = in_first[s, e] + np.arange(n)
    to_sm = np.empty(total, dtype=np.int32)
    to_sm[to_em] = np.arange(total, dtype=np.int32)
    local_seg = np.zeros(E_loc + 1, dtype=np.int64)
    local_seg[1:] = np.cumsum(recv.sum(axis=0)) * GROUP_ROWS
    return ExchangePlan(world, rank, E, E_loc, [int(x) for x in send.sum(axis=1)],
                        [int(x) for x in recv.sum(axis=1)], recv, local_seg, to_em, to_sm)


def exchange_counts(seg_host: np.ndarray, world: int, group=None) -> np.ndarray:
    """All-to-all of the per-(destination, expert) group counts: returns [W, E_loc],
    row s = what rank s sends to this rank."""
    import torch.distributed as dist
    send = torch.from_numpy(group_counts(seg_host).astype(np.int64))
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    send = send.to(dev)
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.cpu().numpy().reshape(world, -1)


def _bytes(t: torch.Tensor) -> torch.Tensor:
    return t.reshape(-1).view(torch.uint8)


def _exchange(send: torch.Tensor, send_groups, recv_groups, group_bytes: int, group=None, recv=None) -> torch.Tensor:
    import torch.distributed as dist
    if recv is None:
        recv = torch.empty(int(sum(recv_groups)) * group_bytes, dtype=torch.uint8, device=send.device)
    dist.all_to_all_single(recv, send, [g * group_bytes for g in recv_groups],
                           [g * group_bytes for g in send_groups], group=group)
    return recv


def _permute(x: torch.Tensor, table: np.ndarray, group_bytes: int, permute) -> torch.Tensor:
    if table.size == 0:
        return torch.empty(0, dtype=torch.uint8, device=x.device)
    t = torch.from_numpy(np.ascontiguousarray(table)).to(x.device)
    return permute(x, t, group_bytes)


def _default_permute():
    from . import api
    return api.moe_permute_row_groups


def dispatch(arrays, M_cap: int, seg: torch.Tensor, world: int, rank: int, group=None, permute=None):
    """Send this rank's expert-major rows to the ranks holding their experts.

    arrays: the row buffer's arrays, each a contiguous tensor whose bytes are
      M_cap rows of equal size in row order (NVFP4 codes [M_cap, D/2], scales in
      the MMA layout, outer scales [M_cap], ...);
    seg: the routing's segment offsets [E+1] (device or host).
    Returns (local arrays as uint8 byte tensors in (local expert, source)
    order, local_seg int64 [E_loc+1] on the arrays' device, plan)."""
    permute = permute or _default_permute()
    seg_host = seg.detach().cpu().numpy() if isinstance(seg, torch.Tensor) else np.asarray(seg)
    plan = make_plan(seg_host, world, rank, exchange_counts(seg_host, world, group))
    rows_sent = plan.send_total * GROUP_ROWS
    out = []
    for a in arrays:
        b = _bytes(a)
        if M_cap <= 0 or b.numel() % M_cap:
            raise ValueError("every array must hold the same number of bytes per row")
        gb = b.numel() // M_cap * GROUP_ROWS
        recv = _exchange(b[:rows_sent // GROUP_ROWS * gb], plan.send_groups, plan.recv_groups, gb, group)
        out.append(_permute(recv, plan.to_expert_major, gb, permute))
    local_seg = torch.from_numpy(plan.local_seg).to(arrays[0].device)
    return out, local_seg, plan


def combine(arrays, plan: ExchangePlan, out_arrays, M_cap: int, group=None, permute=None):
    """Return expert outputs to the ranks their tokens came from.

    arrays: this rank's output rows in (local expert, source) order
      (plan.recv_total * 128 rows of each array's row size);
    out_arrays: the source-side buffers, contiguous, M_cap rows each, whose rows
      [0, seg[E]) receive the rows of this rank's routing, in its expert-major
      order.  Returns out_arrays."""
    permute = permute or _default_permute()
    for a, o in zip(arrays, out_arrays):
        b, ob = _bytes(a), _bytes(o)
        if M_cap <= 0 or ob.numel() % M_cap:
            raise ValueError("every output array must hold M_cap rows of equal size")
        gb = ob.numel() // M_cap * GROUP_ROWS                # bytes of 128 rows, the same on both sides
        if b.numel() < plan.recv_total * gb or ob.numel() < plan.send_total * gb:
            raise ValueError("combine: buffers smaller than the plan's rows")
        src_major = _permute(b[:plan.recv_total * gb], plan.to_source_major, gb, permute)
        _exchange(src_major, plan.recv_groups, plan.send_groups, gb, group, recv=ob[:plan.send_total * gb])
    return out_arrays
