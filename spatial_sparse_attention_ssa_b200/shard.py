"""Data-parallel sharding of a varlen SSA batch over ranks (one process per GPU).

Every SSA step stays inside its own sequence: blocks, windows, the compressed
keys and the selection are all per sequence (Direct3D-S2, hyper.ai, "方法": the
attention runs over the sparse voxels of one shape).  A varlen batch therefore
splits by whole sequences with no exchange in the data path: each rank bins and
attends its own sequences, and only a caller that wants every rank to hold the
whole batch's result gathers it afterwards (`gather_rows`).

The cost of a sequence is dominated by its compressed branch (every query
against every occupied block), so sequences are assigned longest-processing-
time first (LPT): sort by estimated cost, give each to the least-loaded rank.
LPT's makespan is at most (4/3 - 1/(3 * ranks)) of the optimum.

Host-side planning only; the attention itself runs in the CUDA library.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def occupied_cells(coords: np.ndarray, cu_seqlens: np.ndarray, m: int) -> np.ndarray:
    """Occupied m^3 cells per sequence ([S] int64): the block (or window) count."""
    coords = np.asarray(coords, np.int64)
    cu = np.asarray(cu_seqlens, np.int64)
    cells = coords // int(m)
    out = np.zeros(len(cu) - 1, np.int64)
    for s in range(len(cu) - 1):
        c = cells[cu[s]:cu[s + 1]]
        if len(c):
            key = (c[:, 0] << 42) | (c[:, 1] << 21) | c[:, 2]
            out[s] = len(np.unique(key))
    return out


def sequence_costs(coords: np.ndarray, cu_seqlens: np.ndarray, m_cmp: int, m_win: int, topk: int) -> np.ndarray:
    """Estimated scores per query head for each sequence: compressed n*B, selected
    n*k*(n/B) (k blocks of mean size), window n*(n/W) (mean window size)."""
    n = np.diff(np.asarray(cu_seqlens, np.int64)).astype(np.float64)
    b = np.maximum(occupied_cells(coords, cu_seqlens, m_cmp), 1).astype(np.float64)
    w = np.maximum(occupied_cells(coords, cu_seqlens, m_win), 1).astype(np.float64)
    return n * b + n * np.minimum(topk, b) * (n / b) + n * (n / w)


def lpt_assign(costs, world: int) -> np.ndarray:
    """Owner rank of each sequence: longest processing time first; ties between
    sequences by lower index, between ranks by lower rank."""
    costs = np.asarray(costs, np.float64)
    if world < 1:
        raise ValueError("world must be >= 1")
    owner = np.zeros(len(costs), np.int64)
    load = np.zeros(world)
    for s in np.argsort(-costs, kind="stable"):
        r = int(np.argmin(load))  # first minimum: the lowest rank
        owner[s] = r
        load[r] += costs[s]
    return owner


@dataclass
class LocalPlan:
    """One rank's share of a varlen batch."""
    seqs: np.ndarray  # global sequence ids owned by this rank, ascending
    tokens: np.ndarray  # global token indices of those sequences, in order
    cu_seqlens: np.ndarray  # int32 [len(seqs) + 1], offsets into `tokens`


def local_plan(cu_seqlens: np.ndarray, owner: np.ndarray, rank: int) -> LocalPlan:
    cu = np.asarray(cu_seqlens, np.int64)
    seqs = np.nonzero(np.asarray(owner) == rank)[0]
    lens = cu[seqs + 1] - cu[seqs]
    tokens = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]) if len(seqs) else np.zeros(0, np.int64)
    local_cu = np.zeros(len(seqs) + 1, np.int32)
    local_cu[1:] = np.cumsum(lens)
    return LocalPlan(seqs, tokens.astype(np.int64), local_cu)


def gather_rows(local, plan: LocalPlan, n_total: int, group=None):
    """All-gather per-token rows (a torch tensor [n_local, ...]) from every rank
    into the batch's token order ([n_total, ...]) on every rank.  Outside the
    data path: only for callers that want the whole batch's result everywhere."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    sizes = torch.tensor([local.shape[0]], dtype=torch.int64, device=local.device)
    all_sizes = [torch.zeros_like(sizes) for _ in range(world)]
    dist.all_gather(all_sizes, sizes, group=group)
    mx = int(max(int(x.item()) for x in all_sizes))
    pad = torch.zeros((mx,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    idx = torch.full((mx,), -1, dtype=torch.int64, device=local.device)
    idx[:local.shape[0]] = torch.as_tensor(plan.tokens, device=local.device)
    rows = [torch.zeros_like(pad) for _ in range(world)]
    idxs = [torch.zeros_like(idx) for _ in range(world)]
    dist.all_gather(rows, pad, group=group)
    dist.all_gather(idxs, idx, group=group)
    out = torch.zeros((n_total,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    for r, i in zip(rows, idxs):
        ok = i >= 0
        out[i[ok]] = r[ok]
    return out


# ---------------------------------------------------------------------------
# One sequence across ranks (LSRM, "块感知序列并行与负载均衡"): whole blocks per rank
# ---------------------------------------------------------------------------
#
# A rank owns a contiguous range of the sequence's blocks (blocks are numbered in
# cell order, so a range is also spatially compact) and the tokens in them.  Its
# queries attend (a) every compressed block and (b) the tokens of the selected
# blocks, which needs the K / V of the whole sequence: the ranks all-gather K / V
# (and could all-gather Kc / Vc instead of recomputing them); (c) the window
# branch needs only the rank's own tokens when windows are whole blocks
# (m_win = m_cmp).  In the backward, the key gradients of (a) and (b) are partial
# sums over the rank's queries and go back to the owning ranks (a reduce-scatter).
# Queries, outputs and gates never leave their rank.


def block_ranges(counts, world: int) -> list[tuple[int, int]]:
    """Split blocks 0 .. len(counts)-1, with counts[b] tokens each, into `world`
    contiguous ranges [lo, hi) minimising the largest token count of a range (the
    linear partition problem: the least feasible bound by binary search, each
    range filled greedily).  Ranges may be empty when there are fewer blocks than
    ranks; they cover the blocks in order."""
    counts = np.asarray(counts, np.int64)
    if world < 1:
        raise ValueError("world must be >= 1")
    nb = len(counts)
    if nb == 0:
        return [(0, 0)] * world

    def ranges_for(cap):
        out, lo, acc = [], 0, 0
        for b in range(nb):
            if acc + counts[b] > cap and b > lo:
                out.append((lo, b))
                lo, acc = b, 0
            acc += counts[b]
        out.append((lo, nb))
        return out

    lo_c, hi_c = int(counts.max()), int(counts.sum())
    while lo_c < hi_c:
        mid = (lo_c + hi_c) // 2
        if len(ranges_for(mid)) <= world:
            hi_c = mid
        else:
            lo_c = mid + 1
    r = ranges_for(lo_c)
    return r + [(nb, nb)] * (world - len(r))


def range_tokens(blk_perm, blk_ptr, lo: int, hi: int) -> np.ndarray:
    """Tokens of blocks lo .. hi-1, in block order (global token indices)."""
    blk_ptr = np.asarray(blk_ptr, np.int64)
    return np.asarray(blk_perm, np.int64)[blk_ptr[lo]:blk_ptr[hi]]


def all_gather_rows(local, tokens: np.ndarray, n_total: int, group=None):
    """Every rank's rows (a torch tensor [len(tokens), ...] of the given global token
    indices) placed at their token index in a [n_total, ...] tensor, on every rank:
    the K / V exchange of the sequence-parallel forward."""
    from types import SimpleNamespace
    return gather_rows(local, SimpleNamespace(tokens=np.asarray(tokens, np.int64)), n_total, group)


def reduce_to_owners(partial, tokens: np.ndarray, group=None):
    """Sum the [n_total, ...] partial gradients of all ranks and keep this rank's
    rows (`tokens`): the reduce-scatter of the key gradients.  Written as one
    all-reduce for clarity; the rows are disjoint across ranks."""
    import torch
    import torch.distributed as dist

    total = partial.clone()
    dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    return total[torch.as_tensor(np.asarray(tokens, np.int64), device=total.device)]


def sp_local_plan(blk_perm, blk_ptr, blk_cu, cu_seqlens, world: int, rank: int) -> LocalPlan:
    """This rank's tokens when every sequence's blocks are split into `world` contiguous
    ranges balanced by tokens (block_ranges) and rank r owns range r of each sequence:
    `tokens` are global token indices in block order, `cu_seqlens` their per-sequence
    offsets, `seqs` every sequence (a rank may own no block of a short one)."""
    blk_ptr = np.asarray(blk_ptr, np.int64)
    blk_cu = np.asarray(blk_cu, np.int64)
    parts, cu = [], [0]
    for s in range(len(cu_seqlens) - 1):
        b0, b1 = int(blk_cu[s]), int(blk_cu[s + 1])
        lo, hi = block_ranges(np.diff(blk_ptr[b0:b1 + 1]), world)[rank] if b1 > b0 else (0, 0)
        toks = range_tokens(blk_perm, blk_ptr, b0 + lo, b0 + hi)
        parts.append(toks)
        cu.append(cu[-1] + len(toks))
    tokens = np.concatenate(parts) if parts else np.zeros(0, np.int64)
    return LocalPlan(np.arange(len(cu_seqlens) - 1), tokens.astype(np.int64), np.asarray(cu, np.int32))
