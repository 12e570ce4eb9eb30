"""One sequence split across ranks by whole blocks (host logic; CPU, gloo world size 2).

Each rank owns a contiguous range of the sequence's blocks.  It all-gathers K / V,
computes its own queries' compressed and selected branches against the whole
sequence (the cross-attention form: its queries, every voxel's keys), its window
branch on its own tokens only (windows are whole blocks when m_win = m_cmp), and
combines them with its gates.  In the backward its partial key gradients go back to
the owners.  The oracle stands in for the per-rank compute; the test checks that
the ranks' rows reproduce the single-process forward and backward, and the
partition itself against brute force.
"""
import itertools
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import shard
from spatial_sparse_attention_ssa_b200 import workloads as W


def test_block_ranges_minimise_the_largest_range_against_brute_force():
    rng = np.random.default_rng(5)
    for world in (1, 2, 3):
        for _ in range(25):
            counts = rng.integers(1, 20, size=rng.integers(1, 8))
            ranges = shard.block_ranges(counts, world)
            assert len(ranges) == world and ranges[0][0] == 0 and ranges[-1][1] == len(counts)
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            got = max(int(counts[lo:hi].sum()) for lo, hi in ranges)
            best = min(max(int(counts[a:b].sum()) for a, b in zip((0,) + cuts, cuts + (len(counts),)))
                       for cuts in itertools.combinations_with_replacement(range(len(counts) + 1), world - 1)
                       if all(x <= y for x, y in zip(cuts, cuts[1:])))
            assert got == best, (counts, world, ranges)
    assert shard.block_ranges([], 2) == [(0, 0), (0, 0)]
    with pytest.raises(ValueError):
        shard.block_ranges([1], 0)


def _case():
    w = W.small_shell(seed=61, R=32, n_prims=2, lo=4.0, hi=8.0, n_keep=260, n_seqs=1, hq=4, hkv=2, d=8,
                      m_cmp=4, m_win=4, topk=3, dtype="f32")
    t = W.make_tensors(w)
    return w, t


def _rank_main(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, t = _case()
        q, k, v, do = (t.as_f32(x).astype(np.float64) for x in ("q", "k", "v", "do"))
        kw = dict(hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, gate_mode=w.gate_mode, pool_rounding="none")
        blk = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)  # every rank bins the sequence the same way
        # the plan the GPU path uses (ssa_sp_forward's callers): whole blocks per rank
        plan = shard.sp_local_plan(blk["perm"], blk["ptr"], blk["cu"], w.cu_seqlens, world, rank)
        mine = plan.tokens
        lo, hi = shard.block_ranges(np.diff(blk["ptr"]), world)[rank]
        assert np.array_equal(mine, shard.range_tokens(blk["perm"], blk["ptr"], lo, hi))
        n, nr = w.n, len(mine)

        # all-gather of K / V: each rank contributes its own tokens' rows
        kv_full = shard.all_gather_rows(torch.from_numpy(np.concatenate([k[mine], v[mine]], axis=1)), mine, n)
        k_all, v_all = kv_full[:, :w.hkv].numpy(), kv_full[:, w.hkv:].numpy()

        # compressed + selected branches: this rank's queries against every voxel
        cr = O.cross_forward(np.array([0, nr]), w.coords, w.cu_seqlens, q[mine], k_all, v_all, t.gates[mine, :, :2],
                             topk=w.topk, **kw)
        # window branch: this rank's tokens only
        loc = O.forward(w.coords[mine], np.array([0, nr]), q[mine], k[mine], v[mine], t.gates[mine], m_win=w.m_win,
                        topk=w.topk, **kw)
        gw = O.gate_weights(t.gates[mine], w.gate_mode)
        out = gw[..., 0, None] * cr["o"][0] + gw[..., 1, None] * cr["o"][1] + gw[..., 2, None] * loc["o"][2]

        # backward: local queries' gradients; partial key gradients to their owners
        gc = O.cross_backward(cr, do[mine])
        gl = O.backward(loc, do[mine])
        dq = gc["dq"] + gl["parts"]["dq"]["win"]
        dk_part = gc["dk"].copy()
        dv_part = gc["dv"].copy()
        dk_part[mine] += gl["parts"]["dk"]["win"]
        dv_part[mine] += gl["parts"]["dv"]["win"]
        dk = shard.reduce_to_owners(torch.from_numpy(dk_part), mine).numpy()
        dv = shard.reduce_to_owners(torch.from_numpy(dv_part), mine).numpy()
        dg = np.concatenate([gc["dgates"], gl["dgates"][..., 2:]], axis=-1)

        # the single-process reference
        st = O.forward(w.coords, w.cu_seqlens, q, k, v, t.gates, m_win=w.m_win, topk=w.topk, **kw)
        g = O.backward(st, do)
        errs = {"sel": int((cr["sel"] != st["sel"][mine]).sum()),
                "out": float(np.abs(out - st["out"][mine]).max()),
                "dq": float(np.abs(dq - g["dq"][mine]).max()),
                "dk": float(np.abs(dk - g["dk"][mine]).max()),
                "dv": float(np.abs(dv - g["dv"][mine]).max()),
                "dgates": float(np.abs(dg - g["dgates"][mine]).max())}
        result_q.put((rank, nr, int(hi - lo), errs))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_reproduce_one_sequence_forward_and_backward():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(2, _free_port(), q), nprocs=2, join=True, start_method="spawn")
    res = sorted(q.get() for _ in range(2))
    w, _ = _case()
    assert [r[0] for r in res] == [0, 1]
    assert sum(r[1] for r in res) == w.n and all(r[1] > 0 for r in res)
    for _, _, _, e in res:
        assert e["sel"] == 0, e
        for key in ("out", "dq", "dk", "dv", "dgates"):
            assert e[key] <= 1e-12, (key, e)


def test_sp_local_plan_partitions_every_sequence_by_whole_blocks():
    w = W.small_shell(seed=62, R=32, n_prims=2, lo=4.0, hi=8.0, n_keep=300, n_seqs=3, hq=4, hkv=2, d=8,
                      m_cmp=4, m_win=4, topk=3, dtype="f32")
    blk = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)
    for world in (1, 2, 3, 5):
        seen = np.zeros(w.n, np.int64)
        for r in range(world):
            plan = shard.sp_local_plan(blk["perm"], blk["ptr"], blk["cu"], w.cu_seqlens, world, r)
            seen[plan.tokens] += 1
            assert plan.cu_seqlens[-1] == len(plan.tokens) and len(plan.cu_seqlens) == w.s + 1
            for s_ in range(w.s):
                toks = plan.tokens[plan.cu_seqlens[s_]:plan.cu_seqlens[s_ + 1]]
                assert ((toks >= w.cu_seqlens[s_]) & (toks < w.cu_seqlens[s_ + 1])).all()
                ids = blk["id"][toks]
                # whole blocks, consecutive ids, members in block order
                assert (np.diff(ids) >= 0).all() and (np.diff(np.unique(ids)) == 1).all()
                for b in np.unique(ids):
                    assert (ids == b).sum() == blk["ptr"][b + 1] - blk["ptr"][b]
        assert (seen == 1).all()
