"""Data-parallel sharding of a varlen batch (host logic; CPU, gloo world size 2).

The sharded path has no exchange in the data path: each rank runs whole
sequences.  These tests check the LPT assignment against brute force, the cost
model's cell counts against the oracle's binning, and that two gloo ranks, each
running its own sequences and gathering the rows, reproduce the single-process
result on every rank.
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


def test_lpt_assigns_every_sequence_once_within_grahams_bound():
    rng = np.random.default_rng(3)
    for world in (2, 3):
        for _ in range(20):
            costs = rng.integers(1, 100, size=7).astype(float)
            owner = shard.lpt_assign(costs, world)
            assert owner.shape == (7,) and owner.min() >= 0 and owner.max() < world
            makespan = max(costs[owner == r].sum() for r in range(world))
            best = min(max(costs[np.array(a) == r].sum() for r in range(world))
                       for a in itertools.product(range(world), repeat=7))
            assert makespan <= (4 / 3 - 1 / (3 * world)) * best + 1e-9


def test_lpt_ties_and_degenerate_worlds():
    assert shard.lpt_assign([5, 5, 5, 5], 2).tolist() == [0, 1, 0, 1]
    assert shard.lpt_assign([1, 2, 3], 1).tolist() == [0, 0, 0]
    assert shard.lpt_assign([], 4).tolist() == []
    assert sorted(shard.lpt_assign([7, 1], 4).tolist()) == [0, 1]  # more ranks than sequences
    with pytest.raises(ValueError):
        shard.lpt_assign([1.0], 0)


def test_cell_counts_match_the_oracle_binning():
    w = W.small_shell(seed=31, R=48, n_prims=2, lo=4.0, hi=10.0, n_keep=700, n_seqs=4, m_cmp=4, m_win=6)
    for m in (w.m_cmp, w.m_win):
        b = O.bin_tokens(w.coords, w.cu_seqlens, m)
        np.testing.assert_array_equal(shard.occupied_cells(w.coords, w.cu_seqlens, m), np.diff(b["cu"]))


def test_local_plans_partition_the_tokens():
    cu = np.array([0, 5, 5, 12, 20, 21], np.int32)  # includes an empty sequence
    owner = shard.lpt_assign(np.diff(cu), 3)
    plans = [shard.local_plan(cu, owner, r) for r in range(3)]
    allt = np.sort(np.concatenate([p.tokens for p in plans]))
    np.testing.assert_array_equal(allt, np.arange(21))
    for p in plans:
        assert p.cu_seqlens[-1] == len(p.tokens)
        for i, s in enumerate(p.seqs):
            np.testing.assert_array_equal(p.tokens[p.cu_seqlens[i]:p.cu_seqlens[i + 1]], np.arange(cu[s], cu[s + 1]))


def _batch():
    w = W.small_shell(seed=41, R=40, n_prims=2, lo=4.0, hi=9.0, n_keep=300, n_seqs=5, hq=4, hkv=2, d=32,
                      m_cmp=4, m_win=4, topk=4, dtype="f32")
    return w, W.make_tensors(w)


def _oracle_out(w, t, coords, cu, rows):
    st = O.forward(coords, cu, t.as_f32("q")[rows], t.as_f32("k")[rows], t.as_f32("v")[rows], t.gates[rows],
                   hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=w.gate_mode,
                   pool_rounding="f32")
    return st["out"]


def _rank_main(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, t = _batch()
        owner = shard.lpt_assign(shard.sequence_costs(w.coords, w.cu_seqlens, w.m_cmp, w.m_win, w.topk), world)
        plan = shard.local_plan(w.cu_seqlens, owner, rank)
        local = _oracle_out(w, t, w.coords[plan.tokens], plan.cu_seqlens, plan.tokens)
        full = shard.gather_rows(torch.from_numpy(local), plan, w.n).numpy()
        ref = _oracle_out(w, t, w.coords, w.cu_seqlens, np.arange(w.n))
        result_q.put((rank, len(plan.seqs), float(np.abs(full - ref).max())))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_reproduce_the_single_process_batch():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_rank_main, args=(2, _free_port(), q), nprocs=2, join=True, start_method="spawn")
    res = sorted(q.get() for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert sum(r[1] for r in res) == 5 and all(r[1] > 0 for r in res)
    for _, _, err in res:
        assert err <= 1e-12, err
