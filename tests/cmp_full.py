"""Driver of the full-size compressed-branch parity check (test infrastructure).

The oracle's `cmp_branch_range` computes the compressed branch of any range of
query tokens on its own, so the benchmark's 131072 queries are split into ranges
and run in a pool of processes (started with `spawn`; each process uses one BLAS
thread).  Inputs and the GPU's results reach the workers as memory-mapped .npy
files; each worker compares its own rows and returns the error maxima, the rows
whose selection differs from the oracle's (with the oracle's score gap of the
GPU's choice) and its partial sums of dKc / dVc.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import tempfile

import numpy as np

from spatial_sparse_attention_ssa_b200 import workloads as W


class _BF16Rows:
    """Read-only view of a bf16-bits array [N, ...] that converts the rows it returns."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, idx):
        if not isinstance(idx, tuple):
            idx = (idx,)
        rows = W.bf16_bits_to_f32(np.asarray(self.bits[idx[0]]))
        return rows[(slice(None),) + tuple(idx[1:])]


def _max_abs(a, b) -> float:
    d = np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))
    return float(d.max()) if d.size else 0.0


def _work(job):
    path, meta, t0, t1 = job
    from threadpoolctl import threadpool_limits

    from oracle import ssa_oracle as O

    with threadpool_limits(1):
        ld = lambda name: np.load(os.path.join(path, name + ".npy"), mmap_mode="r")  # noqa: E731
        q, do = _BF16Rows(ld("q")), _BF16Rows(ld("do"))
        gates = np.asarray(ld("gates")[t0:t1])
        # the range function indexes gates by absolute token: give it a full-size view
        gfull = ld("gates")
        sel_gpu = np.asarray(ld("sel_gpu")[t0:t1])
        r = O.cmp_branch_range(q, np.asarray(ld("kc")), np.asarray(ld("vc")), meta["blk_cu"], meta["cu"], gfull,
                               hq=meta["hq"], hkv=meta["hkv"], topk=meta["topk"], gate_mode=meta["gate_mode"],
                               t0=t0, t1=t1, dout=do, sel_other=sel_gpu)
        out = {"t0": t0, "t1": t1, "dkc": r["dkc"], "dvc": r["dvc"]}
        o_gpu = np.asarray(ld("o_cmp_gpu")[t0:t1])
        out["o"] = _max_abs(o_gpu, r["o"])
        out["lse"] = _max_abs(np.asarray(ld("lse_gpu")[t0:t1]), r["lse"])
        out["dq"] = _max_abs(np.asarray(ld("dq_gpu")[t0:t1]), r["dq"])
        out["out"] = _max_abs(W.bf16_bits_to_f32(np.asarray(ld("out_gpu")[t0:t1])), r["o"])
        dot = np.einsum("nhd,nhd->nh", do[np.arange(t0, t1)].astype(np.float64), r["o"])
        w = O.gate_weights(gates[:, :, 0], meta["gate_mode"])
        dg = dot if meta["gate_mode"] == 0 else dot * w * (1.0 - w)
        out["dgates_cmp"] = _max_abs(np.asarray(ld("dgates_gpu")[t0:t1, :, 0]), dg)
        diff = (sel_gpu != r["sel"]).any(axis=2)
        tt, gg = np.nonzero(diff)
        out["flips"] = [(int(t0 + a), int(b), float(r["other_gap"][a, b])) for a, b in zip(tt, gg)]
        # structure of the GPU's selection: ascending ids of the token's sequence, -1 padded
        bad = 0
        seq = np.searchsorted(meta["cu"], np.arange(t0, t1), side="right") - 1
        b0, b1 = meta["blk_cu"][seq], meta["blk_cu"][seq + 1]
        keff = np.minimum(meta["topk"], b1 - b0)
        for i in range(t1 - t0):
            for g in range(meta["hkv"]):
                row = sel_gpu[i, g]
                k = int(keff[i])
                ok = (row[k:] == -1).all() and (np.diff(row[:k]) > 0).all() and k > 0 and \
                    row[0] >= b0[i] and row[k - 1] < b1[i]
                bad += 0 if ok else 1
        out["bad_sel_rows"] = bad
    return out


def run(arrays: dict, meta: dict, n: int, procs: int | None = None, pieces_per_proc: int = 4) -> dict:
    """Run the oracle over all n query tokens in a spawn pool; returns the merged
    error maxima, flips, bad-row count and the summed dkc / dvc."""
    if procs is None:
        try:
            procs = len(os.sched_getaffinity(0))
        except AttributeError:
            procs = os.cpu_count() or 1
        procs = max(1, min(64, procs))
    with tempfile.TemporaryDirectory(prefix="ssa_cmp_full_") as path:
        for name, a in arrays.items():
            np.save(os.path.join(path, name + ".npy"), a)
        step = max(1, -(-n // (procs * pieces_per_proc)))
        jobs = [(path, meta, a, min(n, a + step)) for a in range(0, n, step)]
        ctx = mp.get_context("spawn")
        with ctx.Pool(procs) as pool:
            results = list(pool.imap_unordered(_work, jobs))
    merged = {"flips": [], "bad_sel_rows": 0}
    for key in ("o", "lse", "dq", "out", "dgates_cmp"):
        merged[key] = max(r[key] for r in results)
    merged["dkc"] = sum(r["dkc"] for r in results)
    merged["dvc"] = sum(r["dvc"] for r in results)
    for r in results:
        merged["flips"] += r["flips"]
        merged["bad_sel_rows"] += r["bad_sel_rows"]
    merged["procs"] = procs
    return merged
