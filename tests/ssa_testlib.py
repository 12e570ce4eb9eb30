"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, and compare.

Tolerances (written here once, used by every parity test):
  * ids, permutations, CSR pointers, Kc/Vc: bit-exact;
  * outputs and gradients: max-abs 2e-2 for bf16 inputs, 1e-4 for fp32;
  * selected blocks: equal, or a certified near-tie -- the set the GPU picked is
    a top-k of the oracle's fp64 selection scores up to TAU_SEL (the GPU ranks
    fp32 scores, so exact ties can resolve differently).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W

ATOL = {"bf16": 2e-2, "f32": 1e-4}
# fp32 scores carry relative errors of ~1e-6 at most; summed probabilities are
# below 1, so 1e-6 absolute bounds the disagreement a rounding order can cause.
TAU_SEL = 1e-6


def pool_rounding(w: W.Workload) -> str:
    return "bf16" if w.dtype == "bf16" else "f32"


def to_torch(a: np.ndarray, dtype: str, dev="cuda") -> torch.Tensor:
    if dtype == "bf16" and a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class DeviceRun:
    """Inputs on the device and the results of one bin/forward/backward pass."""

    def __init__(self, w: W.Workload, t: W.Tensors, backward: bool = True, dev: str = "cuda"):
        self.w = w
        self.coords = torch.from_numpy(np.ascontiguousarray(w.coords, np.int32)).to(dev)
        self.cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
        self.q = to_torch(t.q, w.dtype, dev)
        self.k = to_torch(t.k, w.dtype, dev)
        self.v = to_torch(t.v, w.dtype, dev)
        self.gates = torch.from_numpy(t.gates).to(dev)
        self.dout = to_torch(t.do, w.dtype, dev) if (backward and t.do is not None) else None
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, tdt, w.gate_mode)

    def run(self, backward: bool = True):
        self.blk, self.win = ssa.ssa_bin(self.coords, self.cu, self.w.R, self.w.m_cmp, self.w.m_win)
        self.out, self.saved = ssa.ssa_forward(self.p, self.cu, self.blk, self.win, self.q, self.k, self.v,
                                               self.gates)
        if backward and self.dout is not None:
            self.grads = ssa.ssa_backward(self.p, self.cu, self.blk, self.win, self.q, self.k, self.v,
                                          self.gates, self.saved, self.dout)
        torch.cuda.synchronize()
        status = ssa.device_status()
        assert status == 0, "device check word: %s" % ssa.STATUS_NAMES.get(status, status)
        return self


def bins_np(b: ssa.Bins) -> dict:
    c = b.count
    return {"id": b.id.cpu().numpy(), "perm": b.perm.cpu().numpy(), "ptr": b.ptr[:c + 1].cpu().numpy(),
            "cu": b.cu.cpu().numpy(), "key": b.key[:c].cpu().numpy(), "count": c}


def assert_bins_equal(gpu: ssa.Bins, ref: dict, what: str) -> None:
    g = bins_np(gpu)
    assert g["count"] == ref["count"], (what, g["count"], ref["count"])
    for key in ("id", "perm", "ptr", "cu", "key"):
        np.testing.assert_array_equal(g[key], np.asarray(ref[key]).astype(g[key].dtype), err_msg=what + "." + key)


def run_oracle(w: W.Workload, t: W.Tensors, tokens=None) -> O.State:
    return O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), t.gates,
                     hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=w.gate_mode,
                     pool_rounding=pool_rounding(w), tokens=tokens)


def check_selection(gpu_sel: np.ndarray, st: O.State, tokens, tau: float = TAU_SEL):
    """Returns the list of (t, g) whose GPU selection differs from the oracle's;
    asserts each is a certified near-tie and a well-formed selection."""
    ref = st["sel"]
    flips = []
    cu = st["cu_seqlens"]
    for t in tokens:
        s = int(np.searchsorted(cu, t, side="right") - 1)
        b0, b1 = int(st["blk"]["cu"][s]), int(st["blk"]["cu"][s + 1])
        for g in range(st["hkv"]):
            a = gpu_sel[t, g]
            keff = min(st["topk"], b1 - b0)
            valid = a[:keff]
            assert (a[keff:] == -1).all(), (t, g, a)
            assert (np.diff(valid) > 0).all() and valid.min() >= b0 and valid.max() < b1, (t, g, a)
            if np.array_equal(a, ref[t, g]):
                continue
            imp = O.importance(st, t, g)
            chosen = np.zeros(b1 - b0, bool)
            chosen[valid - b0] = True
            lo = imp[chosen].min()
            hi = imp[~chosen].max() if (~chosen).any() else -np.inf
            assert lo >= hi - tau, ("selection is not a near-tie", t, g, lo, hi)
            flips.append((int(t), int(g)))
    return flips


def max_abs(a, b) -> float:
    d = np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))
    return float(np.nanmax(d)) if d.size else 0.0


def compare_forward(run: DeviceRun, st: O.State, tokens, atol: float):
    """Element-wise parity of Kc/Vc (bit-exact), selection (near-tie rule), the
    three branch outputs, their lse and the combined output on `tokens`."""
    w = run.w
    tokens = np.asarray(tokens)
    b = run.blk.count
    kc = f64(run.saved.kc[:, :b]).transpose(1, 0, 2)
    vc = f64(run.saved.vc[:, :b]).transpose(1, 0, 2)
    np.testing.assert_array_equal(kc, st["kc"], err_msg="Kc")
    np.testing.assert_array_equal(vc, st["vc"], err_msg="Vc")
    sel = run.saved.sel.cpu().numpy()
    flips = check_selection(sel, st, tokens)
    ob = f64(run.saved.o_branch)
    lse = run.saved.lse.cpu().numpy().astype(np.float64)
    out = f64(run.out)
    G = w.hq // w.hkv
    mask = np.zeros((w.n, w.hq), bool)
    mask[tokens] = True
    flip_rows = np.zeros_like(mask)
    for t, g in flips:
        flip_rows[t, g * G:(g + 1) * G] = True
        # the attention itself, over the blocks the GPU picked
        _, o_ = O.attend_with_sel(st, t, g, sel[t, g])
        assert max_abs(ob[1, t, g * G:(g + 1) * G], o_) <= atol
    errs = {}
    for c, name in enumerate(("o_cmp", "o_slc", "o_win")):
        m = mask & ~flip_rows if c == 1 else mask
        errs[name] = max_abs(ob[c][m], st["o"][c][m])
        errs["lse_" + name[2:]] = max_abs(lse[c][m], st["lse"][c][m])
    m = mask & ~flip_rows
    errs["out"] = max_abs(out[m], st["out"][m])
    for key, e in errs.items():
        assert e <= atol, (key, e, atol)
    return errs, flips


def compare_backward(run: DeviceRun, st: O.State, g: dict, atol: float, flips):
    """Gradients; rows / keys touched by a certified selection flip are left out."""
    w = run.w
    dq, dk, dv, dg = (f64(x) for x in run.grads)
    G = w.hq // w.hkv
    rowmask = np.ones((w.n, w.hq), bool)
    keymask = np.ones((w.n, w.hkv), bool)
    sel_gpu = run.saved.sel.cpu().numpy()
    for t, gg in flips:
        rowmask[t, gg * G:(gg + 1) * G] = False
        blocks = set(sel_gpu[t, gg]) ^ set(st["sel"][t, gg])
        for bb in blocks:
            if bb >= 0:
                keymask[st["blk"]["perm"][st["blk"]["ptr"][bb]:st["blk"]["ptr"][bb + 1]], gg] = False
    errs = {"dq": max_abs(dq[rowmask], g["dq"][rowmask]), "dk": max_abs(dk[keymask], g["dk"][keymask]),
            "dv": max_abs(dv[keymask], g["dv"][keymask]), "dgates": max_abs(dg[rowmask], g["dgates"][rowmask])}
    for key, e in errs.items():
        assert e <= atol, (key, e, atol)
    return errs
