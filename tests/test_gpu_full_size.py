"""Parity at the full benchmark sizes, on outputs the oracle can compute one by one.

Each test runs the whole path through the C ABI at the configuration's real size
(the launch configuration the bench times for config 5) and checks:
  * Kc / Vc of every block bit-exact, and the id arrays bit-exact (test_gpu_bin);
  * for sampled query tokens: selection (near-tie rule), the three branch outputs,
    their lse and the combined output; in backward, dQ and dgates of those rows;
  * window-branch dK / dV of sampled windows (window gates one-hot, so the other
    branches contribute exactly zero to dK / dV);
  * properties that hold at any size: sum_i dV_i = sum over rows of (sum_c w_c) dO
    and sum_i dK_i = 0 per KV head.
"""
import dataclasses
import functools

import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, TAU_SEL, DeviceRun, compare_forward, f64, max_abs, run_oracle

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=2)
def _load(cfg: int):
    """Workload and tensors of a configuration, generated once per module.
    Configs 3 and 5 share geometry, heads and seeded tensors (5 adds dO, which
    make_tensors always draws), so 3 reuses 5's."""
    if cfg == 3:
        return _load(5)
    w = W.config(cfg)
    return w, W.make_tensors(w)


def _sample_tokens(w, n_per_seq: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    out = []
    for s in range(w.s):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        if b <= a:
            continue
        pick = rng.choice(np.arange(a, b), size=min(n_per_seq, b - a), replace=False)
        out.append(np.concatenate([[a, b - 1], pick]))
    return np.unique(np.concatenate(out))


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_forward_sampled_rows_at_full_size(cfg):
    w, t = _load(cfg)
    run = DeviceRun(w, t, backward=False).run(backward=False)
    toks = _sample_tokens(w, 48 if w.s == 1 else 16, seed=cfg)
    st = run_oracle(w, t, tokens=toks)
    errs, flips = compare_forward(run, st, toks, ATOL[w.dtype])
    print(cfg, w.n, len(toks), errs, "flips", len(flips))


def test_backward_sampled_rows_and_sums_at_full_size():
    w, t = _load(5)
    run = DeviceRun(w, t).run()
    toks = _sample_tokens(w, 32, seed=55)
    st = run_oracle(w, t, tokens=toks)
    _, flips = compare_forward(run, st, toks, ATOL[w.dtype])
    flipped = {tt for tt, _ in flips}
    keep = np.array([tt for tt in toks if tt not in flipped])
    do = t.as_f32("do").astype(np.float64)
    dq, dk, dv, dg = (f64(x) for x in run.grads)
    e_dq = max_abs(dq[keep], O.dq_rows(st, do, keep))
    e_dg = max_abs(dg[keep], O.dgates_rows(st, do, keep))
    assert e_dq <= ATOL[w.dtype] and e_dg <= ATOL[w.dtype], (e_dq, e_dg)

    # sums over all tokens.  Softmax rows sum to one in every branch, so
    # sum_i dV_i = sum_rows (sum_c w_c) dO and sum_i dK_i = 0 (the compressed
    # branch included: sum_i dKc_b(i)/n_b = sum_b dKc_b).  The GPU multiplies
    # bf16-rounded P and dS in some tiles; each term then carries a relative
    # error below 2^-9 with independent signs, and sum_j p_j^2 <= 1 per row, so
    # 4 sigma of the rounding noise is below 4 * 2^-9 / sqrt(3) * sqrt(sum_rows
    # |w dO|^2) for dV; dK gets the same bound in terms of its own rows.
    gw = O.gate_weights(t.gates, w.gate_mode)
    G = w.hq // w.hkv
    for g in range(w.hkv):
        hs = slice(g * G, (g + 1) * G)
        wsum = gw[:, hs, :].sum(-1)
        want = np.einsum("nh,nhd->d", wsum, do[:, hs, :])
        noise = np.sqrt(np.einsum("nh,nhd->d", wsum ** 2, do[:, hs, :] ** 2))
        tol_v = 2e-2 + 4 * 2.0 ** -9 / np.sqrt(3) * noise
        assert (np.abs(dv[:, g, :].sum(0) - want) <= tol_v).all(), (g, np.abs(dv[:, g, :].sum(0) - want).max())
        tol_k = 2e-2 + 4 * 2.0 ** -9 / np.sqrt(3) * np.sqrt((dk[:, g, :] ** 2).sum(0))
        assert (np.abs(dk[:, g, :].sum(0)) <= tol_k).all(), (g, np.abs(dk[:, g, :].sum(0)).max())


def test_window_gradients_of_sampled_windows_at_full_size():
    w, t = _load(5)
    w = dataclasses.replace(w, gate_mode=0)
    gates = np.zeros_like(t.gates)
    gates[:, :, 2] = 1.0  # window branch only: the other branches add exact zeros to dK / dV
    t = dataclasses.replace(t, gates=gates)
    run = DeviceRun(w, t).run()
    wb = O.bin_tokens(w.coords, w.cu_seqlens, w.m_win)
    sizes = np.diff(wb["ptr"])
    rng = np.random.default_rng(7)
    wins = np.unique(np.concatenate([np.argsort(-sizes, kind="stable")[:4], rng.choice(len(sizes), 12, replace=False)]))
    members = np.concatenate([wb["perm"][wb["ptr"][x]:wb["ptr"][x + 1]] for x in wins])
    st = run_oracle(w, t, tokens=np.unique(members))
    do = t.as_f32("do").astype(np.float64)
    tk, dk_ref, dv_ref = O.window_kv_grads(st, do, wins)
    dq, dk, dv, _ = (f64(x) for x in run.grads)
    e = {"dk": max_abs(dk[tk], dk_ref), "dv": max_abs(dv[tk], dv_ref),
         "dq": max_abs(dq[tk], O.dq_rows(st, do, tk))}
    print(len(wins), sizes[wins].max(), e)
    for key, val in e.items():
        assert val <= ATOL[w.dtype], (key, val)


# ----------------------------------------------------------------------------
# the compressed branch for every token at the benchmark size, and the selected
# branch's key gradients of sampled blocks
# ----------------------------------------------------------------------------


def _one_hot(t, c):
    gates = np.zeros_like(t.gates)
    gates[:, :, c] = 1.0
    return dataclasses.replace(t, gates=gates)


@functools.lru_cache(maxsize=1)
def _cmp_only_run():
    """Config 5 with the compressed branch alone switched on (gate weights one-hot,
    so the other branches add exact zeros to out, dQ, dK and dV): the GPU's
    results and the oracle's compressed branch over all 131072 query tokens."""
    from tests import cmp_full

    w, t = _load(5)
    w = dataclasses.replace(w, gate_mode=0)
    t = _one_hot(t, 0)
    run = DeviceRun(w, t).run()
    blk = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)
    kc = O.mean_pool(t.as_f32("k").astype(np.float64), blk, "bf16")
    vc = O.mean_pool(t.as_f32("v").astype(np.float64), blk, "bf16")
    dq, dk, dv, dg = (x.cpu().numpy() for x in run.grads)
    arrays = {"q": t.q, "do": t.do, "gates": t.gates, "kc": kc, "vc": vc,
              "sel_gpu": run.saved.sel.cpu().numpy(), "o_cmp_gpu": run.saved.o_branch[0].cpu().numpy(),
              "lse_gpu": run.saved.lse[0].cpu().numpy(), "dq_gpu": dq, "dgates_gpu": dg,
              "out_gpu": run.out.view(torch.int16).cpu().numpy().view(np.uint16)}
    meta = {"blk_cu": blk["cu"], "cu": np.asarray(w.cu_seqlens, np.int64), "hq": w.hq, "hkv": w.hkv,
            "topk": w.topk, "gate_mode": 0}
    res = cmp_full.run(arrays, meta, w.n)
    return w, t, blk, run, res, dk, dv


def test_compressed_branch_every_token_at_full_size():
    """Config 5 (131072 tokens, 2322 blocks, 9.7e9 compressed scores), compressed
    branch only: lse, o_cmp, out, dQ and dgates of every query row, the selection of
    every (token, group) (equal, or a certified near-tie), and dK / dV of every
    token element by element against the oracle at 2e-2."""
    w, t, blk, run, res, dk, dv = _cmp_only_run()
    tol = ATOL[w.dtype]
    flips = res["flips"]
    assert res["bad_sel_rows"] == 0
    assert all(gap >= -TAU_SEL for _, _, gap in flips), [f for f in flips if f[2] < -TAU_SEL][:5]
    dk_ref, dv_ref = O.cmp_token_grads(res["dkc"], res["dvc"], blk)
    errs = {key: res[key] for key in ("o", "lse", "out", "dq", "dgates_cmp")}
    errs["dk"] = max_abs(dk, dk_ref)
    errs["dv"] = max_abs(dv, dv_ref)
    print("every token:", errs, "flips", len(flips), "of", w.n * w.hkv, "procs", res["procs"],
          "max |dK|, |dV|", float(np.abs(dk_ref).max()), float(np.abs(dv_ref).max()))
    for key, e in errs.items():
        assert e <= tol, (key, e, tol)


def test_selected_branch_key_gradients_of_sampled_blocks_at_full_size():
    """Config 5 with the selected branch alone switched on: dK / dV of every token
    of 16 blocks (the 4 most selected, 4 more that are selected, 8 at random, some of
    them selected by nobody, whose gradient must be exactly zero), each against the
    sum over all (token, group) rows whose selection holds the block.  The rows use
    the GPU's selection, which the compressed-branch test certifies."""
    w, t = _load(5)
    w = dataclasses.replace(w, gate_mode=0)
    t = _one_hot(t, 1)
    run = DeviceRun(w, t).run()
    sel = run.saved.sel.cpu().numpy()
    blk = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)
    counts = np.bincount(sel[sel >= 0], minlength=blk["count"])
    rng = np.random.default_rng(9)
    chosen = list(np.argsort(-counts, kind="stable")[:4])
    used = np.nonzero(counts)[0]
    chosen += list(rng.choice(used, 4, replace=False))
    chosen += list(rng.choice(blk["count"], 8, replace=False))
    chosen = sorted(set(int(b) for b in chosen))
    q, k, v, do = (t.as_f32(x).astype(np.float64) for x in ("q", "k", "v", "do"))
    G = w.hq // w.hkv
    scale = 1.0 / np.sqrt(w.d)
    dk_ref = {b: np.zeros((blk["ptr"][b + 1] - blk["ptr"][b], w.hkv, w.d)) for b in chosen}
    dv_ref = {b: np.zeros_like(dk_ref[b]) for b in chosen}
    want = set(chosen)
    rows_seen = 0
    tt_all, gg_all = np.nonzero(np.isin(sel, chosen).any(axis=2))
    for tt, g in zip(tt_all, gg_all):
        row = sel[tt, g]
        js = O.selected_tokens(row, blk)
        hs = slice(g * G, (g + 1) * G)
        s_ = scale * (q[tt, hs] @ k[js, g].T)
        p = np.exp(s_ - O._logsumexp(s_, -1)[:, None])
        dp = do[tt, hs] @ v[js, g].T
        ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
        dkj = scale * (ds.T @ q[tt, hs])
        dvj = p.T @ do[tt, hs]
        off = 0
        for b in row:
            if b < 0:
                continue
            nb = int(blk["ptr"][b + 1] - blk["ptr"][b])
            if b in want:
                dk_ref[b][:, g] += dkj[off:off + nb]
                dv_ref[b][:, g] += dvj[off:off + nb]
            off += nb
        rows_seen += 1
    dk, dv = (x.cpu().numpy() for x in run.grads[1:3])
    errs = {}
    for b in chosen:
        members = blk["perm"][blk["ptr"][b]:blk["ptr"][b + 1]]
        errs[b] = (max_abs(dk[members], dk_ref[b]), max_abs(dv[members], dv_ref[b]), int(counts[b]))
        if counts[b] == 0:
            assert not dk[members].any() and not dv[members].any(), b
    print("selected blocks (dk err, dv err, rows):", errs, "rows", rows_seen)
    for b, (ek, ev, _) in errs.items():
        assert ek <= ATOL[w.dtype] and ev <= ATOL[w.dtype], (b, ek, ev)
