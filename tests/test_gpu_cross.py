"""Cross-attention SSA on the GPU against the oracle (queries from another token set).

The voxel tokens are binned by ssa_bin as usual; the queries (image tokens in LSRM's
cross attention) attend them through the compressed and selected branches.
Compared element by element on every query row: the two branch outputs and their
lse, the combined output, the selection (equal, or a certified near-tie as in the
self-attention tests), and dQ, dK, dV, dgates.  Covered: the tensor-core and MMA
kernels (bf16, d = 64, G = 8 and 16), the SIMT kernels (fp32, d = 32), sequences
with more queries than voxels and the reverse, a sequence without queries, and the
rejection of a sequence that has queries but no voxel tokens.
"""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, TAU_SEL, f64, max_abs, pool_rounding, to_torch

pytestmark = pytest.mark.gpu


def _run(w, t, cq, backward=True):
    dev = "cuda"
    coords = torch.from_numpy(np.ascontiguousarray(w.coords, np.int32)).to(dev)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
    q_cu = torch.from_numpy(cq.q_cu.astype(np.int32)).to(dev)
    q, k, v = to_torch(cq.q, w.dtype), to_torch(t.k, w.dtype), to_torch(t.v, w.dtype)
    gates = torch.from_numpy(cq.gates).to(dev)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, tdt, w.gate_mode)
    blk, _ = ssa.ssa_bin(coords, cu, w.R, w.m_cmp, w.m_win)
    out, saved = ssa.ssa_cross_forward(p, q_cu, blk, q, k, v, gates)
    grads = None
    if backward:
        grads = ssa.ssa_cross_backward(p, q_cu, blk, q, k, v, gates, saved, to_torch(cq.do, w.dtype))
    torch.cuda.synchronize()
    assert ssa.device_status() == 0
    return out, saved, grads


def _oracle(w, t, cq):
    st = O.cross_forward(cq.q_cu, w.coords, w.cu_seqlens, cq.as_f32("q"), t.as_f32("k"), t.as_f32("v"), cq.gates,
                         hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, topk=w.topk, gate_mode=w.gate_mode,
                         pool_rounding=pool_rounding(w))
    return st, O.cross_backward(st, cq.as_f32("do").astype(np.float64))


def _flips(sel, st, tau=TAU_SEL):
    """(t, g) whose GPU selection differs from the oracle's; each must be a
    well-formed selection and a certified near-tie of the oracle's scores."""
    out = []
    q_cu, bcu = st["q_cu"], st["blk"]["cu"]
    G = st["G"]
    for t in range(sel.shape[0]):
        s = int(np.searchsorted(q_cu, t, side="right") - 1)
        b0, b1 = int(bcu[s]), int(bcu[s + 1])
        for g in range(st["hkv"]):
            a = sel[t, g]
            if np.array_equal(a, st["sel"][t, g]):
                continue
            keff = min(st["topk"], b1 - b0)
            valid = a[:keff]
            assert (a[keff:] == -1).all() and (np.diff(valid) > 0).all(), (t, g, a)
            assert valid.min() >= b0 and valid.max() < b1, (t, g, a)
            hs = slice(g * G, (g + 1) * G)
            _, _, p = O.cmp_attention(np.asarray(st["q"][t:t + 1, hs, :], np.float64), st["kc"][b0:b1, g, :],
                                      st["vc"][b0:b1, g, :], st["scale"])
            imp = p[0].sum(axis=0)
            chosen = np.zeros(b1 - b0, bool)
            chosen[valid - b0] = True
            hi = imp[~chosen].max() if (~chosen).any() else -np.inf
            assert imp[chosen].min() >= hi - tau, ("not a near-tie", t, g)
            out.append((t, g))
    return out


def _compare(w, out, saved, grads, st, gr):
    atol = ATOL[w.dtype]
    sel = saved.sel.cpu().numpy()
    flips = _flips(sel, st)
    G = w.hq // w.hkv
    rows = np.ones(st["o"].shape[1:3], bool)
    keys = np.ones((st["k"].shape[0], w.hkv), bool)
    blk = st["blk"]
    for t, g in flips:
        rows[t, g * G:(g + 1) * G] = False
        for b in set(sel[t, g]) ^ set(st["sel"][t, g]):
            if b >= 0:
                keys[blk["perm"][blk["ptr"][b]:blk["ptr"][b + 1]], g] = False
    ob = f64(saved.o_branch)
    lse = saved.lse.cpu().numpy().astype(np.float64)
    errs = {"o_cmp": max_abs(ob[0], st["o"][0]), "lse_cmp": max_abs(lse[0], st["lse"][0]),
            "o_slc": max_abs(ob[1][rows], st["o"][1][rows]), "lse_slc": max_abs(lse[1][rows], st["lse"][1][rows]),
            "out": max_abs(f64(out)[rows], st["out"][rows])}
    if grads is not None:
        dq, dk, dv, dg = (f64(x) for x in grads)
        errs.update({"dq": max_abs(dq[rows], gr["dq"][rows]), "dk": max_abs(dk[keys], gr["dk"][keys]),
                     "dv": max_abs(dv[keys], gr["dv"][keys]), "dgates": max_abs(dg[rows], gr["dgates"][rows])})
    for key, e in errs.items():
        assert e <= atol, (key, e, atol)
    return errs, flips


@pytest.mark.parametrize("hq,d,dtype", [(16, 64, "bf16"), (32, 64, "bf16"), (4, 32, "f32")])
def test_cross_forward_backward_matches_oracle(hq, d, dtype):
    w = W.small_shell(seed=37, R=40, n_prims=2, lo=4.0, hi=9.0, n_keep=600, n_seqs=3, hq=hq, hkv=2, d=d,
                      m_cmp=4, m_win=4, topk=8, dtype=dtype)
    t = W.make_tensors(w)
    cq = W.make_cross_queries(w, [900, 0, 150], seed=1)  # more queries than voxels, none, fewer
    out, saved, grads = _run(w, t, cq)
    st, gr = _oracle(w, t, cq)
    errs, flips = _compare(w, out, saved, grads, st, gr)
    print(errs, "flips", len(flips))
    if dtype == "f32":
        assert not flips


def test_cross_rejects_a_sequence_with_queries_and_no_voxels():
    w = W.small_shell(seed=41, R=32, n_prims=1, lo=4.0, hi=8.0, n_keep=300, n_seqs=2, m_cmp=4, m_win=4, topk=4)
    t = W.make_tensors(w)
    a = int(w.cu_seqlens[1])
    w2 = W.Workload(**{**w.__dict__, "coords": w.coords[:a], "cu_seqlens": np.array([0, a, a], np.int64)})
    cq = W.make_cross_queries(w2, [10, 5], seed=2)  # sequence 1 has queries but no voxel tokens
    t2 = W.Tensors(t.q[:a], t.k[:a], t.v[:a], t.gates[:a], t.do[:a], t.dtype)
    with pytest.raises(ssa.SSAError):
        _run(w2, t2, cq, backward=False)
    assert ssa.device_status() == 0


def test_cross_at_benchmark_size_sampled_rows_and_sum_rules():
    """131072 image-token queries against the 131072 voxel tokens of the benchmark
    shell (the bench's cross-attention leg): sampled query rows element by element,
    and over every row the sum rules of the key gradients (softmax rows sum to one in
    both branches: sum_i dV_i = sum_rows (w_cmp + w_slc) dO, sum_i dK_i = 0 per KV
    head; 4-sigma bound on independent bf16 rounding as in the self-attention test)."""
    w = W.config(5)
    assert w.s == 1
    t = W.make_tensors(w)
    cq = W.make_cross_queries(w, [w.n], seed=3)
    out, saved, grads = _run(w, t, cq)
    rng = np.random.default_rng(21)
    toks = np.unique(np.concatenate([[0, w.n - 1], rng.choice(w.n, 62, replace=False)]))
    st = O.cross_forward(cq.q_cu, w.coords, w.cu_seqlens, cq.as_f32("q"), t.as_f32("k"), t.as_f32("v"), cq.gates,
                         hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, topk=w.topk, gate_mode=w.gate_mode,
                         pool_rounding=pool_rounding(w), tokens=toks)
    atol = ATOL[w.dtype]
    sel = saved.sel.cpu().numpy()
    G = w.hq // w.hkv
    b0, b1 = 0, int(st["blk"]["count"])
    ob = f64(saved.o_branch)
    lse = saved.lse.cpu().numpy().astype(np.float64)
    o = f64(out)
    flips = 0
    for tt in toks:
        np.testing.assert_allclose(ob[0, tt], st["o"][0, tt], rtol=0, atol=atol)
        np.testing.assert_allclose(lse[0, tt], st["lse"][0, tt], rtol=0, atol=atol)
        for g in range(w.hkv):
            hs = slice(g * G, (g + 1) * G)
            if not np.array_equal(sel[tt, g], st["sel"][tt, g]):  # must be a certified near-tie
                _, _, p = O.cmp_attention(np.asarray(st["q"][tt:tt + 1, hs, :], np.float64), st["kc"][b0:b1, g, :],
                                          st["vc"][b0:b1, g, :], st["scale"])
                imp = p[0].sum(axis=0)
                chosen = np.zeros(b1 - b0, bool)
                chosen[sel[tt, g][sel[tt, g] >= 0]] = True
                assert imp[chosen].min() >= imp[~chosen].max() - TAU_SEL, (tt, g)
                flips += 1
                continue
            np.testing.assert_allclose(ob[1, tt, hs], st["o"][1, tt, hs], rtol=0, atol=atol)
            np.testing.assert_allclose(lse[1, tt, hs], st["lse"][1, tt, hs], rtol=0, atol=atol)
            np.testing.assert_allclose(o[tt, hs], st["out"][tt, hs], rtol=0, atol=atol)
    dq, dk, dv, _ = (f64(x) for x in grads)
    do = cq.as_f32("do").astype(np.float64)
    gw = O.gate_weights(cq.gates, w.gate_mode)
    for g in range(w.hkv):
        hs = slice(g * G, (g + 1) * G)
        wsum = gw[:, hs, :].sum(-1)
        want = np.einsum("nh,nhd->d", wsum, do[:, hs, :])
        noise = np.sqrt(np.einsum("nh,nhd->d", wsum ** 2, do[:, hs, :] ** 2))
        assert (np.abs(dv[:, g, :].sum(0) - want) <= 2e-2 + 4 * 2.0 ** -9 / np.sqrt(3) * noise).all(), g
        tol_k = 2e-2 + 4 * 2.0 ** -9 / np.sqrt(3) * np.sqrt((dk[:, g, :] ** 2).sum(0))
        assert (np.abs(dk[:, g, :].sum(0)) <= tol_k).all(), g
    print("flips", flips, "of", len(toks) * w.hkv)
