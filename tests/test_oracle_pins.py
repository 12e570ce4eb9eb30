"""Pins of the CPU oracle against what the pages and the mathematics fix.

The oracle is the plain definition of SSA (Direct3D-S2, hyper.ai, section
"方法"), written in numpy fp64.  These tests pin it to things other than
itself: hand-computed grids, reductions to textbook full attention
(torch's scaled_dot_product_attention), brute force on tiny inputs, exact
invariants, finite differences and torch autograd on an independent
dense-mask re-expression of the forward.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(seed, n_per_seq=(90, 0, 57), R=16, hq=4, hkv=2, d=16, unique=True, dtype=np.float64):
    rng = np.random.default_rng(seed)
    coords = []
    for n in n_per_seq:
        if unique:
            flat = rng.choice(R ** 3, size=n, replace=False)
            c = np.stack(np.unravel_index(flat, (R, R, R)), axis=-1)
        else:
            c = rng.integers(0, R, size=(n, 3))
        coords.append(c)
    coords = np.concatenate(coords).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(n_per_seq)]).astype(np.int64)
    n = len(coords)
    q = rng.standard_normal((n, hq, d)).astype(dtype)
    k = rng.standard_normal((n, hkv, d)).astype(dtype)
    v = rng.standard_normal((n, hkv, d)).astype(dtype)
    gates = rng.standard_normal((n, hq, 3))
    return coords, cu, q, k, v, gates


def _sdpa_full(q, k, v, cu, hq, hkv):
    """Textbook full attention per sequence (torch, fp64, GQA by repeating KV heads)."""
    out = np.zeros_like(q)
    G = hq // hkv
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if a == b:
            continue
        qt = torch.from_numpy(q[a:b]).transpose(0, 1)  # [H, L, d]
        kt = torch.from_numpy(k[a:b]).transpose(0, 1).repeat_interleave(G, 0)
        vt = torch.from_numpy(v[a:b]).transpose(0, 1).repeat_interleave(G, 0)
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
        out[a:b] = o.transpose(0, 1).numpy()
    return out


# ----------------------------------------------------------------------------
# P4 / P12: binning and mean pooling on hand-computed grids
# ----------------------------------------------------------------------------


def test_mean_pool_hand_grids():
    with open(os.path.join(GOLDEN, "mean_pool_hand.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        coords = np.array(c["coords"], np.int32)
        k = np.array(c["k"], np.float64)[:, None, :]  # [N, 1, d]
        blk = O.bin_tokens(coords, np.array([0, len(coords)]), c["m"])
        assert blk["id"].tolist() == c["expect_ids"], c["name"]
        assert blk["ptr"].tolist() == c["expect_ptr"], c["name"]
        kc = O.mean_pool(k, blk, c["rounding"])[:, 0, :]
        np.testing.assert_array_equal(kc, np.array(c["expect_kc"]), err_msg=c["name"])


def test_mean_pool_full_block_of_512():
    # one full 8^3 block; K_i = i mod 16 -> sum = 32 * 120 = 3840, mean 7.5 (exact in bf16)
    g = np.stack(np.meshgrid(np.arange(8), np.arange(8), np.arange(8), indexing="ij"), -1).reshape(-1, 3)
    k = (np.arange(512) % 16).astype(np.float64)[:, None, None]
    blk = O.bin_tokens(g, np.array([0, 512]), 8)
    assert blk["count"] == 1
    assert O.mean_pool(k, blk, "bf16")[0, 0, 0] == 7.5
    # block sizes 1..512 at m = 8: a staircase where block b holds b+1 tokens of value b+1
    coords, vals = [], []
    for b in range(8):
        for j in range(b * 60 + 1):
            coords.append((8 * b + (j // 64) % 8, (j // 8) % 8, j % 8))
            vals.append(b + 1.0)
    coords = np.array(coords)
    blk = O.bin_tokens(coords, np.array([0, len(coords)]), 8)
    kc = O.mean_pool(np.array(vals)[:, None, None], blk, "bf16")[:, 0, 0]
    np.testing.assert_array_equal(kc, np.arange(1, 9, dtype=np.float64))
    np.testing.assert_array_equal(np.diff(blk["ptr"]), [b * 60 + 1 for b in range(8)])


def _brute_bins(coords, cu, m):
    ids = [None] * len(coords)
    base = 0
    cu_out = [0]
    for s in range(len(cu) - 1):
        toks = range(int(cu[s]), int(cu[s + 1]))
        cells = sorted({tuple(int(c) // m for c in coords[t]) for t in toks})
        index = {c: i for i, c in enumerate(cells)}
        for t in toks:
            ids[t] = base + index[tuple(int(c) // m for c in coords[t])]
        base += len(cells)
        cu_out.append(base)
    perm = sorted(range(len(coords)), key=lambda t: (ids[t], t))
    return ids, perm, cu_out


@pytest.mark.parametrize("m", [1, 2, 3, 5, 16])
def test_bin_brute_force(m):
    rng = np.random.default_rng(m)
    lens = [37, 0, 1, 64, 11]
    coords = rng.integers(0, 13, size=(sum(lens), 3))  # duplicates allowed
    cu = np.concatenate([[0], np.cumsum(lens)])
    blk = O.bin_tokens(coords, cu, m)
    ids, perm, cu_out = _brute_bins(coords, cu, m)
    assert blk["id"].tolist() == ids
    assert blk["perm"].tolist() == perm
    assert blk["cu"].tolist() == cu_out
    for b in range(blk["count"]):
        members = blk["perm"][blk["ptr"][b]:blk["ptr"][b + 1]]
        assert all(ids[t] == b for t in members)
        assert (coords[members] // m == blk["key"][b]).all()


# ----------------------------------------------------------------------------
# P1 / P2 / P3: each branch reduces to textbook full attention
# ----------------------------------------------------------------------------


def test_selection_covering_everything_is_full_attention():
    coords, cu, q, k, v, gates = _rand_case(1)
    st = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, m_win=4, topk=10_000,
                   gate_mode=1)
    full = _sdpa_full(q, k, v, cu, 4, 2)
    np.testing.assert_allclose(st["o"][1], full, rtol=1e-12, atol=1e-12)


def test_window_covering_grid_is_full_attention():
    coords, cu, q, k, v, gates = _rand_case(2)
    st = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, m_win=16, topk=3,
                   gate_mode=1)
    full = _sdpa_full(q, k, v, cu, 4, 2)
    np.testing.assert_allclose(st["o"][2], full, rtol=1e-12, atol=1e-12)
    # a window of 1 holds only the query's own token (unique coords): o_win = v_t
    st1 = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, m_win=1, topk=3,
                    gate_mode=1)
    np.testing.assert_allclose(st1["o"][2], np.repeat(v, 2, axis=1), rtol=0, atol=1e-15)


def test_unit_blocks_make_compression_full_attention():
    coords, cu, q, k, v, gates = _rand_case(3)
    for rounding in ("f32", "none"):
        kq = k.astype(np.float32).astype(np.float64)  # fp32-representable: mean of one = itself
        vq = v.astype(np.float32).astype(np.float64)
        st = O.forward(coords, cu, q, kq, vq, gates, hq=4, hkv=2, m_cmp=1, m_win=2, topk=5,
                       gate_mode=1, pool_rounding=rounding)
        full = _sdpa_full(q, kq, vq, cu, 4, 2)
        np.testing.assert_allclose(st["o"][0], full, rtol=1e-12, atol=1e-12)
        # with unit blocks, the selection ranks single tokens by summed probability
        t, g = 5, 1
        s = (q[t, 2:4] @ kq[: 90, g].T) / 4.0
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        top = sorted(np.argsort(-p.sum(0), kind="stable")[:5])
        blk_of_token = st["blk"]["id"][:90]
        assert sorted(blk_of_token[top].tolist()) == st["sel"][t, g].tolist()


# ----------------------------------------------------------------------------
# P5: top-k against brute force, worked example, exact ties
# ----------------------------------------------------------------------------


def test_topk_brute_force_tiny():
    coords, cu, q, k, v, gates = _rand_case(4, n_per_seq=(40, 25), R=8)
    st = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=2, m_win=2, topk=3, gate_mode=1)
    blk = st["blk"]
    for t in range(len(coords)):
        s = 0 if t < 40 else 1
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        for g in range(2):
            imp = []
            for b in range(b0, b1):
                tot = 0.0
                for h in (2 * g, 2 * g + 1):
                    scores = [sum(q[t, h, i] * st["kc"][bb, g, i] for i in range(16)) / 4.0
                              for bb in range(b0, b1)]
                    mx = max(scores)
                    z = sum(math.exp(x - mx) for x in scores)
                    tot += math.exp(scores[b - b0] - mx) / z
                imp.append((-tot, b))
            want = sorted(b for _, b in sorted(imp)[:3])
            assert st["sel"][t, g].tolist() == want


def test_selection_worked_example():
    """Hand example: G = 2 heads, 3 single-token blocks, d = 2, scale 1.

    head 0: q = (1, 0); head 1: q = (0, 1); keys A = (4, 0), B = (0, 2), C = (1.5, 1.5).
    head 0 scores (4, 0, 1.5) -> probs ~ (0.909, 0.017, 0.075)
    head 1 scores (0, 2, 1.5) -> probs ~ (0.078, 0.574, 0.348)
    summed probs ~ (0.987, 0.591, 0.423): top-2 = {A, B}.
    (Summing raw scores would give (4, 2, 3) -> {A, C}; one head alone gives
    {A, C} for head 0.)  So the group sum of softmax probabilities is what picks B.
    """
    coords = np.array([[0, 0, 0], [1, 0, 0], [2, 0, 0], [3, 0, 0]], np.int32)  # A, B, C, query D
    # the query's own block D has key (0, 0): score 0 for both heads, probabilities
    # head 0 ~ (0.894, 0.016, 0.073, 0.016), head 1 ~ (0.072, 0.533, 0.323, 0.072)
    k = np.array([[4.0, 0.0], [0.0, 2.0], [1.5, 1.5], [0.0, 0.0]])[:, None, :]
    v = np.zeros_like(k)
    q = np.zeros((4, 2, 2))
    q[3, 0] = (1.0, 0.0)
    q[3, 1] = (0.0, 1.0)
    gates = np.zeros((4, 2, 3))
    # m_cmp = 1 puts each token in its own block
    st = O.forward(coords, np.array([0, 4]), q, k, v, gates, hq=2, hkv=1, m_cmp=1, m_win=1,
                   topk=2, gate_mode=0, scale=1.0, pool_rounding="none")
    assert st["sel"][3, 0].tolist() == [0, 1]
    imp = O.importance(st, 3, 0)
    assert imp[0] > imp[1] > imp[2] > imp[3]
    np.testing.assert_allclose(imp, [0.96600, 0.54907, 0.39647, 0.08846], atol=5e-5)


def test_topk_exact_ties_go_to_lower_id():
    # blocks 0..3 with identical keys: identical scores for every head -> ties; k = 2 keeps 0, 1
    coords = np.array([[0, 0, 0], [2, 0, 0], [4, 0, 0], [6, 0, 0], [8, 0, 0]], np.int32)
    k = np.ones((5, 1, 4))
    k[4] = -5.0  # the query's own block scores lowest
    rng = np.random.default_rng(0)
    q = rng.standard_normal((5, 2, 4))
    q[4] = np.abs(q[4])
    st = O.forward(coords, np.array([0, 5]), q, k, k, np.zeros((5, 2, 3)), hq=2, hkv=1, m_cmp=2,
                   m_win=2, topk=2, gate_mode=0)
    assert st["sel"][4, 0].tolist() == [0, 1]
    # k larger than the number of blocks: all blocks, padded with -1
    st = O.forward(coords, np.array([0, 5]), q, k, k, np.zeros((5, 2, 3)), hq=2, hkv=1, m_cmp=2,
                   m_win=2, topk=7, gate_mode=0)
    assert st["sel"][4, 0].tolist() == [0, 1, 2, 3, 4, -1, -1]


# ----------------------------------------------------------------------------
# P6 / P7 / P9: invariants
# ----------------------------------------------------------------------------


def _small_workload(seed=0, **kw):
    w = W.small_shell(seed=seed, R=24, n_prims=2, lo=3.0, hi=7.0, hq=4, hkv=2, d=16, m_cmp=4,
                      m_win=4, topk=4, dtype="bf16", gate_mode=1, **kw)
    t = W.make_tensors(w)
    return w, t


def _run(w, t, **kw):
    return O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), t.gates,
                     hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk,
                     gate_mode=w.gate_mode, **kw)


def test_permutation_equivariance():
    w, t = _small_workload(n_seqs=2)
    st = _run(w, t)
    w2, t2, src = W.permute_workload(w, t, seed=5)
    st2 = _run(w2, t2)
    assert (st2["blk"]["id"] == st["blk"]["id"][src]).all()
    assert (st2["win"]["id"] == st["win"]["id"][src]).all()
    assert (st2["sel"] == st["sel"][src]).all()
    np.testing.assert_allclose(st2["out"], st["out"][src], rtol=1e-11, atol=1e-12)
    do = t.as_f32("do").astype(np.float64)
    g1 = O.backward(st, do)
    g2 = O.backward(st2, do[src])
    for key in ("dq", "dk", "dv", "dgates"):
        np.testing.assert_allclose(g2[key], g1[key][src], rtol=1e-10, atol=1e-11)


def test_gates_isolate_branches():
    w, t = _small_workload(seed=1)
    n = w.n
    for c in range(3):
        gates = np.zeros((n, w.hq, 3), np.float32)
        gates[:, :, c] = 1.0
        st = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), gates,
                       hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=0)
        np.testing.assert_array_equal(st["out"], st["o"][c])
    gates = np.zeros((n, w.hq, 3), np.float32)
    st = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), gates,
                   hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=0)
    assert not st["out"].any()
    g = O.backward(st, t.as_f32("do"))
    assert not g["dq"].any() and not g["dk"].any() and not g["dv"].any()
    assert g["dgates"].any()


def test_varlen_batch_equals_separate_calls():
    w, t = _small_workload(seed=2, n_seqs=3)
    st = _run(w, t)
    do = t.as_f32("do").astype(np.float64)
    gb = O.backward(st, do)
    for s in range(w.s):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        st_s = O.forward(w.coords[a:b], np.array([0, b - a]), t.as_f32("q")[a:b], t.as_f32("k")[a:b],
                         t.as_f32("v")[a:b], t.gates[a:b], hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp,
                         m_win=w.m_win, topk=w.topk, gate_mode=w.gate_mode)
        np.testing.assert_allclose(st_s["out"], st["out"][a:b], rtol=1e-12, atol=1e-13)
        off = int(st["blk"]["cu"][s])
        want = np.where(st["sel"][a:b] >= 0, st["sel"][a:b] - off, -1)
        assert (st_s["sel"] == want).all()
        gs = O.backward(st_s, do[a:b])
        for key in ("dq", "dk", "dv", "dgates"):
            np.testing.assert_allclose(gs[key], gb[key][a:b], rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# P8 / P10 / P11: backward
# ----------------------------------------------------------------------------


def _torch_reexpression(coords, cu, q, k, v, gates, st, gate_mode, scale):
    """Independent dense-mask expression of the forward in torch (fp64), with the
    oracle's bins and selection taken as constants; differentiated by autograd."""
    n, hq, d = q.shape
    hkv = k.shape[1]
    G = hq // hkv
    blk_id = torch.from_numpy(st["blk"]["id"])
    win_id = torch.from_numpy(st["win"]["id"])
    nb = int(st["blk"]["count"])
    seq = torch.from_numpy(np.repeat(np.arange(len(cu) - 1), np.diff(cu)))
    blk_seq = torch.from_numpy(np.repeat(np.arange(len(cu) - 1), np.diff(st["blk"]["cu"])))
    qt, kt, vt, gt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, gates))
    onehot = torch.nn.functional.one_hot(blk_id, nb).to(torch.float64)  # [N, B]
    kc = torch.einsum("nb,ngd->bgd", onehot, kt) / onehot.sum(0)[:, None, None]
    vc = torch.einsum("nb,ngd->bgd", onehot, vt) / onehot.sum(0)[:, None, None]
    gw = gt if gate_mode == 0 else torch.sigmoid(gt)
    out = torch.zeros(n, hq, d, dtype=torch.float64)
    sel = torch.from_numpy(st["sel"])
    for h in range(hq):
        g = h // G
        # compressed: mask blocks of other sequences
        s_c = scale * qt[:, h] @ kc[:, g].T
        s_c = s_c.masked_fill(seq[:, None] != blk_seq[None, :], -math.inf)
        o_c = torch.softmax(s_c, -1) @ vc[:, g]
        # selected: key j allowed iff its block is in sel[t, g]
        allowed_blk = torch.zeros(n, nb, dtype=torch.bool)
        for slot in range(sel.shape[2]):
            b = sel[:, g, slot]
            ok = b >= 0
            allowed_blk[torch.nonzero(ok)[:, 0], b[ok]] = True
        mask_s = allowed_blk[:, blk_id]
        s_k = scale * qt[:, h] @ kt[:, g].T
        o_s = torch.softmax(s_k.masked_fill(~mask_s, -math.inf), -1) @ vt[:, g]
        mask_w = (win_id[:, None] == win_id[None, :])
        o_w = torch.softmax(s_k.masked_fill(~mask_w, -math.inf), -1) @ vt[:, g]
        out[:, h] = gw[:, h, 0:1] * o_c + gw[:, h, 1:2] * o_s + gw[:, h, 2:3] * o_w
    return out, (qt, kt, vt, gt)


def test_backward_matches_autograd_of_dense_reexpression():
    coords, cu, q, k, v, gates = _rand_case(7, n_per_seq=(48, 30), R=8, hq=4, hkv=2, d=8, unique=False)
    for gate_mode in (0, 1):
        st = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=2, m_win=4, topk=3,
                       gate_mode=gate_mode, pool_rounding="none")
        out, (qt, kt, vt, gt) = _torch_reexpression(coords, cu, q, k, v, gates, st, gate_mode,
                                                   st["scale"])
        np.testing.assert_allclose(out.detach().numpy(), st["out"], rtol=1e-12, atol=1e-12)
        do = np.random.default_rng(3).standard_normal(q.shape)
        (out * torch.from_numpy(do)).sum().backward()
        g = O.backward(st, do)
        np.testing.assert_allclose(g["dq"], qt.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dk"], kt.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dv"], vt.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dgates"], gt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_central_differences():
    coords, cu, q, k, v, gates = _rand_case(8, n_per_seq=(40,), R=8, hq=4, hkv=2, d=8, unique=False)
    kw = dict(hq=4, hkv=2, m_cmp=2, m_win=4, topk=3, gate_mode=1, pool_rounding="none")
    st = O.forward(coords, cu, q, k, v, gates, **kw)
    do = np.random.default_rng(9).standard_normal(q.shape)
    g = O.backward(st, do)
    rng = np.random.default_rng(10)
    h = 1e-6
    arrays = {"q": q, "k": k, "v": v, "gates": gates}
    grads = {"q": g["dq"], "k": g["dk"], "v": g["dv"], "gates": g["dgates"]}
    for name, arr in arrays.items():
        for _ in range(6):
            idx = tuple(rng.integers(0, s) for s in arr.shape)
            vals = []
            for sgn in (+1, -1):
                a2 = {kk: vv.copy() for kk, vv in arrays.items()}
                a2[name][idx] += sgn * h
                st2 = O.forward(coords, cu, a2["q"], a2["k"], a2["v"], a2["gates"], **kw)
                assert (st2["sel"] == st["sel"]).all()  # selection is locally constant
                vals.append(np.sum(do * st2["out"]))
            fd = (vals[0] - vals[1]) / (2 * h)
            assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd,
                                                                             grads[name][idx])


def test_compression_gradient_conservation():
    w, t = _small_workload(seed=3)
    st = _run(w, t)
    g = O.backward(st, t.as_f32("do"))
    parts = g["parts"]
    np.testing.assert_allclose(parts["dk"]["cmp"].sum(0), parts["dkc"].sum(0), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(parts["dv"]["cmp"].sum(0), parts["dvc"].sum(0), rtol=1e-10, atol=1e-10)
    # softmax rows sum to one: sum_i dV_i = sum over rows and branches of w_c * dO
    gw = O.gate_weights(t.gates, w.gate_mode)
    do = t.as_f32("do").astype(np.float64)
    G = w.hq // w.hkv
    for gi in range(w.hkv):
        hs = slice(gi * G, (gi + 1) * G)
        want = np.einsum("nh,nhd->d", gw[:, hs, :].sum(-1), do[:, hs, :])
        np.testing.assert_allclose(g["dv"][:, gi, :].sum(0), want, rtol=1e-10, atol=1e-9)
        # sum_j dS_j = 0 in every softmax row: keys' gradients sum to zero
        np.testing.assert_allclose(g["dk"][:, gi, :].sum(0), 0.0, atol=1e-9)


def test_dgates_central_differences():
    w, t = _small_workload(seed=4)
    do = t.as_f32("do").astype(np.float64)
    st = _run(w, t)
    g = O.backward(st, do)
    rng = np.random.default_rng(0)
    for _ in range(5):
        idx = (int(rng.integers(0, w.n)), int(rng.integers(0, w.hq)), int(rng.integers(0, 3)))
        h = 1e-5
        vals = []
        for sgn in (1, -1):
            gates = t.gates.astype(np.float64).copy()
            gates[idx] += sgn * h
            st2 = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"),
                            gates, hq=w.hq, hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk,
                            gate_mode=w.gate_mode, tokens=[idx[0]])
            vals.append(np.sum(do[idx[0]] * st2["out"][idx[0]]))
        fd = (vals[0] - vals[1]) / (2 * h)
        assert abs(fd - g["dgates"][idx]) < 1e-7 * max(1, abs(fd))


def test_subset_forward_matches_full():
    w, t = _small_workload(seed=5, n_seqs=2)
    st = _run(w, t)
    toks = np.array([0, 7, w.n - 1, int(w.cu_seqlens[1])])
    st2 = _run(w, t, tokens=toks)
    np.testing.assert_array_equal(st2["out"][toks], st["out"][toks])
    np.testing.assert_array_equal(st2["sel"][toks], st["sel"][toks])


def test_dq_rows_matches_full_backward():
    w, t = _small_workload(seed=6, n_seqs=2)
    st = _run(w, t)
    do = t.as_f32("do").astype(np.float64)
    g = O.backward(st, do)
    toks = np.array([0, 3, w.n - 1, int(w.cu_seqlens[1])])
    st2 = _run(w, t, tokens=toks)
    np.testing.assert_allclose(O.dq_rows(st2, do, toks), g["dq"][toks], rtol=1e-10, atol=1e-12)


def test_dgates_rows_and_window_grads_match_full_backward():
    """The row- and window-restricted gradients used by the full-size GPU tests
    equal the full backward (itself pinned by autograd and central differences)."""
    w, t = _small_workload(seed=7, n_seqs=2)
    st = _run(w, t)
    do = t.as_f32("do").astype(np.float64)
    g = O.backward(st, do)
    wins = np.array([0, 3, st["win"]["count"] - 1])
    members = np.concatenate([st["win"]["perm"][st["win"]["ptr"][x]:st["win"]["ptr"][x + 1]] for x in wins])
    toks = np.unique(np.concatenate([members, [0, w.n - 1]]))
    st2 = _run(w, t, tokens=toks)
    np.testing.assert_allclose(O.dgates_rows(st2, do, toks), g["dgates"][toks], rtol=1e-12, atol=1e-14)
    tk, dk, dv = O.window_kv_grads(st2, do, wins)
    np.testing.assert_array_equal(np.sort(tk), np.sort(members))
    np.testing.assert_allclose(dk, g["parts"]["dk"]["win"][tk], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, g["parts"]["dv"]["win"][tk], rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# geometric block routing
# ----------------------------------------------------------------------------

def _geo_brute(coords, cu, m, k):
    """Python loops over every (token, block, member) triple."""
    out = []
    cells = {}
    for s in range(len(cu) - 1):
        keys = sorted({tuple(int(c) // m for c in coords[i]) for i in range(cu[s], cu[s + 1])})
        cells[s] = keys
    base = 0
    for s in range(len(cu) - 1):
        keys = cells[s]
        for t in range(cu[s], cu[s + 1]):
            dist = []
            for j, key in enumerate(keys):
                dmin = min(sum((int(coords[i][a]) - int(coords[t][a])) ** 2 for a in range(3))
                           for i in range(cu[s], cu[s + 1]) if tuple(int(c) // m for c in coords[i]) == key)
                dist.append((dmin, j))
            picks = sorted(j for _, j in sorted(dist)[:k])
            out.append([base + j for j in picks] + [-1] * (k - len(picks)))
        base += len(keys)
    return np.array(out)


def test_geo_topk_matches_brute_force_with_ties_and_short_sequences():
    rng = np.random.default_rng(4)
    pts = np.unique(rng.integers(0, 12, size=(120, 3)), axis=0)[:90]
    coords = np.concatenate([pts, pts[:7] + 1])  # a short second sequence
    cu = np.array([0, 90, 97])
    for k in (1, 3, 40):
        np.testing.assert_array_equal(O.geo_topk(coords, cu, 4, k), _geo_brute(coords, cu, 4, k))


def test_geo_topk_hand_example():
    # blocks of edge 2 along x: {0,1} | {2,3} | {4,5} | {8,9}; query at x = 3
    coords = np.array([[0, 0, 0], [3, 0, 0], [5, 0, 0], [9, 0, 0], [1, 1, 0]])
    cu = np.array([0, 5])
    # distances^2 from token 1 (3,0,0): block0 min(9, 5)=5, block1 0, block2 4, block4 36
    np.testing.assert_array_equal(O.geo_topk(coords, cu, 2, 2, tokens=[1]), [[1, 2]])
    np.testing.assert_array_equal(O.geo_topk(coords, cu, 2, 3, tokens=[1]), [[0, 1, 2]])
    # a tie (token 4 at (1,1,0): block0 0, block1 (3,0,0): 4+1=5, block2 16+1=17 ... ) and k=1
    np.testing.assert_array_equal(O.geo_topk(coords, cu, 2, 1, tokens=[4]), [[0]])


def test_geo_topk_own_block_always_selected_and_permutation_invariant():
    w, t = _small_workload(seed=8, n_seqs=2)
    sel = O.geo_topk(w.coords, w.cu_seqlens, w.m_cmp, w.topk)
    blk = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)
    assert all(blk["id"][i] in sel[i] for i in range(w.n))
    w2, _, src = W.permute_workload(w, t, seed=3)
    sel2 = O.geo_topk(w2.coords, w2.cu_seqlens, w2.m_cmp, w2.topk)
    np.testing.assert_array_equal(sel2, sel[src])


def test_given_selection_of_every_block_is_full_attention():
    """A given selection listing every block of the token's sequence (in descending
    order, padding first) makes the selected branch full attention."""
    coords, cu, q, k, v, gates = _rand_case(13)
    b = O.bin_tokens(coords, cu, 4)
    nb = np.diff(b["cu"])
    k_sel = int(nb.max()) + 2
    sel = np.full((len(coords), 2, k_sel), -1, np.int64)
    for t in range(len(coords)):
        s = int(np.searchsorted(cu, t, side="right") - 1)
        ids = np.arange(b["cu"][s], b["cu"][s + 1])[::-1]
        sel[t, :, k_sel - len(ids):] = ids
    st = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, m_win=4, topk=k_sel, gate_mode=1,
                   sel_given=sel)
    np.testing.assert_allclose(st["o"][1], _sdpa_full(q, k, v, cu, 4, 2), rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(st["sel"], sel)


def test_geometric_selection_backward_matches_autograd():
    """The geometric routing as the selection: the forward and its backward against
    autograd of the dense re-expression built from that selection."""
    coords, cu, q, k, v, gates = _rand_case(17, n_per_seq=(48, 30), R=8, hq=4, hkv=2, d=8, unique=False)
    geo = O.geo_topk(coords, cu, 2, 3)
    sel = np.repeat(geo[:, None, :], 2, axis=1)
    st = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=2, m_win=4, topk=3, gate_mode=1,
                   pool_rounding="none", sel_given=sel)
    ref = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=2, m_win=4, topk=3, gate_mode=1,
                    pool_rounding="none")
    assert (st["sel"] != ref["sel"]).any()  # the two routings differ on this case
    np.testing.assert_array_equal(st["o"][0], ref["o"][0])  # the compressed branch does not depend on it
    out, (qt, kt, vt, gt) = _torch_reexpression(coords, cu, q, k, v, gates, st, 1, st["scale"])
    np.testing.assert_allclose(out.detach().numpy(), st["out"], rtol=1e-12, atol=1e-12)
    do = np.random.default_rng(5).standard_normal(q.shape)
    (out * torch.from_numpy(do)).sum().backward()
    g = O.backward(st, do)
    for key, tt in (("dq", qt), ("dk", kt), ("dv", vt), ("dgates", gt)):
        np.testing.assert_allclose(g[key], tt.grad.numpy(), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# cross-attention SSA (queries from another token set)
# ----------------------------------------------------------------------------


def _cross_case(seed, nq=(40, 0, 23), nkv=(90, 12, 57), R=16, hq=4, hkv=2, d=16):
    rng = np.random.default_rng(seed)
    coords, _, _, k, v, _ = _rand_case(seed, n_per_seq=nkv, R=R, hq=hq, hkv=hkv, d=d)
    q_cu = np.concatenate([[0], np.cumsum(nq)]).astype(np.int64)
    kv_cu = np.concatenate([[0], np.cumsum(nkv)]).astype(np.int64)
    q = rng.standard_normal((int(q_cu[-1]), hq, d))
    gates = rng.standard_normal((int(q_cu[-1]), hq, 2))
    return q_cu, coords, kv_cu, q, k, v, gates


def _sdpa_cross(q, k, v, q_cu, kv_cu, hq, hkv):
    out = np.zeros_like(q)
    G = hq // hkv
    for s in range(len(q_cu) - 1):
        a, b = int(q_cu[s]), int(q_cu[s + 1])
        c, e = int(kv_cu[s]), int(kv_cu[s + 1])
        if a == b:
            continue
        qt = torch.from_numpy(q[a:b]).transpose(0, 1)
        kt = torch.from_numpy(k[c:e]).transpose(0, 1).repeat_interleave(G, 0)
        vt = torch.from_numpy(v[c:e]).transpose(0, 1).repeat_interleave(G, 0)
        out[a:b] = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).transpose(0, 1).numpy()
    return out


def test_cross_selection_covering_everything_is_full_cross_attention():
    q_cu, coords, kv_cu, q, k, v, gates = _cross_case(31)
    st = O.cross_forward(q_cu, coords, kv_cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, topk=10_000, gate_mode=1)
    np.testing.assert_allclose(st["o"][1], _sdpa_cross(q, k, v, q_cu, kv_cu, 4, 2), rtol=1e-12, atol=1e-12)


def test_cross_unit_blocks_make_compression_full_cross_attention():
    q_cu, coords, kv_cu, q, k, v, gates = _cross_case(32)
    st = O.cross_forward(q_cu, coords, kv_cu, q, k, v, gates, hq=4, hkv=2, m_cmp=1, topk=3, gate_mode=0,
                         pool_rounding="none")
    np.testing.assert_allclose(st["o"][0], _sdpa_cross(q, k, v, q_cu, kv_cu, 4, 2), rtol=1e-12, atol=1e-12)


def test_cross_with_the_voxel_tokens_as_queries_matches_self_attention_branches():
    """Queries = the voxel tokens themselves: the two cross branches, the selection
    and (window gate 0) every gradient equal those of the self-attention oracle."""
    coords, cu, q, k, v, gates = _rand_case(33, n_per_seq=(60, 0, 41), R=8, hq=4, hkv=2, d=8, unique=False)
    g3 = np.abs(gates)
    g3[..., 2] = 0.0
    st = O.forward(coords, cu, q, k, v, g3, hq=4, hkv=2, m_cmp=2, m_win=4, topk=3, gate_mode=0,
                   pool_rounding="none")
    cr = O.cross_forward(cu, coords, cu, q, k, v, g3[..., :2], hq=4, hkv=2, m_cmp=2, topk=3, gate_mode=0,
                         pool_rounding="none")
    np.testing.assert_array_equal(cr["sel"], st["sel"])
    np.testing.assert_allclose(cr["o"], st["o"][:2], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(cr["out"], st["out"], rtol=1e-12, atol=1e-12)
    do = np.random.default_rng(4).standard_normal(q.shape)
    gs, gc = O.backward(st, do), O.cross_backward(cr, do)
    for key in ("dq", "dk", "dv"):
        np.testing.assert_allclose(gc[key], gs[key], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(gc["dgates"], gs["dgates"][..., :2], rtol=1e-10, atol=1e-12)


def test_cross_backward_matches_autograd():
    """Independent dense-mask expression in torch (fp64) of the two cross branches,
    with the oracle's bins and selection as constants, differentiated by autograd."""
    q_cu, coords, kv_cu, q, k, v, gates = _cross_case(34, nq=(21, 9), nkv=(40, 25), R=8, hq=4, hkv=2, d=8)
    for gate_mode in (0, 1):
        st = O.cross_forward(q_cu, coords, kv_cu, q, k, v, gates, hq=4, hkv=2, m_cmp=2, topk=3,
                             gate_mode=gate_mode, pool_rounding="none")
        blk = st["blk"]
        nb = int(blk["count"])
        qt, kt, vt, gt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, gates))
        onehot = torch.nn.functional.one_hot(torch.from_numpy(blk["id"]), nb).to(torch.float64)
        kc = torch.einsum("nb,ngd->bgd", onehot, kt) / onehot.sum(0)[:, None, None]
        vc = torch.einsum("nb,ngd->bgd", onehot, vt) / onehot.sum(0)[:, None, None]
        qseq = torch.from_numpy(np.repeat(np.arange(len(q_cu) - 1), np.diff(q_cu)))
        bseq = torch.from_numpy(np.repeat(np.arange(len(kv_cu) - 1), np.diff(blk["cu"])))
        sel = torch.from_numpy(st["sel"])
        gw = gt if gate_mode == 0 else torch.sigmoid(gt)
        scale = st["scale"]
        out = torch.zeros(q.shape, dtype=torch.float64)
        for h in range(4):
            g = h // 2
            s_c = (scale * qt[:, h] @ kc[:, g].T).masked_fill(qseq[:, None] != bseq[None, :], -math.inf)
            o_c = torch.softmax(s_c, -1) @ vc[:, g]
            allowed = torch.zeros(q.shape[0], nb, dtype=torch.bool)
            for slot in range(sel.shape[2]):
                b = sel[:, g, slot]
                ok = b >= 0
                allowed[torch.nonzero(ok)[:, 0], b[ok]] = True
            mask = allowed[:, torch.from_numpy(blk["id"])]
            o_s = torch.softmax((scale * qt[:, h] @ kt[:, g].T).masked_fill(~mask, -math.inf), -1) @ vt[:, g]
            out[:, h] = gw[:, h, 0:1] * o_c + gw[:, h, 1:2] * o_s
        np.testing.assert_allclose(out.detach().numpy(), st["out"], rtol=1e-12, atol=1e-12)
        do = np.random.default_rng(6).standard_normal(q.shape)
        (out * torch.from_numpy(do)).sum().backward()
        gr = O.cross_backward(st, do)
        for key, tt in (("dq", qt), ("dk", kt), ("dv", vt), ("dgates", gt)):
            np.testing.assert_allclose(gr[key], tt.grad.numpy(), rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------
# learned compression: sparse 3D convolution before the mean pool
# ----------------------------------------------------------------------------


def _conv_weights(seed, hkv, d, scale=0.2):
    rng = np.random.default_rng(seed)
    return {"wk": scale * rng.standard_normal((hkv, 27, d, d)), "bk": rng.standard_normal((hkv, d)),
            "wv": scale * rng.standard_normal((hkv, 27, d, d)), "bv": rng.standard_normal((hkv, d))}


def _dense_conv(coords, cu, x, w, b, R):
    """torch conv3d (cross-correlation, padding 1, one group per KV head) on a dense
    grid per sequence, read back at the tokens (duplicate voxels add up)."""
    hkv, _, d, _ = w.shape
    wt = torch.as_tensor(w, dtype=torch.float64)
    wt = wt.reshape(hkv, 3, 3, 3, d, d).permute(0, 5, 4, 1, 2, 3).reshape(hkv * d, d, 3, 3, 3)
    bt = torch.as_tensor(b, dtype=torch.float64).reshape(-1)
    outs = []
    xt = torch.as_tensor(x, dtype=torch.float64)
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        c = torch.from_numpy(np.asarray(coords[a:e], np.int64))
        flat = (c[:, 0] * R + c[:, 1]) * R + c[:, 2]
        grid = torch.zeros(hkv * d, R * R * R, dtype=torch.float64)
        grid = grid.index_add(1, flat, xt[a:e].reshape(e - a, hkv * d).T)
        y = torch.nn.functional.conv3d(grid.reshape(1, hkv * d, R, R, R), wt, bt, padding=1, groups=hkv)
        outs.append(y.reshape(hkv * d, -1)[:, flat].T.reshape(e - a, hkv, d))
    return torch.cat(outs)


def test_sparse_conv_matches_dense_conv3d_with_duplicates_and_sequences():
    coords, cu, _, k, _, _ = _rand_case(41, n_per_seq=(70, 0, 45), R=6, hq=4, hkv=2, d=5, unique=False)
    cw = _conv_weights(1, 2, 5)
    got = O.sparse_conv3(coords, cu, k, cw["wk"], cw["bk"])
    want = _dense_conv(coords, cu, k, cw["wk"], cw["bk"], 6).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_identity_convolution_is_the_mean_pool():
    coords, cu, _, k, _, _ = _rand_case(42, n_per_seq=(80, 33), R=8, hq=4, hkv=2, d=6)
    w = np.zeros((2, 27, 6, 6))
    w[:, 13] = np.eye(6)  # the centre offset (0, 0, 0)
    blk = O.bin_tokens(coords, cu, 4)
    got = O.conv_pool(coords, cu, k, w, np.zeros((2, 6)), blk, "none")
    np.testing.assert_allclose(got, O.mean_pool(k, blk, "none"), rtol=1e-12, atol=1e-12)


def test_conv_pool_backward_matches_autograd():
    coords, cu, _, k, _, _ = _rand_case(43, n_per_seq=(50, 31), R=6, hq=4, hkv=2, d=4, unique=False)
    cw = _conv_weights(2, 2, 4)
    blk = O.bin_tokens(coords, cu, 2)
    xt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    wt = torch.tensor(cw["wk"], requires_grad=True)
    bt = torch.tensor(cw["bk"], requires_grad=True)
    y = _dense_conv(coords, cu, xt, wt, bt, 6)
    onehot = torch.nn.functional.one_hot(torch.from_numpy(blk["id"]), int(blk["count"])).to(torch.float64)
    xc = torch.einsum("nb,ngd->bgd", onehot, y) / onehot.sum(0)[:, None, None]
    np.testing.assert_allclose(xc.detach().numpy(), O.conv_pool(coords, cu, k, cw["wk"], cw["bk"], blk, "none"),
                               rtol=1e-12, atol=1e-12)
    dxc = np.random.default_rng(9).standard_normal(xc.shape)
    (xc * torch.from_numpy(dxc)).sum().backward()
    dx, dw, db = O.conv_pool_backward(coords, cu, k, cw["wk"], blk, dxc)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_learned_compression_in_the_full_backward_by_central_differences():
    coords, cu, q, k, v, gates = _rand_case(44, n_per_seq=(36,), R=6, hq=4, hkv=2, d=4)
    cw = _conv_weights(3, 2, 4)
    kw = dict(hq=4, hkv=2, m_cmp=2, m_win=3, topk=2, gate_mode=1, pool_rounding="none")
    st = O.forward(coords, cu, q, k, v, gates, conv=cw, **kw)
    do = np.random.default_rng(10).standard_normal(q.shape)
    g = O.backward(st, do)
    rng = np.random.default_rng(11)
    for key, gkey in (("wk", "dwk"), ("bv", "dbv"), ("wv", "dwv")):
        for _ in range(3):
            idx = tuple(rng.integers(0, n) for n in cw[key].shape)
            h = 1e-6
            vals = []
            for sgn in (1, -1):
                c2 = {kk: vv.copy() for kk, vv in cw.items()}
                c2[key][idx] += sgn * h
                s2 = O.forward(coords, cu, q, k, v, gates, conv=c2, sel_given=st["sel"], **kw)
                vals.append(np.sum(do * s2["out"]))
            num = (vals[0] - vals[1]) / (2 * h)
            assert abs(num - g[gkey][idx]) <= 1e-6 * max(1.0, abs(num)), (key, idx, num, g[gkey][idx])
    # dK through the convolution as well
    for _ in range(3):
        idx = tuple(rng.integers(0, n) for n in k.shape)
        vals = []
        for sgn in (1, -1):
            k2 = k.copy()
            k2[idx] += sgn * 1e-6
            s2 = O.forward(coords, cu, q, k2, v, gates, conv=cw, sel_given=st["sel"], **kw)
            vals.append(np.sum(do * s2["out"]))
        num = (vals[0] - vals[1]) / 2e-6
        assert abs(num - g["dk"][idx]) <= 1e-6 * max(1.0, abs(num)), (idx, num, g["dk"][idx])


def test_cross_subset_of_query_rows_matches_full():
    q_cu, coords, kv_cu, q, k, v, gates = _cross_case(35)
    full = O.cross_forward(q_cu, coords, kv_cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, topk=3, gate_mode=1)
    rows = np.array([0, 7, 39, 40, 62])
    sub = O.cross_forward(q_cu, coords, kv_cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, topk=3, gate_mode=1,
                          tokens=rows)
    np.testing.assert_array_equal(sub["sel"][rows], full["sel"][rows])
    np.testing.assert_array_equal(sub["o"][:, rows], full["o"][:, rows])
    np.testing.assert_array_equal(sub["out"][rows], full["out"][rows])


# ----------------------------------------------------------------------------
# the compressed branch over token ranges (used by the full-size GPU checks)
# ----------------------------------------------------------------------------


def _ranges_run(w, t, gates, gate_mode, bounds, sel_other=None):
    st = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), gates, hq=w.hq,
                   hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=gate_mode)
    parts = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        so = None if sel_other is None else sel_other[a:b]
        parts.append(O.cmp_branch_range(t.as_f32("q"), st["kc"], st["vc"], st["blk"]["cu"], w.cu_seqlens, gates,
                                        hq=w.hq, hkv=w.hkv, topk=w.topk, gate_mode=gate_mode, t0=a, t1=b,
                                        dout=t.as_f32("do"), chunk=37, sel_other=so))
    return st, parts


def test_cmp_branch_ranges_match_the_full_forward_and_backward():
    """Split at points inside sequences, the ranges reproduce the compressed branch
    of `forward` / `backward`: lse, output, selection and dQ row by row, and dKc /
    dVc (hence the tokens' dK / dV) as sums over the ranges."""
    w, t = _small_workload(seed=4, n_seqs=3)
    bounds = [0, 17, w.n // 2 + 3, w.n - 5, w.n]
    st, parts = _ranges_run(w, t, t.gates, 1, bounds)
    g = O.backward(st, t.as_f32("do"))
    cat = lambda key: np.concatenate([p[key] for p in parts])  # noqa: E731
    np.testing.assert_allclose(cat("lse"), st["lse"][0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(cat("o"), st["o"][0], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(cat("sel"), st["sel"])
    np.testing.assert_allclose(cat("dq"), g["parts"]["dq"]["cmp"], rtol=0, atol=1e-12)
    dkc = sum(p["dkc"] for p in parts)
    dvc = sum(p["dvc"] for p in parts)
    np.testing.assert_allclose(dkc, g["parts"]["dkc"], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dvc, g["parts"]["dvc"], rtol=0, atol=1e-11)
    dk, dv = O.cmp_token_grads(dkc, dvc, st["blk"])
    np.testing.assert_allclose(dk, g["parts"]["dk"]["cmp"], rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, g["parts"]["dv"]["cmp"], rtol=0, atol=1e-11)


def test_cmp_branch_range_with_unit_blocks_is_full_attention_and_its_gradient():
    """With one token per block (m_cmp = 1, unique coordinates) and the exact mean,
    the compressed branch is textbook full attention: its output, and its dQ / dK /
    dV against torch autograd of scaled_dot_product_attention (fp64)."""
    coords, cu, q, k, v, gates = _rand_case(21)
    hq, hkv, G = 4, 2, 2
    k = k.astype(np.float32).astype(np.float64)  # fp32-representable: the f32 mean of one is itself
    v = v.astype(np.float32).astype(np.float64)
    blk = O.bin_tokens(coords, cu, 1)
    kc, vc = O.mean_pool(k, blk, "f32"), O.mean_pool(v, blk, "f32")
    rng = np.random.default_rng(5)
    do = rng.standard_normal(q.shape)
    gates = np.ones_like(gates)
    r = O.cmp_branch_range(q, kc, vc, blk["cu"], cu, gates, hq=hq, hkv=hkv, topk=3, gate_mode=0, t0=0,
                           t1=len(coords), dout=do)
    np.testing.assert_allclose(r["o"], _sdpa_full(q, k, v, cu, hq, hkv), rtol=0, atol=1e-12)
    dk, dv = O.cmp_token_grads(r["dkc"], r["dvc"], blk)
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        if a == b:
            continue
        qt = torch.from_numpy(q[a:b]).transpose(0, 1).requires_grad_()
        kt = torch.from_numpy(k[a:b]).transpose(0, 1).requires_grad_()
        vt = torch.from_numpy(v[a:b]).transpose(0, 1).requires_grad_()
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt.repeat_interleave(G, 0),
                                                             vt.repeat_interleave(G, 0))
        o.backward(torch.from_numpy(do[a:b]).transpose(0, 1))
        np.testing.assert_allclose(r["dq"][a:b], qt.grad.transpose(0, 1).numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dk[a:b], kt.grad.transpose(0, 1).numpy(), rtol=0, atol=1e-11)
        np.testing.assert_allclose(dv[a:b], vt.grad.transpose(0, 1).numpy(), rtol=0, atol=1e-11)


def test_cmp_branch_gap_certifies_only_top_k_selections():
    """other_gap of the oracle's own selection is >= 0; moving one pick to the best
    block left out makes it exactly minus the score difference of the two blocks."""
    w, t = _small_workload(seed=6, n_seqs=2)
    st0, _ = _ranges_run(w, t, t.gates, 1, [0, w.n])
    sel = st0["sel"].copy()
    st, parts = _ranges_run(w, t, t.gates, 1, [0, w.n], sel_other=sel)
    assert (parts[0]["other_gap"] >= 0).all()
    moved = sel.copy()
    rows = []
    for tt in range(0, w.n, 7):
        s = int(np.searchsorted(w.cu_seqlens, tt, side="right") - 1)
        b0, b1 = int(st["blk"]["cu"][s]), int(st["blk"]["cu"][s + 1])
        if b1 - b0 <= w.topk:
            continue
        imp = O.importance(st, tt, 0)
        chosen = [int(x) for x in sel[tt, 0] if x >= 0]
        rest = [b for b in range(b0, b1) if b not in chosen]
        best = max(rest, key=lambda b: (imp[b - b0], -b))
        worst = min(chosen, key=lambda b: (imp[b - b0], -b))
        moved[tt, 0] = np.sort([b for b in chosen if b != worst] + [best])
        rows.append((tt, imp[worst - b0] - imp[best - b0], imp))
    _, parts2 = _ranges_run(w, t, t.gates, 1, [0, w.n], sel_other=moved)
    for tt, diff, imp in rows:
        gap = parts2[0]["other_gap"][tt, 0]
        # the moved-in block is now the lowest chosen and the moved-out one the highest left out
        assert gap <= 0 and abs(gap - (-(abs(diff)))) <= 1e-12, (tt, gap, diff)


def test_attend_with_sel_equals_the_forward_given_that_selection():
    """attend_with_sel (the check of rows whose selection flipped on the GPU) against
    forward(sel_given=...) with a selection that differs from the score top-k, and
    against textbook attention when the selection covers the sequence."""
    w, t = _small_workload(seed=7, n_seqs=2)
    st = _run(w, t)
    rng = np.random.default_rng(3)
    other = st["sel"].copy()
    for tt in range(w.n):
        s = int(np.searchsorted(w.cu_seqlens, tt, side="right") - 1)
        b0, b1 = int(st["blk"]["cu"][s]), int(st["blk"]["cu"][s + 1])
        k_eff = min(w.topk, b1 - b0)
        for g in range(w.hkv):
            other[tt, g, :k_eff] = np.sort(rng.choice(np.arange(b0, b1), size=k_eff, replace=False))
    assert (other != st["sel"]).any()
    st2 = _run(w, t, sel_given=other)
    G = w.hq // w.hkv
    for tt in range(0, w.n, 3):
        for g in range(w.hkv):
            l_, o_ = O.attend_with_sel(st, tt, g, other[tt, g])
            np.testing.assert_allclose(o_, st2["o"][1][tt, g * G:(g + 1) * G], rtol=0, atol=1e-13)
            np.testing.assert_allclose(l_, st2["lse"][1][tt, g * G:(g + 1) * G], rtol=0, atol=1e-13)
    # every block of the sequence: the selected branch is full attention
    coords, cu, q, k, v, gates = _rand_case(17)
    stf = O.forward(coords, cu, q, k, v, gates, hq=4, hkv=2, m_cmp=4, m_win=4, topk=3, gate_mode=1)
    full = _sdpa_full(q, k, v, cu, 4, 2)
    for tt in (0, 45, 89, 90, 146):
        s = int(np.searchsorted(cu, tt, side="right") - 1)
        ids = np.arange(stf["blk"]["cu"][s], stf["blk"]["cu"][s + 1])
        for g in range(2):
            _, o_ = O.attend_with_sel(stf, tt, g, ids)
            np.testing.assert_allclose(o_, full[tt, 2 * g:2 * g + 2], rtol=0, atol=1e-12)
