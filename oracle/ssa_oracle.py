"""Plain, slow, fp64 CPU oracle of spatial sparse attention (SSA).

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
bench's CPU-baseline leg may import this module.  It shares no code with the
CUDA library and must never be used as a fallback for it.

What it follows (all citations are to the pages as titled):

* Direct3D-S2 (hyper.ai/cn/papers/2505.17412), section "方法", the SSA
  paragraph: tokens are grouped into m_cmp^3 blocks by their 3D coordinates
  (not by 1D index); "sparse 3D compression" mean-pools each block's keys and
  values; "spatial block selection" picks the top-k blocks by the
  query/compressed-block attention score and runs a second, full attention over
  every token of the selected blocks; "sparse 3D window" attends only inside
  non-overlapping m_win^3 windows; the three module outputs are summed with
  predicted gate weights.
* LSRM (shuwu5.cn/article/2502.html), "空间块划分与键值压缩": in-block average
  pooling for the compressed keys/values; "阶段一" for GQA with 32 query and 2
  KV heads and a Linear+Sigmoid gate.

Readings where the pages are silent (each is also listed in the design notes):

* block / window ids: floor(coord / m), per sequence, numbered in
  lexicographic (x, y, z) order of the block coordinate, offset by the number
  of blocks of earlier sequences; members ordered by token index.
* compression is the mean by default; the stored Kc/Vc is computed as
  fp32(sum) / fp32(n), then rounded to the storage dtype (bf16
  round-to-nearest-even) -- "pool_rounding".  The learned form (a submanifold
  sparse 3x3x3 convolution before the mean, weights as inputs) is `conv_pool`.
* selection score: softmax probability over the sequence's compressed blocks,
  summed over the query heads of a GQA group; top-k with ties to the lower
  block id; k_eff = min(k, blocks in sequence); sel stored ascending, padded -1.
* all three branches are outputs (cmp, slc, win), combined with per
  (token, head, branch) gates: the gate value itself (mode 0) or its sigmoid
  (mode 1).  softmax scale 1/sqrt(d) everywhere; no causal mask; a query's own
  token is in its window; selection is a constant for the backward; the
  rounding of Kc/Vc passes the gradient straight through (dKc/dK_i = 1/n_b).

Beyond the self-attention path: `geo_topk` (selection by the shortest distance
between voxel centres, LSRM "3D 感知空间块路由机制", voxel-only case), a given
selection in `forward(sel_given=...)`, and `cross_forward` / `cross_backward`
(queries of another token set, LSRM's cross attention between image and voxel
tokens: compressed and selected branches, no window branch).

Everything is computed in float64 from the exact input values.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# step 1: binning (Direct3D-S2, "方法": spatially coherent block partition)
# ----------------------------------------------------------------------------


def bin_tokens(coords: np.ndarray, cu_seqlens: np.ndarray, m: int) -> dict:
    """Partition each sequence's tokens into m^3 cells of the integer grid.

    Returns id [N] (global, compacted), perm [N] (tokens sorted by (id, index)),
    ptr [B+1] (CSR into perm), cu [S+1] (first id of each sequence) and
    key [B, 3] (the cell coordinate of each id).
    """
    coords = np.asarray(coords, dtype=np.int64)
    cu_seqlens = np.asarray(cu_seqlens, dtype=np.int64)
    n = coords.shape[0]
    ids = np.empty(n, dtype=np.int64)
    cu = [0]
    keys = []
    for s in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        if b == a:
            cu.append(cu[-1])
            continue
        cell = np.floor_divide(coords[a:b], m)
        uniq, inv = np.unique(cell, axis=0, return_inverse=True)  # rows sorted lexicographically
        ids[a:b] = cu[-1] + inv.reshape(-1)
        cu.append(cu[-1] + len(uniq))
        keys.append(uniq)
    total = cu[-1]
    perm = np.argsort(ids, kind="stable")
    counts = np.bincount(ids, minlength=total) if n else np.zeros(0, np.int64)
    ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    key = np.concatenate(keys) if keys else np.zeros((0, 3), np.int64)
    return {"id": ids, "perm": perm, "ptr": ptr, "cu": np.array(cu, np.int64), "key": key,
            "count": total}


# ----------------------------------------------------------------------------
# step 2: sparse 3D compression by mean pooling
# ----------------------------------------------------------------------------


def _round_bf16(x32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 (round to nearest, ties to even) -> value as float64."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def mean_pool(x: np.ndarray, blk: dict, pool_rounding: str) -> np.ndarray:
    """Per block and KV head, the mean of its members' vectors.

    x: [N, Hkv, d] float64 (exact input values).  Returns [B, Hkv, d] float64.
    pool_rounding: "bf16" -> bf16(fp32(sum) / fp32(n)); "f32" -> fp32(sum) / fp32(n);
    "none" -> exact mean (used by derivative checks).
    """
    nb = blk["count"]
    sums = np.zeros((nb,) + x.shape[1:], dtype=np.float64)
    np.add.at(sums, blk["id"], x)  # members in ascending token order
    cnt = np.diff(blk["ptr"]).astype(np.float64)
    if pool_rounding == "none":
        return sums / cnt[:, None, None]
    q = sums.astype(np.float32) / cnt.astype(np.float32)[:, None, None]
    if pool_rounding == "f32":
        return q.astype(np.float64)
    if pool_rounding == "bf16":
        return _round_bf16(q)
    raise ValueError(pool_rounding)


# ----------------------------------------------------------------------------
# step 2, learned form: a sparse 3D convolution before the mean pool
# ----------------------------------------------------------------------------

# offsets of the 3^3 kernel; offset index (dx + 1) * 9 + (dy + 1) * 3 + (dz + 1)
CONV_OFFSETS = [(dx, dy, dz) for dx in (-1, 0, 1) for dy in (-1, 0, 1) for dz in (-1, 0, 1)]


def _neighbours(coords: np.ndarray, cu_seqlens: np.ndarray):
    """For every token i and offset index o, the tokens of i's sequence at
    coords_i + offset_o (all of them if coordinates repeat), as a list of lists."""
    coords = np.asarray(coords, np.int64)
    cu = np.asarray(cu_seqlens, np.int64)
    nbr = [[None] * 27 for _ in range(len(coords))]
    for s in range(len(cu) - 1):
        where = {}
        for t in range(cu[s], cu[s + 1]):
            where.setdefault(tuple(coords[t]), []).append(t)
        for t in range(cu[s], cu[s + 1]):
            c = coords[t]
            for o, off in enumerate(CONV_OFFSETS):
                nbr[t][o] = where.get((c[0] + off[0], c[1] + off[1], c[2] + off[2]), [])
    return nbr


def sparse_conv3(coords, cu_seqlens, x, w, b, nbr=None) -> np.ndarray:
    """Submanifold sparse 3D convolution with a 3^3 kernel (Direct3D-S2, "方法": the
    sparse 3D compression may apply a sparse 3D convolution before pooling): at
    every token i, out_i = b + sum_o W_o^T x_j over the tokens j of i's sequence at
    coords_i + offset_o; empty voxels contribute nothing.
    x [N, Hkv, d], w [Hkv, 27, d_in, d_out], b [Hkv, d] -> [N, Hkv, d] (float64)."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    nbr = _neighbours(coords, cu_seqlens) if nbr is None else nbr
    out = np.broadcast_to(np.asarray(b, np.float64), x.shape).copy()
    for i in range(len(x)):
        for o in range(27):
            for j in nbr[i][o]:
                out[i] += np.einsum("gc,gcd->gd", x[j], w[:, o])
    return out


def conv_pool(coords, cu_seqlens, x, w, b, blk: dict, rounding: str) -> np.ndarray:
    """Learned compression: the block mean of the sparse convolution's output,
    computed exactly and then rounded once to the storage type ("bf16", "f32",
    or "none")."""
    y = sparse_conv3(coords, cu_seqlens, x, w, b)
    sums = np.zeros((blk["count"],) + y.shape[1:])
    np.add.at(sums, blk["id"], y)
    mean = sums / np.diff(blk["ptr"]).astype(np.float64)[:, None, None]
    if rounding == "none":
        return mean
    if rounding == "f32":
        return mean.astype(np.float32).astype(np.float64)
    if rounding == "bf16":
        return _round_bf16(mean.astype(np.float32))
    raise ValueError(rounding)


def conv_pool_backward(coords, cu_seqlens, x, w, blk: dict, dxc: np.ndarray):
    """Gradients of the learned compression given dL/dXc [B, Hkv, d] (the rounding of
    Xc passed straight through): each token's output receives dXc_b / n_b; then
    dx_j = sum over (i, o) with j at coords_i + offset_o of W_o dout_i,
    dW_o = sum over the same pairs of x_j dout_i^T, db = sum_i dout_i."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    nbr = _neighbours(coords, cu_seqlens)
    dout = dxc[blk["id"]] / np.diff(blk["ptr"]).astype(np.float64)[blk["id"]][:, None, None]
    dx = np.zeros_like(x)
    dw = np.zeros_like(w)
    for i in range(len(x)):
        for o in range(27):
            for j in nbr[i][o]:
                dx[j] += np.einsum("gcd,gd->gc", w[:, o], dout[i])
                dw[:, o] += np.einsum("gc,gd->gcd", x[j], dout[i])
    return dx, dw, dout.sum(axis=0)


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------


def _logsumexp(s: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(s, axis=axis, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    return (m + np.log(np.sum(np.exp(s - m), axis=axis, keepdims=True))).squeeze(axis)


def _seq_of_tokens(cu_seqlens: np.ndarray, n: int) -> np.ndarray:
    return np.repeat(np.arange(len(cu_seqlens) - 1), np.diff(cu_seqlens))


def gate_weights(gates: np.ndarray, gate_mode: int) -> np.ndarray:
    g = np.asarray(gates, dtype=np.float64)
    if gate_mode == 0:
        return g
    return 1.0 / (1.0 + np.exp(-g))


# ----------------------------------------------------------------------------
# step 3: compressed attention + top-k block selection
# ----------------------------------------------------------------------------


def cmp_attention(q_rows: np.ndarray, kc: np.ndarray, vc: np.ndarray, scale: float):
    """q_rows [n, G, d] against all compressed blocks kc/vc [B_s, d] of one group.

    Returns lse [n, G], o [n, G, d], p [n, G, B_s] (softmax probabilities)."""
    s = scale * (q_rows @ kc.T)  # [n, G, B]
    lse = _logsumexp(s, -1)
    p = np.exp(s - lse[..., None])
    o = p @ vc
    return lse, o, p


def topk_blocks(importance: np.ndarray, k: int) -> np.ndarray:
    """importance [n, B_s] -> local ids of the k_eff largest (ties: lower id),
    ascending, padded with -1 to k."""
    n, b = importance.shape
    keff = min(k, b)
    order = np.argsort(-importance, axis=1, kind="stable")[:, :keff]
    order = np.sort(order, axis=1)
    out = np.full((n, k), -1, dtype=np.int64)
    out[:, :keff] = order
    return out


# ----------------------------------------------------------------------------
# steps 4/5: selected-block attention and window attention
# ----------------------------------------------------------------------------


def _attend(q: np.ndarray, kk: np.ndarray, vv: np.ndarray, scale: float):
    """q [G, d] against keys kk [L, d]; returns lse [G], o [G, d], p [G, L]."""
    s = scale * (q @ kk.T)
    lse = _logsumexp(s, -1)
    p = np.exp(s - lse[:, None])
    return lse, p @ vv, p


def selected_tokens(sel_row: np.ndarray, blk: dict) -> np.ndarray:
    """Token indices of all members of the selected (global) block ids."""
    parts = [blk["perm"][blk["ptr"][b]:blk["ptr"][b + 1]] for b in sel_row if b >= 0]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


# ----------------------------------------------------------------------------
# full forward
# ----------------------------------------------------------------------------


class State(dict):
    pass


def forward(coords, cu_seqlens, q, k, v, gates, *, hq, hkv, m_cmp, m_win, topk,
            gate_mode, scale=None, pool_rounding="bf16", tokens=None, chunk=256, sel_given=None,
            conv=None) -> State:
    """SSA forward.  q [N, Hq, d], k/v [N, Hkv, d] (any float type; converted to
    float64), gates [N, Hq, 3].

    `conv` (a dict of wk, bk, wv, bv) makes the compression learned: Kc / Vc are the
    block means of a sparse 3D convolution of K / V (`conv_pool`), rounded as
    `pool_rounding` says.

    `sel_given` ([N, Hkv, topk] global block ids or -1) replaces the score top-k:
    the selected branch attends the tokens of those blocks instead (a routing by
    geometry, LSRM "3D 感知空间块路由机制", is one source of such a selection).

    `tokens` restricts the per-query outputs (lse, o_*, sel, O) to a subset of
    query tokens (all other rows are NaN / -2); binning and compression are
    always complete.
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, _, d = q.shape
    assert hq % hkv == 0
    G = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    cu_seqlens = np.asarray(cu_seqlens, dtype=np.int64)
    blk = bin_tokens(coords, cu_seqlens, m_cmp)
    win = bin_tokens(coords, cu_seqlens, m_win)
    if conv is None:
        kc = mean_pool(k, blk, pool_rounding)
        vc = mean_pool(v, blk, pool_rounding)
    else:
        kc = conv_pool(coords, cu_seqlens, k, conv["wk"], conv["bk"], blk, pool_rounding)
        vc = conv_pool(coords, cu_seqlens, v, conv["wv"], conv["bv"], blk, pool_rounding)
    seq = _seq_of_tokens(cu_seqlens, n)
    if tokens is None:
        tokens = np.arange(n)
    tokens = np.asarray(tokens, dtype=np.int64)

    def qrows(idx, hs):  # exact float64 copies of the needed query rows only
        return np.asarray(q[idx, hs, :], dtype=np.float64)

    # rows of tokens outside `tokens` are left unset (lse NaN, sel -2, o/out undefined)
    lse = np.full((3, n, hq), np.nan)
    o = np.empty((3, n, hq, d))
    sel = np.full((n, hkv, topk), -2, dtype=np.int64)

    # --- compressed branch + selection, per sequence and group, chunked over tokens
    for s in range(len(cu_seqlens) - 1):
        toks = tokens[seq[tokens] == s] if len(tokens) else tokens
        if len(toks) == 0:
            continue
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            kcg = kc[b0:b1, g, :]
            vcg = vc[b0:b1, g, :]
            for c0 in range(0, len(toks), chunk):
                tt = toks[c0:c0 + chunk]
                l_, o_, p_ = cmp_attention(qrows(tt, hs), kcg, vcg, scale)
                lse[0, tt, hs] = l_
                o[0, tt, hs, :] = o_
                if sel_given is None:
                    imp = p_.sum(axis=1)  # [n, B_s]: probabilities summed over the group's heads
                    loc = topk_blocks(imp, topk)
                    sel[tt, g, :] = np.where(loc >= 0, loc + b0, -1)
    if sel_given is not None:
        sel[tokens] = np.asarray(sel_given, np.int64)[tokens]

    # --- selected-block attention and window attention, per query token and group
    for t in tokens:
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            qt = qrows(t, hs)
            js = selected_tokens(sel[t, g], blk)
            l_, o_, _ = _attend(qt, k[js, g, :], v[js, g, :], scale)
            lse[1, t, hs] = l_
            o[1, t, hs, :] = o_
            w = win["id"][t]
            jw = win["perm"][win["ptr"][w]:win["ptr"][w + 1]]
            l_, o_, _ = _attend(qt, k[jw, g, :], v[jw, g, :], scale)
            lse[2, t, hs] = l_
            o[2, t, hs, :] = o_

    gw = gate_weights(gates[tokens], gate_mode)  # [T, Hq, 3]
    out = np.empty((n, hq, d))
    out[tokens] = np.einsum("nhc,cnhd->nhd", gw, o[:, tokens])
    st = State(blk=blk, win=win, kc=kc, vc=vc, lse=lse, o=o, sel=sel, out=out, scale=scale,
               q=q, k=k, v=v, gates=np.asarray(gates, np.float64), gate_mode=gate_mode,
               hq=hq, hkv=hkv, G=G, topk=topk, cu_seqlens=cu_seqlens, tokens=tokens, conv=conv,
               coords=np.asarray(coords, np.int64))
    return st


# ----------------------------------------------------------------------------
# cross-attention SSA: queries of another token set attend the voxel tokens
# ----------------------------------------------------------------------------


def cross_forward(q_cu, kv_coords, kv_cu, q, k, v, gates, *, hq, hkv, m_cmp, topk, gate_mode, scale=None,
                  pool_rounding="bf16", chunk=256, sel_given=None, tokens=None) -> State:
    """Cross-attention SSA (LSRM, shuwu5.cn/article/2502.html: the NSA attention is
    also used as cross attention between image tokens and voxel tokens).  The
    queries q [Nq, Hq, d] of sequence s are rows q_cu[s] .. q_cu[s+1]-1; the keys
    and values k/v [Nkv, Hkv, d] of sequence s are the voxel tokens kv_cu[s] ..
    kv_cu[s+1]-1 at kv_coords, grouped into m_cmp^3 blocks and mean-pooled as in
    the self-attention path.  Two branches: compressed attention over all blocks
    of the sequence (with the group-summed top-k selection) and full attention
    over the tokens of the selected blocks.  The queries have no voxel, so there
    is no window branch; gates [Nq, Hq, 2] weight (compressed, selected).

    `tokens` restricts the per-query outputs to a subset of query rows (the other
    rows are left NaN / -1 / 0); compression is always complete."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, _, d = q.shape
    G = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    q_cu = np.asarray(q_cu, dtype=np.int64)
    kv_cu = np.asarray(kv_cu, dtype=np.int64)
    blk = bin_tokens(kv_coords, kv_cu, m_cmp)
    kc = mean_pool(k, blk, pool_rounding)
    vc = mean_pool(v, blk, pool_rounding)
    lse = np.full((2, nq, hq), np.nan)
    o = np.zeros((2, nq, hq, d))
    sel = np.full((nq, hkv, topk), -1, dtype=np.int64)
    rows = np.arange(nq) if tokens is None else np.asarray(tokens, np.int64)
    for s in range(len(q_cu) - 1):
        toks = rows[(rows >= q_cu[s]) & (rows < q_cu[s + 1])]
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        if len(toks) == 0 or b1 == b0:
            continue
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            for c0 in range(0, len(toks), chunk):
                tt = toks[c0:c0 + chunk]
                l_, o_, p_ = cmp_attention(np.asarray(q[tt, hs, :], np.float64), kc[b0:b1, g, :], vc[b0:b1, g, :],
                                           scale)
                lse[0, tt, hs] = l_
                o[0, tt, hs, :] = o_
                if sel_given is None:
                    loc = topk_blocks(p_.sum(axis=1), topk)
                    sel[tt, g, :] = np.where(loc >= 0, loc + b0, -1)
    if sel_given is not None:
        sel = np.asarray(sel_given, np.int64).copy()
    for t in rows:
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            js = selected_tokens(sel[t, g], blk)
            if len(js) == 0:
                continue
            l_, o_, _ = _attend(np.asarray(q[t, hs, :], np.float64), k[js, g, :], v[js, g, :], scale)
            lse[1, t, hs] = l_
            o[1, t, hs, :] = o_
    gw = gate_weights(gates, gate_mode)  # [Nq, Hq, 2]
    out = np.zeros((nq, hq, d))
    out[rows] = np.einsum("nhc,cnhd->nhd", gw[rows], o[:, rows])
    return State(blk=blk, kc=kc, vc=vc, lse=lse, o=o, sel=sel, out=out, scale=scale, q=q, k=k, v=v,
                 gates=np.asarray(gates, np.float64), gate_mode=gate_mode, hq=hq, hkv=hkv, G=G, topk=topk,
                 q_cu=q_cu, kv_cu=kv_cu)


def cross_backward(st: State, dout: np.ndarray, chunk: int = 256) -> dict:
    """Gradients of sum(dout * O) of `cross_forward` w.r.t. q, k, v and gates, by
    the chain rule of its two branches (selection held fixed, the Kc/Vc rounding
    passed straight through, dKc/dK_i = 1/n_b)."""
    q, k, v = np.asarray(st["q"], np.float64), st["k"], st["v"]
    nq, hq, d = q.shape
    hkv, G, scale = st["hkv"], st["G"], st["scale"]
    blk = st["blk"]
    dout = np.asarray(dout, dtype=np.float64)
    gw = gate_weights(st["gates"], st["gate_mode"])
    dots = np.einsum("nhd,cnhd->nhc", dout, st["o"])
    dgates = dots if st["gate_mode"] == 0 else dots * gw * (1.0 - gw)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkc = np.zeros((blk["count"], hkv, d))
    dvc = np.zeros((blk["count"], hkv, d))
    q_cu = st["q_cu"]
    for s in range(len(q_cu) - 1):
        toks = np.arange(q_cu[s], q_cu[s + 1])
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        if len(toks) == 0 or b1 == b0:
            continue
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            kcg, vcg = st["kc"][b0:b1, g, :], st["vc"][b0:b1, g, :]
            for c0 in range(0, len(toks), chunk):
                tt = toks[c0:c0 + chunk]
                qr = q[tt, hs, :]
                dor = dout[tt, hs, :] * gw[tt, hs, 0][..., None]
                p = np.exp(scale * (qr @ kcg.T) - st["lse"][0, tt, hs][..., None])
                dp = dor @ vcg.T
                ds = p * (dp - np.sum(p * dp, axis=-1, keepdims=True))
                dq[tt, hs, :] += scale * (ds @ kcg)
                dkc[b0:b1, g, :] += scale * np.einsum("ngb,ngd->bd", ds, qr)
                dvc[b0:b1, g, :] += np.einsum("ngb,ngd->bd", p, dor)
    cnt = np.diff(blk["ptr"]).astype(np.float64)
    dk += dkc[blk["id"]] / cnt[blk["id"]][:, None, None]
    dv += dvc[blk["id"]] / cnt[blk["id"]][:, None, None]
    for t in range(nq):
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            js = selected_tokens(st["sel"][t, g], blk)
            if len(js) == 0:
                continue
            qr = q[t, hs, :]
            dor = dout[t, hs, :] * gw[t, hs, 1][:, None]
            p = np.exp(scale * (qr @ k[js, g, :].T) - st["lse"][1, t, hs][:, None])
            dp = dor @ v[js, g, :].T
            ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
            dq[t, hs, :] += scale * (ds @ k[js, g, :])
            np.add.at(dk[:, g, :], js, scale * (ds.T @ qr))
            np.add.at(dv[:, g, :], js, p.T @ dor)
    return {"dq": dq, "dk": dk, "dv": dv, "dgates": dgates, "dkc": dkc, "dvc": dvc}


def importance(st: State, t: int, g: int) -> np.ndarray:
    """fp64 selection score of every block of t's sequence for group g (local ids)."""
    cu = st["cu_seqlens"]
    s = int(np.searchsorted(cu, t, side="right") - 1)
    b0, b1 = int(st["blk"]["cu"][s]), int(st["blk"]["cu"][s + 1])
    G = st["G"]
    hs = slice(g * G, (g + 1) * G)
    _, _, p = cmp_attention(np.asarray(st["q"][t:t + 1, hs, :], np.float64), st["kc"][b0:b1, g, :],
                            st["vc"][b0:b1, g, :],
                            st["scale"])
    return p[0].sum(axis=0)


def attend_with_sel(st: State, t: int, g: int, sel_row: np.ndarray):
    """Selected-branch output of (t, g) for a given selection (used to check the
    attention itself when a certified near-tie flipped the selection)."""
    G = st["G"]
    hs = slice(g * G, (g + 1) * G)
    js = selected_tokens(np.asarray(sel_row), st["blk"])
    l_, o_, _ = _attend(np.asarray(st["q"][t, hs, :], np.float64), st["k"][js, g, :], st["v"][js, g, :],
                        st["scale"])
    return l_, o_


# ----------------------------------------------------------------------------
# step 7: backward (analytic chain rule of the forward, selection held fixed)
# ----------------------------------------------------------------------------


def backward(st: State, dout: np.ndarray, chunk: int = 256) -> dict:
    """Gradients of sum(dout * O) w.r.t. q, k, v and gates.  Requires a forward
    over all tokens.  Returns dq, dk, dv, dgates and the per-branch parts."""
    q, k, v = np.asarray(st["q"], np.float64), st["k"], st["v"]
    n, hq, d = q.shape
    hkv, G, scale = st["hkv"], st["G"], st["scale"]
    assert len(st["tokens"]) == n, "backward needs the full forward"
    blk, win = st["blk"], st["win"]
    dout = np.asarray(dout, dtype=np.float64)
    gw = gate_weights(st["gates"], st["gate_mode"])  # [N, Hq, 3]
    o = st["o"]

    # gates: O = sum_c w_c o_c
    dots = np.einsum("nhd,cnhd->nhc", dout, o)
    if st["gate_mode"] == 0:
        dgates = dots
    else:
        dgates = dots * gw * (1.0 - gw)

    dq = {c: np.zeros_like(q) for c in ("cmp", "slc", "win")}
    dk = {c: np.zeros_like(k) for c in ("cmp", "slc", "win")}
    dv = {c: np.zeros_like(v) for c in ("cmp", "slc", "win")}
    nb = blk["count"]
    dkc = np.zeros((nb, hkv, d))
    dvc = np.zeros((nb, hkv, d))
    seq = _seq_of_tokens(st["cu_seqlens"], n)

    def attn_bwd(qr, kk, vv, dor, lse_r):
        # qr [G, d], kk/vv [L, d], dor [G, d] (gate-weighted), lse_r [G]
        s = scale * (qr @ kk.T)
        p = np.exp(s - lse_r[:, None])
        dp = dor @ vv.T
        dsum = np.sum(p * dp, axis=1, keepdims=True)
        ds = p * (dp - dsum)
        return scale * (ds @ kk), scale * (ds.T @ qr), p.T @ dor

    # compressed branch
    for s in range(len(st["cu_seqlens"]) - 1):
        toks = np.nonzero(seq == s)[0]
        if len(toks) == 0:
            continue
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            kcg, vcg = st["kc"][b0:b1, g, :], st["vc"][b0:b1, g, :]
            for c0 in range(0, len(toks), chunk):
                tt = toks[c0:c0 + chunk]
                qr = q[tt, hs, :]
                dor = dout[tt, hs, :] * gw[tt, hs, 0][..., None]
                sc = scale * (qr @ kcg.T)
                p = np.exp(sc - st["lse"][0, tt, hs][..., None])
                dp = dor @ vcg.T
                dsum = np.sum(p * dp, axis=-1, keepdims=True)
                ds = p * (dp - dsum)
                dq["cmp"][tt, hs, :] = scale * (ds @ kcg)
                dkc[b0:b1, g, :] += scale * np.einsum("ngb,ngd->bd", ds, qr)
                dvc[b0:b1, g, :] += np.einsum("ngb,ngd->bd", p, dor)
    cnt = np.diff(blk["ptr"]).astype(np.float64)
    conv = st.get("conv")
    dconv = {}
    if conv is None:
        dk["cmp"] = dkc[blk["id"]] / cnt[blk["id"]][:, None, None]
        dv["cmp"] = dvc[blk["id"]] / cnt[blk["id"]][:, None, None]
    else:
        dk["cmp"], dconv["dwk"], dconv["dbk"] = conv_pool_backward(st["coords"], st["cu_seqlens"], k, conv["wk"],
                                                                   blk, dkc)
        dv["cmp"], dconv["dwv"], dconv["dbv"] = conv_pool_backward(st["coords"], st["cu_seqlens"], v, conv["wv"],
                                                                   blk, dvc)

    # selected-block and window branches
    for t in range(n):
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            js = selected_tokens(st["sel"][t, g], blk)
            a, b_, c_ = attn_bwd(q[t, hs, :], k[js, g, :], v[js, g, :],
                                 dout[t, hs, :] * gw[t, hs, 1][:, None], st["lse"][1, t, hs])
            dq["slc"][t, hs, :] = a
            np.add.at(dk["slc"][:, g, :], js, b_)
            np.add.at(dv["slc"][:, g, :], js, c_)
            w = win["id"][t]
            jw = win["perm"][win["ptr"][w]:win["ptr"][w + 1]]
            a, b_, c_ = attn_bwd(q[t, hs, :], k[jw, g, :], v[jw, g, :],
                                 dout[t, hs, :] * gw[t, hs, 2][:, None], st["lse"][2, t, hs])
            dq["win"][t, hs, :] = a
            np.add.at(dk["win"][:, g, :], jw, b_)
            np.add.at(dv["win"][:, g, :], jw, c_)

    return {
        "dq": dq["cmp"] + dq["slc"] + dq["win"],
        "dk": dk["cmp"] + dk["slc"] + dk["win"],
        "dv": dv["cmp"] + dv["slc"] + dv["win"],
        "dgates": dgates,
        "parts": {"dq": dq, "dk": dk, "dv": dv, "dkc": dkc, "dvc": dvc},
        **dconv,
    }


def dq_rows(st: State, dout: np.ndarray, tokens) -> np.ndarray:
    """dQ of the given query tokens only ([len(tokens), Hq, d]).  The gradient of a
    query row needs only that row's own softmax quantities, so this works on a
    forward restricted to those tokens; same arithmetic as `backward`."""
    q, k, v = st["q"], st["k"], st["v"]
    hkv, G, scale = st["hkv"], st["G"], st["scale"]
    blk, win = st["blk"], st["win"]
    gw = gate_weights(st["gates"], st["gate_mode"])
    cu = st["cu_seqlens"]
    out = np.zeros((len(tokens), q.shape[1], q.shape[2]))
    for i, t in enumerate(tokens):
        s = int(np.searchsorted(cu, t, side="right") - 1)
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            do = np.asarray(dout[t, hs, :], np.float64)
            w = win["id"][t]
            keysets = (
                (st["kc"][b0:b1, g, :], st["vc"][b0:b1, g, :]),
                (k[selected_tokens(st["sel"][t, g], blk), g, :], v[selected_tokens(st["sel"][t, g], blk), g, :]),
                (k[win["perm"][win["ptr"][w]:win["ptr"][w + 1]], g, :],
                 v[win["perm"][win["ptr"][w]:win["ptr"][w + 1]], g, :]),
            )
            for c, (kk, vv) in enumerate(keysets):
                dor = do * gw[t, hs, c][:, None]
                sc = scale * (np.asarray(q[t, hs, :], np.float64) @ kk.T)
                p = np.exp(sc - st["lse"][c, t, hs][:, None])
                dp = dor @ vv.T
                ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
                out[i, hs, :] += scale * (ds @ kk)
    return out


def dgates_rows(st: State, dout: np.ndarray, tokens) -> np.ndarray:
    """dgates of the given tokens only ([len(tokens), Hq, 3]); needs the forward
    rows of those tokens.  Same arithmetic as `backward`."""
    tokens = np.asarray(tokens)
    o = st["o"][:, tokens]
    do = np.asarray(dout[tokens], np.float64)
    dots = np.einsum("nhd,cnhd->nhc", do, o)
    if st["gate_mode"] == 0:
        return dots
    gw = gate_weights(st["gates"][tokens], st["gate_mode"])
    return dots * gw * (1.0 - gw)


def window_kv_grads(st: State, dout: np.ndarray, windows) -> tuple:
    """Window-branch dK, dV of every token of the given windows: (tokens,
    dk [len, Hkv, d], dv [len, Hkv, d]).  A key's window gradient comes only from
    the queries of its own window, so a forward restricted to those windows'
    tokens suffices.  Same arithmetic as `backward`."""
    q, k, v = st["q"], st["k"], st["v"]
    hkv, G, scale = st["hkv"], st["G"], st["scale"]
    win = st["win"]
    gw = gate_weights(st["gates"], st["gate_mode"])
    toks, dks, dvs = [], [], []
    for w in windows:
        jw = win["perm"][win["ptr"][w]:win["ptr"][w + 1]]
        dk = np.zeros((len(jw), hkv, k.shape[2]))
        dv = np.zeros_like(dk)
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            kk, vv = k[jw, g, :], v[jw, g, :]
            for t in jw:
                qr = np.asarray(q[t, hs, :], np.float64)
                dor = np.asarray(dout[t, hs, :], np.float64) * gw[t, hs, 2][:, None]
                p = np.exp(scale * (qr @ kk.T) - st["lse"][2, t, hs][:, None])
                dp = dor @ vv.T
                ds = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
                dk[:, g, :] += scale * (ds.T @ qr)
                dv[:, g, :] += p.T @ dor
        toks.append(jw)
        dks.append(dk)
        dvs.append(dv)
    return np.concatenate(toks), np.concatenate(dks), np.concatenate(dvs)


# ----------------------------------------------------------------------------
# the compressed branch alone over a range of query tokens (full-size checks)
# ----------------------------------------------------------------------------


def cmp_branch_range(q, kc, vc, blk_cu, cu_seqlens, gates, *, hq, hkv, topk, gate_mode, t0, t1,
                     dout=None, scale=None, chunk=256, sel_other=None) -> dict:
    """Forward and backward of the compressed branch (Direct3D-S2 "方法": every
    query attends to all compressed blocks of its sequence; the top-k blocks by
    that score are selected) for the query tokens t0 .. t1-1 only.

    The same definition as the compressed parts of `forward` and `backward`,
    restricted to a token range so that a long sequence can be split over
    processes: a query's lse, output, selection and dQ need only its own row, and
    dKc / dVc are sums over query rows, so the per-range dkc / dvc returned here
    add up to the full ones.  q, dout [N, Hq, d] (any float type, exact values);
    kc, vc [B, Hkv, d] float64 (the stored, rounded block means); blk_cu [S+1]
    block offsets per sequence; gates [N, Hq, 3] (only column 0 is used).

    Returns lse [T, Hq], o [T, Hq, d], sel [T, Hkv, topk] (global ids ascending,
    -1 padded), and with dout: dq [T, Hq, d] (this branch's part), dkc / dvc
    [B, Hkv, d] (these rows' sums).  With `sel_other` (another selection of the
    same rows, [T, Hkv, topk] global ids, -1 padded) also other_gap [T, Hkv]: the
    lowest selection score among the blocks it chose minus the highest among the
    blocks of the sequence it left out (+inf when it chose every block); a valid
    top-k of these scores has other_gap >= 0, a near-tie choice >= -tau.
    """
    n, _, d = q.shape
    G = hq // hkv
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    cu_seqlens = np.asarray(cu_seqlens, np.int64)
    blk_cu = np.asarray(blk_cu, np.int64)
    T = t1 - t0
    lse = np.full((T, hq), np.nan)
    o = np.zeros((T, hq, d))
    sel = np.full((T, hkv, topk), -1, dtype=np.int64)
    res = {"lse": lse, "o": o, "sel": sel}
    if sel_other is not None:
        gap = np.full((T, hkv), np.inf)
        res["other_gap"] = gap
    if dout is not None:
        dq = np.zeros((T, hq, d))
        dkc = np.zeros(kc.shape)
        dvc = np.zeros(vc.shape)
        res.update(dq=dq, dkc=dkc, dvc=dvc)
    for s in range(len(cu_seqlens) - 1):
        a, b = max(t0, int(cu_seqlens[s])), min(t1, int(cu_seqlens[s + 1]))
        if a >= b:
            continue
        b0, b1 = int(blk_cu[s]), int(blk_cu[s + 1])
        for g in range(hkv):
            hs = slice(g * G, (g + 1) * G)
            kcg, vcg = kc[b0:b1, g, :], vc[b0:b1, g, :]
            for c0 in range(a, b, chunk):
                tt = np.arange(c0, min(b, c0 + chunk))
                r = tt - t0
                qr = np.asarray(q[tt, hs, :], np.float64)
                l_, o_, p = cmp_attention(qr, kcg, vcg, scale)
                lse[r, hs] = l_
                o[r, hs, :] = o_
                imp = p.sum(axis=1)  # [n, B_s]: probabilities summed over the group's heads
                loc = topk_blocks(imp, topk)
                sel[r, g, :] = np.where(loc >= 0, loc + b0, -1)
                if sel_other is not None:
                    chosen = np.zeros(imp.shape, bool)
                    for i, row in enumerate(np.asarray(sel_other)[r, g]):
                        ids = row[(row >= b0) & (row < b1)] - b0
                        chosen[i, ids] = True
                    lo = np.where(chosen, imp, np.inf).min(axis=1)
                    hi = np.where(chosen, -np.inf, imp).max(axis=1)
                    gap[r, g] = np.where(chosen.all(axis=1), np.inf, lo - hi)
                if dout is None:
                    continue
                w = gate_weights(gates[tt, hs, 0], gate_mode)
                dor = np.asarray(dout[tt, hs, :], np.float64) * w[..., None]
                dp = dor @ vcg.T
                ds = p * (dp - np.sum(p * dp, axis=-1, keepdims=True))
                dq[r, hs, :] = scale * (ds @ kcg)
                # sums over the chunk's (token, head) rows: [B_s, rows] x [rows, d]
                dkc[b0:b1, g, :] += scale * (ds.reshape(-1, b1 - b0).T @ qr.reshape(-1, d))
                dvc[b0:b1, g, :] += p.reshape(-1, b1 - b0).T @ dor.reshape(-1, d)
    return res


def cmp_token_grads(dkc: np.ndarray, dvc: np.ndarray, blk: dict):
    """dK, dV [N, Hkv, d] of the compressed branch from dKc, dVc: each token gets
    its block's gradient divided by the block size (the mean's derivative)."""
    cnt = np.diff(blk["ptr"]).astype(np.float64)
    return dkc[blk["id"]] / cnt[blk["id"]][:, None, None], dvc[blk["id"]] / cnt[blk["id"]][:, None, None]


# ----------------------------------------------------------------------------
# 3D-aware block routing (selection by geometric distance instead of scores)
# ----------------------------------------------------------------------------


def geo_topk(coords: np.ndarray, cu_seqlens: np.ndarray, m_cmp: int, k: int, tokens=None) -> np.ndarray:
    """Selection by explicit geometric distance (LSRM, shuwu5.cn/article/2502.html,
    "3D 感知空间块路由机制", voxel-only case): a voxel token's point is the centre of
    its voxel; the distance of a query token to a block is the shortest Euclidean
    distance to the points of the block's tokens; each token selects the k blocks of
    its sequence nearest to it (ties: lower block id), stored ascending, padded -1.

    Voxel centres differ by integer vectors, so squared distances are exact integers.
    Returns global block ids [len(tokens), k] (all tokens by default)."""
    coords = np.asarray(coords, np.int64)
    cu = np.asarray(cu_seqlens, np.int64)
    blk = bin_tokens(coords, cu, m_cmp)
    n = len(coords)
    tokens = np.arange(n) if tokens is None else np.asarray(tokens, np.int64)
    seq = _seq_of_tokens(cu, n)
    out = np.full((len(tokens), k), -1, np.int64)
    for row, t in enumerate(tokens):
        s = seq[t]
        b0, b1 = int(blk["cu"][s]), int(blk["cu"][s + 1])
        members = np.arange(cu[s], cu[s + 1])
        d2 = np.sum((coords[members] - coords[t]) ** 2, axis=1)
        best = np.full(b1 - b0, np.iinfo(np.int64).max)
        np.minimum.at(best, blk["id"][members] - b0, d2)
        keff = min(k, b1 - b0)
        order = np.lexsort((np.arange(b1 - b0), best))[:keff]  # by distance, then by id
        out[row, :keff] = np.sort(order) + b0
    return out
