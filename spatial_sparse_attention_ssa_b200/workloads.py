"""Seeded synthetic inputs shaped like the sparse-voxel workloads of the pages.

Direct3D-S2 (hyper.ai, "方法" section) runs SSA on the sparse voxels of a
surface at up to 1024^3, with more than 100k tokens; LSRM (shuwu5.cn,
"活跃 Token 稀疏筛选") keeps only voxels whose SDF is within a threshold of
the surface.  No dataset is used: these generators build surface shells of
random analytic shapes (unions of ellipsoids and thin slabs) and draw the
attention tensors from N(0, 1).

This module is shared by the tests, the bench and the oracle's callers.  It
holds no step of the attention method: only geometry, random numbers and the
rounding of the drawn values to the storage dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# ----------------------------------------------------------------------------
# bf16 helpers (input preparation only)
# ----------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # u + 0x7FFF + lsb stays below 2^32 for every finite float32 (NaN payloads
    # above 0xFFFF8000 are never generated)
    r = (u >> 16) & np.uint32(1)
    r += np.uint32(0x7FFF)
    r += u
    r >>= 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# Surface-shell geometry
# ----------------------------------------------------------------------------


def _ellipsoid_sdf(p: np.ndarray, c: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Approximate signed distance to an axis-aligned ellipsoid.

    The bound k0 (k0 - 1) / k1 with k0 = |(p-c)/r|, k1 = |(p-c)/r^2|
    (I. Quilez's ellipsoid estimate); exact for spheres.
    """
    q = (p - c) / r
    k0 = np.linalg.norm(q, axis=-1)
    k1 = np.linalg.norm(q / r, axis=-1)
    with np.errstate(invalid="ignore", divide="ignore"):
        d = k0 * (k0 - 1.0) / k1
    return np.where(k1 > 0, d, -np.min(r))


def _box_sdf(p: np.ndarray, c: np.ndarray, b: np.ndarray) -> np.ndarray:
    q = np.abs(p - c) - b
    outside = np.linalg.norm(np.maximum(q, 0.0), axis=-1)
    inside = np.minimum(np.max(q, axis=-1), 0.0)
    return outside + inside


@dataclass
class Primitive:
    kind: str  # "ellipsoid" | "box" | "sphere"
    center: np.ndarray
    size: np.ndarray  # semi-axes / half-extents / (radius,)

    def sdf(self, p: np.ndarray) -> np.ndarray:
        if self.kind == "ellipsoid":
            return _ellipsoid_sdf(p, self.center, self.size)
        if self.kind == "box":
            return _box_sdf(p, self.center, self.size)
        if self.kind == "sphere":
            return np.linalg.norm(p - self.center, axis=-1) - self.size[0]
        raise ValueError(self.kind)

    def extent(self) -> np.ndarray:
        if self.kind == "sphere":
            return np.full(3, self.size[0])
        return np.asarray(self.size, dtype=np.float64)


def shell_voxels(R: int, prims: list[Primitive], thresh: float) -> np.ndarray:
    """Integer voxels (i, j, k) of an R^3 grid whose centre (i+.5, j+.5, k+.5)
    lies within `thresh` of the surface of the union (min of SDFs) of `prims`.

    Returned in raster order (x-major, then y, then z), int32 [n, 3].
    """
    cand = []
    for pr in prims:
        ext = pr.extent() + thresh + 1.0
        lo = np.clip(np.floor(pr.center - ext).astype(np.int64), 0, R - 1)
        hi = np.clip(np.ceil(pr.center + ext).astype(np.int64), 0, R - 1)
        # scan slab by slab along x to bound memory
        ys = np.arange(lo[1], hi[1] + 1)
        zs = np.arange(lo[2], hi[2] + 1)
        yy, zz = np.meshgrid(ys, zs, indexing="ij")
        yy = yy.reshape(-1)
        zz = zz.reshape(-1)
        for x in range(lo[0], hi[0] + 1):
            p = np.stack([np.full_like(yy, x), yy, zz], axis=-1).astype(np.float64) + 0.5
            d = pr.sdf(p)
            keep = np.abs(d) < thresh
            if keep.any():
                cand.append(np.stack([np.full(keep.sum(), x), yy[keep], zz[keep]], axis=-1))
    if not cand:
        return np.zeros((0, 3), np.int32)
    v = np.unique(np.concatenate(cand).astype(np.int64), axis=0)
    # inside-any check: a voxel deep inside another primitive is not on the union's surface
    p = v.astype(np.float64) + 0.5
    dmin = np.full(len(v), np.inf)
    for pr in prims:
        dmin = np.minimum(dmin, pr.sdf(p))
    v = v[np.abs(dmin) < thresh]
    # raster order x-major
    order = np.lexsort((v[:, 2], v[:, 1], v[:, 0]))
    return v[order].astype(np.int32)


def _random_ellipsoids(rng, R, n, lo, hi):
    prims = []
    for _ in range(n):
        r = rng.uniform(lo, hi, size=3)
        c = np.array([rng.uniform(r[i], R - r[i]) for i in range(3)])
        prims.append(Primitive("ellipsoid", c, r))
    return prims


def _random_slabs(rng, R, n, lo, hi, half_thickness=1.5):
    prims = []
    for _ in range(n):
        b = rng.uniform(lo, hi, size=3)
        axis = int(rng.integers(0, 3))
        b[axis] = half_thickness
        c = np.array([rng.uniform(b[i], R - b[i]) for i in range(3)])
        prims.append(Primitive("box", c, b))
    return prims


def _subsample(rng, v: np.ndarray, n: int) -> np.ndarray:
    if n >= len(v):
        return v
    idx = np.sort(rng.choice(len(v), size=n, replace=False))
    return v[idx]


# ----------------------------------------------------------------------------
# Workload descriptions
# ----------------------------------------------------------------------------


@dataclass
class Workload:
    name: str
    R: int
    coords: np.ndarray  # int32 [N, 3]
    cu_seqlens: np.ndarray  # int32 [S+1]
    hq: int
    hkv: int
    d: int
    m_cmp: int
    m_win: int
    topk: int
    dtype: str  # "bf16" | "f32"
    gate_mode: int  # 0 weights, 1 logits -> sigmoid
    seed: int
    backward: bool = False
    notes: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])

    @property
    def s(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)


def tiny_sphere(seed: int = 0, n_keep: int = 2048) -> Workload:
    """64^3 grid, voxels within half a cell of a sphere of radius 24 at the
    grid centre (|SDF| < 0.5 reading of "within 1 cell"), subsampled."""
    rng = np.random.default_rng(seed)
    sph = Primitive("sphere", np.array([32.0, 32.0, 32.0]), np.array([24.0]))
    v = shell_voxels(64, [sph], 0.5)
    v = _subsample(rng, v, n_keep)
    return Workload("tiny_fp32_sphere64", 64, v, np.array([0, len(v)], np.int32),
                    hq=2, hkv=1, d=32, m_cmp=4, m_win=4, topk=4, dtype="f32",
                    gate_mode=0, seed=seed)


def ellipsoids256(seed: int = 0) -> Workload:
    """256^3, surface shell (|SDF| < 1) of 3 random ellipsoids, semi-axes U(40,100)."""
    rng = np.random.default_rng(seed)
    prims = _random_ellipsoids(rng, 256, 3, 40.0, 100.0)
    v = shell_voxels(256, prims, 1.0)
    return Workload("bf16_ellipsoids256", 256, v, np.array([0, len(v)], np.int32),
                    hq=16, hkv=2, d=64, m_cmp=8, m_win=8, topk=8, dtype="bf16",
                    gate_mode=1, seed=seed)


def gigascale1024(seed: int = 0, n_keep: int = 131072, backward: bool = False,
                  axis_lo: float = 20.0, axis_hi: float = 50.0) -> Workload:
    """1024^3, shell of 5 random ellipsoids + 2 thin slabs (half-thickness 1.5),
    subsampled to exactly n_keep tokens.  Semi-axes / half-extents U(20, 50)."""
    tries = 0
    s = seed
    while True:
        rng = np.random.default_rng(s)
        prims = _random_ellipsoids(rng, 1024, 5, axis_lo, axis_hi)
        prims += _random_slabs(rng, 1024, 2, axis_lo, axis_hi)
        v = shell_voxels(1024, prims, 1.0)
        if len(v) >= n_keep:
            break
        tries += 1
        s = seed + 1000 * tries
    v = _subsample(rng, v, n_keep)
    return Workload("bf16_gigascale1024" + ("_fwdbwd" if backward else ""), 1024, v,
                    np.array([0, len(v)], np.int32), hq=32, hkv=2, d=64, m_cmp=8,
                    m_win=8, topk=16, dtype="bf16", gate_mode=1, seed=seed,
                    backward=backward, notes={"geometry_seed": s})


def varlen512(seed: int = 100, n_shapes: int = 4, lo: int = 20000, hi: int = 120000,
              scale_counts: float = 1.0) -> Workload:
    """n_shapes sequences, each the shell of 3 ellipsoids (semi-axes U(30,70)) in
    512^3 with a token count drawn U(lo, hi) from the same generator."""
    coords = []
    cu = [0]
    for i in range(n_shapes):
        s = seed + i
        while True:
            rng = np.random.default_rng(s)
            prims = _random_ellipsoids(rng, 512, 3, 30.0, 70.0)
            n_s = int(np.floor(rng.uniform(lo, hi) * scale_counts))
            v = shell_voxels(512, prims, 1.0)
            if len(v) >= n_s:
                break
            s += 1000
        v = _subsample(rng, v, n_s)
        coords.append(v)
        cu.append(cu[-1] + len(v))
    return Workload("bf16_varlen512x%d" % n_shapes, 512, np.concatenate(coords).astype(np.int32),
                    np.array(cu, np.int32), hq=16, hkv=2, d=64, m_cmp=8, m_win=8, topk=8,
                    dtype="bf16", gate_mode=1, seed=seed)


def small_shell(seed: int = 0, R: int = 64, n_prims: int = 2, lo: float = 6.0, hi: float = 14.0,
                n_keep: int | None = None, hq: int = 16, hkv: int = 2, d: int = 64,
                m_cmp: int = 4, m_win: int = 4, topk: int = 8, dtype: str = "bf16",
                gate_mode: int = 1, n_seqs: int = 1) -> Workload:
    """Small shells for parity tests: several tiles and ragged tails, seconds of oracle work."""
    coords = []
    cu = [0]
    for i in range(n_seqs):
        rng = np.random.default_rng(seed * 131 + i)
        prims = _random_ellipsoids(rng, R, n_prims, lo, hi)
        v = shell_voxels(R, prims, 1.0)
        if n_keep is not None:
            v = _subsample(rng, v, n_keep if i == 0 else max(1, n_keep // (i + 1) + 7 * i))
        coords.append(v)
        cu.append(cu[-1] + len(v))
    return Workload("small_shell_R%d" % R, R, np.concatenate(coords).astype(np.int32),
                    np.array(cu, np.int32), hq=hq, hkv=hkv, d=d, m_cmp=m_cmp, m_win=m_win,
                    topk=topk, dtype=dtype, gate_mode=gate_mode, seed=seed)


def config(i: int, seed: int | None = None) -> Workload:
    """The five benchmark configurations (1-based)."""
    if i == 1:
        return tiny_sphere(0 if seed is None else seed)
    if i == 2:
        return ellipsoids256(0 if seed is None else seed)
    if i == 3:
        return gigascale1024(0 if seed is None else seed)
    if i == 4:
        return varlen512(100 if seed is None else seed)
    if i == 5:
        return gigascale1024(0 if seed is None else seed, backward=True)
    raise ValueError(i)


# ----------------------------------------------------------------------------
# Tensors
# ----------------------------------------------------------------------------


@dataclass
class Tensors:
    """Host arrays.  For bf16 workloads q/k/v/do hold uint16 bf16 bits; the
    exact values as float32 are available through `as_f32`."""
    q: np.ndarray  # [N, Hq, d]
    k: np.ndarray  # [N, Hkv, d]
    v: np.ndarray  # [N, Hkv, d]
    gates: np.ndarray  # f32 [N, Hq, 3]
    do: np.ndarray | None  # [N, Hq, d]
    dtype: str

    def as_f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        if self.dtype == "bf16" and a.dtype == np.uint16:
            return bf16_bits_to_f32(a)
        return a.astype(np.float32, copy=False)


def _normal(rng, shape, dtype: str) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x).reshape(shape)
    return x


def make_tensors(w: Workload, seed: int | None = None, with_do: bool | None = None) -> Tensors:
    """Q, K, V ~ N(0,1) in the workload dtype; gates U(0,1) (weights) or
    N(0,1) (logits); upstream gradient dO ~ N(0,1)."""
    rng = np.random.default_rng(np.random.SeedSequence([w.seed if seed is None else seed, 7919]))
    n = w.n
    q = _normal(rng, (n, w.hq, w.d), w.dtype)
    k = _normal(rng, (n, w.hkv, w.d), w.dtype)
    v = _normal(rng, (n, w.hkv, w.d), w.dtype)
    if w.gate_mode == 0:
        gates = rng.uniform(0.0, 1.0, size=(n, w.hq, 3)).astype(np.float32)
    else:
        gates = rng.standard_normal(size=(n, w.hq, 3), dtype=np.float32)
    if with_do is None:
        with_do = True
    do = _normal(rng, (n, w.hq, w.d), w.dtype) if with_do else None
    return Tensors(q, k, v, gates, do, w.dtype)


@dataclass
class CrossQueries:
    """Queries of another token set (image tokens in LSRM's cross attention) for
    the voxel sequences of a workload: sequence s owns rows q_cu[s] .. q_cu[s+1]-1."""
    q_cu: np.ndarray  # int64 [S + 1]
    q: np.ndarray  # [Nq, Hq, d], bf16 bits or f32
    gates: np.ndarray  # f32 [Nq, Hq, 2] (compressed, selected)
    do: np.ndarray  # [Nq, Hq, d]
    dtype: str

    def as_f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        if self.dtype == "bf16" and a.dtype == np.uint16:
            return bf16_bits_to_f32(a)
        return a.astype(np.float32, copy=False)


def make_cross_queries(w: Workload, q_lens, seed: int = 0) -> CrossQueries:
    """Q, dO ~ N(0,1) in the workload dtype for len(q_lens) == S sequences; gates as
    in make_tensors (U(0,1) weights or N(0,1) logits), two columns."""
    q_lens = np.asarray(q_lens, np.int64)
    assert len(q_lens) == w.s
    rng = np.random.default_rng(np.random.SeedSequence([w.seed, seed, 104729]))
    nq = int(q_lens.sum())
    q_cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int64)
    q = _normal(rng, (nq, w.hq, w.d), w.dtype)
    if w.gate_mode == 0:
        gates = rng.uniform(0.0, 1.0, size=(nq, w.hq, 2)).astype(np.float32)
    else:
        gates = rng.standard_normal(size=(nq, w.hq, 2), dtype=np.float32)
    do = _normal(rng, (nq, w.hq, w.d), w.dtype)
    return CrossQueries(q_cu, q, gates, do, w.dtype)


def permute_workload(w: Workload, t: Tensors, seed: int) -> tuple[Workload, Tensors, np.ndarray]:
    """Shuffle tokens inside each sequence (for permutation-equivariance checks).
    Returns the new workload, tensors and `src` with new[i] = old[src[i]]."""
    rng = np.random.default_rng(seed)
    src = np.arange(w.n)
    for s in range(w.s):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        src[a:b] = a + rng.permutation(b - a)
    w2 = Workload(w.name + "_perm", w.R, w.coords[src], w.cu_seqlens.copy(), w.hq, w.hkv, w.d,
                  w.m_cmp, w.m_win, w.topk, w.dtype, w.gate_mode, w.seed, w.backward)
    t2 = Tensors(t.q[src], t.k[src], t.v[src], t.gates[src],
                 None if t.do is None else t.do[src], t.dtype)
    return w2, t2, src
