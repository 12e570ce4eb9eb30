"""ctypes binding of libssa.so (argument marshalling only).

Each call here converts torch tensors to device pointers, sizes and the
current CUDA stream, allocates the caller-owned outputs and workspace with
torch, and calls the C ABI of include/ssa.h.  Every step of the attention
runs in the library's CUDA kernels; there is no CPU path.  A missing or
unloadable library raises immediately.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssa.so")

SSA_OK = 0
STATUS_NAMES = {0: "SSA_OK", 1: "SSA_ERR_INVALID_ARG", 2: "SSA_ERR_UNSUPPORTED", 3: "SSA_ERR_WORKSPACE",
                4: "SSA_ERR_COORD_RANGE", 5: "SSA_ERR_CUDA", 6: "SSA_ERR_TIMEOUT"}
DTYPE_BF16, DTYPE_F32 = 0, 1
GATE_WEIGHTS, GATE_LOGITS = 0, 1
OP_BIN, OP_FORWARD, OP_BACKWARD, OP_GEO_SELECT, OP_CROSS_FORWARD, OP_CROSS_BACKWARD = 0, 1, 2, 3, 4, 5
OP_SP_FORWARD, OP_SP_BACKWARD = 6, 7
SEL_SCORES, SEL_GIVEN = 0, 1

EXPORTS = ("ssa_bin", "ssa_forward", "ssa_backward", "ssa_workspace_size", "ssa_error_string",
           "ssa_get_device_status", "ssa_version", "ssa_launch_count", "ssa_profile_enable",
           "ssa_profile_read", "ssa_geo_select", "ssa_cross_forward", "ssa_cross_backward", "ssa_pool",
           "ssa_diag_wait_timeout", "ssa_diag_ex2", "ssa_sp_forward", "ssa_sp_backward")


class SSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (where, STATUS_NAMES.get(status, status),
                                                 _lib().ssa_error_string(status).decode()))


class Conv(ctypes.Structure):
    _fields_ = [("coords", ctypes.c_void_p), ("wk", ctypes.c_void_p), ("bk", ctypes.c_void_p),
                ("wv", ctypes.c_void_p), ("bv", ctypes.c_void_p), ("dwk", ctypes.c_void_p),
                ("dbk", ctypes.c_void_p), ("dwv", ctypes.c_void_p), ("dbv", ctypes.c_void_p)]


class Params(ctypes.Structure):
    _fields_ = [("hq", ctypes.c_int32), ("hkv", ctypes.c_int32), ("d", ctypes.c_int32),
                ("m_cmp", ctypes.c_int32), ("m_win", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("scale", ctypes.c_float), ("dtype", ctypes.c_int32), ("gate_mode", ctypes.c_int32),
                ("selection", ctypes.c_int32), ("conv", ctypes.POINTER(Conv)), ("deterministic", ctypes.c_int32)]


class Partition(ctypes.Structure):
    _fields_ = [("id", ctypes.c_void_p), ("perm", ctypes.c_void_p), ("ptr", ctypes.c_void_p),
                ("cu", ctypes.c_void_p), ("key", ctypes.c_void_p), ("count", ctypes.c_int64)]


class SpLocalC(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("cu_seqlens", ctypes.c_void_p), ("tokens", ctypes.c_void_p),
                ("win", ctypes.POINTER(Partition)), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("ks", ctypes.c_void_p), ("vs", ctypes.c_void_p)]


class Saved(ctypes.Structure):
    _fields_ = [("kc", ctypes.c_void_p), ("vc", ctypes.c_void_p), ("ks", ctypes.c_void_p),
                ("vs", ctypes.c_void_p), ("o_branch", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("sel", ctypes.c_void_p)]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libssa.so is not built (python -m spatial_sparse_attention_ssa_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        pp = ctypes.POINTER(Partition)
        lib.ssa_bin.argtypes = [vp, vp, i32, i64, i32, i32, i32, pp, pp, vp, sz, vp]
        lib.ssa_bin.restype = ctypes.c_int
        lib.ssa_forward.argtypes = [ctypes.POINTER(Params), vp, i32, i64, pp, pp, vp, vp, vp, vp, vp,
                                    ctypes.POINTER(Saved), vp, sz, vp]
        lib.ssa_forward.restype = ctypes.c_int
        lib.ssa_backward.argtypes = [ctypes.POINTER(Params), vp, i32, i64, pp, pp, vp, vp, vp, vp,
                                     ctypes.POINTER(Saved), vp, vp, vp, vp, vp, vp, sz, vp]
        lib.ssa_backward.restype = ctypes.c_int
        lib.ssa_cross_forward.argtypes = [ctypes.POINTER(Params), vp, i32, i64, i64, pp, vp, vp, vp, vp, vp,
                                          ctypes.POINTER(Saved), vp, sz, vp]
        lib.ssa_cross_forward.restype = ctypes.c_int
        lib.ssa_cross_backward.argtypes = [ctypes.POINTER(Params), vp, i32, i64, i64, pp, vp, vp, vp, vp,
                                           ctypes.POINTER(Saved), vp, vp, vp, vp, vp, vp, sz, vp]
        lib.ssa_cross_backward.restype = ctypes.c_int
        spp = ctypes.POINTER(SpLocalC)
        lib.ssa_sp_forward.argtypes = [ctypes.POINTER(Params), i32, i64, pp, spp, vp, vp, vp, vp, vp,
                                       ctypes.POINTER(Saved), vp, sz, vp]
        lib.ssa_sp_forward.restype = ctypes.c_int
        lib.ssa_sp_backward.argtypes = [ctypes.POINTER(Params), i32, i64, pp, spp, vp, vp, vp, vp,
                                        ctypes.POINTER(Saved), vp, vp, vp, vp, vp, vp, sz, vp]
        lib.ssa_sp_backward.restype = ctypes.c_int
        lib.ssa_diag_wait_timeout.argtypes = [vp, vp]
        lib.ssa_diag_wait_timeout.restype = ctypes.c_int
        lib.ssa_diag_ex2.argtypes = [vp, vp, vp, i64, vp]
        lib.ssa_diag_ex2.restype = ctypes.c_int
        lib.ssa_pool.argtypes = [i32, i32, i32, i64, pp, vp, vp, vp, vp, vp, vp, vp]
        lib.ssa_pool.restype = ctypes.c_int
        lib.ssa_geo_select.argtypes = [vp, vp, i32, i64, i32, pp, i32, i32, i32, vp, vp, sz, vp]
        lib.ssa_geo_select.restype = ctypes.c_int
        lib.ssa_workspace_size.argtypes = [i32, ctypes.POINTER(Params), i32, i64, i64, i64]
        lib.ssa_workspace_size.restype = sz
        lib.ssa_error_string.argtypes = [ctypes.c_int]
        lib.ssa_error_string.restype = ctypes.c_char_p
        lib.ssa_get_device_status.argtypes = [vp]
        lib.ssa_get_device_status.restype = ctypes.c_int
        lib.ssa_version.argtypes = []
        lib.ssa_version.restype = i32
        lib.ssa_launch_count.argtypes = []
        lib.ssa_launch_count.restype = ctypes.c_uint64
        lib.ssa_profile_enable.argtypes = [i32]
        lib.ssa_profile_enable.restype = None
        lib.ssa_profile_read.argtypes = [ctypes.c_char_p, i32, ctypes.POINTER(ctypes.c_float),
                                         ctypes.POINTER(ctypes.c_int32), i32]
        lib.ssa_profile_read.restype = i32
        _LIB = lib
    return _LIB


def lib():
    """The loaded ctypes library (raises if it is not built)."""
    return _lib()


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(device: torch.device | None = None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check(status: int, where: str) -> None:
    if status != SSA_OK:
        raise SSAError(status, where)


def _require_cuda(*ts: torch.Tensor) -> None:
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("SSA tensors must be contiguous CUDA tensors")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# binning
# ---------------------------------------------------------------------------


@dataclass
class Bins:
    """One partition (blocks or windows): device int32 tensors + count."""
    id: torch.Tensor
    perm: torch.Tensor
    ptr: torch.Tensor
    cu: torch.Tensor
    key: torch.Tensor
    count: int

    @staticmethod
    def empty(n: int, s: int, device) -> "Bins":
        z = lambda *shape: torch.empty(*shape, dtype=torch.int32, device=device)  # noqa: E731
        return Bins(z(n), z(n), z(n + 1), z(s + 1), z(max(n, 1), 3), 0)

    def c(self) -> Partition:
        return Partition(_ptr(self.id), _ptr(self.perm), _ptr(self.ptr), _ptr(self.cu), _ptr(self.key),
                         self.count)


def ssa_bin(coords: torch.Tensor, cu_seqlens: torch.Tensor, R: int, m_cmp: int, m_win: int,
            out: tuple[Bins, Bins] | None = None, workspace: torch.Tensor | None = None):
    """Step 1: block and window partitions of the tokens.  Returns (blk, win)."""
    _require_cuda(coords, cu_seqlens)
    n = int(coords.shape[0])
    s = int(cu_seqlens.shape[0]) - 1
    dev = coords.device
    blk, win = out if out is not None else (Bins.empty(n, s, dev), Bins.empty(n, s, dev))
    L = _lib()
    need = L.ssa_workspace_size(OP_BIN, None, s, n, n, n)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, pw = blk.c(), win.c()
    st = L.ssa_bin(_ptr(coords), _ptr(cu_seqlens), s, n, int(R), int(m_cmp), int(m_win),
                   ctypes.byref(pb), ctypes.byref(pw), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ssa_bin")
    blk.count = int(pb.count)
    win.count = int(pw.count)
    return blk, win


def ssa_pool(blk: "Bins", k: torch.Tensor, v: torch.Tensor, out=None):
    """Step 2 alone: (ks, vs, kc, vc) -- K and V gathered in block order, head-major
    [Hkv, N, d], and the block means [Hkv, B, d], in the dtype of k."""
    _require_cuda(k, v)
    n, hkv, d = (int(x) for x in k.shape)
    dt = DTYPE_BF16 if k.dtype == torch.bfloat16 else DTYPE_F32
    if out is None:
        e = lambda *shape: torch.empty(*shape, dtype=k.dtype, device=k.device)  # noqa: E731
        out = (e(hkv, n, d), e(hkv, n, d), e(hkv, max(blk.count, 1), d), e(hkv, max(blk.count, 1), d))
    ks, vs, kc, vc = out
    pb = blk.c()
    st = _lib().ssa_pool(dt, hkv, d, n, ctypes.byref(pb), _ptr(k), _ptr(v), _ptr(ks), _ptr(vs), _ptr(kc), _ptr(vc),
                         _stream(k.device))
    _check(st, "ssa_pool")
    return ks, vs, kc, vc


def ssa_geo_select(coords: torch.Tensor, cu_seqlens: torch.Tensor, R: int, blk: "Bins", m_cmp: int, topk: int,
                   hkv: int, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """3D-aware block routing: the topk blocks nearest to each token (shortest
    distance between voxel centres; ties to the lower id), int32 [N, hkv, topk]
    global block ids, ascending, padded with -1, the same for every KV group."""
    _require_cuda(coords, cu_seqlens)
    n = int(coords.shape[0])
    s = int(cu_seqlens.shape[0]) - 1
    dev = coords.device
    sel = out if out is not None else torch.empty((n, hkv, topk), dtype=torch.int32, device=dev)
    L = _lib()
    need = L.ssa_workspace_size(OP_GEO_SELECT, None, s, n, blk.count, 0)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb = blk.c()
    st = L.ssa_geo_select(_ptr(coords), _ptr(cu_seqlens), s, n, int(R), ctypes.byref(pb), int(m_cmp), int(topk),
                          int(hkv), _ptr(sel), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ssa_geo_select")
    return sel


def ssa_bin_noalloc(coords: torch.Tensor, cu_seqlens: torch.Tensor, R: int, m_cmp: int, m_win: int,
                    out: tuple[Bins, Bins] | None = None):
    """ssa_bin with the library's fixed internal scratch instead of a workspace,
    for callers that cannot allocate device memory at binning time (up to
    SSA_BIN_NOALLOC_MAX_TOKENS tokens; calls that overlap on the GPU race).
    `out` must be preallocated by such callers; without it this wrapper
    allocates the output tensors itself with torch."""
    _require_cuda(coords, cu_seqlens)
    n = int(coords.shape[0])
    s = int(cu_seqlens.shape[0]) - 1
    dev = coords.device
    blk, win = out if out is not None else (Bins.empty(n, s, dev), Bins.empty(n, s, dev))
    L = _lib()
    fn = L.ssa_bin_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                   ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(Partition), ctypes.POINTER(Partition),
                   ctypes.c_void_p]
    fn.restype = ctypes.c_int
    pb, pw = blk.c(), win.c()
    st = fn(_ptr(coords), _ptr(cu_seqlens), s, n, int(R), int(m_cmp), int(m_win), ctypes.byref(pb),
            ctypes.byref(pw), _stream(dev))
    _check(st, "ssa_bin_noalloc")
    blk.count = int(pb.count)
    win.count = int(pw.count)
    return blk, win


# ---------------------------------------------------------------------------
# forward / backward
# ---------------------------------------------------------------------------


@dataclass
class ConvWeights:
    """Learned compression: a sparse 3x3x3 convolution of K and V before the block
    mean.  coords int32 [N, 3]; wk / wv fp32 [Hkv, 27, d, d] (offset, in, out); bk /
    bv fp32 [Hkv, d]; the gradients dwk, dbk, dwv, dbv (same shapes) are written by
    ssa_backward."""
    coords: torch.Tensor
    wk: torch.Tensor
    bk: torch.Tensor
    wv: torch.Tensor
    bv: torch.Tensor
    dwk: torch.Tensor | None = None
    dbk: torch.Tensor | None = None
    dwv: torch.Tensor | None = None
    dbv: torch.Tensor | None = None

    def __post_init__(self):
        for name in ("dwk", "dbk", "dwv", "dbv"):
            if getattr(self, name) is None:
                setattr(self, name, torch.zeros_like(getattr(self, name[1:])))
        self._c = Conv(*(_ptr(getattr(self, f)) for f, _ in Conv._fields_))


def make_params(hq, hkv, d, m_cmp, m_win, topk, dtype: torch.dtype, gate_mode: int,
                scale: float = 0.0, selection: int = SEL_SCORES, conv: ConvWeights | None = None,
                deterministic: bool = False) -> Params:
    dt = DTYPE_BF16 if dtype == torch.bfloat16 else DTYPE_F32 if dtype == torch.float32 else None
    if dt is None:
        raise ValueError("dtype must be torch.bfloat16 or torch.float32")
    prm = Params(hq, hkv, d, m_cmp, m_win, topk, scale, dt, gate_mode, selection,
                 ctypes.pointer(conv._c) if conv is not None else None, 1 if deterministic else 0)
    prm._conv = conv  # keeps the weights (and the struct the pointer refers to) alive
    return prm


@dataclass
class SavedTensors:
    kc: torch.Tensor
    vc: torch.Tensor
    ks: torch.Tensor
    vs: torch.Tensor
    o_branch: torch.Tensor
    lse: torch.Tensor
    sel: torch.Tensor

    @staticmethod
    def empty(p: Params, n: int, btot: int, dtype, device) -> "SavedTensors":
        return SavedTensors(
            torch.empty(p.hkv, max(btot, 1), p.d, dtype=dtype, device=device),
            torch.empty(p.hkv, max(btot, 1), p.d, dtype=dtype, device=device),
            torch.empty(p.hkv, n, p.d, dtype=dtype, device=device),
            torch.empty(p.hkv, n, p.d, dtype=dtype, device=device),
            torch.empty(3, n, p.hq, p.d, dtype=torch.float32, device=device),
            torch.empty(3, n, p.hq, dtype=torch.float32, device=device),
            torch.empty(n, p.hkv, p.topk, dtype=torch.int32, device=device))

    @staticmethod
    def empty_cross(p: Params, nq: int, nkv: int, btot: int, dtype, device) -> "SavedTensors":
        """Buffers of ssa_cross_forward: two branches, keys / values of the voxel tokens."""
        return SavedTensors(
            torch.empty(p.hkv, max(btot, 1), p.d, dtype=dtype, device=device),
            torch.empty(p.hkv, max(btot, 1), p.d, dtype=dtype, device=device),
            torch.empty(p.hkv, nkv, p.d, dtype=dtype, device=device),
            torch.empty(p.hkv, nkv, p.d, dtype=dtype, device=device),
            torch.empty(2, nq, p.hq, p.d, dtype=torch.float32, device=device),
            torch.empty(2, nq, p.hq, dtype=torch.float32, device=device),
            torch.empty(nq, p.hkv, p.topk, dtype=torch.int32, device=device))

    def c(self) -> Saved:
        return Saved(_ptr(self.kc), _ptr(self.vc), _ptr(self.ks), _ptr(self.vs), _ptr(self.o_branch),
                     _ptr(self.lse), _ptr(self.sel))


def workspace_size(op: int, p: Params, s: int, n: int, btot: int, wtot: int) -> int:
    return int(_lib().ssa_workspace_size(op, ctypes.byref(p), s, n, btot, wtot))


def ssa_forward(p: Params, cu_seqlens: torch.Tensor, blk: Bins, win: Bins, q: torch.Tensor,
                k: torch.Tensor, v: torch.Tensor, gates: torch.Tensor, out: torch.Tensor | None = None,
                saved: SavedTensors | None = None, workspace: torch.Tensor | None = None,
                sel: torch.Tensor | None = None):
    """Steps 2-6.  Returns (out [N, Hq, d], saved).  With p.selection == SEL_GIVEN,
    `sel` (int32 [N, Hkv, topk], e.g. from ssa_geo_select) becomes saved.sel and is
    read instead of the score top-k; entries outside the token's sequence are set
    to -1 on the device and reported by device_status()."""
    _require_cuda(cu_seqlens, q, k, v, gates)
    n = int(q.shape[0])
    s = int(cu_seqlens.shape[0]) - 1
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if saved is None:
        saved = SavedTensors.empty(p, n, blk.count, q.dtype, dev)
    if p.selection == SEL_GIVEN:
        if sel is not None:
            if sel.dtype != torch.int32 or not sel.is_contiguous() or tuple(sel.shape) != (n, p.hkv, p.topk):
                raise ValueError("sel must be a contiguous int32 tensor [N, Hkv, topk]")
            saved = dataclasses.replace(saved, sel=sel)
    elif sel is not None:
        raise ValueError("sel is only read with selection=SEL_GIVEN")
    need = workspace_size(OP_FORWARD, p, s, n, blk.count, win.count)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, pw, sv = blk.c(), win.c(), saved.c()
    st = _lib().ssa_forward(ctypes.byref(p), _ptr(cu_seqlens), s, n, ctypes.byref(pb), ctypes.byref(pw),
                            _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(out), ctypes.byref(sv), _ptr(ws),
                            ws.numel(), _stream(dev))
    _check(st, "ssa_forward")
    return out, saved


def ssa_backward(p: Params, cu_seqlens: torch.Tensor, blk: Bins, win: Bins, q, k, v, gates,
                 saved: SavedTensors, dout: torch.Tensor, grads=None, workspace: torch.Tensor | None = None):
    """Step 7.  Returns (dq, dk, dv, dgates), all fp32."""
    _require_cuda(cu_seqlens, q, k, v, gates, dout)
    n = int(q.shape[0])
    s = int(cu_seqlens.shape[0]) - 1
    dev = q.device
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = (torch.empty(q.shape, **f32), torch.empty(k.shape, **f32), torch.empty(v.shape, **f32),
                 torch.empty(gates.shape, **f32))
    dq, dk, dv, dg = grads
    need = workspace_size(OP_BACKWARD, p, s, n, blk.count, win.count)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, pw, sv = blk.c(), win.c(), saved.c()
    st = _lib().ssa_backward(ctypes.byref(p), _ptr(cu_seqlens), s, n, ctypes.byref(pb), ctypes.byref(pw),
                             _ptr(q), _ptr(k), _ptr(v), _ptr(gates), ctypes.byref(sv), _ptr(dout), _ptr(dq),
                             _ptr(dk), _ptr(dv), _ptr(dg), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ssa_backward")
    return dq, dk, dv, dg


@dataclass
class SpLocal:
    """One rank's tokens of a batch split by whole blocks (see ssa_sp_forward in
    include/ssa.h): their per-sequence offsets, their rows among all tokens, their own
    window partition and K / V, and room for their window-ordered K / V copies."""
    cu_seqlens: torch.Tensor  # int32 [S+1]
    tokens: torch.Tensor      # int32 [Nr]
    win: Bins                 # ssa_bin of the rank's coordinates (edge m_win)
    k: torch.Tensor           # [Nr, Hkv, d]
    v: torch.Tensor
    ks: torch.Tensor          # [Hkv, Nr, d]
    vs: torch.Tensor

    @staticmethod
    def make(cu_seqlens, tokens, win: Bins, k, v) -> "SpLocal":
        n, hkv, d = (int(x) for x in k.shape)
        e = lambda: torch.empty(hkv, n, d, dtype=k.dtype, device=k.device)  # noqa: E731
        return SpLocal(cu_seqlens, tokens, win, k, v, e(), e())

    def c(self):
        pw = self.win.c()
        return SpLocalC(int(self.k.shape[0]), _ptr(self.cu_seqlens), _ptr(self.tokens), ctypes.pointer(pw),
                        _ptr(self.k), _ptr(self.v), _ptr(self.ks), _ptr(self.vs)), pw


def ssa_sp_forward(p: Params, blk: Bins, n_all: int, loc: SpLocal, q: torch.Tensor, k: torch.Tensor,
                   v: torch.Tensor, gates: torch.Tensor, out: torch.Tensor | None = None,
                   saved: SavedTensors | None = None, workspace: torch.Tensor | None = None):
    """One rank's forward (sequences split by whole blocks): its query rows q / gates
    [Nr, Hq, *] against all N tokens' k / v binned into `blk`; returns (out, saved)."""
    _require_cuda(q, k, v, gates, loc.cu_seqlens, loc.tokens, loc.k, loc.v)
    nr, s = int(q.shape[0]), int(loc.cu_seqlens.shape[0]) - 1
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if saved is None:  # the cross-attention buffers, with room for the third (window) branch
        saved = dataclasses.replace(SavedTensors.empty_cross(p, nr, n_all, blk.count, q.dtype, dev),
                                    o_branch=torch.empty(3, nr, p.hq, p.d, dtype=torch.float32, device=dev),
                                    lse=torch.empty(3, nr, p.hq, dtype=torch.float32, device=dev))
    need = workspace_size(OP_SP_FORWARD, p, s, nr, blk.count, loc.win.count)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, sv = blk.c(), saved.c()
    lc, _keep = loc.c()
    st = _lib().ssa_sp_forward(ctypes.byref(p), s, int(n_all), ctypes.byref(pb), ctypes.byref(lc), _ptr(q), _ptr(k),
                               _ptr(v), _ptr(gates), _ptr(out), ctypes.byref(sv), _ptr(ws), ws.numel(),
                               _stream(dev))
    _check(st, "ssa_sp_forward")
    return out, saved


def ssa_sp_backward(p: Params, blk: Bins, n_all: int, loc: SpLocal, q, k, v, gates, saved: SavedTensors,
                    dout, grads=None, workspace: torch.Tensor | None = None):
    """One rank's backward: (dq [Nr, Hq, d], dk, dv [N, Hkv, d] = its rows' contributions to every
    token's key gradients, dgates [Nr, Hq, 3])."""
    _require_cuda(q, k, v, gates, dout)
    nr, s = int(q.shape[0]), int(loc.cu_seqlens.shape[0]) - 1
    dev = q.device
    if grads is None:
        grads = (torch.empty(q.shape, dtype=torch.float32, device=dev),
                 torch.empty(k.shape, dtype=torch.float32, device=dev),
                 torch.empty(v.shape, dtype=torch.float32, device=dev),
                 torch.empty(gates.shape, dtype=torch.float32, device=dev))
    dq, dk, dv, dg = grads
    need = workspace_size(OP_SP_BACKWARD, p, s, nr, blk.count, loc.win.count)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, sv = blk.c(), saved.c()
    lc, _keep = loc.c()
    st = _lib().ssa_sp_backward(ctypes.byref(p), s, int(n_all), ctypes.byref(pb), ctypes.byref(lc), _ptr(q), _ptr(k),
                                _ptr(v), _ptr(gates), ctypes.byref(sv), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(dg), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ssa_sp_backward")
    return dq, dk, dv, dg


def ssa_cross_forward(p: Params, q_cu: torch.Tensor, blk: Bins, q: torch.Tensor, k: torch.Tensor,
                      v: torch.Tensor, gates: torch.Tensor, out: torch.Tensor | None = None,
                      saved: SavedTensors | None = None, workspace: torch.Tensor | None = None,
                      sel: torch.Tensor | None = None):
    """Cross-attention SSA: queries q [Nq, Hq, d] (sequence s = rows q_cu[s] ..
    q_cu[s+1]-1) attend the voxel tokens k / v [Nkv, Hkv, d] binned into `blk`
    through the compressed and selected branches; gates [Nq, Hq, 2].
    Returns (out [Nq, Hq, d], saved)."""
    _require_cuda(q_cu, q, k, v, gates)
    nq, nkv = int(q.shape[0]), int(k.shape[0])
    s = int(q_cu.shape[0]) - 1
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if saved is None:
        saved = SavedTensors.empty_cross(p, nq, nkv, blk.count, q.dtype, dev)
    if p.selection == SEL_GIVEN:
        if sel is not None:
            if sel.dtype != torch.int32 or not sel.is_contiguous() or tuple(sel.shape) != (nq, p.hkv, p.topk):
                raise ValueError("sel must be a contiguous int32 tensor [Nq, Hkv, topk]")
            saved = dataclasses.replace(saved, sel=sel)
    elif sel is not None:
        raise ValueError("sel is only read with selection=SEL_GIVEN")
    need = workspace_size(OP_CROSS_FORWARD, p, s, nq, blk.count, 0)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, sv = blk.c(), saved.c()
    st = _lib().ssa_cross_forward(ctypes.byref(p), _ptr(q_cu), s, nq, nkv, ctypes.byref(pb), _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(gates), _ptr(out), ctypes.byref(sv), _ptr(ws), ws.numel(),
                                  _stream(dev))
    _check(st, "ssa_cross_forward")
    return out, saved


def ssa_cross_backward(p: Params, q_cu: torch.Tensor, blk: Bins, q, k, v, gates, saved: SavedTensors,
                       dout: torch.Tensor, grads=None, workspace: torch.Tensor | None = None):
    """Gradients of ssa_cross_forward: (dq, dk, dv, dgates), all fp32."""
    _require_cuda(q_cu, q, k, v, gates, dout)
    nq, nkv = int(q.shape[0]), int(k.shape[0])
    s = int(q_cu.shape[0]) - 1
    dev = q.device
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = (torch.empty(q.shape, **f32), torch.empty(k.shape, **f32), torch.empty(v.shape, **f32),
                 torch.empty(gates.shape, **f32))
    dq, dk, dv, dg = grads
    need = workspace_size(OP_CROSS_BACKWARD, p, s, nq, blk.count, 0)
    ws = workspace if workspace is not None and workspace.numel() >= need else _workspace(need, dev)
    pb, sv = blk.c(), saved.c()
    st = _lib().ssa_cross_backward(ctypes.byref(p), _ptr(q_cu), s, nq, nkv, ctypes.byref(pb), _ptr(q), _ptr(k),
                                   _ptr(v), _ptr(gates), ctypes.byref(sv), _ptr(dout), _ptr(dq), _ptr(dk),
                                   _ptr(dv), _ptr(dg), _ptr(ws), ws.numel(), _stream(dev))
    _check(st, "ssa_cross_backward")
    return dq, dk, dv, dg


def device_status(stream: int | None = None) -> int:
    return int(_lib().ssa_get_device_status(stream if stream is not None else _stream()))


def launch_count() -> int:
    """Kernels this library has launched in this process."""
    return int(_lib().ssa_launch_count())


def profile_enable(on: bool) -> None:
    _lib().ssa_profile_enable(1 if on else 0)


def profile_read(max_entries: int = 128) -> dict:
    """{kernel name: (total ms, launches)} recorded since the last read."""
    L = _lib()
    name_len = 64
    names = ctypes.create_string_buffer(name_len * max_entries)
    ms = (ctypes.c_float * max_entries)()
    cnt = (ctypes.c_int32 * max_entries)()
    n = min(L.ssa_profile_read(names, name_len, ms, cnt, max_entries), max_entries)
    out = {}
    for i in range(n):
        nm = names.raw[i * name_len:(i + 1) * name_len].split(b"\0", 1)[0].decode()
        out[nm] = (float(ms[i]), int(cnt[i]))
    return out


def diag_wait_timeout(device=None) -> tuple[int, int]:
    """Runs the bounded-wait diagnostic; returns (lane wait gave up, warp wait gave up)."""
    out = torch.zeros(2, dtype=torch.int32, device=device or "cuda")
    _check(_lib().ssa_diag_wait_timeout(_ptr(out), _stream(out.device)), "ssa_diag_wait_timeout")
    o = out.cpu().tolist()
    return int(o[0]), int(o[1])


def diag_ex2(x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """(2^x on the FMA pipe as the kernels evaluate it, 2^x from ex2.approx) for fp32 x."""
    _require_cuda(x)
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _check(_lib().ssa_diag_ex2(_ptr(x), _ptr(yp), _ptr(ym), x.numel(), _stream(x.device)), "ssa_diag_ex2")
    return yp, ym


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
