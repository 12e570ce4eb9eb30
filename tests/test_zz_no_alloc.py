"""ssa_bin_noalloc against ssa_bin, through the C ABI.

ssa_bin_noalloc exists for callers that cannot allocate device memory when
they bin tokens (a plugin inside an application that owns every byte of GPU
memory, a latency-critical loop that must not let cudaMalloc synchronise the
device, a process that reserved its memory up front).  It keeps its scratch
in a fixed device array inside the library instead of a caller workspace.

These checks call it twice in a row on different inputs -- so the second call
starts from the first call's leftover scratch -- and require the same ids,
permutations, CSR pointers, per-sequence offsets and cell keys as ssa_bin
(integer work: bit-exact).  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W

pytestmark = pytest.mark.gpu

MAX_TOKENS = 262144  # SSA_BIN_NOALLOC_MAX_TOKENS in include/ssa.h


def _raw_noalloc(coords, cu, R, m_cmp, m_win):
    """Direct ctypes call of the C entry point with preallocated outputs."""
    n, s = int(coords.shape[0]), int(cu.shape[0]) - 1
    blk, win = ssa.Bins.empty(n, s, coords.device), ssa.Bins.empty(n, s, coords.device)
    fn = ssa.lib().ssa_bin_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                   ctypes.c_int32, ctypes.c_int32, ctypes.POINTER(ssa.Partition),
                   ctypes.POINTER(ssa.Partition), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    pb, pw = blk.c(), win.c()
    status = fn(coords.data_ptr(), cu.data_ptr(), s, n, R, m_cmp, m_win, ctypes.byref(pb), ctypes.byref(pw),
                torch.cuda.current_stream().cuda_stream)
    blk.count, win.count = int(pb.count), int(pw.count)
    return status, blk, win


def _same(a: ssa.Bins, b: ssa.Bins):
    assert a.count == b.count
    c = a.count
    for x, y in ((a.id, b.id), (a.perm, b.perm), (a.ptr[:c + 1], b.ptr[:c + 1]), (a.cu, b.cu),
                 (a.key[:c], b.key[:c])):
        assert torch.equal(x, y)


def _inputs(w):
    return (torch.from_numpy(np.ascontiguousarray(w.coords, np.int32)).cuda(),
            torch.from_numpy(w.cu_seqlens.astype(np.int32)).cuda())


def test_noalloc_binning_matches_workspace_binning_twice_in_a_row():
    cases = [W.config(3), W.config(4)]  # 131072 tokens, then a 4-sequence varlen batch
    cases[1].coords = cases[1].coords[:200000]
    cases[1].cu_seqlens = np.minimum(cases[1].cu_seqlens, 200000).astype(np.int32)
    for w, (m_cmp, m_win) in zip(cases, [(8, 8), (8, 4)]):
        coords, cu = _inputs(w)
        want_blk, want_win = ssa.ssa_bin(coords, cu, w.R, m_cmp, m_win)
        status, blk, win = _raw_noalloc(coords, cu, w.R, m_cmp, m_win)
        torch.cuda.synchronize()
        assert status == 0, ssa.lib().ssa_error_string(status)
        _same(blk, want_blk)
        _same(win, want_win)


def test_noalloc_refuses_inputs_above_its_fixed_scratch():
    n = MAX_TOKENS + 1
    coords = torch.zeros(n, 3, dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, n], dtype=torch.int32, device="cuda")
    status, _, _ = _raw_noalloc(coords, cu, 64, 4, 4)
    assert status == 3  # SSA_ERR_WORKSPACE: nothing was enqueued
    status, blk, _ = _raw_noalloc(coords[:MAX_TOKENS].contiguous(),
                                  torch.tensor([0, MAX_TOKENS], dtype=torch.int32, device="cuda"), 64, 4, 4)
    assert status == 0 and blk.count == 1


def test_noalloc_matches_the_oracle_and_recovers_after_a_failed_call():
    """Against the oracle's binning directly; a call with a coordinate outside
    [0, R) reports SSA_ERR_COORD_RANGE, and the next valid call still returns
    SSA_OK with the right partition (the check word left in the shared scratch by
    the failed call is cleared); N = 0 returns zero counts and all-zero offsets."""
    from oracle import ssa_oracle as O
    from tests.ssa_testlib import assert_bins_equal

    w = W.small_shell(seed=12, R=40, n_prims=3, lo=4.0, hi=10.0, n_seqs=3)
    coords, cu = _inputs(w)
    bad = coords.clone()
    bad[5, 1] = w.R  # one coordinate out of range
    status, _, _ = _raw_noalloc(bad, cu, w.R, 4, 2)
    torch.cuda.synchronize()
    assert status == 4  # SSA_ERR_COORD_RANGE
    status, blk, win = _raw_noalloc(coords, cu, w.R, 4, 2)
    torch.cuda.synchronize()
    assert status == 0, ssa.lib().ssa_error_string(status)
    assert_bins_equal(blk, O.bin_tokens(w.coords, w.cu_seqlens, 4), "blk")
    assert_bins_equal(win, O.bin_tokens(w.coords, w.cu_seqlens, 2), "win")
    empty = torch.zeros(0, 3, dtype=torch.int32, device="cuda")
    cu0 = torch.zeros(4, dtype=torch.int32, device="cuda")
    status, blk0, win0 = _raw_noalloc(empty, cu0, 16, 4, 4)
    torch.cuda.synchronize()
    assert status == 0 and blk0.count == 0 and win0.count == 0
    assert not blk0.cu.any() and not win0.cu.any()
