"""Step 1 on the GPU: block / window binning, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import assert_bins_equal

pytestmark = pytest.mark.gpu


def _gpu_bin(coords, cu, R, m_cmp, m_win):
    c = torch.from_numpy(np.ascontiguousarray(coords, np.int32)).cuda()
    u = torch.from_numpy(np.asarray(cu, np.int32)).cuda()
    return ssa.ssa_bin(c, u, R, m_cmp, m_win)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_bins_bit_exact_on_configs(cfg):
    w = W.config(cfg)
    blk, win = _gpu_bin(w.coords, w.cu_seqlens, w.R, w.m_cmp, w.m_win)
    assert_bins_equal(blk, O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp), "blk")
    assert_bins_equal(win, O.bin_tokens(w.coords, w.cu_seqlens, w.m_win), "win")


def test_bins_edge_cases():
    rng = np.random.default_rng(0)
    R = 13  # m = 4 does not divide R
    lens = [0, 1, 37, 0, 5000, 3]  # empty first/middle sequences, a single token
    coords = rng.integers(0, R, size=(sum(lens), 3)).astype(np.int32)  # duplicates included
    coords[1] = (R - 1, R - 1, R - 1)
    cu = np.concatenate([[0], np.cumsum(lens)])
    for m_cmp, m_win in [(4, 4), (4, 2), (1, 13), (3, 64)]:
        blk, win = _gpu_bin(coords, cu, R, m_cmp, m_win)
        assert_bins_equal(blk, O.bin_tokens(coords, cu, m_cmp), "blk m=%d" % m_cmp)
        assert_bins_equal(win, O.bin_tokens(coords, cu, m_win), "win m=%d" % m_win)


def test_bins_wide_keys_and_many_sequences():
    rng = np.random.default_rng(1)
    R = 1 << 20
    lens = rng.integers(0, 300, size=9)
    coords = rng.integers(0, R, size=(int(lens.sum()), 3)).astype(np.int32)
    coords[: min(5, len(coords))] = R - 1
    cu = np.concatenate([[0], np.cumsum(lens)])
    blk, win = _gpu_bin(coords, cu, R, 1, 1 << 19)  # 4 + 3 * 20 = 64 key bits
    assert_bins_equal(blk, O.bin_tokens(coords, cu, 1), "blk")
    assert_bins_equal(win, O.bin_tokens(coords, cu, 1 << 19), "win")
    lens = rng.integers(1, 40, size=3000)  # many short sequences
    coords = rng.integers(0, 64, size=(int(lens.sum()), 3)).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(lens)])
    blk, win = _gpu_bin(coords, cu, 64, 8, 2)
    assert_bins_equal(blk, O.bin_tokens(coords, cu, 8), "blk")
    assert_bins_equal(win, O.bin_tokens(coords, cu, 2), "win")


def test_ids_do_not_depend_on_token_order():
    w = W.config(4)
    t = W.make_tensors(w, with_do=False)
    w2, _, src = W.permute_workload(w, t, seed=3)
    blk, _ = _gpu_bin(w.coords, w.cu_seqlens, w.R, w.m_cmp, w.m_win)
    blk2, _ = _gpu_bin(w2.coords, w2.cu_seqlens, w2.R, w2.m_cmp, w2.m_win)
    np.testing.assert_array_equal(blk2.id.cpu().numpy(), blk.id.cpu().numpy()[src])


def test_range_errors_are_reported_and_cleared():
    coords = np.array([[0, 0, 0], [5, 1, 64], [3, 3, 3]], np.int32)  # z = 64 is outside a 64^3 grid
    with pytest.raises(ssa.SSAError) as e:
        _gpu_bin(coords, [0, 3], 64, 4, 4)
    assert e.value.status == 4
    coords[1, 2] = -1
    with pytest.raises(ssa.SSAError):
        _gpu_bin(coords, [0, 3], 64, 4, 4)
    with pytest.raises(ssa.SSAError) as e:  # decreasing cu_seqlens
        _gpu_bin(np.zeros((3, 3), np.int32), [0, 2, 1, 3], 64, 4, 4)
    assert e.value.status == 4
    blk, _ = _gpu_bin(np.zeros((3, 3), np.int32), [0, 3], 64, 4, 4)  # the check word was cleared
    assert blk.count == 1
    assert ssa.device_status() == 0
