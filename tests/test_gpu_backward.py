"""Step 7 on the GPU against the oracle's analytic backward."""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, DeviceRun, compare_backward, compare_forward, f64, run_oracle

pytestmark = pytest.mark.gpu


def _bwd_parity(w, t):
    run = DeviceRun(w, t).run()
    st = run_oracle(w, t)
    _, flips = compare_forward(run, st, np.arange(w.n), ATOL[w.dtype])
    g = O.backward(st, t.as_f32("do").astype(np.float64))
    errs = compare_backward(run, st, g, ATOL[w.dtype], flips)
    return run, st, g, errs


@pytest.mark.parametrize("kw", [
    dict(hq=16, hkv=2, d=64, m_cmp=4, m_win=4, topk=8, dtype="bf16", gate_mode=1),
    dict(hq=8, hkv=2, d=32, m_cmp=3, m_win=6, topk=5, dtype="bf16", gate_mode=0),
    dict(hq=4, hkv=2, d=64, m_cmp=4, m_win=4, topk=6, dtype="f32", gate_mode=1),
    dict(hq=2, hkv=1, d=32, m_cmp=4, m_win=4, topk=4, dtype="f32", gate_mode=0),
    # head dim 128 (the fp32 CUDA-core kernels), bf16 and fp32
    dict(hq=16, hkv=2, d=128, m_cmp=4, m_win=4, topk=6, dtype="bf16", gate_mode=1),
    dict(hq=8, hkv=2, d=128, m_cmp=4, m_win=8, topk=4, dtype="f32", gate_mode=0),
])
def test_small_shell_backward_parity(kw):
    w = W.small_shell(seed=11, R=32, n_prims=2, lo=4.0, hi=9.0, n_keep=900, n_seqs=2, **kw)
    t = W.make_tensors(w)
    _, _, _, errs = _bwd_parity(w, t)
    print(w.n, errs)


@pytest.mark.parametrize("kw", [
    # 16 heads per KV head, windows and blocks of 16^3 voxels: windows of more than
    # 128 tokens span several key tiles of the tensor-core kernels
    dict(hq=32, hkv=2, d=64, m_cmp=16, m_win=16, topk=4, dtype="bf16", gate_mode=1),
    dict(hq=16, hkv=2, d=64, m_cmp=16, m_win=16, topk=4, dtype="bf16", gate_mode=1),
    dict(hq=32, hkv=2, d=64, m_cmp=4, m_win=4, topk=8, dtype="bf16", gate_mode=1),
])
def test_large_windows_and_16_head_groups(kw):
    w = W.small_shell(seed=21, R=40, n_prims=2, lo=6.0, hi=12.0, n_keep=None, **kw)
    t = W.make_tensors(w)
    sizes = np.bincount(O.bin_tokens(w.coords, w.cu_seqlens, w.m_win)["id"])
    if w.m_win == 16:
        assert sizes.max() > 128  # the case these shapes are for
    _, _, _, errs = _bwd_parity(w, t)
    print(w.n, sizes.max(), errs)


def test_zero_gates_give_zero_input_gradients():
    w = W.small_shell(seed=12, R=32, n_prims=2, lo=4.0, hi=9.0, n_keep=600, gate_mode=0)
    t = W.make_tensors(w)
    t.gates[:] = 0.0
    run = DeviceRun(w, t).run()
    dq, dk, dv, dg = run.grads
    assert not dq.abs().max().item() and not dk.abs().max().item() and not dv.abs().max().item()
    assert dg.abs().max().item() > 0


def test_gradient_sums():
    """Softmax rows sum to one: sum_i dV_i = sum_rows w_c dO; key gradients sum to 0.

    The sums run over ~10^4 rounded terms (the tensor-core kernels multiply bf16
    P and dS), so the tolerance grows with the magnitude of what is summed:
    2e-2 + 1e-3 x (sum of the absolute values of the terms)."""
    w = W.small_shell(seed=13, R=40, n_prims=2, lo=5.0, hi=11.0, n_keep=1500)
    t = W.make_tensors(w)
    run = DeviceRun(w, t).run()
    dq, dk, dv, dg = (f64(x) for x in run.grads)
    gw = O.gate_weights(t.gates, w.gate_mode)
    do = t.as_f32("do").astype(np.float64)
    G = w.hq // w.hkv
    for g in range(w.hkv):
        hs = slice(g * G, (g + 1) * G)
        want = np.einsum("nh,nhd->d", gw[:, hs, :].sum(-1), do[:, hs, :])
        mag_v = np.einsum("nh,nhd->d", gw[:, hs, :].sum(-1), np.abs(do[:, hs, :]))
        assert (np.abs(dv[:, g, :].sum(0) - want) <= 2e-2 + 1e-3 * mag_v).all()
        mag_k = np.abs(dk[:, g, :]).sum(0)
        assert (np.abs(dk[:, g, :].sum(0)) <= 2e-2 + 1e-3 * mag_k).all()
