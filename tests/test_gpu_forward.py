"""Steps 2-6 on the GPU against the oracle, on inputs the oracle finishes in
seconds: several tiles per sequence, ragged tails, varlen batches, edge cases."""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, DeviceRun, compare_forward, f64, run_oracle

pytestmark = pytest.mark.gpu


def _parity(w, t, tokens=None):
    run = DeviceRun(w, t, backward=False).run(backward=False)
    st = run_oracle(w, t)
    toks = np.arange(w.n) if tokens is None else tokens
    errs, flips = compare_forward(run, st, toks, ATOL[w.dtype])
    return run, st, errs, flips


def test_config1_fp32_full_parity():
    w = W.config(1)
    t = W.make_tensors(w, with_do=False)
    _, _, errs, flips = _parity(w, t)
    assert flips == []  # fp32 config: selection bit-exact
    print(errs)


@pytest.mark.parametrize("kw", [
    dict(hq=16, hkv=2, d=64, m_cmp=4, m_win=4, topk=8, dtype="bf16", gate_mode=1),
    dict(hq=16, hkv=2, d=64, m_cmp=4, m_win=8, topk=16, dtype="bf16", gate_mode=1),
    dict(hq=8, hkv=2, d=32, m_cmp=3, m_win=2, topk=5, dtype="bf16", gate_mode=0),
    dict(hq=16, hkv=1, d=64, m_cmp=4, m_win=4, topk=4, dtype="f32", gate_mode=1),
    dict(hq=2, hkv=2, d=64, m_cmp=8, m_win=4, topk=32, dtype="bf16", gate_mode=1),
    # head dim 128 (the fp32 CUDA-core kernels), bf16 and fp32
    dict(hq=16, hkv=2, d=128, m_cmp=4, m_win=4, topk=8, dtype="bf16", gate_mode=1),
    dict(hq=4, hkv=1, d=128, m_cmp=4, m_win=8, topk=4, dtype="f32", gate_mode=0),
])
def test_small_shell_parity(kw):
    w = W.small_shell(seed=3, R=40, n_prims=2, lo=5.0, hi=11.0, n_keep=1500, n_seqs=2, **kw)
    t = W.make_tensors(w, with_do=False)
    _, _, errs, flips = _parity(w, t)
    print(w.n, errs, len(flips))


def test_varlen_with_empty_and_single_token_sequences():
    w = W.small_shell(seed=5, R=32, n_prims=2, lo=4.0, hi=9.0, n_keep=900, n_seqs=3)
    # insert an empty sequence at the front and the middle, and a single-token sequence
    lens = np.diff(w.cu_seqlens).tolist()
    coords = [w.coords[:0]]
    new_lens = [0]
    off = 0
    for i, L in enumerate(lens):
        coords.append(w.coords[off:off + L])
        new_lens.append(L)
        off += L
        if i == 0:
            new_lens.append(0)
            coords.append(w.coords[:0])
    coords.append(np.array([[7, 7, 7]], np.int32))
    new_lens.append(1)
    w.coords = np.concatenate(coords).astype(np.int32)
    w.cu_seqlens = np.concatenate([[0], np.cumsum(new_lens)]).astype(np.int32)
    t = W.make_tensors(w, with_do=False)
    run, st, errs, flips = _parity(w, t)
    # the single-token sequence: every branch is that token's own value row
    last = w.n - 1
    G = w.hq // w.hkv
    v_last = np.repeat(t.as_f32("v")[last], G, axis=0)
    for c in range(3):
        np.testing.assert_allclose(f64(run.saved.o_branch[c, last]), v_last, atol=1e-2)


def test_batch_equals_separate_calls():
    w = W.small_shell(seed=7, R=32, n_prims=2, lo=4.0, hi=9.0, n_keep=800, n_seqs=3)
    t = W.make_tensors(w, with_do=False)
    run = DeviceRun(w, t, backward=False).run(backward=False)
    for s in range(w.s):
        a, b = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
        ws = W.Workload("part", w.R, w.coords[a:b], np.array([0, b - a], np.int32), w.hq, w.hkv, w.d, w.m_cmp,
                        w.m_win, w.topk, w.dtype, w.gate_mode, w.seed)
        ts = W.Tensors(t.q[a:b], t.k[a:b], t.v[a:b], t.gates[a:b], None, t.dtype)
        r2 = DeviceRun(ws, ts, backward=False).run(backward=False)
        np.testing.assert_array_equal(f64(r2.out), f64(run.out[a:b]))
        off = run.blk.cu[s].item()
        sel = run.saved.sel[a:b].cpu().numpy()
        np.testing.assert_array_equal(r2.saved.sel.cpu().numpy(), np.where(sel >= 0, sel - off, -1))


def test_token_permutation_equivariance():
    w = W.small_shell(seed=8, R=40, n_prims=2, lo=5.0, hi=11.0, n_keep=1200)
    t = W.make_tensors(w, with_do=False)
    run = DeviceRun(w, t, backward=False).run(backward=False)
    w2, t2, src = W.permute_workload(w, t, seed=1)
    run2 = DeviceRun(w2, t2, backward=False).run(backward=False)
    np.testing.assert_array_equal(run2.blk.id.cpu().numpy(), run.blk.id.cpu().numpy()[src])
    np.testing.assert_array_equal(run2.saved.sel.cpu().numpy(), run.saved.sel.cpu().numpy()[src])
    np.testing.assert_allclose(f64(run2.out), f64(run.out)[src], atol=1e-2)


def test_one_hot_gates_isolate_each_branch():
    w = W.small_shell(seed=9, R=32, n_prims=2, lo=4.0, hi=9.0, n_keep=700, gate_mode=0)
    t = W.make_tensors(w, with_do=False)
    for c in range(3):
        t.gates[:] = 0.0
        t.gates[:, :, c] = 1.0
        run = DeviceRun(w, t, backward=False).run(backward=False)
        assert torch.equal(run.out, run.saved.o_branch[c].to(run.out.dtype))
    t.gates[:] = 0.0
    run = DeviceRun(w, t, backward=False).run(backward=False)
    assert not run.out.float().abs().max().item()
