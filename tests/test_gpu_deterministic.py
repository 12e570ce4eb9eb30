"""ssa_params.deterministic = 1: the backward's key-gradient sums are 64-bit fixed-point
integer additions, so two runs give bitwise-equal gradients (the default fp32 atomics
may not), the values agree with the default mode and with the oracle, and shapes the
tensor-core backward does not cover are refused."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, DeviceRun, compare_backward, compare_forward, f64, max_abs, run_oracle

pytestmark = pytest.mark.gpu


def _det_run(w, t, det):
    run = DeviceRun(w, t)
    run.p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, torch.bfloat16, w.gate_mode,
                            deterministic=det)
    return run


def test_two_deterministic_backwards_are_bitwise_equal_at_benchmark_size():
    w = W.config(5)
    t = W.make_tensors(w)
    run = _det_run(w, t, True).run()
    first = [x.clone() for x in run.grads]
    again = ssa.ssa_backward(run.p, run.cu, run.blk, run.win, run.q, run.k, run.v, run.gates, run.saved, run.dout)
    torch.cuda.synchronize()
    assert ssa.device_status() == 0
    for a, b in zip(first, again):
        assert torch.equal(a, b)
    # the default mode computes the same sums in another order
    ref = _det_run(w, t, False).run()
    # the default mode's fp32 atomics round every partial sum of key gradients of magnitude up
    # to ~100 (2^-24 relative each, in a varying order); 1.5e-3 has been observed, a quarter of the
    # parity tolerance bounds it
    diffs = [max_abs(f64(a), f64(b)) for a, b in zip(first, ref.grads)]
    print("deterministic vs default, max |difference| of dq, dk, dv, dgates:", diffs)
    assert max(diffs) <= ATOL["bf16"] / 4


def test_deterministic_backward_matches_the_oracle():
    w = W.small_shell(seed=41, R=32, n_prims=2, lo=4.0, hi=9.0, n_keep=900, n_seqs=2, hq=16, hkv=2, d=64,
                      m_cmp=4, m_win=4, topk=8, dtype="bf16", gate_mode=1)
    t = W.make_tensors(w)
    run = _det_run(w, t, True).run()
    st = run_oracle(w, t)
    _, flips = compare_forward(run, st, np.arange(w.n), ATOL["bf16"])
    g = O.backward(st, t.as_f32("do").astype(np.float64))
    print(compare_backward(run, st, g, ATOL["bf16"], flips))


def test_deterministic_is_refused_where_the_tensor_core_backward_does_not_run():
    w = W.small_shell(seed=42, R=24, n_prims=1, lo=3.0, hi=6.0, n_keep=200, hq=4, hkv=2, d=32, m_cmp=4, m_win=4,
                      topk=4, dtype="f32", gate_mode=1)
    t = W.make_tensors(w)
    run = DeviceRun(w, t)
    p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, torch.float32, w.gate_mode, deterministic=True)
    blk, win = ssa.ssa_bin(run.coords, run.cu, w.R, w.m_cmp, w.m_win)
    with pytest.raises(ssa.SSAError) as e:
        ssa.ssa_forward(p, run.cu, blk, win, run.q, run.k, run.v, run.gates)
    assert e.value.status == 2  # SSA_ERR_UNSUPPORTED
