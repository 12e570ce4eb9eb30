"""One batch split across ranks by whole blocks (LSRM, "块感知序列并行与负载均衡"), on one
GPU: each rank's share runs as its own ssa_sp_forward / ssa_sp_backward call (R = 2
and R = 4 ranks, one after the other), its rows of out / dQ / dgates are placed back
and the ranks' partial key gradients summed, as the exchange between ranks would do.
Every row and gradient is compared with the oracle of the whole batch, and with the
single-call GPU path."""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import shard, ssa
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, DeviceRun, check_selection, f64, max_abs, run_oracle, to_torch

pytestmark = pytest.mark.gpu


def _run_ranks(w, t, world):
    run = DeviceRun(w, t).run()  # the single call, for comparison; its binning serves every rank
    dev = "cuda"
    blk_perm, blk_ptr = run.blk.perm.cpu().numpy(), run.blk.ptr[:run.blk.count + 1].cpu().numpy()
    blk_cu = run.blk.cu.cpu().numpy()
    n = w.n
    out = torch.zeros_like(run.q)
    dq = torch.zeros(run.q.shape, dtype=torch.float32, device=dev)
    dg = torch.zeros(run.gates.shape, dtype=torch.float32, device=dev)
    dk = torch.zeros(run.k.shape, dtype=torch.float32, device=dev)
    dv = torch.zeros_like(dk)
    sel = torch.zeros_like(run.saved.sel)
    owned = np.zeros(n, np.int64)
    for r in range(world):
        plan = shard.sp_local_plan(blk_perm, blk_ptr, blk_cu, w.cu_seqlens, world, r)
        nr = len(plan.tokens)
        owned[plan.tokens] += 1
        if nr == 0:
            continue
        tok = torch.from_numpy(plan.tokens).to(dev)
        cu_r = torch.from_numpy(plan.cu_seqlens).to(dev)
        _, win_r = ssa.ssa_bin(run.coords[tok].contiguous(), cu_r, w.R, w.m_cmp, w.m_win)
        loc = ssa.SpLocal.make(cu_r, tok.to(torch.int32), win_r, run.k[tok].contiguous(), run.v[tok].contiguous())
        q_r, g_r, do_r = run.q[tok].contiguous(), run.gates[tok].contiguous(), run.dout[tok].contiguous()
        o_r, saved = ssa.ssa_sp_forward(run.p, run.blk, n, loc, q_r, run.k, run.v, g_r)
        dq_r, dk_r, dv_r, dg_r = ssa.ssa_sp_backward(run.p, run.blk, n, loc, q_r, run.k, run.v, g_r, saved, do_r)
        out[tok], dq[tok], dg[tok], sel[tok] = o_r, dq_r, dg_r, saved.sel
        dk += dk_r  # the reduction of the partial key gradients to their owners
        dv += dv_r
    torch.cuda.synchronize()
    assert ssa.device_status() == 0
    assert (owned == 1).all()  # the ranks' tokens partition the batch
    return run, out, (dq, dk, dv, dg), sel


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", ["bf16", "f32"])
def test_ranks_reproduce_the_whole_batch(world, case):
    if case == "bf16":
        w = W.small_shell(seed=31, R=48, n_prims=3, lo=4.0, hi=11.0, n_keep=2500, n_seqs=2, hq=16, hkv=2, d=64,
                          m_cmp=8, m_win=8, topk=8, dtype="bf16", gate_mode=1)
    else:  # fp32, d = 32 (SIMT kernels), windows smaller than blocks
        w = W.small_shell(seed=32, R=40, n_prims=2, lo=4.0, hi=9.0, n_keep=900, n_seqs=2, hq=4, hkv=2, d=32,
                          m_cmp=8, m_win=4, topk=4, dtype="f32", gate_mode=1)
    t = W.make_tensors(w)
    run, out, grads, sel = _run_ranks(w, t, world)
    st = run_oracle(w, t)
    g = O.backward(st, t.as_f32("do").astype(np.float64))
    tol = ATOL[w.dtype]
    flips = check_selection(sel.cpu().numpy(), st, np.arange(w.n), tau=1e-6)
    assert not flips, flips[:5]
    errs = {"out": max_abs(f64(out), st["out"])}
    for name, a, b in zip(("dq", "dk", "dv", "dgates"), grads, (g["dq"], g["dk"], g["dv"], g["dgates"])):
        errs[name] = max_abs(f64(a), b)
    # against the single-call GPU path: the same arithmetic up to the order of sums
    errs["vs_single_call_out"] = max_abs(f64(out), f64(run.out))
    errs["vs_single_call_dk"] = max_abs(f64(grads[1]), f64(run.grads[1]))
    print(case, world, errs)
    for key, e in errs.items():
        assert e <= tol, (key, e, tol)


def test_a_rank_without_tokens_and_bad_windows_are_handled():
    w = W.small_shell(seed=33, R=24, n_prims=1, lo=3.0, hi=5.0, n_keep=120, hq=16, hkv=2, d=64, m_cmp=8, m_win=8,
                      topk=4, dtype="bf16", gate_mode=1)
    t = W.make_tensors(w)
    run = DeviceRun(w, t).run()
    empty_i = torch.zeros(0, dtype=torch.int32, device="cuda")
    cu0 = torch.zeros(2, dtype=torch.int32, device="cuda")
    _, win0 = ssa.ssa_bin(run.coords[:0].contiguous(), cu0, w.R, w.m_cmp, w.m_win)
    kz = run.k[:0].contiguous()
    loc = ssa.SpLocal.make(cu0, empty_i, win0, kz, kz)
    q0 = run.q[:0].contiguous()
    g0 = run.gates[:0].contiguous()
    saved = ssa.SavedTensors.empty_cross(run.p, 0, w.n, run.blk.count, run.q.dtype, "cuda")
    dq, dk, dv, dg = ssa.ssa_sp_backward(run.p, run.blk, w.n, loc, q0, run.k, run.v, g0, saved, q0)
    torch.cuda.synchronize()
    assert not dk.any() and not dv.any()  # no query rows: nothing flows to any key
    p_bad = ssa.make_params(w.hq, w.hkv, w.d, 8, 3, w.topk, torch.bfloat16, w.gate_mode)  # 8 % 3 != 0
    with pytest.raises(ssa.SSAError):
        ssa.ssa_sp_forward(p_bad, run.blk, w.n, loc, q0, run.k, run.v, g0)
