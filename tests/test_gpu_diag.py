"""Device building blocks through the C ABI: the bounded mbarrier wait gives up,
reports SSA_ERR_TIMEOUT and leaves the context usable; the FMA-pipe exponential
of the tensor-core kernels against fp64 exp2."""
import numpy as np
import pytest
import torch

from spatial_sparse_attention_ssa_b200 import ssa
from tests.ssa_testlib import DeviceRun
from spatial_sparse_attention_ssa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_a_wait_that_nobody_ends_times_out_and_is_reported():
    assert ssa.device_status() == 0
    lane, warp = ssa.diag_wait_timeout()
    assert (lane, warp) == (1, 1)
    assert ssa.STATUS_NAMES[ssa.device_status()] == "SSA_ERR_TIMEOUT"
    assert ssa.device_status() == 0  # read and cleared
    # the context still runs the attention path
    w = W.small_shell(seed=2, R=24, n_prims=2, lo=3.0, hi=7.0, n_keep=300, hq=16, hkv=2, d=64, m_cmp=4, m_win=4,
                      topk=4, dtype="bf16", gate_mode=1)
    DeviceRun(w, W.make_tensors(w)).run()


def test_fma_pipe_exp2_against_fp64():
    """2^x on the FMA pipe (ex2_poly2): relative error at most 2.5 fp32 ulps (3e-7) where the
    result is a normal float (x >= -126), below 2^-125 in absolute value for -127 <= x < -126,
    and the clamp makes every x < -127 give at most 2^-126.  The hardware ex2.approx is
    reported beside it."""
    rng = np.random.default_rng(0)
    xs = np.concatenate([np.linspace(-127.0, 0.0, 2_000_001), rng.uniform(-127.0, 0.0, 1_000_000),
                         -np.arange(0, 128, dtype=np.float64), [-0.5, -1e-7, -126.5, -200.0, -1e30]])
    x = torch.from_numpy(xs.astype(np.float32)).cuda()
    yp, ym = (y.cpu().numpy().astype(np.float64) for y in ssa.diag_ex2(x))
    x32 = xs.astype(np.float32).astype(np.float64)
    ref = np.exp2(x32)
    norm = x32 >= -126.0
    rel_p = np.abs(yp[norm] - ref[norm]) / ref[norm]
    rel_m = np.abs(ym[norm] - ref[norm]) / ref[norm]
    print("max relative error: poly %.3g (%.2f ulp), ex2.approx %.3g" % (rel_p.max(), rel_p.max() / 2 ** -23,
                                                                          rel_m.max()))
    assert rel_p.max() <= 3e-7
    low = (x32 < -126.0) & (x32 >= -127.0)
    assert (np.abs(yp[low]) <= 2.0 ** -125).all() and (yp[low] >= 0).all()
    assert (np.abs(yp[x32 < -127.0]) <= 2.0 ** -126).all()
