"""Step 2 on the GPU through ssa_pool: the block-sorted K_s / V_s copies and the
block means Kc / Vc, bit-exact against the oracle's mean pooling.

Shapes: small shells in bf16 and fp32 with 1, 2 and 4 KV heads and d = 32, 64;
then the 16 * 2^20-token case (128 sequences, each a copy of the 1024^3
benchmark shell) that the bench times for the HBM roofline, checked on sampled
blocks.
"""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _bin(coords, cu, R, m):
    c = torch.from_numpy(np.ascontiguousarray(coords, np.int32)).cuda()
    u = torch.from_numpy(np.asarray(cu, np.int32)).cuda()
    blk, _ = ssa.ssa_bin(c, u, R, m, m)
    return blk


def _check_blocks(blk_ref, k, ks, kc, blocks, rounding):
    """K_s rows of `blocks` equal K[perm]; Kc of `blocks` equals the oracle's mean."""
    perm, ptr = blk_ref["perm"], blk_ref["ptr"]
    k64 = k.astype(np.float64)
    for b in blocks:
        rows = perm[ptr[b]:ptr[b + 1]]
        for g in range(k.shape[1]):
            np.testing.assert_array_equal(ks[g, ptr[b]:ptr[b + 1]], k[rows, g], err_msg="K_s block %d" % b)
        sub = {"id": np.zeros(len(rows), np.int64), "ptr": np.array([0, len(rows)]), "count": 1}
        want = O.mean_pool(k64[rows], sub, rounding)[0]
        np.testing.assert_array_equal(kc[:, b].astype(np.float64), want, err_msg="Kc block %d" % b)


@pytest.mark.parametrize("dtype,hkv,d", [("bf16", 2, 64), ("bf16", 1, 32), ("bf16", 4, 64), ("f32", 1, 32),
                                         ("f32", 2, 64)])
def test_pool_bit_exact_small(dtype, hkv, d):
    w = W.small_shell(seed=3, R=48, n_prims=3, lo=4.0, hi=11.0, n_keep=3000, hq=hkv * 2, hkv=hkv, d=d, m_cmp=4,
                      m_win=4, topk=4, dtype=dtype, gate_mode=1)
    t = W.make_tensors(w)
    blk = _bin(w.coords, w.cu_seqlens, w.R, w.m_cmp)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32

    def dev(x):
        if dtype == "bf16":
            return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()

    k, v = dev(t.k), dev(t.v)
    ks, vs, kc, vc = ssa.ssa_pool(blk, k, v)
    torch.cuda.synchronize()
    ref = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)
    rounding = "bf16" if dtype == "bf16" else "f32"
    kf, vf = t.as_f32("k"), t.as_f32("v")
    for x, xs, xc in ((kf, ks, kc), (vf, vs, vc)):
        xs_ = xs.float().cpu().numpy()
        xc_ = xc[:, :blk.count].float().cpu().numpy()
        _check_blocks(ref, x, xs_, xc_, range(blk.count), rounding)
    assert kc.dtype == tdt


def test_pool_scaled_16m_tokens_sampled_blocks():
    base = W.config(5)
    copies = 128
    n1 = base.n
    coords = np.tile(base.coords, (copies, 1))
    cu = np.arange(copies + 1, dtype=np.int64) * n1
    blk = _bin(coords, cu, base.R, base.m_cmp)
    n = copies * n1
    gen = torch.Generator(device="cuda").manual_seed(0)
    k = torch.randn((n, 2, 64), device="cuda", generator=gen).to(torch.bfloat16)
    v = torch.randn((n, 2, 64), device="cuda", generator=gen).to(torch.bfloat16)
    ks, vs, kc, vc = ssa.ssa_pool(blk, k, v)
    torch.cuda.synchronize()
    assert ssa.device_status() == 0
    one = O.bin_tokens(base.coords, np.array([0, n1]), base.m_cmp)
    assert blk.count == copies * one["count"]
    rng = np.random.default_rng(1)
    picks = [(int(c), int(b)) for c, b in zip(rng.integers(0, copies, 24), rng.integers(0, one["count"], 24))]
    sizes = np.diff(one["ptr"])
    picks.append((copies - 1, int(np.argmax(sizes))))  # the largest block of the last sequence
    for c, b in picks:
        gb = c * one["count"] + b
        p0, p1 = int(one["ptr"][b]) + c * n1, int(one["ptr"][b + 1]) + c * n1
        rows = one["perm"][one["ptr"][b]:one["ptr"][b + 1]] + c * n1
        rows_t = torch.from_numpy(rows.astype(np.int64)).cuda()
        for x, xs, xc in ((k, ks, kc), (v, vs, vc)):
            xr = x[rows_t].float().cpu().numpy()  # [n_b, 2, 64]
            np.testing.assert_array_equal(xs[:, p0:p1].float().cpu().numpy(), xr.transpose(1, 0, 2))
            sub = {"id": np.zeros(len(rows), np.int64), "ptr": np.array([0, len(rows)]), "count": 1}
            want = O.mean_pool(xr.astype(np.float64), sub, "bf16")[0]
            np.testing.assert_array_equal(xc[:, gb].float().cpu().numpy().astype(np.float64), want)
