"""Learned compression on the GPU against the oracle: a submanifold sparse 3x3x3
convolution of K and V before the block mean (Direct3D-S2, "方法").

The GPU evaluates the convolution in fp32 in another order than the oracle (block
sums of the neighbours first, then one product with the weights), so the stored
Kc / Vc may differ from the oracle's by one unit in the last place of the storage
type; everything downstream is compared with the usual tolerances (absolute, the weight
and bias gradients included); where the GPU picked a certified selection near-tie the
oracle is run again with the GPU's selection given, so no row is left out.  fp32 inputs (SIMT attention kernels) and
bf16 inputs (tensor-core kernels); weight and bias gradients included; the table and
the scanning lookups of neighbours, repeated voxels included.
"""
import numpy as np
import pytest
import torch

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import ssa
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests.ssa_testlib import ATOL, f64, max_abs, pool_rounding, to_torch, check_selection

pytestmark = pytest.mark.gpu


def _weights(seed, hkv, d, std):
    rng = np.random.default_rng(seed)
    return {"wk": (std * rng.standard_normal((hkv, 27, d, d))).astype(np.float32),
            "bk": (0.1 * rng.standard_normal((hkv, d))).astype(np.float32),
            "wv": (std * rng.standard_normal((hkv, 27, d, d))).astype(np.float32),
            "bv": (0.1 * rng.standard_normal((hkv, d))).astype(np.float32)}


@pytest.mark.parametrize("hq,d,dtype,m,dup", [(4, 32, "f32", 4, False), (16, 64, "bf16", 4, False),
                                               (4, 32, "f32", 4, True), (4, 32, "f32", 12, False)])
def test_learned_compression_forward_backward(hq, d, dtype, m, dup):
    """m = 4: the per-block voxel table answers the probes; dup: some voxels hold two
    tokens (the table marks them and the probes scan); m = 12: no table, every probe
    scans the neighbouring block."""
    w = W.small_shell(seed=53, R=40, n_prims=2, lo=4.0, hi=9.0, n_keep=700, n_seqs=2, hq=hq, hkv=2, d=d,
                      m_cmp=m, m_win=4, topk=8, dtype=dtype)
    if dup:  # token i + 1 takes the voxel of token i, for every 7th i of each sequence
        coords = w.coords.copy()
        for s in range(w.s):
            a, e = int(w.cu_seqlens[s]), int(w.cu_seqlens[s + 1])
            for i in range(a, e - 1, 7):
                coords[i + 1] = coords[i]
        w = W.Workload(**{**w.__dict__, "coords": coords})
    t = W.make_tensors(w)
    cw = _weights(5, w.hkv, w.d, 0.3 / np.sqrt(9 * w.d))
    dev = "cuda"
    coords = torch.from_numpy(np.ascontiguousarray(w.coords, np.int32)).to(dev)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
    conv = ssa.ConvWeights(coords, *(torch.from_numpy(cw[x]).to(dev) for x in ("wk", "bk", "wv", "bv")))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, tdt, w.gate_mode, conv=conv)
    q, k, v, do = (to_torch(x, dtype) for x in (t.q, t.k, t.v, t.do))
    gates = torch.from_numpy(t.gates).to(dev)
    blk, win = ssa.ssa_bin(coords, cu, w.R, w.m_cmp, w.m_win)
    out, saved = ssa.ssa_forward(p, cu, blk, win, q, k, v, gates)
    dq, dk, dv, dg = ssa.ssa_backward(p, cu, blk, win, q, k, v, gates, saved, do)
    torch.cuda.synchronize()
    assert ssa.device_status() == 0

    st = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), t.gates, hq=w.hq,
                   hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=w.gate_mode,
                   pool_rounding=pool_rounding(w), conv={x: cw[x].astype(np.float64) for x in cw})
    g = O.backward(st, t.as_f32("do").astype(np.float64))

    # Kc / Vc: within one unit in the last place of bf16 storage (2^(e - 7) for a value
    # in [2^e, 2^(e+1))), plus the fp32 rounding of a 27 x d-term sum (values are O(1))
    b = blk.count
    for name, ref in (("kc", st["kc"]), ("vc", st["vc"])):
        got = f64(getattr(saved, name)[:, :b]).transpose(1, 0, 2)
        big = np.maximum(np.abs(got), np.abs(ref))
        ulp = np.exp2(np.floor(np.log2(np.maximum(big, 1e-30))) - 7) if dtype == "bf16" else 0.0
        assert (np.abs(got - ref) <= ulp + 1e-5).all(), (name, np.abs(got - ref).max())
        if dtype == "bf16":
            print(name, "elements one ulp apart:", int((got != ref).sum()), "of", got.size)

    atol = ATOL[dtype]
    toks = np.arange(w.n)
    # bf16: the GPU's Kc may be one ulp (<= 2^-7 relative) off the oracle's (another fp32
    # summation order of the convolution), which moves a score by about |q| * ulp / sqrt(d) and
    # a group's summed probability by well under 1e-3: a near-tie within that is certified
    sel_gpu = saved.sel.cpu().numpy()
    flips = check_selection(sel_gpu, st, toks, tau=1e-6 if dtype == "f32" else 1e-3)
    if flips:
        # the reference for every output and gradient is then the oracle given the GPU's
        # (certified) selection, so nothing is left out of the comparison
        st = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), t.gates, hq=w.hq,
                       hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=w.gate_mode,
                       pool_rounding=pool_rounding(w), conv={x: cw[x].astype(np.float64) for x in cw},
                       sel_given=sel_gpu.astype(np.int64))
        g = O.backward(st, t.as_f32("do").astype(np.float64))
    ob = f64(saved.o_branch)
    errs = {"o_cmp": max_abs(ob[0], st["o"][0]), "o_slc": max_abs(ob[1], st["o"][1]),
            "o_win": max_abs(ob[2], st["o"][2]), "out": max_abs(f64(out), st["out"]),
            "dq": max_abs(f64(dq), g["dq"]), "dk": max_abs(f64(dk), g["dk"]), "dv": max_abs(f64(dv), g["dv"]),
            "dgates": max_abs(f64(dg), g["dgates"])}
    for name in ("dwk", "dbk", "dwv", "dbv"):
        errs[name] = max_abs(f64(getattr(conv, name)), g[name])
    print(dtype, errs, "flips", len(flips), "max |dW|, |db|", float(np.abs(g["dwk"]).max()),
          float(np.abs(g["dbk"]).max()))
    for key, e in errs.items():
        assert e <= atol, (key, e, atol)
