"""The full-size compressed-branch driver (tests/cmp_full.py) on a small case, on the
CPU: given the oracle's own full forward / backward as the "device" results, every
error is zero, no row flips, and the summed dKc / dVc equal the full backward's."""
import numpy as np

from oracle import ssa_oracle as O
from spatial_sparse_attention_ssa_b200 import workloads as W
from tests import cmp_full


def test_driver_reproduces_the_oracle_on_a_small_case():
    w = W.small_shell(seed=8, R=24, n_prims=2, lo=3.0, hi=7.0, hq=4, hkv=2, d=16, m_cmp=4, m_win=4, topk=4,
                      dtype="bf16", gate_mode=0, n_seqs=3)
    t = W.make_tensors(w)
    gates = np.zeros_like(t.gates)
    gates[:, :, 0] = 1.0
    st = O.forward(w.coords, w.cu_seqlens, t.as_f32("q"), t.as_f32("k"), t.as_f32("v"), gates, hq=w.hq,
                   hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=0)
    g = O.backward(st, t.as_f32("do"))
    out_bits = W.f32_to_bf16_bits(st["o"][0].astype(np.float32))
    arrays = {"q": t.q, "do": t.do, "gates": gates, "kc": st["kc"], "vc": st["vc"], "sel_gpu": st["sel"],
              "o_cmp_gpu": st["o"][0], "lse_gpu": st["lse"][0], "dq_gpu": g["dq"], "dgates_gpu": g["dgates"],
              "out_gpu": out_bits}
    meta = {"blk_cu": st["blk"]["cu"], "cu": np.asarray(w.cu_seqlens, np.int64), "hq": w.hq, "hkv": w.hkv,
            "topk": w.topk, "gate_mode": 0}
    res = cmp_full.run(arrays, meta, w.n, procs=2, pieces_per_proc=3)
    assert res["flips"] == [] and res["bad_sel_rows"] == 0
    for key in ("o", "lse", "dq", "dgates_cmp"):
        assert res[key] <= 1e-12, (key, res[key])
    assert res["out"] <= 2.0 ** -8 * np.abs(st["o"][0]).max()  # the bf16 rounding of out
    np.testing.assert_allclose(res["dkc"], g["parts"]["dkc"], rtol=0, atol=1e-11)
    np.testing.assert_allclose(res["dvc"], g["parts"]["dvc"], rtol=0, atol=1e-11)
