"""The bench's JSON line, checked through its CPU arm (the oracle on the host cores):
one line, the metric and config of the GPU arm, and the keys the contract names."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--tokens", "4096",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"]
    assert d["config"]["tokens"] == 4096 and "workload" in d["config"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_algorithmic_work_counts_scores_by_brute_force():
    """The roofline numerators: compressed, selected and window scores counted one
    (query row, key) pair at a time on a small varlen batch, and the flops per score
    of each tensor-core kernel (2d per contraction it performs)."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from oracle import ssa_oracle as O
    from spatial_sparse_attention_ssa_b200 import workloads as W

    w = W.small_shell(seed=71, R=32, n_prims=2, lo=4.0, hi=8.0, n_keep=200, n_seqs=3, hq=8, hkv=2, d=16,
                      m_cmp=4, m_win=3, topk=3, dtype="f32")
    blk = O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)
    win = O.bin_tokens(w.coords, w.cu_seqlens, w.m_win)
    rng = np.random.default_rng(3)
    sel = np.full((w.n, w.hkv, w.topk), -1, np.int64)
    seq = np.repeat(np.arange(w.s), np.diff(w.cu_seqlens))
    for t in range(w.n):
        b0, b1 = blk["cu"][seq[t]], blk["cu"][seq[t] + 1]
        for g in range(w.hkv):
            pick = rng.choice(np.arange(b0, b1), size=min(w.topk, b1 - b0), replace=False)
            sel[t, g, :len(pick)] = np.sort(pick)
    work, stages, scores = bench.kernel_work(w, blk["ptr"], blk["cu"], win["ptr"], sel)
    G = w.hq // w.hkv
    cmp = slc = wnd = 0
    for t in range(w.n):
        for h in range(w.hq):
            cmp += blk["cu"][seq[t] + 1] - blk["cu"][seq[t]]  # every block of the sequence
            slc += sum(blk["ptr"][b + 1] - blk["ptr"][b] for b in sel[t, h // G] if b >= 0)
            wnd += int((win["id"] == win["id"][t]).sum())  # every token of its window
    assert scores == {"cmp": float(cmp), "slc": float(slc), "win": float(wnd)}
    for name, per_score in (("cmp_bwd_dq_tc_kernel", 3), ("cmp_bwd_dkv_tc_kernel", 4), ("cmp_fa_tc_kernel", 2),
                            ("cmp_sel_tc_kernel", 1)):
        assert work[name][1] == 2 * w.d * per_score * cmp, name
    # stages count each contraction of the method once: the compressed forward needs S for the
    # normaliser, S again for the selection's final probabilities and P V (6d); every backward
    # needs S, dP, dQ, dK and dV (10d)
    assert stages["compressed forward"][1:] == (6 * w.d * cmp, 2 * cmp)
    assert stages["compressed backward"][1:] == (10 * w.d * cmp, cmp)
    assert stages["window backward"][1] == 10 * w.d * wnd and stages["selected backward"][1] == 10 * w.d * slc
    assert stages["window forward"][1] == 4 * w.d * wnd and stages["selected forward"][1] == 4 * w.d * slc
