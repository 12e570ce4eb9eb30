#!/usr/bin/env python
"""SSA forward + backward throughput on one B200 per rank.

A step is one pass of the whole SSA hot path -- binning (ssa_bin), compression,
compressed attention + top-k selection, selected-block and window attention,
the gated combine (ssa_forward) and the backward of all of it (ssa_backward) --
over the 1024^3 surface-shell workload with exactly 131072 voxel tokens
(32 query / 2 KV heads, d = 64, m_cmp = m_win = 8, top-k = 16, bf16 inputs,
fp32 accumulation, gate logits).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

For N > 1 launch with torch.distributed.run: every rank runs its own
independent workload (seeded by rank; no data-path collective) and the time is
the max over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSA fwd+bwd voxel tokens/s at 128k tokens; % of bf16 tensor / HBM peak"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
SMS = 148
FP32_LANES_PER_SM = 128
# DRAM bytes per step of the compressed backward's kernels at the 131072-token
# benchmark, from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, one pass;
# profiles/cmp_bwd_dram_gigascale1024_131072.md), valid while the kernels' source text
# (the backward section of csrc/cmp_tc.cu) has the recorded sha1.
BWD_TRAFFIC = {"source_sha1": "aa754fc8a81eeaa6a56e449c60da54af21c20ae5",
               "bytes_per_step": {"cmp_bwd_dq_tc_kernel": 1177.0e6 + 1024.0e6,
                                  "to_f16_kernel": 1073.9e6 + 1014.3e6 + 1.2e6,
                                  "cmp_bwd_dkv_tc_kernel": 1180.7e6 + 2.0e6}}


def _backward_source_sha1() -> str:
    path = os.path.join(ROOT, "spatial_sparse_attention_ssa_b200", "csrc", "cmp_tc.cu")
    with open(path, encoding="utf-8") as f:
        text = f.read()
    a = text.index("// backward, dQ (thread = row)")
    b = text.index("// host side", a)
    return hashlib.sha1(text[a:b].encode()).hexdigest()

def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--tokens", type=int, default=131072,
                    help="tokens of the 1024^3 workload (131072 is the benchmark; smaller only for ncu captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-geo", action="store_true", help="skip the separate timing of geometric block routing")
    ap.add_argument("--no-cross", action="store_true", help="skip the separate timing of cross attention")
    ap.add_argument("--no-conv", action="store_true", help="skip the separate timing of the learned compression")
    ap.add_argument("--no-scaled", action="store_true",
                    help="skip the timing of binning + compression at 16 * 2^20 tokens (HBM roofline)")
    ap.add_argument("--scaled-copies", type=int, default=128,
                    help="sequences of the scaled memory-bound leg (each a copy of the benchmark shell)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def _workload(seed: int, tokens: int = 131072):
    from spatial_sparse_attention_ssa_b200 import workloads as W
    return W.gigascale1024(seed, n_keep=tokens, backward=True)


def _workload_desc(w, nb, nw):
    return {"workload": "1024^3 surface shell of 5 ellipsoids + 2 slabs (semi-axes U(20,50)), subsampled to "
                        "%d voxel tokens; SSA fwd+bwd, 32 query / 2 KV heads, d=64, m_cmp=m_win=8, "
                        "top-k=16, bf16 in / fp32 accumulate, sigmoid gate logits" % w.n,
            "tokens": w.n, "blocks": nb, "windows": nw, "sequences": w.s}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
               "--format=csv,noheader,nounits", "-lms", "100"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.th = threading.Thread(target=self._read, daemon=True)
        self.th.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# algorithmic work per kernel (flops / bytes per launch)
# ---------------------------------------------------------------------------

def _traffic(stage: str, n_tokens: int, row: dict):
    """DRAM bytes per launch of the stage's kernels (ncu), or None when no capture of the
    current source at this size exists."""
    t = BWD_TRAFFIC
    if stage != "compressed backward" or n_tokens != 131072 or not t["source_sha1"]:
        return None
    if _backward_source_sha1() != t["source_sha1"] or set(row["kernels"]) != set(t["bytes_per_step"]):
        return None
    return float(sum(t["bytes_per_step"].values()))


def kernel_work(w, blk_ptr, blk_cu, win_ptr, sel):
    """Algorithmic work per kernel and per stage (a stage is the kernels of one
    branch and direction, e.g. the compressed backward = its dQ and dK/dV kernels;
    a stage lists every kernel that may implement it, and the ones that ran count).

    Scores: compressed = sum over sequences of n_s * Hq * B_s; selected = sum over
    (token, group) of G * (tokens in the selected blocks); window = Hq * sum over
    windows of n_w^2.  Flops per score are 2d for every contraction the method
    needs, counted once per stage: forward 6d for the compressed branch (S for the
    normaliser, S again for the selection's final probabilities, P.V) and 4d for
    the others; backward 10d (S, dP, dQ, dK, dV).  Exponentials per score: 2 in the
    compressed forward (flash pass, selection pass), 1 elsewhere.  Per kernel the same
    count covers the contractions that kernel performs; the bf16 low-part products,
    masked tile padding and the backward's second S / dP are overhead, not work.
    Memory kernels count the bytes they must move.
    """
    d, hq, hkv = w.d, w.hq, w.hkv
    G = hq // hkv
    nb_s = np.diff(blk_cu)
    n_s = np.diff(w.cu_seqlens)
    sc_cmp = float(np.sum(n_s.astype(np.float64) * hq * nb_s))
    bsize = np.diff(blk_ptr).astype(np.float64)
    selv = sel.reshape(-1)
    sc_slc = float(G * np.sum(bsize[selv[selv >= 0]]))
    wsize = np.diff(win_ptr).astype(np.float64)
    sc_win = float(hq * np.sum(wsize ** 2))
    e = 2  # bf16 bytes
    N, B = w.n, len(bsize)
    # per kernel: (kind, contraction flops, exps) for attention, ("bytes", bytes) for memory kernels
    work = {
        "cmp_fa_tc_kernel": ("tc", 4 * d * sc_cmp, sc_cmp),
        "cmp_sel_tc_kernel": ("tc", 2 * d * sc_cmp, sc_cmp),
        "cmp_bwd_dq_tc_kernel": ("tc", 6 * d * sc_cmp, sc_cmp),
        "cmp_bwd_dkv_tc_kernel": ("tc", 8 * d * sc_cmp, sc_cmp),
        "win_fwd_tc_kernel": ("tc", 4 * d * sc_win, sc_win),
        "win_bwd_dq_tc_kernel": ("tc", 6 * d * sc_win, sc_win),
        "win_bwd_dkv_tc_kernel": ("tc", 8 * d * sc_win, sc_win),
        "slc_fwd_mma_kernel": ("tc", 4 * d * sc_slc, sc_slc),
        "slc_bwd_mma_kernel": ("tc", 10 * d * sc_slc, sc_slc),
        "pool_kernel": ("bytes", 4.0 * N * hkv * d * e + 2.0 * B * hkv * d * e),
        "combine_kernel": ("bytes", 3.0 * N * hq * d * 4 + N * hq * 3 * 4 + N * hq * d * e),
        "bwd_pre_kernel": ("bytes", 3.0 * N * hq * d * 4 + N * hq * d * e + N * hq * 3 * 4 * 3),
        # fp16 copies of Q, dO and of Kc, Vc for the compressed dK/dV kernel (two launches per step)
        "to_f16_kernel": ("bytes", 2.0 * 2 * N * hq * d * e + 2.0 * 2 * B * hkv * d * e),
    }
    stages = {
        "compressed forward": (("cmp_fa_tc_kernel", "cmp_sel_tc_kernel"), 6 * d * sc_cmp, 2 * sc_cmp),
        "compressed backward": (("cmp_bwd_dq_tc_kernel", "to_f16_kernel", "cmp_bwd_dkv_tc_kernel"), 10 * d * sc_cmp,
                                sc_cmp),
        "window forward": (("win_fwd_tc_kernel",), 4 * d * sc_win, sc_win),
        "window backward": (("win_bwd_dq_tc_kernel", "win_bwd_dkv_tc_kernel"), 10 * d * sc_win, sc_win),
        "selected forward": (("slc_fwd_mma_kernel",), 4 * d * sc_slc, sc_slc),
        "selected backward": (("slc_bwd_mma_kernel",), 10 * d * sc_slc, sc_slc),
    }
    scores = {"cmp": sc_cmp, "slc": sc_slc, "win": sc_win}
    return work, stages, scores


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(a):
    import torch
    import torch.distributed as dist

    from spatial_sparse_attention_ssa_b200 import ssa
    from spatial_sparse_attention_ssa_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    w = _workload(a.seed + rank, a.tokens)
    t = W.make_tensors(w)

    def to_dev(x, bf=True):
        if bf and x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev)

    coords = to_dev(w.coords.astype(np.int32), False)
    cu = to_dev(w.cu_seqlens.astype(np.int32), False)
    q, k, v, do = to_dev(t.q), to_dev(t.k), to_dev(t.v), to_dev(t.do)
    gates = to_dev(t.gates, False)
    p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, torch.bfloat16, w.gate_mode)
    n, s = w.n, w.s
    bins = (ssa.Bins.empty(n, s, dev), ssa.Bins.empty(n, s, dev))
    ws_bin = torch.empty(ssa.lib().ssa_workspace_size(ssa.OP_BIN, None, s, n, n, n), dtype=torch.uint8, device=dev)
    blk, win = ssa.ssa_bin(coords, cu, w.R, w.m_cmp, w.m_win, out=bins, workspace=ws_bin)
    saved = ssa.SavedTensors.empty(p, n, blk.count, torch.bfloat16, dev)
    out = torch.empty_like(q)
    grads = (torch.empty(q.shape, dtype=torch.float32, device=dev), torch.empty(k.shape, dtype=torch.float32, device=dev),
             torch.empty(v.shape, dtype=torch.float32, device=dev),
             torch.empty(gates.shape, dtype=torch.float32, device=dev))
    ws_f = torch.empty(max(256, ssa.workspace_size(ssa.OP_FORWARD, p, s, n, blk.count, win.count)), dtype=torch.uint8,
                       device=dev)
    ws_b = torch.empty(max(256, ssa.workspace_size(ssa.OP_BACKWARD, p, s, n, blk.count, win.count)),
                       dtype=torch.uint8, device=dev)

    def step(cx=coords, cux=cu, qx=q, kx=k, vx=v, gx=gates, dx=do, outx=out, gradsx=grads):
        b_, w_ = ssa.ssa_bin(cx, cux, w.R, w.m_cmp, w.m_win, out=bins, workspace=ws_bin)
        ssa.ssa_forward(p, cux, b_, w_, qx, kx, vx, gx, out=outx, saved=saved, workspace=ws_f)
        ssa.ssa_backward(p, cux, b_, w_, qx, kx, vx, gx, saved, dx, grads=gradsx, workspace=ws_b)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB L2

    def check_device(where):
        torch.cuda.synchronize()
        code = ssa.device_status()
        if code != 0:
            raise SystemExit("device check word after %s: %s" % (where, ssa.STATUS_NAMES.get(code, code)))

    for i in range(a.warmup):
        step()
        if i == 0:
            check_device("the first step")
    check_device("warm-up")

    # ---- timed region: K steps, device-timed per step, L2 flushed between steps
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", ""))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = ssa.launch_count()
    ssa.profile_read()
    ssa.profile_enable(True)
    sampler.start()
    wall0 = time.perf_counter()
    for i in range(a.steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    ssa.profile_enable(False)
    launches = ssa.launch_count() - launches0
    prof = ssa.profile_read()
    check_device("the timed steps")
    ms = sum(a_.elapsed_time(b_) for a_, b_ in ev) / a.steps
    ms_max = ms
    if world > 1:
        tt = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms_max = float(tt.item())
    total_tokens = n * world

    # ---- end to end through host buffers (pinned), same metric
    e2e = None
    if not a.no_e2e:
        host_in = {"coords": coords.cpu().pin_memory(), "cu": cu.cpu().pin_memory(), "q": q.cpu().pin_memory(),
                   "k": k.cpu().pin_memory(), "v": v.cpu().pin_memory(), "gates": gates.cpu().pin_memory(),
                   "do": do.cpu().pin_memory()}
        h2d = sum(x.numel() * x.element_size() for x in host_in.values())
        d2h = sum(x.numel() * x.element_size() for x in [out, *grads])

        def reduce_max(ms_):
            if world > 1:
                tt = torch.tensor([ms_], device=dev, dtype=torch.float64)
                dist.all_reduce(tt, op=dist.ReduceOp.MAX)
                ms_ = float(tt.item())
            return ms_

        # (1) serial: copy in, step, copy out, one step after the other
        nset = 3  # buffer sets of the pipelined run (3 x ~3 GB on the device)
        dev_in = [{kk: torch.empty_like(vv, device=dev) for kk, vv in host_in.items()} for _ in range(nset)]
        dev_out = [[torch.empty_like(out)] + [torch.empty_like(g_) for g_ in grads] for _ in range(nset)]
        host_out = [[torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in [out, *grads]] for _ in range(nset)]
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(a.steps):
            flush.zero_()
            ee[i][0].record()
            for kk in host_in:
                dev_in[0][kk].copy_(host_in[kk], non_blocking=True)
            di = dev_in[0]
            step(di["coords"], di["cu"], di["q"], di["k"], di["v"], di["gates"], di["do"], dev_out[0][0],
                 tuple(dev_out[0][1:]))
            for src, dst in zip(dev_out[0], host_out[0]):
                dst.copy_(src, non_blocking=True)
            ee[i][1].record()
        torch.cuda.synchronize()
        serial_ms = reduce_max(sum(a_.elapsed_time(b_) for a_, b_ in ee) / a.steps)

        # (2) pipelined: step i's inputs go up on one copy stream while earlier steps
        # compute, its results come down on another while later steps compute; three
        # device buffer sets.  Every step still moves all of its inputs and results.
        comp = torch.cuda.current_stream(dev)
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready = [torch.cuda.Event() for _ in range(nset)]
        in_free = [torch.cuda.Event() for _ in range(nset)]
        out_ready = [torch.cuda.Event() for _ in range(nset)]
        out_free = [torch.cuda.Event() for _ in range(nset)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def upload(j):
            with torch.cuda.stream(up):
                for kk in host_in:
                    dev_in[j][kk].copy_(host_in[kk], non_blocking=True)
                in_ready[j].record(up)

        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start.record(comp)
        up.wait_stream(comp)
        down.wait_stream(comp)
        upload(0)
        for i in range(a.steps):
            j = i % nset
            if i + 1 < a.steps:
                jn = (i + 1) % nset
                if i + 1 >= nset:
                    up.wait_event(in_free[jn])  # step i+1-nset is done with that input set
                upload(jn)
            comp.wait_event(in_ready[j])
            if i >= nset:
                comp.wait_event(out_free[j])  # step i-nset's results are down
            flush.zero_()
            di = dev_in[j]
            step(di["coords"], di["cu"], di["q"], di["k"], di["v"], di["gates"], di["do"], dev_out[j][0],
                 tuple(dev_out[j][1:]))
            in_free[j].record(comp)
            out_ready[j].record(comp)
            down.wait_event(out_ready[j])
            with torch.cuda.stream(down):
                for src, dst in zip(dev_out[j], host_out[j]):
                    dst.copy_(src, non_blocking=True)
                out_free[j].record(down)
        comp.wait_stream(down)
        comp.wait_stream(up)
        t_end.record(comp)
        torch.cuda.synchronize()
        e_ms = reduce_max(t_start.elapsed_time(t_end) / a.steps)
        e2e = {"value": total_tokens / (e_ms / 1e3), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "mode": "pipelined: step i+1's inputs up and earlier steps' results down while step i computes "
                       "(three buffer sets, two copy streams); timed from the first upload to the last download",
               "serial": {"value": total_tokens / (serial_ms / 1e3), "ms_per_step": serial_ms}}

    # ---- roofline of the dominant kernel
    peaks = _peaks()
    blk_ptr = blk.ptr[:blk.count + 1].cpu().numpy()
    blk_cu = blk.cu.cpu().numpy()
    win_ptr = win.ptr[:win.count + 1].cpu().numpy()
    sel = saved.sel.cpu().numpy()
    work, stages, scores = kernel_work(w, blk_ptr, blk_cu, win_ptr, sel)
    mhz = peaks.get("sm_max_mhz", 1965.0)
    tc_peak = peaks.get("bf16_tflops")  # burst: the step is tens of ms, not a seconds-long loop
    mufu_peak = SMS * 16 * mhz * 1e6 / 1e12  # Texp/s: 16 ex2 per clock per SM
    per_kernel = {}
    for name, (tot, cnt) in prof.items():
        ms_l = tot / max(cnt, 1)
        ms_st = tot / a.steps  # the work figures are per step (to_f16_kernel runs twice a step)
        ent = {"ms_per_step": ms_st, "launches": cnt, "ms_per_launch": ms_l}
        wk = work.get(name)
        if wk is not None and wk[0] == "tc":
            ent["tflops"] = wk[1] / (ms_st / 1e3) / 1e12
            ent["tensor_frac"] = ent["tflops"] / tc_peak
            ent["mufu_frac"] = wk[2] / (ms_st / 1e3) / 1e12 / mufu_peak
        elif wk is not None:
            ent["gbs"] = wk[1] / (ms_st / 1e3) / 1e9
            ent["hbm_frac"] = ent["gbs"] / peaks["hbm_gbs"]
        per_kernel[name] = ent
    stage_rows = {}
    for sname, (cands, flops, exps) in stages.items():
        kernels = [k_ for k_ in cands if k_ in prof]  # the stage's kernels that ran
        if not kernels:
            continue
        ms_s = sum(prof[k_][0] / a.steps for k_ in kernels)  # device time of the stage per step
        stage_rows[sname] = {"kernels": list(kernels), "ms": ms_s, "tflops": flops / (ms_s / 1e3) / 1e12,
                             "tensor_frac": flops / (ms_s / 1e3) / 1e12 / tc_peak,
                             "mufu_frac": exps / (ms_s / 1e3) / 1e12 / mufu_peak,
                             "flops": flops, "exps": exps}
    roof = None
    exp_roof = None
    if stage_rows:
        dom = max(stage_rows, key=lambda k_: stage_rows[k_]["ms"])
        r_ = stage_rows[dom]
        roof = {"kernel": " + ".join(r_["kernels"]), "stage": dom, "bound": "tensor", "achieved": r_["tflops"],
                "peak": tc_peak, "unit": "TFLOP/s", "frac": r_["tensor_frac"], "traffic": _traffic(dom, n, r_),
                "peak_source": "%s bf16 dense, burst" % peaks["_source"],
                "algorithmic_per_launch": r_["flops"], "ms_per_launch": r_["ms"],
                "note": "one step's launches of the stage's kernels at its algorithmic flops (each contraction of "
                        "the method once); traffic: ncu DRAM bytes of those launches (null unless captured on this "
                        "source at this size)"}
        exp_roof = {"kernel": roof["kernel"], "bound": "mufu", "achieved": r_["exps"] / (r_["ms"] / 1e3) / 1e12,
                    "peak": mufu_peak, "unit": "Texp/s", "frac": r_["mufu_frac"],
                    "peak_source": "derived: %d SMs x 16 ex2/clock x %.0f MHz" % (SMS, mhz),
                    "exps_per_launch": r_["exps"]}

    # ---- geometric block routing (selection by voxel distance), timed on its own
    geo = None
    if not a.no_geo:
        sel_geo = torch.empty((n, w.hkv, w.topk), dtype=torch.int32, device=dev)
        ws_geo = torch.empty(ssa.lib().ssa_workspace_size(ssa.OP_GEO_SELECT, None, s, n, blk.count, 0),
                             dtype=torch.uint8, device=dev)
        for _ in range(3):
            ssa.ssa_geo_select(coords, cu, w.R, blk, w.m_cmp, w.topk, w.hkv, out=sel_geo, workspace=ws_geo)
        check_device("geometric routing warm-up")
        eg = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
        for i in range(a.steps):
            flush.zero_()
            eg[i][0].record()
            ssa.ssa_geo_select(coords, cu, w.R, blk, w.m_cmp, w.topk, w.hkv, out=sel_geo, workspace=ws_geo)
            eg[i][1].record()
        torch.cuda.synchronize()
        check_device("geometric routing")
        g_ms = sum(a_.elapsed_time(b_) for a_, b_ in eg) / a.steps
        geo = {"ms_per_call": g_ms, "tokens_per_s": n / (g_ms / 1e3), "blocks": int(blk.count),
               "topk": int(w.topk), "launches_per_call": 2}

    # ---- cross attention (queries from another token set), timed on its own: the
    # same voxel tokens as keys / values, Nq = n image-token queries, fwd + bwd
    cross = None
    if not a.no_cross:
        cq = W.make_cross_queries(w, [n], seed=3)
        q_cu = to_dev(cq.q_cu.astype(np.int32), False)
        cq_q, cq_do = to_dev(cq.q), to_dev(cq.do)
        cq_g = to_dev(cq.gates, False)
        c_saved = ssa.SavedTensors.empty_cross(p, n, n, blk.count, torch.bfloat16, dev)
        c_out = torch.empty_like(cq_q)
        c_grads = (torch.empty(cq_q.shape, dtype=torch.float32, device=dev),
                   torch.empty(k.shape, dtype=torch.float32, device=dev),
                   torch.empty(v.shape, dtype=torch.float32, device=dev),
                   torch.empty(cq_g.shape, dtype=torch.float32, device=dev))
        c_wf = torch.empty(ssa.workspace_size(ssa.OP_CROSS_FORWARD, p, 1, n, blk.count, 0), dtype=torch.uint8,
                           device=dev)
        c_wb = torch.empty(ssa.workspace_size(ssa.OP_CROSS_BACKWARD, p, 1, n, blk.count, 0), dtype=torch.uint8,
                           device=dev)

        def cross_step():
            ssa.ssa_cross_forward(p, q_cu, blk, cq_q, k, v, cq_g, out=c_out, saved=c_saved, workspace=c_wf)
            ssa.ssa_cross_backward(p, q_cu, blk, cq_q, k, v, cq_g, c_saved, cq_do, grads=c_grads, workspace=c_wb)

        for _ in range(3):
            cross_step()
        check_device("cross-attention warm-up")
        ec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
        for i in range(a.steps):
            flush.zero_()
            ec[i][0].record()
            cross_step()
            ec[i][1].record()
        torch.cuda.synchronize()
        check_device("cross attention")
        c_ms = sum(a_.elapsed_time(b_) for a_, b_ in ec) / a.steps
        cross = {"ms_per_step": c_ms, "query_tokens_per_s": n / (c_ms / 1e3), "query_tokens": n, "voxel_tokens": n,
                 "what": "ssa_cross_forward + ssa_cross_backward: N(0,1) bf16 image-token queries against the "
                         "voxel tokens (compressed + selected branches, same heads, k, m_cmp)"}
        del c_saved, c_grads, c_wf, c_wb

    # ---- learned compression (sparse 3x3x3 convolution before the block mean), the
    # same step with the convolution on; its own kernels' times from the library's events
    learned = None
    if not a.no_conv:
        rng = np.random.default_rng(11)
        std = 0.3 / np.sqrt(9 * w.d)
        cw = [torch.from_numpy((std * rng.standard_normal((w.hkv, 27, w.d, w.d))).astype(np.float32)).to(dev),
              torch.from_numpy((0.1 * rng.standard_normal((w.hkv, w.d))).astype(np.float32)).to(dev),
              torch.from_numpy((std * rng.standard_normal((w.hkv, 27, w.d, w.d))).astype(np.float32)).to(dev),
              torch.from_numpy((0.1 * rng.standard_normal((w.hkv, w.d))).astype(np.float32)).to(dev)]
        conv = ssa.ConvWeights(coords, *cw)
        pc = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, torch.bfloat16, w.gate_mode, conv=conv)
        l_wf = torch.empty(ssa.workspace_size(ssa.OP_FORWARD, pc, s, n, blk.count, win.count), dtype=torch.uint8,
                           device=dev)
        l_wb = torch.empty(ssa.workspace_size(ssa.OP_BACKWARD, pc, s, n, blk.count, win.count), dtype=torch.uint8,
                           device=dev)

        def conv_step():
            b_, w_ = ssa.ssa_bin(coords, cu, w.R, w.m_cmp, w.m_win, out=bins, workspace=ws_bin)
            ssa.ssa_forward(pc, cu, b_, w_, q, k, v, gates, out=out, saved=saved, workspace=l_wf)
            ssa.ssa_backward(pc, cu, b_, w_, q, k, v, gates, saved, do, grads=grads, workspace=l_wb)

        for _ in range(3):
            conv_step()
        check_device("learned-compression warm-up")
        el = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
        ssa.profile_read()
        ssa.profile_enable(True)
        for i in range(a.steps):
            flush.zero_()
            el[i][0].record()
            conv_step()
            el[i][1].record()
        torch.cuda.synchronize()
        ssa.profile_enable(False)
        cprof = ssa.profile_read()
        check_device("learned compression")
        l_ms = sum(a_.elapsed_time(b_) for a_, b_ in el) / a.steps
        conv_k = {nm: tot / a.steps for nm, (tot, cnt) in cprof.items() if nm.startswith("conv_")}
        learned = {"ms_per_step": l_ms, "tokens_per_s": n / (l_ms / 1e3), "conv_kernels_ms_per_step": conv_k,
                   "what": "the benchmark step with Kc / Vc from a sparse 3x3x3 convolution of K and V (random "
                           "N(0, 0.3^2/(9d)) weights) before the block mean, gradients to the weights included"}
        del l_wf, l_wb

    # ---- the memory-bound steps at scale: binning (ssa_bin) and compression (ssa_pool) of
    # 16 * 2^20 tokens, 128 sequences each holding a copy of the benchmark shell's coordinates,
    # N(0,1) bf16 K / V drawn on the device.  At 131072 tokens these kernels are launch- and
    # latency-bound (1.5 MB of coordinates); at this size their HBM rate shows.
    scaled = None
    if not a.no_scaled:
        del bins, ws_bin
        torch.cuda.empty_cache()
        copies = a.scaled_copies
        ns = copies * n
        sc_coords = coords.repeat(copies, 1).contiguous()
        sc_cu = (torch.arange(copies + 1, device=dev, dtype=torch.int64) * n).to(torch.int32)
        gen = torch.Generator(device=dev).manual_seed(1234)
        sk = torch.randn((ns, w.hkv, w.d), device=dev, generator=gen).to(torch.bfloat16)
        sv = torch.randn((ns, w.hkv, w.d), device=dev, generator=gen).to(torch.bfloat16)
        sbins = (ssa.Bins.empty(ns, copies, dev), ssa.Bins.empty(ns, copies, dev))
        sws = torch.empty(ssa.lib().ssa_workspace_size(ssa.OP_BIN, None, copies, ns, ns, ns), dtype=torch.uint8,
                          device=dev)
        sb, sw = ssa.ssa_bin(sc_coords, sc_cu, w.R, w.m_cmp, w.m_win, out=sbins, workspace=sws)
        pool_out = ssa.ssa_pool(sb, sk, sv)
        torch.cuda.synchronize()
        check_device("scaled warm-up")
        reps = max(3, a.steps)
        ssa.profile_read()
        ssa.profile_enable(True)
        eb = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps):
            flush.zero_()
            eb[i][0].record()
            sb, sw = ssa.ssa_bin(sc_coords, sc_cu, w.R, w.m_cmp, w.m_win, out=sbins, workspace=sws)
            eb[i][1].record()
            flush.zero_()
            ssa.ssa_pool(sb, sk, sv, out=pool_out)
        torch.cuda.synchronize()
        ssa.profile_enable(False)
        sprof = ssa.profile_read()
        check_device("scaled binning and compression")
        bin_ms = sum(a_.elapsed_time(b_) for a_, b_ in eb) / reps
        nb_s, nw_s = int(sb.count), int(sw.count)
        # bytes the steps must move: binning reads the coordinates and writes, per partition, the
        # token ids and permutation and, per cell, its pointer and key; compression reads K and V
        # and writes their block-ordered copies and the block means
        bin_bytes = 12.0 * ns + 2 * 8.0 * ns + 16.0 * (nb_s + nw_s)
        pool_bytes = 4.0 * ns * w.hkv * w.d * 2 + 2.0 * nb_s * w.hkv * w.d * 2
        pool_ms = sprof["pool_kernel"][0] / max(sprof["pool_kernel"][1], 1) if "pool_kernel" in sprof else None
        bin_kernels = {k_: v_[0] / reps for k_, v_ in sprof.items() if k_ != "pool_kernel"}
        bin_kernel_ms = sum(bin_kernels.values())
        hbm = peaks["hbm_gbs"]
        scaled = {"tokens": ns, "sequences": copies, "blocks": nb_s,
                  "pool": {"ms": pool_ms, "bytes": pool_bytes,
                           "gbs": pool_bytes / (pool_ms / 1e3) / 1e9 if pool_ms else None,
                           "hbm_frac": pool_bytes / (pool_ms / 1e3) / 1e9 / hbm if pool_ms else None},
                  "bin": {"ms_call": bin_ms, "ms_kernels": bin_kernel_ms, "bytes": bin_bytes,
                          "gbs_call": bin_bytes / (bin_ms / 1e3) / 1e9,
                          "hbm_frac_call": bin_bytes / (bin_ms / 1e3) / 1e9 / hbm,
                          "gbs_kernels": bin_bytes / (bin_kernel_ms / 1e3) / 1e9,
                          "hbm_frac_kernels": bin_bytes / (bin_kernel_ms / 1e3) / 1e9 / hbm,
                          "kernels_ms": bin_kernels},
                  "peak_gbs": hbm, "peak_source": peaks["_source"],
                  "what": "ssa_bin (device events around the call, which synchronises once) and ssa_pool "
                          "(pool_kernel events) at 16 * 2^20 tokens; algorithmic bytes: binning 12 B of "
                          "coordinates + 2 x 8 B of ids / permutation per token + 16 B per cell; compression "
                          "2 x 2 x Hkv x d x 2 B per token + 2 x Hkv x d x 2 B per block"}
        del sk, sv, sbins, sws, pool_out, sc_coords

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, t, a.cpu_seconds)

    if rank == 0:
        cfg = _workload_desc(w, blk.count, win.count)
        cfg.update({"global_batch": world, "parallelism": "dp%d" % world,
                    "l2": "256 MB buffer written between timed steps (L2 is 126 MB); step working set ~6 GB",
                    "scores": scores})
        line = {"metric": METRIC, "value": total_tokens / (ms_max / 1e3), "unit": UNIT, "n_gpus": world,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms_max, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded surface-shell voxels, N(0,1) bf16 Q/K/V/dO, N(0,1) gate logits)",
                "config": cfg, "roofline": roof, "roofline_exp": exp_roof, "stages": stage_rows,
                "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": int(launches),
                "clocks": clocks, "wall_s_timed": wall, "kernels": per_kernel, "geo_routing": geo,
                "cross_attention": cross, "learned_compression": learned, "memory_bound_scaled": scaled,
                "peaks_source": peaks["_source"]}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# CPU oracle leg
# ---------------------------------------------------------------------------

def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_sample(w, t, tokens):
    """The oracle's forward of the sampled query tokens (binning and pooling of all
    tokens, then the three branches of the sample), and the compressed branch's
    backward of the sampled rows: their dQ and their contributions to dKc / dVc."""
    from oracle import ssa_oracle as O
    q, do = t.as_f32("q"), t.as_f32("do")
    st = O.forward(w.coords, w.cu_seqlens, q, t.as_f32("k"), t.as_f32("v"), t.gates, hq=w.hq,
                   hkv=w.hkv, m_cmp=w.m_cmp, m_win=w.m_win, topk=w.topk, gate_mode=w.gate_mode,
                   pool_rounding="bf16", tokens=tokens)
    for tok in tokens:
        O.cmp_branch_range(q, st["kc"], st["vc"], st["blk"]["cu"], w.cu_seqlens, t.gates, hq=w.hq, hkv=w.hkv,
                           topk=w.topk, gate_mode=w.gate_mode, t0=int(tok), t1=int(tok) + 1, dout=do)


def _sample_tokens(w, n):
    return np.linspace(0, w.n - 1, num=max(1, n)).astype(np.int64)


def cpu_baseline(w, t, seconds: float) -> dict:
    """The oracle as it stands, on a bounded sample: binning + pooling of all
    tokens, then every forward branch and the dQ rows for T sampled query tokens."""
    # two calibration points separate the fixed cost (binning, pooling) from the per-token cost
    t0 = time.perf_counter()
    _oracle_sample(w, t, _sample_tokens(w, 16))
    ta = time.perf_counter() - t0
    t0 = time.perf_counter()
    _oracle_sample(w, t, _sample_tokens(w, 80))
    tb = time.perf_counter() - t0
    per_tok = max((tb - ta) / 64.0, 1e-4)
    fixed = max(ta - 16 * per_tok, 0.0)
    T = int(max(16, min(w.n, (seconds - fixed) / per_tok)))
    t0 = time.perf_counter()
    _oracle_sample(w, t, _sample_tokens(w, T))
    el = time.perf_counter() - t0
    return {"value": T / el, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": "numpy fp64 oracle: binning + mean pooling of all %d tokens, then for %d evenly spaced "
                      "query tokens the forward of all three branches and the compressed branch's backward (dQ "
                      "and the rows' dKc / dVc sums; the selected and window backward, ~3%% of the flops, left "
                      "out); %.1f s" % (w.n, T, el),
            "seconds": el}


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from oracle import ssa_oracle as O
    from spatial_sparse_attention_ssa_b200 import workloads as W
    w = _workload(a.seed, a.tokens)
    t = W.make_tensors(w)
    nb = int(O.bin_tokens(w.coords, w.cu_seqlens, w.m_cmp)["count"])
    nw = int(O.bin_tokens(w.coords, w.cu_seqlens, w.m_win)["count"])
    budget = max(2.0, 150.0 / max(1, a.steps + a.warmup))  # whole run within a few minutes
    t0 = time.perf_counter()
    _oracle_sample(w, t, _sample_tokens(w, 8))
    t1 = time.perf_counter() - t0
    T = int(max(8, min(w.n, 8 * budget / max(t1, 1e-3))))
    for _ in range(a.warmup):
        _oracle_sample(w, t, _sample_tokens(w, T))
    times = []
    for _ in range(a.steps):
        t0 = time.perf_counter()
        _oracle_sample(w, t, _sample_tokens(w, T))
        times.append(time.perf_counter() - t0)
    ms = 1e3 * sum(times) / len(times)
    value = T / (ms / 1e3)
    cores = _blas_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded workload as the GPU arm)",
            "config": dict(_workload_desc(w, nb, nw), global_batch=world, parallelism="dp%d" % world),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "per step: binning + pooling of all tokens, then the forward of all "
                                       "branches and the compressed backward rows of %d evenly spaced query "
                                       "tokens" % T},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    a = _args()
    if a.warmup < 0 or a.steps < 1:
        raise SystemExit("bad --steps / --warmup")
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
