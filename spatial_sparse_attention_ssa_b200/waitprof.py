"""Where the compressed-branch kernels wait: cycle counters around every mbarrier wait.

    python -m spatial_sparse_attention_ssa_b200.waitprof [--tokens N]

Builds a separate, instrumented copy of the library under _build/waitprof/ (the
product library is untouched): in the four tensor-core kernels of the compressed
branch (flash pass, selection pass, dQ, dK/dV) every `mbar_wait` / `mbar_wait_warp`
call is wrapped so that lane 0 of each warp adds the clock64() cycles it spent in
that wait to a per-(CTA, warp, wait site) counter, and each warp's total cycles in
the kernel are counted too.  It then runs the benchmark's forward + backward step on
the 1024^3 shell once through that copy and prints, per kernel and wait site, the
share of each warp's cycles spent waiting there (one JSON object).

The counters add a few instructions per wait, so the kernels run a few per cent
slower under it; the shares, not the absolute times, are the result.  A development
aid: it needs nvcc and a GPU, and no test or benchmark depends on it.
"""
from __future__ import annotations

import argparse
import ctypes
import glob
import json
import os
import re
import shutil
import subprocess
import sys

from . import build as B

KERNELS = ("cmp_fa_tc_kernel(", "cmp_sel_tc_kernel(", "cmp_bwd_dq_tc_kernel(", "cmp_bwd_dkv_tc_kernel(")
SLOTS_PER_KERNEL = 15
MAX_CTAS, MAX_WARPS, NSLOTS = 160, 24, 64  # counter array [cta][warp][slot]; slot 60 + k = kernel k's total

_HEADER = ("__device__ unsigned long long g_wprof[%d][%d][%d];\n"
           "#define PW(slot, expr) ([&]() -> bool { const long long _t0 = clock64(); const bool _r = (expr); "
           "if ((threadIdx.x & 31) == 0 && blockIdx.x < %d) g_wprof[blockIdx.x][threadIdx.x >> 5][slot] += "
           "(unsigned long long)(clock64() - _t0); return _r; }())\n") % (MAX_CTAS, MAX_WARPS, NSLOTS, MAX_CTAS)

_READER = ("\nextern \"C\" __attribute__((visibility(\"default\"))) int ssa_waitprof_read(unsigned long long* host, "
           "int reset) {\n"
           "  if (host && cudaMemcpyFromSymbol(host, g_wprof, sizeof(g_wprof)) != cudaSuccess) return 1;\n"
           "  if (reset) { void* p = nullptr; if (cudaGetSymbolAddress(&p, g_wprof) != cudaSuccess) return 2;\n"
           "    if (cudaMemset(p, 0, sizeof(g_wprof)) != cudaSuccess) return 3; }\n"
           "  return cudaDeviceSynchronize() == cudaSuccess ? 0 : 4;\n}\n")


def instrument(src: str):
    """Return (instrumented cmp_tc.cu text, {slot: (kernel, line, wait call)})."""
    lines = src.split("\n")
    starts = []
    for k in KERNELS:
        idx = [i for i, l in enumerate(lines) if k in l and i > 0 and "__global__" in lines[i - 1] + l]
        if len(idx) != 1:
            raise ValueError("kernel %s found %d times" % (k, len(idx)))
        starts.append(idx[0])
    slots = {}
    for j, a in enumerate(starts):
        e = next(i for i in range(a, len(lines)) if "tmem_dealloc(" in lines[i])
        n = 0
        for i in range(a, e):
            line = lines[i]
            if "mma_done, 0" in line or "last_par" in line:
                continue  # the final drains are not part of the pipeline
            out, pos = [], 0
            while True:
                m = re.search(r"\b(mbar_wait_warp|mbar_wait)\(", line[pos:])
                if not m:
                    out.append(line[pos:])
                    break
                s0 = pos + m.start()
                depth, q = 0, pos + m.end() - 1
                while True:
                    if line[q] == "(":
                        depth += 1
                    elif line[q] == ")":
                        depth -= 1
                        if depth == 0:
                            break
                    q += 1
                call = line[s0:q + 1]
                if n >= SLOTS_PER_KERNEL:
                    raise ValueError("too many wait sites in %s" % KERNELS[j])
                slot = SLOTS_PER_KERNEL * j + n
                slots[slot] = (KERNELS[j][:-1], i + 1, call)
                n += 1
                out += [line[pos:s0], "PW(%d, %s)" % (slot, call)]
                pos = q + 1
            lines[i] = "".join(out)
        t = next(i for i in range(a, e) if "const uint32_t tmem = sm.tmem;" in lines[i])
        lines[t] = lines[t].replace("const uint32_t tmem = sm.tmem;",
                                    "const uint32_t tmem = sm.tmem; const long long _tk0 = clock64();")
        lines[e - 2] += ("\n  if ((threadIdx.x & 31) == 0 && blockIdx.x < %d) g_wprof[blockIdx.x][threadIdx.x >> 5][%d]"
                         " += (unsigned long long)(clock64() - _tk0);" % (MAX_CTAS, 60 + j))
    out = "\n".join(lines)
    ns = out.index("namespace ssa {")
    return out[:ns] + _HEADER + out[ns:] + _READER, slots


def build_instrumented() -> tuple[str, dict]:
    d = os.path.join(B.PKG, "_build", "waitprof")
    if os.path.exists(d):
        shutil.rmtree(d)
    csrc = os.path.join(d, "csrc")
    shutil.copytree(B.CSRC, csrc)
    path = os.path.join(csrc, "cmp_tc.cu")
    with open(path) as f:
        text, slots = instrument(f.read())
    with open(path, "w") as f:
        f.write(text)
    objs, procs = [], []
    flags = [x if x != B.CSRC else csrc for x in B.NVCC_FLAGS]
    for src in sorted(glob.glob(os.path.join(csrc, "*.cu"))):
        obj = src[:-3] + ".o"
        objs.append(obj)
        procs.append(subprocess.Popen([B.nvcc(), *B.ARCH, *flags, "-c", src, "-o", obj], stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT))
    for p in procs:
        out, _ = p.communicate()
        if p.returncode:
            raise RuntimeError(out.decode()[-3000:])
    lib = os.path.join(d, "libssa.so")
    subprocess.check_call([B.nvcc(), *B.ARCH, "-shared", "-o", lib, *objs])
    return lib, slots


def run(tokens: int) -> dict:
    import numpy as np
    import torch

    from . import ssa
    from . import workloads as W

    lib_path, slots = build_instrumented()
    ssa.LIB_PATH = lib_path
    w = W.gigascale1024(0, n_keep=tokens, backward=True)
    t = W.make_tensors(w)
    dev = torch.device("cuda")

    def bf(x):
        return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)

    coords = torch.from_numpy(w.coords.astype(np.int32)).to(dev)
    cu = torch.from_numpy(w.cu_seqlens.astype(np.int32)).to(dev)
    q, k, v, do = bf(t.q), bf(t.k), bf(t.v), bf(t.do)
    gates = torch.from_numpy(t.gates).to(dev)
    p = ssa.make_params(w.hq, w.hkv, w.d, w.m_cmp, w.m_win, w.topk, torch.bfloat16, w.gate_mode)

    def step():
        blk, win = ssa.ssa_bin(coords, cu, w.R, w.m_cmp, w.m_win)
        _, saved = ssa.ssa_forward(p, cu, blk, win, q, k, v, gates)
        ssa.ssa_backward(p, cu, blk, win, q, k, v, gates, saved, do)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    if ssa.device_status() != 0:
        raise RuntimeError("device status after warm-up")
    fn = ssa.lib().ssa_waitprof_read
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int]
    fn.restype = ctypes.c_int
    if fn(None, 1) != 0:
        raise RuntimeError("counter reset failed")
    ssa.profile_read()
    ssa.profile_enable(True)
    step()
    torch.cuda.synchronize()
    ssa.profile_enable(False)
    prof = ssa.profile_read()
    if ssa.device_status() != 0:
        raise RuntimeError("device status after the measured step")
    buf = np.zeros((MAX_CTAS, MAX_WARPS, NSLOTS), np.uint64)
    if fn(buf.ctypes.data, 0) != 0:
        raise RuntimeError("counter read failed")
    res = {"tokens": tokens, "kernels": {}}
    for j, kname in enumerate(KERNELS):
        name = kname[:-1]
        tot = buf[:, :, 60 + j].astype(np.float64)
        ctas = np.nonzero(tot.sum(1))[0]
        ent = {"ms_instrumented": prof.get(name, (0.0, 1))[0], "ctas_counted": int(len(ctas)), "sites": []}
        for s in range(SLOTS_PER_KERNEL * j, SLOTS_PER_KERNEL * (j + 1)):
            if s not in slots:
                continue
            cyc = buf[:, :, s].astype(np.float64)
            warps = np.nonzero(cyc.sum(0))[0]
            share = {int(wi): round(float(cyc[ctas, wi].sum() / max(tot[ctas, wi].sum(), 1.0)), 3) for wi in warps}
            ent["sites"].append({"line": slots[s][1], "wait": slots[s][2], "share_of_warp_cycles": share})
        res["kernels"][name] = ent
    return res


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--tokens", type=int, default=131072)
    a = ap.parse_args(argv)
    print(json.dumps(run(a.tokens)))


if __name__ == "__main__":
    main(sys.argv[1:])
