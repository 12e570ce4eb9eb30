"""The C-ABI library loads and exports every entry point the header declares.

Runs without a GPU: only host-side calls (sizes, error strings, argument checks
that return before any CUDA work) are made.
"""
import ctypes
import os
import re

import pytest
import torch

from spatial_sparse_attention_ssa_b200 import ssa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"SSA_API\s+[\w\s\*]+?\b(ssa_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    lib = ssa.lib()
    declared = _declared()
    assert {"ssa_bin", "ssa_forward", "ssa_backward", "ssa_workspace_size"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(ssa.EXPORTS) <= declared


def test_host_side_calls():
    lib = ssa.lib()
    assert lib.ssa_version() >= 100
    for code in range(7):
        assert lib.ssa_error_string(code)
    p = ssa.Params(32, 2, 64, 8, 8, 16, 0.0, ssa.DTYPE_BF16, ssa.GATE_LOGITS)
    n, b = 131072, 2322
    fw = ssa.workspace_size(ssa.OP_FORWARD, p, 1, n, b, b)
    bw = ssa.workspace_size(ssa.OP_BACKWARD, p, 1, n, b, b)
    assert fw > 0 and bw > 3 * n * 32 * 4
    assert lib.ssa_workspace_size(ssa.OP_BIN, None, 1, n, n, n) > 16 * n
    bad = ssa.Params(30, 4, 64, 8, 8, 16, 0.0, ssa.DTYPE_BF16, ssa.GATE_LOGITS)  # 30 % 4 != 0
    assert ssa.workspace_size(ssa.OP_FORWARD, bad, 1, n, b, b) == 0


@pytest.mark.parametrize("field,value,code", [
    ("hq", 31, 1), ("hq", 30, 2), ("d", 48, 2), ("topk", 0, 1), ("topk", 33, 2), ("m_cmp", 0, 1), ("dtype", 7, 1),
    ("gate_mode", 3, 1), ("scale", -1.0, 1), ("hkv", 1, 2),  # G = 32 with d = 64 is not handled
])
def test_argument_errors_are_status_codes(field, value, code):
    lib = ssa.lib()
    p = ssa.Params(32, 2, 64, 8, 8, 16, 0.0, ssa.DTYPE_BF16, ssa.GATE_LOGITS)
    setattr(p, field, value)
    part = ssa.Partition(1, 1, 1, 1, 1, 10)
    saved = ssa.Saved(1, 1, 1, 1, 1, 1, 1)
    st = lib.ssa_forward(ctypes.byref(p), 1, 1, 100, ctypes.byref(part), ctypes.byref(part), 1, 1, 1, 1, 1,
                         ctypes.byref(saved), 1, 1 << 30, None)
    assert st == code


def test_bin_rejects_bad_arguments_before_launching():
    lib = ssa.lib()
    part = ssa.Partition(1, 1, 1, 1, 1, 0)
    null = ssa.Partition(None, 1, 1, 1, 1, 0)
    assert lib.ssa_bin(1, 1, 1, 10, 64, 0, 4, ctypes.byref(part), ctypes.byref(part), 1, 1 << 20, None) == 1
    assert lib.ssa_bin(1, 1, 1, 10, 64, 4, 4, ctypes.byref(null), ctypes.byref(part), 1, 1 << 20, None) == 1
    assert lib.ssa_bin(1, 1, 1, 10, 1 << 21, 4, 4, ctypes.byref(part), ctypes.byref(part), 1, 1 << 20, None) == 1
    assert lib.ssa_bin(1, 1, 1, 10, 64, 4, 4, ctypes.byref(part), ctypes.byref(part), 1, 16, None) == 3
    # sequence bits + 3 x cell bits above 64: 2^20 grid with unit cells and 2^5 sequences
    assert lib.ssa_bin(1, 1, 32, 10, 1 << 20, 1, 1, ctypes.byref(part), ctypes.byref(part), 1, 1 << 30,
                       None) == 2


def test_geo_select_argument_errors_are_found_on_the_host():
    lib = ssa.lib()
    part = ssa.Partition(1, 1, 1, 1, 1, 10)
    assert lib.ssa_workspace_size(ssa.OP_GEO_SELECT, None, 1, 1000, 100, 0) >= 16 * 1000
    ok = dict(coords=1, cu=1, S=1, N=100, R=64, m=4, topk=8, hkv=2, sel=1, ws=1, ws_bytes=1 << 20)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.ssa_geo_select(a["coords"], a["cu"], a["S"], a["N"], a["R"], ctypes.byref(part), a["m"],
                                  a["topk"], a["hkv"], a["sel"], a["ws"], a["ws_bytes"], None)
    assert call(topk=0) == 1 and call(topk=33) == 1 and call(hkv=0) == 1 and call(m=0) == 1
    assert call(S=0) == 1 and call(N=-1) == 1 and call(sel=None) == 1
    assert call(R=40000) == 2                    # squared distances must fit 32 bits
    assert call(ws_bytes=100) == 3               # workspace too small
    assert call(N=0) == 0                        # nothing to do


def test_cross_attention_argument_errors_are_found_on_the_host():
    lib = ssa.lib()
    p = ssa.make_params(16, 2, 64, 8, 8, 16, torch.bfloat16, 1)
    part = ssa.Partition(1, 1, 1, 1, 1, 10)
    sv = ssa.Saved(1, 1, 1, 1, 1, 1, 1)
    need_f = ssa.workspace_size(ssa.OP_CROSS_FORWARD, p, 1, 1000, 10, 0)
    need_b = ssa.workspace_size(ssa.OP_CROSS_BACKWARD, p, 1, 1000, 10, 0)
    assert need_f > ssa.workspace_size(ssa.OP_FORWARD, p, 1, 1000, 10, 0) - 4096 and need_f > 3 * 1000 * 16 * 4
    assert need_b > 3 * 1000 * 16 * 4

    def fwd(S=1, nq=1000, nkv=500, ws_bytes=None, q=1):
        return lib.ssa_cross_forward(ctypes.byref(p), 1, S, nq, nkv, ctypes.byref(part), q, 1, 1, 1, 1,
                                     ctypes.byref(sv), 1, need_f if ws_bytes is None else ws_bytes, None)
    assert fwd(S=0) == 1 and fwd(nq=-1) == 1 and fwd(q=None) == 1
    assert fwd(nkv=5) == 1                       # fewer voxel tokens than blocks
    assert fwd(ws_bytes=need_f - 1) == 3
    assert fwd(nq=0) == 0                        # nothing to do
    bad = ssa.make_params(16, 2, 64, 8, 8, 16, torch.bfloat16, 1, selection=7)
    assert lib.ssa_cross_forward(ctypes.byref(bad), 1, 1, 10, 10, ctypes.byref(part), 1, 1, 1, 1, 1,
                                 ctypes.byref(sv), 1, need_f, None) == 1
    assert lib.ssa_cross_backward(ctypes.byref(p), 1, 1, 1000, 500, ctypes.byref(part), 1, 1, 1, 1,
                                  ctypes.byref(sv), 1, 1, 1, 1, 1, 1, need_b - 1, None) == 3


C_PROGRAM = r"""
#include "ssa.h"
#include <stdio.h>
int main(void) {
  ssa_params p = {0};
  p.hq = 32; p.hkv = 2; p.d = 64; p.m_cmp = 8; p.m_win = 8; p.topk = 16;
  p.dtype = SSA_DTYPE_BF16; p.gate_mode = SSA_GATE_LOGITS; p.selection = SSA_SEL_SCORES; p.conv = NULL;
  size_t f = ssa_workspace_size(SSA_OP_FORWARD, &p, 1, 131072, 2322, 2322);
  size_t c = ssa_workspace_size(SSA_OP_CROSS_FORWARD, &p, 1, 131072, 2322, 0);
  ssa_status s = ssa_forward(&p, NULL, 1, 10, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL);
  printf("%d %d %d %s\n", ssa_version(), f > 0 && c > f, (int)s, ssa_error_string(s));
  return 0;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    """The boundary is a C ABI: the header compiles as strict C99, a C program links
    against libssa.so and makes host-side calls (no GPU needed)."""
    import shutil
    import subprocess

    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.join(root, "spatial_sparse_attention_ssa_b200")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(root, "include"),
                        str(src), "-L", libdir, "-lssa", "-Wl,-rpath," + libdir, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    version, sizes_ok, status, *msg = out.stdout.split()
    assert int(version) == ssa.lib().ssa_version() and sizes_ok == "1"
    assert int(status) == 1 and " ".join(msg) == "invalid argument"  # null cu_seqlens found on the host
