"""The wait profiler's source instrumentation (CPU): it finds the four compressed
kernels, wraps every pipeline wait of each, and leaves the rest of the source as is."""
import os
import re

from spatial_sparse_attention_ssa_b200 import build as B
from spatial_sparse_attention_ssa_b200 import waitprof


def test_every_pipeline_wait_of_the_four_kernels_is_wrapped():
    with open(os.path.join(B.CSRC, "cmp_tc.cu")) as f:
        src = f.read()
    text, slots = waitprof.instrument(src)
    kernels = {v[0] for v in slots.values()}
    assert kernels == {k[:-1] for k in waitprof.KERNELS}
    assert text.count("PW(") == len(slots) + 1  # the sites and the macro's own definition
    for slot, (_, line, call) in slots.items():
        assert "PW(%d, %s)" % (slot, call) in text
        assert call in src.split("\n")[line - 1]
    # nothing but the wrapping, the counters and the reader differ
    stripped = re.sub(r"PW\(\d+, (mbar_wait(?:_warp)?\()", r"\1", text)
    assert "ssa_waitprof_read" in text and text.count("_tk0") == 2 * len(waitprof.KERNELS)
    assert len(stripped) > len(src)
