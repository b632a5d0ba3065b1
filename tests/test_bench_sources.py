"""bench.py trusts a committed ncu traffic record only while the sources the
tensor-core forward is compiled from are unchanged (a hash over TC_SOURCES).
That list must hold every file of the kernel directory that tc_forward.cu
includes, directly or through another included file."""
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kernelized_linear_attention_fwd_b200", "csrc")


def local_includes(fn, seen):
    if fn in seen:
        return seen
    seen.add(fn)
    for inc in re.findall(r'#include\s+"([^"]+)"', open(os.path.join(CSRC, fn)).read()):
        if os.path.dirname(inc) == "" and os.path.exists(os.path.join(CSRC, inc)):
            local_includes(inc, seen)
    return seen


def test_traffic_hash_covers_every_source_of_the_tensor_core_forward():
    sys.path.insert(0, ROOT)
    import bench

    assert local_includes("tc_forward.cu", set()) <= set(bench.TC_SOURCES)
    assert all(os.path.exists(os.path.join(CSRC, f)) for f in bench.TC_SOURCES)
