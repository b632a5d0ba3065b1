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


def test_clock_sampler_names_the_gpu_by_uuid_or_bus_id():
    # nvidia-smi ignores CUDA_VISIBLE_DEVICES: the sampled GPU must be named by
    # something that does not depend on the visible-device numbering
    import types

    sys.path.insert(0, ROOT)
    import bench

    props = types.SimpleNamespace(uuid="1c0ffee0-0000-4000-8000-000000000001", pci_domain_id=0,
                                  pci_bus_id=0x1B, pci_device_id=0)
    assert bench.smi_device_id(props) == "GPU-1c0ffee0-0000-4000-8000-000000000001"
    props.uuid = "GPU-abc"
    assert bench.smi_device_id(props) == "GPU-abc"
    props.uuid = ""
    assert bench.smi_device_id(props) == "00000000:1b:00.0"
