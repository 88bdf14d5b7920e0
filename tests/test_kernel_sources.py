"""Source-level invariants of the CUDA kernels that no GPU run can show reliably.

The layer's kernels are launched with programmatic dependent launch, so a
kernel may be scheduled while its predecessor in the stream is still running.
That is only safe because every kernel waits on the device for the predecessor
(`griddepcontrol.wait`) before its first global-memory access. These tests pin
that: each kernel's body starts with the wait, and every launch goes through
the helper that sets the attribute (the self-test kernel, launched plainly, is
the one exception)."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "expert_routing_grouped_layer_b200", "csrc")
PLAIN = {"selftest.cu"}  # launched without the attribute, on its own


def kernels():
    out = []
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        text = open(path).read()
        for m in re.finditer(r"__global__ void", text):
            body = text.index("{", m.end())
            sig = re.sub(r"__launch_bounds__\([^)]*\)", "", text[m.end():body])
            name = re.search(r"(\w+)\s*\(", sig).group(1)
            out.append((os.path.basename(path), name, text[body + 1:body + 200]))
    return out


def test_every_layer_kernel_waits_first():
    ks = [k for k in kernels() if k[0] not in PLAIN]
    assert len(ks) >= 18
    for f, name, body in ks:
        first = [s.strip() for s in body.split(";")[:2]]
        assert first == ["pdl_wait()", "pdl_trigger()"], (f, name, first)


def test_every_launch_sets_the_attribute():
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        if os.path.basename(path) in PLAIN:
            continue
        text = re.sub(r"//[^\n]*", "", open(path).read())
        assert "<<<" not in text, os.path.basename(path)


def test_launch_helper_sets_programmatic_serialization():
    text = open(os.path.join(CSRC, "sm100.cuh")).read()
    helper = text[text.index("inline cudaError_t launch_pdl("):]
    helper = helper[:helper.index("\n}\n")]
    assert "cudaLaunchAttributeProgrammaticStreamSerialization" in helper
    assert "programmaticStreamSerializationAllowed = 1" in helper
    assert re.search(r'griddepcontrol\.wait;', text)
