"""Kernels launched as programmatic dependents (CPU, source-level).

A kernel launched with programmatic stream serialization may start while the
kernel before it in the stream is still running, so it must wait for it
(griddepcontrol.wait) before using what that kernel wrote, and it releases the
kernel after it (griddepcontrol.launch_dependents).  This test finds every
kernel the library launches that way and checks that its body does both."""
import os
import re

CSRC = os.path.join(os.path.dirname(__file__), os.pardir, "causal_kernelized_sequence_b200", "csrc")


def _read(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def _pdl_kernels(api):
    names = set(re.findall(r"launch_pdl\(\s*([A-Za-z_]\w*)", api))
    names.discard("void")          # the helper's own declaration
    names.discard("kernel")        # the decode dispatch lambda's parameter
    names |= set(re.findall(r"\bgo\(\s*([A-Za-z_]\w*)", api))
    return names


def _kernel_body(src, name):
    """Text of the body of the __global__ function `name`, or None."""
    m = re.search(r"__global__[^;{]*?\b" + re.escape(name) + r"\s*\(", src, re.S)
    if not m:
        return None
    i = src.index("{", m.end())
    depth = 0
    for j in range(i, len(src)):
        if src[j] == "{":
            depth += 1
        elif src[j] == "}":
            depth -= 1
            if depth == 0:
                return src[i:j + 1]
    return None


def test_every_dependent_launch_waits_and_releases():
    api = _read("la_api.cu")
    kernels = _pdl_kernels(api)
    assert {"fwd_split_state_kernel", "fwd_split_out_kernel", "fwd_tc_kernel", "swa_fwd_tc_kernel",
            "decode_vec_kernel", "swa_decode64_kernel"} <= kernels, kernels
    sources = "".join(_read(f) for f in sorted(os.listdir(CSRC)) if f.endswith(".cuh"))
    for k in sorted(kernels):
        body = _kernel_body(sources, k)
        assert body is not None, k
        assert "grid_dependency_wait()" in body, k
        assert "launch_dependents()" in body, k


def test_one_launch_path_for_dependents():
    """The tensor-core forward and decode kernels are not launched with <<<>>>,
    which would drop the launch attribute."""
    api = _read("la_api.cu")
    for k in ("fwd_split_state_kernel", "fwd_split_out_kernel", "fwd_tc_kernel", "swa_fwd_tc_kernel",
              "decode_vec_kernel", "swa_decode64_kernel"):
        assert not re.search(re.escape(k) + r"[^;(]*<<<", api), k
