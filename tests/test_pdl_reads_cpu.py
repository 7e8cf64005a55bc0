"""Kernels launched with programmatic dependent launch start while the
kernel before them still runs, so what that kernel writes may be read only
after griddepcontrol.wait and only through L2 (plain or __ldcg loads, TMA,
bulk copies): never with __ldg, and never through a const __restrict__
pointer, which lets the compiler serve the load from the read-only path or
issue it ahead of the wait.  A combine that read the decode kernel's work
count through such a pointer once returned without merging.  This checks the
sources of the kernels that read another kernel's output after a wait."""
import os
import re

CSRC = os.path.join(os.path.dirname(__file__), "..", "head_latent_attention_10_b200", "csrc")


def src(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def signature(text, kernel):
    """The parameter list of the kernel's definition."""
    i = text.index(kernel + "(")
    j = text.index(")", i)
    return text[i:j + 1]


def test_combine_reads_the_decode_outputs_without_restrict():
    sig = signature(src("dec_common.cuh"), "\ndec_combine_kernel")
    for p in ("plan", "flags", "part_o", "part_lse2"):
        decl = re.search(r"([^,(]*)\b" + p + r"\b", sig).group(1)
        assert "__restrict__" not in decl, (p, decl)


def test_decode_kernel_reads_its_inputs_without_ldg():
    text = src("tc_decode64.cuh") + src("dec_common.cuh")
    assert "__ldg(" not in text


def test_every_pdl_kernel_waits_before_its_reads():
    # the kernels mla_abi.cu launches with programmatic serialization
    abi = src("mla_abi.cu")
    launched = set(re.findall(r"launch_pdl\((\w+)", abi))
    assert {"dec_combine_kernel", "tc_decode64_kernel"} <= launched, launched
    for name, fn in (("dec_common.cuh", "dec_combine_kernel"), ("tc_decode64.cuh", "tc_decode64_kernel"),
                     ("tc_gemm.cuh", "tc_gemm_kernel")):
        text = src(name)
        body = text[text.index(fn + "("):]
        assert "pdl_wait()" in body[:body.index("\n}\n")], fn
