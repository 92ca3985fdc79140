"""Source rules of the library's launches, checked on the host.

A kernel launched with programmatic stream serialization (launch_pdl) may start
while the kernel before it on the stream is still running, so its first statement
(compile-time declarations aside) must be griddep_wait(): nothing may read an input
or overwrite a buffer before the previous grid has completed.  This test finds every kernel named in a launch_pdl
call and checks the first statement of its definition."""
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "gated_delta_rule_75_b200", "csrc")


def _sources():
    out = {}
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, name)) as f:
                out[name] = f.read()
    return out


def _strip_comments(text):
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def _pdl_kernels(srcs):
    names = set()
    for text in srcs.values():
        for m in re.finditer(r"launch_pdl\(\s*([A-Za-z_:][\w:]*)", _strip_comments(text)):
            names.add(m.group(1).split("::")[-1])
    names.discard("void")     # the helper's own declaration, if matched
    return names


COMPILE_TIME = ("constexpr ", "static_assert", "using ")


def _first_statement(srcs, kernel):
    """The first statement of the __global__ definition of `kernel` that is not a
    compile-time declaration (constexpr constants, static_assert, using)."""
    for text in srcs.values():
        code = _strip_comments(text)
        for m in re.finditer(r"__global__[^;{]*?\b" + re.escape(kernel) + r"\s*\(", code):
            depth, i = 1, m.end()
            while depth:                          # skip the parameter list
                depth += {"(": 1, ")": -1}.get(code[i], 0)
                i += 1
            rest = code[code.index("{", i) + 1:]
            while True:
                stmt, rest = rest.lstrip().split(";", 1)
                if not stmt.strip().startswith(COMPILE_TIME):
                    return stmt.strip()
    return None


def test_every_pdl_kernel_waits_first():
    srcs = _sources()
    kernels = _pdl_kernels(srcs)
    assert {"chunk_prep_tc_kernel", "chunk_state_tc_kernel", "affine_prefix_kernel",
            "chunk_prep_simt_kernel", "chunk_state_simt_kernel", "chunk_offsets_kernel"} <= kernels
    for k in sorted(kernels):
        first = _first_statement(srcs, k)
        assert first is not None, "no __global__ definition found for " + k
        assert first == "griddep_wait()", (k, first)


def test_rule_check_catches_a_late_wait():
    """The check itself: a kernel that reads memory before its wait is reported."""
    srcs = {"x.cu": "__global__ void bad_kernel(const int* p, int* q)\n{\n    int v = *p;\n"
                    "    griddep_wait();\n    *q = v;\n}\n"
                    "void go() { launch_pdl(bad_kernel, 1, 1, 0, 0, p, q); }\n"}
    assert _pdl_kernels(srcs) == {"bad_kernel"}
    assert _first_statement(srcs, "bad_kernel") == "int v = *p"
    srcs["x.cu"] = srcs["x.cu"].replace("{\n    int v", "{\n    constexpr int n = 4;\n    int v")
    assert _first_statement(srcs, "bad_kernel") == "int v = *p"
