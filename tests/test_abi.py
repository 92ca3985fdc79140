"""C-ABI checks that need no GPU: the library loads, exports every function
include/kda.h declares, and rejects bad arguments on the host before any CUDA
call (status codes, never a crash)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda._load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_\s\*]*?\b(kda_[a-z0-9_]+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_the_boundary():
    fns = declared_functions()
    for name in ("kda_chunk_fwd", "kda_chunk_fwd_ex", "kda_recurrent_step", "kda_status_string",
                 "kda_version"):
        assert name in fns, fns


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(6):
        s = lib.kda_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.kda_status_string(99) == b"unknown status"
    assert lib.kda_version() >= 100


FAKE = 0x7f0000000000   # 16-byte aligned, never dereferenced: checks run on the host


def _fwd(lib, q=FAKE, k=FAKE + 16, v=FAKE + 32, g=FAKE + 48, b=FAKE + 64, h0=None, out=FAKE + 80,
         hT=None, cu=None, B=1, T=64, H=2, dk=128, dv=128, io=1, impl=0):
    return lib.kda_chunk_fwd_ex(q, k, v, g, b, h0, out, hT, cu, B, T, H, dk, dv,
                                ctypes.c_float(0.1), io, impl, None)


def _step(lib, q=FAKE, k=FAKE + 16, v=FAKE + 32, g=FAKE + 48, b=FAKE + 64, s=FAKE + 80,
          out=FAKE + 96, N=4, H=2, dk=128, dv=128, io=1):
    return lib.kda_recurrent_step(q, k, v, g, b, s, out, N, H, dk, dv, ctypes.c_float(0.1), io, None)


def test_prefill_argument_errors(lib):
    import gated_delta_rule_75_b200 as kda
    assert _fwd(lib, dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, dv=256) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, io=7) == kda.KDA_ERR_UNSUPPORTED
    assert _fwd(lib, impl=9) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(lib, B=-1) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(lib, T=-5) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(lib, b=None) == kda.KDA_ERR_INVALID_ARG
    assert _fwd(lib, b=FAKE + 66) == kda.KDA_ERR_INVALID_ARG         # beta not 4-byte aligned
    assert _fwd(lib, q=FAKE + 2) == kda.KDA_ERR_INVALID_ARG          # misaligned
    assert _fwd(lib, out=FAKE) == kda.KDA_ERR_INVALID_ARG            # out aliases q
    assert _fwd(lib, h0=FAKE + 8) == kda.KDA_ERR_INVALID_ARG         # misaligned h0
    assert _fwd(lib, cu=FAKE + 2) == kda.KDA_ERR_INVALID_ARG         # misaligned cu_seqlens
    assert _fwd(lib, cu=FAKE + 128, B=0) == kda.KDA_ERR_INVALID_ARG  # varlen needs B >= 1
    assert _fwd(lib, H=70000) == kda.KDA_ERR_UNSUPPORTED
    # empty batch / no heads: nothing to do, no CUDA call
    assert _fwd(lib, B=0) == kda.KDA_OK
    assert _fwd(lib, H=0) == kda.KDA_OK


def test_decode_argument_errors(lib):
    import gated_delta_rule_75_b200 as kda
    assert _step(lib, dk=32) == kda.KDA_ERR_UNSUPPORTED
    assert _step(lib, io=3) == kda.KDA_ERR_UNSUPPORTED
    assert _step(lib, N=-1) == kda.KDA_ERR_INVALID_ARG
    assert _step(lib, s=None) == kda.KDA_ERR_INVALID_ARG
    assert _step(lib, out=FAKE + 80) == kda.KDA_ERR_INVALID_ARG      # out aliases state
    assert _step(lib, v=FAKE + 40) == kda.KDA_ERR_INVALID_ARG        # misaligned
    assert _step(lib, b=FAKE + 66) == kda.KDA_ERR_INVALID_ARG        # beta not 4-byte aligned
    assert _step(lib, N=0) == kda.KDA_OK


def test_python_binding_checks_shapes_on_host():
    import torch
    import gated_delta_rule_75_b200 as kda
    q = torch.zeros(1, 8, 2, 64)
    with pytest.raises(ValueError):
        kda.chunk_fwd(q, q, q, q, torch.zeros(1, 8, 3), 0.1)
    with pytest.raises(TypeError):
        kda.chunk_fwd(q.double(), q.double(), q.double(), q, torch.zeros(1, 8, 2), 0.1)


def test_bounded_wait_selftest_argument_errors(lib):
    import gated_delta_rule_75_b200 as kda
    # (a NULL word is valid: the bits then go to the library's error word)
    for polls, word in ((0, FAKE), (20001, FAKE), (0, None), (10, FAKE + 2)):
        assert lib.kda_debug_bounded_wait(polls, word, None) == kda.KDA_ERR_INVALID_ARG


def test_error_word_and_high_water_argument_errors(lib):
    import gated_delta_rule_75_b200 as kda
    # NULL destinations are refused before any CUDA call
    assert lib.kda_get_error(None, None) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_workspace_high_water(None, 0) == kda.KDA_ERR_INVALID_ARG
