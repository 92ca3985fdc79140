"""GPU test of kda_chunk_fwd_noalloc, the prefill entry point for callers that
cannot allocate device memory (hosts that reserve the whole GPU up front, or
plugin interfaces without an allocator).  It runs on a fixed scratch array
inside the library, so this test checks that two calls in a row -- the second
one finding the first one's data still in the shared scratch -- each match
the ordinary allocating entry point kda_chunk_fwd within the parity
tolerance, and that a problem too large for the scratch is refused before
anything runs.  The file name sorts last so a stop-at-first-failure run has
already run every other test."""
import ctypes

import pytest
import torch

import workloads as W
from kda_testutil import TOL, host, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    lib = kda._load()
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.kda_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                          i64, ctypes.c_float, ctypes.c_int, vp]
    lib.kda_chunk_fwd_noalloc.restype = ctypes.c_int
    return lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call(lib, fn, inp, io):
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    out = torch.full((B, T, H, dv), float("nan"), dtype=q.dtype, device="cuda")
    hT = torch.full((N, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda")
    st = fn(_p(q), _p(inp["k"]), _p(inp["v"]), _p(inp["log_alpha"]), _p(inp["beta"]),
            _p(inp["h0"]), _p(out), _p(hT), _p(cu), N, T, H, dk, dv,
            ctypes.c_float(inp["scale"]), io, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, out, hT


def test_noalloc_matches_allocating_entry_point_twice(lib):
    cases = [
        (W.small_prefill(H=3, dk=128, dv=128, io_dtype="bf16", seed=21, h0_std=0.05,
                         lengths=[130, 1, 64, 0, 77]), 1),
        (W.small_prefill(B=2, T=200, H=2, dk=64, dv=128, io_dtype="f32", seed=22, h0_std=0.05), 0),
    ]
    for cfg, io in cases:                    # two calls in a row on the shared scratch
        inp = W.make_prefill(cfg, "cuda")
        st_a, out_a, hT_a = _call(lib, lib.kda_chunk_fwd_noalloc, inp, io)
        assert st_a == 0, st_a
        st_b, out_b, hT_b = _call(lib, lib.kda_chunk_fwd, inp, io)
        assert st_b == 0, st_b
        assert torch.isfinite(out_a.float()).all() and torch.isfinite(hT_a).all()
        assert rel(out_a, host(out_b).double().numpy()) <= TOL[cfg.io_dtype]
        assert rel(hT_a, host(hT_b).double().numpy()) <= TOL[cfg.io_dtype]


def test_noalloc_refuses_problems_larger_than_its_scratch(lib):
    # 512 chunks of one head at dk = dv = 128 need about 74 MB > 64 MiB of scratch;
    # the refusal happens on the host, before any launch (pointers are never read)
    fake = 0x7f0000000000
    st = lib.kda_chunk_fwd_noalloc(fake, fake + 16, fake + 32, fake + 48, fake + 64, None,
                                   fake + 80, None, None, 1, 512 * 64, 1, 128, 128,
                                   ctypes.c_float(0.1), 1, None)
    assert st == 2      # KDA_ERR_UNSUPPORTED
