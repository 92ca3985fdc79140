"""GPU test of kda_chunk_fwd_noalloc, the prefill entry point for callers that
cannot allocate device memory (hosts that reserve the whole GPU up front, or
plugin interfaces without an allocator).  It runs on a fixed scratch array
inside the library, so this test makes two calls in a row on each input -- the
second one finding the first one's data still in the shared scratch -- and
checks that each matches the fp64 oracle within the parity tolerance, that the
two are bit-identical, that the calls change the device's free memory by nothing,
and that a problem too large for the scratch is refused before anything runs.
The file name sorts last so a stop-at-first-failure run has already run every
other test."""
import ctypes

import pytest
import torch

import workloads as W
from kda_testutil import TOL, oracle_prefill, rel

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


def _outputs(inp):
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    return (torch.full((B, T, H, dv), float("nan"), dtype=q.dtype, device="cuda"),
            torch.full((N, H, dk, dv), float("nan"), dtype=torch.float32, device="cuda"))


def _call(lib, fn, inp, io, bufs=None):
    q = inp["q"]
    B, T, H, dk = q.shape
    dv = inp["v"].shape[-1]
    cu = inp["cu_seqlens"]
    N = B if cu is None else cu.numel() - 1
    out, hT = bufs if bufs is not None else _outputs(inp)
    st = fn(_p(q), _p(inp["k"]), _p(inp["v"]), _p(inp["log_alpha"]), _p(inp["beta"]),
            _p(inp["h0"]), _p(out), _p(hT), _p(cu), N, T, H, dk, dv,
            ctypes.c_float(inp["scale"]), io, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, out, hT


def test_noalloc_matches_oracle_twice_in_a_row(lib):
    cases = [
        (W.small_prefill(H=3, dk=128, dv=128, io_dtype="bf16", seed=21, h0_std=0.05,
                         lengths=[130, 1, 64, 0, 77]), 1),
        (W.small_prefill(B=2, T=200, H=2, dk=64, dv=128, io_dtype="f32", seed=22, h0_std=0.05), 0),
    ]
    for cfg, io in cases:
        inp = W.make_prefill(cfg, "cuda")
        ro, rh = oracle_prefill(inp)
        _call(lib, lib.kda_chunk_fwd_noalloc, inp, io)        # loads the kernels
        bufs_a, bufs_b = _outputs(inp), _outputs(inp)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        st_a, out_a, hT_a = _call(lib, lib.kda_chunk_fwd_noalloc, inp, io, bufs_a)
        st_b, out_b, hT_b = _call(lib, lib.kda_chunk_fwd_noalloc, inp, io, bufs_b)
        free1, _ = torch.cuda.mem_get_info()
        assert st_a == 0 and st_b == 0, (st_a, st_b)
        # the outputs exist before free0 is read; the calls allocate nothing
        assert free1 == free0, (free0, free1)
        for out, hT in ((out_a, hT_a), (out_b, hT_b)):
            assert torch.isfinite(out.float()).all() and torch.isfinite(hT).all()
            assert rel(out, ro) <= TOL[cfg.io_dtype], rel(out, ro)
            assert rel(hT, rh) <= TOL[cfg.io_dtype], rel(hT, rh)
        assert torch.equal(out_a, out_b) and torch.equal(hT_a, hT_b)


def test_noalloc_refuses_problems_larger_than_its_scratch(lib):
    # 512 chunks of one head at dk = dv = 128 need about 74 MB > 64 MiB of scratch;
    # the refusal happens on the host, before any launch (pointers are never read)
    fake = 0x7f0000000000
    st = lib.kda_chunk_fwd_noalloc(fake, fake + 16, fake + 32, fake + 48, fake + 64, None,
                                   fake + 80, None, None, 1, 512 * 64, 1, 128, 128,
                                   ctypes.c_float(0.1), 1, None)
    assert st == 2      # KDA_ERR_UNSUPPORTED
