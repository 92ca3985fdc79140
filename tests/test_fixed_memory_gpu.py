"""Fixed-size state, measured as memory (the pages measure peak memory while the
context grows and credit KDA's fixed-size recurrent state for its flat memory
use).  Through the C ABI (kda_workspace_high_water, the library pool's
used-memory high-water mark): the fused tensor-core prefill's workspace (the
default with many chains) does not change as T doubles; the two-kernel
tensor-core and SIMT forms (and the default with few chains) grow in proportion
to the chunk count; under a small workspace budget the SIMT form stays
under the budget as T grows (heads run in groups); and the decode step allocates
nothing, neither from the library's pool nor anywhere on the device."""
import os
import subprocess
import sys

import pytest
import torch

import workloads as W
from kda_testutil import TOL, oracle_prefill, rel

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def _high_water(kda, cfg, impl):
    inp = W.make_prefill(cfg, "cuda")
    torch.cuda.synchronize()
    kda.workspace_high_water(reset=True)
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], impl=impl)
    torch.cuda.synchronize()
    return kda.workspace_high_water(), inp, out, hT


@pytest.mark.parametrize("varlen", [False, True])
def test_fused_prefill_workspace_does_not_grow_with_T(kda, varlen):
    """96 chains (more than half the SMs): AUTO runs the fused kernel alone."""
    marks = []
    for T in (1024, 2048, 4096):
        if varlen:
            cfg = W.small_prefill(H=24, dk=128, dv=128, io_dtype="bf16", seed=40,
                                  lengths=[T // 2, 1, T, T // 2 - 1])
        else:
            cfg = W.small_prefill(B=2, T=T, H=48, dk=128, dv=128, io_dtype="bf16", seed=40)
        hw, inp, out, hT = _high_water(kda, cfg, "auto")
        marks.append(hw)
        if T == 1024:
            ro, rh = oracle_prefill(inp)
            assert rel(out, ro) <= TOL["bf16"] and rel(hT, rh) <= TOL["bf16"]
    print("fused workspace high water:", marks)
    assert marks[0] == marks[1] == marks[2], marks
    assert 0 < marks[0] <= 4 << 20, marks


@pytest.mark.parametrize("impl,io", [("tensorcore_chain", "bf16"), ("simt", "f32"),
                                     ("auto", "bf16")])
def test_two_kernel_workspace_grows_with_chunk_count(kda, impl, io):
    """8 chains: under AUTO too the two-kernel form runs first (few chains)."""
    marks = []
    for T in (1024, 2048, 4096):
        cfg = W.small_prefill(B=2, T=T, H=4, dk=128, dv=128, io_dtype=io, seed=41)
        hw, *_ = _high_water(kda, cfg, impl)
        marks.append(hw)
    print(impl, "workspace high water:", marks)
    # affine in the chunk count: each doubling of T adds twice what the one before added
    # (the operand images or fp32 blocks; the segment buffers of the segmented walk and
    # the header do not grow)
    d1, d2 = marks[1] - marks[0], marks[2] - marks[1]
    assert d1 > 0 and 1.8 <= d2 / d1 <= 2.2, marks


CHILD = r"""
import sys, torch
sys.path.insert(0, ROOT)
import workloads as W
import gated_delta_rule_75_b200 as kda
marks = []
for T in (4096, 8192, 16384):
    cfg = W.small_prefill(B=1, T=T, H=16, dk=128, dv=128, io_dtype="f32", seed=42)
    inp = W.make_prefill(cfg, "cuda")
    torch.cuda.synchronize()
    kda.workspace_high_water(reset=True)
    kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                  impl="simt")
    torch.cuda.synchronize()
    marks.append(kda.workspace_high_water())
print("capped", marks)
assert all(0 < m <= (64 << 20) + (2 << 20) for m in marks), marks
print("budget ok")
"""


def test_workspace_stays_under_budget_as_T_grows(kda):
    env = dict(os.environ, KDA_WORKSPACE_MB="64")
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "budget ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


def test_decode_allocates_nothing(kda):
    dcfg = W.DecodeConfig("mem", N=64, H=8, dk=128, dv=128, steps=16, seed=43)
    gen = W.decode_generator(dcfg, "cuda")
    S = W.make_decode_state(dcfg, gen, "cuda")
    xs = [W.make_decode_step(dcfg, gen, "cuda") for _ in range(dcfg.steps)]
    o = torch.empty((dcfg.N, dcfg.H, dcfg.dv), dtype=torch.bfloat16, device="cuda")
    kda.recurrent_step(xs[0]["q"], xs[0]["k"], xs[0]["v"], xs[0]["log_alpha"], xs[0]["beta"],
                       S, 0.088, out=o)        # first call loads the kernels
    torch.cuda.synchronize()
    kda.workspace_high_water(reset=True)
    torch.cuda.reset_peak_memory_stats()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for x in xs[1:]:
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, 0.088, out=o)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert kda.workspace_high_water() == 0
    assert torch.cuda.max_memory_allocated() == alloc0
    assert free1 == free0, (free0, free1)
