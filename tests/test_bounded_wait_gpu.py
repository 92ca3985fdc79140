"""The library's bounded device waits (the suspended and the spinning poll), through
the C ABI: a wait on an mbarrier that nothing completes gives up at its limit, is
reported as KDA_ERR_TIMEOUT with a timeout bit in the error word, takes bounded time,
and leaves the context usable (a prefill right after it still matches the fp64
oracle).  These are the waits every kernel uses on its copies, MMAs and warp
hand-offs; nothing here faults or hangs."""
import time

import pytest
import torch

import workloads as W
from kda_testutil import TOL, oracle_prefill, rel

pytestmark = pytest.mark.gpu

TIMEOUT_BITS = 0x7E          # bits 1-6 of the device error word


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


@pytest.mark.parametrize("polls", [1, 40])
def test_wait_that_runs_out_is_reported_and_bounded(kda, polls):
    torch.cuda.synchronize()
    t = time.perf_counter()
    st, word = kda.debug_bounded_wait(polls)
    dt = time.perf_counter() - t
    print(f"bounded wait: polls={polls} status={st} word={word:#x} {dt * 1e3:.2f} ms")
    assert st == kda.KDA_ERR_TIMEOUT, st
    assert word == 0x6, hex(word)             # both waits gave up: suspended and spinning
    assert dt < 1.0, dt                       # at most ~0.1 ms per poll, plus launch


def test_context_usable_after_a_wait_ran_out(kda):
    st, _ = kda.debug_bounded_wait(5)
    assert st == kda.KDA_ERR_TIMEOUT
    cfg = W.small_prefill(B=2, T=130, H=2, dk=128, dv=128, io_dtype="bf16", seed=21, h0_std=0.02)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"])
    torch.cuda.synchronize()
    ro, rh = oracle_prefill(inp)
    assert rel(out, ro) <= TOL["bf16"] and rel(hT, rh) <= TOL["bf16"]
