"""GPU edge cases of the chunkwise prefill: heads processed in several
workspace groups (forced small workspace budget, in a child process since the
budget is read once per process), hT written over h0 in place, and malformed
cu_seqlens (reported in debug mode; offsets are clamped on the device, so the
call never reads or writes out of bounds)."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import workloads as W
from kda_testutil import TOL, host, oracle_prefill, rel

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


@pytest.mark.parametrize("impl,shift", [("simt", 0.0), ("tensorcore_chain", 0.0),
                                        ("tensorcore_fused", 0.0), ("auto", 8.0)])
def test_head_groups_with_small_workspace(cuda_ok, impl, shift):
    """64 MiB budget: 512 chunks per head need about 34 MB (two-kernel tensor-core
    path) or 76 MB (SIMT), so the three heads run in separate groups; the fused
    kernel needs no per-chunk workspace and runs them in one launch.  AUTO with its
    12 chains would take the two-kernel form first, but not when the heads need
    several groups: here, at a decay (about e^-8 per token) that form's prep would
    flag, with the final states written over the initial ones in place, it runs the
    fused kernel alone."""
    code = textwrap.dedent(f"""
        import sys; sys.path.insert(0, {ROOT!r}); sys.path.insert(0, {os.path.join(ROOT, 'tests')!r})
        import workloads as W, gated_delta_rule_75_b200 as kda, torch
        from kda_testutil import TOL, oracle_prefill, rel
        cfg = W.small_prefill(B=4, T=8192, H=3, dk=128, dv=128, io_dtype="bf16", seed=31, h0_std=0.02,
                              gate_shift={shift!r})
        inp = W.make_prefill(cfg, "cuda")
        ro, rh = oracle_prefill(inp)
        state = inp["h0"].clone()
        kda.profiler_read(reset=True)
        out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                inp["scale"], h0=state, hT=state, impl={impl!r})
        torch.cuda.synchronize()
        st = kda.profiler_read(reset=True)
        if {impl!r} == "auto":
            assert st.get("chunk_prep_tc", (0,))[0] == 0 and st["chunk_fused_tc"][0] == 1, st
        eo, eh = rel(out, ro), rel(state, rh)
        print(eo, eh)
        assert eo <= TOL["bf16"] and eh <= TOL["bf16"], (eo, eh)
    """)
    env = dict(os.environ, KDA_WORKSPACE_MB="64", KDA_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr


@pytest.mark.parametrize("impl,io", [("simt", "f32"), ("tensorcore", "bf16"),
                                     ("tensorcore_chain", "bf16")])
def test_final_state_written_over_initial_state(kda, impl, io):
    cfg = W.small_prefill(B=2, T=130, H=2, dk=128, dv=128, io_dtype=io, seed=32, h0_std=0.05)
    inp = W.make_prefill(cfg, "cuda")
    ro, rh = oracle_prefill(inp)
    state = inp["h0"].clone()
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=state, hT=state, impl=impl)
    torch.cuda.synchronize()
    assert hT.data_ptr() == state.data_ptr()
    assert rel(out, ro) <= TOL[io] and rel(state, rh) <= TOL[io]


@pytest.mark.parametrize("impl", ["simt", "tensorcore", "tensorcore_chain"])
@pytest.mark.parametrize("cu", [[0, 100, 50, 200], [0, 200, 0, 200], [0, 64, 300, 200], [5, 64, 128, 200]])
def test_malformed_offsets_are_reported_not_faulted(kda, impl, cu):
    cfg = W.small_prefill(H=2, dk=128, dv=128, io_dtype="bf16", seed=33, lengths=[64, 64, 72])
    inp = W.make_prefill(cfg, "cuda")
    inp["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device="cuda")
    with pytest.raises(kda.KDAError) as e:
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                      cu_seqlens=inp["cu_seqlens"], impl=impl)
    assert e.value.status == kda.KDA_ERR_INVALID_ARG
    # the context is still healthy
    x = torch.ones(4, device="cuda") * 2
    assert float(x.sum()) == 8.0


@pytest.mark.parametrize("H", [4, 6, 9])
def test_many_heads_and_side_stream(kda, H):
    """More heads, and the same call on a side stream gives identical results."""
    cfg = W.small_prefill(B=2, T=300, H=H, dk=128, dv=128, io_dtype="bf16", seed=40 + H, h0_std=0.02)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"])
    torch.cuda.synchronize()
    ro, rh = oracle_prefill(inp)
    assert rel(out, ro) <= TOL["bf16"] and rel(hT, rh) <= TOL["bf16"]
    # and on a side stream, ordered after work queued there
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out2 = torch.zeros_like(out)
        out2, hT2 = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                  inp["scale"], h0=inp["h0"], out=out2)
    s.synchronize()
    torch.testing.assert_close(out2, out, rtol=0, atol=0)
    torch.testing.assert_close(hT2, hT, rtol=0, atol=0)
