"""GPU parity of the chunkwise backward (kda_chunk_bwd through the C ABI)
against the oracle's fp64 token-by-token reverse mode: every gradient
(q, k, v, log_alpha, beta, h0), ragged tails, several chunks, every head
size, packed sequences with an empty one, no final-state gradient, and the
full-length 16-head workload on sampled pairs."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from kda_testutil import host, rel

pytestmark = pytest.mark.gpu

NAMES = ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dh0")


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def _upstream(cfg, inp, seed, with_dhT=True):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    io = inp["q"].dtype
    dout = torch.randn((cfg.B, cfg.T, cfg.H, cfg.dv), generator=gen, device="cuda").to(io)
    dhT = (torch.randn((cfg.N, cfg.H, cfg.dk, cfg.dv), generator=gen, device="cuda")
           if with_dhT else None)
    return dout, dhT


def _check(kda, cfg, seed=0, with_dhT=True, tol=None):
    inp = W.make_prefill(cfg, "cuda")
    dout, dhT = _upstream(cfg, inp, seed, with_dhT)
    got = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                        dout, h0=inp["h0"], dhT=dhT, cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    cu = None if inp["cu_seqlens"] is None else host(inp["cu_seqlens"]).numpy()
    ref = oracle.bwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                     host(inp["beta"]), inp["scale"], host(dout), h0=host(inp["h0"]),
                     dhT=host(dhT), cu_seqlens=cu)
    errs = {name: rel(g, r) for name, g, r in zip(NAMES, got, ref)}
    print(f"PARITY bwd {cfg.name} " + " ".join(f"{k}={v:.3e}" for k, v in errs.items()))
    if tol is not None:
        for name, e in errs.items():
            assert e <= tol[name], (cfg.name, name, e, tol[name])
    return errs


# fp32 I/O: every gradient at the fp32 bar; bf16 I/O: dq, dk, dv are rounded
# to bf16 (about 1.1e-3 rel-L2 by themselves), the fp32 gradients keep fp32
# arithmetic on the same rounded inputs
TOL = {"f32": dict.fromkeys(NAMES, 1e-5),
       "bf16": {"dq": 5e-3, "dk": 5e-3, "dv": 5e-3, "dlog_alpha": 1e-5, "dbeta": 1e-5,
                "dh0": 1e-5}}


@pytest.mark.parametrize("T", [1, 64, 150])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_backward_fp32(kda, T, dk, dv):
    cfg = W.small_prefill(B=2, T=T, H=2, dk=dk, dv=dv, io_dtype="f32", seed=200 + T, h0_std=0.05)
    _check(kda, cfg, seed=T, tol=TOL["f32"])


@pytest.mark.parametrize("T", [64, 300])
def test_backward_bf16(kda, T):
    cfg = W.small_prefill(B=2, T=T, H=2, dk=128, dv=128, io_dtype="bf16", seed=210 + T,
                          h0_std=0.02)
    _check(kda, cfg, seed=T, tol=TOL["bf16"])


def test_backward_packed_and_no_state_gradient(kda):
    cfg = W.small_prefill(H=2, dk=64, dv=64, io_dtype="f32", seed=220, h0_std=0.05,
                          lengths=[70, 0, 1, 128, 33])
    _check(kda, cfg, seed=5, with_dhT=False, tol=TOL["f32"])


def test_backward_without_dh0(kda):
    cfg = W.small_prefill(B=1, T=100, H=1, dk=64, dv=64, io_dtype="f32", seed=230)
    inp = W.make_prefill(cfg, "cuda")
    dout, dhT = _upstream(cfg, inp, 1)
    got = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                        dout, dhT=dhT, need_dh0=False)
    torch.cuda.synchronize()
    assert got[5] is None
    ref = oracle.bwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                     host(inp["beta"]), inp["scale"], host(dout), dhT=host(dhT))
    for g, r in zip(got[:5], ref[:5]):
        assert rel(g, r) <= 1e-5


def _full_size(kda, cfg, pairs):
    """GPU backward on the whole workload; oracle on the listed (sequence, head)
    pairs (each run alone, h0 and dhT sliced)."""
    inp = W.make_prefill(cfg, "cuda")
    dout, dhT = _upstream(cfg, inp, 17)
    got = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                        dout, h0=inp["h0"], dhT=dhT)
    torch.cuda.synchronize()
    worst = dict.fromkeys(NAMES, 0.0)
    for n, h in pairs:
        sl = lambda x: host(x[n:n + 1, :, h:h + 1])
        st = lambda x: None if x is None else host(x[n:n + 1, h:h + 1])
        ref = oracle.bwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                         sl(inp["beta"]), inp["scale"], sl(dout), h0=st(inp["h0"]), dhT=st(dhT))
        mine = [sl(g) for g in got[:5]] + [st(got[5])]
        for name, g, r in zip(NAMES, mine, ref):
            worst[name] = max(worst[name], rel(g, r))
    print(f"PARITY bwd {cfg.name} pairs={len(pairs)} " +
          " ".join(f"{k}={v:.3e}" for k, v in worst.items()))
    for name, e in worst.items():
        assert e <= TOL["bf16"][name], (cfg.name, name, e)


def test_backward_full_16_head_workload(kda):
    """B=1, H=16, T=4096, d=128, bf16, h0 ~ N(0, 0.02): all 16 pairs."""
    _full_size(kda, W.SINGLE, [(0, h) for h in range(W.SINGLE.H)])


@pytest.mark.slow
def test_backward_full_batched_workload_sampled(kda):
    """B=8, H=32, T=8192, d=128, bf16: 4 sampled (sequence, head) pairs."""
    rng = np.random.default_rng(2)
    pairs = [(int(rng.integers(8)), int(rng.integers(32))) for _ in range(4)]
    _full_size(kda, W.BATCHED, pairs)


def test_backward_empty_inputs(kda):
    """T = 0: no token gradients, dh0 = dhT; packed batch of empty sequences likewise."""
    for lengths in (None, [0, 0, 0]):
        cfg = (W.small_prefill(B=2, T=0, H=2, dk=64, dv=64, io_dtype="f32", seed=1, h0_std=0.1)
               if lengths is None else
               W.small_prefill(H=2, dk=64, dv=64, io_dtype="f32", seed=1, h0_std=0.1, lengths=lengths))
        inp = W.make_prefill(cfg, "cuda")
        dout, dhT = _upstream(cfg, inp, 3)
        got = kda.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], dout, h0=inp["h0"], dhT=dhT, cu_seqlens=inp["cu_seqlens"])
        torch.cuda.synchronize()
        torch.testing.assert_close(got[5], dhT, rtol=0, atol=0)
        assert all(g.numel() == 0 for g in got[:5])
