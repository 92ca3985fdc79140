"""Gated DeltaNet (one decay per token and head) through kda_gdn_chunk_fwd and
kda_gdn_recurrent_step, against the fp64 oracle with the gate broadcast over
the key channels (the oracle pins tie that broadcast to the scalar-gate
recurrence).  The SIMT path and the decode step run the KDA arithmetic on the
broadcast gate, so they also match the KDA entry points bit for bit; the
tensor-core prefill has its own prep kernel (the scalar decay factors out of
the key products), checked against the oracle only."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from kda_testutil import TOL, host, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def _expand(log_a, dk):
    return log_a.unsqueeze(-1).expand(*log_a.shape, dk).contiguous()


@pytest.mark.parametrize("io,impl,dk", [("f32", "simt", 64), ("bf16", "simt", 128),
                                        ("bf16", "tensorcore", 128)])
@pytest.mark.parametrize("varlen", [False, True])
def test_gdn_prefill(kda, io, impl, dk, varlen):
    lengths = [100, 1, 64, 150] if varlen else None
    cfg = W.small_prefill(B=2, T=150, H=2, dk=dk, dv=dk, io_dtype=io, seed=60, h0_std=0.03,
                          lengths=lengths)
    inp = W.make_prefill(cfg, "cuda")
    log_a = W.scalar_gates(cfg.B, cfg.T, cfg.H, seed=60, device="cuda")
    out, hT = kda.gdn_chunk_fwd(inp["q"], inp["k"], inp["v"], log_a, inp["beta"], inp["scale"],
                                h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], impl=impl)
    torch.cuda.synchronize()
    cu = None if inp["cu_seqlens"] is None else host(inp["cu_seqlens"]).numpy()
    ro, rh = oracle.fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(_expand(log_a, dk)),
                        host(inp["beta"]), inp["scale"], h0=host(inp["h0"]), cu_seqlens=cu)
    e_out, e_h = rel(out, ro), rel(hT, rh)
    out2, hT2 = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], _expand(log_a, dk), inp["beta"],
                              inp["scale"], h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], impl=impl)
    torch.cuda.synchronize()
    print(f"PARITY gdn_{io}_{impl}_varlen{int(varlen)} out={e_out:.3e} hT={e_h:.3e} "
          f"(kda entry on the broadcast gate: out={rel(out2, ro):.3e} hT={rel(hT2, rh):.3e})")
    assert e_out <= TOL[io] and e_h <= TOL[io]
    if impl == "simt":
        # the KDA entry point with the broadcast gate runs the same arithmetic
        torch.testing.assert_close(out, out2, rtol=0, atol=0)
        torch.testing.assert_close(hT, hT2, rtol=0, atol=0)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_gdn_decode(kda, io):
    cfg = W.DecodeConfig("gdn", N=6, H=3, dk=128, dv=128, steps=3, seed=61, io_dtype=io)
    gen = W.decode_generator(cfg, "cuda")
    S = W.make_decode_state(cfg, gen, "cuda")
    S_ref = host(S).double().numpy()
    scale = 1 / np.sqrt(128)
    for s in range(cfg.steps):
        x = W.make_decode_step(cfg, gen, "cuda")
        log_a = W.scalar_gates(1, cfg.N, cfg.H, seed=61 + s, device="cuda")[0]
        o = kda.gdn_recurrent_step(x["q"], x["k"], x["v"], log_a, x["beta"], S, scale)
        torch.cuda.synchronize()
        ro, S_ref = oracle.step(host(x["q"]), host(x["k"]), host(x["v"]), host(_expand(log_a, 128)),
                                host(x["beta"]), S_ref, scale)
        assert rel(o, ro) <= TOL[io]
        assert rel(S, S_ref) <= 1e-5


@pytest.mark.parametrize("io,dk", [("f32", 64), ("bf16", 128)])
@pytest.mark.parametrize("varlen", [False, True])
def test_gdn_backward(kda, io, dk, varlen):
    """kda_gdn_chunk_bwd against the oracle's reverse mode on the broadcast gate;
    the gate gradient is the channel sum of the per-channel one."""
    lengths = [100, 1, 64, 150] if varlen else None
    cfg = W.small_prefill(B=2, T=150, H=2, dk=dk, dv=dk, io_dtype=io, seed=62, h0_std=0.03,
                          lengths=lengths)
    inp = W.make_prefill(cfg, "cuda")
    log_a = W.scalar_gates(cfg.B, cfg.T, cfg.H, seed=62, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(63)
    dout = torch.randn((cfg.B, cfg.T, cfg.H, dk), generator=gen, device="cuda").to(inp["q"].dtype)
    dhT = torch.randn((cfg.N, cfg.H, dk, dk), generator=gen, device="cuda")
    got = kda.gdn_chunk_bwd(inp["q"], inp["k"], inp["v"], log_a, inp["beta"], inp["scale"], dout,
                            h0=inp["h0"], dhT=dhT, cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    cu = None if inp["cu_seqlens"] is None else host(inp["cu_seqlens"]).numpy()
    ref = oracle.bwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(_expand(log_a, dk)),
                     host(inp["beta"]), inp["scale"], host(dout), h0=host(inp["h0"]),
                     dhT=host(dhT), cu_seqlens=cu)
    ref = list(ref)
    ref[3] = ref[3].sum(axis=-1)
    tol = {"f32": [1e-5] * 6, "bf16": [5e-3, 5e-3, 5e-3, 1e-5, 1e-5, 1e-5]}[io]
    errs = [rel(g, r) for g, r in zip(got, ref)]
    print(f"PARITY gdn_bwd_{io}_varlen{int(varlen)} " + " ".join(f"{e:.3e}" for e in errs))
    assert all(e <= t for e, t in zip(errs, tol)), errs
