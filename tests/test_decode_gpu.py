"""GPU parity of the decode step (kda_recurrent_step through the C ABI)
against the fp64 oracle: one step for every head size and dtype, the full
decode workload (N=256, H=32, d=128, bf16; every head for 8 chained steps,
then 64 sampled (sequence, head) pairs over all 1000 steps), and the
prefill/decode agreement (the final state of a prefill equals the state
reached by chaining decode steps over the same tokens)."""
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


def _step_oracle(x, S, scale):
    return oracle.step(host(x["q"]), host(x["k"]), host(x["v"]), host(x["log_alpha"]),
                       host(x["beta"]), S, scale)


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_single_step(kda, dk, dv, io):
    cfg = W.DecodeConfig("t", N=5, H=3, dk=dk, dv=dv, steps=3, seed=dk * 3 + dv, io_dtype=io)
    gen = W.decode_generator(cfg, "cuda")
    S = W.make_decode_state(cfg, gen, "cuda")
    S_ref = host(S).double().numpy()
    scale = 1.0 / np.sqrt(dk)
    for _ in range(cfg.steps):
        x = W.make_decode_step(cfg, gen, "cuda")
        o = kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, scale)
        torch.cuda.synchronize()
        ro, S_ref = _step_oracle(x, S_ref, scale)
        assert rel(o, ro) <= TOL[io]
        assert rel(S, S_ref) <= TOL["f32"]      # state arithmetic is fp32 on both dtypes


@pytest.mark.slow
def test_decode_workload(kda):
    cfg = W.DECODE
    gen = W.decode_generator(cfg, "cuda")
    S = W.make_decode_state(cfg, gen, "cuda")
    scale = 1.0 / np.sqrt(cfg.dk)
    rng = np.random.default_rng(cfg.seed)
    pairs = rng.choice(cfg.N * cfg.H, size=64, replace=False)
    S_all = host(S).double().numpy()
    S_smp = S_all.reshape(cfg.N * cfg.H, cfg.dk, cfg.dv)[pairs].copy()
    worst = 0.0
    for step in range(cfg.steps):
        x = W.make_decode_step(cfg, gen, "cuda")
        o = kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, scale)
        if step < 8:                                   # every head
            ro, S_all = _step_oracle(x, S_all, scale)
            worst = max(worst, rel(o, ro))
            assert rel(o, ro) <= TOL["bf16"], step
            assert rel(S, S_all) <= 1e-5, step
        sub = {k: host(v).reshape((cfg.N * cfg.H,) + tuple(v.shape[2:]))[pairs].unsqueeze(1)
               for k, v in x.items()}
        ro, S_smp = oracle.step(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                                S_smp[:, None], scale)
        S_smp = S_smp[:, 0]
        o_s = host(o).reshape(cfg.N * cfg.H, cfg.dv)[pairs]
        assert rel(o_s, ro[:, 0]) <= TOL["bf16"], step
    torch.cuda.synchronize()
    S_gpu = host(S).double().numpy().reshape(cfg.N * cfg.H, cfg.dk, cfg.dv)[pairs]
    print(f"PARITY {cfg.name} first-8-steps worst out={worst:.3e}; 1000-step sampled state "
          f"rel={rel(S_gpu, S_smp):.3e}")
    assert rel(S_gpu, S_smp) <= 1e-4


def test_prefill_state_equals_chained_decode(kda):
    cfg = W.small_prefill(B=2, T=70, H=2, dk=128, dv=128, io_dtype="f32", seed=11, h0_std=0.05)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"])
    S = inp["h0"].clone()
    for t in range(cfg.T):
        o = kda.recurrent_step(inp["q"][:, t].contiguous(), inp["k"][:, t].contiguous(),
                               inp["v"][:, t].contiguous(), inp["log_alpha"][:, t].contiguous(),
                               inp["beta"][:, t].contiguous(), S, inp["scale"])
        assert rel(o, host(out[:, t]).double().numpy()) <= 1e-5
    torch.cuda.synchronize()
    assert rel(S, host(hT).double().numpy()) <= 1e-5
