"""GPU parity of the chunkwise prefill (kda_chunk_fwd through the C ABI)
against the fp64 oracle, element by element, on seeded inputs: ragged tails,
several chunks, every supported head size, packed variable-length batches,
continuation across calls, the empty case, and the full-size workloads
(all pairs for the 16-head prefill; sampled pairs for the larger ones)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from kda_testutil import TOL, host, oracle_pairs, oracle_prefill, rel

pytestmark = pytest.mark.gpu

# tensor cores: bf16 with dk = dv = 128 only; "tensorcore_fused" is the one-kernel prefill
# (what AUTO runs with enough chains), "tensorcore_chain" the two-kernel one
IMPLS = ["simt", "tensorcore_fused", "tensorcore_chain"]
TC_IMPLS = ["tensorcore_fused", "tensorcore_chain"]


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def run(kda, inp, impl="auto"):
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], impl=impl)
    torch.cuda.synchronize()
    return out, hT


def check_full(kda, cfg, impl="auto"):
    inp = W.make_prefill(cfg, "cuda")
    out, hT = run(kda, inp, impl)
    ro, rh = oracle_prefill(inp)
    eo, eh = rel(out, ro), rel(hT, rh)
    tol = TOL[cfg.io_dtype]
    print(f"PARITY {cfg.name} impl={impl} out={eo:.3e} hT={eh:.3e} tol={tol:g}")
    assert eo <= tol and eh <= tol, (cfg.name, impl, eo, eh)
    return eo, eh


def test_tiny_fp32_workload(kda):
    """B=1, H=2, T=256, dk=dv=64, fp32 I/O, h0 = 0, seed 0 (SIMT path)."""
    check_full(kda, W.TINY, "simt")
    check_full(kda, W.TINY, "auto")


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("T", [1, 64, 150, 300])
def test_bf16_d128_ragged(kda, impl, T):
    """bf16, dk = dv = 128, h0 != 0, lengths below, at and across chunk boundaries."""
    cfg = W.small_prefill(B=2, T=T, H=3, dk=128, dv=128, io_dtype="bf16", seed=T, h0_std=0.02)
    check_full(kda, cfg, impl)


@pytest.mark.parametrize("impl", TC_IMPLS)
@pytest.mark.parametrize("shift", [3.0, -4.0])
def test_tensorcore_fast_and_slow_decay(kda, shift, impl):
    """Mean per-token decay e^-3.1 (fast) and e^-0.02 (slow): the exponent
    references keep the tensor-core factors in range; parity holds."""
    cfg = W.small_prefill(B=1, T=256, H=2, dk=128, dv=128, io_dtype="bf16", seed=4,
                          gate_shift=shift, h0_std=0.02)
    check_full(kda, cfg, impl)


@pytest.mark.parametrize("impl", ["auto", "tensorcore_fused"])
@pytest.mark.parametrize("shift", [8.0, 40.0])
def test_fused_exact_at_any_decay(kda, shift, impl):
    """Mean per-token decay about e^-8 and e^-40 in bf16 at d = 128 through the
    default path: the one-reference factors would leave the fp32 range, so every
    chunk takes the level passes (all factors <= 1); parity holds."""
    cfg = W.small_prefill(B=2, T=200, H=2, dk=128, dv=128, io_dtype="bf16", seed=12,
                          gate_shift=shift, h0_std=0.05)
    check_full(kda, cfg, impl)


@pytest.mark.parametrize("shift", [0.3, 0.8])
def test_fused_mid_chunk_reference(kda, shift):
    """Mean per-token decay about e^-1.0 and e^-1.3: many (0.3) or all (0.8) chunks
    decay past the chunk-start reference's range (2^100 over 64 tokens) but within
    2^100 of the first half's decay sum, so the fused kernel takes one A/Aqk MMA
    with factors referenced there and writes the image rows back at the chunk start;
    parity holds, the partial last chunk included."""
    cfg = W.small_prefill(B=2, T=300, H=2, dk=128, dv=128, io_dtype="bf16", seed=15,
                          gate_shift=shift, h0_std=0.05)
    check_full(kda, cfg, "tensorcore_fused")


def test_fused_mixed_fast_and_fallback_chunks(kda):
    """Chunks of both kinds in one call (fast decay in one sequence, slow in the
    other, packed): the per-chunk choice of factors is independent."""
    slow = W.small_prefill(B=1, T=190, H=2, dk=128, dv=128, io_dtype="bf16", seed=13, h0_std=0.05)
    fast = W.small_prefill(B=1, T=130, H=2, dk=128, dv=128, io_dtype="bf16", seed=14,
                           gate_shift=8.0, h0_std=0.05)
    a, b = W.make_prefill(slow, "cuda"), W.make_prefill(fast, "cuda")
    inp = {k: (torch.cat([a[k], b[k]], dim=1) if k in ("q", "k", "v", "log_alpha", "beta") else a[k])
           for k in a}
    inp["h0"] = torch.cat([a["h0"], b["h0"]], dim=0)
    inp["cu_seqlens"] = torch.tensor([0, 190, 320], dtype=torch.int32, device="cuda")
    out, hT = run(kda, inp, "tensorcore_fused")
    ro, rh = oracle_prefill(inp)
    eo, eh = rel(out, ro), rel(hT, rh)
    print(f"PARITY mixed-decay fused out={eo:.3e} hT={eh:.3e}")
    assert eo <= TOL["bf16"] and eh <= TOL["bf16"]


@pytest.mark.parametrize("impl", TC_IMPLS)
def test_more_chains_than_sms(kda, impl):
    """160 (sequence, head) chains: the fused kernel's persistent CTAs take
    several chains each (the grid has one CTA per SM)."""
    cfg = W.small_prefill(B=5, T=130, H=32, dk=128, dv=128, io_dtype="bf16", seed=15, h0_std=0.02)
    check_full(kda, cfg, impl)


@pytest.mark.parametrize("impl", ["auto", "tensorcore_fused"])
def test_packed_chains_handed_out_by_tickets(kda, impl):
    """Packed sequences: after its first chain each CTA takes the next one from a
    global ticket counter, and the other roles of the CTA read it from the issuer's
    ring.  400 sequences of 0 to 150 tokens (empty ones included, sorted longest first
    on the device) at H = 2: 800 chains over one CTA per SM, with initial states."""
    rng = np.random.default_rng(16)
    lengths = [int(x) for x in rng.integers(0, 151, size=400)]
    lengths[3] = 0
    lengths[-1] = 0
    cfg = W.small_prefill(H=2, dk=128, dv=128, io_dtype="bf16", seed=16, h0_std=0.02,
                          lengths=lengths)
    check_full(kda, cfg, impl)


@pytest.mark.parametrize("shift", [-4.0, 3.0, 3.6, 8.0])
def test_simt_decay_rates_fp32(kda, shift):
    """fp32 I/O at mean per-token decays from e^-0.02 to e^-8: the SIMT prep factors
    each 16-row diagonal block through its first row while every channel's decay
    across the block stays within 64 nats and takes it pairwise past that.  Over 15
    tokens the channels decay by ~46 nats at shift 3 (factored blocks), ~55 at 3.6
    (the largest of 128 channels passes 64 in about half the blocks: both kinds in
    one chunk) and ~120 at 8 (pairwise blocks); parity holds at the fp32 bar throughout."""
    cfg = W.small_prefill(B=1, T=200, H=2, dk=128, dv=128, io_dtype="f32", seed=11,
                          gate_shift=shift, h0_std=0.05)
    check_full(kda, cfg, "simt")


def test_tensorcore_refuses_unsupported_shapes(kda):
    cfg = W.small_prefill(B=1, T=64, H=1, dk=64, dv=64, io_dtype="bf16", seed=1)
    inp = W.make_prefill(cfg, "cuda")
    with pytest.raises(kda.KDAError):
        run(kda, inp, "tensorcore")
    cfg = W.small_prefill(B=1, T=64, H=1, dk=128, dv=128, io_dtype="f32", seed=1)
    inp = W.make_prefill(cfg, "cuda")
    with pytest.raises(kda.KDAError):
        run(kda, inp, "tensorcore")


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_head_sizes_ragged_tail(kda, dk, dv, io):
    cfg = W.small_prefill(B=2, T=150, H=3, dk=dk, dv=dv, io_dtype=io, seed=dk + dv, h0_std=0.05)
    check_full(kda, cfg, "simt")


@pytest.mark.parametrize("io,impl", [("f32", "simt"), ("bf16", "simt"), ("bf16", "tensorcore_fused"),
                                     ("bf16", "tensorcore_chain")])
def test_packed_variable_lengths(kda, io, impl):
    lens = [1, 63, 64, 65, 0, 130, 200, 7]
    cfg = W.small_prefill(H=2, dk=128, dv=128, io_dtype=io, seed=7, h0_std=0.05, lengths=lens)
    check_full(kda, cfg, impl)


@pytest.mark.parametrize("io,impl", [("f32", "simt"), ("bf16", "tensorcore_fused"),
                                     ("bf16", "tensorcore_chain")])
def test_packed_equals_separate_calls(kda, io, impl):
    lens = [70, 1, 129]
    cfg = W.small_prefill(H=2, dk=128, dv=128, io_dtype=io, seed=8, h0_std=0.05, lengths=lens)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = run(kda, inp, impl)
    cu = [0] + list(np.cumsum(lens))
    for n in range(len(lens)):
        sub = {k: (v[:, cu[n]:cu[n + 1]] if k in ("q", "k", "v", "log_alpha", "beta") else v)
               for k, v in inp.items()}
        sub = {k: (v.contiguous() if isinstance(v, torch.Tensor) else v) for k, v in sub.items()}
        sub["h0"] = inp["h0"][n:n + 1].contiguous()
        sub["cu_seqlens"] = None
        o1, h1 = run(kda, sub, impl)
        # the same per-sequence chunk arithmetic either way: equal to rounding noise
        assert rel(o1, host(out[:, cu[n]:cu[n + 1]]).double().numpy()) <= 1e-6
        assert rel(h1, host(hT[n:n + 1]).double().numpy()) <= 1e-6


@pytest.mark.parametrize("t1", [64, 100])
@pytest.mark.parametrize("io,impl", [("f32", "simt"), ("bf16", "tensorcore_fused"),
                                     ("bf16", "tensorcore_chain")])
def test_continuation_across_calls(kda, t1, io, impl):
    """[0, t1) then [t1, T) with h0 = hT of the first call equals one pass
    (on and off a chunk boundary): the state layout survives the hand-over."""
    cfg = W.small_prefill(B=1, T=256, H=2, dk=128, dv=128, io_dtype=io, seed=9, h0_std=0.05)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = run(kda, inp, impl)
    a = {k: (v[:, :t1].contiguous() if k in ("q", "k", "v", "log_alpha", "beta") else v)
         for k, v in inp.items()}
    o1, h1 = run(kda, a, impl)
    b = {k: (v[:, t1:].contiguous() if k in ("q", "k", "v", "log_alpha", "beta") else v)
         for k, v in inp.items()}
    b["h0"] = h1
    o2, h2 = run(kda, b, impl)
    ro, rh = oracle_prefill(inp)
    assert rel(torch.cat([o1, o2], dim=1), ro) <= TOL[io]
    assert rel(h2, rh) <= TOL[io]


def test_empty_sequence_passes_state_through(kda):
    cfg = W.small_prefill(B=3, T=0, H=2, dk=64, dv=64, io_dtype="f32", seed=1, h0_std=0.1)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = run(kda, inp)
    assert out.numel() == 0
    torch.testing.assert_close(hT, inp["h0"], rtol=0, atol=0)


def test_zero_initial_state_when_h0_absent(kda):
    cfg = W.small_prefill(B=1, T=80, H=1, dk=64, dv=64, io_dtype="f32", seed=2)
    inp = W.make_prefill(cfg, "cuda")
    o1, h1 = run(kda, inp)
    inp["h0"] = torch.zeros(1, 1, 64, 64, device="cuda")
    o2, h2 = run(kda, inp)
    torch.testing.assert_close(o1, o2, rtol=0, atol=0)
    torch.testing.assert_close(h1, h2, rtol=0, atol=0)


@pytest.mark.slow
@pytest.mark.parametrize("impl", ["auto"])
def test_single_head_group_prefill_full(kda, impl):
    """B=1, H=16, T=4096, d=128, bf16, h0 ~ N(0, 0.02^2): every output and state."""
    check_full(kda, W.SINGLE, impl)


@pytest.mark.slow
def test_batched_prefill_sampled_pairs(kda):
    """B=8, H=32, T=8192, bf16 (the benchmark workload, same launch): four
    (batch, head) pairs compared in full against the oracle."""
    cfg = W.BATCHED
    inp = W.make_prefill(cfg, "cuda")
    out, hT = run(kda, inp)
    rng = np.random.default_rng(cfg.seed)
    pairs = [(int(rng.integers(cfg.B)), int(rng.integers(cfg.H))) for _ in range(4)]
    res = oracle_pairs(inp, pairs)
    for (n, h), ((b, t0, t1), ro, rh) in zip(pairs, res):
        eo, eh = rel(out[b, t0:t1, h], ro), rel(hT[n, h], rh)
        print(f"PARITY {cfg.name} pair=({n},{h}) out={eo:.3e} hT={eh:.3e} tol=0.005")
        assert eo <= TOL["bf16"] and eh <= TOL["bf16"], (n, h)


@pytest.mark.slow
def test_long_context_varlen_sampled_pairs(kda):
    """16 packed sequences, 2^20 tokens, H=32, bf16: four (sequence, head)
    pairs (the longest and the shortest sequence among them) in full."""
    cfg = W.varlen_config()
    inp = W.make_prefill(cfg, "cuda")
    out, hT = run(kda, inp)
    L = np.array(cfg.lengths)
    rng = np.random.default_rng(cfg.seed)
    seqs = [int(L.argmax()), int(L.argmin()), int(rng.integers(cfg.N)), int(rng.integers(cfg.N))]
    pairs = [(n, int(rng.integers(cfg.H))) for n in seqs]
    res = oracle_pairs(inp, pairs)
    for (n, h), ((b, t0, t1), ro, rh) in zip(pairs, res):
        eo, eh = rel(out[0, t0:t1, h], ro), rel(hT[n, h], rh)
        print(f"PARITY {cfg.name} pair=({n},{h}) len={t1 - t0} out={eo:.3e} hT={eh:.3e} tol=0.005")
        assert eo <= TOL["bf16"] and eh <= TOL["bf16"], (n, h)
