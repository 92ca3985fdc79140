"""Pooled recurrent states (kda_chunk_fwd_slots / kda_recurrent_step_slots)
against the fp64 oracle: decode on a state pool, chunked prefill continuing
from and returning to pool slots followed by decode steps (the serving path
whose state layout across chunk boundaries "Kimi Linear acaba de superar a la
atencion completa en sus propios terminos" flags as the practical risk),
negative slots (no cached state) and out-of-range slots (reported, not
accessed)."""
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


def _h(x):
    return host(x).double().numpy()


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_on_pool(kda, io):
    P, H, d = 7, 2, 128
    cfg = W.DecodeConfig("pool", N=4, H=H, dk=d, dv=d, steps=1, seed=50, io_dtype=io)
    gen = W.decode_generator(cfg, "cuda")
    pool = torch.randn((P, H, d, d), generator=gen, device="cuda") * 0.05
    before = pool.clone()
    x = W.make_decode_step(cfg, gen, "cuda")
    slots = torch.tensor([5, 0, -1, 3], dtype=torch.int32, device="cuda")
    scale = 1 / np.sqrt(d)
    out = kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, scale,
                             slots=slots)
    torch.cuda.synchronize()
    for n, sl in enumerate([5, 0, -1, 3]):
        if sl < 0:
            assert float(out[n].abs().max()) == 0.0
            continue
        sub = {k: v[n:n + 1] for k, v in x.items()}
        ro, rs = oracle.step(host(sub["q"]), host(sub["k"]), host(sub["v"]), host(sub["log_alpha"]),
                             host(sub["beta"]), _h(before[sl:sl + 1]), scale)
        assert rel(out[n:n + 1], ro) <= TOL[io]
        assert rel(pool[sl:sl + 1], rs) <= 1e-5
    for sl in (1, 2, 4, 6):
        torch.testing.assert_close(pool[sl], before[sl], rtol=0, atol=0)


@pytest.mark.parametrize("io,impl", [("f32", "simt"), ("bf16", "tensorcore"), ("bf16", "simt")])
def test_chunked_prefill_then_decode_through_slots(kda, io, impl):
    """Three sequences (lengths 130, 64, 71) prefilled in two calls split at
    token 70 (off a chunk boundary for two of them), then three decode steps,
    all through pool slots [2, 0, 4] of a 5-slot pool; every output and the
    final states match the oracle run over the whole token sequences."""
    H, d, P = 2, 128, 5
    lens = [130, 64, 71]
    split = 70
    steps = 3
    slots_l = [2, 0, 4]
    full = [L + steps for L in lens]
    cfg = W.small_prefill(H=H, dk=d, dv=d, io_dtype=io, seed=51, lengths=full)
    inp = W.make_prefill(cfg, "cuda")
    cu = np.concatenate([[0], np.cumsum(full)])
    pool = torch.zeros((P, H, d, d), device="cuda")
    h0 = (torch.randn((len(lens), H, d, d), device="cuda") * 0.02)
    for n, sl in enumerate(slots_l):
        pool[sl] = h0[n]
    slots = torch.tensor(slots_l, dtype=torch.int32, device="cuda")

    def take(lo_hi):
        idx = np.concatenate([np.arange(cu[n] + a, cu[n] + b) for n, (a, b) in enumerate(lo_hi)])
        it = torch.from_numpy(idx).to("cuda")
        sub = {k: inp[k][:, it].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        seg = np.concatenate([[0], np.cumsum([b - a for a, b in lo_hi])]).astype(np.int32)
        return sub, torch.from_numpy(seg).to("cuda"), idx

    outs = {}
    for part in ([(0, min(split, L)) for L in lens], [(min(split, L), L) for L in lens]):
        sub, seg, idx = take(part)
        o, _ = kda.chunk_fwd(sub["q"], sub["k"], sub["v"], sub["log_alpha"], sub["beta"],
                             inp["scale"], cu_seqlens=seg, state_pool=pool, slots=slots, impl=impl)
        for j, t in enumerate(idx):
            outs[int(t)] = o[0, j]
    for s in range(steps):
        idx = np.array([cu[n] + lens[n] + s for n in range(len(lens))])
        it = torch.from_numpy(idx).to("cuda")
        x = {k: inp[k][0, it].contiguous() for k in ("q", "k", "v", "log_alpha", "beta")}
        o = kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool,
                               inp["scale"], slots=slots)
        for j, t in enumerate(idx):
            outs[int(t)] = o[j]
    torch.cuda.synchronize()
    gpu_out = torch.stack([outs[t] for t in range(cu[-1])]).unsqueeze(0)
    ro, rh = oracle.fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                        host(inp["beta"]), inp["scale"], h0=host(h0), cu_seqlens=cu)
    assert rel(gpu_out, ro) <= TOL[io]
    for n, sl in enumerate(slots_l):
        assert rel(pool[sl], rh[n]) <= TOL[io]
    assert float(pool[1].abs().max()) == 0.0 and float(pool[3].abs().max()) == 0.0


@pytest.mark.parametrize("impl", ["simt", "tensorcore"])
def test_negative_slot_means_no_cached_state(kda, impl):
    H, d = 2, 128
    cfg = W.small_prefill(H=H, dk=d, dv=d, io_dtype="bf16", seed=52, lengths=[90, 40])
    inp = W.make_prefill(cfg, "cuda")
    pool = torch.randn((3, H, d, d), device="cuda") * 0.05
    before = pool.clone()
    slots = torch.tensor([-1, 1], dtype=torch.int32, device="cuda")
    out, _ = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["scale"], cu_seqlens=inp["cu_seqlens"], state_pool=pool, slots=slots,
                           impl=impl)
    torch.cuda.synchronize()
    h0 = torch.zeros((2, H, d, d), device="cuda")
    h0[1] = before[1]
    ro, rh = oracle.fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                        host(inp["beta"]), inp["scale"], h0=host(h0),
                        cu_seqlens=host(inp["cu_seqlens"]).numpy())
    assert rel(out, ro) <= TOL["bf16"]
    assert rel(pool[1], rh[1]) <= TOL["bf16"]
    torch.testing.assert_close(pool[0], before[0], rtol=0, atol=0)
    torch.testing.assert_close(pool[2], before[2], rtol=0, atol=0)


@pytest.mark.parametrize("lengths", [[300, 130, 0, 200], [700]])
def test_pool_prefill_past_the_two_kernel_decay_range(kda, lengths):
    """AUTO with few chains on a state pool at about e^-8 of decay per token: the two-kernel
    form's prep flags the blocks, its walks leave the pool untouched, and the fused kernel
    continues every sequence from its slot and returns it there (pooled states read and
    written in place); unused slots stay as they were."""
    H, d = 2, 128
    cfg = W.small_prefill(H=H, dk=d, dv=d, io_dtype="bf16", seed=54, gate_shift=8.0,
                          lengths=lengths)
    inp = W.make_prefill(cfg, "cuda")
    N = len(lengths)
    P = N + 2
    pool = torch.randn((P, H, d, d), device="cuda") * 0.05
    before = pool.clone()
    slot_list = [P - 1 - n for n in range(N)]
    slots = torch.tensor(slot_list, dtype=torch.int32, device="cuda")
    kda.profiler_read(reset=True)
    out, _ = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["scale"], cu_seqlens=inp["cu_seqlens"], state_pool=pool, slots=slots)
    torch.cuda.synchronize()
    st = kda.profiler_read(reset=True)
    assert st["chunk_prep_tc"][0] >= 1 and st["chunk_fused_tc"][0] == 1, st
    h0 = before[slot_list]
    ro, rh = oracle.fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                        host(inp["beta"]), inp["scale"], h0=host(h0),
                        cu_seqlens=host(inp["cu_seqlens"]).numpy())
    assert rel(out, ro) <= TOL["bf16"]
    for n, sl in enumerate(slot_list):
        assert rel(pool[sl], rh[n]) <= TOL["bf16"], n
    for sl in range(P - N):
        torch.testing.assert_close(pool[sl], before[sl], rtol=0, atol=0)


@pytest.mark.parametrize("impl", ["simt", "tensorcore"])
def test_slot_beyond_pool_is_reported(kda, impl):
    H, d = 2, 128
    cfg = W.small_prefill(H=H, dk=d, dv=d, io_dtype="bf16", seed=53, lengths=[50, 60])
    inp = W.make_prefill(cfg, "cuda")
    pool = torch.zeros((2, H, d, d), device="cuda")
    slots = torch.tensor([0, 7], dtype=torch.int32, device="cuda")
    with pytest.raises(kda.KDAError) as e:
        kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["scale"],
                      cu_seqlens=inp["cu_seqlens"], state_pool=pool, slots=slots, impl=impl)
    assert e.value.status == kda.KDA_ERR_INVALID_ARG
    x = W.make_decode_step(W.DecodeConfig("p", N=2, H=H, dk=d, dv=d, steps=1, seed=54),
                           W.decode_generator(W.DecodeConfig("p", 2, H, d, d, 1, 54), "cuda"), "cuda")
    with pytest.raises(kda.KDAError) as e:
        kda.recurrent_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], pool, 0.1, slots=slots)
    assert e.value.status == kda.KDA_ERR_INVALID_ARG
