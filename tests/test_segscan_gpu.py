"""Segment-parallel state walk and context parallelism on the GPU, through the
C ABI, against the fp64 oracle.

* the tensor-core prefill with every (sequence, head) chain cut into segments
  (value walk, map walk, composition, final walk), on request;
* kda_chunk_fwd_segmap: (M, B) of each (sequence, head) vs oracle.segment_map;
* kda_affine_prefix vs oracle.compose;
* a sequence split into consecutive pieces run one after another on one GPU
  (what the ranks of a context-parallel group do, without the exchange):
  outputs and final state vs the oracle's single pass.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from kda_testutil import TOL, host, oracle_prefill, rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda(cuda_ok):
    from gated_delta_rule_75_b200 import build
    build.build()
    import gated_delta_rule_75_b200 as kda
    return kda


def _run(kda, inp, impl):
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=inp["h0"], cu_seqlens=inp["cu_seqlens"], impl=impl)
    torch.cuda.synchronize()
    return out, hT


def _check(kda, cfg, impl):
    inp = W.make_prefill(cfg, "cuda")
    out, hT = _run(kda, inp, impl)
    ro, rh = oracle_prefill(inp)
    eo, eh = rel(out, ro), rel(hT, rh)
    print(f"PARITY {cfg.name} impl={impl} out={eo:.3e} hT={eh:.3e} tol={TOL[cfg.io_dtype]:g}")
    assert eo <= TOL[cfg.io_dtype] and eh <= TOL[cfg.io_dtype], (cfg.name, impl, eo, eh)


@pytest.mark.parametrize("T", [1, 64, 150, 300, 700])
@pytest.mark.parametrize("impl", ["tensorcore_segmented", "tensorcore_chain"])
def test_segmented_walk_fixed_length(kda, impl, T):
    cfg = W.small_prefill(B=2, T=T, H=3, dk=128, dv=128, io_dtype="bf16", seed=100 + T,
                          h0_std=0.02)
    _check(kda, cfg, impl)


@pytest.mark.parametrize("impl", ["tensorcore_segmented", "tensorcore_chain"])
def test_segmented_walk_packed(kda, impl):
    """Packed sequences with an empty one, one token, partial and whole chunks."""
    cfg = W.small_prefill(H=2, dk=128, dv=128, io_dtype="bf16", seed=7, h0_std=0.02,
                          lengths=[0, 1, 130, 700, 64, 333])
    _check(kda, cfg, impl)


def test_segmented_walk_in_place_state(kda):
    """hT aliasing h0 (the continuation form): entry states are read by the
    composition before the final walk writes the final states."""
    cfg = W.small_prefill(B=2, T=500, H=2, dk=128, dv=128, io_dtype="bf16", seed=8, h0_std=0.02)
    inp = W.make_prefill(cfg, "cuda")
    ro, rh = oracle_prefill(inp)
    state = inp["h0"].clone()
    out, hT = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                            inp["scale"], h0=state, hT=state, impl="tensorcore_segmented")
    torch.cuda.synchronize()
    assert hT.data_ptr() == state.data_ptr()
    assert rel(out, ro) <= TOL["bf16"] and rel(state, rh) <= TOL["bf16"]


def test_segmented_walk_on_pool_slots(kda):
    P, H, d = 5, 2, 128
    cfg = W.small_prefill(H=H, dk=d, dv=d, io_dtype="bf16", seed=9, lengths=[200, 77, 300])
    inp = W.make_prefill(cfg, "cuda")
    gen = torch.Generator(device="cuda").manual_seed(9)
    pool = torch.randn((P, H, d, d), generator=gen, device="cuda") * 0.02
    before = pool.clone()
    slots_l = [3, -1, 0]
    slots = torch.tensor(slots_l, dtype=torch.int32, device="cuda")
    out, _ = kda.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                           inp["scale"], cu_seqlens=inp["cu_seqlens"], state_pool=pool,
                           slots=slots, impl="tensorcore_segmented")
    torch.cuda.synchronize()
    h0 = torch.stack([before[s] if s >= 0 else torch.zeros_like(before[0]) for s in slots_l])
    ro, rh = oracle.fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                        host(inp["beta"]), inp["scale"], h0=host(h0),
                        cu_seqlens=host(inp["cu_seqlens"]).numpy())
    assert rel(out, ro) <= TOL["bf16"]
    for n, s in enumerate(slots_l):
        if s >= 0:
            assert rel(pool[s], rh[n]) <= TOL["bf16"]
    for s in (1, 2, 4):
        torch.testing.assert_close(pool[s], before[s], rtol=0, atol=0)


def test_automatic_choice(kda):
    """AUTO with few chains (1 sequence x 2 heads) runs the two-kernel form with the
    segment-parallel walk, then launches the fused kernel, which does nothing when no
    chunk left the two-kernel decay range; with half the SMs' worth of chains (2 x 32)
    the one-chain-per-(sequence, head) walk; with many chains (8 x 32) only the fused
    kernel; the segmented walk runs on request too."""
    kda.profiler_read(reset=True)
    cfg = W.small_prefill(B=1, T=2048, H=2, dk=128, dv=128, io_dtype="bf16", seed=11,
                          h0_std=0.02)
    _check(kda, cfg, "auto")
    st = kda.profiler_read(reset=True)
    assert st["chunk_prep_tc"][0] == 1 and st["chunk_state_seg_tc"][0] == 2, st
    assert st["affine_prefix"][0] == 1 and st["chunk_fused_tc"][0] == 1, st
    _check(kda, W.small_prefill(B=2, T=200, H=32, dk=128, dv=128, io_dtype="bf16", seed=14,
                                h0_std=0.02), "auto")
    st = kda.profiler_read(reset=True)
    assert st["chunk_state_tc"][0] == 1 and st["chunk_state_seg_tc"][0] == 0, st
    cfg = W.small_prefill(B=8, T=100, H=32, dk=128, dv=128, io_dtype="bf16", seed=12)
    inp = W.make_prefill(cfg, "cuda")
    _run(kda, inp, "auto")
    st = kda.profiler_read(reset=True)
    assert st["chunk_fused_tc"][0] == 1 and st["chunk_state_tc"][0] == 0, st
    assert st["chunk_prep_tc"][0] == 0, st
    _check(kda, W.small_prefill(B=1, T=2048, H=2, dk=128, dv=128, io_dtype="bf16", seed=11,
                                h0_std=0.02), "tensorcore_segmented")
    st = kda.profiler_read(reset=True)
    assert st["chunk_state_seg_tc"][0] == 2 and st["affine_prefix"][0] == 1, st


@pytest.mark.parametrize("shape", [(1, 2048, 2, None), (2, 200, 32, None),
                                   (1, 0, 2, [900, 0, 130, 1000])])
@pytest.mark.parametrize("shift", [8.0, 40.0])
def test_automatic_choice_falls_back_past_the_decay_range(kda, shape, shift):
    """Few chains under AUTO with fast decay (about e^-8 and e^-40 per token): the
    two-kernel prep flags the 16-token blocks past its range, its walks do nothing and
    the fused kernel computes the call: parity at the bf16 bar, segmented, one chain
    per (sequence, head), and packed."""
    B, T, H, lengths = shape
    cfg = W.small_prefill(B=B, T=T, H=H, dk=128, dv=128, io_dtype="bf16", seed=15,
                          gate_shift=shift, h0_std=0.02, lengths=lengths)
    _check(kda, cfg, "auto")


def test_automatic_choice_one_fast_sequence_moves_the_whole_call(kda):
    """One packed sequence past the range among slow ones: the whole call goes to the
    fused kernel, and the slow sequences' results are still right."""
    slow = W.small_prefill(H=2, dk=128, dv=128, io_dtype="bf16", seed=16, h0_std=0.02,
                           lengths=[700, 64])
    fast = W.small_prefill(B=1, T=300, H=2, dk=128, dv=128, io_dtype="bf16", seed=17,
                           gate_shift=8.0, h0_std=0.02)
    a, b = W.make_prefill(slow, "cuda"), W.make_prefill(fast, "cuda")
    inp = {k: (torch.cat([a[k], b[k]], dim=1) if k in ("q", "k", "v", "log_alpha", "beta") else a[k])
           for k in a}
    inp["h0"] = torch.cat([a["h0"], b["h0"]], dim=0)
    inp["cu_seqlens"] = torch.tensor([0, 700, 764, 1064], dtype=torch.int32, device="cuda")
    kda.profiler_read(reset=True)
    out, hT = _run(kda, inp, "auto")
    st = kda.profiler_read(reset=True)
    assert st["chunk_prep_tc"][0] == 1 and st["chunk_fused_tc"][0] == 1, st
    ro, rh = oracle_prefill(inp)
    assert rel(out, ro) <= TOL["bf16"] and rel(hT, rh) <= TOL["bf16"]


@pytest.mark.parametrize("io,d", [("bf16", 128), ("f32", 64), ("bf16", 64), ("f32", 128)])
def test_segmap_matches_oracle(kda, io, d):
    cfg = W.small_prefill(H=2, dk=d, dv=d, io_dtype=io, seed=13, lengths=[150, 0, 64, 1])
    inp = W.make_prefill(cfg, "cuda")
    maps, offs = kda.chunk_fwd_segmap(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                      inp["beta"], cu_seqlens=inp["cu_seqlens"])
    torch.cuda.synchronize()
    M, Bm = oracle.segment_map(host(inp["q"]), host(inp["k"]), host(inp["v"]),
                               host(inp["log_alpha"]), host(inp["beta"]),
                               cu_seqlens=host(inp["cu_seqlens"]).numpy())
    em, eb = rel(maps, M), rel(offs, Bm)
    print(f"PARITY segmap_{io}_d{d} maps={em:.3e} offs={eb:.3e} tol={TOL[io]:g}")
    assert em <= TOL[io] and eb <= TOL[io]
    # the empty sequence: identity map, zero offset
    torch.testing.assert_close(maps[1], torch.eye(d, device="cuda").expand(2, d, d), rtol=0, atol=0)
    assert float(offs[1].abs().max()) == 0.0


@pytest.mark.parametrize("nseg", [0, 1, 6])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64)])
def test_affine_prefix_matches_compose(kda, nseg, dk, dv):
    gen = torch.Generator(device="cuda").manual_seed(nseg * 1000 + dk + dv)
    NH = 5
    maps = torch.randn((nseg, NH, dk, dk), generator=gen, device="cuda") / np.sqrt(dk)
    offs = torch.randn((nseg, NH, dk, dv), generator=gen, device="cuda")
    h0 = torch.randn((NH, dk, dv), generator=gen, device="cuda")
    out = kda.affine_prefix(maps, offs, h0)
    ref = oracle.compose(host(maps), host(offs), host(h0))
    assert rel(out, ref) <= 1e-5
    # in place on h0, and from zero
    x = h0.clone()
    kda.affine_prefix(maps, offs, x, out=x)
    assert rel(x, ref) <= 1e-5
    z = kda.affine_prefix(maps, offs, None)
    assert rel(z, oracle.compose(host(maps), host(offs), None)) <= 1e-5


def _emulated_context_parallel(kda, inp, cuts):
    """Pieces [cuts[r], cuts[r+1]) of every sequence run in order on this GPU."""
    sl = lambda x, a, c: x[:, a:c].contiguous()
    pieces = list(zip(cuts[:-1], cuts[1:]))
    maps, offs = [], []
    for a, c in pieces:
        m, b = kda.chunk_fwd_segmap(sl(inp["q"], a, c), sl(inp["k"], a, c), sl(inp["v"], a, c),
                                    sl(inp["log_alpha"], a, c), sl(inp["beta"], a, c))
        maps.append(m)
        offs.append(b)
    outs = []
    for r, (a, c) in enumerate(pieces):
        start = (kda.affine_prefix(torch.stack(maps[:r]), torch.stack(offs[:r]), inp["h0"])
                 if r else inp["h0"])
        o, S = kda.chunk_fwd(sl(inp["q"], a, c), sl(inp["k"], a, c), sl(inp["v"], a, c),
                             sl(inp["log_alpha"], a, c), sl(inp["beta"], a, c), inp["scale"],
                             h0=start)
        outs.append(o)
    torch.cuda.synchronize()
    return torch.cat(outs, dim=1), S


@pytest.mark.parametrize("io,d,cuts", [("bf16", 128, [0, 256, 512, 700]),
                                       ("bf16", 128, [0, 100, 700]),
                                       ("f32", 64, [0, 64, 320, 700]),
                                       ("f32", 128, [0, 333, 700])])
def test_context_parallel_pieces(kda, io, d, cuts):
    cfg = W.small_prefill(B=2, T=700, H=2, dk=d, dv=d, io_dtype=io, seed=14, h0_std=0.02)
    inp = W.make_prefill(cfg, "cuda")
    out, hT = _emulated_context_parallel(kda, inp, cuts)
    ro, rh = oracle_prefill(inp)
    eo, eh = rel(out, ro), rel(hT, rh)
    print(f"PARITY context_parallel_{io}_d{d}_cuts{len(cuts) - 1} out={eo:.3e} hT={eh:.3e}")
    assert eo <= TOL[io] and eh <= TOL[io]


def test_context_parallel_helper_over_nccl_one_rank(kda):
    """chunk_fwd_context_parallel with the library's own ops and an NCCL process
    group of one rank (the all-gather runs, the composition has no predecessor):
    the product path end to end, against the oracle."""
    import datetime
    import os
    import socket
    import torch.distributed as dist
    from gated_delta_rule_75_b200.context_parallel import chunk_fwd_context_parallel
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = W.small_prefill(B=2, T=300, H=2, dk=128, dv=128, io_dtype="bf16", seed=15, h0_std=0.02)
        inp = W.make_prefill(cfg, "cuda")
        out, hT = chunk_fwd_context_parallel(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                             inp["beta"], inp["scale"], h0=inp["h0"])
        torch.cuda.synchronize()
        ro, rh = oracle_prefill(inp)
        assert rel(out, ro) <= TOL["bf16"] and rel(hT, rh) <= TOL["bf16"]
    finally:
        dist.destroy_process_group()
