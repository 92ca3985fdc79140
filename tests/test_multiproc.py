"""World-size-2 gloo test of the multi-GPU host logic, on CPU: each rank takes
its head shard (and its share of packed sequences), computes it (with the
fp64 oracle standing in for the per-GPU call), and rank 0 gathers the shards
and checks them against the unsharded result; the max-over-ranks timing
reduction used by bench.py is checked too."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workloads as W
        from gated_delta_rule_75_b200.shard import head_range, sequence_assignment
        import bench

        cfg = W.small_prefill(H=5, dk=8, dv=8, io_dtype="f32", seed=3, h0_std=0.1,
                              lengths=[40, 7, 65, 1, 30])
        inp = W.make_prefill(cfg, "cpu")
        h0, h1 = head_range(cfg.H, world, rank)
        sl = lambda x: x[:, :, h0:h1].contiguous()
        out, hT = oracle.fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["log_alpha"]),
                             sl(inp["beta"]), inp["scale"], h0=inp["h0"][:, h0:h1].contiguous(),
                             cu_seqlens=inp["cu_seqlens"].numpy())
        # gather head shards (sizes differ: pad to the largest shard)
        hmax = max(head_range(cfg.H, world, r)[1] - head_range(cfg.H, world, r)[0]
                   for r in range(world))
        pad = np.zeros(out.shape[:2] + (hmax,) + out.shape[3:])
        pad[:, :, :h1 - h0] = out
        bufs = [torch.zeros_like(torch.from_numpy(pad)) for _ in range(world)]
        dist.all_gather(bufs, torch.from_numpy(pad))
        ok = True
        if rank == 0:
            full, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                 inp["scale"], h0=inp["h0"], cu_seqlens=inp["cu_seqlens"].numpy())
            parts = []
            for r in range(world):
                a, b = head_range(cfg.H, world, r)
                parts.append(bufs[r].numpy()[:, :, :b - a])
            ok &= np.allclose(np.concatenate(parts, axis=2), full, rtol=0, atol=1e-13)
        # sequence shards cover every sequence exactly once
        assign = sequence_assignment(cfg.lengths, world)
        ok &= sorted(i for a in assign for i in a) == list(range(len(cfg.lengths)))
        # the timing reduction bench.py uses
        mx = bench.max_over_ranks(float(rank + 1), world)
        ok &= mx == float(world)
        bench.barrier(world)
        result_q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharding():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    results = dict(q.get(timeout=5) for _ in range(2))
    assert codes == [0, 0], codes
    assert results == {0: True, 1: True}, results


def test_partitions():
    from gated_delta_rule_75_b200.shard import head_range, sequence_assignment
    for H in (1, 5, 32):
        for world in (1, 2, 3, 8):
            rs = [head_range(H, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == H
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in rs]
            assert max(sizes) - min(sizes) <= 1
    a = sequence_assignment([100, 1, 50, 50], 2)
    assert a == [[0, 1], [2, 3]]          # loads 101 and 100
    with pytest.raises(ValueError):
        head_range(4, 2, 2)


class _OracleOps:
    """Per-rank compute of the context-parallel split done by the fp64 oracle
    (CPU), so the gloo test checks the orchestration: pieces, exchange order,
    composition."""

    def segmap(self, q, k, v, g, b):
        import oracle
        M, Bm = oracle.segment_map(q, k, v, g, b)
        return torch.from_numpy(M), torch.from_numpy(Bm)

    def prefix(self, maps, offs, h0):
        import oracle
        return torch.from_numpy(oracle.compose(maps, offs, h0))

    def forward(self, q, k, v, g, b, scale, h0):
        import oracle
        out, hT = oracle.fwd(q, k, v, g, b, scale, h0=h0)
        return torch.from_numpy(out), torch.from_numpy(hT)


def _cp_worker(rank, world, port, result_q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import workloads as W
        from gated_delta_rule_75_b200.context_parallel import (chunk_fwd_context_parallel,
                                                               token_range)
        cfg = W.small_prefill(B=2, T=150, H=2, dk=8, dv=6, io_dtype="f32", seed=9, h0_std=0.1)
        inp = W.make_prefill(cfg, "cpu")
        t0, t1 = token_range(150, world, rank, align=16)
        sl = lambda x: x[:, t0:t1].contiguous()
        out, hT = chunk_fwd_context_parallel(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]),
                                             sl(inp["log_alpha"]), sl(inp["beta"]), inp["scale"],
                                             h0=inp["h0"], ops=_OracleOps())
        full_out, full_hT = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"],
                                       inp["beta"], inp["scale"], h0=inp["h0"])
        ok = np.allclose(out.numpy(), full_out[:, t0:t1], rtol=0, atol=1e-11)
        if rank == world - 1:
            ok &= np.allclose(hT.numpy(), full_hT, rtol=0, atol=1e-11)
        result_q.put((rank, bool(ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_gloo(world):
    """A sequence split across `world` ranks reproduces the single-pass
    outputs and final state (compute by the oracle, exchange over gloo)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    results = dict(q.get(timeout=5) for _ in range(world))
    assert codes == [0] * world, codes
    assert results == {r: True for r in range(world)}, results


def test_token_range():
    from gated_delta_rule_75_b200.context_parallel import token_range
    for T in (0, 1, 63, 64, 150, 4096, 4097):
        for world in (1, 2, 3, 8):
            rs = [token_range(T, world, r) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == T
            assert all(rs[i][1] == rs[i + 1][0] for i in range(world - 1))
            assert all(a % 64 == 0 or a == T for a, _ in rs)
    with pytest.raises(ValueError):
        token_range(10, 2, 2)
