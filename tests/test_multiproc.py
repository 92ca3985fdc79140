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
