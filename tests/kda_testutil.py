"""Helpers shared by the GPU parity tests: run the oracle on host copies of the
exact tensors the GPU consumed, and compare with the rel-L2 metric."""
import numpy as np
import torch

import oracle

TOL = {"f32": 1e-5, "bf16": 5e-3}


def host(x):
    return None if x is None else x.detach().to("cpu")


def oracle_prefill(inp):
    """Full oracle forward over all sequences and heads."""
    return oracle.fwd(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                      host(inp["beta"]), inp["scale"], h0=host(inp["h0"]),
                      cu_seqlens=None if inp["cu_seqlens"] is None else host(inp["cu_seqlens"]).numpy())


def pair_slice(inp, n, h):
    """Token range and per-pair inputs of sequence n, head h, as [1, L, 1, d] host arrays."""
    if inp["cu_seqlens"] is None:
        b, t0, t1 = n, 0, inp["q"].shape[1]
    else:
        cu = host(inp["cu_seqlens"]).numpy()
        b, t0, t1 = 0, int(cu[n]), int(cu[n + 1])
    sl = lambda x: host(x[b, t0:t1, h]).unsqueeze(0).unsqueeze(2)
    h0 = None if inp["h0"] is None else host(inp["h0"][n, h]).unsqueeze(0).unsqueeze(0)
    return (b, t0, t1), dict(q=sl(inp["q"]), k=sl(inp["k"]), v=sl(inp["v"]),
                             log_alpha=sl(inp["log_alpha"]),
                             beta=host(inp["beta"][b, t0:t1, h]).unsqueeze(0).unsqueeze(2), h0=h0)


def oracle_pairs(inp, pairs):
    """Oracle on selected (sequence, head) pairs, run as one packed call so the
    pairs proceed in parallel.  Returns [(range, out [L, dv], hT [dk, dv])]."""
    ranges, parts = zip(*(pair_slice(inp, n, h) for n, h in pairs))
    cat = lambda key: torch.cat([p[key] for p in parts], dim=1)
    lens = [r[2] - r[1] for r in ranges]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    h0 = None
    if inp["h0"] is not None:
        h0 = torch.cat([p["h0"] for p in parts], dim=0)
    out, hT = oracle.fwd(cat("q"), cat("k"), cat("v"), cat("log_alpha"), cat("beta"),
                         inp["scale"], h0=h0, cu_seqlens=cu)
    return [(ranges[i], out[0, cu[i]:cu[i + 1], 0], hT[i, 0]) for i in range(len(pairs))]


def rel(x, ref):
    return oracle.rel_l2(host(x).double() if isinstance(x, torch.Tensor) else x, ref)
