"""fp64 CPU oracle for the KDA recurrence -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package.  The CUDA library never calls it and shares no code with it.

Functions (all inputs are converted exactly to fp64 first, so bf16 inputs are
read with the values the GPU sees):

* :func:`fwd`  -- token-by-token forward over packed sequences
  ("Kimi Delta Attention: la atencion lineal detras de Kimi K2 y Qwen3",
  section "Como funciona Kimi Delta Attention paso a paso": decay, predict,
  beta-scaled error, correct, read).
* :func:`step` -- one decode step, state updated in place (same update, one token).
* :func:`segment_map` -- the affine map S -> M S + B of a run of tokens.  The
  step is linear in S, so M is the state that the same tokens reach from the
  identity with zero values and B the state they reach from zero; both are
  computed with :func:`fwd`.  (The pages do not state this split; it follows
  from the step's linearity and is pinned against dense transition products.)
* :func:`compose` -- X_r of consecutive maps: X_0 = h0, X_{s+1} = M_s X_s + B_s.
* :func:`bwd`  -- gradients of sum(dout * out) + sum(dhT * hT) with respect to
  q, k, v, log_alpha, beta and h0: reverse-mode differentiation of the same
  per-token step, token by token backwards (the pages say the chunk algorithm
  is what the method trains with; the gradient itself is not on the pages and
  is pinned by finite differences and by torch autograd of a separately
  written recurrence).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, reductions to simpler published rules and brute-force matrix products.
"""
import ctypes
import os

import numpy as np

_lib = None


def _load():
    global _lib
    if _lib is None:
        from . import build as _build
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.kda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, i64p,
                                       i64, i64, i64, i64, ctypes.c_double]
        lib.kda_oracle_fwd.restype = ctypes.c_int
        lib.kda_oracle_step.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                        i64, i64, i64, i64, ctypes.c_double]
        lib.kda_oracle_step.restype = ctypes.c_int
        lib.kda_oracle_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                       i64p, i64, i64, i64, i64, ctypes.c_double]
        lib.kda_oracle_bwd.restype = ctypes.c_int
        lib.kda_oracle_threads.argtypes = []
        lib.kda_oracle_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x):
    """Exact conversion to a contiguous fp64 numpy array (torch tensors accepted)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch
        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def threads() -> int:
    return int(_load().kda_oracle_threads())


def fwd(q, k, v, log_alpha, beta, scale, h0=None, cu_seqlens=None, return_state=True):
    """Token-by-token fp64 forward.

    Shapes: q,k [B,T,H,dk]; v [B,T,H,dv]; log_alpha [B,T,H,dk]; beta [B,T,H];
    h0 [N,H,dk,dv] or None.  With ``cu_seqlens`` (N+1 offsets) the batch axis
    must be 1 and the N sequences are packed along T.
    Returns (out [B,T,H,dv], hT [N,H,dk,dv]) as fp64 arrays.
    """
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    h0 = _f64(h0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        if B != 1:
            raise ValueError("packed sequences need batch axis 1")
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != B * T:
        raise ValueError("cu_seqlens must start at 0 and end at the packed length")
    if h0 is not None and h0.shape != (N, H, dk, dv):
        raise ValueError(f"h0 shape {h0.shape} != {(N, H, dk, dv)}")
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    hT = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().kda_oracle_fwd(_p(q), _p(k), _p(v), _p(g), _p(b), _p(h0), _p(out),
                                _p(hT), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                N, H, dk, dv, float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle failed rc={rc}")
    return (out, hT) if return_state else out


def step(q, k, v, log_alpha, beta, state, scale):
    """One fp64 decode step.  q,k [N,H,dk]; v [N,H,dv]; log_alpha [N,H,dk];
    beta [N,H]; state [N,H,dk,dv].  Returns (out [N,H,dv], new_state)."""
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    S = _f64(state).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().kda_oracle_step(_p(q), _p(k), _p(v), _p(g), _p(b), _p(S), _p(out),
                                 N, H, dk, dv, float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle failed rc={rc}")
    return out, S


def bwd(q, k, v, log_alpha, beta, scale, dout, h0=None, dhT=None, cu_seqlens=None):
    """fp64 gradients.  Shapes as for fwd; dout [B,T,H,dv]; dhT [N,H,dk,dv] or
    None (zero).  Returns (dq, dk, dv, dlog_alpha, dbeta, dh0) as fp64 arrays."""
    q, k, v, g, b, do = (_f64(x) for x in (q, k, v, log_alpha, beta, dout))
    h0, dhT = _f64(h0), _f64(dhT)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        if B != 1:
            raise ValueError("packed sequences need batch axis 1")
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[0] != 0 or cu[-1] != B * T:
        raise ValueError("cu_seqlens must start at 0 and end at the packed length")
    if do.shape != (B, T, H, dv):
        raise ValueError(f"dout shape {do.shape} != {(B, T, H, dv)}")
    for name, x in (("h0", h0), ("dhT", dhT)):
        if x is not None and x.shape != (N, H, dk, dv):
            raise ValueError(f"{name} shape {x.shape} != {(N, H, dk, dv)}")
    dq = np.zeros_like(q); dk_ = np.zeros_like(k); dv_ = np.zeros_like(v)
    dg = np.zeros_like(g); db = np.zeros_like(b); dh0 = np.zeros((N, H, dk, dv))
    rc = _load().kda_oracle_bwd(_p(q), _p(k), _p(v), _p(g), _p(b), _p(h0), _p(do), _p(dhT),
                                _p(dq), _p(dk_), _p(dv_), _p(dg), _p(db), _p(dh0),
                                cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                N, H, dk, dv, float(scale))
    if rc != 0:
        raise RuntimeError(f"oracle failed rc={rc}")
    return dq, dk_, dv_, dg, db, dh0


def segment_map(q, k, v, log_alpha, beta, cu_seqlens=None):
    """(M [N,H,dk,dk], B [N,H,dk,dv]) of every (sequence, head): for any entry
    state S0 the state after the tokens is M @ S0 + B.  Inputs as for fwd."""
    q, k, v, g, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    dk = q.shape[-1]
    N = q.shape[0] if cu_seqlens is None else len(np.asarray(
        cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens)) - 1
    H = q.shape[2]
    _, Bm = fwd(q, k, v, g, b, 1.0, h0=None, cu_seqlens=cu_seqlens)
    eye = np.broadcast_to(np.eye(dk), (N, H, dk, dk)).copy()
    v0 = np.zeros(q.shape[:3] + (dk,))
    _, M = fwd(q, k, v0, g, b, 1.0, h0=eye, cu_seqlens=cu_seqlens)
    return M, Bm


def compose(maps, offs, h0=None):
    """State after applying maps[0], maps[1], ... in order to h0 (zeros if None):
    X <- maps[s] @ X + offs[s].  maps [S,...,dk,dk], offs [S,...,dk,dv]."""
    maps, offs = _f64(maps), _f64(offs)
    X = np.zeros(offs.shape[1:]) if h0 is None else _f64(h0).copy()
    for s in range(maps.shape[0]):
        X = maps[s] @ X + offs[s]
    return X


def rel_l2(x, ref):
    """||x - ref||_2 / ||ref||_2 in fp64 (0 when both are zero)."""
    x = _f64(x).ravel()
    ref = _f64(ref).ravel()
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    if den == 0.0:
        return float(num)
    return float(num / den)
