"""Python binding of libkda.so, the B200 (sm_100a) Kimi Delta Attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/kda.h``.  Torch supplies device
memory and the current stream.  There is no CPU fallback: if the shared
library is missing or fails to load, every call raises.

    out, hT = chunk_fwd(q, k, v, log_alpha, beta, scale, h0=None, cu_seqlens=None)
    out     = recurrent_step(q, k, v, log_alpha, beta, state, scale)   # state in place
    maps, offs = chunk_fwd_segmap(q, k, v, log_alpha, beta)            # context parallelism
    start   = affine_prefix(maps, offs, h0)
"""
import ctypes
import os

import torch

__all__ = ["chunk_fwd", "recurrent_step", "gdn_chunk_fwd", "gdn_recurrent_step", "KDAError",
           "chunk_fwd_segmap", "affine_prefix", "chunk_bwd", "gdn_chunk_bwd",
           "library_path", "version",
           "profiler_enable", "profiler_read",
           "KDA_OK", "KDA_ERR_INVALID_ARG", "KDA_ERR_UNSUPPORTED", "KDA_ERR_CUDA",
           "KDA_ERR_NO_MEMORY", "KDA_ERR_TIMEOUT"]

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_NO_MEMORY, \
    KDA_ERR_TIMEOUT = range(6)
_IO = {torch.float32: 0, torch.bfloat16: 1}
_IMPL = {"auto": 0, "simt": 1, "tensorcore": 2, "tensorcore_chain": 3,
         "tensorcore_segmented": 4, "tensorcore_fused": 5}

library_path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkda.so")

_lib = None


class _KernelStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int64),
                ("timed_launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


def _load():
    """Load libkda.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(library_path):
        raise ImportError(f"{library_path} is not built; run "
                          "`python -m gated_delta_rule_75_b200.build`")
    lib = ctypes.CDLL(library_path)
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.kda_chunk_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                     ctypes.c_float, ctypes.c_int, ctypes.c_int, vp]
    lib.kda_chunk_fwd_ex.restype = ctypes.c_int
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                  ctypes.c_float, ctypes.c_int, vp]
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                       ctypes.c_float, ctypes.c_int, vp]
    lib.kda_recurrent_step.restype = ctypes.c_int
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    lib.kda_version.restype = ctypes.c_int
    lib.kda_chunk_fwd_slots.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                        i64, i64, ctypes.c_float, ctypes.c_int, ctypes.c_int, vp]
    lib.kda_chunk_fwd_slots.restype = ctypes.c_int
    lib.kda_recurrent_step_slots.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                             i64, ctypes.c_float, ctypes.c_int, vp]
    lib.kda_recurrent_step_slots.restype = ctypes.c_int
    lib.kda_gdn_chunk_fwd.argtypes = lib.kda_chunk_fwd_ex.argtypes
    lib.kda_gdn_chunk_fwd.restype = ctypes.c_int
    lib.kda_gdn_recurrent_step.argtypes = lib.kda_recurrent_step.argtypes
    lib.kda_gdn_recurrent_step.restype = ctypes.c_int
    lib.kda_chunk_fwd_segmap.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i64,
                                         i64, ctypes.c_int, vp]
    lib.kda_chunk_fwd_segmap.restype = ctypes.c_int
    lib.kda_affine_prefix.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, vp]
    lib.kda_affine_prefix.restype = ctypes.c_int
    lib.kda_chunk_bwd.argtypes = [vp] * 15 + [i64, i64, i64, i64, i64, ctypes.c_float,
                                              ctypes.c_int, vp]
    lib.kda_chunk_bwd.restype = ctypes.c_int
    lib.kda_gdn_chunk_bwd.argtypes = lib.kda_chunk_bwd.argtypes
    lib.kda_gdn_chunk_bwd.restype = ctypes.c_int
    lib.kda_debug_prep_image.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, ctypes.c_int, vp]
    lib.kda_debug_prep_image.restype = ctypes.c_int
    lib.kda_debug_bounded_wait.argtypes = [ctypes.c_int32, vp, vp]
    lib.kda_debug_bounded_wait.restype = ctypes.c_int
    lib.kda_workspace_high_water.argtypes = [ctypes.POINTER(ctypes.c_int64), ctypes.c_int]
    lib.kda_workspace_high_water.restype = ctypes.c_int
    lib.kda_get_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.kda_get_error.restype = ctypes.c_int
    lib.kda_profiler_enable.argtypes = [ctypes.c_int]
    lib.kda_profiler_enable.restype = None
    lib.kda_profiler_read.argtypes = [ctypes.POINTER(_KernelStat), ctypes.c_int, ctypes.c_int]
    lib.kda_profiler_read.restype = ctypes.c_int
    _lib = lib
    return lib


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_load().kda_status_string(status).decode()} (status {status})")


def version() -> int:
    return int(_load().kda_version())


def profiler_enable(on: bool = True) -> None:
    """Record CUDA events on the launching stream around each library kernel."""
    _load().kda_profiler_enable(1 if on else 0)


def profiler_read(reset: bool = True) -> dict:
    """{kernel name: (launches, timed launches, total event ms)}; waits for the
    recorded events.  Launches are counted whether or not timing is on."""
    lib = _load()
    arr = (_KernelStat * 32)()
    n = lib.kda_profiler_read(arr, 32, 1 if reset else 0)
    if n < 0:
        raise RuntimeError("kda_profiler_read: an event could not be read")
    return {arr[i].name.decode(): (int(arr[i].launches), int(arr[i].timed_launches),
                                   float(arr[i].total_ms)) for i in range(n)}


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check(t, name, dtype, shape, device):
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def chunk_fwd(q, k, v, log_alpha, beta, scale, h0=None, cu_seqlens=None, out=None,
              hT=None, output_final_state=True, impl="auto", state_pool=None, slots=None):
    """Chunkwise KDA prefill (C ABI ``kda_chunk_fwd_ex``, or ``kda_chunk_fwd_slots``
    when ``slots`` is given).

    q, k [B,T,H,dk] and v [B,T,H,dv] in fp32 or bf16; log_alpha [B,T,H,dk] and
    beta [B,T,H] fp32; h0 [N,H,dk,dv] fp32 or None.  With ``cu_seqlens`` (int32,
    N+1 entries, on the device) B must be 1 and N sequences are packed along T.
    With ``slots`` (int32 [N] on the device) and ``state_pool`` [P,H,dk,dv] fp32,
    sequence n starts from and writes back to state_pool[slots[n]] (h0/hT unused).
    Returns (out [B,T,H,dv] in the I/O dtype, hT [N,H,dk,dv] fp32 or None; with
    slots: (out, state_pool)).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    io = q.dtype
    if io not in _IO:
        raise TypeError(f"unsupported I/O dtype {io}")
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv))):
        _check(t, name, io, shp, dev)
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H, dk), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    if cu_seqlens is not None:
        if B != 1:
            raise ValueError("cu_seqlens needs a leading axis of 1")
        if cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor on the same device")
        N = cu_seqlens.numel() - 1
        n_arg, T_arg = N, T
    else:
        N = B
        n_arg, T_arg = B, T
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=io, device=dev)
    else:
        _check(out, "out", io, (B, T, H, dv), dev)
    if slots is not None:
        if state_pool is None or h0 is not None or hT is not None:
            raise ValueError("slots go with state_pool (and without h0 / hT)")
        _check(slots, "slots", torch.int32, (N,), dev)
        P = state_pool.shape[0]
        _check(state_pool, "state_pool", torch.float32, (P, H, dk, dv), dev)
        st = _load().kda_chunk_fwd_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                         _ptr(state_pool), _ptr(slots), _ptr(out), _ptr(cu_seqlens),
                                         n_arg, T_arg, P, H, dk, dv, float(scale), _IO[io],
                                         _IMPL[impl], _stream(dev))
        if st != KDA_OK:
            raise KDAError(st, "kda_chunk_fwd_slots")
        return out, state_pool
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif hT is not None:
        _check(hT, "hT", torch.float32, (N, H, dk, dv), dev)
    st = _load().kda_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(h0),
                               _ptr(out), _ptr(hT), _ptr(cu_seqlens), n_arg, T_arg, H, dk, dv,
                               float(scale), _IO[io], _IMPL[impl], _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd")
    return out, hT


def gdn_chunk_fwd(q, k, v, log_a, beta, scale, h0=None, cu_seqlens=None, out=None, hT=None,
                  output_final_state=True, impl="auto"):
    """Gated DeltaNet prefill (C ABI ``kda_gdn_chunk_fwd``): as :func:`chunk_fwd`
    with one gate per (token, head), log_a [B,T,H] fp32."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, io = q.device, q.dtype
    if io not in _IO:
        raise TypeError(f"unsupported I/O dtype {io}")
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv))):
        _check(t, name, io, shp, dev)
    _check(log_a, "log_a", torch.float32, (B, T, H), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and (B != 1 or cu_seqlens.dtype != torch.int32):
        raise ValueError("cu_seqlens needs int32 offsets and a leading axis of 1")
    if h0 is not None:
        _check(h0, "h0", torch.float32, (N, H, dk, dv), dev)
    out = torch.empty((B, T, H, dv), dtype=io, device=dev) if out is None else out
    _check(out, "out", io, (B, T, H, dv), dev)
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    st = _load().kda_gdn_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(beta), _ptr(h0),
                                   _ptr(out), _ptr(hT), _ptr(cu_seqlens), N, T, H, dk, dv,
                                   float(scale), _IO[io], _IMPL[impl], _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_gdn_chunk_fwd")
    return out, hT


def gdn_recurrent_step(q, k, v, log_a, beta, state, scale, out=None):
    """Gated DeltaNet decode step (C ABI ``kda_gdn_recurrent_step``); log_a [N,H]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev, io = q.device, q.dtype
    _check(log_a, "log_a", torch.float32, (N, H), dev)
    _check(beta, "beta", torch.float32, (N, H), dev)
    _check(state, "state", torch.float32, (N, H, dk, dv), dev)
    out = torch.empty((N, H, dv), dtype=io, device=dev) if out is None else out
    st = _load().kda_gdn_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_a), _ptr(beta),
                                        _ptr(state), _ptr(out), N, H, dk, dv, float(scale),
                                        _IO[io], _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_gdn_recurrent_step")
    return out


def recurrent_step(q, k, v, log_alpha, beta, state, scale, out=None, slots=None):
    """One decode token per sequence (C ABI ``kda_recurrent_step``); ``state``
    [N,H,dk,dv] fp32 is updated in place.  With ``slots`` (int32 [N] on the
    device), ``state`` is a pool [P,H,dk,dv] and sequence n uses slot slots[n]
    (``kda_recurrent_step_slots``).  Returns out [N,H,dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    io = q.dtype
    if io not in _IO:
        raise TypeError(f"unsupported I/O dtype {io}")
    _check(q, "q", io, (N, H, dk), dev)
    _check(k, "k", io, (N, H, dk), dev)
    _check(v, "v", io, (N, H, dv), dev)
    _check(log_alpha, "log_alpha", torch.float32, (N, H, dk), dev)
    _check(beta, "beta", torch.float32, (N, H), dev)
    if out is None:
        out = torch.empty((N, H, dv), dtype=io, device=dev)
    else:
        _check(out, "out", io, (N, H, dv), dev)
    if slots is not None:
        _check(slots, "slots", torch.int32, (N,), dev)
        P = state.shape[0]
        _check(state, "state", torch.float32, (P, H, dk, dv), dev)
        st = _load().kda_recurrent_step_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                              _ptr(beta), _ptr(state), _ptr(slots), _ptr(out),
                                              N, P, H, dk, dv, float(scale), _IO[io], _stream(dev))
        if st != KDA_OK:
            raise KDAError(st, "kda_recurrent_step_slots")
        return out
    _check(state, "state", torch.float32, (N, H, dk, dv), dev)
    st = _load().kda_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                 _ptr(state), _ptr(out), N, H, dk, dv, float(scale), _IO[io],
                                 _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_recurrent_step")
    return out


def chunk_fwd_segmap(q, k, v, log_alpha, beta, cu_seqlens=None, maps=None, offs=None):
    """Affine map of every (sequence, head) of a prefill input (C ABI
    ``kda_chunk_fwd_segmap``): for any entry state S0 the final state is
    maps[n, h] @ S0 + offs[n, h].  Inputs as for :func:`chunk_fwd`.  Returns
    (maps [N,H,dk,dk], offs [N,H,dk,dv]), fp32."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, io = q.device, q.dtype
    if io not in _IO:
        raise TypeError(f"unsupported I/O dtype {io}")
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv))):
        _check(t, name, io, shp, dev)
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H, dk), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    if cu_seqlens is not None:
        if B != 1 or cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev:
            raise ValueError("cu_seqlens needs int32 offsets on the device and a leading axis of 1")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if maps is None:
        maps = torch.empty((N, H, dk, dk), dtype=torch.float32, device=dev)
    if offs is None:
        offs = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    _check(maps, "maps", torch.float32, (N, H, dk, dk), dev)
    _check(offs, "offs", torch.float32, (N, H, dk, dv), dev)
    st = _load().kda_chunk_fwd_segmap(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                      _ptr(maps), _ptr(offs), _ptr(cu_seqlens), N, T, H, dk, dv,
                                      _IO[io], _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_chunk_fwd_segmap")
    return maps, offs


def affine_prefix(maps, offs, h0=None, out=None):
    """State after consecutive affine maps (C ABI ``kda_affine_prefix``).

    maps [S, ..., dk, dk] and offs [S, ..., dk, dv] fp32 hold S segments in
    order (segment-major); h0 [..., dk, dv] fp32 or None (zeros).  Returns
    out [..., dk, dv] = M_{S-1}(...(M_0 h0 + B_0)...) + B_{S-1}."""
    nseg = maps.shape[0]
    lead = tuple(offs.shape[1:-2])
    dk, dv = offs.shape[-2], offs.shape[-1]
    dev = offs.device
    NH = 1
    for x in lead:
        NH *= x
    _check(maps, "maps", torch.float32, (nseg,) + lead + (dk, dk), dev)
    _check(offs, "offs", torch.float32, (nseg,) + lead + (dk, dv), dev)
    if h0 is not None:
        _check(h0, "h0", torch.float32, lead + (dk, dv), dev)
    if out is None:
        out = torch.empty(lead + (dk, dv), dtype=torch.float32, device=dev)
    _check(out, "out", torch.float32, lead + (dk, dv), dev)
    st = _load().kda_affine_prefix(_ptr(maps), _ptr(offs), _ptr(h0), _ptr(out), nseg, NH, dk, dv,
                                   _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_affine_prefix")
    return out


def chunk_bwd(q, k, v, log_alpha, beta, scale, dout, h0=None, dhT=None, cu_seqlens=None,
              need_dh0=True, _gdn=False):
    """Gradients of sum(dout * out) + sum(dhT * hT) for the prefill
    :func:`chunk_fwd` computes on the same inputs (C ABI ``kda_chunk_bwd``).
    dout [B,T,H,dv] in the I/O dtype; dhT [N,H,dk,dv] fp32 or None.  Returns
    (dq, dk, dv in the I/O dtype; dlog_alpha, dbeta, dh0 in fp32; dh0 is None
    when need_dh0 is False)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, io = q.device, q.dtype
    if io not in _IO:
        raise TypeError(f"unsupported I/O dtype {io}")
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("v", v, (B, T, H, dv)),
                         ("dout", dout, (B, T, H, dv))):
        _check(t, name, io, shp, dev)
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H) if _gdn else (B, T, H, dk), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    if cu_seqlens is not None:
        if B != 1 or cu_seqlens.dtype != torch.int32 or cu_seqlens.device != dev:
            raise ValueError("cu_seqlens needs int32 offsets on the device and a leading axis of 1")
        N = cu_seqlens.numel() - 1
    else:
        N = B
    for name, t in (("h0", h0), ("dhT", dhT)):
        if t is not None:
            _check(t, name, torch.float32, (N, H, dk, dv), dev)
    dq = torch.empty_like(q)
    dk_ = torch.empty_like(k)
    dv_ = torch.empty_like(v)
    dg = torch.empty_like(log_alpha)
    db = torch.empty_like(beta)
    dh0 = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev) if need_dh0 else None
    fn = _load().kda_gdn_chunk_bwd if _gdn else _load().kda_chunk_bwd
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(h0), _ptr(dout),
            _ptr(dhT), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dg), _ptr(db), _ptr(dh0),
            _ptr(cu_seqlens), N, T, H, dk, dv, float(scale), _IO[io], _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_gdn_chunk_bwd" if _gdn else "kda_chunk_bwd")
    return dq, dk_, dv_, dg, db, dh0


def gdn_chunk_bwd(q, k, v, log_a, beta, scale, dout, h0=None, dhT=None, cu_seqlens=None,
                  need_dh0=True):
    """Gated DeltaNet gradients (C ABI ``kda_gdn_chunk_bwd``): as :func:`chunk_bwd`
    with one gate per (token, head), log_a [B,T,H] fp32; returns dlog_a [B,T,H]."""
    return chunk_bwd(q, k, v, log_a, beta, scale, dout, h0=h0, dhT=dhT, cu_seqlens=cu_seqlens,
                     need_dh0=need_dh0, _gdn=True)


IMAGE_BYTES = 66560   # one (chunk, head) operand image of the tensor-core prefill


def get_error(device="cuda") -> int:
    """C ABI ``kda_get_error``: takes (reads and clears) the device's error word
    after the work queued on the current stream; bit 0 = malformed cu_seqlens or a
    slot out of range, bits 1-6 = a bounded device wait gave up."""
    dev = torch.device(device)
    word = ctypes.c_int32(0)
    with torch.cuda.device(dev):
        st = _load().kda_get_error(_stream(dev), ctypes.byref(word))
    if st != 0:
        raise KDAError(st, "kda_get_error")
    return int(word.value)


def workspace_high_water(reset=False, device="cuda") -> int:
    """C ABI ``kda_workspace_high_water``: the most workspace bytes the library had
    allocated at once on ``device`` since the last reset; ``reset`` restarts it."""
    v = ctypes.c_int64(0)
    with torch.cuda.device(torch.device(device)):
        st = _load().kda_workspace_high_water(ctypes.byref(v), 1 if reset else 0)
    if st != 0:
        raise KDAError(st, "kda_workspace_high_water")
    return int(v.value)


def debug_bounded_wait(polls, device="cuda", to_library_word=False):
    """Self-test (C ABI ``kda_debug_bounded_wait``): a device wait on a barrier that
    nothing completes, given up after ``polls`` polls.  Returns the status code
    (KDA_ERR_TIMEOUT expected) and the error word the kernel wrote; with
    ``to_library_word`` the bits go to the library's error word instead (read them
    with ``get_error``) and the word returned is None."""
    dev = torch.device(device)
    if to_library_word:
        with torch.cuda.device(dev):
            st = _load().kda_debug_bounded_wait(int(polls), None, _stream(dev))
        return st, None
    word = torch.zeros(1, dtype=torch.int32, device=dev)
    st = _load().kda_debug_bounded_wait(int(polls), _ptr(word), _stream(dev))
    return st, int(word.item())


def debug_prep_image(q, k, log_alpha, beta, gate_scalar=False):
    """Test hook (C ABI ``kda_debug_prep_image``): the tensor-core prep kernel's
    operand images of a fixed-length bf16 batch, uint8 [B*ceil(T/64)*H, 66560]
    (Q e^G and Aqk without the attention scale)."""
    B, T, H, dk = q.shape
    dev = q.device
    _check(q, "q", torch.bfloat16, (B, T, H, 128), dev)
    _check(k, "k", torch.bfloat16, (B, T, H, 128), dev)
    _check(log_alpha, "log_alpha", torch.float32, (B, T, H) if gate_scalar else (B, T, H, 128), dev)
    _check(beta, "beta", torch.float32, (B, T, H), dev)
    n = B * ((T + 63) // 64) * H
    image = torch.zeros((n, IMAGE_BYTES), dtype=torch.uint8, device=dev)
    st = _load().kda_debug_prep_image(_ptr(q), _ptr(k), _ptr(log_alpha), _ptr(beta), _ptr(image),
                                      B, T, H, 1 if gate_scalar else 0, _stream(dev))
    if st != KDA_OK:
        raise KDAError(st, "kda_debug_prep_image")
    return image
