"""Kimi Delta Attention (KDA) token mixer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/kda.h`` (``libkda_b200.so``):
argument marshalling only.  Tensors must be CUDA tensors; every step of the
computation runs in the library's kernels.  There is no CPU path: if the
shared library is missing or cannot be loaded, calls raise.

Entry points (same names as the C ABI):
    kda_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None,
                  out=None, final_state=None, output_final_state=True)
        -> (out, final_state or None)
    kda_recurrent_step(q, k, v, g, beta, state, out=None) -> out
    kda_recurrent_steps(q, k, v, g, beta, state_pool, slots=None, out=None,
                        flags=0, q_scale=1.0) -> out
    kda_chunk_fwd_ex(..., flags=0, q_scale=1.0), kda_recurrent_step_ex(..., flags=0,
                     q_scale=1.0): with the in-kernel input prologue
                     (KDA_QK_L2NORM, KDA_BETA_SIGMOID)
    kda_chunk_fwd_host(q, k, v, g, beta, initial_state=None, cu_seqlens=None, out=None,
                       final_state=None, output_final_state=True, range_tokens=0)
        -> (out, final_state or None)   (CPU tensors; valid after the stream syncs)
    kda_chunk_fwd_noalloc(...): kda_chunk_fwd over the library's fixed
                     scratch array (bf16, dk = dv = 128; pass out and
                     final_state to keep the call free of allocations)
    kda_gated_rmsnorm(x, gate, weight, eps=1e-5, out=None) -> out
    kda_recurrent_bwd(q, k, v, g, beta, do, initial_state=None, dsT=None)
        -> (dq, dk, dv, dg, dbeta, ds0)
    kda_chunk_fwd_save(q, k, v, g, beta, initial_state=None, cu_seqlens=None, ...)
        -> (out, final_state, saved): kda_chunk_fwd that also keeps the
        intermediates for the backward (a uint8 CUDA tensor)
    kda_chunk_bwd(..., cu_seqlens=None, saved=None): the same gradients by the chunked form
                     (bf16, dk = dv = 128; tensor cores)
    kda_state_affine(M, B, S_in, out=None) -> S_out
    kda_get_device_error(stream=None) -> int
    kda_selftest_bounded_wait(limit=1000): one CTA's bounded wait that always
                     runs out (sets device error code 1; no fault)
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["kda_chunk_fwd", "kda_chunk_fwd_ex", "kda_chunk_fwd_host", "kda_chunk_fwd_noalloc",
           "kda_recurrent_step",
           "kda_recurrent_step_ex", "kda_recurrent_steps", "kda_gated_rmsnorm", "kda_state_affine",
           "kda_recurrent_bwd", "kda_chunk_bwd", "kda_chunk_fwd_save", "kda_chunk_saved_bytes",
           "kda_chunk_bwd_saved",
           "kda_get_device_error", "kda_selftest_bounded_wait",
           "KDAError",
           "KDA_QK_L2NORM", "KDA_BETA_SIGMOID", "KDA_STEPS_CHUNK",
           "library_path", "load_library"]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libkda_b200.so")
_lib = None
_lock = threading.Lock()

KDA_F32, KDA_BF16 = 0, 1
KDA_QK_L2NORM, KDA_BETA_SIGMOID = 1, 2     # input prologue flags (the *_ex calls)
KDA_STEPS_CHUNK = 4                        # kda_recurrent_steps: chunk form on tensor cores
_STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED",
           3: "KDA_ERR_CUDA", 4: "KDA_ERR_DEVICE"}


class KDAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def load_library():
    """Load libkda_b200.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"{library_path} not found: build it with "
                "`python -m gated_delta_rule_88_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(library_path)
        vp, i = ctypes.c_void_p, ctypes.c_int
        lib.kda_chunk_fwd.argtypes = [vp] * 9 + [i] * 7 + [vp]
        lib.kda_chunk_fwd.restype = i
        lib.kda_chunk_fwd_ex.argtypes = [vp] * 9 + [i] * 7 + [ctypes.c_uint, ctypes.c_float, vp]
        lib.kda_chunk_fwd_ex.restype = i
        lib.kda_chunk_fwd_noalloc.argtypes = [vp] * 9 + [i] * 7 + [vp]
        lib.kda_chunk_fwd_noalloc.restype = i
        lib.kda_recurrent_step_ex.argtypes = [vp] * 7 + [i] * 5 + [ctypes.c_uint, ctypes.c_float, vp]
        lib.kda_recurrent_step_ex.restype = i
        lib.kda_recurrent_step.argtypes = [vp] * 7 + [i] * 5 + [vp]
        lib.kda_recurrent_step.restype = i
        lib.kda_recurrent_steps.argtypes = ([vp] * 7 + [i] + [vp] + [i] * 6 +
                                            [ctypes.c_uint, ctypes.c_float, vp])
        lib.kda_recurrent_steps.restype = i
        lib.kda_chunk_fwd_host.argtypes = [vp] * 9 + [i] * 8 + [vp]
        lib.kda_chunk_fwd_host.restype = i
        lib.kda_gated_rmsnorm.argtypes = [vp, vp, vp, ctypes.c_float, vp, ctypes.c_longlong, i, i, vp]
        lib.kda_gated_rmsnorm.restype = i
        lib.kda_state_affine.argtypes = [vp] * 4 + [i] * 3 + [vp]
        lib.kda_recurrent_bwd.argtypes = [vp] * 14 + [i] * 6 + [vp]
        lib.kda_recurrent_bwd.restype = i
        lib.kda_chunk_bwd.argtypes = [vp] * 15 + [i] * 7 + [vp]
        lib.kda_chunk_bwd.restype = i
        ll = ctypes.c_longlong
        lib.kda_chunk_bwd_saved.argtypes = [vp] * 15 + [i] * 7 + [vp, ll, vp]
        lib.kda_chunk_bwd_saved.restype = i
        lib.kda_chunk_fwd_save.argtypes = [vp] * 9 + [i] * 7 + [vp, ll, vp]
        lib.kda_chunk_fwd_save.restype = i
        lib.kda_chunk_saved_bytes.argtypes = [i] * 5
        lib.kda_chunk_saved_bytes.restype = ll
        lib.kda_state_affine.restype = i
        lib.kda_get_device_error.argtypes = [vp, ctypes.POINTER(i)]
        lib.kda_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
        lib.kda_selftest_bounded_wait.restype = i
        lib.kda_get_device_error.restype = i
        lib.kda_last_error_message.restype = ctypes.c_char_p
        lib.kda_status_string.restype = ctypes.c_char_p
        lib.kda_status_string.argtypes = [i]
        lib.kda_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _check(rc: int):
    if rc != 0:
        msg = load_library().kda_last_error_message().decode(errors="replace")
        raise KDAError(rc, msg)


def _dptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _need(t: torch.Tensor, name: str, device, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def kda_chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, out=None,
                  final_state=None, output_final_state: bool = True):
    """Chunkwise KDA prefill.  q,k,g [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H];
    states [N,H,dk,dv] fp32 (N = B, or len(cu_seqlens)-1 in varlen mode)."""
    return _chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                      output_final_state, None)


def kda_chunk_fwd_ex(q, k, v, g, beta, initial_state=None, cu_seqlens=None, out=None,
                     final_state=None, output_final_state: bool = True, flags: int = 0,
                     q_scale: float = 1.0):
    """kda_chunk_fwd with the in-kernel input prologue: flags KDA_QK_L2NORM
    (q, k L2-normalised per token and head), KDA_BETA_SIGMOID (beta given as a
    logit); q is then scaled by q_scale."""
    return _chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                      output_final_state, (int(flags), float(q_scale)))


def kda_chunk_fwd_noalloc(q, k, v, g, beta, initial_state=None, cu_seqlens=None, out=None,
                          final_state=None, output_final_state: bool = True):
    """kda_chunk_fwd through the allocation-free entry point: the library
    allocates nothing (its scratch is a fixed 32 MiB array); bf16 with
    dk = dv = 128.  Pass out (and final_state) to make the whole call
    allocation-free; otherwise they are allocated here, as torch tensors."""
    return _chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
                      output_final_state, None, noalloc=True)


def _chunk_fwd(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state,
               output_final_state, pro, noalloc: bool = False):
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_chunk_fwd needs CUDA tensors (no CPU path)")
    dt = q.dtype
    _dtype_code(q)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dev, dt)
    _need(g, "g", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    if k.shape != q.shape or g.shape != q.shape or v.shape[:3] != q.shape[:3] or beta.shape != q.shape[:3]:
        raise ValueError("shape mismatch among q, k, v, g, beta")
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", dev, torch.int32)
        N = cu_seqlens.numel() - 1
    else:
        N = B
    if initial_state is not None:
        _need(initial_state, "initial_state", dev, torch.float32)
        if tuple(initial_state.shape) != (N, H, dk, dv):
            raise ValueError(f"initial_state must be [{N},{H},{dk},{dv}]")
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=dt, device=dev)
    else:
        _need(out, "out", dev, dt)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    elif final_state is not None:
        _need(final_state, "final_state", dev, torch.float32)
    args = (_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta), _dptr(initial_state),
            _dptr(cu_seqlens), _dptr(out), _dptr(final_state), B, T, H, dk, dv, N, _dtype_code(q))
    with torch.cuda.device(dev):
        if noalloc:
            rc = lib.kda_chunk_fwd_noalloc(*args, _stream_handle(dev))
        elif pro is None:
            rc = lib.kda_chunk_fwd(*args, _stream_handle(dev))
        else:
            rc = lib.kda_chunk_fwd_ex(*args, pro[0], pro[1], _stream_handle(dev))
    _check(rc)
    return out, final_state


def kda_chunk_fwd_host(q, k, v, g, beta, initial_state=None, cu_seqlens=None, out=None,
                       final_state=None, output_final_state: bool = True, range_tokens: int = 0,
                       device=None):
    """kda_chunk_fwd on host (CPU) tensors, dense [B,T,H,*] layouts or (with a
    CPU int32 ``cu_seqlens``) varlen [1,T,H,*]; the copies are pipelined
    against the computation on ``device`` (default: the current CUDA device).
    Pinned tensors overlap; results are valid once the current stream of that
    device has synchronised.  Returns (out, final_state)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    cpu = torch.device("cpu")
    dt = q.dtype
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, cpu, dt)
    _need(g, "g", cpu, torch.float32)
    _need(beta, "beta", cpu, torch.float32)
    N = B
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", cpu, torch.int32)
        N = cu_seqlens.numel() - 1
    if initial_state is not None:
        _need(initial_state, "initial_state", cpu, torch.float32)
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=dt, pin_memory=True)
    else:
        _need(out, "out", cpu, dt)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, pin_memory=True)
    with torch.cuda.device(dev):
        rc = lib.kda_chunk_fwd_host(_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta),
                                    _dptr(initial_state), _dptr(cu_seqlens), _dptr(out),
                                    _dptr(final_state), B, T, H, dk, dv, N, _dtype_code(q),
                                    int(range_tokens), _stream_handle(dev))
    _check(rc)
    return out, final_state


def kda_recurrent_step(q, k, v, g, beta, state, out=None):
    """One decode token per sequence.  q,k,g [N,H,dk]; v [N,H,dv]; beta [N,H];
    state [N,H,dk,dv] fp32 updated in place.  Returns out [N,H,dv]."""
    return _recurrent_step(q, k, v, g, beta, state, out, None)


def kda_recurrent_step_ex(q, k, v, g, beta, state, out=None, flags: int = 0, q_scale: float = 1.0):
    """kda_recurrent_step with the in-kernel input prologue (see kda_chunk_fwd_ex)."""
    return _recurrent_step(q, k, v, g, beta, state, out, (int(flags), float(q_scale)))


def _recurrent_step(q, k, v, g, beta, state, out, pro):
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_recurrent_step needs CUDA tensors (no CPU path)")
    dt = q.dtype
    N, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dev, dt)
    _need(g, "g", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    _need(state, "state", dev, torch.float32)
    if tuple(state.shape) != (N, H, dk, dv):
        raise ValueError(f"state must be [{N},{H},{dk},{dv}]")
    if out is None:
        out = torch.empty(N, H, dv, dtype=dt, device=dev)
    else:
        _need(out, "out", dev, dt)
    args = (_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta), _dptr(state), _dptr(out), N, H,
            dk, dv, _dtype_code(q))
    with torch.cuda.device(dev):
        if pro is None:
            rc = lib.kda_recurrent_step(*args, _stream_handle(dev))
        else:
            rc = lib.kda_recurrent_step_ex(*args, pro[0], pro[1], _stream_handle(dev))
    _check(rc)
    return out


def kda_recurrent_steps(q, k, v, g, beta, state_pool, slots=None, out=None, flags: int = 0,
                        q_scale: float = 1.0):
    """L decode tokens per sequence on a slot-indexed state pool.  q,k,g
    [N,L,H,dk]; v [N,L,H,dv]; beta [N,L,H]; state_pool [S,H,dk,dv] fp32,
    entry slots[n] updated in place (slots: int32 [N] or None for n).
    Returns out [N,L,H,dv]."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_recurrent_steps needs CUDA tensors (no CPU path)")
    dt = q.dtype
    N, L, H, dk = q.shape
    dv = v.shape[-1]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, dev, dt)
    _need(g, "g", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    _need(state_pool, "state_pool", dev, torch.float32)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != (H, dk, dv):
        raise ValueError(f"state_pool must be [S,{H},{dk},{dv}]")
    if slots is not None:
        _need(slots, "slots", dev, torch.int32)
        if tuple(slots.shape) != (N,):
            raise ValueError(f"slots must be [{N}]")
    if out is None:
        out = torch.empty(N, L, H, dv, dtype=dt, device=dev)
    else:
        _need(out, "out", dev, dt)
    with torch.cuda.device(dev):
        rc = lib.kda_recurrent_steps(_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta),
                                     _dptr(state_pool), _dptr(slots), state_pool.shape[0],
                                     _dptr(out), N, L, H, dk, dv, _dtype_code(q), int(flags),
                                     float(q_scale), _stream_handle(dev))
    _check(rc)
    return out


def kda_gated_rmsnorm(x, gate, weight, eps: float = 1e-5, out=None):
    """The layer's output epilogue: x / sqrt(mean(x^2) + eps) * weight *
    sigmoid(gate) over the last dimension (dv = 64 or 128).  x, gate [..., dv]
    in the output dtype; weight [dv] fp32.  out may be x (in place)."""
    lib = load_library()
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("kda_gated_rmsnorm needs CUDA tensors (no CPU path)")
    dv = x.shape[-1]
    _need(x, "x", dev, x.dtype)
    _need(gate, "gate", dev, x.dtype)
    _need(weight, "weight", dev, torch.float32)
    if gate.shape != x.shape or tuple(weight.shape) != (dv,):
        raise ValueError("gate must match x and weight must be [dv]")
    if out is None:
        out = torch.empty_like(x)
    else:
        _need(out, "out", dev, x.dtype)
    rows = x.numel() // dv
    with torch.cuda.device(dev):
        rc = lib.kda_gated_rmsnorm(_dptr(x), _dptr(gate), _dptr(weight), float(eps), _dptr(out),
                                   rows, dv, _dtype_code(x), _stream_handle(dev))
    _check(rc)
    return out


def kda_recurrent_bwd(q, k, v, g, beta, do, initial_state=None, dsT=None,
                      want_initial_state_grad: bool = True):
    """Gradients of the recurrence (dense layout): q,k,g [B,T,H,dk]; v, do
    [B,T,H,dv]; beta [B,T,H]; initial_state, dsT (the final-state gradient)
    [B,H,dk,dv] fp32 or None.  Returns fp32 (dq, dk, dv, dg, dbeta, ds0)
    (ds0 None unless wanted)."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_recurrent_bwd needs CUDA tensors (no CPU path)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    for t, name in ((k, "k"), (v, "v"), (do, "do")):
        _need(t, name, dev, q.dtype)
    _need(q, "q", dev)
    _need(g, "g", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    for t, name in ((initial_state, "initial_state"), (dsT, "dsT")):
        if t is not None:
            _need(t, name, dev, torch.float32)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk_, dg = (torch.empty(B, T, H, dk, **f32) for _ in range(3))
    dv_ = torch.empty(B, T, H, dv, **f32)
    db = torch.empty(B, T, H, **f32)
    ds0 = torch.empty(B, H, dk, dv, **f32) if want_initial_state_grad else None
    with torch.cuda.device(dev):
        rc = lib.kda_recurrent_bwd(_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta),
                                   _dptr(initial_state), _dptr(do), _dptr(dsT), _dptr(dq),
                                   _dptr(dk_), _dptr(dv_), _dptr(dg), _dptr(db), _dptr(ds0),
                                   B, T, H, dk, dv, dt, _stream_handle(dev))
    _check(rc)
    return dq, dk_, dv_, dg, db, ds0


def kda_chunk_saved_bytes(B: int, T: int, H: int, num_seqs: int = 0, varlen: bool = False) -> int:
    """Bytes of the forward intermediates kda_chunk_fwd_save keeps."""
    n = load_library().kda_chunk_saved_bytes(int(B), int(T), int(H), int(num_seqs), int(bool(varlen)))
    if n < 0:
        raise ValueError("kda_chunk_saved_bytes: bad sizes")
    return int(n)


def kda_chunk_fwd_save(q, k, v, g, beta, initial_state=None, cu_seqlens=None, out=None,
                       final_state=None, output_final_state: bool = True, saved=None):
    """kda_chunk_fwd (bf16, dk = dv = 128) that also writes the intermediates
    the chunked backward needs into ``saved`` (allocated here if None).
    Returns (out, final_state, saved); pass ``saved`` to kda_chunk_bwd."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_chunk_fwd_save needs CUDA tensors (no CPU path)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for t, name in ((k, "k"), (v, "v")):
        _need(t, name, dev, q.dtype)
    _need(q, "q", dev)
    _need(g, "g", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    N = B
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", dev, torch.int32)
        N = cu_seqlens.numel() - 1
    if initial_state is not None:
        _need(initial_state, "initial_state", dev, torch.float32)
    nbytes = kda_chunk_saved_bytes(B, T, H, N, cu_seqlens is not None)
    if saved is None:
        saved = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    else:
        _need(saved, "saved", dev, torch.uint8)
    if out is None:
        out = torch.empty(B, T, H, dv, dtype=q.dtype, device=dev)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = lib.kda_chunk_fwd_save(_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta),
                                    _dptr(initial_state), _dptr(cu_seqlens), _dptr(out),
                                    _dptr(final_state), B, T, H, dk, dv, N, _dtype_code(q),
                                    _dptr(saved), saved.numel(), _stream_handle(dev))
    _check(rc)
    return out, final_state, saved


def kda_chunk_bwd(q, k, v, g, beta, do, initial_state=None, dsT=None, cu_seqlens=None,
                  want_initial_state_grad: bool = True, saved=None):
    """Gradients by the chunked form on the tensor cores (bf16, dk = dv = 128):
    arguments and results as kda_recurrent_bwd, plus cu_seqlens (varlen, B == 1;
    states then [N,H,dk,dv]) and ``saved`` (from kda_chunk_fwd_save on the same
    inputs: the forward is then not recomputed)."""
    lib = load_library()
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("kda_chunk_bwd needs CUDA tensors (no CPU path)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    for t, name in ((k, "k"), (v, "v"), (do, "do")):
        _need(t, name, dev, q.dtype)
    _need(q, "q", dev)
    _need(g, "g", dev, torch.float32)
    _need(beta, "beta", dev, torch.float32)
    N = B
    if cu_seqlens is not None:
        _need(cu_seqlens, "cu_seqlens", dev, torch.int32)
        N = cu_seqlens.numel() - 1
    for t, name in ((initial_state, "initial_state"), (dsT, "dsT")):
        if t is not None:
            _need(t, name, dev, torch.float32)
    if saved is not None:
        _need(saved, "saved", dev, torch.uint8)
    f32 = dict(dtype=torch.float32, device=dev)
    dq, dk_, dg = (torch.empty(B, T, H, dk, **f32) for _ in range(3))
    dv_ = torch.empty(B, T, H, dv, **f32)
    db = torch.empty(B, T, H, **f32)
    ds0 = torch.empty(N, H, dk, dv, **f32) if want_initial_state_grad else None
    args = (_dptr(q), _dptr(k), _dptr(v), _dptr(g), _dptr(beta), _dptr(initial_state),
            _dptr(cu_seqlens), _dptr(do), _dptr(dsT), _dptr(dq), _dptr(dk_), _dptr(dv_), _dptr(dg),
            _dptr(db), _dptr(ds0), B, T, H, dk, dv, N, dt)
    with torch.cuda.device(dev):
        if saved is None:
            rc = lib.kda_chunk_bwd(*args, _stream_handle(dev))
        else:
            rc = lib.kda_chunk_bwd_saved(*args, _dptr(saved), saved.numel(), _stream_handle(dev))
    _check(rc)
    return dq, dk_, dv_, dg, db, ds0


def kda_chunk_bwd_saved(q, k, v, g, beta, do, saved, initial_state=None, dsT=None,
                        cu_seqlens=None, want_initial_state_grad: bool = True):
    """kda_chunk_bwd given the intermediates of kda_chunk_fwd_save."""
    return kda_chunk_bwd(q, k, v, g, beta, do, initial_state, dsT, cu_seqlens,
                         want_initial_state_grad, saved=saved)


def kda_state_affine(M, B, S_in, out=None):
    """S_out = M S_in + B per block: M [..., dk, dk]; B (or None), S_in
    [..., dk, dv] fp32 CUDA tensors.  Returns S_out (a new tensor unless out
    is given; out must not overlap S_in or M)."""
    lib = load_library()
    dev = S_in.device
    if dev.type != "cuda":
        raise ValueError("kda_state_affine needs CUDA tensors (no CPU path)")
    dk, dv = S_in.shape[-2], S_in.shape[-1]
    _need(M, "M", dev, torch.float32)
    _need(S_in, "S_in", dev, torch.float32)
    if B is not None:
        _need(B, "B", dev, torch.float32)
        if B.shape != S_in.shape:
            raise ValueError("B must match S_in")
    if M.shape[:-2] != S_in.shape[:-2] or M.shape[-2:] != (dk, dk):
        raise ValueError("M must be [..., dk, dk] over the same blocks as S_in")
    out = torch.empty_like(S_in) if out is None else out
    _need(out, "out", dev, torch.float32)
    count = S_in.numel() // (dk * dv)
    with torch.cuda.device(dev):
        rc = lib.kda_state_affine(_dptr(M), _dptr(B), _dptr(S_in), _dptr(out), count, dk, dv,
                                  _stream_handle(dev))
    _check(rc)
    return out


def kda_get_device_error(stream=None) -> int:
    """Synchronise the stream and read-and-clear the device error word."""
    lib = load_library()
    code = ctypes.c_int(0)
    handle = ctypes.c_void_p(stream.cuda_stream if stream is not None
                             else torch.cuda.current_stream().cuda_stream)
    rc = lib.kda_get_device_error(handle, ctypes.byref(code))
    if rc not in (0, 4):
        _check(rc)
    return code.value


def kda_selftest_bounded_wait(limit: int = 1000, device=None) -> None:
    """Launch one CTA whose bounded mbarrier wait always runs out: it sets the
    device error word to 1 (read it with kda_get_device_error) and returns."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _check(lib.kda_selftest_bounded_wait(int(limit), _stream_handle(dev)))
