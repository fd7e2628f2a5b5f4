"""fp64 CPU oracle for the Kimi Delta Attention (KDA) token mixer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg / ``--impl reference`` arm may import this
package.  The product package ``gated_delta_rule_88_b200`` never imports it, and
this package imports nothing from the product package: the two share no code.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64, token by token; see its
header for the cited recurrence).  This module only marshals arguments: it
slices each (sequence, head) out of the caller's tensors, widens them exactly to
fp64, calls the C routine, and scatters the results.  Independent
(sequence, head) recurrences run on a thread pool (ctypes releases the GIL).

Layouts follow the library's C ABI:
  dense : q,k,g [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H]; states [B,H,dk,dv]
  varlen: B == 1, cu_seqlens [N+1] int; states [N,H,dk,dv]
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None
_lib_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into libkda_oracle.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lib_lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            f = lib.kda_oracle_recurrence
            dp = ctypes.POINTER(ctypes.c_double)
            L = ctypes.c_long
            f.argtypes = [L, ctypes.c_int, ctypes.c_int,
                          dp, L, dp, L, dp, L, dp, L, dp, L, dp, dp, L]
            f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recurrence(q, k, v, g, beta, S0=None):
    """One (sequence, head): q,k,g [T,dk]; v [T,dv]; beta [T]; S0 [dk,dv].

    Inputs are any real arrays/tensors; they are widened to fp64.
    Returns (o [T,dv] fp64, S_T [dk,dv] fp64) as numpy arrays.
    """
    lib = _load()
    q = _f64(q); k = _f64(k); v = _f64(v); g = _f64(g); beta = _f64(beta)
    T, dk = q.shape
    dv = v.shape[1]
    assert k.shape == (T, dk) and g.shape == (T, dk) and v.shape == (T, dv)
    assert beta.shape == (T,)
    S = np.zeros((dk, dv)) if S0 is None else _f64(S0).copy()
    assert S.shape == (dk, dv)
    o = np.zeros((T, dv))
    rc = lib.kda_oracle_recurrence(T, dk, dv, _ptr(q), dk, _ptr(k), dk,
                                   _ptr(v), dv, _ptr(g), dk, _ptr(beta), 1,
                                   _ptr(S), _ptr(o), dv)
    if rc != 0:
        raise RuntimeError("kda_oracle_recurrence failed")
    return o, S


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        return np.ascontiguousarray(x.detach().cpu().to(torch.float64).numpy())
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _threads(n_tasks: int, threads: int | None) -> int:
    if threads is None:
        threads = os.cpu_count() or 1
    return max(1, min(threads, n_tasks))


def forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None,
            threads: int | None = None, heads=None, seqs=None,
            want_output: bool = True):
    """Full KDA forward over all (sequence, head) pairs, fp64.

    q,k,g: [B,T,H,dk]; v: [B,T,H,dv]; beta: [B,T,H] (CPU tensors, any dtype).
    initial_state: None (zeros) or [N,H,dk,dv].  cu_seqlens: None (dense, N=B)
    or [N+1] offsets into T with B == 1.
    heads / seqs: optional subsets to evaluate (others left as NaN).
    Returns (o [B,T,H,dv] float64 tensor, final_state [N,H,dk,dv] float64).
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        N = B
        ranges = [(b, 0, T) for b in range(B)]
    else:
        assert B == 1
        cu = [int(x) for x in torch.as_tensor(cu_seqlens).tolist()]
        N = len(cu) - 1
        ranges = [(0, cu[n], cu[n + 1]) for n in range(N)]
    heads = list(range(H)) if heads is None else list(heads)
    seqs = list(range(N)) if seqs is None else list(seqs)
    o = torch.full((B, T, H, dv), float("nan"), dtype=torch.float64)
    sT = torch.full((N, H, dk, dv), float("nan"), dtype=torch.float64)

    def task(n, h):
        b, s, e = ranges[n]
        S0 = None if initial_state is None else initial_state[n, h]
        on, Sn = recurrence(q[b, s:e, h], k[b, s:e, h], v[b, s:e, h],
                            g[b, s:e, h], beta[b, s:e, h], S0)
        if want_output:
            o[b, s:e, h] = torch.from_numpy(on)
        sT[n, h] = torch.from_numpy(Sn)

    jobs = [(n, h) for n in seqs for h in heads]
    with ThreadPoolExecutor(_threads(len(jobs), threads)) as ex:
        for f in [ex.submit(task, n, h) for n, h in jobs]:
            f.result()
    return o, sT


def decode_step(q, k, v, g, beta, state, threads: int | None = None):
    """One recurrent step for N sequences: q,k,g [N,H,dk]; v [N,H,dv];
    beta [N,H]; state [N,H,dk,dv].  Returns (o [N,H,dv], new state), fp64."""
    o, sT = forward(q.unsqueeze(1), k.unsqueeze(1), v.unsqueeze(1),
                    g.unsqueeze(1), beta.unsqueeze(1), initial_state=state,
                    threads=threads)
    return o[:, 0], sT


def prologue(q, k, beta, qk_l2norm: bool = False, beta_sigmoid: bool = False,
             q_scale: float = 1.0):
    """The input prologue of the library's *_ex calls, in fp64, on the values
    as given (bf16 inputs widened exactly).  Kimi Linear paper notes, section 7:
    the layer normalises q and k inside the kernel (use_qk_l2norm_in_kernel)
    and takes beta as the sigmoid of a projection.  Per (token, head):
        q <- q_scale * q / |q|_2,   k <- k / |k|_2      (qk_l2norm; 0 -> 0)
        q <- q_scale * q                                 (otherwise)
        beta <- 1 / (1 + exp(-beta))                     (beta_sigmoid)
    Returns fp64 tensors (q, k, beta) of the same shapes."""
    q64, k64, b64 = q.double(), k.double(), beta.double()
    if qk_l2norm:
        def unit(x):
            n = torch.linalg.vector_norm(x, dim=-1, keepdim=True)
            return torch.where(n > 0, x / torch.where(n > 0, n, torch.ones_like(n)),
                               torch.zeros_like(x))
        q64, k64 = unit(q64), unit(k64)
    q64 = q64 * float(q_scale)
    if beta_sigmoid:
        b64 = 1.0 / (1.0 + torch.exp(-b64))
    return q64, k64, b64


def gated_rmsnorm(x, gate, weight, eps: float):
    """The layer's output epilogue in fp64 (Kimi Linear paper notes, section 7:
    FusedRMSNormGated with a sigmoid output gate), over the last dimension:
        y = x / sqrt(mean(x^2) + eps) * weight * 1 / (1 + exp(-gate))"""
    x64, z64, w64 = x.double(), gate.double(), weight.double()
    r = torch.rsqrt((x64 * x64).mean(dim=-1, keepdim=True) + eps)
    return x64 * r * w64 / (1.0 + torch.exp(-z64))


def state_affine(M, B, S):
    """S_out = M S + B per block in fp64: M [..., dk, dk]; B (or None), S
    [..., dk, dv].  Kimi Linear paper notes, section 2: the recurrence is
    affine in the state, so a segment of tokens acts on its start state as
    such a map (used to check the context-parallel fold)."""
    out = M.double() @ S.double()
    return out if B is None else out + B.double()


def _recurrence_torch(q, k, v, g, beta, S0):
    """The recurrence of ``recurrence`` in plain fp64 torch ops (differentiable).
    One (sequence, head): q,k,g [T,dk]; v [T,dv]; beta [T]; S0 [dk,dv].
    Kimi Linear paper notes, section 2: per token
        S' = Diag(exp g) S;  S = S' + beta k (v - S'^T k)^T;  o = S^T q."""
    S = S0
    outs = []
    for t in range(q.shape[0]):
        Sp = torch.exp(g[t])[:, None] * S
        u = beta[t] * (v[t] - Sp.T @ k[t])
        S = Sp + torch.outer(k[t], u)
        outs.append(S.T @ q[t])
    return torch.stack(outs) if outs else q.new_zeros((0, v.shape[1])), S


def backward(q, k, v, g, beta, do, initial_state=None, dsT=None):
    """Gradients of the forward (dense layout q,k,g [B,T,H,dk]; v [B,T,H,dv];
    beta [B,T,H]; initial_state [B,H,dk,dv] or None) for the output gradient
    do [B,T,H,dv] and the final-state gradient dsT [B,H,dk,dv] (or None = 0):
    returns fp64 (dq, dk, dv, dg, dbeta, ds0) of the inputs' shapes.

    The chain rule through the recurrence of section 2 (``_recurrence_torch``),
    taken by torch autograd in fp64 on the CPU; pinned against central finite
    differences of ``recurrence`` (tests/test_oracle_pins.py)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    outs = {n: torch.zeros(x.shape, dtype=torch.float64) for n, x in
            (("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dbeta", beta))}
    ds0 = torch.zeros(B, H, dk, dv, dtype=torch.float64)
    for b in range(B):
        for h in range(H):
            xs = [x[b, :, h].detach().double().clone().requires_grad_(True) for x in (q, k, v, g)]
            bt = beta[b, :, h].detach().double().clone().requires_grad_(True)
            s0 = (torch.zeros(dk, dv, dtype=torch.float64) if initial_state is None
                  else initial_state[b, h].detach().double().clone())
            s0.requires_grad_(True)
            o, sT = _recurrence_torch(xs[0], xs[1], xs[2], xs[3], bt, s0)
            loss = (o * do[b, :, h].double()).sum()
            if dsT is not None:
                loss = loss + (sT * dsT[b, h].double()).sum()
            grads = torch.autograd.grad(loss, xs + [bt, s0], allow_unused=True)
            for name, gr in zip(("dq", "dk", "dv", "dg", "dbeta"), grads[:5]):
                if gr is not None:
                    outs[name][b, :, h] = gr
            if grads[5] is not None:
                ds0[b, h] = grads[5]
    return outs["dq"], outs["dk"], outs["dv"], outs["dg"], outs["dbeta"], ds0
