"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every function include/kda.h declares, and
reject bad arguments synchronously (before any CUDA call) with the status the
header documents.
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_88_b200 as kda
from gated_delta_rule_88_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(kda_\w+)\s*\(", src, flags=re.M)
    return names


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("kda_chunk_fwd", "kda_chunk_fwd_ex", "kda_chunk_fwd_host", "kda_recurrent_step",
              "kda_recurrent_step_ex", "kda_recurrent_steps", "kda_gated_rmsnorm",
              "kda_status_string",
              "kda_get_device_error", "kda_last_error_message", "kda_version"):
        assert n in names


def test_every_computing_entry_point_has_a_binding_of_the_same_name():
    """The Python package binds every entry point of the C ABI that computes
    (the status helpers are used internally), under the same name, and each
    refuses CPU tensors instead of computing on the host."""
    import torch
    helpers = {"kda_status_string", "kda_last_error_message", "kda_version"}
    for n in declared_functions():
        if n in helpers:
            continue
        assert hasattr(kda, n) and n in kda.__all__, f"{n} has no Python binding"
    x = torch.zeros(1, 4, 1, 128)
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_chunk_fwd_noalloc(x, x, x, x, torch.zeros(1, 4, 1))


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_status_strings(lib):
    assert lib.kda_status_string(0) == b"KDA_OK"
    assert lib.kda_status_string(1) == b"KDA_ERR_INVALID_ARG"
    assert lib.kda_status_string(2) == b"KDA_ERR_UNSUPPORTED"
    assert lib.kda_version().decode().count(".") == 2


FAKE = 0x10000  # a 16-byte aligned fake device address; never dereferenced


def chunk(lib, *, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, s0=None, cu=None, out=FAKE,
          sT=None, B=1, T=64, H=1, dk=128, dv=128, N=1, dtype=1):
    P = ctypes.c_void_p
    return lib.kda_chunk_fwd(P(q), P(k), P(v), P(g), P(b), P(s0), P(cu), P(out), P(sT),
                             B, T, H, dk, dv, N, dtype, None)


def step(lib, *, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, s=FAKE, out=FAKE, N=1, H=1,
         dk=128, dv=128, dtype=1):
    P = ctypes.c_void_p
    return lib.kda_recurrent_step(P(q), P(k), P(v), P(g), P(b), P(s), P(out), N, H, dk, dv,
                                  dtype, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "b", "out"])
def test_chunk_null_pointer_rejected(lib, field):
    assert chunk(lib, **{field: 0}) == 1
    assert b"null" in lib.kda_last_error_message()


@pytest.mark.parametrize("kw", [dict(B=0), dict(T=-1), dict(H=0), dict(dk=0), dict(dv=-3),
                                dict(dtype=7), dict(B=2, cu=FAKE, N=2),
                                dict(cu=FAKE, N=0), dict(q=FAKE + 8), dict(s0=FAKE + 4),
                                dict(cu=FAKE + 2, N=1), dict(b=FAKE + 2), dict(B=70000),
                                dict(T=1 << 30, B=4)])
def test_chunk_bad_arguments_rejected(lib, kw):
    assert chunk(lib, **kw) == 1


@pytest.mark.parametrize("kw", [dict(dk=96, dv=96), dict(dk=32, dv=64), dict(dk=128, dv=256),
                                dict(dtype=0, dk=32, dv=64), dict(dtype=0, dk=128, dv=256)])
def test_chunk_unsupported_rejected(lib, kw):
    assert chunk(lib, **kw) == 2


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "b", "s", "out"])
def test_step_null_pointer_rejected(lib, field):
    assert step(lib, **{field: 0}) == 1


@pytest.mark.parametrize("kw", [dict(N=-1), dict(H=0), dict(dtype=5), dict(s=FAKE + 8), dict(b=FAKE + 1),
                                dict(N=1 << 20, H=1 << 12)])
def test_step_bad_arguments_rejected(lib, kw):
    assert step(lib, **kw) == 1


@pytest.mark.parametrize("kw", [dict(dk=32), dict(dv=96), dict(dk=256, dv=256)])
def test_step_unsupported_rejected(lib, kw):
    assert step(lib, **kw) == 2


def test_step_empty_batch_is_a_no_op(lib):
    assert step(lib, N=0) == 0


def steps(lib, *, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, pool=FAKE, slots=None, S=4, out=FAKE,
          N=1, L=2, H=1, dk=128, dv=128, dtype=1, flags=0, q_scale=1.0):
    P = ctypes.c_void_p
    return lib.kda_recurrent_steps(P(q), P(k), P(v), P(g), P(b), P(pool), P(slots), S, P(out),
                                   N, L, H, dk, dv, dtype, flags, q_scale, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "b", "pool", "out"])
def test_steps_null_pointer_rejected(lib, field):
    assert steps(lib, **{field: 0}) == 1


@pytest.mark.parametrize("kw", [dict(N=-1), dict(L=0), dict(H=0), dict(S=0), dict(N=5, S=4),
                                dict(dtype=3), dict(pool=FAKE + 8), dict(b=FAKE + 1),
                                dict(slots=FAKE + 2), dict(N=1 << 20, H=1 << 12),
                                dict(flags=8), dict(flags=0xFFFFFFFF), dict(q_scale=float("nan")),
                                dict(q_scale=float("inf"))])
def test_steps_bad_arguments_rejected(lib, kw):
    assert steps(lib, **kw) == 1


def test_steps_slots_allow_a_pool_smaller_than_the_batch(lib):
    # with a slot array the pool size is independent of N (checked on device)
    assert steps(lib, N=0, S=1, slots=FAKE) == 0


@pytest.mark.parametrize("kw", [dict(dk=32), dict(dv=96)])
def test_steps_unsupported_rejected(lib, kw):
    assert steps(lib, **kw) == 2


def host(lib, *, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, s0=None, cu=None, out=FAKE, sT=None,
         B=1, T=64, H=1, dk=128, dv=128, N=1, dtype=1, rt=0):
    P = ctypes.c_void_p
    cu_arr = None if cu is None else (ctypes.c_int32 * len(cu))(*cu)
    return lib.kda_chunk_fwd_host(P(q), P(k), P(v), P(g), P(b), P(s0), cu_arr, P(out), P(sT), B,
                                  T, H, dk, dv, N, dtype, rt, None)


@pytest.mark.parametrize("kw", [dict(flags=8), dict(flags=4), dict(flags=0xFFFFFFFF),
                                dict(q_scale=float("nan")), dict(q_scale=float("-inf"))])
def test_ex_prologue_arguments_rejected(lib, kw):
    P = ctypes.c_void_p
    flags, q_scale = kw.get("flags", 1), kw.get("q_scale", 1.0)
    assert lib.kda_chunk_fwd_ex(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None, P(FAKE),
                                None, 1, 64, 1, 128, 128, 1, 1, flags, q_scale, None) == 1
    assert lib.kda_recurrent_step_ex(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                     1, 1, 128, 128, 1, flags, q_scale, None) == 1


def norm(lib, *, x=FAKE, z=FAKE, w=FAKE, eps=1e-5, out=FAKE, rows=4, dv=128, dtype=1):
    P = ctypes.c_void_p
    return lib.kda_gated_rmsnorm(P(x), P(z), P(w), eps, P(out), rows, dv, dtype, None)


@pytest.mark.parametrize("kw", [dict(x=0), dict(z=0), dict(w=0), dict(out=0), dict(rows=-1),
                                dict(dtype=4), dict(eps=-1.0), dict(eps=float("nan")),
                                dict(x=FAKE + 8), dict(w=FAKE + 2)])
def test_norm_bad_arguments_rejected(lib, kw):
    assert norm(lib, **kw) == 1


def test_norm_unsupported_rejected(lib):
    assert norm(lib, dv=96) == 2


def test_norm_empty_is_a_no_op(lib):
    assert norm(lib, rows=0) == 0


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "b", "out"])
def test_host_null_pointer_rejected(lib, field):
    assert host(lib, **{field: 0}) == 1


@pytest.mark.parametrize("kw", [dict(B=0), dict(T=-1), dict(H=0), dict(rt=-64), dict(dtype=9),
                                dict(B=70000), dict(T=1 << 30, B=4)])
def test_host_bad_arguments_rejected(lib, kw):
    assert host(lib, **kw) == 1


@pytest.mark.parametrize("kw", [dict(cu=[1, 64], N=1), dict(cu=[0, 32], N=1), dict(cu=[0, 40, 30, 64], N=3),
                                dict(cu=[0, 64], N=0), dict(cu=[0, 64], N=1, B=2)])
def test_host_bad_varlen_offsets_rejected(lib, kw):
    # cu_seqlens is a host array here: it is checked in full before any CUDA call
    assert host(lib, **kw) == 1


@pytest.mark.parametrize("kw", [dict(dk=96, dv=96), dict(dtype=0, dk=32, dv=64)])
def test_host_unsupported_rejected(lib, kw):
    assert host(lib, **kw) == 2


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_chunk_fwd(x, x, x, x, torch.zeros(1, 4, 1))
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_recurrent_step(x[0], x[0], x[0], x[0], torch.zeros(4, 1), torch.zeros(4, 1, 64, 64))


def affine(lib, *, M=FAKE, B=0, S=FAKE + (1 << 24), out=FAKE + (1 << 25), count=2, dk=128, dv=128):
    P = ctypes.c_void_p
    return lib.kda_state_affine(P(M), P(B), P(S), P(out), count, dk, dv, None)


@pytest.mark.parametrize("kw", [dict(M=0), dict(S=0), dict(out=0), dict(count=-1), dict(dk=0),
                                dict(dv=5000), dict(M=FAKE + 2), dict(B=FAKE + 6),
                                dict(out=FAKE + (1 << 24) + 64), dict(out=FAKE + 4)])
def test_affine_bad_arguments_rejected(lib, kw):
    assert affine(lib, **kw) == 1


def test_affine_empty_is_a_no_op(lib):
    assert affine(lib, count=0) == 0


def bwd(lib, *, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, s0=None, do=FAKE, dsT=None, dq=FAKE,
        dk=FAKE, dv=FAKE, dg=FAKE, db=FAKE, ds0=None, B=1, T=8, H=1, d_k=128, d_v=128, dtype=1):
    P = ctypes.c_void_p
    return lib.kda_recurrent_bwd(P(q), P(k), P(v), P(g), P(b), P(s0), P(do), P(dsT), P(dq), P(dk),
                                 P(dv), P(dg), P(db), P(ds0), B, T, H, d_k, d_v, dtype, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "b", "do", "dq", "dk", "dv", "dg", "db"])
def test_bwd_null_pointer_rejected(lib, field):
    assert bwd(lib, **{field: 0}) == 1


@pytest.mark.parametrize("kw", [dict(B=0), dict(T=0), dict(H=-1), dict(dtype=5), dict(q=FAKE + 4),
                                dict(db=FAKE + 2), dict(s0=FAKE + 8), dict(B=70000)])
def test_bwd_bad_arguments_rejected(lib, kw):
    assert bwd(lib, **kw) == 1


@pytest.mark.parametrize("kw", [dict(d_k=32), dict(d_v=96), dict(d_k=256)])
def test_bwd_unsupported_rejected(lib, kw):
    assert bwd(lib, **kw) == 2


def cbwd(lib, *, q=FAKE, k=FAKE, v=FAKE, g=FAKE, b=FAKE, s0=None, cu=None, do=FAKE, dsT=None,
         dq=FAKE, dk=FAKE, dv=FAKE, dg=FAKE, db=FAKE, ds0=None, B=1, T=8, H=1, d_k=128, d_v=128,
         N=1, dtype=1):
    P = ctypes.c_void_p
    return lib.kda_chunk_bwd(P(q), P(k), P(v), P(g), P(b), P(s0), P(cu), P(do), P(dsT), P(dq),
                             P(dk), P(dv), P(dg), P(db), P(ds0), B, T, H, d_k, d_v, N, dtype, None)


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "b", "do", "dq", "dk", "dv", "dg", "db"])
def test_chunk_bwd_null_pointer_rejected(lib, field):
    assert cbwd(lib, **{field: 0}) == 1


@pytest.mark.parametrize("kw", [dict(B=0), dict(T=-1), dict(H=-1), dict(dtype=5), dict(q=FAKE + 4),
                                dict(db=FAKE + 2), dict(s0=FAKE + 8), dict(B=70000),
                                dict(cu=FAKE, B=2), dict(cu=FAKE, N=0), dict(cu=FAKE + 2)])
def test_chunk_bwd_bad_arguments_rejected(lib, kw):
    assert cbwd(lib, **kw) == 1


@pytest.mark.parametrize("kw", [dict(d_k=64), dict(d_v=64), dict(dtype=0)])
def test_chunk_bwd_unsupported_rejected(lib, kw):
    assert cbwd(lib, **kw) == 2


def test_saved_bytes_rule(lib):
    lib.kda_chunk_saved_bytes.restype = ctypes.c_longlong
    per = 74240 + 32768 + 16384
    # dense: B * ceil(T / 64) chunk slots per head, plus the 256-byte plan
    assert lib.kda_chunk_saved_bytes(2, 130, 3, 0, 0) == 256 + 2 * 3 * 3 * per
    # varlen: ceil(T / 64) + num_seqs slots
    assert lib.kda_chunk_saved_bytes(1, 300, 2, 4, 1) == 256 + (5 + 4) * 2 * per
    for bad in ((0, 64, 1, 0, 0), (1, -1, 1, 0, 0), (2, 64, 1, 3, 1), (1, 64, 1, 0, 1)):
        assert lib.kda_chunk_saved_bytes(*bad) == -1


def save_fwd(lib, *, saved=FAKE, nbytes=1 << 30, T=64, dtype=1, dk=128):
    P = ctypes.c_void_p
    lib.kda_chunk_fwd_save.argtypes = [P] * 9 + [ctypes.c_int] * 7 + [P, ctypes.c_longlong, P]
    return lib.kda_chunk_fwd_save(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None, P(FAKE),
                                  None, 1, T, 1, dk, 128, 1, dtype, P(saved), nbytes, None)


@pytest.mark.parametrize("kw,code", [(dict(saved=0), 1), (dict(saved=FAKE + 16), 1),
                                     (dict(nbytes=1000), 1), (dict(dtype=0), 2), (dict(dk=64), 2)])
def test_save_fwd_bad_arguments_rejected(lib, kw, code):
    assert save_fwd(lib, **kw) == code
