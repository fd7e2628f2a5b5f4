"""kda_chunk_fwd_noalloc: the prefill entry point for callers that cannot
allocate device memory (for instance a plugin inside an engine that owns all
device memory).  It runs the same kernels as kda_chunk_fwd over a fixed
32 MiB scratch array inside the library instead of pool memory.

The GPU test calls it through the C ABI twice in a row, on different inputs
(so the second call starts from the first call's leftovers in the shared
array), and requires each result to be bitwise equal to kda_chunk_fwd's: both
entry points run the same kernels with the same launch shapes, only the
scratch memory differs.  It also checks that the second call leaves the
device's free memory unchanged (the first call may load the module that holds
the array; later calls allocate nothing).  This file is collected last.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_88_b200 as kda
from gated_delta_rule_88_b200 import build as kbuild
from gated_delta_rule_88_b200 import workloads as W

BF = torch.bfloat16


def _lib():
    kbuild.build()
    lib = kda.load_library()
    f = lib.kda_chunk_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7 + [ctypes.c_void_p]
    f.restype = ctypes.c_int
    return lib


def _noalloc(lib, inp, out, sT):
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    B, T, H, dk = inp.q.shape
    N = B if inp.cu_seqlens is None else inp.cu_seqlens.numel() - 1
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.kda_chunk_fwd_noalloc(P(inp.q), P(inp.k), P(inp.v), P(inp.g), P(inp.beta),
                                     P(inp.initial_state), P(inp.cu_seqlens), P(out), P(sT),
                                     B, T, H, dk, inp.v.shape[-1], N, 1, stream)


def test_noalloc_rejects_oversize_before_touching_the_gpu():
    lib = _lib()
    FAKE = 0x10000
    P = ctypes.c_void_p
    # T = 8192, H = 32: 4096 (chunk, head) slots x 74240 B > 32 MiB
    rc = lib.kda_chunk_fwd_noalloc(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None,
                                   P(FAKE), None, 1, 8192, 32, 128, 128, 1, 1, None)
    assert rc == 1
    assert b"static maximum" in lib.kda_last_error_message()
    rc = lib.kda_chunk_fwd_noalloc(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None,
                                   P(FAKE), None, 1, 64, 1, 64, 64, 1, 1, None)
    assert rc == 2


@pytest.mark.gpu
def test_noalloc_matches_pool_entry_point_twice():
    lib = _lib()
    dev = "cuda"
    cases = [
        # varlen, per-sequence initial states, ragged tails (3 + 4 + 2 chunks x 8 heads)
        W.prefill(1, 0, 8, 128, 128, BF, seed=41, initial_state_std=0.02,
                  seq_lens=[150, 200, 100]),
        # dense, fewer heads, zero initial state: leaves stale records behind
        W.prefill(2, 130, 3, 128, 128, BF, seed=42),
    ]
    for i, inp in enumerate(cases):
        d = inp.to(dev)
        ref_o, ref_s = kda.kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state,
                                         d.cu_seqlens)
        out = torch.full_like(ref_o, float("nan"))
        sT = torch.full_like(ref_s, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        rc = _noalloc(lib, d, out, sT)
        assert rc == 0, lib.kda_last_error_message()
        torch.cuda.synchronize()
        if i > 0:
            assert torch.cuda.mem_get_info()[0] == free_before, "the call changed free device memory"
        assert kda.kda_get_device_error() == 0
        assert torch.equal(out, ref_o), f"call {i}: o differs from kda_chunk_fwd"
        assert torch.equal(sT, ref_s), f"call {i}: final state differs from kda_chunk_fwd"
