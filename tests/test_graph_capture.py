"""The device entry points inside a CUDA graph.

A serving loop replays one captured graph per step instead of launching
kernels from Python.  This needs every call on the path to be stream-ordered
with no allocation and no host synchronisation: kda_recurrent_step,
kda_recurrent_steps and kda_chunk_fwd_noalloc are.  Each test captures a few
calls, replays the graph, and requires the result to equal the same calls
run eagerly, bit for bit (same kernels, same inputs).
"""
import ctypes

import pytest
import torch

import gated_delta_rule_88_b200 as kda
from gated_delta_rule_88_b200 import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _capture(fn):
    """Run fn once eagerly on a side stream (one-time launcher set-up stays
    outside the capture), then capture it into a graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_steps_graph_equals_eager():
    N, H, d, steps = 6, 4, 128, 5
    s0 = W.decode_initial_state(N, H, d, d, seed=81).to(DEV)
    toks = [tuple(t.to(DEV) for t in W.decode_tokens(i, N, H, d, d, seed=81)) for i in range(steps)]
    out_g = torch.empty(steps, N, H, d, dtype=torch.bfloat16, device=DEV)
    state_g = s0.clone()

    def run():
        for i, (q, k, v, g, b) in enumerate(toks):
            kda.kda_recurrent_step(q, k, v, g, b, state_g, out_g[i])

    graph = _capture(run)
    state_g.copy_(s0)
    graph.replay()
    torch.cuda.synchronize()
    assert kda.kda_get_device_error() == 0

    state_e = s0.clone()
    out_e = torch.stack([kda.kda_recurrent_step(q, k, v, g, b, state_e) for (q, k, v, g, b) in toks])
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e)
    assert torch.equal(state_g, state_e)


def test_serving_decode_graph_equals_eager():
    N, L, H, d, pool_n = 5, 8, 3, 128, 9
    pool0 = W.decode_initial_state(pool_n, H, d, d, seed=82)
    slots = torch.randperm(pool_n, generator=torch.Generator().manual_seed(82))[:N].to(torch.int32).to(DEV)
    st = [W.decode_tokens(l, N, H, d, d, seed=82) for l in range(L)]
    q, k, v, g, b = [torch.stack([s[i] for s in st], dim=1).contiguous().to(DEV) for i in range(5)]
    pool_g = pool0.to(DEV)
    out_g = torch.empty(N, L, H, d, dtype=torch.bfloat16, device=DEV)
    graph = _capture(lambda: kda.kda_recurrent_steps(q, k, v, g, b, pool_g, slots, out=out_g))
    pool_g.copy_(pool0.to(DEV))
    graph.replay()
    graph.replay()      # two calls: 16 tokens
    torch.cuda.synchronize()
    assert kda.kda_get_device_error() == 0

    pool_e = pool0.to(DEV)
    kda.kda_recurrent_steps(q, k, v, g, b, pool_e, slots)
    out_e = kda.kda_recurrent_steps(q, k, v, g, b, pool_e, slots)
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e)
    assert torch.equal(pool_g, pool_e)


def test_noalloc_prefill_graph_equals_eager():
    lib = kda.load_library()
    f = lib.kda_chunk_fwd_noalloc
    f.argtypes = [ctypes.c_void_p] * 9 + [ctypes.c_int] * 7 + [ctypes.c_void_p]
    f.restype = ctypes.c_int
    inp = W.prefill(1, 1000, 4, 128, 128, torch.bfloat16, seed=83, initial_state_std=0.02).to(DEV)
    B, T, H, dk = inp.q.shape

    def call(out, sT):
        P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = f(P(inp.q), P(inp.k), P(inp.v), P(inp.g), P(inp.beta), P(inp.initial_state), None,
               P(out), P(sT), B, T, H, dk, dk, B, 1, stream)
        assert rc == 0, kda.load_library().kda_last_error_message()

    out_g = torch.empty(B, T, H, dk, dtype=torch.bfloat16, device=DEV)
    s_g = torch.empty(B, H, dk, dk, dtype=torch.float32, device=DEV)
    graph = _capture(lambda: call(out_g, s_g))
    out_g.zero_()
    s_g.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert kda.kda_get_device_error() == 0

    out_e = torch.empty_like(out_g)
    s_e = torch.empty_like(s_g)
    call(out_e, s_e)
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_e)
    assert torch.equal(s_g, s_e)
