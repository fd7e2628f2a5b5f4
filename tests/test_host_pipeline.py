"""GPU: kda_chunk_fwd_host (host buffers, copies pipelined over token ranges)
gives exactly what kda_chunk_fwd gives on device buffers, dense and varlen.

The packed token axis is cut into ranges that end at a sequence end or a whole
number of chunks into a sequence, each resuming its sequences from the fp32
states the previous range left on the device (the checkpoint semantics of the
whoami-wesleyyou blog, "context modification and checkpoint"), so the chunk
grid and hence every rounding step equal those of one call over the whole
batch: the comparison is bitwise.
"""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_chunk_fwd, kda_chunk_fwd_host
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(B, T, H, d, dtype, seed, s0):
    inp = W.prefill(B, T, H, d, d, dtype, seed=seed, gate="softplus8",
                    initial_state_std=0.05 if s0 else None)
    return inp


def _both(inp, range_tokens, pin=True):
    host = [t.contiguous() for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
    if pin:
        host = [t.pin_memory() for t in host]
    s0, cu = inp.initial_state, inp.cu_seqlens
    o_h, s_h = kda_chunk_fwd_host(*host, initial_state=None if s0 is None else s0.contiguous(),
                                  cu_seqlens=cu, range_tokens=range_tokens)
    torch.cuda.synchronize()
    d = [t.to(DEV) for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
    o_d, s_d = kda_chunk_fwd(*d, initial_state=None if s0 is None else s0.to(DEV),
                             cu_seqlens=None if cu is None else cu.to(DEV))
    torch.cuda.synchronize()
    return o_h, s_h, o_d.cpu(), s_d.cpu()


@pytest.mark.parametrize("B,T,rt,s0", [(1, 1000, 256, False), (2, 300, 128, True),
                                        (1, 640, 0, True), (3, 70, 64, False), (1, 200, 4096, False)])
def test_host_pipeline_bitwise_bf16(B, T, rt, s0):
    o_h, s_h, o_d, s_d = _both(_inputs(B, T, 4, 128, torch.bfloat16, seed=41, s0=s0), rt)
    assert torch.equal(o_h, o_d)
    assert torch.equal(s_h, s_d)


def test_host_pipeline_f32_small_heads():
    o_h, s_h, o_d, s_d = _both(_inputs(2, 200, 3, 64, torch.float32, seed=42, s0=True), 64)
    assert torch.equal(o_h, o_d)
    assert torch.equal(s_h, s_d)


def test_host_pipeline_pageable_memory():
    o_h, s_h, o_d, s_d = _both(_inputs(1, 500, 2, 128, torch.bfloat16, seed=43, s0=False), 128,
                               pin=False)
    assert torch.equal(o_h, o_d)
    assert torch.equal(s_h, s_d)


def test_host_pipeline_against_oracle():
    inp = _inputs(1, 333, 2, 128, torch.bfloat16, seed=44, s0=True)
    o_h, s_h = kda_chunk_fwd_host(inp.q.pin_memory(), inp.k.pin_memory(), inp.v.pin_memory(),
                                  inp.g.pin_memory(), inp.beta.pin_memory(),
                                  initial_state=inp.initial_state.pin_memory(), range_tokens=128)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta,
                                  initial_state=inp.initial_state.double())
    assert_close(o_h, o_ref, torch.bfloat16, "o")
    assert_close(s_h, s_ref, torch.bfloat16, "final state")


def test_host_pipeline_without_final_state():
    inp = _inputs(1, 256, 2, 128, torch.bfloat16, seed=45, s0=False)
    o_h, s_h = kda_chunk_fwd_host(inp.q, inp.k, inp.v, inp.g, inp.beta, output_final_state=False,
                                  range_tokens=64)
    torch.cuda.synchronize()
    assert s_h is None
    o_d, _ = kda_chunk_fwd(*[t.to(DEV) for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)])
    assert torch.equal(o_h, o_d.cpu())


@pytest.mark.parametrize("lens,rt,s0", [
    ([300, 0, 129, 64, 1000], 128, True),     # ranges straddle sequences, an empty one inside
    ([0, 700, 1, 0], 256, False),             # empty sequences at both ends, a one-token one
    ([65, 63, 640, 200], 0, True),            # everything in one range
    ([1500, 2100], 64, True),                 # one chunk per range
])
def test_host_pipeline_varlen_bitwise_bf16(lens, rt, s0):
    inp = W.prefill(1, 0, 3, 128, 128, torch.bfloat16, seed=46,
                    initial_state_std=0.05 if s0 else None, seq_lens=lens)
    o_h, s_h, o_d, s_d = _both(inp, rt)
    assert torch.equal(o_h, o_d)
    assert torch.equal(s_h, s_d)


def test_host_pipeline_varlen_f32():
    inp = W.prefill(1, 0, 2, 64, 64, torch.float32, seed=47, initial_state_std=0.05,
                    seq_lens=[100, 0, 37, 250])
    o_h, s_h, o_d, s_d = _both(inp, 64)
    assert torch.equal(o_h, o_d)
    assert torch.equal(s_h, s_d)


def test_host_pipeline_varlen_workload_sampled_against_oracle():
    """The 8-sequence varlen workload through host buffers (the bench's e2e
    call): bitwise equal to the device call, and its first and last sequences
    within the bf16 tolerance of the oracle on two heads."""
    inp = W.named_prefill("varlen8_h32_d128_resume")
    o_h, s_h, o_d, s_d = _both(inp, 0)
    assert torch.equal(o_h, o_d)
    assert torch.equal(s_h, s_d)
    cu = inp.cu_seqlens.tolist()
    for n in (0, len(cu) - 2):
        for h in (3, 30):
            a, b = cu[n], cu[n + 1]
            sl = lambda t: t[:, a:b, h:h + 1].contiguous()
            o_ref, s_ref = oracle.forward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.beta),
                                          initial_state=inp.initial_state[n:n + 1, h:h + 1].double())
            assert_close(o_h[:, a:b, h:h + 1], o_ref, torch.bfloat16, f"o seq {n} head {h}")
            assert_close(s_h[n:n + 1, h:h + 1], s_ref, torch.bfloat16, f"state seq {n} head {h}")
