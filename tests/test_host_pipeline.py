"""GPU: kda_chunk_fwd_host (host buffers, copies pipelined over token ranges)
gives exactly what kda_chunk_fwd gives on device buffers.

The sequence is cut into ranges of whole chunks, each resuming from the fp32
state the previous range left on the device (the checkpoint semantics of the
whoami-wesleyyou blog, "context modification and checkpoint"), so the chunk
grid and hence every rounding step equal those of one call over the whole
sequence: the comparison is bitwise.
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
    s0 = inp.initial_state
    o_h, s_h = kda_chunk_fwd_host(*host, initial_state=None if s0 is None else s0.contiguous(),
                                  range_tokens=range_tokens)
    torch.cuda.synchronize()
    d = [t.to(DEV) for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
    o_d, s_d = kda_chunk_fwd(*d, initial_state=None if s0 is None else s0.to(DEV))
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
