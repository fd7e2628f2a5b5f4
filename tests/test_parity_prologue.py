"""GPU parity: the in-kernel input prologue (kda_chunk_fwd_ex,
kda_recurrent_step_ex, kda_recurrent_steps flags) vs the fp64 oracle.

Inputs are raw projections: q and k not normalised (rows of different
scales, one all-zero padding row), beta given as logits.  The expected result
is oracle.prologue (fp64, on the same bf16/fp32 values) followed by the
oracle's recurrence.  Kimi Linear paper notes, section 7: the layer hands raw
projections to the kernels with the q/k L2 norm inside the kernel and beta as
the sigmoid of a projection.
"""
import math

import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import (KDA_BETA_SIGMOID, KDA_QK_L2NORM, kda_chunk_fwd,
                                      kda_chunk_fwd_ex, kda_recurrent_step, kda_recurrent_step_ex,
                                      kda_recurrent_steps)
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
ALL = KDA_QK_L2NORM | KDA_BETA_SIGMOID


def _raw(shape_tok, dk, dv, dtype, seed):
    """Raw per-token inputs: q, k with per-row scales in [0.1, 10) and one zero
    row; v ~ N(0,1); g = -softplus(N(0,1))/8; beta logits ~ N(0,1)."""
    gen = torch.Generator().manual_seed(seed)
    scale = 10.0 ** (torch.rand(*shape_tok, 1, generator=gen) * 2 - 1)
    q = torch.randn(*shape_tok, dk, generator=gen) * scale
    k = torch.randn(*shape_tok, dk, generator=gen) * scale.flip(0)
    v = torch.randn(*shape_tok, dv, generator=gen)
    g = -torch.nn.functional.softplus(torch.randn(*shape_tok, dk, generator=gen)) / 8
    b = torch.randn(*shape_tok, generator=gen)
    q.view(-1, dk)[1] = 0.0                           # a padding row stays zero
    return q.to(dtype), k.to(dtype), v.to(dtype), g.float(), b.float()


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
@pytest.mark.parametrize("flags", [ALL, KDA_QK_L2NORM, KDA_BETA_SIGMOID])
def test_chunk_prologue(dtype, d, flags):
    B, T, H = 2, 200, 3
    q, k, v, g, b = _raw((B, T, H), d, d, dtype, seed=51)
    qs = 1.0 / math.sqrt(d)
    # a step the kernel does not take is done here, so the recurrence sees
    # unit keys and beta in (0, 1) either way
    if not (flags & KDA_QK_L2NORM):
        unit = lambda x: (x.float() / x.float().norm(dim=-1, keepdim=True).clamp_min(1e-30)).to(dtype)
        q, k = unit(q), unit(k)
    if not (flags & KDA_BETA_SIGMOID):
        b = torch.sigmoid(b)
    o, s = kda_chunk_fwd_ex(*[t.to(DEV) for t in (q, k, v, g, b)], flags=flags, q_scale=qs)
    torch.cuda.synchronize()
    qp, kp, bp = oracle.prologue(q, k, b, qk_l2norm=bool(flags & KDA_QK_L2NORM),
                                 beta_sigmoid=bool(flags & KDA_BETA_SIGMOID), q_scale=qs)
    o_ref, s_ref = oracle.forward(qp, kp, v, g, bp)
    assert not torch.isnan(o).any()
    assert_close(o, o_ref, dtype, "o")
    assert_close(s, s_ref, dtype if dtype == torch.bfloat16 else torch.float32, "final state")


def test_chunk_prologue_with_strong_decay_chunks():
    """bf16 prefill with the prologue where chunk 1 of head 0 decays by more
    than e^80 (g = -2 on some channels): that chunk takes the 16-token
    exponent path, the others the chunk-start path, both normalising q, k
    and taking the sigmoid of beta inside the kernel."""
    B, T, H, d = 1, 256, 2, 128
    q, k, v, g, b = _raw((B, T, H), d, d, torch.bfloat16, seed=57)
    g[:, 64:128, 0, ::4] = -2.0
    qs = 1.0 / math.sqrt(d)
    o, s = kda_chunk_fwd_ex(*[t.to(DEV) for t in (q, k, v, g, b)], flags=ALL, q_scale=qs)
    torch.cuda.synchronize()
    qp, kp, bp = oracle.prologue(q, k, b, qk_l2norm=True, beta_sigmoid=True, q_scale=qs)
    o_ref, s_ref = oracle.forward(qp, kp, v, g, bp)
    assert not torch.isnan(o).any()
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(s, s_ref, torch.bfloat16, "final state")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_chunk_prologue_identity_is_bitwise_the_plain_call(dtype):
    from gated_delta_rule_88_b200 import workloads as W
    d = 128 if dtype == torch.bfloat16 else 64
    inp = W.prefill(1, 300, 2, d, d, dtype, seed=52)
    x = [t.to(DEV) for t in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
    o0, s0 = kda_chunk_fwd(*x)
    o1, s1 = kda_chunk_fwd_ex(*x, flags=0, q_scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(o0, o1) and torch.equal(s0, s1)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_decode_step_prologue(dtype, d):
    N, H, steps = 4, 3, 5
    qs = 1.0 / math.sqrt(d)
    gen = torch.Generator().manual_seed(53)
    state0 = torch.randn(N, H, d, d, generator=gen) * 0.02
    state = state0.to(DEV)
    ref = state0.double()
    for t in range(steps):
        q, k, v, g, b = _raw((N, H), d, d, dtype, seed=60 + t)
        o = kda_recurrent_step_ex(*[x.to(DEV) for x in (q, k, v, g, b)], state, flags=ALL,
                                  q_scale=qs)
        qp, kp, bp = oracle.prologue(q, k, b, qk_l2norm=True, beta_sigmoid=True, q_scale=qs)
        o_ref, ref = oracle.decode_step(qp, kp, v, g, bp, ref)
        assert_close(o, o_ref, dtype, f"o step {t}")
    torch.cuda.synchronize()
    assert_close(state, ref, dtype if dtype == torch.bfloat16 else torch.float32, "state")


def test_decode_step_prologue_identity_is_bitwise_the_plain_call():
    q, k, v, g, b = [x.to(DEV) for x in _raw((3, 2), 128, 128, torch.bfloat16, seed=54)]
    q, k = q / 12.0, k / 12.0
    s0 = torch.randn(3, 2, 128, 128, device=DEV) * 0.02
    sa, sb = s0.clone(), s0.clone()
    oa = kda_recurrent_step(q, k, v, g, b, sa)
    ob = kda_recurrent_step_ex(q, k, v, g, b, sb, flags=0, q_scale=1.0)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob) and torch.equal(sa, sb)


def test_decode_steps_prologue():
    N, L, H, d, S = 3, 6, 2, 128, 5
    qs = 1.0 / math.sqrt(d)
    q, k, v, g, b = _raw((N, L, H), d, d, torch.bfloat16, seed=55)
    gen = torch.Generator().manual_seed(56)
    pool0 = torch.randn(S, H, d, d, generator=gen) * 0.02
    slots = torch.tensor([4, 0, 2], dtype=torch.int32)
    pool = pool0.to(DEV)
    out = kda_recurrent_steps(*[x.to(DEV) for x in (q, k, v, g, b)], pool, slots.to(DEV),
                              flags=ALL, q_scale=qs)
    torch.cuda.synchronize()
    qp, kp, bp = oracle.prologue(q, k, b, qk_l2norm=True, beta_sigmoid=True, q_scale=qs)
    o_ref, s_ref = oracle.forward(qp, kp, v, g, bp, initial_state=pool0[slots.long()].double())
    assert_close(out, o_ref, torch.bfloat16, "o")
    assert_close(pool[slots.long().to(DEV)], s_ref, torch.bfloat16, "states")
