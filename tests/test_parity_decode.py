"""GPU parity: kda_recurrent_step (through the C ABI) vs the fp64 oracle.

The decode step is the fused recurrent form (Kimi Linear paper notes,
section 3: the mode used for short queries outside training).
"""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_recurrent_step
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run_steps(N, H, dk, dv, dtype, steps, seed, s0_std=0.02, gate="softplus8"):
    state0 = W.decode_initial_state(N, H, dk, dv, seed=seed, std=s0_std)
    state = state0.to(DEV)
    ref_state = state0.double()
    for t in range(steps):
        q, k, v, g, b = W.decode_tokens(t, N, H, dk, dv, dtype, seed=seed, gate=gate)
        o = kda_recurrent_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), state)
        o_ref, ref_state = oracle.decode_step(q, k, v, g, b, ref_state)
        assert_close(o, o_ref, dtype, f"o step {t}")
    torch.cuda.synchronize()
    assert_close(state, ref_state, torch.float32 if dtype == torch.float32 else dtype,
                 "final state")


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_shapes(dk, dv, dtype):
    _run_steps(N=3, H=5, dk=dk, dv=dv, dtype=dtype, steps=6, seed=11)


def test_decode_strong_decay_and_zero_state():
    # g far below the prefill range: the decode path takes exp(g) directly
    N, H, d = 2, 3, 128
    state = torch.zeros(N, H, d, d, device=DEV)
    ref = torch.zeros(N, H, d, d, dtype=torch.float64)
    for t in range(4):
        q, k, v, g, b = W.decode_tokens(t, N, H, d, d, torch.bfloat16, seed=5)
        g = g * 200.0
        o = kda_recurrent_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), state)
        o_ref, ref = oracle.decode_step(q, k, v, g, b, ref)
        assert_close(o, o_ref, torch.bfloat16, f"o step {t}")
    assert_close(state, ref, torch.bfloat16, "state")


def test_decode_full_batch_sampled():
    """The full decode workload (256 sequences x 32 heads, d = 128, bf16):
    all pairs for 16 steps against the oracle, then 64 seeded (seq, head)
    pairs carried for 128 more steps."""
    N, H, d = W.DECODE_N, W.DECODE_H, W.DECODE_D
    state0 = W.decode_initial_state()
    state = state0.to(DEV)
    ref = state0.double()
    for t in range(16):
        q, k, v, g, b = W.decode_tokens(t)
        o = kda_recurrent_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), state)
        o_ref, ref = oracle.decode_step(q, k, v, g, b, ref)
        assert_close(o, o_ref, torch.bfloat16, f"o step {t}")
    gen = torch.Generator().manual_seed(99)
    pairs = torch.randperm(N * H, generator=gen)[:64]
    ns, hs = pairs // H, pairs % H
    ref_s = ref[ns, hs]                         # [64, d, d]
    for t in range(16, 144):
        q, k, v, g, b = W.decode_tokens(t)
        o = kda_recurrent_step(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), state)
        o_ref, ref_s4 = oracle.decode_step(q[ns, hs][:, None], k[ns, hs][:, None],
                                           v[ns, hs][:, None], g[ns, hs][:, None],
                                           b[ns, hs][:, None], ref_s[:, None])
        ref_s = ref_s4[:, 0]
        assert_close(o[ns, hs], o_ref[:, 0], torch.bfloat16, f"o step {t}")
    assert_close(state[ns, hs], ref_s, torch.bfloat16, "sampled states")


def test_decode_repeated_equals_prefill_oracle():
    """T decode steps from S_0 give the prefill recurrence's outputs/state."""
    N, H, d, T = 2, 2, 64, 20
    gen = torch.Generator().manual_seed(3)
    q, k, v, g, b = W.draw_tokens(gen, (N, T, H), d, d, torch.float32)
    s0 = torch.randn(N, H, d, d, generator=gen) * 0.1
    o_ref, s_ref = oracle.forward(q, k, v, g, b, s0)
    state = s0.to(DEV)
    for t in range(T):
        o = kda_recurrent_step(q[:, t].contiguous().to(DEV), k[:, t].contiguous().to(DEV),
                               v[:, t].contiguous().to(DEV), g[:, t].contiguous().to(DEV),
                               b[:, t].contiguous().to(DEV), state)
        assert_close(o, o_ref[:, t], torch.float32, f"o[{t}]")
    assert_close(state, s_ref, torch.float32, "state")
