"""GPU parity: kda_recurrent_bwd (gradients of the recurrence, for training)
vs the fp64 oracle's backward (autograd through the recurrence, pinned by
finite differences).  The kernel computes in fp32 from the exact (widened)
inputs, so the bound is an fp32 rounding bound: ||x - ref||_inf / ||ref||_inf
<= 2e-3 per gradient tensor, for bf16 and fp32 inputs alike.  Lengths cover
one token, partial and whole 8-token blocks and several blocks."""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_recurrent_bwd
from gated_delta_rule_88_b200 import workloads as W
from helpers import rel_inf

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-3


def _check(B, T, H, d, dtype, seed, with_s0=True, with_dsT=True, gate="softplus8"):
    inp = W.prefill(B, T, H, d, d, dtype, seed=seed, gate=gate,
                    initial_state_std=0.05 if with_s0 else None)
    gen = torch.Generator().manual_seed(seed + 7)
    do = torch.randn(B, T, H, d, generator=gen).to(dtype)
    dsT = torch.randn(B, H, d, d, generator=gen) * 0.1 if with_dsT else None
    dd = inp.to(DEV)
    got = kda_recurrent_bwd(dd.q, dd.k, dd.v, dd.g, dd.beta, do.to(DEV), dd.initial_state,
                            None if dsT is None else dsT.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.backward(inp.q, inp.k, inp.v, inp.g, inp.beta, do, inp.initial_state, dsT)
    for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta", "ds0"), got, ref):
        assert torch.isfinite(x).all(), name
        e = rel_inf(x, r)
        assert e <= TOL, f"{name}: relative inf-norm error {e:.3e}"


@pytest.mark.parametrize("T", [1, 7, 8, 9, 33])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_backward_d128(T, dtype):
    _check(B=2, T=T, H=2, d=128, dtype=dtype, seed=200 + T)


@pytest.mark.parametrize("with_s0,with_dsT", [(False, False), (True, False), (False, True)])
def test_backward_optional_states(with_s0, with_dsT):
    _check(B=1, T=20, H=3, d=64, dtype=torch.bfloat16, seed=210, with_s0=with_s0,
           with_dsT=with_dsT)


def test_backward_offset_gates_and_longer_sequence():
    _check(B=1, T=100, H=2, d=128, dtype=torch.bfloat16, seed=211, gate="offset16")
