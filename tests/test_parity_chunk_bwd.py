"""GPU parity: kda_chunk_bwd (the chunked tensor-core backward) vs the fp64
oracle's backward (autograd through the recurrence, pinned by finite
differences).  The products take bf16 operands with fp32 accumulation, like
the bf16 forward, so the bound is the forward's: ||x - ref||_inf /
||ref||_inf <= 2e-2 per gradient tensor (a CPU replay of the rounding points
gives 1.5-4e-3 on an 8192-token head).  Lengths cover one token, a partial
chunk, whole chunks and ragged tails over several chunks."""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_chunk_bwd, kda_get_device_error, kda_recurrent_bwd
from gated_delta_rule_88_b200 import workloads as W
from helpers import rel_inf

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 2e-2


def _inputs(B, T, H, seed, with_s0=True, with_dsT=True, gate="softplus8"):
    inp = W.prefill(B, T, H, 128, 128, torch.bfloat16, seed=seed, gate=gate,
                    initial_state_std=0.05 if with_s0 else None)
    gen = torch.Generator().manual_seed(seed + 7)
    do = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16)
    dsT = torch.randn(B, H, 128, 128, generator=gen) * 0.1 if with_dsT else None
    return inp, do, dsT


def _check(B, T, H, seed, **kw):
    inp, do, dsT = _inputs(B, T, H, seed, **kw)
    dd = inp.to(DEV)
    got = kda_chunk_bwd(dd.q, dd.k, dd.v, dd.g, dd.beta, do.to(DEV), dd.initial_state,
                        None if dsT is None else dsT.to(DEV))
    torch.cuda.synchronize()
    ref = oracle.backward(inp.q, inp.k, inp.v, inp.g, inp.beta, do, inp.initial_state, dsT)
    for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta", "ds0"), got, ref):
        assert torch.isfinite(x).all(), name
        e = rel_inf(x, r)
        assert e <= TOL, f"{name}: relative inf-norm error {e:.3e}"


@pytest.mark.parametrize("T", [1, 50, 64, 65, 200, 333])
def test_chunk_bwd_lengths(T):
    _check(B=2, T=T, H=2, seed=300 + T)


@pytest.mark.parametrize("with_s0,with_dsT", [(False, False), (True, False), (False, True)])
def test_chunk_bwd_optional_states(with_s0, with_dsT):
    _check(B=1, T=130, H=3, seed=310, with_s0=with_s0, with_dsT=with_dsT)


def test_chunk_bwd_offset_gates_longer():
    _check(B=1, T=1024, H=2, seed=311, gate="offset16")


def test_chunk_bwd_matches_recurrent_bwd_full_size_sampled():
    """T = 8192, H = 32: the chunked backward against the recurrent one (itself
    within 2e-3 of the oracle) on all heads, and against the oracle on two."""
    inp, do, dsT = _inputs(1, 8192, 32, 312)
    dd = inp.to(DEV)
    a = kda_chunk_bwd(dd.q, dd.k, dd.v, dd.g, dd.beta, do.to(DEV), dd.initial_state, dsT.to(DEV))
    b = kda_recurrent_bwd(dd.q, dd.k, dd.v, dd.g, dd.beta, do.to(DEV), dd.initial_state, dsT.to(DEV))
    torch.cuda.synchronize()
    for name, x, y in zip(("dq", "dk", "dv", "dg", "dbeta", "ds0"), a, b):
        assert rel_inf(x, y) <= TOL, name
    for h in (0, 17):
        sl = lambda t: None if t is None else t[:, :, h:h + 1].contiguous()
        ref = oracle.backward(sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.beta), sl(do),
                              inp.initial_state[:, h:h + 1].contiguous(), dsT[:, h:h + 1].contiguous())
        for name, x, r in zip(("dq", "dk", "dv", "dg", "dbeta"), a, ref):
            assert rel_inf(x[:, :, h:h + 1].cpu(), r) <= TOL, (name, h)


@pytest.mark.parametrize("case", ["dense_6_units", "dense_32_units", "dense_64_units", "varlen_256_units"])
def test_saved_intermediates_bitwise(case):
    """kda_chunk_fwd_save gives kda_chunk_fwd's outputs bitwise, and the
    backward from its saved intermediates gives kda_chunk_bwd's gradients
    bitwise (the saved state images are the same whatever state-tile width
    the forward chain ran with: 16, 32, 64 or 128 columns here)."""
    from gated_delta_rule_88_b200 import kda_chunk_fwd, kda_chunk_fwd_save
    if case == "varlen_256_units":
        inp = W.prefill(1, 0, 32, 128, 128, torch.bfloat16, seed=320, initial_state_std=0.05,
                        seq_lens=[70, 0, 130, 64, 1, 200, 65, 90, 33])
    else:
        B, T, H = {"dense_6_units": (2, 150, 3), "dense_32_units": (1, 200, 32),
                   "dense_64_units": (2, 100, 32)}[case]
        inp = W.prefill(B, T, H, 128, 128, torch.bfloat16, seed=321, initial_state_std=0.05)
    d = inp.to(DEV)
    B, T, H, _ = d.q.shape
    gen = torch.Generator().manual_seed(322)
    do = torch.randn(B, T, H, 128, generator=gen).to(torch.bfloat16).to(DEV)
    N = inp.num_seqs
    dsT = (torch.randn(N, H, 128, 128, generator=gen) * 0.1).to(DEV)
    o1, s1 = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state, d.cu_seqlens)
    o2, s2, saved = kda_chunk_fwd_save(d.q, d.k, d.v, d.g, d.beta, d.initial_state, d.cu_seqlens)
    g1 = kda_chunk_bwd(d.q, d.k, d.v, d.g, d.beta, do, d.initial_state, dsT, d.cu_seqlens)
    g2 = kda_chunk_bwd(d.q, d.k, d.v, d.g, d.beta, do, d.initial_state, dsT, d.cu_seqlens,
                       saved=saved)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    for name, x, y in zip(("dq", "dk", "dv", "dg", "dbeta", "ds0"), g1, g2):
        assert torch.equal(x, y), name
