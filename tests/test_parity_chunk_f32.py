"""GPU parity: kda_chunk_fwd with fp32 inputs (exact-fp32 chunk path) vs the
fp64 oracle, max-abs tolerance 1e-3."""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_chunk_fwd
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
F32 = torch.float32


def _check(inp, dtype=F32):
    d = inp.to(DEV)
    o, sT = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state, d.cu_seqlens)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state,
                                  inp.cu_seqlens)
    torch.cuda.synchronize()
    assert_close(o, o_ref, dtype, "o")
    assert_close(sT, s_ref, dtype, "final state")
    return o, sT


def test_config_t256_h1_d64():
    """The fp32 workload: B=1, H=1, T=256, dk=dv=64, zero initial state."""
    _check(W.named_prefill("prefill_t256_h1_d64_f32"))


@pytest.mark.parametrize("T", [1, 63, 64, 65, 127, 200])
def test_ragged_lengths(T):
    _check(W.prefill(2, T, 3, 64, 64, F32, seed=T, initial_state_std=0.1))


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128)])
def test_head_dims(dk, dv):
    _check(W.prefill(1, 150, 2, dk, dv, F32, seed=7, initial_state_std=0.05))


def test_varlen_with_empty_sequences():
    inp = W.prefill(1, 0, 2, 64, 64, F32, seed=21, initial_state_std=0.1,
                    seq_lens=[70, 0, 1, 128, 0, 33])
    o, sT = _check(inp)
    # zero-length sequences return their initial state unchanged
    assert torch.equal(sT[1].cpu(), inp.initial_state[1])
    assert torch.equal(sT[4].cpu(), inp.initial_state[4])


def test_split_resume_matches_unsplit():
    inp = W.prefill(1, 300, 2, 64, 64, F32, seed=5, initial_state_std=0.1)
    d = inp.to(DEV)
    o, s = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state)
    cut = 77
    oa, sa = kda_chunk_fwd(d.q[:, :cut].contiguous(), d.k[:, :cut].contiguous(),
                           d.v[:, :cut].contiguous(), d.g[:, :cut].contiguous(),
                           d.beta[:, :cut].contiguous(), d.initial_state)
    ob, sb = kda_chunk_fwd(d.q[:, cut:].contiguous(), d.k[:, cut:].contiguous(),
                           d.v[:, cut:].contiguous(), d.g[:, cut:].contiguous(),
                           d.beta[:, cut:].contiguous(), sa)
    assert_close(torch.cat([oa, ob], 1), o, F32, "o split")
    assert_close(sb, s, F32, "state split")


def test_inplace_resume_state():
    inp = W.prefill(1, 100, 2, 64, 64, F32, seed=8, initial_state_std=0.1)
    d = inp.to(DEV)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state)
    st = d.initial_state.clone()
    o, s = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, st, final_state=st)
    assert s.data_ptr() == st.data_ptr()
    assert_close(st, s_ref, F32, "in-place state")
