"""GPU parity: kda_chunk_fwd with bf16 inputs (tensor-core chunk path) vs the
fp64 oracle.  Tolerance: ||x - ref||_inf / ||ref||_inf <= 2e-2 on outputs and
on each final state (fp32 state)."""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_chunk_fwd, kda_get_device_error
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close, rel_inf, rms_rel

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16


def _run(inp, **kw):
    d = inp.to(DEV)
    o, sT = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state, d.cu_seqlens, **kw)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    return o, sT


def _check(inp, heads=None):
    o, sT = _run(inp)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state,
                                  inp.cu_seqlens, heads=heads)
    if heads is not None:
        o, sT = o[:, :, heads], sT[:, heads]
        o_ref, s_ref = o_ref[:, :, heads], s_ref[:, heads]
    assert_close(o, o_ref, BF, "o")
    for n in range(sT.shape[0]):
        assert_close(sT[n], s_ref[n], BF, f"final state {n}")
    return o, sT, o_ref, s_ref


@pytest.mark.parametrize("T", [1, 16, 63, 64, 65, 127, 200, 333])
def test_ragged_lengths(T):
    _check(W.prefill(2, T, 3, 128, 128, BF, seed=100 + T, initial_state_std=0.02))


def test_zero_initial_state_null_pointer():
    _check(W.prefill(1, 300, 4, 128, 128, BF, seed=9))


@pytest.mark.parametrize("gate", ["offset16", "zero"])
def test_gate_variants(gate):
    _check(W.prefill(1, 257, 3, 128, 128, BF, seed=4, gate=gate, initial_state_std=0.02))


def test_strongest_supported_decay():
    """per-token g at the documented floor (-5) on a third of the channels:
    every sub-chunk exponent sits at its extreme"""
    inp = W.prefill(1, 256, 2, 128, 128, BF, seed=12, initial_state_std=0.02)
    inp.g[..., ::3] = -5.0
    _check(inp)


@pytest.mark.parametrize("g_strong", [-6.0, -20.0, -90.0])
def test_any_decay_below_the_factorised_range(g_strong):
    """per-token g far below -5 on some channels and heads (down to a decay of
    e^-90 per token): the sub-chunk factor 1 / a_j would overflow, so those
    sub-chunks' diagonal blocks of A and P are formed from e^{G_i - G_j}
    directly; mixed with ordinary chunks in one call"""
    inp = W.prefill(1, 333, 3, 128, 128, BF, seed=44, initial_state_std=0.02)
    inp.g[:, :, 0, ::4] = g_strong          # every chunk of head 0
    inp.g[:, 100:180, 2, 1::3] = g_strong   # a span of head 2 (chunks 1 and 2)
    o, sT, _, _ = _check(inp)
    assert torch.isfinite(o.float()).all() and torch.isfinite(sT).all()


def test_any_decay_prologue_path():
    """the same with the in-kernel prologue (the fallback re-reads q and k
    and applies the L2-norm factors itself)"""
    from gated_delta_rule_88_b200 import kda_chunk_fwd_ex, KDA_QK_L2NORM
    inp = W.prefill(1, 150, 2, 128, 128, BF, seed=45, initial_state_std=0.02)
    inp.g[:, :, 1, ::2] = -30.0
    raw_q = (inp.q.float() * 3.0).to(BF)     # not normalised: the prologue does it
    d = inp.to(DEV)
    o, sT = kda_chunk_fwd_ex(raw_q.to(DEV), d.k, d.v, d.g, d.beta, d.initial_state,
                             flags=KDA_QK_L2NORM, q_scale=1.0 / 128 ** 0.5)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    qn, kn, _ = oracle.prologue(raw_q, inp.k, inp.beta, qk_l2norm=True, q_scale=1.0 / 128 ** 0.5)
    o_ref, s_ref = oracle.forward(qn, kn, inp.v, inp.g, inp.beta, inp.initial_state)
    assert_close(o, o_ref, BF, "o (prologue, strong decay)")
    assert_close(sT[0], s_ref[0], BF, "state (prologue, strong decay)")


@pytest.mark.parametrize("g_floor", [-1.2, -1.3, -2.0])
def test_mixed_exponent_ranges(g_floor):
    """Chunks whose decay over the chunk stays within e^80 use one exponent
    reference per chunk, the others 16-token references: a per-token g of
    -1.2 on some channels keeps a 64-token chunk inside (|G_C| = 76.8),
    -1.3 and -2 push it outside.  The strong decay sits on chunks 1 and 3 of
    one head only, so both kinds of chunk meet in one call and in one chain."""
    inp = W.prefill(1, 320, 3, 128, 128, BF, seed=41, initial_state_std=0.02)
    inp.g[:, 64:128, 1, ::5] = g_floor
    inp.g[:, 192:250, 1, 3::7] = g_floor
    _check(inp)


def test_varlen_with_empty_and_short_sequences():
    inp = W.prefill(1, 0, 3, 128, 128, BF, seed=21, initial_state_std=0.02,
                    seq_lens=[70, 0, 1, 128, 0, 200, 64, 65])
    o, sT, _, _ = _check(inp)
    assert torch.equal(sT[1].cpu(), inp.initial_state[1])
    assert torch.equal(sT[4].cpu(), inp.initial_state[4])


def test_varlen_equals_separate_runs():
    lens = [100, 37, 256]
    inp = W.prefill(1, 0, 2, 128, 128, BF, seed=31, initial_state_std=0.02, seq_lens=lens)
    o, sT = _run(inp)
    d = inp.to(DEV)
    cu = inp.cu_seqlens.tolist()
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        on, sn = kda_chunk_fwd(d.q[:, s:e].contiguous(), d.k[:, s:e].contiguous(),
                               d.v[:, s:e].contiguous(), d.g[:, s:e].contiguous(),
                               d.beta[:, s:e].contiguous(), d.initial_state[n:n + 1].contiguous())
        # same kernels, same chunk boundaries -> identical results
        assert torch.equal(on, o[:, s:e])
        assert torch.equal(sn[0], sT[n])


def test_split_resume_matches_unsplit():
    inp = W.prefill(1, 400, 2, 128, 128, BF, seed=5, initial_state_std=0.02)
    d = inp.to(DEV)
    o, s = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state)
    cut = 150   # not a multiple of the chunk length
    sl = lambda x, a, b: x[:, a:b].contiguous()
    oa, sa = kda_chunk_fwd(sl(d.q, 0, cut), sl(d.k, 0, cut), sl(d.v, 0, cut), sl(d.g, 0, cut),
                           sl(d.beta, 0, cut), d.initial_state)
    ob, sb = kda_chunk_fwd(sl(d.q, cut, 400), sl(d.k, cut, 400), sl(d.v, cut, 400),
                           sl(d.g, cut, 400), sl(d.beta, cut, 400), sa)
    assert_close(torch.cat([oa, ob], 1), o, BF, "o split")
    assert_close(sb, s, BF, "state split")
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state)
    assert_close(torch.cat([oa, ob], 1), o_ref, BF, "o split vs oracle")
    assert_close(sb, s_ref, BF, "state split vs oracle")


def test_inplace_state_and_no_final_state():
    inp = W.prefill(1, 130, 2, 128, 128, BF, seed=8, initial_state_std=0.02)
    d = inp.to(DEV)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state)
    st = d.initial_state.clone()
    o, s = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, st, final_state=st)
    torch.cuda.synchronize()
    assert_close(st, s_ref, BF, "in-place state")
    o2, s2 = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state, output_final_state=False)
    assert s2 is None
    assert torch.equal(o2, o)


def test_prefill_t8192_h32_full():
    """The T = 8192, H = 32 workload, every head against the oracle."""
    inp = W.named_prefill("prefill_t8192_h32_d128")
    o, sT, o_ref, s_ref = _check(inp)
    print(f"o rel {rel_inf(o, o_ref):.2e} rms {rms_rel(o, o_ref):.2e}; "
          f"S rel {rel_inf(sT, s_ref):.2e}")


def _margins(name, o, sT, o_ref, s_ref):
    msg = (f"{name}: o rel-inf {rel_inf(o, o_ref):.2e} rms {rms_rel(o, o_ref):.2e}; "
           f"S rel-inf {rel_inf(sT, s_ref):.2e} rms {rms_rel(sT, s_ref):.2e}")
    print(msg)
    return msg


def test_prefill_t65536_h32_all_heads():
    """The T = 65536, H = 32 long-memory workload, every head against the
    oracle over the full length."""
    inp = W.named_prefill("prefill_t65536_h32_d128")
    o, sT, o_ref, s_ref = _check(inp)
    _margins("prefill_t65536_h32_d128", o, sT, o_ref, s_ref)


def test_varlen8_resume_all_heads():
    """8 packed sequences, lengths U[1024, 32768], per-sequence initial states,
    every head of every sequence against the oracle.  Each sequence is also
    split at a non-multiple of 64 and resumed; the resumed run must match the
    oracle too."""
    inp = W.named_prefill("varlen8_h32_d128_resume")
    o, sT, o_ref, s_ref = _check(inp)
    _margins("varlen8_h32_d128_resume", o, sT, o_ref, s_ref)
    d = inp.to(DEV)
    cu = inp.cu_seqlens.tolist()
    for n in range(8):
        s, e = cu[n], cu[n + 1]
        cut = s + (e - s) // 3 + 17
        sl = lambda x, a, b: x[:, a:b].contiguous()
        _, sa = kda_chunk_fwd(sl(d.q, s, cut), sl(d.k, s, cut), sl(d.v, s, cut), sl(d.g, s, cut),
                              sl(d.beta, s, cut), d.initial_state[n:n + 1].contiguous())
        ob, sb = kda_chunk_fwd(sl(d.q, cut, e), sl(d.k, cut, e), sl(d.v, cut, e), sl(d.g, cut, e),
                               sl(d.beta, cut, e), sa)
        assert_close(sb[0], s_ref[n], BF, f"resumed state {n}")
        assert_close(ob, o_ref[:, cut:e], BF, f"resumed o {n}")


# ---- bf16 inputs at head dimension 64 (fp32 arithmetic on the CUDA cores) ----

@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64)])
def test_head_dim_64_ragged(T, dk, dv):
    _check(W.prefill(2, T, 3, dk, dv, BF, seed=700 + T + dk + dv, initial_state_std=0.02))


def test_head_dim_64_varlen_and_resume():
    """Varlen with an empty and a one-token sequence, then each sequence split
    at a non-multiple of 64 and resumed from its checkpoint."""
    inp = W.prefill(1, 0, 4, 64, 64, BF, seed=710, initial_state_std=0.05,
                    seq_lens=[300, 0, 1, 129])
    o, sT, o_ref, s_ref = _check(inp)
    d = inp.to(DEV)
    cu = inp.cu_seqlens.tolist()
    for n in (0, 3):
        s, e = cu[n], cu[n + 1]
        cut = s + 77
        sl = lambda x, a, b: x[:, a:b].contiguous()
        _, sa = kda_chunk_fwd(sl(d.q, s, cut), sl(d.k, s, cut), sl(d.v, s, cut), sl(d.g, s, cut),
                              sl(d.beta, s, cut), d.initial_state[n:n + 1].contiguous())
        ob, sb = kda_chunk_fwd(sl(d.q, cut, e), sl(d.k, cut, e), sl(d.v, cut, e), sl(d.g, cut, e),
                               sl(d.beta, cut, e), sa)
        assert_close(sb[0], s_ref[n], BF, f"resumed state {n}")
        assert_close(ob, o_ref[:, cut:e], BF, f"resumed o {n}")
