"""GPU parity: kda_recurrent_steps (through the C ABI) vs the fp64 oracle.

Serving decode: up to L tokens per sequence in the fused recurrent mode
(Kimi Linear paper notes, section 3: queries of at most 64 tokens outside
training) against a slot-indexed state pool.  Each sequence's expected result
is the oracle's recurrence over its L tokens from the pool entry it names.
"""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_get_device_error, kda_recurrent_step, kda_recurrent_steps
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tokens(N, L, H, dk, dv, dtype, seed, gate="softplus8"):
    """[N, L, H, *] token tensors: step l of the decode workload generator."""
    steps = [W.decode_tokens(l, N, H, dk, dv, dtype, seed=seed, gate=gate) for l in range(L)]
    return [torch.stack([s[i] for s in steps], dim=1).contiguous() for i in range(5)]


def _check(N, L, H, dk, dv, dtype, pool_size, seed, slots=True):
    pool0 = W.decode_initial_state(pool_size, H, dk, dv, seed=seed, std=0.02)
    gen = torch.Generator().manual_seed(seed + 1)
    sl = torch.randperm(pool_size, generator=gen)[:N].to(torch.int32) if slots else None
    q, k, v, g, b = _tokens(N, L, H, dk, dv, dtype, seed)
    pool = pool0.to(DEV)
    out = kda_recurrent_steps(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), pool,
                              None if sl is None else sl.to(DEV))
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    idx = sl.long() if sl is not None else torch.arange(N)
    o_ref, s_ref = oracle.forward(q, k, v, g, b, initial_state=pool0[idx].double())
    sdt = torch.float32 if dtype == torch.float32 else dtype
    assert_close(out, o_ref, dtype, "o")
    assert_close(pool[idx.to(DEV)], s_ref, sdt, "named pool entries")
    rest = torch.ones(pool_size, dtype=torch.bool)
    rest[idx] = False
    assert torch.equal(pool.cpu()[rest], pool0[rest]), "pool entries not named were written"


@pytest.mark.parametrize("L", [1, 4, 17, 64])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_steps_slots_d128(L, dtype):
    _check(N=5, L=L, H=3, dk=128, dv=128, dtype=dtype, pool_size=9, seed=21)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128)])
def test_steps_other_shapes(dk, dv):
    _check(N=4, L=6, H=2, dk=dk, dv=dv, dtype=torch.bfloat16, pool_size=7, seed=22)


def test_steps_without_slots():
    _check(N=3, L=8, H=4, dk=128, dv=128, dtype=torch.bfloat16, pool_size=3, seed=23, slots=False)


def test_steps_match_repeated_single_steps():
    """L tokens in one call equal L calls of kda_recurrent_step (same
    arithmetic per token, one state read and write instead of L)."""
    N, L, H, d = 6, 12, 3, 128
    q, k, v, g, b = [t.to(DEV) for t in _tokens(N, L, H, d, d, torch.bfloat16, seed=24)]
    s0 = W.decode_initial_state(N, H, d, d, seed=24).to(DEV)
    pool = s0.clone()
    out = kda_recurrent_steps(q, k, v, g, b, pool)
    st = s0.clone()
    outs = [kda_recurrent_step(q[:, l].contiguous(), k[:, l].contiguous(), v[:, l].contiguous(),
                               g[:, l].contiguous(), b[:, l].contiguous(), st) for l in range(L)]
    torch.cuda.synchronize()
    assert torch.equal(out, torch.stack(outs, dim=1))
    assert torch.equal(pool, st)


def test_steps_bad_slot_reported_and_skipped():
    N, L, H, d, S = 4, 3, 2, 64, 6
    q, k, v, g, b = [t.to(DEV) for t in _tokens(N, L, H, d, d, torch.bfloat16, seed=25)]
    pool0 = W.decode_initial_state(S, H, d, d, seed=25)
    pool = pool0.to(DEV)
    slots = torch.tensor([2, -1, 5, 6], dtype=torch.int32, device=DEV)   # -1 and 6 are invalid
    out = torch.full((N, L, H, d), 7.0, dtype=torch.bfloat16, device=DEV)
    kda_recurrent_steps(q, k, v, g, b, pool, slots, out=out)
    assert kda_get_device_error() == 3
    assert torch.all(out[1] == 7.0) and torch.all(out[3] == 7.0)
    ok = torch.tensor([0, 2])
    o_ref, s_ref = oracle.forward(q.cpu()[ok], k.cpu()[ok], v.cpu()[ok], g.cpu()[ok], b.cpu()[ok],
                                  initial_state=pool0[[2, 5]].double())
    assert_close(out[ok.to(DEV)], o_ref, torch.bfloat16, "o of the valid sequences")
    assert_close(pool[[2, 5]], s_ref, torch.bfloat16, "their pool entries")
    keep = [0, 1, 3, 4]
    assert torch.equal(pool.cpu()[keep], pool0[keep])


def test_steps_decode_workload_sampled():
    """The decode workload's shape (256 sequences x 32 heads, d = 128, bf16)
    with 8 tokens per call on a pool of 512 entries: 48 seeded sequences
    (all heads) against the oracle."""
    N, H, d, L, S = W.DECODE_N, W.DECODE_H, W.DECODE_D, 8, 2 * W.DECODE_N
    pool0 = W.decode_initial_state(S, H, d, d)
    gen = torch.Generator().manual_seed(31)
    slots = torch.randperm(S, generator=gen)[:N].to(torch.int32)
    q, k, v, g, b = _tokens(N, L, H, d, d, torch.bfloat16, seed=W.DECODE_SEED)
    pool = pool0.to(DEV)
    out = kda_recurrent_steps(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), pool,
                              slots.to(DEV))
    torch.cuda.synchronize()
    ns = torch.randperm(N, generator=gen)[:48]
    o_ref, s_ref = oracle.forward(q[ns], k[ns], v[ns], g[ns], b[ns],
                                  initial_state=pool0[slots[ns].long()].double())
    assert_close(out[ns.to(DEV)], o_ref, torch.bfloat16, "sampled o")
    assert_close(pool[slots[ns].long().to(DEV)], s_ref, torch.bfloat16, "sampled states")
