"""GPU parity: kda_recurrent_steps with KDA_STEPS_CHUNK (the chunk form of
the L tokens on tensor cores, blocks of 16 tokens) vs the fp64 oracle.

Kimi Linear paper notes, section 3: the chunkwise form gathers a block's
writes in a WY-like representation and touches the state with one product;
the result is the recurrence's.  Tolerance: the bf16 bound of the other
parity tests (the state-product operands are bf16, as in the prefill).
Lengths cover one partial block (2, 8), a full block (16), a block plus one
token (17) and several blocks (32, 33, 40, 64, 100); gates cover the decode
workload's and a stronger, channel-dependent decay.
"""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import (KDA_STEPS_CHUNK, kda_get_device_error, kda_recurrent_steps)
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close, rel_inf

pytestmark = pytest.mark.gpu
DEV = "cuda"
BF = torch.bfloat16


def _tokens(N, L, H, d, seed, gate="softplus8"):
    steps = [W.decode_tokens(l, N, H, d, d, BF, seed=seed, gate=gate) for l in range(L)]
    return [torch.stack([s[i] for s in steps], dim=1).contiguous() for i in range(5)]


def _run(N, L, H, pool_n, seed, gate="softplus8", slots=True):
    d = 128
    pool0 = W.decode_initial_state(pool_n, H, d, d, seed=seed, std=0.02)
    gen = torch.Generator().manual_seed(seed + 1)
    sl = torch.randperm(pool_n, generator=gen)[:N].to(torch.int32) if slots else None
    q, k, v, g, b = _tokens(N, L, H, d, seed, gate)
    pool = pool0.to(DEV)
    out = kda_recurrent_steps(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), pool,
                              None if sl is None else sl.to(DEV), flags=KDA_STEPS_CHUNK)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    idx = sl.long() if sl is not None else torch.arange(N)
    o_ref, s_ref = oracle.forward(q, k, v, g, b, initial_state=pool0[idx].double())
    return pool0, pool, idx, out, o_ref, s_ref, (q, k, v, g, b), sl


@pytest.mark.parametrize("L", [2, 8, 16, 17, 32, 33, 40, 64, 100])
def test_chunk_steps_vs_oracle(L):
    pool0, pool, idx, out, o_ref, s_ref, _, _ = _run(N=5, L=L, H=3, pool_n=9, seed=90 + L)
    assert_close(out, o_ref, BF, "o")
    for n in range(idx.numel()):
        assert_close(pool[idx[n]], s_ref[n], BF, f"state {n}")
    rest = torch.ones(pool0.shape[0], dtype=torch.bool)
    rest[idx] = False
    assert torch.equal(pool.cpu()[rest], pool0[rest]), "pool entries not named were written"


@pytest.mark.parametrize("gate", ["offset16", "zero"])
def test_chunk_steps_gates(gate):
    _, pool, idx, out, o_ref, s_ref, _, _ = _run(N=4, L=24, H=2, pool_n=4, seed=97, gate=gate,
                                                 slots=False)
    assert_close(out, o_ref, BF, f"o ({gate})")
    for n in range(idx.numel()):
        assert_close(pool[idx[n]], s_ref[n], BF, f"state {n} ({gate})")


@pytest.mark.parametrize("L", [20, 70])
def test_chunk_steps_strong_decay(L):
    """g = -20 per token on every channel: the block forms use e^{G_i - G_j}
    <= 1 directly, so nothing overflows."""
    N, H, d = 3, 2, 128
    q, k, v, g, b = _tokens(N, L, H, d, seed=98)
    g = torch.full_like(g, -20.0)
    pool0 = W.decode_initial_state(N, H, d, d, seed=98, std=0.02)
    pool = pool0.to(DEV)
    out = kda_recurrent_steps(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), pool,
                              flags=KDA_STEPS_CHUNK)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all() and torch.isfinite(pool).all()
    o_ref, s_ref = oracle.forward(q, k, v, g, b, initial_state=pool0.double())
    assert_close(out, o_ref, BF, "o")
    for n in range(N):
        assert_close(pool[n], s_ref[n], BF, f"state {n}")


def test_chunk_steps_close_to_recurrent_on_the_decode_workload():
    """256 x 32 heads, 8 tokens, pool of 512: the chunk form against the
    recurrent kernel on every output (both bf16-tolerance from the oracle,
    which a sample checks)."""
    N, H, d, L, S = W.DECODE_N, W.DECODE_H, W.DECODE_D, 8, 2 * W.DECODE_N
    pool0 = W.decode_initial_state(S, H, d, d)
    gen = torch.Generator().manual_seed(31)
    slots = torch.randperm(S, generator=gen)[:N].to(torch.int32).to(DEV)
    q, k, v, g, b = [t.to(DEV) for t in _tokens(N, L, H, d, seed=W.DECODE_SEED)]
    pool_c, pool_r = pool0.to(DEV), pool0.to(DEV)
    out_c = kda_recurrent_steps(q, k, v, g, b, pool_c, slots, flags=KDA_STEPS_CHUNK)
    out_r = kda_recurrent_steps(q, k, v, g, b, pool_r, slots)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    assert rel_inf(out_c, out_r) <= 2e-2
    assert rel_inf(pool_c, pool_r) <= 2e-2
    ns = torch.randperm(N, generator=gen)[:16]
    sl = slots.cpu()[ns].long()
    o_ref, s_ref = oracle.forward(q.cpu()[ns], k.cpu()[ns], v.cpu()[ns], g.cpu()[ns], b.cpu()[ns],
                                  initial_state=pool0[sl].double())
    assert_close(out_c[ns.to(DEV)], o_ref, BF, "sampled o")
    assert_close(pool_c[sl.to(DEV)], s_ref, BF, "sampled states")


def test_chunk_flag_falls_back_where_unsupported():
    """fp32 inputs or d = 64 with the flag run the recurrent kernel: bitwise
    equal to the call without the flag."""
    N, L, H, d = 3, 5, 2, 64
    steps = [W.decode_tokens(l, N, H, d, d, torch.float32, seed=99) for l in range(L)]
    q, k, v, g, b = [torch.stack([s[i] for s in steps], dim=1).contiguous().to(DEV) for i in range(5)]
    s0 = W.decode_initial_state(N, H, d, d, seed=99).to(DEV)
    p1, p2 = s0.clone(), s0.clone()
    o1 = kda_recurrent_steps(q, k, v, g, b, p1, flags=KDA_STEPS_CHUNK)
    o2 = kda_recurrent_steps(q, k, v, g, b, p2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(p1, p2)


def test_chunk_steps_bad_slot_reported_and_skipped_long():
    """A slot outside the pool skips its sequence (no output, no pool entry
    written) and reports device error code 3; the other sequences are
    computed (several 16-token blocks per call)."""
    N, L, H, d, S = 4, 40, 2, 128, 6
    q, k, v, g, b = [t.to(DEV) for t in _tokens(N, L, H, d, seed=26)]
    pool0 = W.decode_initial_state(S, H, d, d, seed=26)
    pool = pool0.to(DEV)
    slots = torch.tensor([2, -1, 5, 6], dtype=torch.int32, device=DEV)   # -1 and 6 are invalid
    out = torch.full((N, L, H, d), 7.0, dtype=BF, device=DEV)
    kda_recurrent_steps(q, k, v, g, b, pool, slots, out=out, flags=KDA_STEPS_CHUNK)
    assert kda_get_device_error() == 3
    assert torch.all(out[1] == 7.0) and torch.all(out[3] == 7.0)
    ok = torch.tensor([0, 2])
    o_ref, s_ref = oracle.forward(q.cpu()[ok], k.cpu()[ok], v.cpu()[ok], g.cpu()[ok], b.cpu()[ok],
                                  initial_state=pool0[[2, 5]].double())
    assert_close(out[ok.to(DEV)], o_ref, BF, "o of the valid sequences")
    assert_close(pool[[2, 5]], s_ref, BF, "their pool entries")
    keep = [0, 1, 3, 4]
    assert torch.equal(pool.cpu()[keep], pool0[keep])


def test_chunk_steps_out_of_range_from_a_later_chunk():
    """From 33 tokens on the chunk form takes 64-token chunks on tcgen05; a
    chunk whose decay leaves the chunk-start range sends its item, from that
    chunk's first token on, to the 16-token blocks.  Sequence 1 head 0 leaves
    the range in its second chunk only, sequence 2 head 1 in its first, the
    rest stays in range: all of it against the oracle."""
    N, L, H, d = 4, 100, 2, 128
    q, k, v, g, b = _tokens(N, L, H, d, seed=61)
    g[1, 64:, 0] = -20.0
    g[2, :, 1] = -20.0
    pool0 = W.decode_initial_state(N, H, d, d, seed=61, std=0.02)
    pool = pool0.to(DEV)
    out = kda_recurrent_steps(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), pool,
                              flags=KDA_STEPS_CHUNK)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    assert torch.isfinite(out.float()).all() and torch.isfinite(pool).all()
    o_ref, s_ref = oracle.forward(q, k, v, g, b, initial_state=pool0.double())
    assert_close(out, o_ref, BF, "o")
    for n in range(N):
        assert_close(pool[n], s_ref[n], BF, f"state {n}")


def test_chunk_steps_decode_workload_64_tokens():
    """256 sequences x 32 heads, 64 tokens each, pool of 512 (the serving
    decode's chunk-form workload): every output finite and within the bf16
    bound of the recurrent kernel; 16 sampled sequences against the oracle."""
    N, H, d, L, S = W.DECODE_N, W.DECODE_H, W.DECODE_D, 64, 2 * W.DECODE_N
    pool0 = W.decode_initial_state(S, H, d, d)
    gen = torch.Generator().manual_seed(33)
    slots = torch.randperm(S, generator=gen)[:N].to(torch.int32).to(DEV)
    q, k, v, g, b = [t.to(DEV) for t in _tokens(N, L, H, d, seed=W.DECODE_SEED)]
    pool_c, pool_r = pool0.to(DEV), pool0.to(DEV)
    out_c = kda_recurrent_steps(q, k, v, g, b, pool_c, slots, flags=KDA_STEPS_CHUNK)
    out_r = kda_recurrent_steps(q, k, v, g, b, pool_r, slots)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    assert torch.isfinite(out_c.float()).all() and torch.isfinite(pool_c).all()
    assert rel_inf(out_c, out_r) <= 2e-2
    assert rel_inf(pool_c, pool_r) <= 2e-2
    ns = torch.randperm(N, generator=gen)[:16]
    sl = slots.cpu()[ns].long()
    o_ref, s_ref = oracle.forward(q.cpu()[ns], k.cpu()[ns], v.cpu()[ns], g.cpu()[ns], b.cpu()[ns],
                                  initial_state=pool0[sl].double())
    assert_close(out_c[ns.to(DEV)], o_ref, BF, "sampled o")
    assert_close(pool_c[sl.to(DEV)], s_ref, BF, "sampled states")


def test_chunk_steps_16_byte_aligned_buffers():
    """The 64-token path moves the state and the output in 32-byte pieces; a
    pool and an output that are only 16-byte aligned (the entry point's
    contract) take the 16-token blocks instead, and match the oracle."""
    N, L, H, d = 3, 64, 2, 128
    q, k, v, g, b = _tokens(N, L, H, d, seed=63)
    pool0 = W.decode_initial_state(N, H, d, d, seed=63, std=0.02)
    pool_buf = torch.zeros(pool0.numel() + 4, dtype=torch.float32, device=DEV)
    pool = pool_buf[4:].view(pool0.shape)                 # 16 bytes past a 256-byte boundary
    pool.copy_(pool0.to(DEV))
    out_buf = torch.zeros(N * L * H * d + 8, dtype=BF, device=DEV)
    out = out_buf[8:].view(N, L, H, d)                    # likewise
    assert pool.data_ptr() % 32 == 16 and out.data_ptr() % 32 == 16
    kda_recurrent_steps(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), b.to(DEV), pool, out=out,
                        flags=KDA_STEPS_CHUNK)
    torch.cuda.synchronize()
    assert kda_get_device_error() == 0
    o_ref, s_ref = oracle.forward(q, k, v, g, b, initial_state=pool0.double())
    assert_close(out, o_ref, BF, "o")
    for n in range(N):
        assert_close(pool[n], s_ref[n], BF, f"state {n}")
