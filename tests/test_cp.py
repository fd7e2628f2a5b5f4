"""Context-parallel prefill (gated_delta_rule_88_b200.cp): a sequence split
along time into W segments, one per rank, joined by one all-gather of each
segment's affine chunk map S_end = M S_start + B.

  * CPU: the oracle's recurrence is affine in the state (the pin the fold
    rests on), and the protocol over two gloo ranks with oracle-backed ops
    reproduces the unsplit oracle run.
  * GPU: kda_state_affine against the fp64 product, and W segments emulated
    in one process (segment maps and folds through the kernels, no
    collective) against the unsplit oracle run and the unsplit kernel.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_88_b200 import cp
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """The protocol's two device ops computed by the fp64 oracle (CPU)."""

    @staticmethod
    def chunk_fwd(q, k, v, g, beta, initial_state):
        return oracle.forward(q, k, v, g, beta, initial_state=initial_state)

    @staticmethod
    def affine(M, B, S):
        return oracle.state_affine(M, B, S)


def _split(x, bounds):
    return [x[:, a:b].contiguous() for a, b in zip(bounds[:-1], bounds[1:])]


def _inputs(T, H, seed, dtype=torch.float32, dk=64, dv=64):
    return W.prefill(1, T, H, dk, dv, dtype, seed=seed, initial_state_std=0.05)


def test_oracle_chunk_map_is_affine_in_the_state():
    inp = _inputs(T=23, H=2, seed=301)
    S0 = inp.initial_state.double()
    M, Bm = cp.segment_map(inp.q, inp.k, inp.v, inp.g, inp.beta, ops=OracleOps)
    _, sT = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, initial_state=S0)
    assert torch.allclose(oracle.state_affine(M, Bm, S0), sT, atol=1e-12, rtol=0)
    # and the map composes: two halves folded equal the whole
    bounds = [0, 9, 23]
    parts = [_split(x, bounds) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
    maps = [cp.segment_map(*[p[i] for p in parts], ops=OracleOps) for i in range(2)]
    S = cp.start_state(maps, S0, ops=OracleOps)
    assert torch.allclose(S, sT, atol=1e-12, rtol=0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cp_worker(rank, world, port, bounds, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs(T=bounds[-1], H=2, seed=302)
        seg = [_split(x, bounds)[rank] for x in (inp.q, inp.k, inp.v, inp.g, inp.beta)]
        o, sT = cp.cp_chunk_fwd(*seg, initial_state=inp.initial_state.double(), ops=OracleOps)
        torch.save({"o": o, "sT": sT}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world,bounds", [(2, [0, 40, 71]), (3, [0, 1, 30, 47])])
def test_cp_protocol_gloo(tmp_path, world, bounds):
    mp.start_processes(_cp_worker, args=(world, _free_port(), bounds, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    got = [torch.load(tmp_path / f"r{r}.pt") for r in range(world)]
    inp = _inputs(T=bounds[-1], H=2, seed=302)
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta,
                                  initial_state=inp.initial_state.double())
    o = torch.cat([g["o"] for g in got], dim=1)
    assert torch.allclose(o, o_ref, atol=1e-10, rtol=0)
    assert torch.allclose(got[-1]["sT"], s_ref, atol=1e-10, rtol=0)
    _, s_mid = oracle.forward(*[x[:, :bounds[1]] for x in (inp.q, inp.k, inp.v, inp.g, inp.beta)],
                              initial_state=inp.initial_state.double())
    assert torch.allclose(got[0]["sT"], s_mid, atol=1e-10, rtol=0)


# ---------------------------------------------------------------------------
# GPU

@pytest.mark.gpu
@pytest.mark.parametrize("count,dk,dv", [(1, 128, 128), (7, 64, 128), (3, 128, 64), (2, 5, 3)])
@pytest.mark.parametrize("with_b", [True, False])
def test_state_affine_kernel(count, dk, dv, with_b):
    from gated_delta_rule_88_b200 import kda_state_affine
    gen = torch.Generator().manual_seed(303 + dk + dv)
    M = torch.randn(count, dk, dk, generator=gen) / dk ** 0.5
    S = torch.randn(count, dk, dv, generator=gen)
    B = torch.randn(count, dk, dv, generator=gen) if with_b else None
    out = kda_state_affine(M.cuda(), None if B is None else B.cuda(), S.cuda())
    ref = oracle.state_affine(M, B, S)
    assert_close(out, ref, torch.float32, "state affine")


def _emulate(inp, bounds):
    """W ranks in one process: each segment's map, the fold, the re-run."""
    d = inp.to("cuda")
    parts = [_split(x, bounds) for x in (d.q, d.k, d.v, d.g, d.beta)]
    segs = [[p[i] for p in parts] for i in range(len(bounds) - 1)]
    maps = [cp.segment_map(*s) for s in segs]
    S0 = d.initial_state
    outs, states = [], []
    for r, s in enumerate(segs):
        S = cp.start_state(maps[:r], S0)
        o, sT = cp.KernelOps.chunk_fwd(*s, S)
        outs.append(o)
        states.append(sT)
    torch.cuda.synchronize()
    return torch.cat(outs, dim=1), states


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("bounds", [[0, 512, 1024], [0, 64, 200, 333, 1000]])
def test_cp_emulated_segments_match_unsplit(dtype, bounds):
    from gated_delta_rule_88_b200 import kda_chunk_fwd, kda_get_device_error
    inp = W.prefill(2, bounds[-1], 3, 128, 128, dtype, seed=304, initial_state_std=0.02)
    o, states = _emulate(inp, bounds)
    assert kda_get_device_error() == 0
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state)
    assert_close(o, o_ref, dtype, "cp o")
    for n in range(2):
        assert_close(states[-1][n], s_ref[n], dtype, f"cp final state {n}")
    d = inp.to("cuda")
    o_one, s_one = kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state)
    assert_close(o, o_one.double().cpu(), dtype, "cp o vs unsplit kernel")
