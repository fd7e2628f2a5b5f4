"""CPU: the error budget of the bf16 chunk path, from its rounding points.

The bf16 prefill kernels round to bf16 exactly where a value becomes a
tensor-core operand: the decayed forms (Q e^G, beta K e^G, K e^{-G},
K e^{G_C-G}, beta V), P, T, W, U, the state S before each product, and
V_new before P V_new and Kt^T V_new; everything else (G, A, the inverse, the
state update, the accumulators) stays fp32.  This test replays those rounding
points in plain PyTorch over a whole 8192-token sequence (128 chunks; chunk
form of Kimi Linear paper notes, section 3, derived from the section 2
recurrence) and checks the result against the same chunk form in fp64: the
error must sit inside the bf16 tolerance (2e-2 relative) with room to spare,
so the kernels' measured error (about 7e-3 on this workload) is what the
rounding points imply.  It does not call the CUDA path or the oracle.
"""
import torch

from gated_delta_rule_88_b200 import workloads

BF = torch.bfloat16
C = 64


def _r(x):
    return x.to(BF).float()


def _forms(q, k, v, g, beta):
    G = torch.cumsum(g, 0)
    GC = G[-1]
    return (q * torch.exp(G), beta[:, None] * k * torch.exp(G), k * torch.exp(-G),
            k * torch.exp(GC - G), beta[:, None] * v, torch.exp(GC))


def _chain(q, k, v, g, beta, rounded):
    dt = torch.float32 if rounded else torch.float64
    q, k, v, g, beta = (x.to(dt) for x in (q, k, v, g, beta))
    r = _r if rounded else (lambda x: x)
    S = torch.zeros(q.shape[1], v.shape[1], dtype=dt)
    outs = []
    eye = torch.eye(C, dtype=dt)
    for c in range(0, q.shape[0], C):
        sl = slice(c, c + C)
        Qg, bKg, Kinv, Kt, bV, eGC = _forms(q[sl], k[sl], v[sl], g[sl], beta[sl])
        Qg, bKg, Kinv, Kt, bV = r(Qg), r(bKg), r(Kinv), r(Kt), r(bV)
        A = torch.tril(bKg @ Kinv.T, -1)
        P = r(torch.tril(Qg @ Kinv.T))
        T = r(torch.linalg.inv(eye + A))
        W, U = r(T @ bKg), r(T @ bV)
        Sb = r(S)
        Vn = r(U - W @ Sb)
        outs.append(Qg @ Sb + P @ Vn)
        S = eGC[:, None] * S + Kt.T @ Vn
    return torch.cat(outs).double(), S.double()


def test_rounding_points_stay_inside_the_bf16_tolerance():
    inp = workloads.named_prefill("prefill_t8192_h32_d128")
    h = 0
    q, k, v, g, beta = (x[0, :, h].float() for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    O64, S64 = _chain(q, k, v, g, beta, rounded=False)
    O, S = _chain(q, k, v, g, beta, rounded=True)
    eo = float((O - O64).abs().max() / O64.abs().max())
    es = float((S - S64).abs().max() / S64.abs().max())
    assert eo < 1e-2 and es < 1e-2, (eo, es)
    # the rounding is really there: an fp32 path without it would be ~1e-6
    assert eo > 1e-4, eo
