"""CPU, fp64: the chunked backward algorithm end to end, against torch autograd.

Kimi Linear paper notes (paper-notes-site), section 3 notes that training
uses the chunked kernels and their backward; the pages give no backward
equations.  This file writes out the chunked backward derived by reverse mode
through the chunk form (section 3 in words; equations from the section 2
recurrence) as three passes, the structure a tensor-core backward follows:

1. forward recompute: per chunk the forms, A, P, T, W, U, V_new and the state
   S entering the chunk;
2. reverse chain over chunks (last first), with dS' the gradient of the state
   leaving the chunk:
       dV_new = P^T dO + Kt dS',   dS = Qg^T dO + Diag(e^{G_C}) dS' - W^T dV_new;
3. per chunk, independently: the gradients of the forms, then dq, dk, dv,
   dbeta, and dg as the reverse cumsum, within the chunk, of the per-token dG
   (the last token also collects the e^{G_C} and K e^{G_C-G} terms).

The result must equal autograd through the token recurrence to rounding
(1e-10 relative), on several chunks with a ragged tail, a nonzero initial
state and a nonzero gradient of the final state.  It does not call the CUDA
path or the oracle.
"""
import pytest
import torch

DT = torch.float64
C = 16          # chunk length for the check (the algorithm is independent of C)


def _inputs(T, dk, dv, seed):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(T, dk, generator=gen, dtype=DT)
    k = torch.randn(T, dk, generator=gen, dtype=DT)
    q = q / q.norm(dim=1, keepdim=True) / dk ** 0.5
    k = k / k.norm(dim=1, keepdim=True)
    v = torch.randn(T, dv, generator=gen, dtype=DT)
    g = -torch.rand(T, dk, generator=gen, dtype=DT) * 0.4
    beta = torch.rand(T, generator=gen, dtype=DT)
    S0 = torch.randn(dk, dv, generator=gen, dtype=DT) * 0.3
    dO = torch.randn(T, dv, generator=gen, dtype=DT)
    dSf = torch.randn(dk, dv, generator=gen, dtype=DT)
    return q, k, v, g, beta, S0, dO, dSf


def _token_recurrence(q, k, v, g, beta, S):
    outs = []
    for t in range(q.shape[0]):
        S = torch.exp(g[t])[:, None] * S
        u = beta[t] * (v[t] - S.T @ k[t])
        S = S + torch.outer(k[t], u)
        outs.append(S.T @ q[t])
    return torch.stack(outs), S


def _chunks(T):
    return [slice(c, min(c + C, T)) for c in range(0, T, C)]


def _forms(q, k, v, g, beta):
    G = torch.cumsum(g, 0)
    GC = G[-1]
    eG, em, eGC = torch.exp(G), torch.exp(-G), torch.exp(GC)
    n = q.shape[0]
    f = dict(G=G, eG=eG, em=em, eGC=eGC,
             Qg=q * eG, bKg=beta[:, None] * k * eG, Kinv=k * em,
             Kt=k * em * eGC, bV=beta[:, None] * v)
    f["A"] = torch.tril(f["bKg"] @ f["Kinv"].T, -1)
    f["P"] = torch.tril(f["Qg"] @ f["Kinv"].T, 0)
    f["T"] = torch.linalg.inv(torch.eye(n, dtype=DT) + f["A"])
    f["W"] = f["T"] @ f["bKg"]
    f["U"] = f["T"] @ f["bV"]
    return f


def chunked_backward(q, k, v, g, beta, S0, dO, dSf, mutant=None):
    """mutant (tests only): a named slip planted in the algorithm."""
    T = q.shape[0]
    # 1. forward recompute
    recs, S = [], S0
    for sl in _chunks(T):
        f = _forms(q[sl], k[sl], v[sl], g[sl], beta[sl])
        f["S"] = S
        f["Vn"] = f["U"] - f["W"] @ S
        S = f["eGC"][:, None] * S + f["Kt"].T @ f["Vn"]
        recs.append(f)
    # 2. reverse chain
    dS = dSf
    for f, sl in zip(reversed(recs), reversed(_chunks(T))):
        f["dS2"] = dS
        f["dVn"] = f["P"].T @ dO[sl] + f["Kt"] @ dS
        decay = 1.0 if mutant == "no_decay_in_reverse_chain" else f["eGC"][:, None]
        dS = f["Qg"].T @ dO[sl] + decay * dS - f["W"].T @ f["dVn"]
    dS0 = dS
    # 3. per chunk
    out = [torch.zeros_like(x) for x in (q, k, v, g, beta)]
    dq, dk, dv, dg, db = out
    for f, sl in zip(recs, _chunks(T)):
        S, dS2, dVn, dOc = f["S"], f["dS2"], f["dVn"], dO[sl]
        dP = torch.tril(dOc @ f["Vn"].T, 0)
        dKt = f["Vn"] @ dS2.T
        deGC = (S * dS2).sum(1)
        dW = -dVn @ S.T
        dT = dVn @ f["bV"].T + dW @ f["bKg"].T
        Tt = f["T"] if mutant == "untransposed_T_in_dA" else f["T"].T
        dA = torch.tril(-Tt @ dT @ Tt, -1)
        dbV = f["T"].T @ dVn
        dbKg = f["T"].T @ dW + dA @ f["Kinv"]
        dKinv = dA.T @ f["bKg"] + dP.T @ f["Qg"]
        dQg = dOc @ S.T + (0.0 if mutant == "no_dP_in_dQg" else dP @ f["Kinv"])
        eG, em, eGC = f["eG"], f["em"], f["eGC"]
        bt = beta[sl, None]
        dq[sl] = dQg * eG
        dk[sl] = dbKg * bt * eG + dKinv * em + dKt * em * eGC
        dv[sl] = dbV * bt
        db[sl] = (dbKg * k[sl] * eG).sum(1) + (dbV * v[sl]).sum(1)
        dG = dQg * f["Qg"] + dbKg * f["bKg"] - dKinv * f["Kinv"] - dKt * f["Kt"]
        if mutant != "no_G_C_terms":
            dG[-1] += (dKt * f["Kt"]).sum(0) + deGC * eGC
        dg[sl] = torch.flip(torch.cumsum(torch.flip(dG, [0]), 0), [0])
    return dq, dk, dv, dg, db, dS0


@pytest.mark.parametrize("T,dk,dv,seed", [(53, 6, 5, 0), (64, 8, 8, 1), (40, 5, 7, 2)])
def test_chunked_backward_equals_autograd(T, dk, dv, seed):
    q, k, v, g, beta, S0, dO, dSf = _inputs(T, dk, dv, seed)
    xs = [x.clone().requires_grad_(True) for x in (q, k, v, g, beta, S0)]
    O, Sf = _token_recurrence(*xs)
    ((O * dO).sum() + (Sf * dSf).sum()).backward()
    mine = chunked_backward(q, k, v, g, beta, S0, dO, dSf)
    for name, m, x in zip(("dq", "dk", "dv", "dg", "dbeta", "dS0"), mine, xs):
        ref = x.grad
        err = float((m - ref).abs().max() / ref.abs().max())
        assert err < 1e-10, f"{name}: {err}"


@pytest.mark.parametrize("mutant", ["no_G_C_terms", "untransposed_T_in_dA",
                                    "no_dP_in_dQg", "no_decay_in_reverse_chain"])
def test_planted_slips_are_caught(mutant):
    """The comparison has teeth: each plausible slip moves some gradient far
    outside the bound."""
    q, k, v, g, beta, S0, dO, dSf = _inputs(53, 6, 5, 4)
    xs = [x.clone().requires_grad_(True) for x in (q, k, v, g, beta, S0)]
    O, Sf = _token_recurrence(*xs)
    ((O * dO).sum() + (Sf * dSf).sum()).backward()
    wrong = chunked_backward(q, k, v, g, beta, S0, dO, dSf, mutant=mutant)
    worst = max(float((m - x.grad).abs().max() / x.grad.abs().max()) for m, x in zip(wrong, xs))
    assert worst > 1e-3, (mutant, worst)
