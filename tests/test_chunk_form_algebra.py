"""CPU, fp64: the chunk form the bf16 prefill kernels compute, and its
reverse mode, checked against the token recurrence and torch autograd.

Kimi Linear paper notes (paper-notes-site), section 3 describes the chunkwise
form in words (the old state through the chunk's transitions plus the
intra-chunk writes in a WY-like form); the equations here are derived from
the recurrence of section 2 and written out in plain PyTorch, independent of
the CUDA path and of the oracle.  Forward per chunk (G the chunk-local
cumsum of g, S the entering state):

    A = tril_-1(beta K e^G (K e^-G)^T),  P = tril_0(Q e^G (K e^-G)^T)
    T = (I + A)^-1,  W = T beta K e^G,  U = T beta V
    V_new = U - W S,  O = Q e^G S + P V_new,  S' = e^{G_C} S + (K e^{G_C - G})^T V_new

and the backward equations of the chunked backward plan (given dO, dS').
"""
import pytest
import torch

DT = torch.float64


def _chunk(C=16, dk=6, dv=5, seed=0):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(C, dk, generator=gen, dtype=DT)
    k = torch.randn(C, dk, generator=gen, dtype=DT)
    v = torch.randn(C, dv, generator=gen, dtype=DT)
    q, k = q / q.norm(dim=1, keepdim=True), k / k.norm(dim=1, keepdim=True)
    g = -torch.rand(C, dk, generator=gen, dtype=DT) * 0.3
    beta = torch.rand(C, generator=gen, dtype=DT)
    S = torch.randn(dk, dv, generator=gen, dtype=DT) * 0.3
    return q, k, v, g, beta, S


def _forward(q, k, v, g, beta, S):
    C = q.shape[0]
    G = torch.cumsum(g, 0)
    GC = G[-1]
    f = dict(Qg=q * torch.exp(G), Kg=k * torch.exp(G), Kinv=k * torch.exp(-G),
             Kt=k * torch.exp(GC - G), eGC=torch.exp(GC))
    f["bKg"] = beta[:, None] * f["Kg"]
    f["bV"] = beta[:, None] * v
    f["A"] = torch.tril(f["bKg"] @ f["Kinv"].T, -1)
    f["P"] = torch.tril(f["Qg"] @ f["Kinv"].T, 0)
    f["T"] = torch.linalg.inv(torch.eye(C, dtype=DT) + f["A"])
    f["W"] = f["T"] @ f["bKg"]
    f["U"] = f["T"] @ f["bV"]
    f["Vn"] = f["U"] - f["W"] @ S
    O = f["Qg"] @ S + f["P"] @ f["Vn"]
    S2 = f["eGC"][:, None] * S + f["Kt"].T @ f["Vn"]
    return O, S2, f


def test_chunk_form_equals_token_recurrence():
    q, k, v, g, beta, S = _chunk()
    O, S2, _ = _forward(q, k, v, g, beta, S)
    Sr, outs = S.clone(), []
    for t in range(q.shape[0]):
        Sr = torch.exp(g[t])[:, None] * Sr
        u = beta[t] * (v[t] - Sr.T @ k[t])
        Sr = Sr + torch.outer(k[t], u)
        outs.append(Sr.T @ q[t])
    assert torch.allclose(O, torch.stack(outs), atol=1e-13, rtol=0)
    assert torch.allclose(S2, Sr, atol=1e-13, rtol=0)


@pytest.mark.parametrize("seed", [0, 1])
def test_chunk_backward_equations_match_autograd(seed):
    q, k, v, g, beta, S = _chunk(seed=seed)
    for t in (q, k, v, g, beta, S):
        t.requires_grad_(True)
    O, S2, f = _forward(q, k, v, g, beta, S)
    for name in ("Qg", "Kinv", "Kt", "bKg", "bV", "A", "P", "T", "W", "U", "Vn"):
        f[name].retain_grad()
    gen = torch.Generator().manual_seed(100 + seed)
    dO = torch.randn(O.shape, generator=gen, dtype=DT)
    dS2 = torch.randn(S2.shape, generator=gen, dtype=DT)
    ((O * dO).sum() + (S2 * dS2).sum()).backward()
    d = {n: t.detach() for n, t in f.items()}
    Sd = S.detach()
    with torch.no_grad():
        dVn = d["P"].T @ dO + d["Kt"] @ dS2
        dS = d["Qg"].T @ dO + d["eGC"][:, None] * dS2 - d["W"].T @ dVn
        dU, dW = dVn, -dVn @ Sd.T
        dT = dU @ d["bV"].T + dW @ d["bKg"].T
        dA = torch.tril(-d["T"].T @ dT @ d["T"].T, -1)
        dP = torch.tril(dO @ d["Vn"].T, 0)
        dKt = d["Vn"] @ dS2.T
        dbV = d["T"].T @ dU
        dbKg = d["T"].T @ dW + dA @ d["Kinv"]
        dKinv = dA.T @ d["bKg"] + dP.T @ d["Qg"]
        dQg = dO @ Sd.T + dP @ d["Kinv"]
    checks = {
        "dS": (dS, S.grad), "dV_new": (dVn, f["Vn"].grad), "dU": (dU, f["U"].grad),
        "dW": (dW, f["W"].grad), "dT": (dT, f["T"].grad),
        "dA": (dA, torch.tril(f["A"].grad, -1)), "dP": (dP, torch.tril(f["P"].grad, 0)),
        "dKt": (dKt, f["Kt"].grad), "d(beta V)": (dbV, f["bV"].grad),
        "d(beta K e^G)": (dbKg, f["bKg"].grad), "d(K e^-G)": (dKinv, f["Kinv"].grad),
        "dQg": (dQg, f["Qg"].grad),
    }
    for name, (mine, ref) in checks.items():
        err = float((mine - ref).abs().max() / ref.abs().max())
        assert err < 1e-12, f"{name}: {err}"
