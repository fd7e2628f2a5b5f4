"""Pins for the fp64 oracle: it is checked against what the pages and the
mathematics fix, never against itself.

Each pin is a function of a ``run(q, k, v, g, beta, S0) -> (o, S_T)`` callable
for one (sequence, head).  The oracle must pass every pin; every planted
mistake (a mutant of the recurrence with a dropped term, wrong sign, wrong
index or transposed operand) must fail at least one pin.

Sources of the pins (pages named by title and section):
  - KDA recurrence: Kimi Linear paper notes (paper-notes-site), section 2.
  - DeltaNet and Gated DeltaNet formulas: zhichai.net account, the DeltaNet /
    GDN / KDA formula paragraph; hnts03 summary, "Kimi Delta Attention"
    (GDN = scalar decay, KDA = per-channel diagonal decay).
  - Prefix checkpoint / resume: whoami-wesleyyou blog, "context modification
    and checkpoint" section (the state summarises the whole prefix).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(12345)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(T=9, dk=5, dv=3, g_scale=0.3, beta=None, seed=0, s0=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, dk))
    k = r.standard_normal((T, dk)) / math.sqrt(dk)
    v = r.standard_normal((T, dv))
    g = -np.abs(r.standard_normal((T, dk))) * g_scale
    b = r.uniform(0.1, 0.9, T) if beta is None else np.full(T, float(beta))
    S0 = r.standard_normal((dk, dv)) if s0 else np.zeros((dk, dv))
    return q, k, v, g, b, S0


# --------------------------------------------------------------------------
# pins (each returns the max abs deviation; the caller compares to a bound)
# --------------------------------------------------------------------------

def pin_deltanet(run):
    """g == 0 (alpha = 1): the recurrence is DeltaNet,
    S_t = (I - b k k^T) S_{t-1} + b k v^T, written with dense matrices."""
    q, k, v, _, b, S0 = _rand_case(seed=1)
    g = np.zeros_like(q)
    o, S = run(q, k, v, g, b, S0)
    Sd = S0.copy()
    err = 0.0
    for t in range(q.shape[0]):
        M = np.eye(q.shape[1]) - b[t] * np.outer(k[t], k[t])
        Sd = M @ Sd + b[t] * np.outer(k[t], v[t])
        err = max(err, np.abs(o[t] - Sd.T @ q[t]).max())
    return max(err, np.abs(S - Sd).max())


def pin_gdn_scalar(run):
    """alpha_t constant across channels: Gated DeltaNet's scalar decay,
    S_t = gamma_t (I - b k k^T) S_{t-1} + b k v^T."""
    q, k, v, _, b, S0 = _rand_case(seed=2)
    gam = -np.abs(np.random.default_rng(3).standard_normal(q.shape[0])) * 0.5
    g = np.repeat(gam[:, None], q.shape[1], axis=1)
    o, S = run(q, k, v, g, b, S0)
    Sd = S0.copy()
    err = 0.0
    for t in range(q.shape[0]):
        M = np.eye(q.shape[1]) - b[t] * np.outer(k[t], k[t])
        Sd = math.exp(gam[t]) * (M @ Sd) + b[t] * np.outer(k[t], v[t])
        err = max(err, np.abs(o[t] - Sd.T @ q[t]).max())
    return max(err, np.abs(S - Sd).max())


def pin_beta_zero(run):
    """beta == 0: nothing is written; S_t = Diag(exp(sum_{s<=t} g_s)) S_0
    (closed form) and o_t = S_t^T q_t.  dk != dv fixes the decay to rows."""
    q, k, v, g, _, S0 = _rand_case(seed=4, T=11, dk=4, dv=6)
    b = np.zeros(q.shape[0])
    o, S = run(q, k, v, g, b, S0)
    G = np.cumsum(g, axis=0)
    err = 0.0
    for t in range(q.shape[0]):
        St = np.exp(G[t])[:, None] * S0
        err = max(err, np.abs(o[t] - St.T @ q[t]).max())
    return max(err, np.abs(S - np.exp(G[-1])[:, None] * S0).max())


def pin_one_token_dense(run):
    """One token: S_1 = (I - b k k^T) Diag(alpha) S_0 + b k v^T, dense."""
    q, k, v, g, b, S0 = _rand_case(seed=5, T=1, dk=6, dv=4)
    o, S = run(q, k, v, g, b, S0)
    A = np.diag(np.exp(g[0]))
    S1 = (np.eye(6) - b[0] * np.outer(k[0], k[0])) @ A @ S0 + b[0] * np.outer(k[0], v[0])
    return max(np.abs(S - S1).max(), np.abs(o[0] - S1.T @ q[0]).max())


def pin_bruteforce_product(run):
    """S_T = (prod_t M_t) S_0 + sum_t (prod_{s>t} M_s) b_t k_t v_t^T with
    M_t = (I - b_t k_t k_t^T) Diag(alpha_t); every o_t from its own prefix
    products (no recursion on S)."""
    q, k, v, g, b, S0 = _rand_case(seed=6, T=7, dk=4, dv=3)
    T, dk = q.shape
    M = [(np.eye(dk) - b[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) for t in range(T)]

    def state_at(t):  # S_t (1-based count of tokens consumed = t+1)
        P = np.eye(dk)
        for s in range(t + 1):
            P = M[s] @ P
        acc = P @ S0
        for s in range(t + 1):
            Ps = np.eye(dk)
            for r in range(s + 1, t + 1):
                Ps = M[r] @ Ps
            acc = acc + Ps @ (b[s] * np.outer(k[s], v[s]))
        return acc

    o, S = run(q, k, v, g, b, S0)
    err = np.abs(S - state_at(T - 1)).max()
    for t in range(T):
        err = max(err, np.abs(o[t] - state_at(t).T @ q[t]).max())
    return err


def pin_retrieval(run):
    """With b |k|^2 = 1 the delta rule overwrites: S_t^T k_t = v_t exactly,
    for any decay; with q_t = k_t the readout returns v_t (post-update)."""
    q, k, v, g, _, S0 = _rand_case(seed=7, T=10, dk=5, dv=4)
    b = 1.0 / (k * k).sum(axis=1)
    o, _ = run(k.copy(), k, v, g, b, S0)
    return np.abs(o - v).max()


def pin_linearity(run):
    """(o, S_T) are jointly linear in (S_0, v)."""
    q, k, v1, g, b, S1 = _rand_case(seed=8)
    _, _, v2, _, _, S2 = _rand_case(seed=9)
    a1, a2 = 0.7, -1.3
    o1, T1 = run(q, k, v1, g, b, S1)
    o2, T2 = run(q, k, v2, g, b, S2)
    o3, T3 = run(q, k, a1 * v1 + a2 * v2, g, b, a1 * S1 + a2 * S2)
    return max(np.abs(o3 - (a1 * o1 + a2 * o2)).max(), np.abs(T3 - (a1 * T1 + a2 * T2)).max())


def pin_split_resume(run):
    """A prefix's final state resumes the suffix exactly (checkpoint semantics)."""
    q, k, v, g, b, S0 = _rand_case(seed=10, T=13)
    o, S = run(q, k, v, g, b, S0)
    oa, Sa = run(q[:5], k[:5], v[:5], g[:5], b[:5], S0)
    ob, Sb = run(q[5:], k[5:], v[5:], g[5:], b[5:], Sa)
    return max(np.abs(np.concatenate([oa, ob]) - o).max(), np.abs(Sb - S).max())


def _golden():
    vals = {}
    with open(os.path.join(GOLDEN, "kda_tiny_dk2_dv2.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, *nums = line.split()
            vals[name] = np.array([float(x) for x in nums])
    return vals


def pin_golden_hand_example(run):
    """The hand-derived dk=dv=2, T=2 example in tests/golden."""
    G = _golden()
    q = np.stack([G["q_1"], G["q_2"]])
    k = np.stack([G["k_1"], G["k_2"]])
    v = np.stack([G["v_1"], G["v_2"]])
    g = np.log(np.stack([G["alpha_1"], G["alpha_2"]]))
    b = np.array([G["beta_1"][0], G["beta_2"][0]])
    S0 = G["S0"].reshape(2, 2)
    o, S = run(q, k, v, g, b, S0)
    o1, S1 = run(q[:1], k[:1], v[:1], g[:1], b[:1], S0)
    return max(np.abs(o[0] - G["o_1"]).max(), np.abs(o[1] - G["o_2"]).max(),
               np.abs(S - G["S_2"].reshape(2, 2)).max(),
               np.abs(S1 - G["S_1"].reshape(2, 2)).max())


PINS = [pin_deltanet, pin_gdn_scalar, pin_beta_zero, pin_one_token_dense,
        pin_bruteforce_product, pin_retrieval, pin_linearity, pin_split_resume,
        pin_golden_hand_example]
TOL = 1e-11


def oracle_run(q, k, v, g, b, S0):
    return oracle.recurrence(q, k, v, g, b, S0)


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    assert pin(oracle_run) < TOL


# --------------------------------------------------------------------------
# planted mistakes: each mutant of the recurrence must fail at least one pin
# --------------------------------------------------------------------------

def _mutant(kind):
    def run(q, k, v, g, b, S0):
        q, k, v, g = (np.asarray(x, float) for x in (q, k, v, g))
        b = np.asarray(b, float)
        S = np.array(S0, float, copy=True)
        T = q.shape[0]
        o = np.zeros((T, v.shape[1]))
        for t in range(T):
            a = np.exp(g[t])
            if kind == "decay_after_write":
                u = b[t] * (v[t] - S.T @ k[t])
                S = a[:, None] * (S + np.outer(k[t], u))
            else:
                if kind == "no_decay":
                    Sp = S.copy()
                elif kind == "decay_columns":
                    Sp = S * np.resize(a, S.shape[1])[None, :]
                elif kind == "decay_exp_neg":
                    Sp = np.exp(-g[t])[:, None] * S
                else:
                    Sp = a[:, None] * S
                if kind == "kS_pre_decay":
                    kS = S.T @ k[t]
                else:
                    kS = Sp.T @ k[t]
                if kind == "sign_flip":
                    u = b[t] * (v[t] + kS)
                elif kind == "beta_on_v_only":
                    u = b[t] * v[t] - kS
                elif kind == "no_erase":
                    u = b[t] * v[t]
                else:
                    u = b[t] * (v[t] - kS)
                S = Sp + np.outer(k[t], u)
            if kind == "readout_pre_update":
                o[t] = Sp.T @ q[t]
            elif kind == "readout_transposed":
                o[t] = S @ q[t]          # shape error unless dk == dv
            elif kind == "readout_k":
                o[t] = S.T @ k[t]
            else:
                o[t] = S.T @ q[t]
        return o, S
    return run


MUTANTS = ["no_decay", "decay_columns", "decay_exp_neg", "kS_pre_decay",
           "sign_flip", "beta_on_v_only", "no_erase", "decay_after_write",
           "readout_pre_update", "readout_transposed", "readout_k"]


def test_reference_mutant_is_exact():
    """The mutant harness with no mutation agrees with the oracle (sanity)."""
    for pin in PINS:
        assert pin(_mutant("none")) < 1e-10


@pytest.mark.parametrize("kind", MUTANTS)
def test_pins_catch_planted_mistake(kind):
    run = _mutant(kind)
    worst = 0.0
    for pin in PINS:
        try:
            worst = max(worst, pin(run))
        except (ValueError, IndexError):
            worst = float("inf")
    assert worst > 1e-6, f"no pin caught mutant {kind}"


# --------------------------------------------------------------------------
# the batched wrapper: layouts, varlen packing, head independence
# --------------------------------------------------------------------------

def test_forward_dense_matches_per_sequence():
    torch.manual_seed(0)
    B, T, H, dk, dv = 2, 7, 3, 4, 5
    q = torch.randn(B, T, H, dk); k = torch.randn(B, T, H, dk) * 0.4
    v = torch.randn(B, T, H, dv); g = -torch.rand(B, T, H, dk) * 0.3
    beta = torch.rand(B, T, H); s0 = torch.randn(B, H, dk, dv)
    o, sT = oracle.forward(q, k, v, g, beta, s0)
    for b in range(B):
        for h in range(H):
            o1, S1 = oracle.recurrence(q[b, :, h], k[b, :, h], v[b, :, h], g[b, :, h],
                                       beta[b, :, h], s0[b, h])
            assert np.abs(o[b, :, h].numpy() - o1).max() == 0
            assert np.abs(sT[b, h].numpy() - S1).max() == 0


def test_forward_varlen_matches_dense_pieces():
    torch.manual_seed(1)
    lens = [3, 0, 6, 1]
    T, H, dk, dv = sum(lens), 2, 4, 3
    q = torch.randn(1, T, H, dk); k = torch.randn(1, T, H, dk) * 0.4
    v = torch.randn(1, T, H, dv); g = -torch.rand(1, T, H, dk) * 0.3
    beta = torch.rand(1, T, H); s0 = torch.randn(len(lens), H, dk, dv)
    cu = torch.tensor([0, 3, 3, 9, 10], dtype=torch.int32)
    o, sT = oracle.forward(q, k, v, g, beta, s0, cu)
    for n in range(len(lens)):
        s, e = int(cu[n]), int(cu[n + 1])
        on, Sn = oracle.forward(q[:, s:e], k[:, s:e], v[:, s:e], g[:, s:e], beta[:, s:e],
                                s0[n:n + 1])
        assert torch.equal(o[:, s:e], on)
        assert torch.equal(sT[n], Sn[0])
    # a zero-length sequence returns its initial state
    assert torch.equal(sT[1], s0[1].double())


def test_decode_step_equals_one_token_forward():
    torch.manual_seed(2)
    N, H, d = 3, 2, 4
    q = torch.randn(N, H, d); k = torch.randn(N, H, d) * 0.5
    v = torch.randn(N, H, d); g = -torch.rand(N, H, d); beta = torch.rand(N, H)
    s0 = torch.randn(N, H, d, d)
    o, s1 = oracle.decode_step(q, k, v, g, beta, s0)
    for n in range(N):
        for h in range(H):
            o1, S1 = oracle.recurrence(q[n, h][None], k[n, h][None], v[n, h][None],
                                       g[n, h][None], beta[n, h][None], s0[n, h])
            assert np.abs(o[n, h].numpy() - o1[0]).max() == 0
            assert np.abs(s1[n, h].numpy() - S1).max() == 0


# ---- input prologue (the *_ex calls): pinned by properties, not by retyping ----

def test_prologue_l2norm_unit_rows_direction_and_zero_rows():
    gen = torch.Generator().manual_seed(7)
    q = torch.randn(2, 5, 3, 8, generator=gen, dtype=torch.float64) * 3.0
    k = torch.randn(2, 5, 3, 8, generator=gen, dtype=torch.float64)
    q[1, 2, 0] = 0.0                                    # a padding row
    b = torch.zeros(2, 5, 3, dtype=torch.float64)
    qn, kn, bn = oracle.prologue(q, k, b, qk_l2norm=True)
    norms_q = torch.linalg.vector_norm(qn, dim=-1)
    norms_k = torch.linalg.vector_norm(kn, dim=-1)
    mask = torch.ones_like(norms_q, dtype=torch.bool)
    mask[1, 2, 0] = False
    assert torch.allclose(norms_q[mask], torch.ones_like(norms_q[mask]), atol=1e-14)
    assert torch.allclose(norms_k, torch.ones_like(norms_k), atol=1e-14)
    assert torch.all(qn[1, 2, 0] == 0)
    # same direction: <q_hat, q> = |q|
    dots = (qn * q).sum(-1)
    assert torch.allclose(dots[mask], torch.linalg.vector_norm(q, dim=-1)[mask], rtol=1e-13)
    assert torch.equal(bn, b)                          # beta untouched without the flag


def test_prologue_q_scale_only_scales_q():
    gen = torch.Generator().manual_seed(8)
    q = torch.randn(1, 4, 2, 8, generator=gen, dtype=torch.float64)
    k = torch.randn(1, 4, 2, 8, generator=gen, dtype=torch.float64)
    b = torch.randn(1, 4, 2, generator=gen, dtype=torch.float64)
    qs, ks, bs = oracle.prologue(q, k, b, q_scale=0.25)
    assert torch.equal(qs, q * 0.25) and torch.equal(ks, k) and torch.equal(bs, b)
    qn, kn, _ = oracle.prologue(q, k, b, qk_l2norm=True, q_scale=0.5)
    assert torch.allclose(torch.linalg.vector_norm(qn, dim=-1), torch.full((1, 4, 2), 0.5,
                          dtype=torch.float64), atol=1e-14)


def test_prologue_sigmoid_closed_forms():
    b = torch.tensor([0.0, math.log(3.0), -math.log(3.0), 40.0, -40.0], dtype=torch.float64)
    _, _, s = oracle.prologue(torch.zeros(5, 1), torch.zeros(5, 1), b, beta_sigmoid=True)
    assert s[0] == 0.5
    assert abs(s[1] - 0.75) < 1e-15 and abs(s[2] - 0.25) < 1e-15   # sigma(ln 3) = 3/4
    x = torch.linspace(-6, 6, 25, dtype=torch.float64)
    _, _, sx = oracle.prologue(torch.zeros(25, 1), torch.zeros(25, 1), x, beta_sigmoid=True)
    _, _, smx = oracle.prologue(torch.zeros(25, 1), torch.zeros(25, 1), -x, beta_sigmoid=True)
    assert torch.allclose(sx + smx, torch.ones_like(sx), atol=1e-15)   # sigma(x) + sigma(-x) = 1
    assert torch.all(sx[1:] > sx[:-1])                                # increasing
    assert s[3] > 1 - 1e-15 and s[4] < 1e-15


# ---- output epilogue (gated RMSNorm): pinned by properties ----

def test_gated_rmsnorm_unit_rms_scale_invariance_and_gate():
    gen = torch.Generator().manual_seed(9)
    x = torch.randn(6, 16, generator=gen, dtype=torch.float64) * 5.0
    ones = torch.ones(16, dtype=torch.float64)
    big = torch.full((6, 16), 60.0, dtype=torch.float64)          # sigmoid -> 1
    y = oracle.gated_rmsnorm(x, big, ones, 0.0)
    assert torch.allclose(y.pow(2).mean(-1), torch.ones(6, dtype=torch.float64), atol=1e-12)
    assert torch.allclose(oracle.gated_rmsnorm(3.7 * x, big, ones, 0.0), y, atol=1e-13)
    half = oracle.gated_rmsnorm(x, torch.zeros(6, 16, dtype=torch.float64), ones, 0.0)
    assert torch.allclose(half, 0.5 * y, atol=1e-13)              # sigmoid(0) = 1/2
    w = torch.linspace(-2, 2, 16, dtype=torch.float64)
    assert torch.allclose(oracle.gated_rmsnorm(x, big, w, 0.0), y * w, atol=1e-13)
    # eps enters as mean(x^2) + eps: a row with mean square m maps to x / sqrt(m + eps)
    row = torch.full((1, 16), 2.0, dtype=torch.float64)
    assert torch.allclose(oracle.gated_rmsnorm(row, big[:1], ones, 5.0),
                          torch.full((1, 16), 2.0 / 3.0, dtype=torch.float64), atol=1e-13)


# ---------------------------------------------------------------------------
# The backward oracle (autograd through the fp64 recurrence), pinned by
# central finite differences of the C recurrence and by closed forms.

def _bwd_case(seed, T=6, dk=4, dv=3, with_s0=True):
    gen = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=gen, dtype=torch.float64)
    q, k, v = r(1, T, 1, dk), 0.6 * r(1, T, 1, dk), r(1, T, 1, dv)
    g = -torch.rand(1, T, 1, dk, generator=gen, dtype=torch.float64)
    b = torch.rand(1, T, 1, generator=gen, dtype=torch.float64)
    s0 = r(1, 1, dk, dv) if with_s0 else None
    do, dsT = r(1, T, 1, dv), r(1, 1, dk, dv)
    return q, k, v, g, b, s0, do, dsT


def _loss(q, k, v, g, b, s0, do, dsT):
    o, sT = oracle.recurrence(q[0, :, 0], k[0, :, 0], v[0, :, 0], g[0, :, 0], b[0, :, 0],
                              None if s0 is None else s0[0, 0])
    return float((o * do[0, :, 0].numpy()).sum() + (sT * dsT[0, 0].numpy()).sum())


@pytest.mark.parametrize("seed", [1, 2])
def test_backward_matches_finite_differences(seed):
    q, k, v, g, b, s0, do, dsT = _bwd_case(seed)
    grads = oracle.backward(q, k, v, g, b, do, s0, dsT)
    args = [q, k, v, g, b, s0]
    gen = torch.Generator().manual_seed(100 + seed)
    eps = 1e-6
    for ai, (x, gx) in enumerate(zip(args, grads)):
        for _ in range(4):
            idx = tuple(int(torch.randint(0, n, (1,), generator=gen)) for n in x.shape)
            xp, xm = x.clone(), x.clone()
            xp[idx] += eps
            xm[idx] -= eps
            ap, am = list(args), list(args)
            ap[ai], am[ai] = xp, xm
            fd = (_loss(*ap, do, dsT) - _loss(*am, do, dsT)) / (2 * eps)
            assert abs(fd - float(gx[idx])) <= 1e-6 * max(1.0, abs(fd)), (ai, idx, fd, float(gx[idx]))


def test_backward_one_token_closed_form():
    """T = 1, S0 = 0: o = beta (k.q) v, S_1 = beta k v^T, so
    dv = beta ((k.q) do + dS^T k), dq = beta (v.do) k."""
    q, k, v, g, b, _, do, dsT = _bwd_case(3, T=1)
    dq, dk_, dv_, dg, db, ds0 = oracle.backward(q, k, v, g, b, do, None, dsT)
    qq, kk, vv, bb, dd, SS = q[0, 0, 0], k[0, 0, 0], v[0, 0, 0], b[0, 0, 0], do[0, 0, 0], dsT[0, 0]
    assert torch.allclose(dv_[0, 0, 0], bb * ((kk @ qq) * dd + SS.T @ kk), atol=1e-12)
    assert torch.allclose(dq[0, 0, 0], bb * (vv @ dd) * kk, atol=1e-12)
    assert torch.allclose(dg[0, 0, 0], torch.zeros_like(dg[0, 0, 0]), atol=1e-12)   # S0 = 0


def test_backward_pure_decay_state_gradient():
    """beta = 0: S_t = Diag(prod_{s<=t} a_s) S0 and o_t = S_t^T q_t, so
    dS0 = sum_t Diag(prod_{s<=t} a_s) q_t do_t^T + Diag(prod_s a_s) dS_T."""
    q, k, v, g, b, s0, do, dsT = _bwd_case(4, T=5)
    b = torch.zeros_like(b)
    ds0 = oracle.backward(q, k, v, g, b, do, s0, dsT)[5][0, 0]
    a = torch.exp(torch.cumsum(g[0, :, 0], dim=0))      # [T, dk]
    ref = sum(a[t][:, None] * torch.outer(q[0, t, 0], do[0, t, 0]) for t in range(5))
    ref = ref + a[-1][:, None] * dsT[0, 0]
    assert torch.allclose(ds0, ref, atol=1e-12)
