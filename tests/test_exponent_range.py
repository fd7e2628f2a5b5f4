"""CPU: the exponent range behind the bf16 prefill's two ways of forming the
intra-chunk products.

With every exponent of a chunk referenced at the chunk start, a product
e^{G_i - G_j} (j <= i) is formed as (x_i e^{G_i}) . (y_j e^{-G_j}) from two
factors rounded to bf16.  Both factors are normal bf16 numbers while |G| <=
80, so the products keep bf16 accuracy however strong the decay inside that
bound; past ~88 the factor e^{-G} overflows.  The kernel therefore takes the
chunk-start form only when every |G| and G_C - G of the chunk is at most 80
and forms other chunks with 16-token references (where per-token g >= -5
keeps each factor within e^{+-80}).  These checks emulate the factor
rounding in plain PyTorch; they do not call the CUDA path.
"""
import math

import torch

BF = torch.bfloat16


def _pairwise(G, x, y):
    """P_ij = sum_c x_ic y_jc e^{G_ic - G_jc} two ways: fp64 directly, and from
    bf16-rounded chunk-start factors with fp32 accumulation (the kernel's
    operand precision)."""
    exact = torch.einsum("ic,jc,ijc->ij", x.double(), y.double(),
                         torch.exp(G.double()[:, None, :] - G.double()[None, :, :]))
    left = (x.float() * torch.exp(G.float())).to(BF).float()
    right = (y.float() * torch.exp(-G.float())).to(BF).float()
    return exact, left @ right.T


def _lower_rel_err(exact, approx):
    C = exact.shape[0]
    mask = torch.tril(torch.ones(C, C, dtype=torch.bool))
    e, a = exact[mask], approx[mask].double()
    return float((e - a).abs().max() / e.abs().max())


def test_chunk_start_factors_keep_bf16_accuracy_up_to_80():
    gen = torch.Generator().manual_seed(0)
    C, d = 64, 32
    x = torch.randn(C, d, generator=gen)
    y = torch.randn(C, d, generator=gen)
    for total in (1.0, 20.0, 60.0, 79.0):
        # a constant per-token decay reaching -total at the last token on half
        # of the channels, weak decay elsewhere
        g = torch.full((C, d), -0.01)
        g[:, : d // 2] = -total / C
        G = torch.cumsum(g, 0)
        assert float(G.abs().max()) <= 80.0
        exact, approx = _pairwise(G, x, y)
        err = _lower_rel_err(exact, approx)
        assert err < 1e-2, (total, err)          # bf16 operands, fp32 accumulation


def test_chunk_start_factor_overflows_past_the_bound():
    # e^{-G} for G = -90 is beyond the bf16 range (max ~3.39e38 = e^{88.7})
    assert math.exp(88.0) < float(torch.finfo(BF).max) < math.exp(89.0)
    f = torch.tensor([math.exp(90.0)], dtype=torch.float32).to(BF)
    assert torch.isinf(f).all()
    # while the 16-token reference bound keeps every factor finite
    assert math.exp(16 * 5.0) < float(torch.finfo(BF).max)
