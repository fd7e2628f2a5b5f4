"""GPU parity: kda_gated_rmsnorm (the layer's output epilogue, Kimi Linear
paper notes section 7: RMSNorm with a sigmoid output gate) vs the fp64 oracle."""
import pytest
import torch

import oracle
from gated_delta_rule_88_b200 import kda_gated_rmsnorm
from helpers import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("dv", [128, 64])
def test_gated_rmsnorm(dtype, dv):
    gen = torch.Generator().manual_seed(71)
    x = (torch.randn(3, 37, 4, dv, generator=gen) * 3.0).to(dtype)
    z = torch.randn(3, 37, 4, dv, generator=gen).to(dtype)
    w = torch.randn(dv, generator=gen) * 0.5 + 1.0
    y = kda_gated_rmsnorm(x.to(DEV), z.to(DEV), w.to(DEV), eps=1e-5)
    ref = oracle.gated_rmsnorm(x, z, w, 1e-5)
    assert_close(y, ref, dtype, "gated rmsnorm")


def test_gated_rmsnorm_in_place_and_zero_rows():
    gen = torch.Generator().manual_seed(72)
    x = torch.randn(64, 128, generator=gen).to(torch.bfloat16)
    x[5] = 0.0
    z = torch.randn(64, 128, generator=gen).to(torch.bfloat16)
    w = torch.ones(128)
    xd = x.to(DEV)
    y = kda_gated_rmsnorm(xd, z.to(DEV), w.to(DEV), eps=1e-6, out=xd)
    assert y.data_ptr() == xd.data_ptr()
    ref = oracle.gated_rmsnorm(x, z, w, 1e-6)
    assert torch.all(y[5] == 0)
    assert_close(y, ref, torch.bfloat16, "in place")
