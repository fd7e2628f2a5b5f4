"""Failure detection without a GPU fault.

Every mbarrier wait in the library's kernels is bounded: when the bound runs
out the kernel sets the device error word (code 1) and returns.  The GPU test
makes such a wait run out on purpose (kda_selftest_bounded_wait: one CTA
waiting on an mbarrier nothing arrives on, no copy or MMA in flight), then
checks that the host reads code 1, that reading clears it, and that the
context still computes correctly afterwards.  The CPU tests check the call's
argument rules.
"""
import ctypes

import pytest
import torch

import oracle
import gated_delta_rule_88_b200 as kda
from gated_delta_rule_88_b200 import build as kbuild
from gated_delta_rule_88_b200 import workloads as W
from helpers import assert_close


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


@pytest.mark.parametrize("limit", [0, 65537, 1 << 31])
def test_selftest_limit_out_of_range_rejected(lib, limit):
    assert lib.kda_selftest_bounded_wait(ctypes.c_uint(limit), None) == 1
    assert b"limit" in lib.kda_last_error_message()


@pytest.mark.gpu
def test_bounded_wait_timeout_reaches_the_host_and_clears():
    torch.cuda.set_device(0)
    assert kda.kda_get_device_error() == 0          # clean start
    kda.kda_selftest_bounded_wait(limit=1000)
    assert kda.kda_get_device_error() == 1          # kErrWaitTimeout
    assert kda.kda_get_device_error() == 0          # read-and-clear
    # twice in a row on one stream: the first code stays until it is read
    kda.kda_selftest_bounded_wait(limit=64)
    kda.kda_selftest_bounded_wait(limit=64)
    assert kda.kda_get_device_error() == 1
    assert kda.kda_get_device_error() == 0
    # the context is still usable: a prefill right after matches the oracle
    inp = W.prefill(1, 100, 2, 128, 128, torch.bfloat16, seed=90, initial_state_std=0.02)
    d = inp.to("cuda")
    o, s = kda.kda_chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.initial_state)
    torch.cuda.synchronize()
    assert kda.kda_get_device_error() == 0
    o_ref, s_ref = oracle.forward(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state)
    assert_close(o, o_ref, torch.bfloat16, "o after a timeout")
    assert_close(s, s_ref, torch.bfloat16, "state after a timeout")
