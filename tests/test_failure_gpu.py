"""Failure detection without faulting the GPU.

Every wait in the kernels is bounded; when one runs out, the kernel records
RA_ERR_TIMEOUT in the library's device status word, stops issuing work and returns, so the
context stays usable.  The self-test kernel makes such a wait run out (it waits on an
mbarrier that nothing arrives on, with a 50 ms limit), and the host reads the status back.
"""
import time

import pytest
import torch

import oracle
from long_context_exact_fwd_b200.workloads import random_qkv
from parity import assert_close_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    from long_context_exact_fwd_b200 import build
    build.ensure_built()
    from long_context_exact_fwd_b200 import ring_attn
    return ring_attn


def test_bounded_wait_reports_timeout_and_the_context_survives(ra):
    assert ra.device_status() == 0
    t0 = time.perf_counter()
    ra.wait_selftest(0.05)
    assert ra.device_status() == ra.RA_ERR_TIMEOUT      # read ...
    assert time.perf_counter() - t0 < 5.0
    assert ra.device_status() == 0                      # ... and cleared
    inp = random_qkv(1, 1, 256, 128, seed=9)
    o, _ = ra.fwd(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), 2, True)
    assert ra.device_status() == 0
    O, _ = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], True)
    assert_close_bf16(o.float().cpu().numpy(), O)


def test_selftest_argument_checks(ra):
    with pytest.raises(ra.RingAttnError):
        ra.wait_selftest(0.0)
    with pytest.raises(ra.RingAttnError):
        ra.wait_selftest(100.0)
