"""ring_attn_bwd_noalloc, the backward entry point for callers that cannot allocate.

Some callers may not allocate device memory on their path -- code embedded in a host
framework that owns every device allocation, or latency-critical code that cannot absorb
cudaMalloc's implicit synchronisation -- so they cannot hand ring_attn_bwd its workspace.
ring_attn_bwd_noalloc keeps that scratch in a static device array of the library instead.
These tests call it through the C ABI and compare it with ring_attn_bwd (given a workspace)
and with the float64 oracle, within the parity tolerances; consecutive calls check that
leftovers in the shared scratch from the previous call do not leak into the next result, and
that a call with caller-provided outputs allocates no device memory.

This file is collected last on purpose, so a stop-at-first-failure run reaches it only
after every other test has run.
"""
import ctypes

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


def _problem(ra, B, H, S, D, causal, seed):
    inp = random_qkv(B, H, S, 128, seed=seed, with_do=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = ra.fwd(q, k, v, D, causal)
    return q, k, v, o, lse, do


def _oracle_grads(q, k, v, do, causal):
    return oracle.attn_bwd_heads(*(x.cpu() for x in (q, k, v, do)), causal)


def _compare(got, ref):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert_close_bf16(g.float().cpu().numpy(), r.float().cpu().numpy(), name)


@pytest.mark.parametrize("causal", [True, False])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(ra, causal):
    q, k, v, o, lse, do = _problem(ra, 1, 2, 1000, 8, causal, seed=41)
    ref = ra.bwd(q, k, v, o, lse, do, 8, causal)
    want = _oracle_grads(q, k, v, do, causal)
    torch.cuda.synchronize()
    outs = [torch.empty_like(q) for _ in range(3)]   # caller-owned outputs
    for i in range(2):   # the second call starts from the first call's leftovers
        if i == 1:
            alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        got = ra.bwd_noalloc(q, k, v, o, lse, do, 8, causal, *outs)
        assert ra.device_status() == 0
        if i == 1:   # a warmed-up call allocates nothing, through torch or behind its back
            assert torch.cuda.memory_allocated() == alloc0
            assert torch.cuda.mem_get_info()[0] == free0
        _compare(got, ref)
        for name, g, r in zip(("dq", "dk", "dv"), got, want):
            assert_close_bf16(g.float().cpu().numpy(), r, name)
    # a different, smaller problem right after: nothing of the larger one may remain
    q2, k2, v2, o2, lse2, do2 = _problem(ra, 2, 1, 384, 3, causal, seed=43)
    ref2 = ra.bwd(q2, k2, v2, o2, lse2, do2, 3, causal)
    got2 = ra.bwd_noalloc(q2, k2, v2, o2, lse2, do2, 3, causal)
    assert ra.device_status() == 0
    _compare(got2, ref2)


def test_noalloc_rejects_problems_beyond_its_scratch(ra):
    limit = ra.bwd_noalloc_max_bytes()
    assert limit == 96 << 20
    S = 262144   # needs 512 B of dQ accumulator per row: 128 MiB > the scratch
    assert ra.bwd_workspace_bytes(1, 1, S, 128) > limit
    f = ra.raw.ring_attn_bwd_noalloc
    P = ctypes.c_void_p
    ptrs = [P(256)] * 5 + [P(256)] * 4     # never dereferenced: the size check comes first
    code = f(*ptrs[:5], ptrs[5], *ptrs[6:9], 1, 1, S, 128, 1, 1, P(0))
    assert code == ra.RA_ERR_WORKSPACE
