"""The sequence-sharded ring's block-pair work on one B200, through the CUDA library.

ring_dist.ring_fwd_emulated / ring_bwd_emulated run every rank of a D-rank ring in one process
with the same ring_steps schedule as the distributed ring_fwd / ring_bwd (no communication: the
blocks come from lists), so each block pair goes through ring_attn_fwd_partial (float32 partial) /
ring_attn_bwd_accumulate (float32 gradients added in place) with the mask the ring gives it, and
the partials through ring_attn_merge.  The zig-zag ring (ring_fwd_zigzag_emulated /
ring_bwd_zigzag_emulated) does the same on half blocks.  Compared with the float64 oracle over
the whole sequence at the bf16 parity bar (max-abs 2e-2, mean-abs 2e-3, LSE 1e-3): nothing is
rounded to bf16 before the end, so the ring's error is the single-call kernels' error.
"""
import pytest
import torch

import oracle
from long_context_exact_fwd_b200.workloads import random_qkv
from parity import assert_close_bf16, assert_lse

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rd():
    from long_context_exact_fwd_b200 import build
    build.ensure_built()
    from long_context_exact_fwd_b200 import ring_dist
    return ring_dist


def _blocks(x, D):
    return [b.contiguous() for b in x.chunk(D, dim=2)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D,c", [(2, 384), (4, 256)])
def test_emulated_ring_forward_and_backward(rd, causal, D, c):
    inp = random_qkv(1, 2, D * c, 128, seed=61 + D, with_do=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    outs = rd.ring_fwd_emulated(_blocks(q, D), _blocks(k, D), _blocks(v, D), causal)
    o = torch.cat([x for x, _ in outs], dim=2)
    lse = torch.cat([l for _, l in outs], dim=2)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    assert_close_bf16(o.float().cpu().numpy(), O, "ring o")
    assert_lse(lse.cpu().numpy(), L)

    dq, dk, dv = rd.ring_bwd_emulated(_blocks(q, D), _blocks(k, D), _blocks(v, D), _blocks(o, D), _blocks(lse, D),
                                      _blocks(do, D), causal)
    ref = oracle.attn_bwd_heads(inp["q"], inp["k"], inp["v"], inp["do"], causal)
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_close_bf16(torch.cat(got, dim=2).float().cpu().numpy(), want, "ring " + name)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D,c", [(2, 384), (4, 256)])
def test_emulated_zigzag_ring_forward_and_backward(rd, causal, D, c):
    # zig-zag shards: rank r holds chunks r and 2D - 1 - r of 2D; every half-block pair goes
    # through the library
    inp = random_qkv(1, 2, D * c, 128, seed=71 + D, with_do=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    sh = lambda x: [rd.zigzag_shard(x, r, D) for r in range(D)]
    outs = rd.ring_fwd_zigzag_emulated(sh(q), sh(k), sh(v), causal)
    o = rd.zigzag_unshard([x for x, _ in outs])
    lse = rd.zigzag_unshard([l for _, l in outs])
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    assert_close_bf16(o.float().cpu().numpy(), O, "zig-zag ring o")
    assert_lse(lse.cpu().numpy(), L)

    dq, dk, dv = rd.ring_bwd_zigzag_emulated(sh(q), sh(k), sh(v), [x for x, _ in outs], [l for _, l in outs],
                                             sh(do), causal)
    ref = oracle.attn_bwd_heads(inp["q"], inp["k"], inp["v"], inp["do"], causal)
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert_close_bf16(rd.zigzag_unshard(got).float().cpu().numpy(), want, "zig-zag ring " + name)


def test_one_rank_ring_is_the_plain_forward(rd):
    # no process group: a ring of one rank, one block, one merge of a single part
    from long_context_exact_fwd_b200 import ring_attn as ra
    inp = random_qkv(1, 2, 640, 128, seed=3)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = rd.ring_fwd(q, k, v, True)
    o2, l2 = ra.fwd(q, k, v, 1, True)
    assert torch.equal(o1, o2)
    assert torch.allclose(l1, l2, atol=1e-6, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_accumulating_backward_adds_the_plain_backward_in_float32(causal):
    # ring_attn_bwd_accumulate into cleared accumulators is ring_attn_bwd before its bf16
    # rounding: dK, dV bit for bit once rounded (fixed summation order), dQ up to the order of
    # its fp32 reduce-adds; a second call doubles them
    from long_context_exact_fwd_b200 import build
    build.ensure_built()
    from long_context_exact_fwd_b200 import ring_attn as ra
    inp = random_qkv(1, 2, 1000, 128, seed=81, with_do=True)
    q, k, v, do = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = ra.fwd(q, k, v, 4, causal)
    dq, dk, dv = ra.bwd(q, k, v, o, lse, do, 4, causal)
    acc = [torch.zeros(q.shape, dtype=torch.float32, device="cuda") for _ in range(3)]
    ra.bwd_accumulate(q, k, v, o, lse, do, 4, causal, *acc)
    assert ra.device_status() == 0
    assert torch.equal(acc[1].to(torch.bfloat16), dk)
    assert torch.equal(acc[2].to(torch.bfloat16), dv)
    assert torch.allclose(acc[0].to(torch.bfloat16).float(), dq.float(), atol=2e-2, rtol=1e-2)
    once = [a.clone() for a in acc]
    ra.bwd_accumulate(q, k, v, o, lse, do, 4, causal, *acc)
    assert torch.equal(acc[1], 2 * once[1])
    assert torch.equal(acc[2], 2 * once[2])
    assert torch.allclose(acc[0], 2 * once[0], atol=1e-4, rtol=1e-4)
