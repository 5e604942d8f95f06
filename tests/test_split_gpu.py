"""Split-ring forward (ring_attn_fwd_split): each 256-row query pair's ring of key tiles is
cut into n_parts pieces run as separate work items, and the normalised partials are merged
through their log-sum-exp ("精读笔记 ..." §3.1: partials over disjoint key/value blocks
combine exactly in any order).

Checked against the float64 oracle: the merged output at the forward's parity bar, and every
partial left in the workspace against the oracle's attention over exactly that piece's keys.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_fwd_b200.workloads import WORKLOADS, make_inputs, random_qkv, sample_rows
from parity import assert_close_bf16, assert_lse

pytestmark = pytest.mark.gpu

ROWS = 256   # query rows per work item (two 128-row tiles)
BN = 128     # keys per key tile


@pytest.fixture(scope="module")
def ra():
    from long_context_exact_fwd_b200 import build
    build.ensure_built()
    from long_context_exact_fwd_b200 import ring_attn
    return ring_attn


def _split(ra, inp, D, causal, n_parts):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    B, H, S, Dh = q.shape
    ws = torch.empty(ra.fwd_split_workspace_bytes(B, H, S, Dh, n_parts), dtype=torch.uint8, device="cuda")
    o, lse = ra.fwd_split(q, k, v, D, causal, n_parts=n_parts, workspace=ws)
    assert ra.device_status() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy(), ws


def _partials(ws, n_parts, B, H, S, Dh):
    rows = B * H * S
    o_bytes = n_parts * rows * Dh * 4
    o_part = ws[:o_bytes].view(torch.float32).reshape(n_parts, B, H, S, Dh).cpu().numpy()
    lse_part = ws[o_bytes:o_bytes + n_parts * rows * 4].view(torch.float32).reshape(n_parts, B, H, S).cpu().numpy()
    return o_part, lse_part


def _piece_keys(ra, S, D, causal, q0, part, n_parts):
    tiles = ra.visit_tiles(S, D, causal, q0, ROWS)
    n = len(tiles)
    piece = tiles[n * part // n_parts: n * (part + 1) // n_parts]
    keys = [j for kt in piece for j in range(kt * BN, min(kt * BN + BN, S))]
    return keys


SPLIT_SHAPES = [  # (B, H, S, Dh, D): ragged tails, short rings, one head, Dh 64
    (1, 1, 1000, 128, 8),
    (2, 2, 768, 128, 3),
    (1, 3, 1536, 64, 4),
    (1, 1, 4096, 128, 16),
]


@pytest.mark.parametrize("n_parts", [2, 3, 5, 16])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,S,Dh,D", SPLIT_SHAPES)
def test_split_matches_oracle_every_row(ra, B, H, S, Dh, D, causal, n_parts):
    inp = random_qkv(B, H, S, Dh, seed=100 + S + n_parts)
    o, lse = _split(ra, inp, D, causal, n_parts)[:2]
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    assert_close_bf16(o, O)
    assert_lse(lse, L)


@pytest.mark.parametrize("causal", [False, True])
def test_each_partial_is_attention_over_its_piece(ra, causal):
    B, H, S, Dh, D, n_parts = 1, 2, 1000, 128, 4, 3
    inp = random_qkv(B, H, S, Dh, seed=77)
    _, _, ws = _split(ra, inp, D, causal, n_parts)
    o_part, lse_part = _partials(ws, n_parts, B, H, S, Dh)
    qn, kn, vn = (inp[n].float().numpy() for n in ("q", "k", "v"))
    empty = 0
    for h in range(H):
        for q0 in range(0, S, ROWS):
            rows = np.arange(q0, min(q0 + ROWS, S))
            for part in range(n_parts):
                keys = _piece_keys(ra, S, D, causal, q0, part, n_parts)
                Op, Lp = oracle.attn_fwd_keys(qn[0, h], kn[0, h], vn[0, h], keys, causal, rows=rows)
                got_l = lse_part[part, 0, h, rows]
                assert np.array_equal(np.isneginf(got_l), np.isneginf(Lp)), (h, q0, part)
                fin = np.isfinite(Lp)
                empty += int((~fin).sum())
                if fin.any():
                    assert np.abs(got_l[fin] - Lp[fin]).max() <= 1e-3
                assert_close_bf16(o_part[part, 0, h, rows], Op, f"o_part[{part}] h{h} q0 {q0}")
    if causal:
        assert empty > 0   # the first pairs have fewer tiles than pieces: empty pieces occur


def test_one_part_is_the_plain_forward(ra):
    inp = random_qkv(1, 2, 1280, 128, seed=5)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = ra.fwd(q, k, v, 5, True)
    o2, l2 = ra.fwd_split(q, k, v, 5, True, n_parts=1, workspace=torch.empty(1, dtype=torch.uint8, device="cuda"))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.slow
def test_s32k_outliers_split_sampled_rows(ra):
    # the full-size outlier workload, cut into 4 pieces per pair, on the oracle's sampled rows
    w = WORKLOADS["s32k_outliers"]
    inp = make_inputs(w)
    rows = sample_rows(w).numpy()
    o, lse, _ = _split(ra, inp, w.D, w.causal, 4)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], w.causal, rows=rows)
    g = lambda x: np.stack([np.stack([x[b, h, rows[b, h]] for h in range(w.H)]) for b in range(w.B)])
    assert_close_bf16(g(o), O)
    assert_lse(g(lse), L)


def test_split_errors(ra):
    inp = random_qkv(1, 1, 512, 128, seed=1)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ra.RingAttnError) as e:
        ra.fwd_split(q, k, v, 4, True, n_parts=2, workspace=small)
    assert e.value.code == ra.RA_ERR_WORKSPACE
    for bad in (0, 17):
        with pytest.raises(ra.RingAttnError) as e:
            ra.fwd_split(q, k, v, 4, True, n_parts=bad)
        assert e.value.code == ra.RA_ERR_ARG


def test_auto_parts_choice(ra):
    # a single head of 1024 rows is 4 work items: well under two per SM, so the hint splits
    assert ra.split_parts_hint(1, 1, 1024) == 2
    assert ra.split_parts_hint(1, 64, 32768) == 1
    inp = random_qkv(1, 1, 1024, 128, seed=9)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = ra.fwd_split(q, k, v, 4, True)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], True)
    assert_close_bf16(o.float().cpu().numpy(), O)
    assert_lse(lse.cpu().numpy(), L)


@pytest.mark.parametrize("B,H,S,Dh,D", SPLIT_SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_partial_forward_is_the_plain_forward_in_float32(ra, B, H, S, Dh, D, causal):
    # ring_attn_fwd_partial: the whole ring as one float32 part; merged alone it must give the
    # bf16 forward bit for bit (weight exp(0) = 1, one rounding to bf16 in both)
    inp = random_qkv(B, H, S, Dh, seed=90 + S % 97 + D)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o32, l32 = ra.fwd_partial(q, k, v, D, causal)
    o16, l16 = ra.fwd(q, k, v, D, causal)
    assert o32.dtype == torch.float32 and ra.device_status() == 0
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    assert_close_bf16(o32.cpu().numpy(), O, "fp32 partial o")
    assert_lse(l32.cpu().numpy(), L)
    om, lm = ra.merge(o32[None].contiguous(), l32[None].contiguous())
    assert torch.equal(om, o16)
    assert torch.allclose(lm, l16, atol=1e-6, rtol=0)
    assert torch.equal(o32.to(torch.bfloat16), o16)
