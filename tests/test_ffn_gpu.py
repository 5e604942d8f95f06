"""Blockwise feedforward after attention (ring_attn_ffn_fwd / ring_attn_ffn_block through the
C ABI) against the float64 oracle.  The hidden activation is rounded to bf16 between the two
matrices on the GPU (the stored activation), the oracle keeps it exact; bar as for attention
with bf16 inputs: max-abs 2e-2, mean-abs 2e-3."""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_fwd_b200.workloads import WORKLOADS, ffn_weights, make_inputs, random_qkv
from parity import assert_close_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    from long_context_exact_fwd_b200 import build
    build.ensure_built()
    from long_context_exact_fwd_b200 import ring_attn
    return ring_attn


def _weights(h, f, seed):
    w = ffn_weights(h, f, seed)
    return w, {n: t.cuda() for n, t in w.items()}


# (B, H, S, Dh, D, f): ragged blocks (c = 100, 125 < 128 rows), a partial last N tile
# (f = 320, h = 192), both head dims; K = h or f an odd multiple of 64 (a 64-wide last K step),
# with two batch entries where the first product's last step ends at a batch entry's last head;
# one block (one activation buffer) and seven blocks (three buffers, reused up to twice); D = S
# (one-token blocks)
FFN_SHAPES = [(1, 2, 256, 64, 2, 256), (2, 1, 300, 128, 3, 320), (1, 4, 1000, 64, 8, 1024),
              (1, 3, 384, 64, 3, 512), (2, 2, 512, 128, 4, 1024), (2, 3, 256, 64, 2, 192),
              (1, 2, 256, 64, 1, 256), (1, 1, 1792, 128, 7, 256), (1, 1, 64, 128, 64, 128)]


@pytest.mark.parametrize("B,H,S,Dh,D,f", FFN_SHAPES)
def test_ffn_matches_oracle(ra, B, H, S, Dh, D, f):
    o = random_qkv(B, H, S, Dh, seed=500 + S)["q"]          # stands in for an attention output
    w, wd = _weights(H * Dh, f, seed=600 + f)
    y = ra.ffn(o.cuda(), wd["w1"], wd["b1"], wd["w2"], wd["b2"], D)
    assert ra.device_status() == 0
    ref, _ = oracle.ffn_rows(oracle.heads_to_tokens(o), w["w1"], w["b1"], w["w2"], w["b2"])
    assert_close_bf16(y.float().cpu().numpy(), ref, "y")


def test_ffn_single_block_writes_only_its_rows_and_matches_the_full_call(ra):
    B, H, S, Dh, D, f = 2, 2, 600, 64, 3, 512
    o = random_qkv(B, H, S, Dh, seed=7)["q"].cuda()
    _, wd = _weights(H * Dh, f, seed=8)
    full = ra.ffn(o, wd["w1"], wd["b1"], wd["w2"], wd["b2"], D)
    c = S // D
    for r in range(D):
        y = torch.full((B, S, H * Dh), float("nan"), dtype=torch.bfloat16, device="cuda")
        ra.ffn(o, wd["w1"], wd["b1"], wd["w2"], wd["b2"], D, block=r, out=y)
        assert ra.device_status() == 0
        blk = slice(r * c, (r + 1) * c)
        assert torch.equal(y[:, blk], full[:, blk])                 # same tiles, same arithmetic
        rest = torch.ones(S, dtype=torch.bool)
        rest[blk] = False
        assert torch.isnan(y[:, rest].float()).all()                # nothing outside the block


@pytest.mark.slow
def test_ffn_after_attention_at_16k_tokens_on_sampled_rows(ra):
    """The 16K-token workload: attention output of the forward, then the blockwise feedforward
    (h = 2048, f = 4h = 8192, D = 8 blocks of 2048 tokens); 96 sampled token rows + first/last."""
    w = WORKLOADS["s16k_fwd_bwd"]
    inp = make_inputs(w)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, _ = ra.fwd(q, k, v, w.D, w.causal)
    h = w.H * w.Dh
    wt, wd = _weights(h, 4 * h, seed=9)
    y = ra.ffn(o, wd["w1"], wd["b1"], wd["w2"], wd["b2"], w.D)
    assert ra.device_status() == 0
    rows = np.sort(np.concatenate([np.random.default_rng(10).choice(w.S, 96, replace=False), [0, w.S - 1]]))
    x = oracle.heads_to_tokens(o.cpu())[0, rows]
    ref, _ = oracle.ffn_rows(x, wt["w1"], wt["b1"], wt["w2"], wt["b2"])
    assert_close_bf16(y[0, rows].float().cpu().numpy(), ref, "y")
