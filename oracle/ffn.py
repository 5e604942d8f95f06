"""Float64 oracle of the blockwise feedforward that follows attention in each layer.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never imports it.

Sources (page title, section):
  [CR]  "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context":
        §2.2 (BPT): the feedforward network attached to each self-attention sub-layer is
        computed block by block, which caps its largest activation at 2bsh bytes instead of
        8bsh (b batch, s sequence, h hidden size); §1 and the summary: attention and
        feedforward are both computed in blocks, so a device holds one block at a time;
        §3.5 Algorithm 1: per transformer layer, each host's block goes through attention and
        then the feedforward.

Readings where the pages are silent (each also listed in the design notes):
  F1 shape: 8bsh bytes of bf16 activation is a hidden layer of width 4h, so the
     feedforward is the two-matrix MLP  Y = act(X W1^T + b1) W2^T + b2  with
     W1 [f, h], W2 [h, f], f = 4h by default (weights in the [out, in] layout).
  F2 activation: not named; GELU in its exact form  x * Phi(x) = x/2 (1 + erf(x / sqrt 2)).
  F3 input: the attention output of the block with its heads side by side per token,
     X[b, s, head * Dh + d] = O[b, head, s, d]  (hidden size h = H * Dh).
  F4 blocks: the D ring blocks of c = S / D tokens; the feedforward is row-wise, so any
     partition of the tokens gives the same result as the whole sequence at once.
"""
from __future__ import annotations

import math
from typing import Tuple

import numpy as np
from scipy.special import erf

from .attention import _as64


def gelu(x) -> np.ndarray:
    """Exact GELU (F2): x * Phi(x), Phi the standard normal CDF, via the error function."""
    x = _as64(x)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def heads_to_tokens(o) -> np.ndarray:
    """[B, H, S, Dh] attention output -> [B, S, H * Dh] token rows (F3)."""
    o = _as64(o)
    B, H, S, Dh = o.shape
    return np.ascontiguousarray(o.transpose(0, 2, 1, 3).reshape(B, S, H * Dh))


def ffn_rows(x, w1, b1, w2, b2) -> Tuple[np.ndarray, np.ndarray]:
    """Feedforward of token rows x [..., h] (F1): returns (Y [..., h], Z [..., f]) with
    Z = gelu(x W1^T + b1) the hidden activation and Y = Z W2^T + b2."""
    x, w1, b1, w2, b2 = (_as64(a) for a in (x, w1, b1, w2, b2))
    z = gelu(x @ w1.T + b1)
    return z @ w2.T + b2, z


def ffn_blockwise(x, w1, b1, w2, b2, c: int) -> Tuple[np.ndarray, int]:
    """BPT's blockwise feedforward ([CR] §2.2) over x [B, S, h]: the sequence is taken c tokens
    at a time, each block's hidden activation [B, c, f] computed, used and dropped before the
    next.  Returns (Y [B, S, h], the largest hidden activation held, in elements)."""
    x = _as64(x)
    B, S, _ = x.shape
    out = np.empty((B, S, _as64(w2).shape[0]))
    peak = 0
    for s0 in range(0, S, c):
        y, z = ffn_rows(x[:, s0:s0 + c], w1, b1, w2, b2)
        out[:, s0:s0 + c] = y
        peak = max(peak, z.size)
    return out, peak
