"""Pins of the blockwise-feedforward oracle against things other than itself (CPU only).

A dropped bias, a transposed weight, a wrong GELU form (tanh instead of erf, a missing 1/2),
a head/token layout slip or a block boundary error each fails at least one of these.
"""
import math

import numpy as np
import pytest
import torch

from oracle import ffn_blockwise, ffn_rows, gelu, heads_to_tokens


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_gelu_against_tabulated_normal_cdf():
    # Phi(0) = 1/2, Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208 (normal tables)
    for x, phi in ((0.5, None), (1.0, 0.8413447460685429), (2.0, 0.9772498680518208), (-1.0, 1 - 0.8413447460685429)):
        if phi is not None:
            assert abs(gelu(np.array([x]))[0] - x * phi) < 1e-15
    assert gelu(np.array([0.0]))[0] == 0.0
    # odd-part identity: x Phi(x) - (-x) Phi(-x) = x
    x = np.linspace(-6, 6, 101)
    np.testing.assert_allclose(gelu(x) - gelu(-x), x, atol=1e-14)
    # limits: GELU(x) -> x for large x, -> 0 for very negative x
    assert abs(gelu(np.array([12.0]))[0] - 12.0) < 1e-12 and abs(gelu(np.array([-12.0]))[0]) < 1e-12


def _brute_ffn(x, w1, b1, w2, b2):
    """Scalar loops, pure Python floats and math.erf."""
    out = []
    for row in x.tolist():
        z = []
        for j in range(len(b1)):
            a = b1[j] + sum(w1[j][i] * row[i] for i in range(len(row)))
            z.append(0.5 * a * (1.0 + math.erf(a / math.sqrt(2.0))))
        out.append([b2[m] + sum(w2[m][j] * z[j] for j in range(len(z))) for m in range(len(b2))])
    return np.array(out)


def test_ffn_matches_scalar_loops():
    h, f = 5, 12
    x = _rand((7, h), 1)
    w1, b1, w2, b2 = _rand((f, h), 2, 0.5), _rand(f, 3), _rand((h, f), 4, 0.3), _rand(h, 5)
    y, z = ffn_rows(x, w1, b1, w2, b2)
    np.testing.assert_allclose(y, _brute_ffn(x, w1.tolist(), b1.tolist(), w2.tolist(), b2.tolist()), atol=1e-12)
    assert z.shape == (7, f)


def test_ffn_matches_torch_library_calls():
    h, f = 16, 64
    x = _rand((3, 9, h), 6)
    w1, b1, w2, b2 = _rand((f, h), 7, 0.25), _rand(f, 8), _rand((h, f), 9, 0.125), _rand(h, 10)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    ref = torch.nn.functional.linear(torch.nn.functional.gelu(torch.nn.functional.linear(t(x), t(w1), t(b1)),
                                                              approximate="none"), t(w2), t(b2))
    np.testing.assert_allclose(ffn_rows(x, w1, b1, w2, b2)[0], ref.numpy(), atol=1e-12)


def test_heads_to_tokens_layout():
    B, H, S, Dh = 2, 3, 5, 4
    o = _rand((B, H, S, Dh), 11)
    x = heads_to_tokens(o)
    assert x.shape == (B, S, H * Dh)
    for b in range(B):
        for s in range(S):
            for hh in range(H):
                for d in range(Dh):
                    assert x[b, s, hh * Dh + d] == o[b, hh, s, d]


@pytest.mark.parametrize("c", [1, 3, 4, 6, 12, 13])
def test_blockwise_equals_whole_sequence_and_bounds_the_activation(c):
    """[CR] §2.2: the blockwise feedforward is exact and holds one block's hidden activation."""
    B, S, h, f = 2, 12, 6, 24
    x = _rand((B, S, h), 12)
    w1, b1, w2, b2 = _rand((f, h), 13, 0.4), _rand(f, 14), _rand((h, f), 15, 0.2), _rand(h, 16)
    whole = ffn_rows(x, w1, b1, w2, b2)[0]
    blk, peak = ffn_blockwise(x, w1, b1, w2, b2, c)
    np.testing.assert_allclose(blk, whole, atol=1e-12)
    assert peak == B * min(c, S) * f   # the whole-sequence activation would be B * S * f
