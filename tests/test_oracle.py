"""Pins of the float64 oracle against things other than itself (CPU only).

Each group is chosen so that a plausible slip in the oracle (dropped scale, wrong
causal direction, transposed operand, wrong log base, a missing term in the
gradient, a wrong merge weight) fails at least one test.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import (attn_bwd, attn_bwd_given_stats, attn_fwd, attn_fwd_heads, attn_fwd_keys, lse_merge, ring_attention_blockwise,
                    ring_attention_partials, ring_order)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- brute force
def _brute_fwd(q, k, v, causal, scale):
    """Scalar triple loop, pure Python floats."""
    S, Dh, Dv = len(q), len(q[0]), len(v[0])
    O, L = [], []
    for i in range(S):
        s = []
        for j in range(len(k)):
            if causal and j > i:
                continue
            dot = 0.0
            for d in range(Dh):
                dot += q[i][d] * k[j][d]
            s.append((j, dot * scale))
        M = max(x for _, x in s)
        Z = sum(math.exp(x - M) for _, x in s)
        lse = M + math.log(Z)
        o = [0.0] * Dv
        for j, x in s:
            w = math.exp(x - lse)
            for d in range(Dv):
                o[d] += w * v[j][d]
        O.append(o)
        L.append(lse)
    return np.array(O), np.array(L)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("S,Dh", [(1, 3), (7, 4), (13, 5)])
def test_fwd_matches_brute_force(causal, S, Dh):
    q, k, v = (_rand((S, Dh), s) * 1.5 for s in (1, 2, 3))
    sc = 1.0 / math.sqrt(Dh)
    Ob, Lb = _brute_fwd(q.tolist(), k.tolist(), v.tolist(), causal, sc)
    O, L = attn_fwd(q, k, v, causal)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=1e-12, atol=1e-12)


def _brute_fwd_keys(q, k, v, keys, causal, scale):
    """Scalar loops over an explicit key subset; global positions decide the mask."""
    S, Dh, Dv = len(q), len(q[0]), len(v[0])
    O, L = [], []
    for i in range(S):
        s = []
        for j in keys:
            if causal and j > i:
                continue
            s.append((j, sum(q[i][d] * k[j][d] for d in range(Dh)) * scale))
        if not s:
            O.append([0.0] * Dv)
            L.append(-math.inf)
            continue
        M = max(x for _, x in s)
        lse = M + math.log(sum(math.exp(x - M) for _, x in s))
        o = [0.0] * Dv
        for j, x in s:
            for d in range(Dv):
                o[d] += math.exp(x - lse) * v[j][d]
        O.append(o)
        L.append(lse)
    return np.array(O), np.array(L)


@pytest.mark.parametrize("causal", [False, True])
def test_key_subset_matches_brute_force(causal):
    S, Dh = 11, 4
    q, k, v = (_rand((S, Dh), s) * 1.3 for s in (21, 22, 23))
    keys = [9, 2, 5, 6]   # any order; rows 0 and 1 see none of them under the causal mask
    Ob, Lb = _brute_fwd_keys(q.tolist(), k.tolist(), v.tolist(), keys, causal, 1.0 / math.sqrt(Dh))
    O, L = attn_fwd_keys(q, k, v, keys, causal)
    np.testing.assert_allclose(O, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(L), np.isinf(Lb))
    fin = np.isfinite(Lb)
    np.testing.assert_allclose(L[fin], Lb[fin], rtol=1e-12, atol=1e-12)
    if causal:
        assert np.isneginf(L[:2]).all() and not O[:2].any()


@pytest.mark.parametrize("causal", [False, True])
def test_key_partition_merges_to_full(causal):
    # pieces of the key positions (one empty), merged through their lse, give the plain result
    S, Dh = 50, 6
    q, k, v = (_rand((S, Dh), s) for s in (31, 32, 33))
    perm = np.random.default_rng(34).permutation(S)
    pieces = [perm[:7], perm[7:7], perm[7:30], perm[30:]]
    parts = [attn_fwd_keys(q, k, v, p, causal) for p in pieces]
    O, L = lse_merge(np.stack([o for o, _ in parts]), np.stack([l for _, l in parts]))
    Of, Lf = attn_fwd(q, k, v, causal)
    np.testing.assert_allclose(O, Of, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(L, Lf, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_block_gradients_with_full_row_statistics_sum_to_the_gradient(causal):
    # two blocks of c positions; per-pair gradients with the full rows' O and LSE, summed over
    # the pairs a block takes part in, reproduce attn_bwd (whose own forward is the plain one)
    c, Dh = 9, 5
    q, k, v, do = (_rand((2 * c, Dh), s) for s in (41, 42, 43, 44))
    O, L = attn_fwd(q, k, v, causal)
    dQ, dK, dV = attn_bwd(q, k, v, do, causal)
    blk = [slice(0, c), slice(c, 2 * c)]
    dq = [np.zeros((c, Dh)) for _ in blk]
    dk = [np.zeros((c, Dh)) for _ in blk]
    dv = [np.zeros((c, Dh)) for _ in blk]
    for r, qs in enumerate(blk):
        for j, ks in enumerate(blk):
            if causal and j > r:
                continue
            a, b, e = attn_bwd_given_stats(q[qs], k[ks], v[ks], O[qs], L[qs], do[qs], causal and j == r)
            dq[r] += a
            dk[j] += b
            dv[j] += e
    np.testing.assert_allclose(np.concatenate(dq), dQ, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(dk), dK, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(np.concatenate(dv), dV, rtol=1e-11, atol=1e-12)


def test_fwd_row_subset_and_chunking():
    q, k, v = (_rand((40, 6), s) for s in (4, 5, 6))
    O, L = attn_fwd(q, k, v, True)
    rows = [39, 0, 17, 17, 3]
    O2, L2 = attn_fwd(q, k, v, True, rows=rows, chunk=2)
    np.testing.assert_allclose(O2, O[rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(L2, L[rows], rtol=0, atol=1e-14)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_values(causal):
    S, Dh = 11, 4
    q, v = _rand((S, Dh), 7), _rand((S, Dh), 8)
    kappa = _rand((Dh,), 9)
    k = np.tile(kappa, (S, 1))
    O, L = attn_fwd(q, k, v, causal)
    sc = 1.0 / math.sqrt(Dh)
    for i in range(S):
        n = i + 1 if causal else S
        np.testing.assert_allclose(O[i], v[:n].mean(axis=0), atol=1e-13)
        assert abs(L[i] - (sc * q[i] @ kappa + math.log(n))) < 1e-13


def test_one_hot_score_selects_one_value_row():
    S, Dh = 9, 4
    rng = np.random.default_rng(10)
    k = rng.standard_normal((S, Dh)) * 0.01
    J = 5
    k[J] = np.array([60.0, 0, 0, 0])
    q = np.tile(np.array([2.0, 0, 0, 0]), (S, 1))   # q . k_J * scale = 60
    v = rng.standard_normal((S, Dh))
    O, _ = attn_fwd(q, k, v, False)
    np.testing.assert_allclose(O, np.tile(v[J], (S, 1)), atol=1e-15)


def test_causal_row0_is_v0_and_lse_is_its_score():
    S, Dh = 8, 16
    q, k, v = (_rand((S, Dh), s) for s in (11, 12, 13))
    O, L = attn_fwd(q, k, v, True)
    np.testing.assert_allclose(O[0], v[0], atol=1e-15)
    assert abs(L[0] - q[0] @ k[0] / 4.0) < 1e-14


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_and_zero_q(causal):
    S, Dh = 10, 8
    q, k = _rand((S, Dh), 14), _rand((S, Dh), 15)
    cvec = _rand((Dh,), 16)
    O, _ = attn_fwd(q, k, np.tile(cvec, (S, 1)), causal)
    np.testing.assert_allclose(O, np.tile(cvec, (S, 1)), atol=1e-14)
    v = _rand((S, Dh), 17)
    O, L = attn_fwd(np.zeros((S, Dh)), k, v, causal)
    for i in range(S):
        n = i + 1 if causal else S
        np.testing.assert_allclose(O[i], v[:n].mean(axis=0), atol=1e-14)
        assert abs(L[i] - math.log(n)) < 1e-14


def test_explicit_scale_overrides_default():
    q, k, v = (_rand((6, 4), s) for s in (18, 19, 20))
    O1, L1 = attn_fwd(q, k, v, False, scale=0.3)
    O2, L2 = attn_fwd(q * 0.3 / 0.5, k, v, False)  # default scale 1/sqrt(4) = 0.5
    np.testing.assert_allclose(O1, O2, atol=1e-14)
    np.testing.assert_allclose(L1, L2, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_output_is_linear_in_v_and_lse_does_not_depend_on_v(causal):
    # O is a convex combination of V rows with weights fixed by Q and K
    S, Dh = 11, 5
    q, k, v1, v2 = (_rand((S, Dh), s) for s in (33, 34, 35, 36))
    O1, L1 = attn_fwd(q, k, v1, causal)
    O2, L2 = attn_fwd(q, k, v2, causal)
    O3, L3 = attn_fwd(q, k, 2.5 * v1 - 0.75 * v2, causal)
    np.testing.assert_allclose(O3, 2.5 * O1 - 0.75 * O2, atol=1e-13)
    np.testing.assert_allclose(L3, L1, atol=0)
    np.testing.assert_allclose(L2, L1, atol=0)


def test_permutations_of_keys_and_queries():
    # without a mask, attention is a function of the set of (key, value) pairs and acts row by
    # row on the queries
    S, Dh = 12, 4
    q, k, v = (_rand((S, Dh), s) for s in (37, 38, 39))
    O, L = attn_fwd(q, k, v, False)
    pk = np.random.default_rng(40).permutation(S)
    Ok, Lk = attn_fwd(q, k[pk], v[pk], False)
    np.testing.assert_allclose(Ok, O, atol=1e-13)
    np.testing.assert_allclose(Lk, L, atol=1e-13)
    pq = np.random.default_rng(41).permutation(S)
    Oq, Lq = attn_fwd(q[pq], k, v, False)
    np.testing.assert_allclose(Oq, O[pq], atol=1e-14)
    np.testing.assert_allclose(Lq, L[pq], atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_shifting_every_key_shifts_each_lse_by_its_score_offset(causal):
    # k_j + u adds scale * q_i . u to every visible score of row i: O unchanged,
    # LSE_i + scale * q_i . u
    S, Dh = 9, 6
    q, k, v = (_rand((S, Dh), s) for s in (42, 43, 44))
    u = _rand((Dh,), 45)
    O, L = attn_fwd(q, k, v, causal)
    Os, Ls = attn_fwd(q, k + u, v, causal)
    np.testing.assert_allclose(Os, O, atol=1e-13)
    np.testing.assert_allclose(Ls, L + (q @ u) / math.sqrt(Dh), atol=1e-13)


# ---------------------------------------------------------------- backward
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_is_linear_in_do(causal):
    S, Dh = 10, 4
    q, k, v, do1, do2 = (_rand((S, Dh), s) for s in (46, 47, 48, 49, 50))
    g1 = attn_bwd(q, k, v, do1, causal)
    g2 = attn_bwd(q, k, v, do2, causal)
    g3 = attn_bwd(q, k, v, -1.5 * do1 + 0.5 * do2, causal)
    for a, b, c in zip(g1, g2, g3):
        np.testing.assert_allclose(c, -1.5 * a + 0.5 * b, atol=1e-12)


def _loss(q, k, v, do, causal):
    O, _ = attn_fwd(q, k, v, causal)
    return float((O * do).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_central_finite_differences(causal):
    S, Dh = 6, 3
    q, k, v, do = (_rand((S, Dh), s) for s in (21, 22, 23, 24))
    dq, dk, dv = attn_bwd(q, k, v, do, causal)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in itertools.product(range(S), range(Dh)):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do, causal)
                        - _loss(args_m["q"], args_m["k"], args_m["v"], do, causal)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_torch_float64_autograd(causal):
    S, Dh = 33, 8
    q, k, v, do = (_rand((S, Dh), s) for s in (25, 26, 27, 28))
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = (tq @ tk.T) / math.sqrt(Dh)
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    o.backward(torch.tensor(do))
    dq, dk, dv = attn_bwd(q, k, v, do, causal, chunk=7)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_column_sum_identities(causal):
    """sum_j dK_j = 0 (each row of dS sums to zero) and sum_j dV_j = sum_i dO_i
    (each row of P sums to one)."""
    S, Dh = 40, 8
    q, k, v, do = (_rand((S, Dh), s) for s in (29, 30, 31, 32))
    dq, dk, dv = attn_bwd(q, k, v, do, causal)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)


# ---------------------------------------------------------------- merge
def test_merge_single_part_is_identity_and_neg_inf_part_is_noop():
    O = _rand((5, 4), 33)
    L = _rand((5,), 34)
    O1, L1 = lse_merge(O[None], L[None])
    np.testing.assert_allclose(O1, O, atol=1e-15)
    np.testing.assert_allclose(L1, L, atol=1e-15)
    O2, L2 = lse_merge(np.stack([O, _rand((5, 4), 35)]), np.stack([L, np.full(5, -np.inf)]))
    np.testing.assert_allclose(O2, O, atol=1e-15)
    np.testing.assert_allclose(L2, L, atol=1e-15)


def test_merge_all_neg_inf_gives_zero_and_neg_inf():
    O, L = lse_merge(_rand((3, 2, 4), 36), np.full((3, 2), -np.inf))
    assert np.all(O == 0.0) and np.all(np.isneginf(L))


def test_merge_permutation_and_associativity():
    Op, Lp = _rand((4, 6, 3), 37), _rand((4, 6), 38) * 3
    O, L = lse_merge(Op, Lp)
    perm = [2, 0, 3, 1]
    Oq, Lq = lse_merge(Op[perm], Lp[perm])
    np.testing.assert_allclose(Oq, O, atol=1e-14)
    np.testing.assert_allclose(Lq, L, atol=1e-14)
    Oa, La = lse_merge(Op[:2], Lp[:2])
    Ob, Lb = lse_merge(np.stack([Oa, Op[2], Op[3]]), np.stack([La, Lp[2], Lp[3]]))
    np.testing.assert_allclose(Ob, O, atol=1e-14)
    np.testing.assert_allclose(Lb, L, atol=1e-14)


def test_merge_of_key_halves_equals_full_attention():
    S, Dh = 24, 8
    q, k, v = (_rand((S, Dh), s) for s in (39, 40, 41))
    O, L = attn_fwd(q, k, v, False)
    parts = [attn_fwd(q, k[a:b], v[a:b], False) for a, b in ((0, 5), (5, 24))]
    Om, Lm = lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(Om, O, atol=1e-13)
    np.testing.assert_allclose(Lm, L, atol=1e-13)


# ---------------------------------------------------------------- ring algorithm
def test_ring_order_matches_the_pages_worked_example():
    rows = [tuple(int(x) for x in ln.split()) for ln in open(os.path.join(GOLDEN, "ring_walkthrough_d4.txt"))
            if ln.strip() and not ln.startswith("#")]
    for dev, rnd, blk in rows:
        assert ring_order(4, dev, False)[rnd - 1] == blk
    for dev in range(4):  # after four rounds every device has used every block once
        assert sorted(ring_order(4, dev, False)) == [0, 1, 2, 3]


def test_ring_order_causal_drops_later_blocks():
    assert ring_order(8, 0, True) == [0]
    assert ring_order(8, 5, True) == [5, 4, 3, 2, 1, 0]
    assert ring_order(8, 7, True) == [7, 6, 5, 4, 3, 2, 1, 0]
    assert ring_order(8, 2, False) == [2, 1, 0, 7, 6, 5, 4, 3]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [1, 2, 3, 4, 6, 12])
def test_blockwise_ring_equals_definition(causal, D):
    S, Dh = 36, 8
    q, k, v = (_rand((S, Dh), s) * 2 for s in (42, 43, 44))
    O, L = attn_fwd(q, k, v, causal)
    Ob, Lb = ring_attention_blockwise(q, k, v, D, causal)
    np.testing.assert_allclose(Ob, O, atol=1e-12)
    np.testing.assert_allclose(Lb, L, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_blockwise_ring_is_order_independent(causal):
    S, Dh, D = 32, 4, 8
    q, k, v = (_rand((S, Dh), s) * 3 for s in (45, 46, 47))
    O, L = attn_fwd(q, k, v, causal)
    rng = np.random.default_rng(48)
    reverse = [list(reversed(ring_order(D, r, causal))) for r in range(D)]
    shuffled = [list(rng.permutation(ring_order(D, r, causal))) for r in range(D)]
    for orders in (reverse, shuffled):
        Ob, Lb = ring_attention_blockwise(q, k, v, D, causal, orders=orders)
        np.testing.assert_allclose(Ob, O, atol=1e-12)
        np.testing.assert_allclose(Lb, L, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_merged_ring_partials_equal_definition(causal):
    S, Dh, D = 24, 8, 4
    q, k, v = (_rand((S, Dh), s) for s in (49, 50, 51))
    O, L = attn_fwd(q, k, v, causal)
    Op, Lp = ring_attention_partials(q, k, v, D, causal)
    Om, Lm = lse_merge(Op, Lp)
    np.testing.assert_allclose(Om, O, atol=1e-12)
    np.testing.assert_allclose(Lm, L, atol=1e-12)


def test_uneven_split_is_rejected():
    with pytest.raises(ValueError):
        ring_attention_blockwise(np.zeros((10, 2)), np.zeros((10, 2)), np.zeros((10, 2)), 3, False)


def test_heads_wrapper_accepts_bf16_torch_inputs():
    from long_context_exact_fwd_b200.workloads import random_qkv
    t = random_qkv(1, 2, 16, 8, seed=3)
    O, L = attn_fwd_heads(t["q"], t["k"], t["v"], True)
    O0, L0 = attn_fwd(t["q"][0, 1].double().numpy(), t["k"][0, 1].double().numpy(),
                      t["v"][0, 1].double().numpy(), True)
    np.testing.assert_allclose(O[0, 1], O0, atol=0)
    np.testing.assert_allclose(L[0, 1], L0, atol=0)


def _torch_batched_grads(q, k, v, do, causal, scale):
    """float64 autograd of the plain batched formula over [B, H, S, Dh] (a library check
    independent of the oracle's per-head code)."""
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = torch.einsum("bhid,bhjd->bhij", qt, kt) * scale
    if causal:
        S = s.shape[-1]
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.einsum("bhij,bhjd->bhid", torch.softmax(s, dim=-1), vt)
    (o * torch.tensor(do, dtype=torch.float64)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_heads_wrapper_matches_batched_autograd(causal):
    """attn_bwd_heads over [B=2, H=3]: every head equals batched float64 autograd (catches a
    head-index or batch/head transposition slip), with a non-default scale passed through."""
    B, H, S, Dh = 2, 3, 11, 5
    q, k, v, do = (_rand((B, H, S, Dh), s) for s in (61, 62, 63, 64))
    sc = 0.37
    dq, dk, dv = oracle.attn_bwd_heads(q, k, v, do, causal, scale=sc)
    tq, tk, tv = _torch_batched_grads(q, k, v, do, causal, sc)
    np.testing.assert_allclose(dq, tq, atol=1e-12)
    np.testing.assert_allclose(dk, tk, atol=1e-12)
    np.testing.assert_allclose(dv, tv, atol=1e-12)


def test_bwd_heads_wrapper_filters_heads_and_accepts_bf16_torch_inputs():
    """Listed heads equal attn_bwd on that head's float64 slices exactly; unlisted heads are NaN."""
    from long_context_exact_fwd_b200.workloads import random_qkv
    t = random_qkv(2, 3, 16, 8, seed=5, with_do=True)
    heads = [(0, 2), (1, 0)]
    dq, dk, dv = oracle.attn_bwd_heads(t["q"], t["k"], t["v"], t["do"], True, heads=heads)
    for b in range(2):
        for h in range(3):
            if (b, h) in heads:
                ref = attn_bwd(*(t[n][b, h].double().numpy() for n in ("q", "k", "v", "do")), True)
                for got, want in zip((dq, dk, dv), ref):
                    np.testing.assert_allclose(got[b, h], want, atol=0)
            else:
                assert np.isnan(dq[b, h]).all() and np.isnan(dk[b, h]).all() and np.isnan(dv[b, h]).all()
