"""Sequence-sharded ring (ring_dist.ring_fwd / ring_bwd) on CPU: 2 and 4 gloo ranks.

Each rank holds one block of the sequence and the key/value blocks travel around the ring
("精读笔记 ..." §3.2-§3.5).  The per-block work is injected here as the float64 oracle (the
product binds the CUDA library instead), so these tests check the orchestration -- ring order,
causal block skipping, neighbour send/receive pairing, the LSE merge, and the travelling dK/dV
accumulators -- against the oracle's full-sequence attention and gradient.  No GPU.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _per_head(fn, *xs):
    B, H = xs[0].shape[:2]
    outs = None
    for b in range(B):
        for h in range(H):
            res = fn(*[x[b, h].numpy() if isinstance(x, torch.Tensor) else x for x in xs])
            if outs is None:
                outs = [np.zeros((B, H) + np.shape(r)) for r in res]
            for o, r in zip(outs, res):
                o[b, h] = r
    return [torch.from_numpy(o) for o in outs]


def _full_inputs(B, H, S, Dh, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, S, Dh, generator=g, dtype=torch.float64) for _ in range(4)]


def _rank_main(rank, world, port, causal, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import oracle
    from long_context_exact_fwd_b200 import ring_dist

    def block_fwd(q, k, v, masked):
        return _per_head(lambda a, b, c: oracle.attn_fwd(a, b, c, masked), q, k, v)

    def merge(o_parts, lse_parts):
        o, l = oracle.lse_merge(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o), torch.from_numpy(l)

    def block_bwd(q, k, v, o, lse, do, masked):
        return _per_head(lambda a, b, c, d, e, f: oracle.attn_bwd_given_stats(a, b, c, d, e, f, masked),
                         q, k, v, o, lse, do)

    B, H, c, Dh = 1, 2, 6, 4
    q, k, v, do = _full_inputs(B, H, world * c, Dh, seed=11)
    blk = slice(rank * c, (rank + 1) * c)
    stats = {}
    o, lse = ring_dist.ring_fwd(q[:, :, blk].contiguous(), k[:, :, blk].contiguous(), v[:, :, blk].contiguous(),
                                causal, block_fwd=block_fwd, merge=merge, stats=stats)
    dq, dk, dv = ring_dist.ring_bwd(q[:, :, blk].contiguous(), k[:, :, blk].contiguous(), v[:, :, blk].contiguous(),
                                    o, lse, do[:, :, blk].contiguous(), causal, block_bwd=block_bwd)
    O, L = _per_head(lambda a, b, cc: oracle.attn_fwd(a, b, cc, causal), q, k, v)
    dQ, dK, dV = _per_head(lambda a, b, cc, d: oracle.attn_bwd(a, b, cc, d, causal), q, k, v, do)
    err = lambda x, y: float((x.double() - y[:, :, blk]).abs().max())
    out[rank] = (err(o, O), err(lse, L), err(dq, dQ), err(dk, dK), err(dv, dV), stats["peak_partials"])
    dist.barrier()
    dist.destroy_process_group()


def _zigzag_rank_main(rank, world, port, causal, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import oracle
    from long_context_exact_fwd_b200 import ring_dist as rd

    def block_fwd(q, k, v, masked):
        return _per_head(lambda a, b, c: oracle.attn_fwd(a, b, c, masked), q, k, v)

    def merge(o_parts, lse_parts):
        o, l = oracle.lse_merge(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o), torch.from_numpy(l)

    def block_bwd(q, k, v, o, lse, do, masked):
        return _per_head(lambda a, b, c, d, e, f: oracle.attn_bwd_given_stats(a, b, c, d, e, f, masked),
                         q, k, v, o, lse, do)

    B, H, c, Dh = 1, 2, 6, 4
    q, k, v, do = _full_inputs(B, H, world * c, Dh, seed=13)
    sh = lambda x: rd.zigzag_shard(x, rank, world)
    o, lse = rd.ring_fwd_zigzag(sh(q), sh(k), sh(v), causal, block_fwd=block_fwd, merge=merge)
    dq, dk, dv = rd.ring_bwd_zigzag(sh(q), sh(k), sh(v), o, lse, sh(do), causal, block_bwd=block_bwd)
    O, L = _per_head(lambda a, b, cc: oracle.attn_fwd(a, b, cc, causal), q, k, v)
    dQ, dK, dV = _per_head(lambda a, b, cc, d: oracle.attn_bwd(a, b, cc, d, causal), q, k, v, do)
    err = lambda x, y: float((x.double() - sh(y)).abs().max())
    out[rank] = (err(o, O), err(lse, L), err(dq, dQ), err(dk, dK), err(dv, dV))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, False), (2, True), (3, True), (4, False), (4, True)])
def test_ring_over_gloo_ranks_matches_the_full_oracle(world, causal):
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), causal, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == list(range(world))
    for rank, errs in res.items():
        # the ring accumulates float32 partials of float64 blocks
        assert max(errs[:5]) < 1e-5, (rank, errs)
        # the fold keeps at most the running result and one new partial, whatever the ring
        # length (fixed per-host memory); the last rank of a 4-rank ring has 4 partials
        assert 1 <= errs[5] <= 2, (rank, errs)


def test_ring_steps_follow_the_pages_ring_order():
    sys.path.insert(0, ROOT)
    import oracle
    from long_context_exact_fwd_b200.ring_dist import ring_steps
    for world in (1, 2, 4, 7):
        for rank in range(world):
            for causal in (False, True):
                steps = ring_steps(rank, world, causal)
                assert [j for _, j, _ in steps] == oracle.ring_order(world, rank, causal)
                assert [m for _, j, m in steps] == [causal and j == rank for _, j, _ in steps]
                assert steps[0][:2] == (0, rank)   # own block first


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (4, False), (4, True)])
def test_zigzag_ring_over_gloo_ranks_matches_the_full_oracle(world, causal):
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_zigzag_rank_main, args=(world, _free_port(), causal, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == list(range(world))
    for rank, errs in res.items():
        assert max(errs) < 1e-5, (rank, errs)


def test_zigzag_shards_hold_chunks_r_and_2d_minus_1_minus_r():
    sys.path.insert(0, ROOT)
    from long_context_exact_fwd_b200 import ring_dist as rd
    for world in (1, 2, 3, 4, 8):
        S = 2 * world * 3
        pos = torch.arange(S).view(1, 1, S, 1).expand(2, 3, S, 5).contiguous()
        shards = [rd.zigzag_shard(pos, r, world) for r in range(world)]
        for r, x in enumerate(shards):
            want = list(range(3 * r, 3 * r + 3)) + list(range(3 * (2 * world - 1 - r), 3 * (2 * world - r)))
            assert x[1, 2, :, 4].tolist() == want
            assert x.is_contiguous()
        assert torch.equal(rd.zigzag_unshard(shards), pos)
        lse_like = pos[..., 0].contiguous()   # [B, H, S]: the sequence is dim 2 there too
        assert torch.equal(rd.zigzag_unshard([rd.zigzag_shard(lse_like, r, world) for r in range(world)]), lse_like)
    with pytest.raises(ValueError):
        rd.zigzag_shard(torch.zeros(1, 1, 10, 4), 0, 4)


def test_zigzag_schedule_covers_every_visible_chunk_pair_once_and_balances_the_steps():
    sys.path.insert(0, ROOT)
    from long_context_exact_fwd_b200 import ring_dist as rd
    for world in range(1, 9):
        n = 2 * world
        for causal in (False, True):
            seen = []
            for r in range(world):
                steps = rd.zigzag_steps(r, world, causal)
                assert [(t, j) for t, j, _ in steps] == [(t, (r - t) % world) for t in range(world)]
                for t, j, pairs in steps:
                    qc, kc = rd.zigzag_chunks(r, world), rd.zigzag_chunks(j, world)
                    seen += [(qc[a], kc[b], m) for a, b, m in pairs]
                    # work per step in units of one unmasked half-block pair; a masked diagonal
                    # pair holds half of one
                    work = sum(0.5 if m else 1.0 for _, _, m in pairs)
                    assert work == (2.0 if causal else 4.0), (world, r, t, pairs)
            want = [(a, b, causal and a == b) for a in range(n) for b in range(n) if not causal or b <= a]
            assert sorted(seen) == sorted(want)
    # the contiguous assignment, for contrast: rank r has r + 1 blocks of causal work
    work = [sum(0.5 if m else 1.0 for _, _, m in rd.ring_steps(r, 4, True)) for r in range(4)]
    assert work == [0.5, 1.5, 2.5, 3.5]


@pytest.mark.parametrize("n_parts", [1, 2, 5, 8])
def test_running_merge_holds_two_partials_and_equals_the_oracle_merge(n_parts):
    """The forward's running fold of per-step partials: at most two held at once for any ring
    length, and the same result as merging all partials together (order independence)."""
    sys.path.insert(0, ROOT)
    import oracle
    from long_context_exact_fwd_b200 import ring_dist as rd

    S, Dh = 5, 3
    rng = np.random.default_rng(7 + n_parts)
    q = torch.from_numpy(rng.standard_normal((1, 1, S, Dh)))
    ks = [torch.from_numpy(rng.standard_normal((1, 1, S, Dh))) for _ in range(n_parts)]
    vs = [torch.from_numpy(rng.standard_normal((1, 1, S, Dh))) for _ in range(n_parts)]

    def block_fwd(q_, k_, v_, masked):
        return _per_head(lambda a, b, c: oracle.attn_fwd(a, b, c, masked), q_, k_, v_)

    def merge(o_parts, lse_parts):
        o, l = oracle.lse_merge(o_parts.numpy(), lse_parts.numpy())
        return torch.from_numpy(o), torch.from_numpy(l)

    run = rd._RunningMerge(q, block_fwd, merge)
    for k_, v_ in zip(ks, vs):
        run.add(q, k_, v_, False)
        assert run.held <= 2
    o, l = run.result(q.dtype)
    assert run.peak == min(n_parts, 2)
    parts = [block_fwd(q, k_, v_, False) for k_, v_ in zip(ks, vs)]
    O, L = merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    np.testing.assert_allclose(o.numpy(), O.numpy(), atol=1e-12)
    np.testing.assert_allclose(l.numpy(), L.numpy(), atol=1e-12)
