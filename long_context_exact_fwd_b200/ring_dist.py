"""Sequence-sharded ring attention over several GPUs (one process per GPU).

This is the pages' own system ("精读笔记 · Ring Attention with Blockwise Transformers for
Near-Infinite Context", §3.2-§3.5; "RingAttention large-context attention", 架构与算法): the
sequence is cut into D = world-size blocks, rank r holds block r of Q, K, V (and dO), and the
key/value blocks travel around the ring while every rank computes its queries against the block
it currently holds.  At ring step t rank r holds block (r - t) mod D (its own block first, the
§3.5 walk-through); the transfer of the next block is posted before the compute of the current
one, so the two overlap (§3.3).  Partial results combine through their log-sum-exp (§3.1).

The per-block work runs in the CUDA library (ring_attn_fwd / ring_attn_bwd on one block pair,
ring_attn_merge for the partials); this module is host orchestration only: torch.distributed
point-to-point sends and receives between neighbours (NCCL over NVLink on GPUs), no collective.

Causal masking is on global positions: block j is entirely visible to block r when j < r, masked
per element when j == r (the kernel's own causal mask, same positions), and skipped when j > r.
The skipped blocks still travel on, so every rank forwards D - 1 blocks.

Backward: rank r keeps dQ for its queries; the dK/dV accumulators (fp32) of a key/value block
travel with that block, collect every rank's contribution, and are back at the block's owner
after D hops.  The per-block backward uses the global O and lse, so each contribution is exact.
"""
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

BlockFwd = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, bool], Tuple[torch.Tensor, torch.Tensor]]
BlockBwd = Callable[..., Tuple[torch.Tensor, torch.Tensor, torch.Tensor]]
Merge = Callable[[torch.Tensor, torch.Tensor], Tuple[torch.Tensor, torch.Tensor]]


def _cuda_block_fwd(q, k, v, causal):
    from . import ring_attn as ra
    return ra.fwd(q, k, v, 1, causal)


def _cuda_block_bwd(q, k, v, o, lse, do, causal):
    from . import ring_attn as ra
    return ra.bwd(q, k, v, o, lse, do, 1, causal)


def _cuda_merge(o_parts, lse_parts):
    from . import ring_attn as ra
    return ra.merge(o_parts, lse_parts, out_dtype=torch.bfloat16)


def ring_steps(rank: int, world: int, causal: bool):
    """The blocks rank `rank` works on, in ring order: (step t, key/value block j, mask) for
    t = 0..world-1 with j = (rank - t) mod world; causal drops j > rank (nothing visible) and
    masks per element only for j == rank (same positions)."""
    out = []
    for t in range(world):
        j = (rank - t) % world
        if causal and j > rank:
            continue
        out.append((t, j, causal and j == rank))
    return out


class _Ring:
    """Neighbour exchange: send to rank + 1, receive from rank - 1 (mod D)."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self._reqs = []

    def _global(self, r):
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def start(self, sends, recvs):
        nxt, prv = self._global((self.rank + 1) % self.world), self._global((self.rank - 1) % self.world)
        ops = [dist.P2POp(dist.isend, s, nxt, self.group) for s in sends]
        ops += [dist.P2POp(dist.irecv, r, prv, self.group) for r in recvs]
        self._reqs = dist.batch_isend_irecv(ops)

    def wait(self):
        for r in self._reqs:
            r.wait()
        self._reqs = []


def ring_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, group=None,
             block_fwd: Optional[BlockFwd] = None, merge: Optional[Merge] = None
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward of this rank's query block.  q, k, v: [B, H, c, Dh], this rank's block of the
    sequence (rank r holds positions [r c, r c + c)).  Returns (o [B, H, c, Dh], lse [B, H, c])."""
    ring = _Ring(group)
    block_fwd = block_fwd or _cuda_block_fwd
    merge = merge or _cuda_merge
    kv = torch.stack((k, v)).contiguous()
    nxt = torch.empty_like(kv)
    parts_o, parts_l = [], []
    work = {t: masked for t, _, masked in ring_steps(ring.rank, ring.world, causal)}
    for t in range(ring.world):
        more = t + 1 < ring.world
        if more:   # the next block is in flight while this one is computed
            ring.start([kv], [nxt])
        if t in work:
            o_t, l_t = block_fwd(q, kv[0], kv[1], work[t])
            parts_o.append(o_t.float())
            parts_l.append(l_t.float())
        if more:
            ring.wait()
            kv, nxt = nxt, kv
    return merge(torch.stack(parts_o).contiguous(), torch.stack(parts_l).contiguous())


def ring_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
             do: torch.Tensor, causal: bool = True, group=None, block_bwd: Optional[BlockBwd] = None
             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Backward of this rank's blocks, given the ring forward's o and lse.  Returns
    (dq, dk, dv) for this rank's block, in the dtype of q."""
    ring = _Ring(group)
    block_bwd = block_bwd or _cuda_block_bwd
    kv = torch.stack((k, v)).contiguous()
    g = torch.zeros(kv.shape, dtype=torch.float32, device=kv.device)   # dK, dV of the block held
    kv_n, g_n = torch.empty_like(kv), torch.empty_like(g)
    dq = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    work = {t: masked for t, _, masked in ring_steps(ring.rank, ring.world, causal)}
    for t in range(ring.world):
        if t in work:
            dq_t, dk_t, dv_t = block_bwd(q, kv[0], kv[1], o, lse, do, work[t])
            dq += dq_t.float()
            g[0] += dk_t.float()
            g[1] += dv_t.float()
        if ring.world > 1:   # D hops in all: the accumulators end at their block's owner
            ring.start([kv, g], [kv_n, g_n])
            ring.wait()
            kv, kv_n = kv_n, kv
            g, g_n = g_n, g
    return dq.to(q.dtype), g[0].to(q.dtype), g[1].to(q.dtype)


def ring_fwd_emulated(q_blocks, k_blocks, v_blocks, causal: bool = True, block_fwd: Optional[BlockFwd] = None,
                      merge: Optional[Merge] = None):
    """All ranks of ring_fwd in one process, without communication: rank r's output from the
    same ring_steps schedule, the blocks taken from the lists.  For checking the block-pair
    work of a D-rank ring on one device."""
    block_fwd = block_fwd or _cuda_block_fwd
    merge = merge or _cuda_merge
    world = len(q_blocks)
    outs = []
    for r in range(world):
        parts = [block_fwd(q_blocks[r], k_blocks[j], v_blocks[j], masked) for _, j, masked in ring_steps(r, world, causal)]
        outs.append(merge(torch.stack([o.float() for o, _ in parts]).contiguous(),
                          torch.stack([l.float() for _, l in parts]).contiguous()))
    return outs


def ring_bwd_emulated(q_blocks, k_blocks, v_blocks, o_blocks, lse_blocks, do_blocks, causal: bool = True,
                      block_bwd: Optional[BlockBwd] = None):
    """All ranks of ring_bwd in one process: dQ of block r summed over its steps, dK/dV of block
    j summed over every rank that visits it (what the travelling accumulators collect)."""
    block_bwd = block_bwd or _cuda_block_bwd
    world = len(q_blocks)
    dq = [torch.zeros(b.shape, dtype=torch.float32, device=b.device) for b in q_blocks]
    dk = [torch.zeros(b.shape, dtype=torch.float32, device=b.device) for b in k_blocks]
    dv = [torch.zeros(b.shape, dtype=torch.float32, device=b.device) for b in v_blocks]
    for r in range(world):
        for _, j, masked in ring_steps(r, world, causal):
            a, b, c = block_bwd(q_blocks[r], k_blocks[j], v_blocks[j], o_blocks[r], lse_blocks[r], do_blocks[r], masked)
            dq[r] += a.float()
            dk[j] += b.float()
            dv[j] += c.float()
    dt = q_blocks[0].dtype
    return [x.to(dt) for x in dq], [x.to(dt) for x in dk], [x.to(dt) for x in dv]
