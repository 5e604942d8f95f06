"""Sequence-sharded ring attention over several GPUs (one process per GPU).

This is the pages' own system ("精读笔记 · Ring Attention with Blockwise Transformers for
Near-Infinite Context", §3.2-§3.5; "RingAttention large-context attention", 架构与算法): the
sequence is cut into D = world-size blocks, rank r holds block r of Q, K, V (and dO), and the
key/value blocks travel around the ring while every rank computes its queries against the block
it currently holds.  At ring step t rank r holds block (r - t) mod D (its own block first, the
§3.5 walk-through); the transfer of the next block is posted before the compute of the current
one, so the two overlap (§3.3).  Partial results combine through their log-sum-exp (§3.1).

The per-block work runs in the CUDA library (ring_attn_fwd_partial / ring_attn_bwd_accumulate on
one block pair, ring_attn_merge for the partials: each step's forward output and gradients stay
float32 until the end); this module is host orchestration only: torch.distributed
point-to-point sends and receives between neighbours (NCCL over NVLink on GPUs), no collective.

Causal masking is on global positions: block j is entirely visible to block r when j < r, masked
per element when j == r (the kernel's own causal mask, same positions), and skipped when j > r.
The skipped blocks still travel on, so every rank forwards D - 1 blocks.

Backward: rank r keeps dQ for its queries; the dK/dV accumulators (fp32) of a key/value block
travel with that block, collect every rank's contribution, and are back at the block's owner
after D hops.  The per-block backward uses the global O and lse, so each contribution is exact.

Zig-zag assignment (ring_fwd_zigzag / ring_bwd_zigzag; the striped/zig-zag variant that the
"Ring Attention" pages name as a follow-up): with contiguous blocks and a causal mask, rank r has
r + 1 blocks of work and rank D - 1 has D, so the ring waits on the last rank.  Cutting the
sequence into 2D chunks and giving rank r chunks r and 2D - 1 - r (an early and a late one) gives
every rank the same work at every ring step: two of the four half-block pairs are visible at every
step but the first, where three are (two of them on the diagonal).  The ring itself is unchanged;
only which positions a rank holds, and so which half-block pairs it computes, differ.
"""
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

BlockFwd = Callable[[torch.Tensor, torch.Tensor, torch.Tensor, bool], Tuple[torch.Tensor, torch.Tensor]]
BlockBwd = Callable[..., Tuple[torch.Tensor, torch.Tensor, torch.Tensor]]
Merge = Callable[[torch.Tensor, torch.Tensor], Tuple[torch.Tensor, torch.Tensor]]


def _cuda_block_fwd(q, k, v, causal):
    from . import ring_attn as ra
    return ra.fwd_partial(q, k, v, 1, causal)   # float32 partial, rounded to bf16 only by the merge


def _cuda_block_bwd_acc(q, k, v, o, lse, do, causal, dq32, dk32, dv32):
    from . import ring_attn as ra
    ra.bwd_accumulate(q, k, v, o, lse, do, 1, causal, dq32, dk32, dv32)   # float32, added in place


def _accumulating(block_bwd: Optional[BlockBwd]):
    """A block backward that adds its gradients to float32 accumulators: the library's
    (ring_attn_bwd_accumulate) by default, else one adding what `block_bwd` returns."""
    if block_bwd is None:
        return _cuda_block_bwd_acc

    def acc(q, k, v, o, lse, do, causal, dq32, dk32, dv32):
        a, b, c = block_bwd(q, k, v, o, lse, do, causal)
        dq32 += a.to(dq32.dtype)
        dk32 += b.to(dk32.dtype)
        dv32 += c.to(dv32.dtype)
    return acc


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
    block_acc = _accumulating(block_bwd)
    kv = torch.stack((k, v)).contiguous()
    g = torch.zeros(kv.shape, dtype=torch.float32, device=kv.device)   # dK, dV of the block held
    kv_n, g_n = torch.empty_like(kv), torch.empty_like(g)
    dq = torch.zeros(q.shape, dtype=torch.float32, device=q.device)
    work = {t: masked for t, _, masked in ring_steps(ring.rank, ring.world, causal)}
    for t in range(ring.world):
        if t in work:
            block_acc(q, kv[0], kv[1], o, lse, do, work[t], dq, g[0], g[1])
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
    block_acc = _accumulating(block_bwd)
    world = len(q_blocks)
    dq = [torch.zeros(b.shape, dtype=torch.float32, device=b.device) for b in q_blocks]
    dk = [torch.zeros(b.shape, dtype=torch.float32, device=b.device) for b in k_blocks]
    dv = [torch.zeros(b.shape, dtype=torch.float32, device=b.device) for b in v_blocks]
    for r in range(world):
        for _, j, masked in ring_steps(r, world, causal):
            block_acc(q_blocks[r], k_blocks[j], v_blocks[j], o_blocks[r], lse_blocks[r], do_blocks[r], masked,
                      dq[r], dk[j], dv[j])
    dt = q_blocks[0].dtype
    return [x.to(dt) for x in dq], [x.to(dt) for x in dk], [x.to(dt) for x in dv]


def zigzag_chunks(rank: int, world: int) -> Tuple[int, int]:
    """The two chunks (of 2 * world equal chunks of the sequence) that rank `rank` holds under the
    zig-zag assignment, in local order: chunk rank, then chunk 2 * world - 1 - rank."""
    return rank, 2 * world - 1 - rank


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 2) -> torch.Tensor:
    """Rank `rank`'s zig-zag shard of a full-sequence tensor (sequence along `dim`): its two
    chunks concatenated, early chunk first."""
    S = x.shape[dim]
    if S % (2 * world):
        raise ValueError(f"sequence length {S} is not a multiple of 2 * world = {2 * world}")
    ch = x.chunk(2 * world, dim=dim)
    a, b = zigzag_chunks(rank, world)
    return torch.cat((ch[a], ch[b]), dim=dim).contiguous()


def zigzag_unshard(shards, dim: int = 2) -> torch.Tensor:
    """The full-sequence tensor from every rank's zig-zag shard (the inverse of zigzag_shard)."""
    world = len(shards)
    chunks = [None] * (2 * world)
    for r, x in enumerate(shards):
        a, b = zigzag_chunks(r, world)
        chunks[a], chunks[b] = x.chunk(2, dim=dim)
    return torch.cat(chunks, dim=dim)


def zigzag_steps(rank: int, world: int, causal: bool):
    """The work of rank `rank` under the zig-zag assignment, in ring order: (step t, key/value rank
    j, pairs) for t = 0..world-1 with j = (rank - t) mod world, where pairs lists the half-block
    pairs (query half a, key/value half b, masked) to compute.  Half a of a rank is its chunk
    zigzag_chunks(rank)[a].  Causal: a chunk pair is visible when the key chunk does not come
    after the query chunk, and masked per element when it is the same chunk."""
    out = []
    for t in range(world):
        j = (rank - t) % world
        qc, kc = zigzag_chunks(rank, world), zigzag_chunks(j, world)
        pairs = [(a, b, causal and qc[a] == kc[b]) for a in (0, 1) for b in (0, 1)
                 if not causal or kc[b] <= qc[a]]
        out.append((t, j, pairs))
    return out


def _halves(x: torch.Tensor):
    """The two chunks of a zig-zag shard (sequence along dim 2), each contiguous."""
    if x.shape[2] % 2:
        raise ValueError(f"a zig-zag shard holds two equal chunks; length {x.shape[2]} is odd")
    return [h.contiguous() for h in x.chunk(2, dim=2)]


def _kv_halves(k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """[half][k or v][B, H, c/2, Dh]: the travelling key/value buffer of a zig-zag shard."""
    return torch.stack([torch.stack(p) for p in zip(_halves(k), _halves(v))]).contiguous()


def _merge_halves(parts, merge):
    outs = [merge(torch.stack([o for o, _ in p]).contiguous(), torch.stack([l for _, l in p]).contiguous())
            for p in parts]
    return torch.cat([o for o, _ in outs], dim=2), torch.cat([l for _, l in outs], dim=2)


def ring_fwd_zigzag(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, group=None,
                    block_fwd: Optional[BlockFwd] = None, merge: Optional[Merge] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward of this rank's zig-zag shard.  q, k, v: [B, H, c, Dh], zigzag_shard of the full
    sequence for this rank (c = S / world, even).  Returns (o, lse) in the same shard layout."""
    ring = _Ring(group)
    block_fwd = block_fwd or _cuda_block_fwd
    merge = merge or _cuda_merge
    qh = _halves(q)
    kv = _kv_halves(k, v)
    nxt = torch.empty_like(kv)
    parts = ([], [])
    for t, _, pairs in zigzag_steps(ring.rank, ring.world, causal):
        more = t + 1 < ring.world
        if more:   # the next shard is in flight while this one is computed
            ring.start([kv], [nxt])
        for a, b, masked in pairs:
            o_t, l_t = block_fwd(qh[a], kv[b, 0], kv[b, 1], masked)
            parts[a].append((o_t.float(), l_t.float()))
        if more:
            ring.wait()
            kv, nxt = nxt, kv
    return _merge_halves(parts, merge)


def ring_bwd_zigzag(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                    do: torch.Tensor, causal: bool = True, group=None, block_bwd: Optional[BlockBwd] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Backward of this rank's zig-zag shard, given ring_fwd_zigzag's o and lse (all tensors in
    the shard layout).  Returns (dq, dk, dv) in the shard layout, in the dtype of q."""
    ring = _Ring(group)
    block_acc = _accumulating(block_bwd)
    qh, oh, lh, dh = _halves(q), _halves(o), _halves(lse), _halves(do)
    kv = _kv_halves(k, v)
    g = torch.zeros(kv.shape, dtype=torch.float32, device=kv.device)   # dK, dV of the halves held
    kv_n, g_n = torch.empty_like(kv), torch.empty_like(g)
    dq = [torch.zeros(h.shape, dtype=torch.float32, device=h.device) for h in qh]
    for t, _, pairs in zigzag_steps(ring.rank, ring.world, causal):
        for a, b, masked in pairs:
            block_acc(qh[a], kv[b, 0], kv[b, 1], oh[a], lh[a], dh[a], masked, dq[a], g[b, 0], g[b, 1])
        if ring.world > 1:   # D hops in all: the accumulators end at their shard's owner
            ring.start([kv, g], [kv_n, g_n])
            ring.wait()
            kv, kv_n = kv_n, kv
            g, g_n = g_n, g
    dt = q.dtype
    return (torch.cat(dq, dim=2).to(dt), torch.cat((g[0, 0], g[1, 0]), dim=2).to(dt),
            torch.cat((g[0, 1], g[1, 1]), dim=2).to(dt))


def ring_fwd_zigzag_emulated(q_shards, k_shards, v_shards, causal: bool = True,
                             block_fwd: Optional[BlockFwd] = None, merge: Optional[Merge] = None):
    """All ranks of ring_fwd_zigzag in one process, without communication: rank r's (o, lse)
    from the same zigzag_steps schedule, the shards taken from the lists."""
    block_fwd = block_fwd or _cuda_block_fwd
    merge = merge or _cuda_merge
    world = len(q_shards)
    kvs = [_kv_halves(k, v) for k, v in zip(k_shards, v_shards)]
    outs = []
    for r in range(world):
        qh = _halves(q_shards[r])
        parts = ([], [])
        for _, j, pairs in zigzag_steps(r, world, causal):
            for a, b, masked in pairs:
                o_t, l_t = block_fwd(qh[a], kvs[j][b, 0], kvs[j][b, 1], masked)
                parts[a].append((o_t.float(), l_t.float()))
        outs.append(_merge_halves(parts, merge))
    return outs


def ring_bwd_zigzag_emulated(q_shards, k_shards, v_shards, o_shards, lse_shards, do_shards, causal: bool = True,
                             block_bwd: Optional[BlockBwd] = None):
    """All ranks of ring_bwd_zigzag in one process: dQ of each half summed over its pairs, dK/dV
    of each key/value half summed over every rank that visits it."""
    block_acc = _accumulating(block_bwd)
    world = len(q_shards)
    kvs = [_kv_halves(k, v) for k, v in zip(k_shards, v_shards)]
    gs = [torch.zeros(kv.shape, dtype=torch.float32, device=kv.device) for kv in kvs]
    dqs = []
    for r in range(world):
        qh, oh, lh, dh = _halves(q_shards[r]), _halves(o_shards[r]), _halves(lse_shards[r]), _halves(do_shards[r])
        dq = [torch.zeros(h.shape, dtype=torch.float32, device=h.device) for h in qh]
        for _, j, pairs in zigzag_steps(r, world, causal):
            for a, b, masked in pairs:
                block_acc(qh[a], kvs[j][b, 0], kvs[j][b, 1], oh[a], lh[a], dh[a], masked, dq[a], gs[j][b, 0],
                          gs[j][b, 1])
        dqs.append(torch.cat(dq, dim=2))
    dt = q_shards[0].dtype
    return ([x.to(dt) for x in dqs], [torch.cat((g[0, 0], g[1, 0]), dim=2).to(dt) for g in gs],
            [torch.cat((g[0, 1], g[1, 1]), dim=2).to(dt) for g in gs])
