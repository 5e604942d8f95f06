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

Forward memory: each step's partial is folded into a running (o, lse) as soon as it is computed
(_RunningMerge), so a rank holds two partials at most, whatever D -- the fixed per-host memory of
§3.4 -- rather than one per ring step.

Backward: rank r keeps dQ for its queries; the dK/dV accumulators (fp32) of a key/value block
travel with that block, collect every rank's contribution, and are back at the block's owner
after D hops.  The per-block backward uses the global O and lse, so each contribution is exact.
K and V do not change during a step, so their transfer to the next rank is posted before the
step's compute (overlapping it, §3.3); the accumulators follow once the step has added to them.

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


def _cuda_merge_f32(o_parts, lse_parts):
    from . import ring_attn as ra
    return ra.merge(o_parts, lse_parts, out_dtype=torch.float32)


def _raise_on_device_status():
    """After a ring call on the CUDA library: synchronise and raise if a kernel gave up on a
    bounded wait (its result would be incomplete).  One synchronisation per ring call."""
    from . import ring_attn as ra
    code = ra.device_status()
    if code != ra.RA_OK:
        raise ra.RingAttnError(code, "ring kernel")


class _RunningMerge:
    """The running log-sum-exp fold of one query block's per-step partials ("精读笔记 ...",
    §3.1: blocks combined in any order through their statistics).  Each new partial is merged
    into the running (o, lse) at once, so a rank holds at most two partials whatever the ring
    length -- the fixed per-host memory of §3.4 -- instead of one per ring step.

    Default (block_fwd and merge None): the CUDA library.  Each partial is written by
    ring_attn_fwd_partial into slot 1 of a preallocated float32 pair [2][B, H, c, Dh] whose
    slot 0 holds the running result; ring_attn_merge_ex folds the pair into slot 0 of a second
    pair (float32, nothing rounded before the end), and the two pairs swap roles.  result()
    rounds once, to the input dtype.  With callables: the same fold through `merge` on two
    stacked parts (the caller's precision)."""

    def __init__(self, q, block_fwd: Optional[BlockFwd], merge: Optional[Merge]):
        self.cuda = block_fwd is None and merge is None
        self.block_fwd = block_fwd or _cuda_block_fwd
        self.merge = merge or _cuda_merge_f32     # running folds: nothing rounded yet
        self.final = merge or _cuda_merge         # the last one rounds to the output dtype
        self.state = None
        self.held = 0          # partials (running result included) alive in the fold
        self.peak = 0
        if self.cuda:
            B, H, c, Dh = q.shape
            self.pairs = [torch.empty((2, B, H, c, Dh), dtype=torch.float32, device=q.device) for _ in range(2)]
            self.lses = [torch.empty((2, B, H, c), dtype=torch.float32, device=q.device) for _ in range(2)]
            self.n = 0

    def _note(self, n):
        self.held = n
        self.peak = max(self.peak, n)

    def add(self, q, k, v, masked):
        if self.cuda:
            from . import ring_attn as ra
            a, la = self.pairs[0], self.lses[0]
            slot = 0 if self.n == 0 else 1
            ra.fwd_partial(q, k, v, 1, masked, out=a[slot], lse=la[slot])
            self._note(slot + 1)
            if self.n > 0:
                ra.merge(a, la, out_dtype=torch.float32, out=self.pairs[1][0], lse=self.lses[1][0])
                self.pairs.reverse()
                self.lses.reverse()
                self._note(1)
            self.n += 1
            return
        o_t, l_t = self.block_fwd(q, k, v, masked)
        if self.state is None:
            self.state = (o_t, l_t)
            self._note(1)
            return
        self._note(2)
        o_r, l_r = self.state
        self.state = self.merge(torch.stack((o_r.to(o_t.dtype), o_t)).contiguous(),
                                torch.stack((l_r.to(l_t.dtype), l_t)).contiguous())
        self._note(1)

    def result(self, dtype):
        if self.cuda:
            from . import ring_attn as ra
            if self.n == 0:
                raise ValueError("no partial was added")
            return ra.merge(self.pairs[0][:1], self.lses[0][:1], out_dtype=dtype)
        if self.state is None:
            raise ValueError("no partial was added")
        o, l = self.state
        return self.final(o.unsqueeze(0).contiguous(), l.unsqueeze(0).contiguous())


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
        """Post the sends to rank + 1 and the receives from rank - 1; requests accumulate
        until wait().  Every rank posts the same sequence of start() calls, so the batches
        pair up in order."""
        nxt, prv = self._global((self.rank + 1) % self.world), self._global((self.rank - 1) % self.world)
        ops = [dist.P2POp(dist.isend, s, nxt, self.group) for s in sends]
        ops += [dist.P2POp(dist.irecv, r, prv, self.group) for r in recvs]
        self._reqs += dist.batch_isend_irecv(ops)

    def wait(self):
        for r in self._reqs:
            r.wait()
        self._reqs = []


def ring_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, group=None,
             block_fwd: Optional[BlockFwd] = None, merge: Optional[Merge] = None, stats: Optional[dict] = None
             ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward of this rank's query block.  q, k, v: [B, H, c, Dh], this rank's block of the
    sequence (rank r holds positions [r c, r c + c)).  Returns (o [B, H, c, Dh], lse [B, H, c]).
    Each step's partial is folded into a running result at once (_RunningMerge), so the memory
    a rank holds does not grow with the ring length.  `stats`, if given, receives
    "peak_partials": the most partials held at once."""
    ring = _Ring(group)
    run = _RunningMerge(q, block_fwd, merge)
    kv = torch.stack((k, v)).contiguous()
    nxt = torch.empty_like(kv)
    work = {t: masked for t, _, masked in ring_steps(ring.rank, ring.world, causal)}
    for t in range(ring.world):
        more = t + 1 < ring.world
        if more:   # the next block is in flight while this one is computed
            ring.start([kv], [nxt])
        if t in work:
            run.add(q, kv[0], kv[1], work[t])
        if more:
            ring.wait()
            kv, nxt = nxt, kv
    out = run.result(q.dtype)
    if stats is not None:
        stats["peak_partials"] = run.peak
    if run.cuda:
        _raise_on_device_status()
    return out


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
        hop = ring.world > 1   # D hops in all: the accumulators end at their block's owner
        if hop:   # K, V do not change during the step: their transfer overlaps the compute
            ring.start([kv], [kv_n])
        if t in work:
            block_acc(q, kv[0], kv[1], o, lse, do, work[t], dq, g[0], g[1])
        if hop:   # the block's dK, dV accumulators leave once this step's share is in
            ring.start([g], [g_n])
            ring.wait()
            kv, kv_n = kv_n, kv
            g, g_n = g_n, g
    if block_bwd is None:
        _raise_on_device_status()
    return dq.to(q.dtype), g[0].to(q.dtype), g[1].to(q.dtype)


def ring_fwd_emulated(q_blocks, k_blocks, v_blocks, causal: bool = True, block_fwd: Optional[BlockFwd] = None,
                      merge: Optional[Merge] = None):
    """All ranks of ring_fwd in one process, without communication: rank r's output from the
    same ring_steps schedule, the blocks taken from the lists.  For checking the block-pair
    work of a D-rank ring on one device."""
    world = len(q_blocks)
    outs = []
    for r in range(world):
        run = _RunningMerge(q_blocks[r], block_fwd, merge)
        for _, j, masked in ring_steps(r, world, causal):
            run.add(q_blocks[r], k_blocks[j], v_blocks[j], masked)
        outs.append(run.result(q_blocks[r].dtype))
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


def ring_fwd_zigzag(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = True, group=None,
                    block_fwd: Optional[BlockFwd] = None, merge: Optional[Merge] = None
                    ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward of this rank's zig-zag shard.  q, k, v: [B, H, c, Dh], zigzag_shard of the full
    sequence for this rank (c = S / world, even).  Returns (o, lse) in the same shard layout."""
    ring = _Ring(group)
    qh = _halves(q)
    runs = [_RunningMerge(h, block_fwd, merge) for h in qh]   # one running fold per query half
    kv = _kv_halves(k, v)
    nxt = torch.empty_like(kv)
    for t, _, pairs in zigzag_steps(ring.rank, ring.world, causal):
        more = t + 1 < ring.world
        if more:   # the next shard is in flight while this one is computed
            ring.start([kv], [nxt])
        for a, b, masked in pairs:
            runs[a].add(qh[a], kv[b, 0], kv[b, 1], masked)
        if more:
            ring.wait()
            kv, nxt = nxt, kv
    outs = [r.result(q.dtype) for r in runs]
    if runs[0].cuda:
        _raise_on_device_status()
    return torch.cat([o for o, _ in outs], dim=2), torch.cat([l for _, l in outs], dim=2)


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
        hop = ring.world > 1   # D hops in all: the accumulators end at their shard's owner
        if hop:   # K, V do not change during the step: their transfer overlaps the compute
            ring.start([kv], [kv_n])
        for a, b, masked in pairs:
            block_acc(qh[a], kv[b, 0], kv[b, 1], oh[a], lh[a], dh[a], masked, dq[a], g[b, 0], g[b, 1])
        if hop:   # the halves' dK, dV accumulators leave once this step's share is in
            ring.start([g], [g_n])
            ring.wait()
            kv, kv_n = kv_n, kv
            g, g_n = g_n, g
    if block_bwd is None:
        _raise_on_device_status()
    dt = q.dtype
    return (torch.cat(dq, dim=2).to(dt), torch.cat((g[0, 0], g[1, 0]), dim=2).to(dt),
            torch.cat((g[0, 1], g[1, 1]), dim=2).to(dt))


def ring_fwd_zigzag_emulated(q_shards, k_shards, v_shards, causal: bool = True,
                             block_fwd: Optional[BlockFwd] = None, merge: Optional[Merge] = None):
    """All ranks of ring_fwd_zigzag in one process, without communication: rank r's (o, lse)
    from the same zigzag_steps schedule, the shards taken from the lists."""
    world = len(q_shards)
    kvs = [_kv_halves(k, v) for k, v in zip(k_shards, v_shards)]
    outs = []
    for r in range(world):
        qh = _halves(q_shards[r])
        runs = [_RunningMerge(h, block_fwd, merge) for h in qh]
        for _, j, pairs in zigzag_steps(r, world, causal):
            for a, b, masked in pairs:
                runs[a].add(qh[a], kvs[j][b, 0], kvs[j][b, 1], masked)
        res = [run.result(q_shards[r].dtype) for run in runs]
        outs.append((torch.cat([o for o, _ in res], dim=2), torch.cat([l for _, l in res], dim=2)))
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
