"""Float64 oracle: exact attention, its gradient, the LSE merge and the ring algorithm.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never imports it.

Sources (page title, section):
  [CR]  "精读笔记 · Ring Attention with Blockwise Transformers for Near-Infinite Context"
        (close reading): §2.1 blockwise attention without materialising the s x s
        matrix; §3.1 a query block against a group of key/value blocks may be computed
        in any order if each block's statistics are combined with rescaling; §3.2 the
        ring; §3.5 Algorithm 1 and its 4-device walk-through (the first ring step uses
        the own block, the second on device 0 uses block 3); summary: the result equals global
        attention with no approximation.
  [HB]  "Ring Attention 与序列并行" (agent handbook): conceptual pseudocode — per ring
        step, attention of the local queries against the current K/V block, folded in
        with online softmax.
  [NW]  "RingAttention large-context attention" (news deep-dive), "架构与算法": the
        per-block partial outputs are aggregated into the final output.

Readings where the pages are silent or garbled (each also listed in the design notes):
  R1 causal mask: the pages never mention one; read it as the standard autoregressive
     mask on global positions, key j allowed for query i iff j <= i.
  R2 ring order: [CR] §3.5 has step 0 on the own block, then block (p - t) mod D;
     [HB]'s pseudocode receives before the first compute.  Follow [CR].
  R3 aggregation: [NW] says the partials are summed; a plain sum of normalised
     partials is not attention.  Read it as the log-sum-exp weighted merge that
     [CR] §3.1's "statistics combined for rescaling" implies.
  R4 a partial with no allowed key has lse = -inf and weight 0; if every partial is
     -inf the merged output is O = 0, lse = -inf (never NaN).
  R5 LSE is the natural log of sum_j exp(scale * q_i . k_j), scale = 1/sqrt(Dh).
  R6 backward: the pages give no formulas; the oracle uses the analytic softmax
     gradient (textbook derivation).
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


def _as64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu")
        import torch  # local: only for dtype conversion of test inputs

        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _default_scale(Dh: int, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(Dh) if scale is None or scale <= 0 else float(scale)


# --------------------------------------------------------------------------------------
# Forward: the plain definition ([CR] summary: exact global attention, R1, R5)
# --------------------------------------------------------------------------------------
def attn_fwd(q, k, v, causal: bool, scale: Optional[float] = None,
             rows: Optional[Sequence[int]] = None, chunk: int = 512
             ) -> Tuple[np.ndarray, np.ndarray]:
    """One head.  q, k, v: [S, Dh].  Returns (O [n, Dh], LSE [n]) for the query rows
    ``rows`` (all rows when None).

    For query row i with allowed key set A_i (all keys, or j <= i when causal):
        s_ij  = scale * q_i . k_j
        LSE_i = M_i + ln sum_{j in A_i} exp(s_ij - M_i),  M_i = max_j s_ij
        O_i   = sum_{j in A_i} exp(s_ij - LSE_i) v_j
    Each row sees all of its keys at once: no blocks, no running statistics.
    """
    q, k, v = _as64(q), _as64(k), _as64(v)
    S, Dh = q.shape
    sc = _default_scale(Dh, scale)
    idx = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    O = np.zeros((idx.size, v.shape[1]), dtype=np.float64)
    L = np.full((idx.size,), NEG_INF, dtype=np.float64)
    keys = np.arange(k.shape[0])
    for a in range(0, idx.size, chunk):
        ii = idx[a:a + chunk]
        s = (q[ii] @ k.T) * sc                       # [n, S_k]
        if causal:
            s = np.where(keys[None, :] <= ii[:, None], s, NEG_INF)
        m = s.max(axis=1)
        ok = np.isfinite(m)
        m_safe = np.where(ok, m, 0.0)
        e = np.exp(s - m_safe[:, None])              # exp(-inf) = 0 for masked keys
        z = e.sum(axis=1)
        lse = np.where(ok, m_safe + np.log(np.where(ok, z, 1.0)), NEG_INF)
        w = np.where(ok[:, None], np.exp(s - np.where(ok, lse, 0.0)[:, None]), 0.0)
        O[a:a + chunk] = w @ v
        L[a:a + chunk] = lse
    return O, L


def attn_fwd_keys(q, k, v, keys: Sequence[int], causal: bool, scale: Optional[float] = None,
                  rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """One head, attention over the key positions ``keys`` only (global indices, any order):
    for query row i the allowed set is {j in keys} (and j <= i when causal), and O_i, LSE_i
    are attn_fwd's definition over that set; a row with no allowed key gets LSE = -inf and
    O = 0.  This is one partial of "精读笔记 ..." §3.1: a query block against a subset of the
    key/value blocks, to be combined with the others through lse_merge."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    S, Dh = q.shape
    sc = _default_scale(Dh, scale)
    idx = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    kk = np.asarray(keys, dtype=np.int64)
    O = np.zeros((idx.size, v.shape[1]), dtype=np.float64)
    L = np.full((idx.size,), NEG_INF, dtype=np.float64)
    if kk.size == 0:
        return O, L
    s = (q[idx] @ k[kk].T) * sc
    if causal:
        s = np.where(kk[None, :] <= idx[:, None], s, NEG_INF)
    m = s.max(axis=1)
    ok = np.isfinite(m)
    m_safe = np.where(ok, m, 0.0)
    z = np.exp(s - m_safe[:, None]).sum(axis=1)
    lse = np.where(ok, m_safe + np.log(np.where(ok, z, 1.0)), NEG_INF)
    w = np.where(ok[:, None], np.exp(s - np.where(ok, lse, 0.0)[:, None]), 0.0)
    O[:] = w @ v[kk]
    L[:] = lse
    return O, L


def attn_fwd_heads(q, k, v, causal: bool, scale: Optional[float] = None,
                   rows=None, heads: Optional[Iterable[Tuple[int, int]]] = None
                   ) -> Tuple[np.ndarray, np.ndarray]:
    """[B, H, S, Dh] inputs.  ``rows``: None, or an int array [B, H, n] of query rows.
    Returns O [B, H, n, Dh] and LSE [B, H, n] (only for ``heads`` if given; other
    entries stay NaN)."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    B, H, S, Dh = q.shape
    n = S if rows is None else np.asarray(rows).shape[-1]
    O = np.full((B, H, n, v.shape[-1]), np.nan)
    L = np.full((B, H, n), np.nan)
    hs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    for b, h in hs:
        r = None if rows is None else np.asarray(rows)[b, h]
        O[b, h], L[b, h] = attn_fwd(q[b, h], k[b, h], v[b, h], causal, scale, r)
    return O, L


# --------------------------------------------------------------------------------------
# Backward: analytic softmax gradient (R6)
# --------------------------------------------------------------------------------------
def attn_bwd(q, k, v, do, causal: bool, scale: Optional[float] = None, chunk: int = 512
             ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One head, gradients of L = sum(dO * O) for O = attn(q, k, v):
        P_ij    = exp(s_ij - LSE_i)              (0 for masked keys)
        dV      = P^T dO
        dP      = dO V^T
        Delta_i = sum_j P_ij dP_ij
        dS      = P * (dP - Delta)
        dQ      = scale * dS K,   dK = scale * dS^T Q
    Query rows are processed in chunks, each chunk against every key."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    S, Dh = q.shape
    sc = _default_scale(Dh, scale)
    _, lse = attn_fwd(q, k, v, causal, sc, chunk=chunk)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    keys = np.arange(k.shape[0])
    for a in range(0, S, chunk):
        ii = np.arange(a, min(S, a + chunk))
        s = (q[ii] @ k.T) * sc
        if causal:
            s = np.where(keys[None, :] <= ii[:, None], s, NEG_INF)
        P = np.exp(s - lse[ii][:, None])
        dP = do[ii] @ v.T
        delta = (P * dP).sum(axis=1)
        dS = P * (dP - delta[:, None])
        dv += P.T @ do[ii]
        dq[ii] = sc * (dS @ k)
        dk += sc * (dS.T @ q[ii])
    return dq, dk, dv


def attn_bwd_given_stats(q, k, v, o, lse, do, causal: bool, scale: Optional[float] = None
                         ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One head, one query block against one key/value block, with the row statistics O and
    LSE of the full rows (every key block): P = exp(S - LSE), dV = P^T dO, dP = dO V^T,
    Delta = rowsum(dO * O), dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q.
    ``causal`` masks key i > query i inside the pair (the diagonal block, same positions).
    Summing dQ over a row's key blocks, and dK, dV over a key block's query blocks, gives
    attn_bwd -- the ring backward's per-step contribution."""
    q, k, v, o, do = _as64(q), _as64(k), _as64(v), _as64(o), _as64(do)
    lse = np.asarray(lse, dtype=np.float64)
    sc = _default_scale(q.shape[1], scale)
    s = (q @ k.T) * sc
    if causal:
        n, m = s.shape
        s = np.where(np.arange(m)[None, :] <= np.arange(n)[:, None], s, NEG_INF)
    p = np.exp(s - lse[:, None])
    dv = p.T @ do
    dp = do @ v.T
    delta = (do * o).sum(axis=1)
    ds = p * (dp - delta[:, None])
    return sc * (ds @ k), sc * (ds.T @ q), dv


def attn_bwd_heads(q, k, v, do, causal: bool, scale: Optional[float] = None,
                   heads: Optional[Iterable[Tuple[int, int]]] = None):
    """[B, H, S, Dh] inputs; gradients for the listed (b, h) heads (others NaN)."""
    q, k, v, do = _as64(q), _as64(k), _as64(v), _as64(do)
    B, H, S, Dh = q.shape
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    hs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    for b, h in hs:
        dq[b, h], dk[b, h], dv[b, h] = attn_bwd(q[b, h], k[b, h], v[b, h], do[b, h], causal, scale)
    return dq, dk, dv


# --------------------------------------------------------------------------------------
# LSE merge of normalised partial outputs (R3, R4; [CR] §3.1, [NW] aggregation)
# --------------------------------------------------------------------------------------
def lse_merge(o_parts, lse_parts) -> Tuple[np.ndarray, np.ndarray]:
    """o_parts [P, ..., Dh], lse_parts [P, ...]  ->  (O [..., Dh], LSE [...]).
        LSE = ln sum_p exp(lse_p)
        O   = sum_p exp(lse_p - LSE) * O_p
    A part with lse_p = -inf has weight 0; if all parts are -inf, O = 0, LSE = -inf."""
    o_parts, lse_parts = _as64(o_parts), _as64(lse_parts)
    m = lse_parts.max(axis=0)
    ok = np.isfinite(m)
    m_safe = np.where(ok, m, 0.0)
    z = np.exp(lse_parts - m_safe[None]).sum(axis=0)
    lse = np.where(ok, m_safe + np.log(np.where(ok, z, 1.0)), NEG_INF)
    w = np.where(ok[None], np.exp(lse_parts - np.where(ok, lse, 0.0)[None]), 0.0)
    O = (w[..., None] * o_parts).sum(axis=0)
    return O, lse


# --------------------------------------------------------------------------------------
# The ring algorithm itself, in the pages' order ([CR] §3.2, §3.5; [HB] pseudocode)
# --------------------------------------------------------------------------------------
def ring_order(D: int, r: int, causal: bool) -> List[int]:
    """KV blocks visited by ring position r, in order.  At ring step t the position
    works on block (r - t) mod D; step 0 is its own block (R2).  Under the causal mask
    blocks j > r hold only later keys and are dropped (R1)."""
    order = [(r - t) % D for t in range(D)]
    if causal:
        order = [j for j in order if j <= r]
    return order


def ring_attention_blockwise(q, k, v, D: int, causal: bool, scale: Optional[float] = None,
                             orders: Optional[Sequence[Sequence[int]]] = None
                             ) -> Tuple[np.ndarray, np.ndarray]:
    """One head, the algorithm step by step.  The S tokens are cut into D blocks of
    c = S/D.  Query block r keeps a running max m, running sum l and an accumulator
    acc; for each KV block j it visits (ring order unless ``orders[r]`` is given):
        s      = scale * Q_r K_j^T          (masked entries -inf)
        m_new  = max(m, rowmax s)
        alpha  = exp(m - m_new)             (0 while m is still -inf)
        p      = exp(s - m_new)
        l      = alpha * l + rowsum p
        acc    = alpha * acc + p V_j
        m      = m_new
    and finally O_r = acc / l, LSE_r = m + ln l."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    S, Dh = q.shape
    if S % D != 0:
        raise ValueError("the sequence must split evenly into D blocks")
    c = S // D
    sc = _default_scale(Dh, scale)
    O = np.zeros((S, v.shape[1]))
    LSE = np.full((S,), NEG_INF)
    for r in range(D):
        qi = np.arange(r * c, (r + 1) * c)
        m = np.full((c,), NEG_INF)
        l = np.zeros((c,))
        acc = np.zeros((c, v.shape[1]))
        visit = ring_order(D, r, causal) if orders is None else list(orders[r])
        for j in visit:
            kj = np.arange(j * c, (j + 1) * c)
            s = (q[qi] @ k[kj].T) * sc
            if causal:
                s = np.where(kj[None, :] <= qi[:, None], s, NEG_INF)
            m_new = np.maximum(m, s.max(axis=1))
            fin = np.isfinite(m_new)
            ref = np.where(fin, m_new, 0.0)
            alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
            p = np.exp(s - ref[:, None])
            l = alpha * l + p.sum(axis=1)
            acc = alpha[:, None] * acc + p @ v[kj]
            m = m_new
        ok = l > 0
        O[qi] = np.where(ok[:, None], acc / np.where(ok, l, 1.0)[:, None], 0.0)
        LSE[qi] = np.where(ok, m + np.log(np.where(ok, l, 1.0)), NEG_INF)
    return O, LSE


def ring_attention_partials(q, k, v, D: int, causal: bool, scale: Optional[float] = None
                            ) -> Tuple[np.ndarray, np.ndarray]:
    """One head: each ring step's normalised partial (O_t, lse_t) of every query block,
    stacked [D, S, Dh] and [D, S] (lse = -inf and O = 0 for a step with no allowed
    key).  ``lse_merge`` of these is the full output (R3)."""
    q, k, v = _as64(q), _as64(k), _as64(v)
    S, Dh = q.shape
    c = S // D
    sc = _default_scale(Dh, scale)
    Op = np.zeros((D, S, v.shape[1]))
    Lp = np.full((D, S), NEG_INF)
    for r in range(D):
        qi = np.arange(r * c, (r + 1) * c)
        for t in range(D):
            j = (r - t) % D
            kj = np.arange(j * c, (j + 1) * c)
            s = (q[qi] @ k[kj].T) * sc
            if causal:
                s = np.where(kj[None, :] <= qi[:, None], s, NEG_INF)
            m = s.max(axis=1)
            ok = np.isfinite(m)
            ref = np.where(ok, m, 0.0)
            e = np.exp(s - ref[:, None])
            z = e.sum(axis=1)
            Op[t, qi] = np.where(ok[:, None], (e @ v[kj]) / np.where(ok, z, 1.0)[:, None], 0.0)
            Lp[t, qi] = np.where(ok, ref + np.log(np.where(ok, z, 1.0)), NEG_INF)
    return Op, Lp
