"""Seeded synthetic workloads for ring attention (inputs only, no attention arithmetic).

This module is the one piece shared by the CUDA path's tests/bench and the float64
oracle: it draws the Q/K/V(/dO) tensors and the sampled query rows.  It holds none
of the method's arithmetic, so either side may use it without depending on the other.

The five workloads follow the shapes on the Ring Attention pages' setting (exact
blockwise self-attention, sequence cut into D ring blocks; "Ring Attention with
Blockwise Transformers for Near-Infinite Context", §3.5 Algorithm 1 and the 4-device
walk-through): an fp32 exactness case, and bf16 causal cases at S = 8K, 32K (with
score outliers in K), 128K, and 16K forward+backward.

Generation recipe (identical for every consumer):
  * a CPU ``torch.Generator`` seeded with the workload's seed draws ``randn`` in
    float32, in the order q, k, v, then dO (backward workloads only), each of shape
    [B, H, S, Dh];
  * for the outlier workload, after q/k/v are drawn, the same generator draws, for
    each (b, h) in row-major order, ``randperm(S)`` and keeps the first
    ``round(frac * S)`` rows; those K rows are multiplied by ``scale`` in float32;
  * the tensors are then cast to the workload dtype (bf16 rounds to nearest even).
Sampled query rows: a second generator seeded ``seed + 1000`` draws ``randperm(S)``
per (b, h) and keeps the first n rows; rows 0 and S-1 are always appended.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    Dh: int
    D: int                      # number of ring blocks (virtual ring positions)
    dtype: str                  # "bf16" or "fp32"
    causal: bool
    seed: int
    backward: bool = False
    k_outlier_frac: float = 0.0
    k_outlier_scale: float = 1.0
    sample_rows: Optional[int] = None       # oracle checks this many rows per head
    oracle_heads: Optional[Tuple[int, ...]] = None   # backward: heads the oracle covers
    note: str = ""

    @property
    def c(self) -> int:
        """Tokens per ring block."""
        return self.S // self.D

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def fwd_flops(self) -> float:
        """Causal-adjusted forward FLOPs: 4*Dh per (query, key) pair of a dense
        S x S score matrix, halved under the causal mask (S^2/2 convention)."""
        f = 4.0 * self.B * self.H * self.S * self.S * self.Dh
        return f * 0.5 if self.causal else f

    def bwd_flops(self) -> float:
        """Backward FLOPs = 2.5 x forward (five S x S x Dh contractions vs two)."""
        return 2.5 * self.fwd_flops()

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in (
        Workload("tiny_fp32", B=1, H=2, S=256, Dh=64, D=4, dtype="fp32", causal=False,
                 seed=0, note="exactness case, checked in full against the oracle"),
        Workload("s8k", B=1, H=16, S=8192, Dh=128, D=8, dtype="bf16", causal=True, seed=1,
                 note="oracle over every row"),
        Workload("s32k_outliers", B=1, H=32, S=32768, Dh=128, D=8, dtype="bf16", causal=True,
                 seed=2, k_outlier_frac=0.001, k_outlier_scale=8.0, sample_rows=256,
                 note="0.1% of K rows per head scaled x8 (score outliers)"),
        Workload("s128k", B=1, H=8, S=131072, Dh=128, D=16, dtype="bf16", causal=True, seed=3,
                 sample_rows=128),
        Workload("s16k_fwd_bwd", B=1, H=16, S=16384, Dh=128, D=8, dtype="bf16", causal=True,
                 seed=4, backward=True, oracle_heads=(0, 15)),
        Workload("s32k_h2", B=1, H=2, S=32768, Dh=128, D=8, dtype="bf16", causal=True, seed=5,
                 sample_rows=256,
                 note="few heads, long rows: 256 query-pair items for 148 SMs (split-ring case)"),
    )
}


def make_inputs(w: Workload, device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Draw the workload's tensors on the CPU (seeded), cast, then move to ``device``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.H, w.S, w.Dh)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    out = {"q": q, "k": k, "v": v}
    if w.k_outlier_frac > 0.0:
        n_out = int(round(w.k_outlier_frac * w.S))
        for b in range(w.B):
            for h in range(w.H):
                rows = torch.randperm(w.S, generator=g)[:n_out]
                k[b, h, rows, :] *= w.k_outlier_scale
        out["k_outlier_rows"] = _outlier_rows(w)  # for reporting only
    if w.backward:
        out["do"] = torch.randn(shape, generator=g, dtype=torch.float32)
    dt = w.torch_dtype
    for name in ("q", "k", "v", "do"):
        if name in out:
            out[name] = out[name].to(dt).contiguous().to(device)
    return out


def _outlier_rows(w: Workload) -> torch.Tensor:
    """Re-derive the outlier row indices [B, H, n] drawn by ``make_inputs``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    shape = (w.B, w.H, w.S, w.Dh)
    for _ in range(3):
        torch.randn(shape, generator=g, dtype=torch.float32)
    n_out = int(round(w.k_outlier_frac * w.S))
    rows = torch.empty((w.B, w.H, n_out), dtype=torch.long)
    for b in range(w.B):
        for h in range(w.H):
            rows[b, h] = torch.randperm(w.S, generator=g)[:n_out]
    return rows


def sample_rows(w: Workload, n: Optional[int] = None) -> torch.Tensor:
    """Query rows [B, H, n+2] the oracle checks: n seeded random rows + rows 0, S-1."""
    n = w.sample_rows if n is None else n
    if n is None or n >= w.S:
        return torch.arange(w.S).expand(w.B, w.H, w.S).clone()
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed + 1000)
    rows = torch.empty((w.B, w.H, n + 2), dtype=torch.long)
    for b in range(w.B):
        for h in range(w.H):
            r = torch.randperm(w.S, generator=g)[:n]
            rows[b, h, :n] = r
            rows[b, h, n] = 0
            rows[b, h, n + 1] = w.S - 1
    return rows


def ffn_weights(h: int, f: int, seed: int, dtype=torch.bfloat16, device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Seeded synthetic feedforward weights (no trained model exists here): a CPU generator
    seeded ``seed`` draws, in float32 and in this order, W1 [f, h] ~ N(0, 1/h), b1 [f] ~
    N(0, 0.1^2), W2 [h, f] ~ N(0, 1/f), b2 [h] ~ N(0, 0.1^2) (fan-in scaling keeps the
    activations O(1)); the weights are cast to ``dtype``, the biases stay float32."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    w1 = torch.randn((f, h), generator=g, dtype=torch.float32) * h ** -0.5
    b1 = torch.randn((f,), generator=g, dtype=torch.float32) * 0.1
    w2 = torch.randn((h, f), generator=g, dtype=torch.float32) * f ** -0.5
    b2 = torch.randn((h,), generator=g, dtype=torch.float32) * 0.1
    return {"w1": w1.to(dtype).contiguous().to(device), "b1": b1.to(device),
            "w2": w2.to(dtype).contiguous().to(device), "b2": b2.to(device)}


def random_qkv(B: int, H: int, S: int, Dh: int, seed: int, dtype=torch.bfloat16,
               with_do: bool = False, device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Ad-hoc seeded N(0,1) tensors for shape sweeps (same recipe, no outliers)."""
    w = Workload("adhoc", B=B, H=H, S=S, Dh=Dh, D=1, dtype="bf16" if dtype == torch.bfloat16 else "fp32",
                 causal=False, seed=seed, backward=with_do)
    return make_inputs(w, device=device)
