"""Float64 CPU oracle for exact ring attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference
legs may import or run it.  It shares no code with the CUDA path (no kernels, headers,
helpers, tables or pre/post-processing); the only module both sides use is the
seeded input generator ``long_context_exact_fwd_b200.workloads``, which holds no
attention arithmetic.

Every function restates a definition or algorithm step from the Ring Attention pages
("Ring Attention with Blockwise Transformers for Near-Infinite Context" close reading,
§2.1, §3.1, §3.5; "Ring Attention 与序列并行" handbook, conceptual pseudocode) in plain
NumPy float64, with library matmuls as the only primitive.  Readings of points the
pages leave open are listed in the module docstrings.

Parity pins (all in tests/test_oracle*.py, CPU only): brute-force scalar loops on tiny
inputs, closed forms (identical keys, one-hot scores, causal row 0, constant V, Q=0),
invariances (linearity in V with the LSE independent of V, key/value and query
permutations without a mask, a common shift of all keys moving each LSE by its score
offset), central finite differences, an independent torch float64 autograd check and
linearity in dO for the backward, merge identities, and order/partition independence of the blockwise ring
algorithm against the plain definition; the key-subset attention against a brute-force
loop and, over a key partition, merged to the full result; the block-pair gradient with
full-row statistics summed over block pairs to the full gradient; the per-head wrappers
(forward and backward) against per-slice calls and, for the backward over several batch
entries and heads, against batched torch float64 autograd.  The blockwise feedforward
(``ffn.py``): GELU against the normal CDF's tabulated values and its odd-part identity, the
two-matrix feedforward against a scalar loop and torch float64 library calls, the head-to-token
layout against an explicit index loop, and blockwise = whole sequence for every block size.
No function here is "parity unpinned".
"""
from .ffn import ffn_blockwise, ffn_rows, gelu, heads_to_tokens  # noqa: F401
from .attention import (  # noqa: F401
    attn_fwd,
    attn_fwd_keys,
    attn_fwd_heads,
    attn_bwd,
    attn_bwd_given_stats,
    attn_bwd_heads,
    lse_merge,
    ring_order,
    ring_attention_blockwise,
    ring_attention_partials,
)
