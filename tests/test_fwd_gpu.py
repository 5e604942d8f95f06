"""Forward parity: the CUDA path against the float64 oracle, through the C ABI.

Bar (from the workload definitions): bf16 inputs -> max-abs 2e-2 and mean-abs 2e-3 on O,
fp32 inputs -> 1e-4, LSE within 1e-3 absolute.  Large workloads are checked on the seeded
sampled rows the oracle can afford (plus rows 0 and S-1), in the same launch
configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_exact_fwd_b200.workloads import WORKLOADS, make_inputs, random_qkv, sample_rows
from parity import assert_close_bf16, assert_close_f32, assert_lse

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ra():
    from long_context_exact_fwd_b200 import build
    build.ensure_built()
    from long_context_exact_fwd_b200 import ring_attn
    return ring_attn


def _gpu_fwd(ra, inp, D, causal, **kw):
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o, lse = ra.fwd(q, k, v, D, causal, **kw)
    assert ra.device_status() == 0
    return o.float().cpu().numpy(), lse.cpu().numpy()


def _gather(x, rows):
    B, H = rows.shape[:2]
    return np.stack([np.stack([x[b, h, rows[b, h]] for h in range(H)]) for b in range(B)])


def test_tiny_fp32_exact(ra):
    w = WORKLOADS["tiny_fp32"]
    inp = make_inputs(w)
    o, lse = _gpu_fwd(ra, inp, w.D, w.causal)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], w.causal)
    assert_close_f32(o, O)
    assert_close_f32(lse, L, "lse")


def test_s8k_causal_all_rows(ra):
    w = WORKLOADS["s8k"]
    inp = make_inputs(w)
    o, lse = _gpu_fwd(ra, inp, w.D, w.causal)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], w.causal)
    assert_close_bf16(o, O)
    assert_lse(lse, L)


@pytest.mark.slow
def test_s32k_outliers_sampled_rows(ra):
    w = WORKLOADS["s32k_outliers"]
    inp = make_inputs(w)
    rows = sample_rows(w).numpy()
    o, lse = _gpu_fwd(ra, inp, w.D, w.causal)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], w.causal, rows=rows)
    assert_close_bf16(_gather(o, rows), O)
    assert_lse(_gather(lse, rows), L)
    # rows whose visible keys include an outlier row exercise the running-max tracking
    out_rows = inp["k_outlier_rows"].numpy()
    hit = sum(int((out_rows[b, h][None, :] <= rows[b, h][:, None]).any(axis=1).sum())
              for b in range(w.B) for h in range(w.H))
    assert hit > rows.size // 2


@pytest.mark.slow
def test_s128k_sampled_rows(ra):
    w = WORKLOADS["s128k"]
    inp = make_inputs(w)
    rows = sample_rows(w).numpy()
    o, lse = _gpu_fwd(ra, inp, w.D, w.causal)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], w.causal, rows=rows)
    assert_close_bf16(_gather(o, rows), O)
    assert_lse(_gather(lse, rows), L)


def test_s16k_forward_on_oracle_heads(ra):
    w = WORKLOADS["s16k_fwd_bwd"]
    inp = make_inputs(w)
    o, lse = _gpu_fwd(ra, inp, w.D, w.causal)
    heads = [(0, h) for h in w.oracle_heads]
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], w.causal, heads=heads)
    for b, h in heads:
        assert_close_bf16(o[b, h], O[b, h])
        assert_lse(lse[b, h], L[b, h])


SHAPES = [  # (B, H, S, Dh, D): tiles, ragged tails, blocks smaller than a tile
    (1, 1, 1, 128, 1), (1, 2, 100, 128, 4), (2, 2, 128, 128, 2), (1, 2, 129, 128, 3), (1, 3, 255, 128, 5),
    (1, 2, 256, 128, 8), (1, 2, 257, 128, 1), (2, 1, 384, 128, 3), (1, 2, 1000, 128, 8), (1, 1, 2125, 128, 5),
    (1, 2, 777, 64, 7), (2, 2, 512, 64, 4), (1, 1, 64, 64, 2),
    (1, 2, 64, 128, 64),   # D = S: every ring block one token
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,H,S,Dh,D", SHAPES)
def test_small_shapes_every_row(ra, B, H, S, Dh, D, causal):
    inp = random_qkv(B, H, S, Dh, seed=S * 7 + Dh + D)
    o, lse = _gpu_fwd(ra, inp, D, causal)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    assert_close_bf16(o, O)
    assert_lse(lse, L)


@pytest.mark.parametrize("causal", [False, True])
def test_result_independent_of_ring_block_count(ra, causal):
    """Order independence (close reading §3.1): every D gives the oracle's result."""
    inp = random_qkv(1, 4, 2048, 128, seed=77)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    outs = []
    for D in (1, 2, 4, 8, 16):
        o, lse = _gpu_fwd(ra, inp, D, causal)
        assert_close_bf16(o, O)
        assert_lse(lse, L)
        outs.append(o)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2e-2


def test_explicit_scale_and_fp32_path(ra):
    inp = random_qkv(1, 2, 300, 96, seed=5, dtype=torch.float32)
    o, lse = _gpu_fwd(ra, inp, 3, True, scale=0.05)
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], True, scale=0.05)
    assert_close_f32(o, O)
    assert_close_f32(lse, L, "lse")


def test_outputs_do_not_write_past_their_end(ra):
    B, H, S, Dh = 1, 2, 300, 128
    inp = random_qkv(B, H, S, Dh, seed=11)
    n = B * H * S * Dh
    guard = 4096
    obuf = torch.full((n + guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((B * H * S + guard,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[:n].view(B, H, S, Dh)
    lse = lbuf[:B * H * S].view(B, H, S)
    ra.fwd(inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda(), 3, True, out=o, lse=lse)
    assert ra.device_status() == 0
    assert torch.all(obuf[n:] == 7.0) and torch.all(lbuf[B * H * S:] == 7.0)


def test_argument_errors_raise(ra):
    inp = random_qkv(1, 1, 256, 128, seed=1)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    with pytest.raises(ra.RingAttnError) as e:
        ra.fwd(q, k, v, 3, True)          # 256 % 3 != 0
    assert e.value.code == ra.RA_ERR_SHAPE
    with pytest.raises(ValueError):
        ra.fwd(q, k.float(), v, 4, True)  # mixed dtypes


# ---------------------------------------------------------------- merge
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_merge_matches_oracle(ra, out_dtype):
    g = torch.Generator().manual_seed(3)
    P, B, H, S, Dh = 5, 2, 3, 301, 128
    o_parts = torch.randn((P, B, H, S, Dh), generator=g)
    lse_parts = torch.randn((P, B, H, S), generator=g) * 4
    lse_parts[1, 0, 0, :50] = float("-inf")      # some parts with no visible key
    lse_parts[:, 1, 2, 7] = float("-inf")        # a row where every part is empty
    o, lse = ra.merge(o_parts.cuda(), lse_parts.cuda(), out_dtype=out_dtype)
    assert ra.device_status() == 0
    O, L = oracle.lse_merge(o_parts, lse_parts)
    if out_dtype == torch.float32:
        assert_close_f32(o.cpu().numpy(), O, tol=1e-5)
    else:
        assert_close_bf16(o.float().cpu().numpy(), O)
    assert_lse(lse.cpu().numpy(), L, tol=1e-5)
    assert np.isneginf(lse[1, 2, 7].item()) and torch.all(o[1, 2, 7] == 0)


@pytest.mark.parametrize("P,Dh", [(1, 128), (4, 64), (9, 256), (3, 36)])
def test_merge_part_counts_head_dims_and_ignored_parts(ra, P, Dh):
    # chunks of four partials with remainders, Dh not a multiple of 128, and partials marked
    # -inf whose O holds NaN: they weigh 0 and must not reach the result
    g = torch.Generator().manual_seed(20 + P)
    B, H, S = 1, 2, 77
    o_parts = torch.randn((P, B, H, S, Dh), generator=g)
    lse_parts = torch.randn((P, B, H, S), generator=g) * 3
    if P > 1:
        lse_parts[P - 1, 0, 1, ::3] = float("-inf")
        o_parts[P - 1, 0, 1, ::3] = float("nan")
    o, lse = ra.merge(o_parts.cuda(), lse_parts.cuda(), out_dtype=torch.float32)
    assert ra.device_status() == 0
    O, L = oracle.lse_merge(torch.nan_to_num(o_parts, nan=0.0), lse_parts)
    assert torch.isfinite(o).all()
    assert_close_f32(o.cpu().numpy(), O, tol=1e-5)
    assert_lse(lse.cpu().numpy(), L, tol=1e-5)


@pytest.mark.parametrize("causal", [False, True])
def test_ring_steps_as_separate_calls_then_merged(ra, causal):
    """The pages' decomposition done literally: each ring position r computes one
    partial per ring step t against block (r - t) mod D (one library call each), and the
    partials are combined with ring_attn_merge; the result is the full attention."""
    B, H, S, Dh, D = 1, 2, 1024, 128, 4
    c = S // D
    inp = random_qkv(B, H, S, Dh, seed=21)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o_parts = torch.zeros((D, B, H, S, Dh), dtype=torch.float32, device="cuda")
    lse_parts = torch.full((D, B, H, S), float("-inf"), dtype=torch.float32, device="cuda")
    for r in range(D):
        for t, j in enumerate(ra.ring_order(D, r, False)):
            if causal and j > r:
                continue
            qr = q[:, :, r * c:(r + 1) * c].contiguous()
            kj = k[:, :, j * c:(j + 1) * c].contiguous()
            vj = v[:, :, j * c:(j + 1) * c].contiguous()
            o, lse = ra.fwd(qr, kj, vj, 1, causal and j == r)
            o_parts[t, :, :, r * c:(r + 1) * c] = o.float()
            lse_parts[t, :, :, r * c:(r + 1) * c] = lse
    o, lse = ra.merge(o_parts, lse_parts, out_dtype=torch.bfloat16)
    assert ra.device_status() == 0
    O, L = oracle.attn_fwd_heads(inp["q"], inp["k"], inp["v"], causal)
    assert_close_bf16(o.float().cpu().numpy(), O)
    assert_lse(lse.cpu().numpy(), L)


def test_fma_pipe_exp2_against_exp2_and_its_bound(ra):
    """The polynomial 2^x spread onto the FMA pipes stays within its 1.0e-4 relative bound
    of the exact value (float64) on [-126, 8], returns exactly-representable powers of two
    at integers within the bound, and maps -inf to a negligible 2^-126."""
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20), torch.arange(-126, 9, dtype=torch.float32),
                   torch.tensor([float("-inf"), -1000.0])]).cuda()
    y_fma, y_mufu = ra.exp2_check(x)
    assert ra.device_status() == 0
    xs = x[:-2].double().cpu()
    exact = torch.exp2(xs)
    rel = ((y_fma[:-2].double().cpu() - exact).abs() / exact)
    assert rel.max().item() <= 1.05e-4, rel.max().item()
    rel_hw = ((y_mufu[:-2].double().cpu() - exact).abs() / exact)
    assert rel_hw.max().item() <= 2e-6              # hardware unit, for reference
    assert y_fma[-2].item() <= 1.2e-38 and y_fma[-1].item() <= 1.2e-38
    assert y_fma[-2].item() >= 0.0 and y_fma[-1].item() >= 0.0
