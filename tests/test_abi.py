"""C ABI checks that need no GPU: the library loads, exports every declared symbol,
validates arguments before touching the device, and its host-side ring schedule matches
the oracle's ring order and the pages' worked example."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"RA_API\s+[\w\s\*]+?\b(ring_attn_\w+)\s*\(", txt)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_symbols()
    for required in ("ring_attn_fwd", "ring_attn_bwd", "ring_attn_merge"):
        assert required in names


def test_library_exports_every_declared_symbol(lib_path):
    lib = ctypes.CDLL(lib_path)
    missing = [n for n in _declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


@pytest.fixture(scope="module")
def ra(lib_path):
    from long_context_exact_fwd_b200 import ring_attn
    return ring_attn


def test_version_and_strerror(ra):
    assert ra.version() >= 100
    for code in range(8):
        assert isinstance(ra.strerror(code), str) and ra.strerror(code)
    assert "unknown" in ra.strerror(999)


def test_argument_errors_are_reported_before_any_device_work(ra):
    f = ra.raw.ring_attn_fwd_ex
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    args = lambda **kw: [P(kw.get("q", 16)), P(16), P(16), P(16), P(16), kw.get("B", 1), 2, kw.get("S", 256),
                         kw.get("Dh", 128), kw.get("D", 4), 1, kw.get("dtype", 0), ctypes.c_float(0.0), P(0)]
    assert f(*args(q=0)) == ra.RA_ERR_ARG                 # null pointer
    assert f(*args(B=0)) == ra.RA_ERR_ARG                 # non-positive size
    assert f(*args(dtype=7)) == ra.RA_ERR_ARG             # unknown dtype
    assert f(*args(S=250, D=4)) == ra.RA_ERR_SHAPE        # uneven ring split
    assert f(*args(S=4, D=8)) == ra.RA_ERR_SHAPE          # more blocks than tokens
    assert f(*args(q=18)) == ra.RA_ERR_ALIGN              # misaligned TMA source
    assert f(*args(Dh=96)) in (ra.RA_ERR_SHAPE,)          # no bf16 kernel for Dh=96
    # valid arguments on a machine without a usable sm_100 device: reported, not crashed
    import torch
    if not torch.cuda.is_available():
        assert f(*args()) in (ra.RA_ERR_CUDA, ra.RA_ERR_DEVICE)


def test_merge_and_bwd_argument_errors(ra):
    m = ra.raw.ring_attn_merge_ex
    P = ctypes.c_void_p
    assert m(P(0), P(16), 2, P(16), P(16), 1, 1, 8, 128, 0, P(0)) == ra.RA_ERR_ARG
    assert m(P(16), P(16), 0, P(16), P(16), 1, 1, 8, 128, 0, P(0)) == ra.RA_ERR_ARG
    assert m(P(16), P(16), 2, P(16), P(16), 1, 1, 8, 126, 0, P(0)) == ra.RA_ERR_SHAPE
    assert ra.bwd_workspace_bytes(1, 2, 256, 128) >= 1 * 2 * 256 * 128 * 4 + 1 * 2 * 256 * 4
    assert ra.bwd_workspace_bytes(0, 2, 256, 128) == 0


def test_backward_ex_argument_errors(ra):
    f = ra.raw.ring_attn_bwd_ex
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    big = 1 << 30
    args = lambda **kw: [P(kw.get("q", 256))] + [P(256)] * 8 + [1, 2, kw.get("S", 256), kw.get("Dh", 128),
                                                                 kw.get("D", 4), 1, ctypes.c_float(0.3),
                                                                 P(kw.get("ws", 256)),
                                                                 ctypes.c_size_t(kw.get("wsb", big)), P(0)]
    assert f(*args(q=0)) == ra.RA_ERR_ARG
    assert f(*args(Dh=96)) == ra.RA_ERR_SHAPE          # backward kernels: Dh 64 and 128
    assert f(*args(S=250)) == ra.RA_ERR_SHAPE          # uneven ring split
    assert f(*args(q=264)) == ra.RA_ERR_ALIGN
    assert f(*args(ws=0)) == ra.RA_ERR_WORKSPACE
    assert f(*args(ws=272)) == ra.RA_ERR_WORKSPACE     # not 256-byte aligned
    assert f(*args(wsb=16)) == ra.RA_ERR_WORKSPACE     # too small
    assert ra.bwd_workspace_bytes(1, 2, 256, 64) >= 1 * 2 * 256 * 64 * 4


def test_ffn_argument_errors(ra):
    f = ra.raw.ring_attn_ffn_block
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    big = 1 << 40
    args = lambda **kw: [P(kw.get("o", 256)), 1, 2, kw.get("S", 300), kw.get("Dh", 64), kw.get("D", 3),
                         kw.get("r", 0), P(256), P(kw.get("b1", 256)), P(256), P(256), kw.get("f", 256), P(256),
                         P(kw.get("ws", 256)), ctypes.c_size_t(kw.get("wsb", big)), P(0)]
    assert f(*args(o=0)) == ra.RA_ERR_ARG
    assert f(*args(r=3)) == ra.RA_ERR_ARG           # ring block out of range
    assert f(*args(r=-1)) == ra.RA_ERR_ARG
    assert f(*args(f=0)) == ra.RA_ERR_ARG
    assert f(*args(f=100)) == ra.RA_ERR_SHAPE       # hidden width: a multiple of 64
    assert f(*args(Dh=96)) == ra.RA_ERR_SHAPE
    assert f(*args(S=301)) == ra.RA_ERR_SHAPE       # uneven ring split
    assert f(*args(b1=260)) == ra.RA_ERR_ALIGN
    assert f(*args(ws=0)) == ra.RA_ERR_WORKSPACE
    assert f(*args(wsb=3 * 100 * 256 * 2)) == ra.RA_ERR_WORKSPACE   # no room for the counters
    # min(3, D) blocks' hidden activations, bf16 [nbuf][B][S/D][f], then 2 * nbuf * (B * ceil(c / 256))
    # counters (one per 256-row tile of a CTA pair and buffer), each region rounded up to 256 bytes
    r256 = lambda x: (x + 255) // 256 * 256
    assert ra.ffn_workspace_bytes(1, 300, 3, 256) == r256(3 * 100 * 256 * 2) + r256(6 * 1 * 4)
    assert ra.ffn_workspace_bytes(2, 300, 3, 64) == r256(3 * 2 * 100 * 64 * 2) + r256(6 * 2 * 4)
    assert ra.ffn_workspace_bytes(1, 1024, 2, 64) == r256(2 * 512 * 64 * 2) + r256(4 * 2 * 4)
    assert ra.ffn_workspace_bytes(64, 65536, 1, 64) == r256(64 * 65536 * 64 * 2) + r256(2 * 64 * 256 * 4)
    assert ra.ffn_workspace_bytes(1, 8192, 8, 1024) == r256(3 * 1024 * 1024 * 2) + r256(6 * 4 * 4)
    assert ra.ffn_workspace_bytes(1, 300, 7, 256) == 0


def test_split_forward_workspace_and_argument_errors(ra):
    rows = 1 * 2 * 1000
    lse_block = (rows * 4 + 255) // 256 * 256
    assert ra.fwd_split_workspace_bytes(1, 2, 1000, 128, 3) == 3 * rows * 128 * 4 + 3 * lse_block
    assert ra.fwd_split_workspace_bytes(1, 2, 1000, 128, 0) == 0
    f = ra.raw.ring_attn_fwd_split
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    args = lambda **kw: [P(kw.get("q", 256)), P(256), P(256), P(256), P(256), 1, 2, 1024, 128, 4, 1,
                         kw.get("n_parts", 2), P(kw.get("ws", 256)), ctypes.c_size_t(kw.get("ws_bytes", 1 << 40)),
                         P(0)]
    # all rejected before anything is enqueued (no device needed)
    assert f(*args(q=0)) == ra.RA_ERR_ARG
    assert f(*args(n_parts=0)) == ra.RA_ERR_ARG
    assert f(*args(n_parts=17)) == ra.RA_ERR_ARG
    assert f(*args(ws=0)) == ra.RA_ERR_WORKSPACE
    assert f(*args(ws_bytes=1024)) == ra.RA_ERR_WORKSPACE
    assert f(*args(ws=272)) == ra.RA_ERR_ALIGN          # workspace must be 256-byte aligned
    assert f(*args(q=24)) == ra.RA_ERR_ALIGN


def test_partial_forward_argument_errors(ra):
    f = ra.raw.ring_attn_fwd_partial
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    args = lambda **kw: [P(kw.get("q", 256)), P(256), P(256), P(kw.get("o", 256)), P(kw.get("lse", 256)), 1, 2,
                         kw.get("S", 1024), kw.get("Dh", 128), kw.get("D", 4), 1, P(0)]
    # all rejected before anything is enqueued (no device needed)
    assert f(*args(q=0)) == ra.RA_ERR_ARG
    assert f(*args(o=0)) == ra.RA_ERR_ARG
    assert f(*args(lse=0)) == ra.RA_ERR_ARG
    assert f(*args(S=1000, D=3)) == ra.RA_ERR_SHAPE      # S % D != 0
    assert f(*args(Dh=96)) == ra.RA_ERR_SHAPE
    assert f(*args(q=24)) == ra.RA_ERR_ALIGN
    assert f(*args(o=264)) == ra.RA_ERR_ALIGN


def test_accumulating_backward_argument_errors(ra):
    f = ra.raw.ring_attn_bwd_accumulate
    f.restype = ctypes.c_int
    P = ctypes.c_void_p
    args = lambda **kw: [P(kw.get("q", 256))] + [P(256)] * 5 + [P(kw.get("dq32", 256)), P(256), P(256), 1, 2,
                                                                 kw.get("S", 1024), kw.get("Dh", 128), 4, 1,
                                                                 P(kw.get("ws", 256)),
                                                                 ctypes.c_size_t(kw.get("ws_bytes", 1 << 40)), P(0)]
    # all rejected before anything is enqueued (no device needed)
    assert f(*args(q=0)) == ra.RA_ERR_ARG
    assert f(*args(dq32=0)) == ra.RA_ERR_ARG
    assert f(*args(S=1001)) == ra.RA_ERR_SHAPE
    assert f(*args(Dh=96)) == ra.RA_ERR_SHAPE          # backward kernels: Dh 64 and 128
    assert f(*args(dq32=264)) == ra.RA_ERR_ALIGN
    assert f(*args(ws=0)) == ra.RA_ERR_WORKSPACE
    assert f(*args(ws=272)) == ra.RA_ERR_WORKSPACE
    assert f(*args(ws_bytes=1024)) == ra.RA_ERR_WORKSPACE


@pytest.mark.parametrize("causal", [False, True])
def test_library_ring_order_matches_oracle(ra, causal):
    for D in (1, 2, 3, 4, 7, 8, 16):
        for r in range(D):
            assert ra.ring_order(D, r, causal) == oracle.ring_order(D, r, causal)


def test_library_ring_order_reproduces_the_pages_worked_example(ra):
    rows = [tuple(int(x) for x in ln.split())
            for ln in open(os.path.join(ROOT, "tests", "golden", "ring_walkthrough_d4.txt"))
            if ln.strip() and not ln.startswith("#")]
    for dev, rnd, blk in rows:
        assert ra.ring_order(4, dev, False)[rnd - 1] == blk


def _expected_tiles(S, D, causal, q0, rows, KT=128):
    """Independent restatement: ring order of the tile's block, each block's tiles
    (first key inside the block) ascending, tiles beyond the last query row dropped."""
    c = S // D
    q_last = min(q0 + rows, S) - 1
    out = []
    for j in oracle.ring_order(D, q0 // c, False):
        for kt in range(-(-j * c // KT), -(-(j + 1) * c // KT)):
            if causal and kt * KT > q_last:
                continue
            out.append(kt)
    return out


@pytest.mark.parametrize("S,D", [(256, 1), (1024, 4), (8192, 8), (1000, 8), (384, 3), (1536, 6), (130, 2),
                                 (4096, 16), (257, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_visit_tiles_schedule_and_coverage(ra, S, D, causal):
    n_tiles = -(-S // 128)
    for q0 in range(0, S, 256):
        got = ra.visit_tiles(S, D, causal, q0, 256)
        assert got == _expected_tiles(S, D, causal, q0, 256)
        # every key tile holding a key visible to some row of the query tile, exactly once
        last = min(q0 + 256, S) - 1
        need = [kt for kt in range(n_tiles) if not causal or kt * 128 <= last]
        assert sorted(got) == need


def _expected_q_tiles(S, D, causal, k0, rows=128):
    """Independent restatement for the backward: block j of the key tile travels the ring,
    visiting query blocks j, j+1, ... (mod D); each block's query tiles (first row inside
    the block) ascending; under the causal mask tiles ending before k0 are dropped."""
    c = S // D
    j = k0 // c
    out = []
    for t in range(D):
        p = (j + t) % D
        for qt in range(-(-p * c // rows), -(-(p + 1) * c // rows)):
            if causal and (qt + 1) * rows - 1 < k0:
                continue
            out.append(qt)
    return out


@pytest.mark.parametrize("S,D", [(256, 1), (1024, 4), (8192, 8), (1000, 8), (384, 3), (130, 2), (16384, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_visit_tiles_schedule_and_coverage(ra, S, D, causal):
    n_qt = -(-S // 128)
    for k0 in range(0, S, 128):
        got = ra.bwd_visit_tiles(S, D, causal, k0)
        assert got == _expected_q_tiles(S, D, causal, k0)
        need = [qt for qt in range(n_qt) if not causal or (qt + 1) * 128 - 1 >= k0]
        assert sorted(got) == need


def test_bwd_ring_order_is_the_forward_ring_seen_from_the_key_side():
    """At ring step t query block r meets key block (r - t) mod D (forward view) exactly
    when key block j meets query block (j + t) mod D (backward view)."""
    D = 8
    for r in range(D):
        for t, j in enumerate(oracle.ring_order(D, r, False)):
            assert (j + t) % D == r
