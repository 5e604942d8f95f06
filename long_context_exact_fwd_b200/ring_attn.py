"""ctypes binding of libringattn.so (include/ring_attn.h): argument marshalling only.

Every step of the forward, backward and merge runs in the library's CUDA kernels; this
module only checks tensor properties, allocates outputs with torch (device memory
plumbing) and passes raw pointers plus the current CUDA stream.  There is no fallback:
importing this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libringattn.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m long_context_exact_fwd_b200.build` "
        "(there is no CPU fallback)")
_lib = ctypes.CDLL(_LIB_PATH)

RA_OK, RA_ERR_ARG, RA_ERR_SHAPE, RA_ERR_ALIGN, RA_ERR_WORKSPACE, RA_ERR_CUDA, RA_ERR_TIMEOUT, RA_ERR_DEVICE = range(8)
RA_BF16, RA_F32 = 0, 1

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_ip = ctypes.POINTER(ctypes.c_int)


def _sig(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_fwd = _sig("ring_attn_fwd", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp)
_fwd_ex = _sig("ring_attn_fwd_ex", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp)
_bwd_ws = _sig("ring_attn_bwd_workspace_size", _sz, _i, _i, _i, _i)
_split_ws = _sig("ring_attn_fwd_split_workspace_size", _sz, _i, _i, _i, _i, _i)
_fwd_split = _sig("ring_attn_fwd_split", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp)
_fwd_partial = _sig("ring_attn_fwd_partial", _i, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp)
_bwd = _sig("ring_attn_bwd", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz, _vp)
_bwd_ex = _sig("ring_attn_bwd_ex", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp,
               _sz, _vp)
_merge_ex = _sig("ring_attn_merge_ex", _i, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp)
_ring_order = _sig("ring_attn_ring_order", _i, _i, _i, _i, _ip, _i)
_visit_tiles = _sig("ring_attn_visit_tiles", _i, _i, _i, _i, _i, _i, _ip, _i)
_device_status = _sig("ring_attn_device_status", _i, _vp)
_strerror = _sig("ring_attn_strerror", ctypes.c_char_p, _i)
_version = _sig("ring_attn_version", _i)
_last_cuda = _sig("ring_attn_last_cuda_error", _i, ctypes.POINTER(ctypes.c_char_p))
_bwd_visit_tiles = _sig("ring_attn_bwd_visit_tiles", _i, _i, _i, _i, _i, _i, _ip, _i)
_launch_count = _sig("ring_attn_launch_count", ctypes.c_ulonglong)
_bwd_acc = _sig("ring_attn_bwd_accumulate", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                _i, _vp, _sz, _vp)
_bwd_noalloc = _sig("ring_attn_bwd_noalloc", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp)
_noalloc_max = _sig("ring_attn_bwd_noalloc_max_bytes", _sz)
_ffn_ws = _sig("ring_attn_ffn_workspace_size", _sz, _i, _i, _i, _i)
_ffn_fwd = _sig("ring_attn_ffn_fwd", _i, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _sz, _vp)
_ffn_block = _sig("ring_attn_ffn_block", _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _i, _vp, _vp, _sz, _vp)
_exp2_check = _sig("ring_attn_exp2_check", _i, _vp, _vp, _vp, ctypes.c_longlong, _vp)
_wait_selftest = _sig("ring_attn_wait_selftest", _i, ctypes.c_longlong, _vp)


class RingAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: status {code} ({strerror(code)})"
        if code == RA_ERR_CUDA:
            err, site = last_cuda_error()
            msg += f"; last CUDA failure {err} in {site}"
        super().__init__(msg)


def last_cuda_error() -> Tuple[int, str]:
    site = ctypes.c_char_p()
    code = _last_cuda(ctypes.byref(site))
    return int(code), (site.value or b"").decode()


def strerror(code: int) -> str:
    return _strerror(code).decode()


def version() -> int:
    return _version()


def lib_path() -> str:
    return _LIB_PATH


def _check(code: int, where: str) -> None:
    if code != RA_OK:
        raise RingAttnError(code, where)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    # the library launches on the current device (and uses its static scratch there)
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device} but the current device is cuda:{torch.cuda.current_device()}; "
                         "make the tensors' device current (torch.cuda.device) before the call")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, D: int, causal: bool = True,
        scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
        lse: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Ring-attention forward.  q, k, v: [B, H, S, Dh] bf16 (or float32) CUDA tensors.
    Returns (o [B, H, S, Dh] in the input dtype, lse [B, H, S] float32)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, S, Dh]")
    B, H, S, Dh = q.shape
    dt = q.dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise ValueError("inputs must be bfloat16 or float32")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, dt, q.shape)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    _need(out, "out", dt, q.shape)
    _need(lse, "lse", torch.float32, (B, H, S))
    code = _fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, S, Dh, D,
                   1 if causal else 0, RA_BF16 if dt == torch.bfloat16 else RA_F32,
                   float(scale) if scale else 0.0, _stream(stream))
    _check(code, "ring_attn_fwd")
    return out, lse


def fwd_split_workspace_bytes(B: int, H: int, S: int, Dh: int, n_parts: int) -> int:
    return int(_split_ws(B, H, S, Dh, n_parts))


def split_parts_hint(B: int, H: int, S: int, device=None) -> int:
    """Pieces per query pair worth using: 2 while the forward has fewer than two 256-row work
    items per SM (measured on B200: H=1 S=64K +50 %, H=2 S=32K +31 %; from four items per SM
    on, splitting only adds the merge), else 1."""
    sms = torch.cuda.get_device_properties(device if device is not None else torch.cuda.current_device()) \
        .multi_processor_count
    items = B * H * ((S + 255) // 256)
    return 2 if items < 2 * sms else 1


def fwd_split(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, D: int, causal: bool = True,
              n_parts: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
              out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
              stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward with each query pair's ring cut into n_parts pieces merged through their
    log-sum-exp (ring_attn_fwd_split); n_parts None picks split_parts_hint.  q, k, v:
    [B, H, S, Dh] bf16.  Returns (o, lse); after the call `workspace` (if given) holds the
    partials."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, S, Dh]")
    B, H, S, Dh = q.shape
    if n_parts is None:
        n_parts = split_parts_hint(B, H, S, q.device)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, q.shape)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(out, "out", torch.bfloat16, q.shape)
    _need(lse, "lse", torch.float32, (B, H, S))
    need = fwd_split_workspace_bytes(B, H, S, Dh, n_parts)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    code = _fwd_split(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, S, Dh, D,
                      1 if causal else 0, n_parts, workspace.data_ptr(),
                      workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "ring_attn_fwd_split")
    return out, lse


def fwd_partial(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, D: int, causal: bool = True,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward with a float32 output (ring_attn_fwd_partial): (o [B, H, S, Dh] f32, lse
    [B, H, S] f32), one part for merge().  q, k, v: [B, H, S, Dh] bf16."""
    if q.dim() != 4:
        raise ValueError("q must be [B, H, S, Dh]")
    B, H, S, Dh = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, q.shape)
    out = torch.empty(q.shape, dtype=torch.float32, device=q.device) if out is None else out
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(out, "out", torch.float32, q.shape)
    _need(lse, "lse", torch.float32, (B, H, S))
    code = _fwd_partial(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, H, S, Dh, D,
                        1 if causal else 0, _stream(stream))
    _check(code, "ring_attn_fwd_partial")
    return out, lse


def bwd_workspace_bytes(B: int, H: int, S: int, Dh: int) -> int:
    return int(_bwd_ws(B, H, S, Dh))


def bwd(q, k, v, o, lse, do, D: int, causal: bool = True, dq=None, dk=None, dv=None,
        workspace: Optional[torch.Tensor] = None, stream=None, scale: Optional[float] = None):
    """Ring-attention backward (bf16, Dh 64 or 128; ring_attn_bwd_ex).  `scale` must be the
    forward's (None: 1/sqrt(Dh)).  Returns (dq, dk, dv), each [B, H, S, Dh] bf16."""
    B, H, S, Dh = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _need(t, name, torch.bfloat16, q.shape)
    _need(lse, "lse", torch.float32, (B, H, S))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, torch.bfloat16, q.shape)
    need = bwd_workspace_bytes(B, H, S, Dh)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    code = _bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                   dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, S, Dh, D, 1 if causal else 0,
                   float(scale) if scale else 0.0, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                   _stream(stream))
    _check(code, "ring_attn_bwd_ex")
    return dq, dk, dv


def bwd_accumulate(q, k, v, o, lse, do, D: int, causal: bool, dq32: torch.Tensor, dk32: torch.Tensor,
                   dv32: torch.Tensor, workspace: Optional[torch.Tensor] = None, stream=None):
    """Backward whose gradients are added to float32 accumulators (ring_attn_bwd_accumulate):
    dq32 += dQ, dk32 += dK, dv32 += dV, each [B, H, S, Dh] float32 cleared by the caller
    before the first call."""
    B, H, S, Dh = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _need(t, name, torch.bfloat16, q.shape)
    _need(lse, "lse", torch.float32, (B, H, S))
    for name, t in (("dq32", dq32), ("dk32", dk32), ("dv32", dv32)):
        _need(t, name, torch.float32, q.shape)
    need = bwd_workspace_bytes(B, H, S, Dh)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _need(workspace, "workspace")
    code = _bwd_acc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                    dq32.data_ptr(), dk32.data_ptr(), dv32.data_ptr(), B, H, S, Dh, D, 1 if causal else 0,
                    workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "ring_attn_bwd_accumulate")
    return dq32, dk32, dv32


def bwd_noalloc(q, k, v, o, lse, do, D: int, causal: bool = True, dq=None, dk=None, dv=None, stream=None):
    """Backward through ring_attn_bwd_noalloc: no workspace argument; the library's static
    device scratch (bwd_noalloc_max_bytes()) holds the dQ accumulator.  Calls that overlap
    on the GPU race on that scratch."""
    B, H, S, Dh = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _need(t, name, torch.bfloat16, q.shape)
    _need(lse, "lse", torch.float32, (B, H, S))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, torch.bfloat16, q.shape)
    code = _bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), do.data_ptr(),
                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, S, Dh, D, 1 if causal else 0,
                        _stream(stream))
    _check(code, "ring_attn_bwd_noalloc")
    return dq, dk, dv


def ffn_workspace_bytes(B: int, S: int, D: int, f: int) -> int:
    return int(_ffn_ws(B, S, D, f))


def ffn(o: torch.Tensor, w1: torch.Tensor, b1: torch.Tensor, w2: torch.Tensor, b2: torch.Tensor, D: int,
        block: Optional[int] = None, out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
        stream=None) -> torch.Tensor:
    """Blockwise feedforward after attention (ring_attn_ffn_fwd, or ring_attn_ffn_block for one
    ring block): o [B, H, S, Dh] bf16 attention output; w1 [f, H*Dh], w2 [H*Dh, f] bf16; b1 [f],
    b2 [H*Dh] float32.  Returns y [B, S, H*Dh] bf16 = gelu(x w1^T + b1) w2^T + b2 with
    x[b, s] the heads of token s side by side (only block `block`'s rows are written when given)."""
    if o.dim() != 4:
        raise ValueError("o must be [B, H, S, Dh]")
    B, H, S, Dh = o.shape
    h, f = H * Dh, w1.shape[0]
    _need(o, "o", torch.bfloat16)
    _need(w1, "w1", torch.bfloat16, (f, h))
    _need(w2, "w2", torch.bfloat16, (h, f))
    _need(b1, "b1", torch.float32, (f,))
    _need(b2, "b2", torch.float32, (h,))
    out = torch.empty((B, S, h), dtype=torch.bfloat16, device=o.device) if out is None else out
    _need(out, "out", torch.bfloat16, (B, S, h))
    if workspace is None:
        workspace = torch.empty(max(ffn_workspace_bytes(B, S, D, f), 1), dtype=torch.uint8, device=o.device)
    _need(workspace, "workspace")
    wsb = workspace.numel() * workspace.element_size()
    if block is None:
        code = _ffn_fwd(o.data_ptr(), B, H, S, Dh, D, w1.data_ptr(), b1.data_ptr(), w2.data_ptr(), b2.data_ptr(), f,
                        out.data_ptr(), workspace.data_ptr(), wsb, _stream(stream))
        _check(code, "ring_attn_ffn_fwd")
    else:
        code = _ffn_block(o.data_ptr(), B, H, S, Dh, D, int(block), w1.data_ptr(), b1.data_ptr(), w2.data_ptr(),
                          b2.data_ptr(), f, out.data_ptr(), workspace.data_ptr(), wsb, _stream(stream))
        _check(code, "ring_attn_ffn_block")
    return out


def bwd_noalloc_max_bytes() -> int:
    return int(_noalloc_max())


def merge(o_parts: torch.Tensor, lse_parts: torch.Tensor, out_dtype=torch.bfloat16,
          out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, stream=None):
    """LSE merge of P partials: o_parts [P, B, H, S, Dh] f32, lse_parts [P, B, H, S] f32."""
    P, B, H, S, Dh = o_parts.shape
    _need(o_parts, "o_parts", torch.float32)
    _need(lse_parts, "lse_parts", torch.float32, (P, B, H, S))
    if out is None:
        out = torch.empty((B, H, S, Dh), dtype=out_dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, H, S), dtype=torch.float32, device=o_parts.device)
    _need(out, "out", out_dtype, (B, H, S, Dh))
    _need(lse, "lse", torch.float32, (B, H, S))
    code = _merge_ex(o_parts.data_ptr(), lse_parts.data_ptr(), P, out.data_ptr(), lse.data_ptr(), B, H, S, Dh,
                     RA_BF16 if out_dtype == torch.bfloat16 else RA_F32, _stream(stream))
    _check(code, "ring_attn_merge")
    return out, lse


def ring_order(D: int, r: int, causal: bool) -> List[int]:
    """Host-side ring schedule of the library (blocks visited by position r, in order)."""
    buf = (ctypes.c_int * max(D, 1))()
    n = _ring_order(D, r, 1 if causal else 0, buf, D)
    if n < 0:
        raise RingAttnError(-n, "ring_attn_ring_order")
    return list(buf[:n])


def visit_tiles(S: int, D: int, causal: bool, q0: int, rows: int) -> List[int]:
    """Host-side copy of the forward kernel's key-tile visit order for one query tile."""
    cap = S // 128 + 2
    buf = (ctypes.c_int * cap)()
    n = _visit_tiles(S, D, 1 if causal else 0, q0, rows, buf, cap)
    if n < 0:
        raise RingAttnError(-n, "ring_attn_visit_tiles")
    return list(buf[:n])


def bwd_visit_tiles(S: int, D: int, causal: bool, k0: int, rows: int = 128) -> List[int]:
    """Host-side copy of the backward kernel's query-tile visit order for one key tile."""
    cap = S // max(rows, 1) + 2
    buf = (ctypes.c_int * cap)()
    n = _bwd_visit_tiles(S, D, 1 if causal else 0, k0, rows, buf, cap)
    if n < 0:
        raise RingAttnError(-n, "ring_attn_bwd_visit_tiles")
    return list(buf[:n])


def exp2_check(x: torch.Tensor, stream=None):
    """Evaluate the kernels' two base-2 exponentials on x (float32, CUDA): returns
    (polynomial on the FMA pipes, hardware ex2.approx)."""
    _need(x, "x", torch.float32)
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    _check(_exp2_check(x.data_ptr(), y1.data_ptr(), y2.data_ptr(), x.numel(), _stream(stream)), "ring_attn_exp2_check")
    return y1, y2


def wait_selftest(timeout_s: float = 0.05, stream=None) -> None:
    """Run the bounded-wait self-test kernel (it records RA_ERR_TIMEOUT on purpose)."""
    _check(_wait_selftest(int(timeout_s * 1e9), _stream(stream)), "ring_attn_wait_selftest")


def launch_count() -> int:
    """Kernels launched by the library since it was loaded."""
    return int(_launch_count())


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device status word."""
    return int(_device_status(_stream(stream)))


# raw entry points (for tests of the C ABI itself)
raw = _lib
