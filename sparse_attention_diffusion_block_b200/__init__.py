"""Python binding of libpisa.so, the B200 PISA piecewise sparse attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/pisa.h.  PyTorch provides device
memory and streams.  There is no CPU fallback: importing this module fails
loudly when the library has not been built.

Entry points mirror the C names (without the ``pisa_`` prefix):
block_stats, cov_norm, cov_norm_spectral, block_first_order, select, select_route,
attn_fwd_with_sel, attn_fwd_blockwise_with_sel, attn_fwd,
attn_fwd_host, attn_fwd_with_sel_noalloc, keep_count, workspace_size, stats_workspace_size,
fused_workspace_size, host_workspace_size, autotune, set_tuning, clear_tuning, get_tuning,
tuning_save, tuning_load, set_wait_limit, device_status, status_string.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpisa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m sparse_attention_diffusion_block_b200.build` "
        "(nvcc, sm_100a).  There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

PISA_OK = 0
PISA_ERR_INVALID_ARG = -1
PISA_ERR_UNSUPPORTED = -2
PISA_ERR_WORKSPACE = -3
PISA_ERR_CUDA = -4
PISA_ERR_TIMEOUT = -5
PISA_ERR_DEVICE_CHECK = -6
PISA_BF16 = 0
PISA_FP32 = 1
PISA_ROUTE_COVARIANCE = 0
PISA_ROUTE_POOLED = 1
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # PISA_NOALLOC_SCRATCH_BYTES

EXPORTS = (
    "pisa_status_string", "pisa_keep_count", "pisa_stats_workspace_size",
    "pisa_fused_workspace_size", "pisa_workspace_size", "pisa_block_stats", "pisa_cov_norm",
    "pisa_block_first_order", "pisa_select", "pisa_attn_fwd_with_sel", "pisa_attn_fwd",
    "pisa_device_status", "pisa_attn_fwd_with_sel_noalloc", "pisa_host_workspace_size",
    "pisa_attn_fwd_host", "pisa_select_route", "pisa_cov_norm_spectral", "pisa_autotune",
    "pisa_set_tuning", "pisa_get_tuning", "pisa_tuning_save", "pisa_tuning_load",
    "pisa_set_wait_limit", "pisa_attn_fwd_blockwise_with_sel",
)

_p = ctypes.c_void_p
_i = ctypes.c_int
_z = ctypes.c_size_t
_f = ctypes.c_float


def _sig(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_lib_status_string = _sig("pisa_status_string", ctypes.c_char_p, _i)
_lib_keep_count = _sig("pisa_keep_count", _i, _i, _i, _f)
_lib_stats_ws = _sig("pisa_stats_workspace_size", _z, _i, _i, _i, _i, _i)
_lib_fused_ws = _sig("pisa_fused_workspace_size", _z, _i, _i, _i, _i, _i)
_lib_ws = _sig("pisa_workspace_size", _z, _i, _i, _i, _i, _i, _i)
_lib_block_stats = _sig("pisa_block_stats", _i, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                        _p, _p, _p, _p, _p, _z, _p)
_lib_cov_norm = _sig("pisa_cov_norm", _i, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p)
_lib_first_order = _sig("pisa_block_first_order", _i, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p)
_lib_select = _sig("pisa_select", _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p)
_lib_fwd_sel = _sig("pisa_attn_fwd_with_sel", _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                    _p, _p, _p, _p, _i, _p, _z, _p)
_lib_fwd_sel_noalloc = _sig("pisa_attn_fwd_with_sel_noalloc", _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                            _p, _p, _p, _p, _i, _p)
_lib_fwd = _sig("pisa_attn_fwd", _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _z, _p)
_lib_device_status = _sig("pisa_device_status", _i, _p, _i)
_lib_host_ws = _sig("pisa_host_workspace_size", _z, _i, _i, _i, _i, _i, _i, _i, _i)
_lib_select_route = _sig("pisa_select_route", _i, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p)
_lib_cov_spectral = _sig("pisa_cov_norm_spectral", _i, _p, _p, _i, _i, _i, _i, _i, _p, _p)
class _Tuning(ctypes.Structure):
    _fields_ = [("cov_blocks_per_cta", ctypes.c_int), ("select_rows_per_cta", ctypes.c_int),
                ("fused_ctas", ctypes.c_int)]


_TP = ctypes.POINTER(_Tuning)
_lib_autotune = _sig("pisa_autotune", _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p, _z, _p, _TP)
_lib_set_tuning = _sig("pisa_set_tuning", _i, _i, _i, _i, _i, _i, _TP)
_lib_get_tuning = _sig("pisa_get_tuning", _i, _i, _i, _i, _i, _i, _TP)
_lib_tuning_save = _sig("pisa_tuning_save", _i, ctypes.c_char_p)
_lib_tuning_load = _sig("pisa_tuning_load", _i, ctypes.c_char_p)
_lib_fwd_blockwise = _sig("pisa_attn_fwd_blockwise_with_sel", _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i,
                          _p, _p, _p, _p, _i, _p)
_lib_set_wait_limit = _sig("pisa_set_wait_limit", _i, ctypes.c_uint64, _p)
_lib_fwd_host = _sig("pisa_attn_fwd_host", _i, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _i, _p, _z, _p)


class PisaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} ({code})")
        self.code = code


def raw_lib() -> ctypes.CDLL:
    """The loaded ctypes library (for tests of the raw C ABI)."""
    return _lib


def status_string(code: int) -> str:
    return _lib_status_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != PISA_OK:
        raise PisaError(code, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return PISA_BF16
    if t.dtype == torch.float32:
        return PISA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}: bf16 or fp32")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _qkv_shape(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("q, k, v must be [batch, heads, L, d]")
    b, h, L, d = q.shape
    return b, h, L, d


def _need_cuda(*ts):
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")


def keep_count(L: int, block: int, keep_ratio: float) -> int:
    return int(_lib_keep_count(int(L), int(block), float(keep_ratio)))


def stats_workspace_size(batch, heads, L, d, block) -> int:
    return int(_lib_stats_ws(batch, heads, L, d, block))


def fused_workspace_size(batch, heads, L, d, block) -> int:
    return int(_lib_fused_ws(batch, heads, L, d, block))


def workspace_size(batch, heads, L, d, block, k) -> int:
    return int(_lib_ws(batch, heads, L, d, block, k))


def host_workspace_size(dtype: torch.dtype, batch, heads, L, d, block, k, chunk) -> int:
    code = PISA_BF16 if dtype == torch.bfloat16 else PISA_FP32 if dtype == torch.float32 else -1
    return int(_lib_host_ws(code, batch, heads, L, d, block, k, chunk))


def _workspace(nbytes: int, device, given: Optional[torch.Tensor]):
    if given is not None:
        return given
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def block_stats(q, k, v, block, workspace=None, stream=None, out=None):
    """(qbar, kbar, vsum, hbar) float32 for [b,h,L,d] inputs (``out``: the four
    tensors, preallocated)."""
    _need_cuda(q, k, v)
    b, h, L, d = _qkv_shape(q)
    nb = -(-L // block)
    f = dict(dtype=torch.float32, device=q.device)
    if out is None:
        out = (torch.empty(b, h, nb, d, **f), torch.empty(b, h, nb, d, **f),
               torch.empty(b, h, nb, d, **f), torch.empty(b, h, d, d, **f))
    qbar, kbar, vsum, hbar = out
    ws = _workspace(stats_workspace_size(b, h, L, d, block), q.device, workspace)
    _check(_lib_block_stats(_ptr(q), _ptr(k), _ptr(v), _dtype_code(q), b, h, L, d, block,
                            _ptr(qbar), _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(ws), ws.numel(),
                            _stream(stream)), "pisa_block_stats")
    return qbar, kbar, vsum, hbar


def cov_norm(k, v, block, kbar, vsum, hbar, stream=None, out=None):
    _need_cuda(k, v, kbar, vsum, hbar)
    b, h, L, d = _qkv_shape(k)
    M = out if out is not None else torch.empty(b, h, -(-L // block), dtype=torch.float32, device=k.device)
    _check(_lib_cov_norm(_ptr(k), _ptr(v), _dtype_code(k), b, h, L, d, block, _ptr(kbar), _ptr(vsum),
                         _ptr(hbar), _ptr(M), _stream(stream)), "pisa_cov_norm")
    return M


def block_first_order(k, v, block, kbar, vsum, stream=None):
    _need_cuda(k, v, kbar, vsum)
    b, h, L, d = _qkv_shape(k)
    H = torch.empty(b, h, -(-L // block), d, d, dtype=torch.float32, device=k.device)
    _check(_lib_first_order(_ptr(k), _ptr(v), _dtype_code(k), b, h, L, d, block, _ptr(kbar),
                            _ptr(vsum), _ptr(H), _stream(stream)), "pisa_block_first_order")
    return H


def select(qbar, kbar, M, L, block, k, stream=None, out=None):
    _need_cuda(qbar, kbar, M)
    b, h, nb, d = qbar.shape
    sel = out if out is not None else torch.empty(b, h, nb, k, dtype=torch.int32, device=qbar.device)
    _check(_lib_select(_ptr(qbar), _ptr(kbar), _ptr(M), b, h, L, d, block, k, _ptr(sel),
                       _stream(stream)), "pisa_select")
    return sel


def select_route(qbar, kbar, M, L, block, k, route="covariance", stream=None, out=None):
    """Routing with a chosen score: "covariance" (pisa_select) or "pooled"
    (no covariance term; ``M`` may be None)."""
    code = {"covariance": PISA_ROUTE_COVARIANCE, "pooled": PISA_ROUTE_POOLED}[route]
    _need_cuda(qbar, kbar, *(() if M is None else (M,)))
    b, h, nb, d = qbar.shape
    sel = out if out is not None else torch.empty(b, h, nb, k, dtype=torch.int32, device=qbar.device)
    _check(_lib_select_route(_ptr(qbar), _ptr(kbar), _ptr(M), b, h, L, d, block, k, code, _ptr(sel),
                             _stream(stream)), "pisa_select_route")
    return sel


def cov_norm_spectral(H, hbar, L, block, stream=None, out=None):
    """M_j = ||H_j - Hbar||_2 (largest singular value) from the block-wise
    matrices of block_first_order."""
    _need_cuda(H, hbar)
    b, h, nb, d, _ = H.shape
    M = out if out is not None else torch.empty(b, h, nb, dtype=torch.float32, device=H.device)
    _check(_lib_cov_spectral(_ptr(H), _ptr(hbar), b, h, L, d, block, _ptr(M), _stream(stream)),
           "pisa_cov_norm_spectral")
    return M


def attn_fwd_with_sel(q, k, v, block, kbar, vsum, hbar, sel, out=None, workspace=None, stream=None):
    _need_cuda(q, k, v, kbar, vsum, hbar, sel)
    b, h, L, d = _qkv_shape(q)
    if out is None:
        out = torch.empty_like(q)
    ws = _workspace(fused_workspace_size(b, h, L, d, block), q.device, workspace)
    _check(_lib_fwd_sel(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), b, h, L, d, block,
                        _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(sel), int(sel.shape[-1]), _ptr(ws),
                        ws.numel(), _stream(stream)), "pisa_attn_fwd_with_sel")
    return out


def attn_fwd_with_sel_noalloc(q, k, v, block, kbar, vsum, hbar, sel, out=None, stream=None):
    """attn_fwd_with_sel for callers that cannot allocate device scratch: the
    library's fixed device array is used instead of a workspace.  Concurrent
    calls on different streams race on that array."""
    _need_cuda(q, k, v, kbar, vsum, hbar, sel)
    b, h, L, d = _qkv_shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(_lib_fwd_sel_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), b, h, L, d, block,
                                _ptr(kbar), _ptr(vsum), _ptr(hbar), _ptr(sel), int(sel.shape[-1]),
                                _stream(stream)), "pisa_attn_fwd_with_sel_noalloc")
    return out


def attn_fwd_blockwise_with_sel(q, k, v, block, kbar, vsum, H, sel, out=None, stream=None):
    """The forward with each unselected block's own first-order term s alpha
    (q_t H_j) instead of s beta (q_t Hbar); H from block_first_order.  CUDA
    cores, (nb - k) d^2 per row: a comparison variant for small shapes."""
    _need_cuda(q, k, v, kbar, vsum, H, sel)
    b, h, L, d = _qkv_shape(q)
    if out is None:
        out = torch.empty_like(q)
    _check(_lib_fwd_blockwise(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), b, h, L, d, block,
                              _ptr(kbar), _ptr(vsum), _ptr(H), _ptr(sel), int(sel.shape[-1]),
                              _stream(stream)), "pisa_attn_fwd_blockwise_with_sel")
    return out


def attn_fwd(q, k, v, block, keep_ratio, out=None, workspace=None, stream=None):
    """PISA forward: out [b,h,L,d] with the dtype of q."""
    _need_cuda(q, k, v)
    b, h, L, d = _qkv_shape(q)
    if out is None:
        out = torch.empty_like(q)
    kk = keep_count(L, block, keep_ratio)
    ws = _workspace(workspace_size(b, h, L, d, block, kk), q.device, workspace)
    _check(_lib_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), b, h, L, d, block,
                    float(keep_ratio), _ptr(ws), ws.numel(), _stream(stream)), "pisa_attn_fwd")
    return out


def attn_fwd_host(q, k, v, block, keep_ratio, out=None, chunk=4, workspace=None, stream=None,
                  device=None):
    """PISA forward on HOST tensors [b,h,L,d]: the library copies chunks of
    ``chunk`` (batch, head) slices in, runs the forward and copies the result
    back, overlapping copies with compute.  Pin the host tensors
    (``tensor.pin_memory()``) for the copies to overlap.  Asynchronous on
    ``stream``: synchronise it before reading ``out``.  ``workspace`` is a
    device byte tensor of at least host_workspace_size(...) bytes."""
    for t in (q, k, v):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous host tensors")
    b, h, L, d = _qkv_shape(q)
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    if out.is_cuda or not out.is_contiguous() or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("out must be a contiguous host tensor shaped and typed like q")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    kk = keep_count(L, block, keep_ratio)
    ws = _workspace(host_workspace_size(q.dtype, b, h, L, d, block, kk, chunk), dev, workspace)
    _check(_lib_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), b, h, L, d, block,
                         float(keep_ratio), int(chunk), _ptr(ws), ws.numel(), _stream(stream)),
           "pisa_attn_fwd_host")
    return out


def _tuning_dict(t: _Tuning) -> dict:
    return {"cov_blocks_per_cta": t.cov_blocks_per_cta, "select_rows_per_cta": t.select_rows_per_cta,
            "fused_ctas": t.fused_ctas}


def autotune(q, k, v, block, keep_ratio, out=None, workspace=None, stream=None) -> dict:
    """Times the result-invariant launch parameters for this shape on the
    current device, keeps the fastest and returns them (blocking).  ``out``
    receives the forward's result."""
    _need_cuda(q, k, v)
    b, h, L, d = _qkv_shape(q)
    if out is None:
        out = torch.empty_like(q)
    kk = keep_count(L, block, keep_ratio)
    ws = _workspace(workspace_size(b, h, L, d, block, kk), q.device, workspace)
    t = _Tuning()
    _check(_lib_autotune(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q), b, h, L, d, block,
                         float(keep_ratio), _ptr(ws), ws.numel(), _stream(stream), ctypes.byref(t)),
           "pisa_autotune")
    return _tuning_dict(t)


def set_tuning(batch, heads, L, d, block, cov_blocks_per_cta=0, select_rows_per_cta=0, fused_ctas=0):
    t = _Tuning(cov_blocks_per_cta, select_rows_per_cta, fused_ctas)
    _check(_lib_set_tuning(batch, heads, L, d, block, ctypes.byref(t)), "pisa_set_tuning")


def clear_tuning(batch, heads, L, d, block):
    _check(_lib_set_tuning(batch, heads, L, d, block, None), "pisa_set_tuning")


def get_tuning(batch, heads, L, d, block) -> dict:
    t = _Tuning()
    _check(_lib_get_tuning(batch, heads, L, d, block, ctypes.byref(t)), "pisa_get_tuning")
    return _tuning_dict(t)


def tuning_save(path: str):
    _check(_lib_tuning_save(os.fsencode(path)), "pisa_tuning_save")


def tuning_load(path: str):
    _check(_lib_tuning_load(os.fsencode(path)), "pisa_tuning_load")


def launches(entry: str, dtype: torch.dtype = torch.bfloat16) -> int:
    """Number of kernels an entry point launches (launch accounting)."""
    fused = 2 if dtype == torch.bfloat16 else 1  # bf16: operand prep + tensor-core kernel
    table = {"block_stats": 2, "cov_norm": 1, "select": 1, "attn_fwd_with_sel": fused}
    table["attn_fwd"] = sum(table.values())
    return table[entry]


def device_status(stream=None, reset: bool = True) -> int:
    return int(_lib_device_status(_stream(stream), 1 if reset else 0))


def set_wait_limit(limit_ns: int = 0, stream=None) -> None:
    """Limit of the tensor-core kernels' bounded waits on the current device,
    in ns (0 restores the 2 s default).  Blocking."""
    if limit_ns < 0:
        raise ValueError("limit_ns must be >= 0")
    _check(_lib_set_wait_limit(int(limit_ns), _stream(stream)), "set_wait_limit")
