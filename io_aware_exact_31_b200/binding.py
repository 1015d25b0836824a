"""ctypes binding of libfa_sm100.so (argument marshalling only).

PyTorch supplies device memory and the current stream; every step of the
attention path runs in the library's CUDA kernels.  There is no fallback: if
the library is missing or the device is not sm_100, calls raise ``FaError``.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_sm100.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(5)

# Every entry point include/fa.h declares.
EXPORTS = ("fa_forward", "fa_forward_gqa", "fa_forward_varlen", "fa_forward_dropout",
           "fa_forward_fp8", "fa_backward_workspace_bytes",
           "fa_backward", "fa_backward_gqa", "fa_backward_varlen", "fa_backward_dropout",
           "fa_backward_deterministic", "fa_backward_noalloc",
           "fa_check_device_error", "fa_selftest_bounded_wait", "fa_status_str", "fa_version")

# Size of the library's built-in workspace used by fa_backward_noalloc.
NOALLOC_MAX_SCRATCH_BYTES = 64 * 1024 * 1024

_lib = None


class FaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} (status {status})")


def load_library(path: str | None = None):
    """Open the C-ABI library (once).  Raises FaError if it was not built."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise FaError(FA_ERR_UNSUPPORTED,
                      f"{p} not found; build it with `python -m io_aware_exact_31_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_forward.restype = i
    lib.fa_backward_workspace_bytes.argtypes = [i, i, i, i]
    lib.fa_backward_workspace_bytes.restype = sz
    lib.fa_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
    lib.fa_backward.restype = i
    lib.fa_forward_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.fa_forward_gqa.restype = i
    lib.fa_backward_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f,
                                    i, vp]
    lib.fa_backward_gqa.restype = i
    lib.fa_forward_varlen.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    lib.fa_forward_varlen.restype = i
    lib.fa_backward_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, i, i, i, i,
                                       i, f, i, vp]
    lib.fa_backward_varlen.restype = i
    u64, u32 = ctypes.c_ulonglong, ctypes.c_uint
    lib.fa_forward_dropout.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, f, u64, u32,
                                       vp]
    lib.fa_forward_dropout.restype = i
    lib.fa_backward_dropout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp, i, i, i, i,
                                        i, f, i, f, u64, u32, vp]
    lib.fa_backward_dropout.restype = i
    lib.fa_backward_deterministic.argtypes = list(lib.fa_backward_dropout.argtypes)
    lib.fa_backward_deterministic.restype = i
    lib.fa_forward_fp8.argtypes = [vp, vp, vp, vp, vp, f, f, f, i, i, i, i, i, f, i, vp]
    lib.fa_forward_fp8.restype = i
    lib.fa_backward_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_backward_noalloc.restype = i
    lib.fa_check_device_error.argtypes = [vp, ctypes.POINTER(ctypes.c_uint)]
    lib.fa_check_device_error.restype = i
    lib.fa_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, vp]
    lib.fa_selftest_bounded_wait.restype = i
    lib.fa_status_str.argtypes = [i]
    lib.fa_status_str.restype = ctypes.c_char_p
    lib.fa_version.restype = i
    if path is None:
        _lib = lib
    return lib


def status_str(status: int) -> str:
    try:
        return load_library().fa_status_str(status).decode()
    except FaError:
        return "library not loaded"


def _stream_handle(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check_qkv(*ts):
    shape = ts[0].shape
    for t in ts:
        if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("tensors must be contiguous bf16 CUDA tensors [B, H, N, d]")
        if t.shape != shape or t.dim() != 4:
            raise ValueError(f"shape mismatch: {tuple(t.shape)} vs {tuple(shape)}")
    return shape


def _check_kv_heads(q, k, v):
    """(B, H, N, d, H_kv): K and V may have H_kv heads dividing H (grouped-query)."""
    B, H, N, d = _check_qkv(q)
    _check_qkv(k, v)
    if k.shape[0] != B or k.shape[2] != N or k.shape[3] != d or H % k.shape[1] != 0:
        raise ValueError(f"K/V shape {tuple(k.shape)} incompatible with Q {tuple(q.shape)}")
    return B, H, N, d, k.shape[1]


def forward_raw(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d, scale, causal, stream=0) -> int:
    """fa_forward on raw device addresses; returns the status code."""
    return load_library().fa_forward(q_ptr, k_ptr, v_ptr, o_ptr, lse_ptr, B, H, N, d,
                                     float(scale), int(bool(causal)), ctypes.c_void_p(stream))


def backward_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(load_library().fa_backward_workspace_bytes(B, H, N, d))


def _seqlens_ptr(seqlens, B, device):
    if seqlens is None:
        return None, None
    t = seqlens.to(device=device, dtype=torch.int32).contiguous()
    if t.shape != (B,):
        raise ValueError("seqlens must have shape [B]")
    return t, t.data_ptr()


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
            scale: float | None = None, out: torch.Tensor | None = None,
            lse: torch.Tensor | None = None, stream=None, seqlens: torch.Tensor | None = None,
            dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """O, LSE = softmax(scale Q K^T [+causal]) V and its per-row logsumexp.
    K and V may have fewer heads than Q (grouped-/multi-query attention);
    seqlens [B] marks tokens >= seqlens[b] of batch b as padding; dropout_p > 0
    applies attention dropout with the Philox keep mask of (seed, offset)."""
    B, H, N, d, Hkv = _check_kv_heads(q, k, v)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    _check_qkv(q, o)
    if l.dtype != torch.float32 or not l.is_contiguous() or tuple(l.shape) != (B, H, N):
        raise ValueError("lse must be a contiguous float32 tensor [B, H, N]")
    keep, sl = _seqlens_ptr(seqlens, B, q.device)
    lib = load_library()
    if dropout_p:
        st = lib.fa_forward_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                    l.data_ptr(), sl, B, H, Hkv, N, d, scale, int(bool(causal)),
                                    float(dropout_p), int(seed), int(offset),
                                    _stream_handle(stream))
    else:
        st = lib.fa_forward_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   l.data_ptr(), sl, B, H, Hkv, N, d, scale, int(bool(causal)),
                                   _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_forward")
    return o, l


def forward_fp8(q8, k8, v8, descale_q: float, descale_k: float, descale_v: float,
                causal: bool = False, scale: float | None = None, out=None, lse=None,
                stream=None):
    """FP8 forward: q8/k8/v8 are torch.float8_e4m3fn [B,H,N,128] ([B,H_kv,N,128]
    for K/V); the real inputs are q8 * descale_q etc.  Returns bf16 O and LSE."""
    for t in (q8, k8, v8):
        if not t.is_cuda or t.dtype != torch.float8_e4m3fn or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("inputs must be contiguous float8_e4m3fn CUDA tensors [B, H, N, d]")
    B, H, N, d = q8.shape
    Hkv = k8.shape[1]
    if k8.shape != v8.shape or k8.shape[0] != B or k8.shape[2:] != q8.shape[2:]:
        raise ValueError("K/V shape incompatible with Q")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    o = torch.empty(q8.shape, device=q8.device, dtype=torch.bfloat16) if out is None else out
    l = torch.empty((B, H, N), device=q8.device, dtype=torch.float32) if lse is None else lse
    st = load_library().fa_forward_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), o.data_ptr(),
                                       l.data_ptr(), float(descale_q), float(descale_k),
                                       float(descale_v), B, H, Hkv, N, d, scale, int(bool(causal)),
                                       _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_forward_fp8")
    return o, l


def backward(q, k, v, o, do, lse, causal: bool = False, scale: float | None = None,
             dq=None, dk=None, dv=None, workspace: torch.Tensor | None = None, stream=None,
             seqlens: torch.Tensor | None = None, dropout_p: float = 0.0, seed: int = 0,
             offset: int = 0, deterministic: bool = False):
    """dQ, dK, dV of <O, dO> (scores recomputed from the saved LSE).  With K/V
    of fewer heads, dK/dV are summed over each group of query heads.  The
    dropout arguments must be those of the forward call.  deterministic=True
    adds the key blocks' dQ parts in a fixed order (fa_backward_deterministic),
    so that dQ is bitwise reproducible from run to run."""
    B, H, N, d, Hkv = _check_kv_heads(q, k, v)
    _check_qkv(q, o, do)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    lib = load_library()
    ws_bytes = int(lib.fa_backward_workspace_bytes(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    keep, sl = _seqlens_ptr(seqlens, B, q.device)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), sl, B, H, Hkv, N, d, scale,
            int(bool(causal)))
    if deterministic:
        st = lib.fa_backward_deterministic(*args, float(dropout_p), int(seed), int(offset),
                                           _stream_handle(stream))
    elif dropout_p:
        st = lib.fa_backward_dropout(*args, float(dropout_p), int(seed), int(offset),
                                     _stream_handle(stream))
    else:
        st = lib.fa_backward_varlen(*args, _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_backward")
    return dq, dk, dv


def check_device_error(stream=None) -> tuple[int, int]:
    """Synchronise and read/clear the device error word: (status, raw site code)."""
    site = ctypes.c_uint(0)
    st = load_library().fa_check_device_error(_stream_handle(stream), ctypes.byref(site))
    return st, site.value


def selftest_bounded_wait(timeout_ns: int = 20_000_000, stream=None) -> tuple[int, int]:
    """Run the bounded-wait self-test and return check_device_error()'s result."""
    st = load_library().fa_selftest_bounded_wait(int(timeout_ns), _stream_handle(stream))
    if st != FA_OK:
        raise FaError(st, "fa_selftest_bounded_wait")
    return check_device_error(stream)


class _Attention(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, causal, scale, dropout_p, seed, offset):
        o, lse = forward(q, k, v, causal=causal, scale=scale, dropout_p=dropout_p, seed=seed,
                         offset=offset)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.causal, ctx.scale = causal, scale
        ctx.dropout = (dropout_p, seed, offset)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        p, seed, offset = ctx.dropout
        dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, causal=ctx.causal,
                              scale=ctx.scale, dropout_p=p, seed=seed, offset=offset)
        return dq, dk, dv, None, None, None, None, None


def attention(q, k, v, causal: bool = False, scale: float | None = None, dropout_p: float = 0.0,
              seed: int | None = None, offset: int = 0):
    """Differentiable exact attention (autograd wrapper over forward/backward).
    With dropout_p > 0 and no seed, a seed is drawn from torch's default CPU
    generator, so torch.manual_seed makes the mask reproducible; the backward
    regenerates the same mask."""
    if dropout_p and seed is None:
        seed = int(torch.randint(0, 2 ** 62, (1,)).item())
    return _Attention.apply(q, k, v, causal, scale, float(dropout_p), int(seed or 0), int(offset))
