"""fp64 CPU oracle for exact scaled-dot-product attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares no code with it.  The arithmetic lives in ``attn_oracle.c`` (plain C,
IEEE double); this module only builds it with gcc and marshals numpy arrays.

What each function computes, and the passage it follows, is stated in the C
file.  Pins (tests that tie the oracle to the pages and to mathematics rather
than to itself) are in ``tests/test_oracle.py``.  Parity status of every
function: pinned (closed forms, invariants, brute force, library special
cases, finite differences).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F64 = 0
BF16 = 1

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build())
    i64, dbl, vp, ip = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
    lib.oracle_attention_forward.argtypes = [vp, vp, vp, ip, i64, i64, i64, i64, dbl, ip, vp, vp]
    lib.oracle_attention_forward_rows.argtypes = [vp, vp, vp, ip, i64, i64, i64, i64, dbl, ip,
                                                  vp, i64, vp, vp]
    lib.oracle_attention_backward.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, dbl, ip,
                                              vp, vp, vp]
    lib.oracle_attention_forward_gqa.argtypes = [vp, vp, vp, ip, i64, i64, i64, i64, i64, dbl, ip,
                                                 vp, vp]
    lib.oracle_attention_backward_gqa.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, i64, dbl,
                                                  ip, vp, vp, vp]
    lib.oracle_attention_forward_varlen.argtypes = [vp, vp, vp, ip, vp, i64, i64, i64, i64, i64,
                                                    dbl, ip, vp, vp]
    lib.oracle_attention_backward_varlen.argtypes = [vp, vp, vp, vp, ip, vp, i64, i64, i64, i64,
                                                     i64, dbl, ip, vp, vp, vp]
    u64, u32 = ctypes.c_uint64, ctypes.c_uint32
    lib.oracle_attention_forward_dropout.argtypes = [vp, vp, vp, ip, vp, i64, i64, i64, i64, i64,
                                                     dbl, ip, dbl, u64, u32, vp, vp]
    lib.oracle_attention_backward_dropout.argtypes = [vp, vp, vp, vp, ip, vp, i64, i64, i64, i64,
                                                      i64, dbl, ip, dbl, u64, u32, vp, vp, vp]
    lib.oracle_attention_forward_dropout_rows.argtypes = [vp, vp, vp, ip, i64, i64, i64, i64, i64,
                                                          dbl, ip, dbl, u64, u32, vp, i64, vp, vp]
    lib.oracle_attention_backward_dropout_heads.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64,
                                                            i64, dbl, ip, dbl, u64, u32, vp, i64,
                                                            vp, vp, vp]
    lib.oracle_philox4x32_10.argtypes = [vp, vp, vp]
    lib.oracle_philox4x32_10.restype = None
    lib.oracle_philox4x32_7.argtypes = [vp, vp, vp]
    lib.oracle_philox4x32_7.restype = None
    lib.oracle_dropout_keep_mask.argtypes = [i64, i64, i64, dbl, u64, u32, vp]
    lib.oracle_softmax_partial.argtypes = [vp, i64, vp, i64, vp, vp, vp]
    lib.oracle_softmax_merge.argtypes = [dbl, dbl, vp, dbl, dbl, vp, i64, vp, vp, vp]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_set_num_threads.argtypes = [ip]
    for name in ("oracle_attention_forward", "oracle_attention_forward_rows",
                 "oracle_attention_backward", "oracle_softmax_partial",
                 "oracle_softmax_merge", "oracle_attention_forward_gqa",
                 "oracle_attention_backward_gqa", "oracle_attention_forward_varlen",
                 "oracle_attention_backward_varlen", "oracle_attention_forward_dropout",
                 "oracle_attention_backward_dropout", "oracle_dropout_keep_mask",
                 "oracle_attention_forward_dropout_rows",
                 "oracle_attention_backward_dropout_heads"):
        getattr(lib, name).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _as_input(x):
    """Return (contiguous array, dtype code).  bf16 arrives as uint16 bits."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float64:
        return x, F64
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle inputs must be float64 or bf16 bits (uint16), got {x.dtype}")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what} failed with code {rc}")


def attention_forward(Q, K, V, scale: float, causal: bool, lib=None):
    """O [B,H,N,d] and LSE [B,H,N] (float64) of softmax(Q K^T scale [+causal]) V."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv) = _as_input(Q), _as_input(K), _as_input(V)
    assert dt == dk == dv and Q.shape == K.shape == V.shape and Q.ndim == 4
    B, H, N, d = Q.shape
    O = np.empty((B, H, N, d), np.float64)
    LSE = np.empty((B, H, N), np.float64)
    _check(lib.oracle_attention_forward(_ptr(Q), _ptr(K), _ptr(V), dt, B, H, N, d,
                                        float(scale), int(bool(causal)), _ptr(O), _ptr(LSE)),
           "oracle_attention_forward")
    return O, LSE


def attention_forward_rows(Q, K, V, scale: float, causal: bool, rows, lib=None):
    """Rows of the forward: rows[k] = bh*N + i.  Returns O_rows [n,d], LSE_rows [n]."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv) = _as_input(Q), _as_input(K), _as_input(V)
    assert dt == dk == dv and Q.shape == K.shape == V.shape and Q.ndim == 4
    B, H, N, d = Q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.empty((rows.size, d), np.float64)
    LSE = np.empty((rows.size,), np.float64)
    _check(lib.oracle_attention_forward_rows(_ptr(Q), _ptr(K), _ptr(V), dt, B, H, N, d,
                                             float(scale), int(bool(causal)), _ptr(rows),
                                             rows.size, _ptr(O), _ptr(LSE)),
           "oracle_attention_forward_rows")
    return O, LSE


def attention_backward(Q, K, V, dO, scale: float, causal: bool, lib=None):
    """dQ, dK, dV [B,H,N,d] (float64): exact gradient of <O, dO>."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv), (dO, dd) = (_as_input(Q), _as_input(K), _as_input(V),
                                           _as_input(dO))
    assert dt == dk == dv == dd and Q.shape == K.shape == V.shape == dO.shape
    B, H, N, d = Q.shape
    dQ = np.empty((B, H, N, d), np.float64)
    dK = np.empty_like(dQ)
    dV = np.empty_like(dQ)
    _check(lib.oracle_attention_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), dt, B, H, N, d,
                                         float(scale), int(bool(causal)),
                                         _ptr(dQ), _ptr(dK), _ptr(dV)),
           "oracle_attention_backward")
    return dQ, dK, dV


def attention_forward_gqa(Q, K, V, scale: float, causal: bool, lib=None):
    """Grouped-query forward: Q [B,H,N,d], K/V [B,Hkv,N,d] -> O [B,H,N,d], LSE [B,H,N]."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv) = _as_input(Q), _as_input(K), _as_input(V)
    assert dt == dk == dv and K.shape == V.shape and Q.ndim == 4
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    O = np.empty((B, H, N, d), np.float64)
    LSE = np.empty((B, H, N), np.float64)
    _check(lib.oracle_attention_forward_gqa(_ptr(Q), _ptr(K), _ptr(V), dt, B, H, Hkv, N, d,
                                            float(scale), int(bool(causal)), _ptr(O), _ptr(LSE)),
           "oracle_attention_forward_gqa")
    return O, LSE


def attention_backward_gqa(Q, K, V, dO, scale: float, causal: bool, lib=None):
    """Grouped-query backward: dQ [B,H,N,d]; dK, dV [B,Hkv,N,d] (sums over each group)."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv), (dO, dd) = (_as_input(Q), _as_input(K), _as_input(V),
                                           _as_input(dO))
    assert dt == dk == dv == dd and K.shape == V.shape and Q.shape == dO.shape
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    dQ = np.empty((B, H, N, d), np.float64)
    dK = np.empty((B, Hkv, N, d), np.float64)
    dV = np.empty_like(dK)
    _check(lib.oracle_attention_backward_gqa(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), dt, B, H, Hkv,
                                             N, d, float(scale), int(bool(causal)),
                                             _ptr(dQ), _ptr(dK), _ptr(dV)),
           "oracle_attention_backward_gqa")
    return dQ, dK, dV


def attention_forward_varlen(Q, K, V, seqlens, scale: float, causal: bool, lib=None):
    """Padded batches: seqlens[b] real tokens per batch (keys beyond masked,
    padding query rows O = 0, LSE = 0).  K/V may have fewer heads (grouped)."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv) = _as_input(Q), _as_input(K), _as_input(V)
    assert dt == dk == dv and K.shape == V.shape and Q.ndim == 4
    B, H, N, d = Q.shape
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    assert sl.shape == (B,)
    O = np.empty((B, H, N, d), np.float64)
    LSE = np.empty((B, H, N), np.float64)
    _check(lib.oracle_attention_forward_varlen(_ptr(Q), _ptr(K), _ptr(V), dt, _ptr(sl), B, H,
                                               K.shape[1], N, d, float(scale), int(bool(causal)),
                                               _ptr(O), _ptr(LSE)),
           "oracle_attention_forward_varlen")
    return O, LSE


def attention_backward_varlen(Q, K, V, dO, seqlens, scale: float, causal: bool, lib=None):
    """Gradients for padded batches (all gradients of padding tokens are 0)."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv), (dO, dd) = (_as_input(Q), _as_input(K), _as_input(V),
                                           _as_input(dO))
    assert dt == dk == dv == dd and K.shape == V.shape and Q.shape == dO.shape
    B, H, N, d = Q.shape
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    assert sl.shape == (B,)
    dQ = np.empty((B, H, N, d), np.float64)
    dK = np.empty(K.shape, np.float64)
    dV = np.empty(K.shape, np.float64)
    _check(lib.oracle_attention_backward_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), dt, _ptr(sl),
                                                B, H, K.shape[1], N, d, float(scale),
                                                int(bool(causal)), _ptr(dQ), _ptr(dK), _ptr(dV)),
           "oracle_attention_backward_varlen")
    return dQ, dK, dV


def _seqlens_arg(seqlens, B):
    if seqlens is None:
        return None, None
    sl = np.ascontiguousarray(seqlens, dtype=np.int32)
    assert sl.shape == (B,)
    return sl, _ptr(sl)


def attention_forward_dropout(Q, K, V, scale: float, causal: bool, p_drop: float, seed: int,
                              offset: int = 0, seqlens=None, lib=None):
    """Forward with attention dropout (Philox-4x32-10 keep mask; see the C
    file).  K/V may have fewer heads; seqlens optional.  p_drop = 0 is the
    plain forward."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv) = _as_input(Q), _as_input(K), _as_input(V)
    assert dt == dk == dv and K.shape == V.shape and Q.ndim == 4
    B, H, N, d = Q.shape
    sl, slp = _seqlens_arg(seqlens, B)
    O = np.empty((B, H, N, d), np.float64)
    LSE = np.empty((B, H, N), np.float64)
    _check(lib.oracle_attention_forward_dropout(_ptr(Q), _ptr(K), _ptr(V), dt, slp, B, H,
                                                K.shape[1], N, d, float(scale), int(bool(causal)),
                                                float(p_drop), int(seed), int(offset),
                                                _ptr(O), _ptr(LSE)),
           "oracle_attention_forward_dropout")
    return O, LSE


def attention_backward_dropout(Q, K, V, dO, scale: float, causal: bool, p_drop: float, seed: int,
                               offset: int = 0, seqlens=None, lib=None):
    """Exact gradient of the dropout forward for the same (p_drop, seed, offset)."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv), (dO, dd) = (_as_input(Q), _as_input(K), _as_input(V),
                                           _as_input(dO))
    assert dt == dk == dv == dd and K.shape == V.shape and Q.shape == dO.shape
    B, H, N, d = Q.shape
    sl, slp = _seqlens_arg(seqlens, B)
    dQ = np.empty((B, H, N, d), np.float64)
    dK = np.empty(K.shape, np.float64)
    dV = np.empty(K.shape, np.float64)
    _check(lib.oracle_attention_backward_dropout(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), dt, slp, B,
                                                 H, K.shape[1], N, d, float(scale),
                                                 int(bool(causal)), float(p_drop), int(seed),
                                                 int(offset), _ptr(dQ), _ptr(dK), _ptr(dV)),
           "oracle_attention_backward_dropout")
    return dQ, dK, dV


def attention_forward_dropout_rows(Q, K, V, scale: float, causal: bool, p_drop: float, seed: int,
                                   offset: int, rows, lib=None):
    """Sampled rows (rows[k] = bh*N + i) of attention_forward_dropout (no padding;
    K/V may have fewer heads).  p_drop = 0: plain attention."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv) = _as_input(Q), _as_input(K), _as_input(V)
    assert dt == dk == dv and K.shape == V.shape and Q.ndim == 4
    B, H, N, d = Q.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    O = np.empty((rows.size, d), np.float64)
    LSE = np.empty((rows.size,), np.float64)
    _check(lib.oracle_attention_forward_dropout_rows(_ptr(Q), _ptr(K), _ptr(V), dt, B, H,
                                                     K.shape[1], N, d, float(scale),
                                                     int(bool(causal)), float(p_drop), int(seed),
                                                     int(offset), _ptr(rows), rows.size, _ptr(O),
                                                     _ptr(LSE)),
           "oracle_attention_forward_dropout_rows")
    return O, LSE


def attention_backward_dropout_heads(Q, K, V, dO, scale: float, causal: bool, p_drop: float,
                                     seed: int, offset: int, heads, lib=None):
    """attention_backward_dropout restricted to the listed (distinct) query heads
    bh = b*H + h; other heads' gradients are 0."""
    lib = lib or load()
    (Q, dt), (K, dk), (V, dv), (dO, dd) = (_as_input(Q), _as_input(K), _as_input(V),
                                           _as_input(dO))
    assert dt == dk == dv == dd and K.shape == V.shape and Q.shape == dO.shape
    B, H, N, d = Q.shape
    hs = np.ascontiguousarray(heads, dtype=np.int64)
    dQ = np.empty((B, H, N, d), np.float64)
    dK = np.empty(K.shape, np.float64)
    dV = np.empty(K.shape, np.float64)
    _check(lib.oracle_attention_backward_dropout_heads(_ptr(Q), _ptr(K), _ptr(V), _ptr(dO), dt, B,
                                                       H, K.shape[1], N, d, float(scale),
                                                       int(bool(causal)), float(p_drop),
                                                       int(seed), int(offset), _ptr(hs), hs.size,
                                                       _ptr(dQ), _ptr(dK), _ptr(dV)),
           "oracle_attention_backward_dropout_heads")
    return dQ, dK, dV


def _philox(fn, counter, key):
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    assert c.shape == (4,) and k.shape == (2,)
    out = np.empty(4, np.uint32)
    fn(_ptr(c), _ptr(k), _ptr(out))
    return out


def philox4x32_10(counter, key, lib=None):
    """The four 32-bit output words of Philox-4x32-10 for a 4-word counter and 2-word key."""
    return _philox((lib or load()).oracle_philox4x32_10, counter, key)


def philox4x32_7(counter, key, lib=None):
    """Philox-4x32 with 7 rounds (the dropout generator)."""
    return _philox((lib or load()).oracle_philox4x32_7, counter, key)


def dropout_keep_mask(B: int, H: int, N: int, p_drop: float, seed: int, offset: int = 0,
                      lib=None):
    """Keep mask z [B,H,N,N] (bool; row = query, column = key) of the dropout forward."""
    lib = lib or load()
    m = np.empty((B, H, N, N), np.uint8)
    _check(lib.oracle_dropout_keep_mask(B, H, N, float(p_drop), int(seed), int(offset), _ptr(m)),
           "oracle_dropout_keep_mask")
    return m.astype(bool)


def softmax_partial(s, Vblk, lib=None):
    """(m, l, o) of one block of scores s [n] with value rows Vblk [n, d]."""
    lib = lib or load()
    s = np.ascontiguousarray(s, np.float64)
    Vblk = np.ascontiguousarray(Vblk, np.float64)
    d = Vblk.shape[1]
    m, l = ctypes.c_double(), ctypes.c_double()
    o = np.empty((d,), np.float64)
    _check(lib.oracle_softmax_partial(_ptr(s), s.size, _ptr(Vblk), d, ctypes.byref(m),
                                      ctypes.byref(l), _ptr(o)), "oracle_softmax_partial")
    return m.value, l.value, o


def softmax_merge(part_x, part_y, lib=None):
    """Merge two (m, l, o) partials into the partial of the union of both blocks."""
    lib = lib or load()
    (mx, lx, ox), (my, ly, oy) = part_x, part_y
    ox = np.ascontiguousarray(ox, np.float64)
    oy = np.ascontiguousarray(oy, np.float64)
    m, l = ctypes.c_double(), ctypes.c_double()
    o = np.empty_like(ox)
    _check(lib.oracle_softmax_merge(mx, lx, _ptr(ox), my, ly, _ptr(oy), ox.size,
                                    ctypes.byref(m), ctypes.byref(l), _ptr(o)),
           "oracle_softmax_merge")
    return m.value, l.value, o


def num_threads(lib=None) -> int:
    return (lib or load()).oracle_num_threads()


def set_num_threads(n: int, lib=None) -> None:
    (lib or load()).oracle_set_num_threads(int(n))
