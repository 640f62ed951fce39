"""CPU oracle for the host-streamed NF4 LoRA hot path (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
(``host_streamed_nf4_b200``) never imports it and never falls back to it.

The arithmetic lives in ``nf4_oracle.c`` (plain C11, fp32 data, double
accumulation); this module only compiles it with gcc and marshals numpy
arrays.  bf16 tensors travel as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

# -O2, IEEE semantics: no fast-math, no FMA contraction, no x87.
CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fno-fast-math",
          "-ffp-contract=off", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> str:
    """Compile nf4_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "nf4_oracle.h"))):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm", "-lpthread"],
                       check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct)) if a is not None else None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        f32p, u8p, u16p, i64p = (ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_uint8),
                                 ctypes.POINTER(ctypes.c_uint16), ctypes.POINTER(ctypes.c_int64))
        f64p = ctypes.POINTER(ctypes.c_double)
        i64, i32 = ctypes.c_int64, ctypes.c_int
        L.orc_nf4_codebook.argtypes = [f32p]
        L.orc_normal_quantile.argtypes = [ctypes.c_double]
        L.orc_normal_quantile.restype = ctypes.c_double
        L.orc_nf4_nearest.argtypes = [ctypes.c_float]
        L.orc_nf4_nearest.restype = i32
        L.orc_nf4_storage_bytes.argtypes = [i64, i64]
        L.orc_nf4_storage_bytes.restype = i64
        L.orc_nf4_quantize.argtypes = [u16p, i64, i64, u8p, f32p]
        L.orc_nf4_dequant.argtypes = [u8p, f32p, i64, i64, u16p]
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_lora_fwd_f64.argtypes = [f64p, f64p, f64p, f64p, i64, i64, i64, i32,
                                       ctypes.c_double, f64p, f64p]
        L.orc_lora_bwd_f64.argtypes = [f64p, f64p, f64p, f64p, f64p, i64, i64, i64, i32,
                                       ctypes.c_double, f64p, f64p, f64p]
        L.orc_lora_fwd.argtypes = [u8p, f32p, i64, i64, u16p, i64, u16p, u16p, i32,
                                   ctypes.c_float, i64p, i64, f32p, f32p, i32]
        L.orc_lora_bwd.argtypes = [u8p, f32p, i64, i64, u16p, i64, u16p, u16p, i32,
                                   ctypes.c_float, u16p, i64p, i64, f32p, f32p, f32p, i32]
        L.orc_lora_fwd_bf16w.argtypes = [u16p, i64, i64, u16p, i64, u16p, u16p, i32,
                                         ctypes.c_float, i64p, i64, f32p, f32p, i32]
        L.orc_lora_bwd_bf16w.argtypes = [u16p, i64, i64, u16p, i64, u16p, u16p, i32,
                                         ctypes.c_float, u16p, i64p, i64, f32p, f32p, f32p, i32]
        L.orc_lora_merge.argtypes = [u8p, f32p, u16p, i64, i64, u16p, u16p, i32,
                                     ctypes.c_float, u16p]
        u32p, u64 = ctypes.POINTER(ctypes.c_uint32), ctypes.c_uint64
        L.orc_philox4x32_10.argtypes = [u32p, u32p, u32p]
        L.orc_dropout_keep.argtypes = [u64, u64, ctypes.c_float, i64, i64, u8p]
        L.orc_dropout_apply.argtypes = [u16p, i64, i64, u64, u64, ctypes.c_float, u16p]
        L.orc_lora_fwd_f64m.argtypes = [f64p, f64p, f64p, f64p, f64p, i64, i64, i64, i32,
                                        ctypes.c_double, f64p, f64p]
        L.orc_lora_bwd_f64m.argtypes = [f64p, f64p, f64p, f64p, f64p, f64p, i64, i64, i64, i32,
                                        ctypes.c_double, f64p, f64p, f64p]
        L.orc_lora_fwd_drop.argtypes = [u8p, f32p, i64, i64, u16p, i64, u16p, u16p, i32,
                                        ctypes.c_float, ctypes.c_float, u64, u64, i64p, i64,
                                        f32p, f32p, i32]
        L.orc_lora_bwd_drop.argtypes = [u8p, f32p, i64, i64, u16p, i64, u16p, u16p, i32,
                                        ctypes.c_float, ctypes.c_float, u64, u64, u16p, i64p,
                                        i64, f32p, f32p, f32p, i32]
        L.orc_rmsnorm_fwd.argtypes = [f64p, f64p, i64, i64, ctypes.c_double, f64p]
        L.orc_rmsnorm_bwd.argtypes = [f64p, f64p, f64p, i64, i64, ctypes.c_double, f64p]
        L.orc_silu_mul_fwd.argtypes = [f64p, f64p, i64, f64p]
        L.orc_silu_mul_bwd.argtypes = [f64p, f64p, f64p, i64, f64p, f64p]
        L.orc_attention_fwd.argtypes = [f64p, f64p, f64p, i64, i32, i32, i32, ctypes.c_double,
                                        f64p, f64p]
        L.orc_attention_bwd.argtypes = [f64p, f64p, f64p, f64p, i64, i32, i32, i32,
                                        ctypes.c_double, f64p, f64p, f64p]
        for fn in ("orc_nf4_quantize", "orc_nf4_dequant", "orc_lora_fwd", "orc_lora_bwd",
                   "orc_lora_fwd_bf16w", "orc_lora_bwd_bf16w", "orc_lora_merge",
                   "orc_dropout_keep", "orc_dropout_apply", "orc_lora_fwd_drop",
                   "orc_lora_bwd_drop"):
            getattr(L, fn).restype = i32
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def default_threads() -> int:
    return os.cpu_count() or 1


def codebook() -> np.ndarray:
    out = np.zeros(16, np.float32)
    lib().orc_nf4_codebook(_p(out, ctypes.c_float))
    return out


def normal_quantile(p: float) -> float:
    return lib().orc_normal_quantile(float(p))


def nearest(x: float) -> int:
    return lib().orc_nf4_nearest(float(np.float32(x)))


def storage_bytes(n_out: int, k_in: int) -> int:
    return lib().orc_nf4_storage_bytes(n_out, k_in)


def f32_to_bf16(x: float) -> int:
    return lib().orc_f32_to_bf16(float(np.float32(x)))


def bf16_to_f32(h: int) -> float:
    return lib().orc_bf16_to_f32(int(h))


def quantize(w_bf16: np.ndarray):
    """w_bf16: uint16 [N, K] -> (codes uint8 [N*K/2], absmax float32 [N*K/64])."""
    w = _c(w_bf16, np.uint16)
    n, k = w.shape
    codes = np.zeros(n * k // 2, np.uint8)
    absmax = np.zeros(n * k // 64, np.float32)
    rc = lib().orc_nf4_quantize(_p(w, ctypes.c_uint16), n, k, _p(codes, ctypes.c_uint8),
                                _p(absmax, ctypes.c_float))
    if rc != 0:
        raise ValueError(f"orc_nf4_quantize rejected shape {w.shape}")
    return codes, absmax


def dequant(codes: np.ndarray, absmax: np.ndarray, n: int, k: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    absmax = _c(absmax, np.float32)
    out = np.zeros((n, k), np.uint16)
    rc = lib().orc_nf4_dequant(_p(codes, ctypes.c_uint8), _p(absmax, ctypes.c_float), n, k,
                               _p(out, ctypes.c_uint16))
    if rc != 0:
        raise ValueError(f"orc_nf4_dequant rejected shape ({n}, {k})")
    return out


def lora_fwd_f64(W, X, A, B, s):
    W, X, A, B = (_c(np.asarray(a, np.float64), np.float64) for a in (W, X, A, B))
    T, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    Y = np.zeros((T, N), np.float64)
    t = np.zeros((T, r), np.float64)
    f = ctypes.c_double
    lib().orc_lora_fwd_f64(_p(W, f), _p(X, f), _p(A, f), _p(B, f), T, N, K, r, float(s),
                           _p(Y, f), _p(t, f))
    return Y, t


def lora_bwd_f64(W, X, A, B, dY, s):
    W, X, A, B, dY = (_c(np.asarray(a, np.float64), np.float64) for a in (W, X, A, B, dY))
    T, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    dX = np.zeros((T, K), np.float64)
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    f = ctypes.c_double
    lib().orc_lora_bwd_f64(_p(W, f), _p(X, f), _p(A, f), _p(B, f), _p(dY, f), T, N, K, r,
                           float(s), _p(dX, f), _p(dA, f), _p(dB, f))
    return dX, dA, dB


def lora_fwd(codes, absmax, N, K, X, A, B, alpha, rows=None, n_threads=None):
    """Returns (Y fp32 [len(rows) or T, N], t fp32 [T, r])."""
    codes, absmax = _c(codes, np.uint8), _c(absmax, np.float32)
    X, A, B = _c(X, np.uint16), _c(A, np.uint16), _c(B, np.uint16)
    T = X.shape[0]
    r = A.shape[0]
    if rows is not None:
        rows = _c(np.asarray(rows, np.int64), np.int64)
    nr = T if rows is None else rows.shape[0]
    Y = np.zeros((nr, N), np.float32)
    t = np.zeros((T, r), np.float32)
    rc = lib().orc_lora_fwd(_p(codes, ctypes.c_uint8), _p(absmax, ctypes.c_float), N, K,
                            _p(X, ctypes.c_uint16), T, _p(A, ctypes.c_uint16),
                            _p(B, ctypes.c_uint16), r, float(alpha), _p(rows, ctypes.c_int64),
                            nr, _p(Y, ctypes.c_float), _p(t, ctypes.c_float),
                            n_threads or default_threads())
    if rc != 0:
        raise ValueError("orc_lora_fwd rejected its arguments")
    return Y, t


def lora_bwd(codes, absmax, N, K, X, A, B, dY, alpha, rows=None, n_threads=None):
    """Returns (dX fp32 [len(rows) or T, K], dA fp32 [r, K], dB fp32 [N, r])."""
    codes, absmax = _c(codes, np.uint8), _c(absmax, np.float32)
    X, A, B, dY = (_c(a, np.uint16) for a in (X, A, B, dY))
    T = X.shape[0]
    r = A.shape[0]
    if rows is not None:
        rows = _c(np.asarray(rows, np.int64), np.int64)
    nr = T if rows is None else rows.shape[0]
    dX = np.zeros((nr, K), np.float32)
    dA = np.zeros((r, K), np.float32)
    dB = np.zeros((N, r), np.float32)
    rc = lib().orc_lora_bwd(_p(codes, ctypes.c_uint8), _p(absmax, ctypes.c_float), N, K,
                            _p(X, ctypes.c_uint16), T, _p(A, ctypes.c_uint16),
                            _p(B, ctypes.c_uint16), r, float(alpha), _p(dY, ctypes.c_uint16),
                            _p(rows, ctypes.c_int64), nr, _p(dX, ctypes.c_float),
                            _p(dA, ctypes.c_float), _p(dB, ctypes.c_float),
                            n_threads or default_threads())
    if rc != 0:
        raise ValueError("orc_lora_bwd rejected its arguments")
    return dX, dA, dB


def lora_fwd_bf16w(W, X, A, B, alpha, rows=None, n_threads=None):
    """Forward with a dense bf16 base W (uint16 bits [N, K]).  Returns (Y, t) as lora_fwd."""
    W, X, A, B = (_c(a, np.uint16) for a in (W, X, A, B))
    N, K = W.shape
    T, r = X.shape[0], A.shape[0]
    if rows is not None:
        rows = _c(np.asarray(rows, np.int64), np.int64)
    nr = T if rows is None else rows.shape[0]
    Y = np.zeros((nr, N), np.float32)
    t = np.zeros((T, r), np.float32)
    u16 = ctypes.c_uint16
    rc = lib().orc_lora_fwd_bf16w(_p(W, u16), N, K, _p(X, u16), T, _p(A, u16), _p(B, u16), r,
                                  float(alpha), _p(rows, ctypes.c_int64), nr,
                                  _p(Y, ctypes.c_float), _p(t, ctypes.c_float),
                                  n_threads or default_threads())
    if rc != 0:
        raise ValueError("orc_lora_fwd_bf16w rejected its arguments")
    return Y, t


def lora_bwd_bf16w(W, X, A, B, dY, alpha, rows=None, n_threads=None):
    """Backward with a dense bf16 base W.  Returns (dX, dA, dB) as lora_bwd."""
    W, X, A, B, dY = (_c(a, np.uint16) for a in (W, X, A, B, dY))
    N, K = W.shape
    T, r = X.shape[0], A.shape[0]
    if rows is not None:
        rows = _c(np.asarray(rows, np.int64), np.int64)
    nr = T if rows is None else rows.shape[0]
    dX = np.zeros((nr, K), np.float32)
    dA = np.zeros((r, K), np.float32)
    dB = np.zeros((N, r), np.float32)
    u16, f = ctypes.c_uint16, ctypes.c_float
    rc = lib().orc_lora_bwd_bf16w(_p(W, u16), N, K, _p(X, u16), T, _p(A, u16), _p(B, u16), r,
                                  float(alpha), _p(dY, u16), _p(rows, ctypes.c_int64), nr,
                                  _p(dX, f), _p(dA, f), _p(dB, f), n_threads or default_threads())
    if rc != 0:
        raise ValueError("orc_lora_bwd_bf16w rejected its arguments")
    return dX, dA, dB


def lora_merge(A, B, alpha, codes=None, absmax=None, W=None, N=None, K=None):
    """merge_and_unload: bf16 bits [N, K] of deq(W) + (alpha/r) B A, one rounding.
    The base is NF4 (codes, absmax, N, K) or dense bf16 (W bits [N, K])."""
    A, B = _c(A, np.uint16), _c(B, np.uint16)
    r = A.shape[0]
    if W is not None:
        W = _c(W, np.uint16)
        N, K = W.shape
    else:
        codes, absmax = _c(codes, np.uint8), _c(absmax, np.float32)
    out = np.zeros((N, K), np.uint16)
    rc = lib().orc_lora_merge(_p(codes, ctypes.c_uint8), _p(absmax, ctypes.c_float),
                              _p(W, ctypes.c_uint16), N, K, _p(A, ctypes.c_uint16),
                              _p(B, ctypes.c_uint16), r, float(alpha), _p(out, ctypes.c_uint16))
    if rc != 0:
        raise ValueError("orc_lora_merge rejected its arguments")
    return out


def philox4x32_10(ctr, key):
    """Philox4x32-10 of a 4-word counter under a 2-word key -> 4 words."""
    c = np.ascontiguousarray(ctr, np.uint32)
    k = np.ascontiguousarray(key, np.uint32)
    out = np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(_p(c, ctypes.c_uint32), _p(k, ctypes.c_uint32),
                            _p(out, ctypes.c_uint32))
    return out


def dropout_keep(seed: int, offset: int, p: float, T: int, K: int) -> np.ndarray:
    keep = np.zeros((T, K), np.uint8)
    if lib().orc_dropout_keep(seed, offset, p, T, K, _p(keep, ctypes.c_uint8)) != 0:
        raise ValueError("orc_dropout_keep rejected its arguments")
    return keep


def dropout_apply(X, seed: int, offset: int, p: float) -> np.ndarray:
    X = _c(X, np.uint16)
    T, K = X.shape
    out = np.zeros((T, K), np.uint16)
    if lib().orc_dropout_apply(_p(X, ctypes.c_uint16), T, K, seed, offset, p,
                               _p(out, ctypes.c_uint16)) != 0:
        raise ValueError("orc_dropout_apply rejected its arguments")
    return out


def lora_fwd_f64m(W, X, Xl, A, B, s):
    W, X, Xl, A, B = (_c(np.asarray(a, np.float64), np.float64) for a in (W, X, Xl, A, B))
    T, K = X.shape
    N, r = W.shape[0], A.shape[0]
    Y = np.zeros((T, N), np.float64)
    t = np.zeros((T, r), np.float64)
    f = ctypes.c_double
    lib().orc_lora_fwd_f64m(_p(W, f), _p(X, f), _p(Xl, f), _p(A, f), _p(B, f), T, N, K, r,
                            float(s), _p(Y, f), _p(t, f))
    return Y, t


def lora_bwd_f64m(W, Xl, g, A, B, dY, s):
    W, Xl, A, B, dY = (_c(np.asarray(a, np.float64), np.float64) for a in (W, Xl, A, B, dY))
    g = None if g is None else _c(np.asarray(g, np.float64), np.float64)
    T, K = Xl.shape
    N, r = W.shape[0], A.shape[0]
    dX = np.zeros((T, K), np.float64)
    dA = np.zeros((r, K), np.float64)
    dB = np.zeros((N, r), np.float64)
    f = ctypes.c_double
    lib().orc_lora_bwd_f64m(_p(W, f), _p(Xl, f), _p(g, f), _p(A, f), _p(B, f), _p(dY, f), T, N,
                            K, r, float(s), _p(dX, f), _p(dA, f), _p(dB, f))
    return dX, dA, dB


def lora_fwd_drop(codes, absmax, N, K, X, A, B, alpha, p, seed, offset, rows=None,
                  n_threads=None):
    """lora_fwd with dropout p under (seed, offset) on the adapter branch."""
    codes, absmax = _c(codes, np.uint8), _c(absmax, np.float32)
    X, A, B = _c(X, np.uint16), _c(A, np.uint16), _c(B, np.uint16)
    T, r = X.shape[0], A.shape[0]
    if rows is not None:
        rows = _c(np.asarray(rows, np.int64), np.int64)
    nr = T if rows is None else rows.shape[0]
    Y = np.zeros((nr, N), np.float32)
    t = np.zeros((T, r), np.float32)
    u16 = ctypes.c_uint16
    rc = lib().orc_lora_fwd_drop(_p(codes, ctypes.c_uint8), _p(absmax, ctypes.c_float), N, K,
                                 _p(X, u16), T, _p(A, u16), _p(B, u16), r, float(alpha),
                                 float(p), seed, offset, _p(rows, ctypes.c_int64), nr,
                                 _p(Y, ctypes.c_float), _p(t, ctypes.c_float),
                                 n_threads or default_threads())
    if rc != 0:
        raise ValueError("orc_lora_fwd_drop rejected its arguments")
    return Y, t


def lora_bwd_drop(codes, absmax, N, K, X, A, B, dY, alpha, p, seed, offset, rows=None,
                  n_threads=None):
    """lora_bwd with dropout p under (seed, offset) on the adapter branch."""
    codes, absmax = _c(codes, np.uint8), _c(absmax, np.float32)
    X, A, B, dY = (_c(a, np.uint16) for a in (X, A, B, dY))
    T, r = X.shape[0], A.shape[0]
    if rows is not None:
        rows = _c(np.asarray(rows, np.int64), np.int64)
    nr = T if rows is None else rows.shape[0]
    dX = np.zeros((nr, K), np.float32)
    dA = np.zeros((r, K), np.float32)
    dB = np.zeros((N, r), np.float32)
    u16, f = ctypes.c_uint16, ctypes.c_float
    rc = lib().orc_lora_bwd_drop(_p(codes, ctypes.c_uint8), _p(absmax, f), N, K, _p(X, u16), T,
                                 _p(A, u16), _p(B, u16), r, float(alpha), float(p), seed, offset,
                                 _p(dY, u16), _p(rows, ctypes.c_int64), nr, _p(dX, f), _p(dA, f),
                                 _p(dB, f), n_threads or default_threads())
    if rc != 0:
        raise ValueError("orc_lora_bwd_drop rejected its arguments")
    return dX, dA, dB


# ---------------------------------------------------------------- decoder glue

def _d(a):
    return _c(np.asarray(a, np.float64), np.float64)


def rmsnorm_fwd(x, g, eps):
    x, g = _d(x), _d(g)
    T, n = x.shape
    y = np.zeros_like(x)
    f = ctypes.c_double
    lib().orc_rmsnorm_fwd(_p(x, f), _p(g, f), T, n, float(eps), _p(y, f))
    return y


def rmsnorm_bwd(x, g, dy, eps):
    x, g, dy = _d(x), _d(g), _d(dy)
    T, n = x.shape
    dx = np.zeros_like(x)
    f = ctypes.c_double
    lib().orc_rmsnorm_bwd(_p(x, f), _p(g, f), _p(dy, f), T, n, float(eps), _p(dx, f))
    return dx


def silu_mul_fwd(a, b):
    a, b = _d(a), _d(b)
    m = np.zeros_like(a)
    f = ctypes.c_double
    lib().orc_silu_mul_fwd(_p(a, f), _p(b, f), a.size, _p(m, f))
    return m


def silu_mul_bwd(a, b, dm):
    a, b, dm = _d(a), _d(b), _d(dm)
    da, db = np.zeros_like(a), np.zeros_like(a)
    f = ctypes.c_double
    lib().orc_silu_mul_bwd(_p(a, f), _p(b, f), _p(dm, f), a.size, _p(da, f), _p(db, f))
    return da, db


def attention_fwd(q, k, v, H, KV, d, scale):
    q, k, v = _d(q), _d(k), _d(v)
    T = q.shape[0]
    o = np.zeros_like(q)
    lse = np.zeros((H, T), np.float64)
    f = ctypes.c_double
    lib().orc_attention_fwd(_p(q, f), _p(k, f), _p(v, f), T, H, KV, d, float(scale), _p(o, f),
                            _p(lse, f))
    return o, lse


def attention_bwd(q, k, v, do, H, KV, d, scale):
    q, k, v, do = _d(q), _d(k), _d(v), _d(do)
    T = q.shape[0]
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    f = ctypes.c_double
    lib().orc_attention_bwd(_p(q, f), _p(k, f), _p(v, f), _p(do, f), T, H, KV, d, float(scale),
                            _p(dq, f), _p(dk, f), _p(dv, f))
    return dq, dk, dv
