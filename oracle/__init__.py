"""CPU oracle for the online INT8 W8A8 linear / routed-MoE hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py`` may import this package.
The product (``moe_gemm_absmax_b200``) never imports it, and this package
never imports the product: the two share no code.

The arithmetic lives in ``w8a8_oracle.c`` (plain scalar C, fp32 with one
IEEE round-to-nearest step per operator, fp contraction off).  This module
compiles it with gcc on first use and wraps each function with ctypes over
numpy arrays.  bf16 values travel as ``np.uint16`` bit patterns.

Parity pins: every function here is checked in ``tests/test_oracle_*.py``
against closed forms, invariants, library routines or brute force; the
only bits left unpinned are the last fp32 rounding steps of the dequant
epilogues, which the tests bound by one bf16 ulp.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w8a8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_w8a8.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            L = _lib
            vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
            L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_f32.restype = ctypes.c_float
            L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
            L.oracle_f32_to_bf16.restype = ctypes.c_uint16
            L.oracle_quant_row_f32.argtypes = [vp, i64, vp, vp]
            L.oracle_quant_rows_bf16.argtypes = [vp, i64, i64, i64, vp, vp]
            L.oracle_quant_rows_f32.argtypes = [vp, i64, i64, vp, vp]
            L.oracle_gemm_s32.argtypes = [vp, vp, i64, i64, i64, vp]
            L.oracle_gemm_s32.restype = i64
            L.oracle_gemm_s32_at.argtypes = [vp, vp, i64, vp, vp, i64, vp]
            L.oracle_dequant.argtypes = [vp, vp, vp, i64, i64, vp, vp, vp]
            L.oracle_linear.argtypes = [vp, vp, vp, i64, i64, i64, vp, vp, vp, vp]
            L.oracle_exp_proj.argtypes = [ctypes.c_float]
            L.oracle_exp_proj.restype = ctypes.c_float
            L.oracle_silu.argtypes = [ctypes.c_float]
            L.oracle_silu.restype = ctypes.c_float
            L.oracle_exp_proj_array.argtypes = [vp, vp, i64]
            L.oracle_silu_array.argtypes = [vp, vp, i64]
            L.oracle_f32_to_bf16_array.argtypes = [vp, vp, i64]
            L.oracle_route.argtypes = [vp, i64, i32, i32, vp, vp]
            L.oracle_moe_histogram.argtypes = [vp, i64, i32, vp]
            L.oracle_moe_forward.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32,
                                             vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.oracle_mlp_forward.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp, vp, vp]
            L.oracle_fwht128.argtypes = [vp]
            L.oracle_fwht128_quant.argtypes = [vp, i64, i64, vp, vp, vp]
            L.oracle_gemm_g128.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
            L.oracle_fwht128_quant_f32.argtypes = [vp, i64, i64, vp, vp]
            L.oracle_group128_quant.argtypes = [vp, i64, i64, vp, vp]
            L.oracle_trunk_weight_quant.argtypes = [vp, i64, i64, vp, vp, vp]
            L.oracle_gemm_trunk.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, vp, vp]
            L.oracle_shared_expert_forward.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32,
                                                       vp, vp, vp, vp, vp, vp]
            L.oracle_gemm_group128.argtypes = [vp, vp, vp, vp, i64, i64, i64, vp, vp]
            L.oracle_moe_g128_forward.argtypes = [vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32,
                                                  vp, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            L.oracle_set_threads.argtypes = [i32]
            L.oracle_get_threads.restype = i32
        return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


# ---------------------------------------------------------------- bf16

def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (upper half of binary32)."""
    h = np.asarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (scalar C loop)."""
    f = np.ascontiguousarray(f, dtype=np.float32)
    out = np.empty(f.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_array(_p(f), _p(out), f.size)
    return out


# ---------------------------------------------------------------- quant

def quant_row_f32(v: np.ndarray):
    v = _c(v, np.float32)
    q = np.empty(v.shape[-1], dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    lib().oracle_quant_row_f32(_p(v), v.shape[-1], _p(q), _p(s))
    return q, np.float32(s[0])


def quant_rows_bf16(x_bits: np.ndarray):
    """a1: per-token absmax quant of bf16 rows [M, K] -> (int8 [M,K], fp32 [M])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.int8)
    s = np.empty(M, dtype=np.float32)
    lib().oracle_quant_rows_bf16(_p(x), M, K, K, _p(q), _p(s))
    return q, s


def quant_rows_f32(w: np.ndarray):
    """a0: per-output-channel absmax quant of fp32 rows [N, K]."""
    w = _c(w, np.float32)
    N, K = w.shape
    q = np.empty((N, K), dtype=np.int8)
    s = np.empty(N, dtype=np.float32)
    lib().oracle_quant_rows_f32(_p(w), N, K, _p(q), _p(s))
    return q, s


# ---------------------------------------------------------------- gemm

def gemm_s32(qa: np.ndarray, qb: np.ndarray) -> np.ndarray:
    """a2: acc[m,n] = sum_k qa[m,k] qb[n,k] (int32; raises on overflow)."""
    qa, qb = _c(qa, np.int8), _c(qb, np.int8)
    M, K = qa.shape
    N = qb.shape[0]
    acc = np.empty((M, N), dtype=np.int32)
    bad = lib().oracle_gemm_s32(_p(qa), _p(qb), M, N, K, _p(acc))
    if bad:
        raise OverflowError(f"{bad} accumulators outside int32")
    return acc


def gemm_s32_at(qa, qb, ms, ns) -> np.ndarray:
    qa, qb = _c(qa, np.int8), _c(qb, np.int8)
    ms, ns = _c(ms, np.int64), _c(ns, np.int64)
    out = np.empty(ms.size, dtype=np.int32)
    lib().oracle_gemm_s32_at(_p(qa), _p(qb), qa.shape[1], _p(ms), _p(ns), ms.size, _p(out))
    return out


def dequant(acc, sx, sw):
    """a3: returns (y bf16 bits, y fp32, y fp64)."""
    acc = _c(acc, np.int32)
    sx, sw = _c(sx, np.float32), _c(sw, np.float32)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.uint16)
    y32 = np.empty((M, N), dtype=np.float32)
    y64 = np.empty((M, N), dtype=np.float64)
    lib().oracle_dequant(_p(acc), _p(sx), _p(sw), M, N, _p(y), _p(y32), _p(y64))
    return y, y32, y64


def linear(x_bits, qw, sw):
    """a1 + a2 + a3: returns (y bf16 bits, y fp32, qx, sx)."""
    x = _c(x_bits, np.uint16)
    qw, sw = _c(qw, np.int8), _c(sw, np.float32)
    M, K = x.shape
    N = qw.shape[0]
    qx = np.empty((M, K), dtype=np.int8)
    sx = np.empty(M, dtype=np.float32)
    y = np.empty((M, N), dtype=np.uint16)
    y32 = np.empty((M, N), dtype=np.float32)
    lib().oracle_linear(_p(x), _p(qw), _p(sw), M, N, K, _p(qx), _p(sx), _p(y), _p(y32))
    return y, y32, qx, sx


# ---------------------------------------------------------------- exp / silu

def exp_proj(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    y = np.empty_like(x)
    lib().oracle_exp_proj_array(_p(x), _p(y), x.size)
    return y


def silu(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    y = np.empty_like(x)
    lib().oracle_silu_array(_p(x), _p(y), x.size)
    return y


# ---------------------------------------------------------------- routing / MoE

def route(logits_bits, topk: int):
    """a5: (ids int32 [T,k] descending, weights fp32 [T,k])."""
    lg = _c(logits_bits, np.uint16)
    T, E = lg.shape
    ids = np.empty((T, topk), dtype=np.int32)
    w = np.empty((T, topk), dtype=np.float32)
    lib().oracle_route(_p(lg), T, E, topk, _p(ids), _p(w))
    return ids, w


def histogram(ids, E: int):
    ids = _c(ids, np.int32).reshape(-1)
    counts = np.empty(E, dtype=np.int32)
    lib().oracle_moe_histogram(_p(ids), ids.size, E, _p(counts))
    return counts


def moe_forward(x_bits, logits_bits, w13, s13, w2, s2, topk: int, tokens=None):
    """a5-a11 for the listed tokens (all when None).  Returns a dict."""
    x = _c(x_bits, np.uint16)
    lg = _c(logits_bits, np.uint16)
    w13, w2 = _c(w13, np.int8), _c(w2, np.int8)
    s13, s2 = _c(s13, np.float32), _c(s2, np.float32)
    T, H = x.shape
    E, I2, H2 = w13.shape
    assert H2 == H and I2 % 2 == 0 and w2.shape == (E, H, I2 // 2)
    I = I2 // 2
    toks = np.arange(T, dtype=np.int64) if tokens is None else _c(tokens, np.int64)
    n = toks.size
    out = dict(
        y=np.empty((n, H), np.uint16), y32=np.empty((n, H), np.float32),
        yabs=np.empty((n, H), np.float32), ids=np.empty((n, topk), np.int32),
        wts=np.empty((n, topk), np.float32), qx=np.empty((n, H), np.int8),
        sx=np.empty(n, np.float32), qa=np.empty((n, topk, I), np.int8),
        sa=np.empty((n, topk), np.float32))
    lib().oracle_moe_forward(_p(x), _p(lg), _p(w13), _p(s13), _p(w2), _p(s2), T, E, H, I, topk,
                             _p(toks), n, _p(out["y"]), _p(out["y32"]), _p(out["yabs"]),
                             _p(out["ids"]), _p(out["wts"]), _p(out["qx"]), _p(out["sx"]),
                             _p(out["qa"]), _p(out["sa"]))
    out["tokens"] = toks
    return out


def mlp_forward(x_bits, w13, s13, w2, s2):
    """Dense gated MLP block (x -> gate_up + SiLU*up -> requant -> down) for
    all tokens.  w13 int8 [2I, H], s13 [2I], w2 int8 [H, I], s2 [H].
    Returns a dict with y (bf16 bits), y32, qx, sx, qa, sa."""
    x = _c(x_bits, np.uint16)
    w13, w2 = _c(w13, np.int8), _c(w2, np.int8)
    s13, s2 = _c(s13, np.float32), _c(s2, np.float32)
    M, H = x.shape
    I2, H2 = w13.shape
    assert H2 == H and I2 % 2 == 0 and w2.shape == (H, I2 // 2)
    I = I2 // 2
    out = dict(y=np.empty((M, H), np.uint16), y32=np.empty((M, H), np.float32),
               qx=np.empty((M, H), np.int8), sx=np.empty(M, np.float32),
               qa=np.empty((M, I), np.int8), sa=np.empty(M, np.float32))
    lib().oracle_mlp_forward(_p(x), _p(w13), _p(s13), _p(w2), _p(s2), M, H, I, _p(out["y"]), _p(out["y32"]),
                             _p(out["qx"]), _p(out["sx"]), _p(out["qa"]), _p(out["sa"]))
    return out


# ---------------------------------------------------------------- FWHT128

def fwht128(v: np.ndarray) -> np.ndarray:
    v = np.array(v, dtype=np.float32).reshape(128).copy()
    lib().oracle_fwht128(_p(v))
    return v


def fwht128_quant(x_bits):
    """a12: returns (codes int8 [M,K], scales bf16 bits [M,K/128], rotated fp32 [M,K])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    assert K % 128 == 0
    q = np.empty((M, K), np.int8)
    s = np.empty((M, K // 128), np.uint16)
    xr = np.empty((M, K), np.float32)
    lib().oracle_fwht128_quant(_p(x), M, K, _p(q), _p(s), _p(xr))
    return q, s, xr


def fwht128_quant_f32(x):
    """a12 on fp32 rows: returns (codes int8 [M,K], scales bf16 bits [M,K/128])."""
    x = _c(x, np.float32)
    M, K = x.shape
    assert K % 128 == 0
    q = np.empty((M, K), np.int8)
    s = np.empty((M, K // 128), np.uint16)
    lib().oracle_fwht128_quant_f32(_p(x), M, K, _p(q), _p(s))
    return q, s


def moe_g128_forward(x_bits, logits_bits, w13, s13_bits, w2, s2_bits, topk: int, tokens=None):
    """Routed experts on the FWHT128 grid for the listed tokens (all when
    None).  w13 int8 [E,2I,H] + bf16 bits [E,2I,H/128]; w2 int8 [E,H,I] +
    bf16 bits [E,H,I/128].  Returns a dict like moe_forward, with the scales
    sx [n,H/128] and sa [n,k,I/128] as bf16 bits."""
    x = _c(x_bits, np.uint16)
    lg = _c(logits_bits, np.uint16)
    w13, w2 = _c(w13, np.int8), _c(w2, np.int8)
    s13, s2 = _c(s13_bits, np.uint16), _c(s2_bits, np.uint16)
    T, H = x.shape
    E, I2, H2 = w13.shape
    assert H2 == H and I2 % 2 == 0 and H % 128 == 0
    I = I2 // 2
    assert I % 128 == 0 and w2.shape == (E, H, I)
    assert s13.shape == (E, I2, H // 128) and s2.shape == (E, H, I // 128)
    toks = np.arange(T, dtype=np.int64) if tokens is None else _c(tokens, np.int64)
    n = toks.size
    out = dict(
        y=np.empty((n, H), np.uint16), y32=np.empty((n, H), np.float32),
        yabs=np.empty((n, H), np.float32), ids=np.empty((n, topk), np.int32),
        wts=np.empty((n, topk), np.float32), qx=np.empty((n, H), np.int8),
        sx=np.empty((n, H // 128), np.uint16), qa=np.empty((n, topk, I), np.int8),
        sa=np.empty((n, topk, I // 128), np.uint16))
    lib().oracle_moe_g128_forward(_p(x), _p(lg), _p(w13), _p(s13), _p(w2), _p(s2), T, E, H, I, topk,
                                  _p(toks), n, _p(out["y"]), _p(out["y32"]), _p(out["yabs"]),
                                  _p(out["ids"]), _p(out["wts"]), _p(out["qx"]), _p(out["sx"]),
                                  _p(out["qa"]), _p(out["sa"]))
    out["tokens"] = toks
    return out


def gemm_g128(qx, sx_bits, qw, sw_bits):
    """a13: returns (y bf16 bits [M,N], y fp32)."""
    qx, qw = _c(qx, np.int8), _c(qw, np.int8)
    sx, sw = _c(sx_bits, np.uint16), _c(sw_bits, np.uint16)
    M, K = qx.shape
    N = qw.shape[0]
    y = np.empty((M, N), np.uint16)
    y32 = np.empty((M, N), np.float32)
    lib().oracle_gemm_g128(_p(qx), _p(sx), _p(qw), _p(sw), M, N, K, _p(y), _p(y32))
    return y, y32


def group128_quant(x_bits):
    """Group-128 quant without the rotation (the head's grid): returns
    (codes int8 [M,K], scales bf16 bits [M,K/128])."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    assert K % 128 == 0
    q = np.empty((M, K), np.int8)
    s = np.empty((M, K // 128), np.uint16)
    lib().oracle_group128_quant(_p(x), M, K, _p(q), _p(s))
    return q, s


def gemm_group128(qx, sx_bits, qw, sw_bits):
    """Group-128 GEMM on the unrotated grid (no 1/128): returns (y bf16 bits, y fp32)."""
    qx, qw = _c(qx, np.int8), _c(qw, np.int8)
    sx, sw = _c(sx_bits, np.uint16), _c(sw_bits, np.uint16)
    M, K = qx.shape
    N = qw.shape[0]
    y = np.empty((M, N), np.uint16)
    y32 = np.empty((M, N), np.float32)
    lib().oracle_gemm_group128(_p(qx), _p(sx), _p(qw), _p(sw), M, N, K, _p(y), _p(y32))
    return y, y32


def trunk_weight_quant(w_bits):
    """Two-level trunk format of bf16 rows [N,K] (K % 256 == 0): returns
    (codes int8 [N,K], u8 group scales [N,K/256], bf16 row scales [N])."""
    w = _c(w_bits, np.uint16)
    N, K = w.shape
    assert K % 256 == 0
    q = np.empty((N, K), np.int8)
    su8 = np.empty((N, K // 256), np.uint8)
    s2 = np.empty(N, np.uint16)
    lib().oracle_trunk_weight_quant(_p(w), N, K, _p(q), _p(su8), _p(s2))
    return q, su8, s2


def gemm_trunk(qx, sx_bits, qw, su8, s2_bits):
    """Trunk GEMM (x rotated with bf16 group-128 scales, W two-level): returns
    (y bf16 bits [M,N], y fp32)."""
    qx, qw = _c(qx, np.int8), _c(qw, np.int8)
    sx, su8, s2 = _c(sx_bits, np.uint16), _c(su8, np.uint8), _c(s2_bits, np.uint16)
    M, K = qx.shape
    N = qw.shape[0]
    y = np.empty((M, N), np.uint16)
    y32 = np.empty((M, N), np.float32)
    lib().oracle_gemm_trunk(_p(qx), _p(sx), _p(qw), _p(su8), _p(s2), M, N, K, _p(y), _p(y32))
    return y, y32


def shared_expert_forward(x_bits, w13, u13, r13_bits, w2, s2_bits):
    """The shared expert on the rotated grid: x bf16 bits [M,H]; gate_up in the
    trunk format (w13 int8 [2I,H], u8 [2I,H/256], bf16 row scales [2I]); down
    on the group-128 grid (w2 int8 [H,I], bf16 [H,I/128]).  Returns a dict
    with y (bf16 bits), y32, qx, sx, qa, sa (scales as bf16 bits)."""
    x = _c(x_bits, np.uint16)
    w13, w2 = _c(w13, np.int8), _c(w2, np.int8)
    u13, r13, s2 = _c(u13, np.uint8), _c(r13_bits, np.uint16), _c(s2_bits, np.uint16)
    M, H = x.shape
    I2 = w13.shape[0]
    I = I2 // 2
    assert w13.shape == (I2, H) and u13.shape == (I2, H // 256) and r13.shape == (I2,)
    assert w2.shape == (H, I) and s2.shape == (H, I // 128)
    out = dict(y=np.empty((M, H), np.uint16), y32=np.empty((M, H), np.float32),
               qx=np.empty((M, H), np.int8), sx=np.empty((M, H // 128), np.uint16),
               qa=np.empty((M, I), np.int8), sa=np.empty((M, I // 128), np.uint16))
    lib().oracle_shared_expert_forward(_p(x), _p(w13), _p(u13), _p(r13), _p(w2), _p(s2), M, H, I,
                                       _p(out["y"]), _p(out["y32"]), _p(out["qx"]), _p(out["sx"]),
                                       _p(out["qa"]), _p(out["sa"]))
    return out


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())
