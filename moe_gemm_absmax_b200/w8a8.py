"""Thin ctypes binding of libw8a8.so, with the C entry points' names.

Argument marshalling only: each function checks dtypes/devices, allocates
outputs with torch (device memory), passes raw pointers and the current CUDA
stream to the library, and raises :class:`W8A8Error` on a non-zero status.
Every step of the computation runs in the library's CUDA kernels; there is
no CPU path.  If the library has not been built, :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw8a8.so")

OK, ERR_INVALID_ARG, ERR_WORKSPACE, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
PATH_AUTO, PATH_TCGEN05, PATH_GEMV = 0, 1, 2

# Every function the header include/w8a8.h declares.
EXPORTS = (
    "w8a8_quant_act", "w8a8_quant_rows_f32", "w8a8_linear_workspace_size", "w8a8_linear",
    "w8a8_linear_noalloc_scratch_size", "w8a8_linear_noalloc",
    "w8a8_gemm_workspace_size", "w8a8_gemm_q", "w8a8_gemm_s32", "w8a8_moe_workspace_size",
    "w8a8_moe_forward", "w8a8_moe_set_combine", "w8a8_moe_g128_workspace_size", "w8a8_moe_g128_forward", "w8a8_mlp_workspace_size", "w8a8_mlp_forward", "fwht128_quant", "w8a8_linear_g128",
    "group128_quant", "w8a8_linear_group128", "w8a8_trunk_weight_quant", "w8a8_linear_trunk",
    "w8a8_shared_expert_workspace_size", "w8a8_shared_expert_forward",
    "w8a8_exp_proj",
    "w8a8_get_device_error", "w8a8_debug_wait_timeout", "w8a8_status_str", "w8a8_version",
)

_lib = None


class W8A8Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


class MoeG128Debug(ctypes.Structure):
    _fields_ = [("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("qx", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("qa", ctypes.c_void_p),
                ("sa", ctypes.c_void_p)]


class SharedExpertDebug(ctypes.Structure):
    _fields_ = [("qx", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("qa", ctypes.c_void_p), ("sa", ctypes.c_void_p)]


class MlpDebug(ctypes.Structure):
    _fields_ = [("qx", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("qa", ctypes.c_void_p), ("sa", ctypes.c_void_p)]


class MoeDebug(ctypes.Structure):
    _fields_ = [("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("qx", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("qa", ctypes.c_void_p),
                ("sa", ctypes.c_void_p)]


def lib() -> ctypes.CDLL:
    """Loads the library (raises if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libw8a8.so not built ({LIB_PATH}); run moe_gemm_absmax_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    sig = {
        "w8a8_quant_act": ([vp, i64, i64, i64, vp, vp, vp], i32),
        "w8a8_quant_rows_f32": ([vp, i64, i64, vp, vp, vp], i32),
        "w8a8_linear_workspace_size": ([i64, i64, i64], sz),
        "w8a8_linear": ([vp, vp, vp, vp, i64, i64, i64, vp, sz, vp], i32),
        "w8a8_linear_noalloc_scratch_size": ([i64, i64, i64], sz),
        "w8a8_linear_noalloc": ([vp, vp, vp, vp, i64, i64, i64, vp], i32),
        "w8a8_gemm_workspace_size": ([i64, i64, i64, i32], sz),
        "w8a8_gemm_q": ([vp, vp, vp, vp, vp, i64, i64, i64, i32, vp, sz, vp], i32),
        "w8a8_gemm_s32": ([vp, vp, vp, i64, i64, i64, i32, vp, sz, vp], i32),
        "w8a8_moe_workspace_size": ([i64, i32, i32, i32, i32], sz),
        "w8a8_moe_set_combine": ([i32], i32),
        "w8a8_moe_forward": ([vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, vp, sz,
                              ctypes.POINTER(MoeDebug), vp], i32),
        "w8a8_moe_g128_workspace_size": ([i64, i32, i32, i32, i32], sz),
        "w8a8_moe_g128_forward": ([vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, i32, i32, vp, sz,
                                   ctypes.POINTER(MoeG128Debug), vp], i32),
        "w8a8_mlp_workspace_size": ([i64, i64, i64], sz),
        "w8a8_mlp_forward": ([vp, vp, vp, vp, vp, vp, i64, i64, i64, vp, sz, ctypes.POINTER(MlpDebug), vp], i32),
        "fwht128_quant": ([vp, i64, i64, vp, vp, vp], i32),
        "w8a8_linear_g128": ([vp, vp, vp, vp, vp, i64, i64, i64, vp], i32),
        "group128_quant": ([vp, i64, i64, vp, vp, vp], i32),
        "w8a8_linear_group128": ([vp, vp, vp, vp, vp, i64, i64, i64, vp], i32),
        "w8a8_trunk_weight_quant": ([vp, i64, i64, vp, vp, vp, vp], i32),
        "w8a8_linear_trunk": ([vp, vp, vp, vp, vp, vp, i64, i64, i64, vp], i32),
        "w8a8_shared_expert_workspace_size": ([i64, i32, i32], sz),
        "w8a8_shared_expert_forward": ([vp, vp, vp, vp, vp, vp, vp, i64, i32, i32, vp, sz,
                                        ctypes.POINTER(SharedExpertDebug), vp], i32),
        "w8a8_exp_proj": ([vp, vp, i64, vp], i32),
        "w8a8_get_device_error": ([vp, ctypes.POINTER(ctypes.c_int)], i32),
        "w8a8_debug_wait_timeout": ([i64, vp], i32),
        "w8a8_status_str": ([i32], ctypes.c_char_p),
        "w8a8_version": ([], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def status_str(status: int) -> str:
    try:
        return lib().w8a8_status_str(int(status)).decode()
    except RuntimeError:
        return "library not loaded"


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise W8A8Error(rc, what)


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ quant

def quant_act(x: torch.Tensor, stream=None):
    """Per-token int8 quant of bf16 x [M,K] -> (codes int8 [M,K], scales fp32 [M]).

    x may be a row-strided view (unit column stride, row stride = ldx)."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise TypeError("x must be a CUDA tensor")
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise TypeError("x must be a 2-D bfloat16 tensor")
    M, K = x.shape
    ldx = x.stride(0) if M > 1 else K
    if x.stride(1) != 1 or ldx < K:
        raise ValueError("x rows must be contiguous (unit column stride, row stride >= K)")
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().w8a8_quant_act(_ptr(x), M, K, ldx, _ptr(q), _ptr(s), _stream(stream)), "w8a8_quant_act")
    return q, s


def quant_rows_f32(w: torch.Tensor, stream=None):
    """Per-output-channel int8 quant of fp32 weights [N,K] -> (int8 [N,K], fp32 [N])."""
    _need(w, torch.float32, "w")
    K = w.shape[-1]
    N = w.numel() // K
    q = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    s = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    _check(lib().w8a8_quant_rows_f32(_ptr(w), N, K, _ptr(q), _ptr(s), _stream(stream)), "w8a8_quant_rows_f32")
    return q, s


# ------------------------------------------------------------------ dense

def linear_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().w8a8_linear_workspace_size(M, N, K))


def linear(x: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, y: torch.Tensor | None = None,
           ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Dense W8A8 linear: bf16 x [M,K] against int8 qw [N,K] / fp32 sw [N] -> bf16 [M,N]."""
    _need(x, torch.bfloat16, "x", 2)
    _need(qw, torch.int8, "qw", 2)
    _need(sw, torch.float32, "sw", 1)
    M, K = x.shape
    N = qw.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    need = linear_workspace_size(M, N, K)
    if ws is None:
        ws = _workspace(need, x.device)
    _check(lib().w8a8_linear(_ptr(x), _ptr(qw), _ptr(sw), _ptr(y), M, N, K, _ptr(ws), ws.numel(),
                             _stream(stream)), "w8a8_linear")
    return y


NOALLOC_SCRATCH_BYTES = 4 << 20


def linear_noalloc(x: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor, y: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """The dense W8A8 linear for callers that cannot allocate device memory
    while it runs: same result as :func:`linear`, scratch kept in the
    library's static device array (at most NOALLOC_SCRATCH_BYTES), so only
    x, the weights and y are passed.  Calls that overlap on the GPU race on
    that array; the first call on a device must come before stream capture.
    (The output tensor is allocated here only when the caller passes none.)"""
    _need(x, torch.bfloat16, "x", 2)
    _need(qw, torch.int8, "qw", 2)
    _need(sw, torch.float32, "sw", 1)
    M, K = x.shape
    N = qw.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().w8a8_linear_noalloc(_ptr(x), _ptr(qw), _ptr(sw), _ptr(y), M, N, K, _stream(stream)),
           "w8a8_linear_noalloc")
    return y


def gemm_workspace_size(M: int, N: int, K: int, path: int = PATH_AUTO) -> int:
    return int(lib().w8a8_gemm_workspace_size(M, N, K, path))


def gemm_q(qx, sx, qw, sw, path: int = PATH_AUTO, y=None, ws=None, stream=None) -> torch.Tensor:
    _need(qx, torch.int8, "qx", 2)
    _need(qw, torch.int8, "qw", 2)
    _need(sx, torch.float32, "sx", 1)
    _need(sw, torch.float32, "sw", 1)
    M, K = qx.shape
    N = qw.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    if ws is None:
        ws = _workspace(gemm_workspace_size(M, N, K, path), qx.device)
    _check(lib().w8a8_gemm_q(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(y), M, N, K, path, _ptr(ws),
                             ws.numel(), _stream(stream)), "w8a8_gemm_q")
    return y


def gemm_s32(qx, qw, path: int = PATH_AUTO, acc=None, ws=None, stream=None) -> torch.Tensor:
    _need(qx, torch.int8, "qx", 2)
    _need(qw, torch.int8, "qw", 2)
    M, K = qx.shape
    N = qw.shape[0]
    if acc is None:
        acc = torch.empty((M, N), dtype=torch.int32, device=qx.device)
    if ws is None:
        ws = _workspace(gemm_workspace_size(M, N, K, path), qx.device)
    _check(lib().w8a8_gemm_s32(_ptr(qx), _ptr(qw), _ptr(acc), M, N, K, path, _ptr(ws), ws.numel(),
                               _stream(stream)), "w8a8_gemm_s32")
    return acc


# ------------------------------------------------------------------ MoE

def moe_workspace_size(T: int, E: int, H: int, I: int, topk: int) -> int:
    return int(lib().w8a8_moe_workspace_size(T, E, H, I, topk))


MOE_COMBINE_AUTO, MOE_COMBINE_EXACT = 0, 1


def moe_set_combine(mode: int) -> int:
    """Combine mode of moe_forward (process-wide); returns the previous one."""
    r = int(lib().w8a8_moe_set_combine(int(mode)))
    if r < 0:
        raise W8A8Error(r, "w8a8_moe_set_combine")
    return r


def moe_forward(x, logits, w13, s13, w2, s2, topk: int = 8, y=None, ws=None, debug: bool = False,
                stream=None):
    """Routed W8A8 MoE layer.  Returns y bf16 [T,H], or (y, debug dict) when debug."""
    _need(x, torch.bfloat16, "x", 2)
    _need(logits, torch.bfloat16, "logits", 2)
    _need(w13, torch.int8, "w13", 3)
    _need(w2, torch.int8, "w2", 3)
    _need(s13, torch.float32, "s13", 2)
    _need(s2, torch.float32, "s2", 2)
    T, H = x.shape
    E, I2, _ = w13.shape
    I = I2 // 2
    dev = x.device
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(moe_workspace_size(T, E, H, I, topk), dev)
    dbg_t = None
    dbg_p = None
    if debug:
        dbg_t = dict(topk_ids=torch.empty((T, topk), dtype=torch.int32, device=dev),
                     topk_w=torch.empty((T, topk), dtype=torch.float32, device=dev),
                     counts=torch.empty(E, dtype=torch.int32, device=dev),
                     qx=torch.empty((T, H), dtype=torch.int8, device=dev),
                     sx=torch.empty(T, dtype=torch.float32, device=dev),
                     qa=torch.empty((T, topk, I), dtype=torch.int8, device=dev),
                     sa=torch.empty((T, topk), dtype=torch.float32, device=dev))
        dbg_p = ctypes.pointer(MoeDebug(*[v.data_ptr() for v in dbg_t.values()]))
    _check(lib().w8a8_moe_forward(_ptr(x), _ptr(logits), _ptr(w13), _ptr(s13), _ptr(w2), _ptr(s2), _ptr(y),
                                  T, E, H, I, topk, _ptr(ws), ws.numel(), dbg_p, _stream(stream)),
           "w8a8_moe_forward")
    return (y, dbg_t) if debug else y


# ------------------------------------------------------------------ MoE on the FWHT128 grid

def moe_g128_workspace_size(T: int, E: int, H: int, I: int, topk: int) -> int:
    return int(lib().w8a8_moe_g128_workspace_size(T, E, H, I, topk))


def moe_g128_forward(x, logits, w13, s13, w2, s2, topk: int = 8, y=None, ws=None, debug: bool = False,
                     stream=None):
    """Routed experts on the FWHT128 grid: bf16 x [T,H] (unrotated), bf16 logits [T,E];
    w13 int8 [E,2I,H] with bf16 group scales s13 [E,2I,H/128]; w2 int8 [E,H,I] with
    s2 [E,H,I/128] (rows rotated along K and group-quantized, e.g. by fwht128_quant).
    Returns y bf16 [T,H], or (y, debug dict) when debug."""
    _need(x, torch.bfloat16, "x", 2)
    _need(logits, torch.bfloat16, "logits", 2)
    _need(w13, torch.int8, "w13", 3)
    _need(w2, torch.int8, "w2", 3)
    _need(s13, torch.bfloat16, "s13", 3)
    _need(s2, torch.bfloat16, "s2", 3)
    T, H = x.shape
    E, I2, _ = w13.shape
    I = I2 // 2
    dev = x.device
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(moe_g128_workspace_size(T, E, H, I, topk), dev)
    dbg_t = None
    dbg_p = None
    if debug:
        dbg_t = dict(topk_ids=torch.empty((T, topk), dtype=torch.int32, device=dev),
                     topk_w=torch.empty((T, topk), dtype=torch.float32, device=dev),
                     counts=torch.empty(E, dtype=torch.int32, device=dev),
                     qx=torch.empty((T, H), dtype=torch.int8, device=dev),
                     sx=torch.empty((T, H // 128), dtype=torch.bfloat16, device=dev),
                     qa=torch.empty((T, topk, I), dtype=torch.int8, device=dev),
                     sa=torch.empty((T, topk, I // 128), dtype=torch.bfloat16, device=dev))
        dbg_p = ctypes.pointer(MoeG128Debug(*[v.data_ptr() for v in dbg_t.values()]))
    _check(lib().w8a8_moe_g128_forward(_ptr(x), _ptr(logits), _ptr(w13), _ptr(s13), _ptr(w2), _ptr(s2), _ptr(y),
                                       T, E, H, I, topk, _ptr(ws), ws.numel(), dbg_p, _stream(stream)),
           "w8a8_moe_g128_forward")
    return (y, dbg_t) if debug else y


# ------------------------------------------------------------------ dense gated MLP block

def mlp_workspace_size(M: int, H: int, I: int) -> int:
    return int(lib().w8a8_mlp_workspace_size(M, H, I))


def mlp_forward(x, w13, s13, w2, s2, y=None, ws=None, debug: bool = False, stream=None):
    """Dense gated MLP block: bf16 x [M,H] -> gate_up (w13 int8 [2I,H], rows 2i gate /
    2i+1 up, s13 [2I]) with SiLU(gate)*up -> requant -> down (w2 int8 [H,I], s2 [H])
    -> bf16 y [M,H].  Returns y, or (y, debug dict) when debug."""
    _need(x, torch.bfloat16, "x", 2)
    _need(w13, torch.int8, "w13", 2)
    _need(w2, torch.int8, "w2", 2)
    _need(s13, torch.float32, "s13", 1)
    _need(s2, torch.float32, "s2", 1)
    M, H = x.shape
    I = w13.shape[0] // 2
    dev = x.device
    if y is None:
        y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(mlp_workspace_size(M, H, I), dev)
    dbg_t = dbg_p = None
    if debug:
        dbg_t = dict(qx=torch.empty((M, H), dtype=torch.int8, device=dev),
                     sx=torch.empty(M, dtype=torch.float32, device=dev),
                     qa=torch.empty((M, I), dtype=torch.int8, device=dev),
                     sa=torch.empty(M, dtype=torch.float32, device=dev))
        dbg_p = ctypes.pointer(MlpDebug(*[v.data_ptr() for v in dbg_t.values()]))
    _check(lib().w8a8_mlp_forward(_ptr(x), _ptr(w13), _ptr(s13), _ptr(w2), _ptr(s2), _ptr(y), M, H, I, _ptr(ws),
                                  ws.numel(), dbg_p, _stream(stream)), "w8a8_mlp_forward")
    return (y, dbg_t) if debug else y


# ------------------------------------------------------------------ FWHT128

def fwht128_quant(x: torch.Tensor, stream=None):
    """Rotated group-128 quant of bf16 x [M,K] -> (int8 [M,K], bf16 scales [M,K/128])."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.bfloat16, device=x.device)
    _check(lib().fwht128_quant(_ptr(x), M, K, _ptr(q), _ptr(s), _stream(stream)), "fwht128_quant")
    return q, s


def linear_g128(qx, sx, qw, sw, y=None, stream=None) -> torch.Tensor:
    _need(qx, torch.int8, "qx", 2)
    _need(qw, torch.int8, "qw", 2)
    _need(sx, torch.bfloat16, "sx", 2)
    _need(sw, torch.bfloat16, "sw", 2)
    M, K = qx.shape
    N = qw.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    _check(lib().w8a8_linear_g128(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(y), M, N, K, _stream(stream)),
           "w8a8_linear_g128")
    return y


def group128_quant(x: torch.Tensor, stream=None):
    """Group-128 quant without the rotation (the head's grid): bf16 x [M,K] ->
    (int8 [M,K], bf16 scales [M,K/128])."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.int8, device=x.device)
    s = torch.empty((M, K // 128), dtype=torch.bfloat16, device=x.device)
    _check(lib().group128_quant(_ptr(x), M, K, _ptr(q), _ptr(s), _stream(stream)), "group128_quant")
    return q, s


def linear_group128(qx, sx, qw, sw, y=None, stream=None) -> torch.Tensor:
    """Group-128 GEMM on the unrotated grid (no 1/128): -> bf16 y [M,N]."""
    _need(qx, torch.int8, "qx", 2)
    _need(qw, torch.int8, "qw", 2)
    _need(sx, torch.bfloat16, "sx", 2)
    _need(sw, torch.bfloat16, "sw", 2)
    M, K = qx.shape
    N = qw.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    _check(lib().w8a8_linear_group128(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(sw), _ptr(y), M, N, K, _stream(stream)),
           "w8a8_linear_group128")
    return y


def trunk_weight_quant(w: torch.Tensor, stream=None):
    """The trunk's two-level format of bf16 rows [N,K] (K % 256 == 0): returns
    (codes int8 [N,K], u8 group scales [N,K/256], bf16 row scales [N])."""
    _need(w, torch.bfloat16, "w", 2)
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.int8, device=w.device)
    su8 = torch.empty((N, K // 256), dtype=torch.uint8, device=w.device)
    s2 = torch.empty(N, dtype=torch.bfloat16, device=w.device)
    _check(lib().w8a8_trunk_weight_quant(_ptr(w), N, K, _ptr(q), _ptr(su8), _ptr(s2), _stream(stream)),
           "w8a8_trunk_weight_quant")
    return q, su8, s2


def linear_trunk(qx, sx, qw, su8, s2, y=None, stream=None) -> torch.Tensor:
    """x codes + bf16 group scales (fwht128_quant) times W in the trunk format -> bf16 y [M,N]."""
    _need(qx, torch.int8, "qx", 2)
    _need(qw, torch.int8, "qw", 2)
    _need(sx, torch.bfloat16, "sx", 2)
    _need(su8, torch.uint8, "su8", 2)
    _need(s2, torch.bfloat16, "s2", 1)
    M, K = qx.shape
    N = qw.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    _check(lib().w8a8_linear_trunk(_ptr(qx), _ptr(sx), _ptr(qw), _ptr(su8), _ptr(s2), _ptr(y), M, N, K,
                                   _stream(stream)), "w8a8_linear_trunk")
    return y


def shared_expert_workspace_size(M: int, H: int, I: int) -> int:
    return int(lib().w8a8_shared_expert_workspace_size(M, H, I))


def shared_expert_forward(x, w13, u13, r13, w2, s2, y=None, ws=None, debug: bool = False, stream=None):
    """The shared expert on the rotated grid: bf16 x [M,H]; gate_up in the trunk format
    (w13 int8 [2I,H], u13 uint8 [2I,H/256], r13 bf16 [2I]); down on the group-128 grid
    (w2 int8 [H,I], s2 bf16 [H,I/128]).  Returns y bf16 [M,H], or (y, debug dict)."""
    _need(x, torch.bfloat16, "x", 2)
    _need(w13, torch.int8, "w13", 2)
    _need(u13, torch.uint8, "u13", 2)
    _need(r13, torch.bfloat16, "r13", 1)
    _need(w2, torch.int8, "w2", 2)
    _need(s2, torch.bfloat16, "s2", 2)
    M, H = x.shape
    I = w13.shape[0] // 2
    dev = x.device
    if y is None:
        y = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = _workspace(shared_expert_workspace_size(M, H, I), dev)
    dbg_t = dbg_p = None
    if debug:
        dbg_t = dict(qx=torch.empty((M, H), dtype=torch.int8, device=dev),
                     sx=torch.empty((M, H // 128), dtype=torch.bfloat16, device=dev),
                     qa=torch.empty((M, I), dtype=torch.int8, device=dev),
                     sa=torch.empty((M, I // 128), dtype=torch.bfloat16, device=dev))
        dbg_p = ctypes.pointer(SharedExpertDebug(*[v.data_ptr() for v in dbg_t.values()]))
    _check(lib().w8a8_shared_expert_forward(_ptr(x), _ptr(w13), _ptr(u13), _ptr(r13), _ptr(w2), _ptr(s2), _ptr(y),
                                            M, H, I, _ptr(ws), ws.numel(), dbg_p, _stream(stream)),
           "w8a8_shared_expert_forward")
    return (y, dbg_t) if debug else y


# ------------------------------------------------------------------ diagnostics

def exp_proj(x: torch.Tensor, stream=None) -> torch.Tensor:
    _need(x, torch.float32, "x")
    y = torch.empty_like(x)
    _check(lib().w8a8_exp_proj(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "w8a8_exp_proj")
    return y


def get_device_error(stream=None):
    """Synchronizes the stream; returns (status, site) and clears the error word."""
    site = ctypes.c_int(0)
    rc = lib().w8a8_get_device_error(_stream(stream), ctypes.byref(site))
    return int(rc), int(site.value)


def debug_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(lib().w8a8_debug_wait_timeout(int(limit_ns), _stream(stream)), "w8a8_debug_wait_timeout")


def version() -> str:
    return lib().w8a8_version().decode()
