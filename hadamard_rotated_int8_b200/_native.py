"""ctypes binding of ``libsdnq.so`` (C ABI in ``include/sdnq.h``).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
Tensors are torch CUDA tensors; bf16 tensors are passed by pointer and read as raw 16-bit
patterns. Calls are asynchronous on torch's current CUDA stream. There is no fallback: if
the library is missing or the device is not a B200 (sm_100), calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from . import _build

_lib = None
_lock = threading.Lock()

SDNQ_OK = 0
SDNQ_ERR_NULL = 1
SDNQ_ERR_SHAPE = 2
SDNQ_ERR_ALIGN = 3
SDNQ_ERR_UNSUPPORTED = 4
SDNQ_ERR_CUDA = 5
SDNQ_ERR_TIMEOUT = 6

MAX_K = 131072
MIN_GROUP = 8
MAX_GROUP = 256
MAX_RANK = 256

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_F = ctypes.c_float

SIGNATURES = {
    "sdnq_rotate_quant_weight": [_P, _I64, _I64, _I64, _I32, _P, _P, _P],
    "sdnq_rotquant_act": [_P, _I64, _I64, _I64, _I32, _P, _P, _P],
    "sdnq_int8_linear": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _P],
    "sdnq_int8_linear_gelu": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _P],
    "sdnq_int8_linear_fused": [_P, _I64, _I32, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P, _I64,
                               _P, _I32, _P],
    "sdnq_int8_linear_fused_plan": [_I64, _I64, _I64, _I32, _P],
    "sdnq_int8_linear_grad_input": [_P, _I64, _P, _P, _I64, _I64, _I64, _I32, _P, _P, _P, _I64,
                                    _P, _P],
    "sdnq_quant_grad_output": [_P, _I64, _P, _I64, _I64, _P, _P, _P],
    "sdnq_int8_grad_input_gemm": [_P, _P, _P, _I64, _I64, _I64, _I32, _P, _I64, _P, _P],
    "sdnq_int8_linear_lora": [_P, _P, _P, _P, _P, _P, _I64, _P, _P, _I32, _F, _P, _I64, _I64,
                              _I64, _P, _I64, _P, _P],
    "sdnq_int8_linear_lora_noalloc": [_P, _P, _P, _P, _P, _P, _I64, _P, _P, _I32, _F, _I64,
                                      _I64, _I64, _P, _I64, _P, _P],
    "sdnq_lora_down": [_P, _I64, _P, _I32, _I64, _I64, _P, _P],
    "sdnq_int8_linear_lora_up": [_P, _P, _P, _P, _P, _P, _P, _I32, _F, _I64, _I64, _I64, _P,
                                 _I64, _P, _P],
    "sdnq_gelu_bf16": [_P, _I64, _I64, _I64, _P, _I64, _P],
    "sdnq_rotquant_fp8": [_P, _I64, _I64, _I64, _I32, _P, _P, _P],
    "sdnq_attention_workspace": [_I64, _I64, _I64, _I64, _I64, _P],
    "sdnq_attention_int8qk": [_P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I32, _F, _I32, _P, _I64,
                              _P, _P],
    "sdnq_attention_prep": [_P, _P, _I64, _I64, _I64, _I64, _I64, _I32, _I32, _P, _I64, _P],
    "sdnq_attention_core": [_P, _I64, _I64, _I64, _I64, _I64, _F, _P, _I64, _P, _P],
    "sdnq_fp8_linear": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I64, _P, _P],
    "sdnq_device_status": [_P],
    "sdnq_selftest_wait_timeout": [_I64, _P],
    "sdnq_status_string": [ctypes.c_int],
    "sdnq_version": [],
}


class SdnqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib_path() -> str:
    return _build.LIB


def lib():
    """The loaded ``libsdnq.so`` (ctypes.CDLL with argument types set). Raises if the
    library has not been built (``python -m hadamard_rotated_int8_b200._build``)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                path = lib_path()
                if not os.path.exists(path):
                    raise RuntimeError(
                        f"libsdnq.so not found at {path}: build it with "
                        "`python -m hadamard_rotated_int8_b200._build` (needs nvcc); "
                        "there is no non-CUDA fallback")
                cdll = ctypes.CDLL(path)
                for name, args in SIGNATURES.items():
                    fn = getattr(cdll, name)
                    fn.argtypes = args
                    fn.restype = ctypes.c_char_p if name in ("sdnq_status_string",
                                                             "sdnq_version") else ctypes.c_int
                _lib = cdll
    return _lib


def status_string(status: int) -> str:
    return lib().sdnq_status_string(int(status)).decode()


def version() -> str:
    return lib().sdnq_version().decode()


def _check(status: int, where: str):
    if status != SDNQ_OK:
        raise SdnqError(status, where)


def _stream(stream):
    if stream is None:
        return _P(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return _P(stream.cuda_stream)
    return _P(int(stream))


def _ptr(t: torch.Tensor | None):
    return _P(t.data_ptr()) if t is not None else _P(0)


def _on_current_device(t: torch.Tensor, name: str):
    """The library launches on the current CUDA device; a tensor elsewhere would be read
    through a peer mapping or fault, so it is refused here."""
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor (no CPU path)")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def _req(t: torch.Tensor, dtype, name: str, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    _on_current_device(t, name)
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got {t.dim()}")
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: last dimension must be contiguous")


def _vec(t, dtype, n: int, name: str, optional: bool = False):
    """A dense 1-D tensor of at least n elements (a scale or bias vector the kernels index
    up to n - 1); None is accepted only where the argument is optional."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name}: required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    _on_current_device(t, name)
    if t.dim() != 1 or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous 1-D tensor")
    if t.numel() < n:
        raise ValueError(f"{name}: has {t.numel()} elements, needs {n}")


def _mat(t, dtype, rows: int, cols: int, name: str, dense: bool = False):
    """A 2-D tensor of exactly [rows, cols] with unit column stride (dense if asked)."""
    _req(t, dtype, name, 2)
    if tuple(t.shape) != (rows, cols):
        raise ValueError(f"{name}: expected shape {(rows, cols)}, got {tuple(t.shape)}")
    if dense:
        _dense(t, name)


def _dense(t: torch.Tensor, name: str):
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _rows_out(M: int, N: int, dtype, device) -> torch.Tensor:
    """[M, N] output whose row stride is padded to a multiple of 8 elements (the library
    wants 16-byte aligned rows); returned as a view of the first N columns."""
    ld = (N + 7) // 8 * 8
    buf = torch.empty((M, ld), dtype=dtype, device=device)
    return buf[:, :N] if ld != N else buf


# ---------------------------------------------------------------- the C ABI, by name

def sdnq_rotate_quant_weight(W: torch.Tensor, group: int = 256, qW=None, sW=None, stream=None):
    """W [N, K] bf16 -> (qW [N, K] int8, sW [N] fp32)."""
    _req(W, torch.bfloat16, "W", 2)
    N, K = W.shape
    qW = torch.empty((N, K), dtype=torch.int8, device=W.device) if qW is None else qW
    sW = torch.empty((N,), dtype=torch.float32, device=W.device) if sW is None else sW
    _mat(qW, torch.int8, N, K, "qW", dense=True)
    _vec(sW, torch.float32, N, "sW")
    _check(lib().sdnq_rotate_quant_weight(_ptr(W), N, K, W.stride(0), group, _ptr(qW), _ptr(sW),
                                          _stream(stream)), "sdnq_rotate_quant_weight")
    return qW, sW


def sdnq_rotquant_act(x: torch.Tensor, group: int = 256, qx=None, sx=None, stream=None):
    """x [M, K] bf16 -> (qx [M, K] int8, sx [M] fp32)."""
    _req(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    qx = torch.empty((M, K), dtype=torch.int8, device=x.device) if qx is None else qx
    sx = torch.empty((M,), dtype=torch.float32, device=x.device) if sx is None else sx
    _mat(qx, torch.int8, M, K, "qx", dense=True)
    _vec(sx, torch.float32, M, "sx")
    _check(lib().sdnq_rotquant_act(_ptr(x), M, K, x.stride(0), group, _ptr(qx), _ptr(sx),
                                   _stream(stream)), "sdnq_rotquant_act")
    return qx, sx


def _linear_operands(qx, sx, qW, sW, bias, out, acc_out, code_dtype=torch.int8,
                     acc_dtype=torch.int32):
    """Checks the operands of a linear call; returns (M, N, K, out)."""
    _req(qx, code_dtype, "qx", 2)
    _req(qW, code_dtype, "qW", 2)
    _dense(qx, "qx")
    _dense(qW, "qW")
    M, K = qx.shape
    N = qW.shape[0]
    if qW.shape[1] != K:
        raise ValueError("qx and qW disagree on K")
    _vec(sx, torch.float32, M, "sx")
    _vec(sW, torch.float32, N, "sW")
    _vec(bias, torch.bfloat16, N, "bias", optional=True)
    out = _rows_out(M, N, torch.bfloat16, qx.device) if out is None else out
    _mat(out, torch.bfloat16, M, N, "out")
    if acc_out is not None:
        _mat(acc_out, acc_dtype, M, N, "acc_out", dense=True)
    return M, N, K, out


def _linear_call(name, qx, sx, qW, sW, bias, out, acc_out, stream):
    M, N, K, out = _linear_operands(qx, sx, qW, sW, bias, out, acc_out)
    _check(getattr(lib(), name)(_ptr(qx), _ptr(sx), _ptr(qW), _ptr(sW), _ptr(bias), M, N, K,
                                _ptr(out), out.stride(0), _ptr(acc_out), _stream(stream)), name)
    return out


def sdnq_int8_linear(qx, sx, qW, sW, bias=None, out=None, acc_out=None, stream=None):
    """out [M, N] bf16 = bf16(float(qx qW^T) * (sx sW^T) + bias)."""
    return _linear_call("sdnq_int8_linear", qx, sx, qW, sW, bias, out, acc_out, stream)


def sdnq_rotquant_fp8(x, group: int, q=None, s=None, stream=None):
    """Rows of x [M, K] bf16 -> (e4m3 codes uint8 [M, K], fp32 scales [M]), rotated."""
    _req(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device) if q is None else q
    s = torch.empty((M,), dtype=torch.float32, device=x.device) if s is None else s
    _mat(q, torch.uint8, M, K, "q", dense=True)
    _vec(s, torch.float32, M, "s")
    _check(lib().sdnq_rotquant_fp8(_ptr(x), M, K, x.stride(0), group, _ptr(q), _ptr(s),
                                   _stream(stream)), "sdnq_rotquant_fp8")
    return q, s


def sdnq_fp8_linear(qx, sx, qW, sW, bias=None, out=None, acc_out=None, stream=None):
    """out [M, N] bf16 from e4m3 codes qx [M, K], qW [N, K] (uint8) and their scales."""
    M, N, K, out = _linear_operands(qx, sx, qW, sW, bias, out, acc_out, torch.uint8,
                                    torch.float32)
    _check(lib().sdnq_fp8_linear(_ptr(qx), _ptr(sx), _ptr(qW), _ptr(sW), _ptr(bias), M, N, K,
                                 _ptr(out), out.stride(0), _ptr(acc_out), _stream(stream)),
           "sdnq_fp8_linear")
    return out


def attention_workspace(B: int, Lq: int, Lk: int, H: int, D: int):
    """(total bytes, offsets of: Q codes, K codes, Q scales, K scales, mu, scratch)."""
    off = (ctypes.c_int64 * 6)()
    total = lib().sdnq_attention_workspace(B, Lq, Lk, H, D, ctypes.cast(off, _P))
    if total < 0:
        raise ValueError("bad attention shape")
    return int(total), [int(x) for x in off]


def sdnq_attention_int8qk(q, k, v, group: int = 256, scale: float | None = None,
                          smooth_k: bool = True, ws=None, out=None, stream=None):
    """o [B, Lq, H, D] bf16: attention with Hadamard-rotated int8 QK^T and a bf16 PV. ``ws``
    (uint8, attention_workspace bytes) receives the codes, scales and key means."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _req(t, torch.bfloat16, n, 4)
        _dense(t, n)
    B, Lq, H, D = q.shape
    Lk = k.shape[1]
    if k.shape != (B, Lk, H, D) or v.shape != k.shape:
        raise ValueError("q, k, v shapes disagree")
    total, _ = attention_workspace(B, Lq, Lk, H, D)
    ws = torch.empty(total, dtype=torch.uint8, device=q.device) if ws is None else ws
    _vec(ws, torch.uint8, total, "ws")
    out = torch.empty_like(q) if out is None else out
    _req(out, torch.bfloat16, "out", 4)
    _dense(out, "out")
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    scale = float(1.0 / math.sqrt(D)) if scale is None else float(scale)
    _check(lib().sdnq_attention_int8qk(_ptr(q), _ptr(k), _ptr(v), B, Lq, Lk, H, D, group, scale,
                                       1 if smooth_k else 0, _ptr(ws), ws.numel(), _ptr(out),
                                       _stream(stream)), "sdnq_attention_int8qk")
    return out


def sdnq_attention_prep(q, k, group: int = 256, smooth_k: bool = True, ws=None, stream=None):
    """The preparation half: smooth_k means and Q / K codes and scales into ``ws``."""
    for t, n in ((q, "q"), (k, "k")):
        _req(t, torch.bfloat16, n, 4)
        _dense(t, n)
    B, Lq, H, D = q.shape
    Lk = k.shape[1]
    if k.shape[0] != B or k.shape[2:] != q.shape[2:]:
        raise ValueError("q and k shapes disagree")
    total, _ = attention_workspace(B, Lq, Lk, H, D)
    ws = torch.empty(total, dtype=torch.uint8, device=q.device) if ws is None else ws
    _vec(ws, torch.uint8, total, "ws")
    _check(lib().sdnq_attention_prep(_ptr(q), _ptr(k), B, Lq, Lk, H, D, group,
                                     1 if smooth_k else 0, _ptr(ws), ws.numel(), _stream(stream)),
           "sdnq_attention_prep")
    return ws


def sdnq_attention_core(v, Lq: int, ws, scale: float | None = None, out=None, stream=None):
    """The attention kernel on a prepared ``ws``: o [B, Lq, H, D] bf16."""
    _req(v, torch.bfloat16, "v", 4)
    _dense(v, "v")
    B, Lk, H, D = v.shape
    total, _ = attention_workspace(B, Lq, Lk, H, D)
    _vec(ws, torch.uint8, total, "ws")
    out = torch.empty((B, Lq, H, D), dtype=torch.bfloat16, device=v.device) if out is None else out
    _req(out, torch.bfloat16, "out", 4)
    _dense(out, "out")
    if tuple(out.shape) != (B, Lq, H, D):
        raise ValueError(f"out: expected shape {(B, Lq, H, D)}")
    scale = float(1.0 / math.sqrt(D)) if scale is None else float(scale)
    _check(lib().sdnq_attention_core(_ptr(v), B, Lq, Lk, H, D, scale, _ptr(ws), ws.numel(),
                                     _ptr(out), _stream(stream)), "sdnq_attention_core")
    return out


def fused_sync_words(M: int) -> int:
    return 2 * ((M + 127) // 128)


_SYNC_CACHE = {}


def _sync_buffer(device, stream_handle: int, M: int):
    """A zeroed counter buffer for sdnq_int8_linear_fused, one per (device, stream); the
    kernel leaves it zero after every successful call, so it is reused as it is."""
    key = (device.index, stream_handle)
    need = fused_sync_words(M)
    buf = _SYNC_CACHE.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.zeros(max(need, 256), dtype=torch.int32, device=device)
        _SYNC_CACHE[key] = buf
    return buf


FUSE_AUTO, FUSE_ALWAYS, FUSE_NEVER = 0, 1, 2


def sdnq_int8_linear_fused(x, group: int, qW, sW, bias=None, qx_ws=None, sx_ws=None,
                           sync_ws=None, out=None, acc_out=None, policy: int = FUSE_AUTO,
                           stream=None):
    """out [M, N] bf16 = the rotated int8 linear of x [M, K] bf16, in one launch (activation
    quantizer inside the GEMM kernel) when ``policy`` and the shape call for it, else in two.
    qx_ws / sx_ws receive the activation codes and scales."""
    _req(x, torch.bfloat16, "x", 2)
    _req(qW, torch.int8, "qW", 2)
    _dense(qW, "qW")
    M, K = x.shape
    N = qW.shape[0]
    if qW.shape[1] != K:
        raise ValueError("x and qW disagree on K")
    dev = x.device
    qx_ws = torch.empty((M, K), dtype=torch.int8, device=dev) if qx_ws is None else qx_ws
    sx_ws = torch.empty((M,), dtype=torch.float32, device=dev) if sx_ws is None else sx_ws
    _, _, _, out = _linear_operands(qx_ws, sx_ws, qW, sW, bias, out, acc_out)
    if sync_ws is not None:
        _vec(sync_ws, torch.int32, fused_sync_words(M), "sync_ws")
    st = _stream(stream)
    if sync_ws is None:
        sync_ws = _sync_buffer(dev, st.value or 0, M)
    _check(lib().sdnq_int8_linear_fused(_ptr(x), x.stride(0), group, _ptr(qW), _ptr(sW),
                                        _ptr(bias), M, N, K, _ptr(qx_ws), _ptr(sx_ws),
                                        _ptr(sync_ws), _ptr(out), out.stride(0), _ptr(acc_out),
                                        int(policy), st), "sdnq_int8_linear_fused")
    return out


def sdnq_int8_linear_fused_plan(M: int, N: int, K: int, policy: int = FUSE_AUTO) -> bool:
    """True if sdnq_int8_linear_fused takes one launch for these sizes on the current
    device, False for the two launches (the library's own rule; nothing is launched)."""
    one = ctypes.c_int32(0)
    _check(lib().sdnq_int8_linear_fused_plan(M, N, K, int(policy), ctypes.byref(one)),
           "sdnq_int8_linear_fused_plan")
    return bool(one.value)


def sdnq_int8_linear_gelu(qx, sx, qW, sW, bias=None, out=None, acc_out=None, stream=None):
    """out [M, N] bf16 = GELU of sdnq_int8_linear's output, rounded once more to bf16."""
    return _linear_call("sdnq_int8_linear_gelu", qx, sx, qW, sW, bias, out, acc_out, stream)


def sdnq_int8_linear_grad_input(dy, qW, sW, group: int, qg_ws=None, sg_ws=None, out=None,
                                acc_out=None, stream=None):
    """dx [M, K] bf16 of the frozen rotated int8 layer (qW [N, K], sW [N]) for output
    gradients dy [M, N] bf16. qg_ws [M, N] int8 / sg_ws [M] fp32 receive the quantized dy * sW."""
    _req(dy, torch.bfloat16, "dy", 2)
    _req(qW, torch.int8, "qW", 2)
    _dense(qW, "qW")
    M, N = dy.shape
    if qW.shape[0] != N:
        raise ValueError("dy and qW disagree on N")
    K = qW.shape[1]
    dev = dy.device
    _vec(sW, torch.float32, N, "sW")
    qg_ws = torch.empty((M, N), dtype=torch.int8, device=dev) if qg_ws is None else qg_ws
    sg_ws = torch.empty((M,), dtype=torch.float32, device=dev) if sg_ws is None else sg_ws
    _mat(qg_ws, torch.int8, M, N, "qg_ws", dense=True)
    _vec(sg_ws, torch.float32, M, "sg_ws")
    out = _rows_out(M, K, torch.bfloat16, dev) if out is None else out
    _mat(out, torch.bfloat16, M, K, "out")
    if acc_out is not None:
        _mat(acc_out, torch.int32, M, K, "acc_out", dense=True)
    _check(lib().sdnq_int8_linear_grad_input(_ptr(dy), dy.stride(0), _ptr(qW), _ptr(sW), M, N, K,
                                             group, _ptr(qg_ws), _ptr(sg_ws), _ptr(out),
                                             out.stride(0), _ptr(acc_out), _stream(stream)),
           "sdnq_int8_linear_grad_input")
    return out


def sdnq_quant_grad_output(dy, sW, qg=None, sg=None, stream=None):
    """(qg [M, N] int8, sg [M] fp32): per-token int8 of fp32(dy) * sW."""
    _req(dy, torch.bfloat16, "dy", 2)
    M, N = dy.shape
    _vec(sW, torch.float32, N, "sW")
    qg = torch.empty((M, N), dtype=torch.int8, device=dy.device) if qg is None else qg
    sg = torch.empty((M,), dtype=torch.float32, device=dy.device) if sg is None else sg
    _mat(qg, torch.int8, M, N, "qg", dense=True)
    _vec(sg, torch.float32, M, "sg")
    _check(lib().sdnq_quant_grad_output(_ptr(dy), dy.stride(0), _ptr(sW), M, N, _ptr(qg),
                                        _ptr(sg), _stream(stream)), "sdnq_quant_grad_output")
    return qg, sg


def sdnq_int8_grad_input_gemm(qg, sg, qW, group: int, out=None, acc_out=None, stream=None):
    """dx [M, K] bf16 from the quantized output gradient (qg, sg) and the layer's codes qW."""
    _req(qg, torch.int8, "qg", 2)
    _req(qW, torch.int8, "qW", 2)
    _dense(qg, "qg")
    _dense(qW, "qW")
    M, N = qg.shape
    if qW.shape[0] != N:
        raise ValueError("qg and qW disagree on N")
    K = qW.shape[1]
    _vec(sg, torch.float32, M, "sg")
    out = _rows_out(M, K, torch.bfloat16, qg.device) if out is None else out
    _mat(out, torch.bfloat16, M, K, "out")
    if acc_out is not None:
        _mat(acc_out, torch.int32, M, K, "acc_out", dense=True)
    _check(lib().sdnq_int8_grad_input_gemm(_ptr(qg), _ptr(sg), _ptr(qW), M, N, K, group,
                                           _ptr(out), out.stride(0), _ptr(acc_out),
                                           _stream(stream)), "sdnq_int8_grad_input_gemm")
    return out


def _lora_operands(qx, sx, qW, sW, bias, x, A, B, out, acc_out):
    """Checks the operands of a LoRA linear call; returns (M, N, K, rank, out)."""
    M, N, K, out = _linear_operands(qx, sx, qW, sW, bias, out, acc_out)
    _req(x, torch.bfloat16, "x", 2)
    if tuple(x.shape) != (M, K):
        raise ValueError(f"x: expected shape {(M, K)}, got {tuple(x.shape)}")
    _req(A, torch.bfloat16, "A", 2)
    _req(B, torch.bfloat16, "B", 2)
    _dense(A, "A")
    _dense(B, "B")
    rank = A.shape[1]
    if A.shape[0] != K or tuple(B.shape) != (rank, N):
        raise ValueError("LoRA shapes disagree: A must be [K, rank] and B [rank, N]")
    return M, N, K, rank, out


def sdnq_int8_linear_lora(qx, sx, qW, sW, bias, x, A, B, lora_scale: float = 1.0, u_ws=None,
                          out=None, acc_out=None, stream=None):
    """As sdnq_int8_linear plus lora_scale * bf16(x A) B; u_ws [M, rank] receives bf16(x A)."""
    M, N, K, rank, out = _lora_operands(qx, sx, qW, sW, bias, x, A, B, out, acc_out)
    u_ws = torch.empty((M, rank), dtype=torch.bfloat16, device=qx.device) if u_ws is None else u_ws
    _mat(u_ws, torch.bfloat16, M, rank, "u_ws", dense=True)
    _check(lib().sdnq_int8_linear_lora(_ptr(qx), _ptr(sx), _ptr(qW), _ptr(sW), _ptr(bias),
                                       _ptr(x), x.stride(0), _ptr(A), _ptr(B), rank,
                                       float(lora_scale), _ptr(u_ws), M, N, K, _ptr(out),
                                       out.stride(0), _ptr(acc_out), _stream(stream)),
           "sdnq_int8_linear_lora")
    return out


def sdnq_lora_down(x, A, u=None, stream=None):
    """u [M, rank] = bf16(x A): the LoRA down-projection of sdnq_int8_linear_lora alone
    (x the unrotated bf16 layer input [M, K], A [K, rank] bf16)."""
    _req(x, torch.bfloat16, "x", 2)
    _req(A, torch.bfloat16, "A", 2)
    _dense(A, "A")
    M, K = x.shape
    if A.shape[0] != K:
        raise ValueError(f"A: expected {K} rows, got {A.shape[0]}")
    rank = A.shape[1]
    u = torch.empty((M, rank), dtype=torch.bfloat16, device=x.device) if u is None else u
    _mat(u, torch.bfloat16, M, rank, "u", dense=True)
    _check(lib().sdnq_lora_down(_ptr(x), x.stride(0), _ptr(A), rank, M, K, _ptr(u),
                                _stream(stream)), "sdnq_lora_down")
    return u


def sdnq_int8_linear_lora_up(qx, sx, qW, sW, bias, u, B, lora_scale: float = 1.0, out=None,
                             acc_out=None, stream=None):
    """sdnq_int8_linear plus lora_scale * u B from a given u [M, rank] (as written by
    sdnq_lora_down); B [rank, N] bf16."""
    M, N, K, out = _linear_operands(qx, sx, qW, sW, bias, out, acc_out)
    _req(B, torch.bfloat16, "B", 2)
    _dense(B, "B")
    rank = B.shape[0]
    if B.shape[1] != N:
        raise ValueError(f"B: expected shape {(rank, N)}, got {tuple(B.shape)}")
    _mat(u, torch.bfloat16, M, rank, "u", dense=True)
    _check(lib().sdnq_int8_linear_lora_up(_ptr(qx), _ptr(sx), _ptr(qW), _ptr(sW), _ptr(bias),
                                          _ptr(u), _ptr(B), rank, float(lora_scale), M, N, K,
                                          _ptr(out), out.stride(0), _ptr(acc_out),
                                          _stream(stream)), "sdnq_int8_linear_lora_up")
    return out


NOALLOC_MAX_U_ELEMS = 1 << 22


def sdnq_int8_linear_lora_noalloc(qx, sx, qW, sW, bias, x, A, B, lora_scale: float = 1.0,
                                  out=None, acc_out=None, stream=None):
    """sdnq_int8_linear_lora for callers that cannot provide device memory for the u
    workspace: u lives in a fixed 8 MiB array inside the library (M * rank must not exceed
    NOALLOC_MAX_U_ELEMS). Calls that overlap on the GPU share that array and race."""
    M, N, K, rank, out = _lora_operands(qx, sx, qW, sW, bias, x, A, B, out, acc_out)
    if M * rank > NOALLOC_MAX_U_ELEMS:
        raise ValueError(f"M * rank = {M * rank} exceeds the library's fixed scratch of "
                         f"{NOALLOC_MAX_U_ELEMS} values; use sdnq_int8_linear_lora with u_ws")
    _check(lib().sdnq_int8_linear_lora_noalloc(_ptr(qx), _ptr(sx), _ptr(qW), _ptr(sW),
                                               _ptr(bias), _ptr(x), x.stride(0), _ptr(A),
                                               _ptr(B), rank, float(lora_scale), M, N, K,
                                               _ptr(out), out.stride(0), _ptr(acc_out),
                                               _stream(stream)),
           "sdnq_int8_linear_lora_noalloc")
    return out


def sdnq_gelu_bf16(x: torch.Tensor, out=None, stream=None):
    """Exact-erf GELU, bf16 -> bf16 (the MLP glue between up and down projections)."""
    _req(x, torch.bfloat16, "x", 2)
    M, N = x.shape
    out = _rows_out(M, N, torch.bfloat16, x.device) if out is None else out
    _mat(out, torch.bfloat16, M, N, "out")
    _check(lib().sdnq_gelu_bf16(_ptr(x), M, N, x.stride(0), _ptr(out), out.stride(0),
                                _stream(stream)), "sdnq_gelu_bf16")
    return out


def sdnq_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word status."""
    return lib().sdnq_device_status(_stream(stream))


def sdnq_selftest_wait_timeout(limit_ns: int, stream=None):
    _check(lib().sdnq_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "sdnq_selftest_wait_timeout")
