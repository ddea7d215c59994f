"""CPU oracle for the Hadamard-rotated ("ConvRot") INT8 linear layer.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package. The product path (the CUDA library and its
Python binding) never imports, links or runs anything here, and this package imports
nothing from the product.

The arithmetic lives in ``oracle.c`` (plain C, fp contraction off); this module only
builds it with gcc, loads it with ctypes and marshals numpy arrays. bf16 values travel as
their raw 16-bit patterns in ``numpy.uint16`` arrays.

Every function follows the readings stated in ``oracle.c``'s header, with the pages cited
there ("ConvRot / Hadamard SDNQ", "SDNQ: SD.Next Quantization Engine",
"Hybrid-Sensitivity-Weighted-Quantization").

Parity status: every function here is pinned by tests in ``tests/test_oracle_pins.py``
except the summation order of the LoRA terms, which is pinned only to within the
fp64-sum bound (see ``lora_down`` / ``lora_up``).
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-shared", "-fPIC"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (gcc) unless it is up to date."""
    with _lock:
        stale = (not os.path.exists(_LIB)
                 or os.path.getmtime(_LIB) < os.path.getmtime(_SRC))
        if force or stale:
            tmp = _LIB + f".tmp{os.getpid()}"
            subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
            os.replace(tmp, _LIB)
    return _LIB


def _open(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    INT = ctypes.c_int
    F = ctypes.c_float
    sig = {
        "oracle_bf16_to_f32": [P, I64, P],
        "oracle_f32_to_bf16": [P, I64, P],
        "oracle_f64_to_bf16": [P, I64, P],
        "oracle_fwht_f32": [P, I64, I64],
        "oracle_fwht_f64": [P, I64, I64],
        "oracle_rotate_quantize": [P, I64, I64, I64, I64, P, P, INT],
        "oracle_gemm_s8": [P, P, I64, I64, I64, P, INT],
        "oracle_dequant_epilogue": [P, P, P, P, P, F, I64, I64, P, INT],
        "oracle_lora_down": [P, I64, I64, I64, P, I64, P, INT],
        "oracle_lora_up": [P, P, I64, I64, I64, P, INT],
        "oracle_gelu_bf16": [P, I64, P, INT],
        "oracle_colscale_quantize": [P, I64, I64, I64, P, P, P, INT],
        "oracle_e4m3_encode": [P, I64, P],
        "oracle_attn_prep": [P, P, I64, I64, I64, I64, I64, I64, INT, P, P, P, P, P, INT],
        "oracle_attn_logits": [P, P, P, P, I64, I64, I64, I64, I64, F, P, INT],
        "oracle_attn_softmax_pv": [P, P, I64, I64, I64, I64, I64, P, INT],
        "oracle_e4m3_decode": [P, I64, P],
        "oracle_rotate_quantize_fp8": [P, I64, I64, I64, I64, P, P, INT],
        "oracle_gemm_fp8": [P, P, I64, I64, I64, P, INT],
        "oracle_dequant_epilogue_f32": [P, P, P, P, I64, I64, P, INT],
        "oracle_gemm_s8_nn": [P, P, I64, I64, I64, P, INT],
        "oracle_grad_input_epilogue": [P, P, I64, I64, I64, P, INT],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = None if name in ("oracle_bf16_to_f32", "oracle_f32_to_bf16",
                                      "oracle_f64_to_bf16", "oracle_e4m3_encode",
                                      "oracle_e4m3_decode") else ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _open(_LIB)
    return _lib


@contextlib.contextmanager
def built_from(source_text: str, workdir: str):
    """Test hook: run this wrapper against a build of another version of ``oracle.c``
    (used to plant a mistake in the oracle and check that the pins catch it)."""
    global _lib
    src = os.path.join(workdir, "oracle_variant.c")
    so = os.path.join(workdir, "liboracle_variant.so")
    with open(src, "w") as f:
        f.write(source_text)
    subprocess.run(["gcc", *_CFLAGS, src, "-o", so, "-lm"], check=True)
    saved = _lib
    _lib = _open(so)
    try:
        yield
    finally:
        _lib = saved


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: oracle returned error {rc}")


def default_threads() -> int:
    return os.cpu_count() or 1


# ---- number formats ---------------------------------------------------------------

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, np.float32)
    _load().oracle_bf16_to_f32(_ptr(bits), bits.size, _ptr(out))
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().oracle_f64_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


# ---- the method ---------------------------------------------------------------------

def fwht_f32(v: np.ndarray, g: int) -> np.ndarray:
    """Unnormalised block-diagonal Walsh-Hadamard butterfly (fp32, ascending stages)
    along the last axis, in groups of ``g``. Returns a new array."""
    out = np.array(v, dtype=np.float32, copy=True, order="C")
    _check(_load().oracle_fwht_f32(_ptr(out), out.size, g), "fwht_f32")
    return out


def fwht_f64(v: np.ndarray, g: int) -> np.ndarray:
    """The same butterfly in fp64 (quality reports and pins only)."""
    out = np.array(v, dtype=np.float64, copy=True, order="C")
    _check(_load().oracle_fwht_f64(_ptr(out), out.size, g), "fwht_f64")
    return out


def rotate_quantize(x_bits: np.ndarray, g: int, nthreads: int | None = None):
    """Rotate each row by the block-diagonal H_g and quantize it to int8 with one fp32
    scale per row. ``x_bits``: bf16 patterns [rows, K]. Returns (codes int8 [rows, K],
    scales fp32 [rows])."""
    x_bits = _c(x_bits, np.uint16)
    rows, K = x_bits.shape
    q = np.empty((rows, K), np.int8)
    s = np.empty((rows,), np.float32)
    rc = _load().oracle_rotate_quantize(_ptr(x_bits), rows, K, K, g, _ptr(q), _ptr(s),
                                        nthreads or default_threads())
    _check(rc, "rotate_quantize")
    return q, s


def gemm_s8(a: np.ndarray, b: np.ndarray, nthreads: int | None = None) -> np.ndarray:
    """acc[m, n] = sum_k a[m, k] * b[n, k] in int32."""
    a = _c(a, np.int8)
    b = _c(b, np.int8)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("K mismatch")
    acc = np.empty((M, N), np.int32)
    _check(_load().oracle_gemm_s8(_ptr(a), _ptr(b), M, N, K, _ptr(acc),
                                  nthreads or default_threads()), "gemm_s8")
    return acc


def dequant_epilogue(acc, sx, sw, bias_bits=None, L=None, lora_scale=1.0,
                     nthreads: int | None = None) -> np.ndarray:
    """fp32 de-quant epilogue; returns bf16 patterns [M, N]."""
    acc = _c(acc, np.int32)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    M, N = acc.shape
    out = np.empty((M, N), np.uint16)
    bias_p = None
    L_p = None
    if bias_bits is not None:
        bias_bits = _c(bias_bits, np.uint16)
        bias_p = _ptr(bias_bits)
    if L is not None:
        L = _c(L, np.float32)
        L_p = _ptr(L)
    rc = _load().oracle_dequant_epilogue(_ptr(acc), _ptr(sx), _ptr(sw), bias_p, L_p,
                                         float(lora_scale), M, N, _ptr(out),
                                         nthreads or default_threads())
    _check(rc, "dequant_epilogue")
    return out


def lora_down(x_bits, A_bits, nthreads: int | None = None) -> np.ndarray:
    """u = bf16(x @ A), fp64 sums. x [M, K], A [K, r] bf16 patterns -> u [M, r]."""
    x_bits = _c(x_bits, np.uint16)
    A_bits = _c(A_bits, np.uint16)
    M, K = x_bits.shape
    K2, r = A_bits.shape
    if K != K2:
        raise ValueError("K mismatch")
    u = np.empty((M, r), np.uint16)
    _check(_load().oracle_lora_down(_ptr(x_bits), M, K, K, _ptr(A_bits), r, _ptr(u),
                                    nthreads or default_threads()), "lora_down")
    return u


def lora_up(u_bits, B_bits, nthreads: int | None = None) -> np.ndarray:
    """L = fp32(u @ B), fp64 sums. u [M, r], B [r, N] bf16 patterns -> fp32 [M, N]."""
    u_bits = _c(u_bits, np.uint16)
    B_bits = _c(B_bits, np.uint16)
    M, r = u_bits.shape
    r2, N = B_bits.shape
    if r != r2:
        raise ValueError("rank mismatch")
    L = np.empty((M, N), np.float32)
    _check(_load().oracle_lora_up(_ptr(u_bits), _ptr(B_bits), M, N, r, _ptr(L),
                                  nthreads or default_threads()), "lora_up")
    return L


def gelu_bf16(x_bits, nthreads: int | None = None) -> np.ndarray:
    """Exact-erf GELU in fp64, rounded once to bf16."""
    x_bits = _c(x_bits, np.uint16)
    out = np.empty(x_bits.shape, np.uint16)
    _check(_load().oracle_gelu_bf16(_ptr(x_bits), x_bits.size, _ptr(out),
                                    nthreads or default_threads()), "gelu_bf16")
    return out


def linear(x_bits, qw, sw, g, bias_bits=None, A_bits=None, B_bits=None, lora_scale=1.0,
           nthreads: int | None = None):
    """Whole quantized linear for the rows given: rotate+quantize x, int8 GEMM against the
    (already rotated and quantized) weight codes, fp32 epilogue, optional LoRA.
    Returns a dict with every intermediate."""
    qx, sx = rotate_quantize(x_bits, g, nthreads)
    acc = gemm_s8(qx, qw, nthreads)
    res = {"qx": qx, "sx": sx, "acc": acc}
    L = None
    if A_bits is not None:
        u = lora_down(x_bits, A_bits, nthreads)
        L = lora_up(u, B_bits, nthreads)
        res["u"] = u
        res["L"] = L
    res["out"] = dequant_epilogue(acc, sx, sw, bias_bits, L, lora_scale, nthreads)
    return res


# ---- input gradient through the frozen rotated base ----------------------------------

def colscale_quantize(dy_bits, sw, nthreads: int | None = None):
    """Per-row int8 quantization of dy * sw (sw [N] multiplies column n). Returns (codes
    int8 [rows, N], scales fp32 [rows])."""
    dy_bits = _c(dy_bits, np.uint16)
    sw = _c(sw, np.float32)
    rows, N = dy_bits.shape
    if sw.shape != (N,):
        raise ValueError("sw must have one scale per column")
    q = np.empty((rows, N), np.int8)
    s = np.empty((rows,), np.float32)
    _check(_load().oracle_colscale_quantize(_ptr(dy_bits), rows, N, N, _ptr(sw), _ptr(q),
                                            _ptr(s), nthreads or default_threads()),
           "colscale_quantize")
    return q, s


def gemm_s8_nn(a, b, nthreads: int | None = None) -> np.ndarray:
    """acc[m, k] = sum_n a[m, n] * b[n, k] in int32."""
    a = _c(a, np.int8)
    b = _c(b, np.int8)
    M, N = a.shape
    N2, K = b.shape
    if N != N2:
        raise ValueError("N mismatch")
    acc = np.empty((M, K), np.int32)
    _check(_load().oracle_gemm_s8_nn(_ptr(a), _ptr(b), M, N, K, _ptr(acc),
                                     nthreads or default_threads()), "gemm_s8_nn")
    return acc


def grad_input_epilogue(acc, s, g, nthreads: int | None = None) -> np.ndarray:
    """bf16 patterns of fp32(acc * s[m]), rotated back by the butterfly, times 1/sqrt(g)."""
    acc = _c(acc, np.int32)
    s = _c(s, np.float32)
    M, K = acc.shape
    dx = np.empty((M, K), np.uint16)
    _check(_load().oracle_grad_input_epilogue(_ptr(acc), _ptr(s), M, K, g, _ptr(dx),
                                              nthreads or default_threads()),
           "grad_input_epilogue")
    return dx


def grad_input(dy_bits, qw, sw, g, nthreads: int | None = None):
    """dx of the frozen rotated int8 layer for output gradients dy [M, N] (bf16 patterns),
    given its stored codes qw [N, K] and row scales sw [N]. Returns every intermediate."""
    qg, sg = colscale_quantize(dy_bits, sw, nthreads)
    acc = gemm_s8_nn(qg, qw, nthreads)
    return {"qg": qg, "sg": sg, "acc": acc, "dx": grad_input_epilogue(acc, sg, g, nthreads)}


# ---- FP8 (e4m3) variant ----------------------------------------------------------------

def e4m3_encode(x) -> np.ndarray:
    """fp32 values -> e4m3 codes (round to nearest, ties to even, saturating at +-448)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    _load().oracle_e4m3_encode(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float32)
    _load().oracle_e4m3_decode(_ptr(c), c.size, _ptr(out))
    return out


def rotate_quantize_fp8(x_bits, g: int, nthreads: int | None = None):
    """Rotate each row by H_g and quantize it to e4m3 with one fp32 scale per row (absmax
    onto +-448). Returns (codes uint8 [rows, K], scales fp32 [rows])."""
    x_bits = _c(x_bits, np.uint16)
    rows, K = x_bits.shape
    q = np.empty((rows, K), np.uint8)
    s = np.empty((rows,), np.float32)
    _check(_load().oracle_rotate_quantize_fp8(_ptr(x_bits), rows, K, K, g, _ptr(q), _ptr(s),
                                              nthreads or default_threads()),
           "rotate_quantize_fp8")
    return q, s


def gemm_fp8(a, b, nthreads: int | None = None) -> np.ndarray:
    """acc[m, n] = fp32(sum_k dec(a[m, k]) dec(b[n, k])), summed in fp64."""
    a = _c(a, np.uint8)
    b = _c(b, np.uint8)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("K mismatch")
    acc = np.empty((M, N), np.float32)
    _check(_load().oracle_gemm_fp8(_ptr(a), _ptr(b), M, N, K, _ptr(acc),
                                   nthreads or default_threads()), "gemm_fp8")
    return acc


def dequant_epilogue_f32(acc, sx, sw, bias_bits=None, nthreads: int | None = None):
    acc = _c(acc, np.float32)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    M, N = acc.shape
    out = np.empty((M, N), np.uint16)
    bias_p = None
    if bias_bits is not None:
        bias_bits = _c(bias_bits, np.uint16)
        bias_p = _ptr(bias_bits)
    _check(_load().oracle_dequant_epilogue_f32(_ptr(acc), _ptr(sx), _ptr(sw), bias_p, M, N,
                                               _ptr(out), nthreads or default_threads()),
           "dequant_epilogue_f32")
    return out


def linear_fp8(x_bits, qw, sw, g, bias_bits=None, nthreads: int | None = None):
    """The FP8 variant of ``linear``: every intermediate in a dict."""
    qx, sx = rotate_quantize_fp8(x_bits, g, nthreads)
    acc = gemm_fp8(qx, qw, nthreads)
    return {"qx": qx, "sx": sx, "acc": acc,
            "out": dequant_epilogue_f32(acc, sx, sw, bias_bits, nthreads)}


# ---- Hadamard-rotated int8 QK inside attention ----------------------------------------

def attn_prep(q_bits, k_bits, g: int, smooth_k: bool = True, nthreads: int | None = None):
    """q [B, Lq, H, D], k [B, Lk, H, D] bf16 patterns -> dict(qq, sq [B, H, Lq], kq, sk
    [B, H, Lk], mu [B, H, D]): smooth_k means, rotated per-row int8 codes and scales."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    B, Lq, H, D = q_bits.shape
    Lk = k_bits.shape[1]
    out = {"qq": np.empty((B, Lq, H, D), np.int8), "sq": np.empty((B, H, Lq), np.float32),
           "kq": np.empty((B, Lk, H, D), np.int8), "sk": np.empty((B, H, Lk), np.float32),
           "mu": np.empty((B, H, D), np.float32)}
    _check(_load().oracle_attn_prep(_ptr(q_bits), _ptr(k_bits), B, Lq, Lk, H, D, g,
                                    1 if smooth_k else 0, _ptr(out["qq"]), _ptr(out["sq"]),
                                    _ptr(out["kq"]), _ptr(out["sk"]), _ptr(out["mu"]),
                                    nthreads or default_threads()), "attn_prep")
    return out


def attn_logits(prep, scale: float, nthreads: int | None = None) -> np.ndarray:
    B, Lq, H, D = prep["qq"].shape
    Lk = prep["kq"].shape[1]
    logits = np.empty((B, H, Lq, Lk), np.float32)
    _check(_load().oracle_attn_logits(_ptr(prep["qq"]), _ptr(prep["sq"]), _ptr(prep["kq"]),
                                      _ptr(prep["sk"]), B, Lq, Lk, H, D, float(scale),
                                      _ptr(logits), nthreads or default_threads()), "attn_logits")
    return logits


def attn_softmax_pv(logits, v_bits, nthreads: int | None = None) -> np.ndarray:
    logits = _c(logits, np.float32)
    v_bits = _c(v_bits, np.uint16)
    B, H, Lq, Lk = logits.shape
    D = v_bits.shape[3]
    o = np.empty((B, Lq, H, D), np.uint16)
    _check(_load().oracle_attn_softmax_pv(_ptr(logits), _ptr(v_bits), B, Lq, Lk, H, D, _ptr(o),
                                          nthreads or default_threads()), "attn_softmax_pv")
    return o


def attention(q_bits, k_bits, v_bits, g: int = 256, scale: float | None = None,
              smooth_k: bool = True, nthreads: int | None = None):
    """Attention with Hadamard-rotated int8 QK and a bf16 PV; every intermediate in a dict."""
    D = q_bits.shape[3]
    scale = float(np.float32(1.0 / np.sqrt(D))) if scale is None else scale
    res = attn_prep(q_bits, k_bits, g, smooth_k, nthreads)
    res["logits"] = attn_logits(res, scale, nthreads)
    res["o"] = attn_softmax_pv(res["logits"], v_bits, nthreads)
    return res
