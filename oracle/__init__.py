"""Plain CPU oracle for block-quantized dequantize + GEMV (numpy wrapper).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``dequant_gemv_q4_b200`` and its CUDA library) never imports, links or falls
back to it, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one weight at
a time); this module only compiles it with the system C compiler, loads it with
ctypes and marshals numpy arrays.  Definitions and citations are in the C file.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

Q8_0_BLOCK_ELEMS = 32
Q8_0_BLOCK_BYTES = 34
Q4K_BLOCK_ELEMS = 256
Q4K_BLOCK_BYTES = 144


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` (IEEE semantics, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, p = ctypes.c_int64, ctypes.c_void_p
            lib.oracle_fp16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_fp16_to_double.restype = ctypes.c_double
            lib.oracle_q4k_scale_min.argtypes = [p, ctypes.c_int, p, p]
            lib.oracle_q4k_scale_min.restype = None
            lib.oracle_q4k_quant.argtypes = [p, ctypes.c_int]
            lib.oracle_q4k_quant.restype = ctypes.c_int
            lib.oracle_q4k_block.argtypes = [p, p]
            lib.oracle_q4k_block.restype = None
            lib.oracle_q8_0_block.argtypes = [p, p]
            lib.oracle_q8_0_block.restype = None
            lib.oracle_q4k_repack_soa.argtypes = [p, i64, i64, p]
            lib.oracle_q8_0_dequant.argtypes = [p, i64, i64, p]
            lib.oracle_q4k_dequant.argtypes = [p, ctypes.c_int, i64, i64, p]
            lib.oracle_q4k_dequant_f32.argtypes = [p, ctypes.c_int, i64, i64, p]
            lib.oracle_q8_0_dequant_f32.argtypes = [p, i64, i64, p]
            lib.oracle_q4k_gemv_rows.argtypes = [p, ctypes.c_int, i64, i64, p, ctypes.c_int,
                                                 p, i64, p, p]
            lib.oracle_q8_0_gemv_rows.argtypes = [p, i64, i64, p, ctypes.c_int, p, i64, p, p]
            lib.oracle_swiglu.argtypes = [p, p, i64, p]
            lib.oracle_swiglu.restype = None
            lib.oracle_argmax.argtypes = [p, i64]
            lib.oracle_split_qg.argtypes = [p, i64, i64, i64, p, p]
            lib.oracle_argmax.restype = i64
            lib.oracle_float_to_fp16.argtypes = [ctypes.c_float]
            lib.oracle_float_to_fp16.restype = ctypes.c_uint16
            lib.oracle_float_to_fp16_array.argtypes = [p, i64, p]
            lib.oracle_float_to_fp16_array.restype = None
            lib.oracle_q4k_dequant_f16.argtypes = [p, ctypes.c_int, i64, i64, p]
            lib.oracle_q4k_prefill_rows.argtypes = [p, ctypes.c_int, i64, i64, p, i64, p, i64,
                                                    p, p]
            for name in ("oracle_q4k_repack_soa", "oracle_q8_0_dequant", "oracle_q4k_dequant",
                         "oracle_q4k_dequant_f32", "oracle_q8_0_dequant_f32",
                         "oracle_q4k_gemv_rows", "oracle_q8_0_gemv_rows", "oracle_split_qg",
                         "oracle_q4k_dequant_f16", "oracle_q4k_prefill_rows"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _u8(w) -> np.ndarray:
    w = np.ascontiguousarray(w)
    if w.dtype != np.uint8:
        raise TypeError("weight bytes must be uint8")
    return w


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError("oracle %s rejected its arguments (code %d)" % (what, rc))


def _layout_flag(layout: str) -> int:
    if layout not in ("aos", "soa"):
        raise ValueError("layout must be 'aos' or 'soa'")
    return 1 if layout == "soa" else 0


# --- element decoders -------------------------------------------------------

def fp16_to_double(h: int) -> float:
    """IEEE binary16 bit pattern -> exact double."""
    return _load().oracle_fp16_to_double(int(h))


def q4k_scale_min(scales12) -> tuple[list[int], list[int]]:
    """The 8 (scale, min) six-bit pairs packed in 12 scale bytes."""
    s = _u8(np.asarray(scales12, dtype=np.uint8).reshape(12))
    sc = ctypes.c_int()
    mn = ctypes.c_int()
    out_s, out_m = [], []
    for j in range(8):
        _load().oracle_q4k_scale_min(_ptr(s), j, ctypes.byref(sc), ctypes.byref(mn))
        out_s.append(sc.value)
        out_m.append(mn.value)
    return out_s, out_m


def q4k_quant(qs128, i: int) -> int:
    """Quant i (0..255) of a super-block's 128 quant bytes."""
    qs = _u8(np.asarray(qs128, dtype=np.uint8).reshape(128))
    return _load().oracle_q4k_quant(_ptr(qs), int(i))


def q4k_block(block144) -> np.ndarray:
    b = _u8(np.asarray(block144, dtype=np.uint8).reshape(Q4K_BLOCK_BYTES))
    out = np.empty(Q4K_BLOCK_ELEMS, np.float64)
    _load().oracle_q4k_block(_ptr(b), _ptr(out))
    return out


def q8_0_block(block34) -> np.ndarray:
    b = _u8(np.asarray(block34, dtype=np.uint8).reshape(Q8_0_BLOCK_BYTES))
    out = np.empty(Q8_0_BLOCK_ELEMS, np.float64)
    _load().oracle_q8_0_block(_ptr(b), _ptr(out))
    return out


# --- whole matrices ---------------------------------------------------------

def q8_0_dequant(w, N: int, K: int) -> np.ndarray:
    w = _u8(w)
    out = np.empty((N, K), np.float64)
    _check(_load().oracle_q8_0_dequant(_ptr(w), N, K, _ptr(out)), "q8_0_dequant")
    return out


def q8_0_dequant_f32(w, N: int, K: int) -> np.ndarray:
    w = _u8(w)
    out = np.empty((N, K), np.float32)
    _check(_load().oracle_q8_0_dequant_f32(_ptr(w), N, K, _ptr(out)), "q8_0_dequant_f32")
    return out


def q4k_dequant(w, N: int, K: int, layout: str = "aos") -> np.ndarray:
    w = _u8(w)
    out = np.empty((N, K), np.float64)
    _check(_load().oracle_q4k_dequant(_ptr(w), _layout_flag(layout), N, K, _ptr(out)),
           "q4k_dequant")
    return out


def q4k_dequant_f32(w, N: int, K: int, layout: str = "aos") -> np.ndarray:
    w = _u8(w)
    out = np.empty((N, K), np.float32)
    _check(_load().oracle_q4k_dequant_f32(_ptr(w), _layout_flag(layout), N, K, _ptr(out)),
           "q4k_dequant_f32")
    return out


def q4k_repack_soa(w, N: int, K: int) -> np.ndarray:
    w = _u8(w)
    out = np.empty_like(w)
    _check(_load().oracle_q4k_repack_soa(_ptr(w), N, K, _ptr(out)), "q4k_repack_soa")
    return out


def _rows_arg(rows, N):
    if rows is None:
        rows = np.arange(N, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))


def _x_arg(x, K):
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if x.ndim == 1:
        x = x.reshape(1, -1)
    if x.shape[1] != K:
        raise ValueError("x must have K columns")
    return x


def q4k_gemv(w, N: int, K: int, x, rows=None, layout: str = "aos"):
    """y, A for the listed rows (default: all), each of shape (B, nrows), float64."""
    w = _u8(w)
    x = _x_arg(x, K)
    rows = _rows_arg(rows, N)
    B = x.shape[0]
    y = np.empty((B, rows.size), np.float64)
    a = np.empty((B, rows.size), np.float64)
    _check(_load().oracle_q4k_gemv_rows(_ptr(w), _layout_flag(layout), N, K, _ptr(x), B,
                                        _ptr(rows), rows.size, _ptr(y), _ptr(a)), "q4k_gemv")
    return y, a


def q8_0_gemv(w, N: int, K: int, x, rows=None):
    w = _u8(w)
    x = _x_arg(x, K)
    rows = _rows_arg(rows, N)
    B = x.shape[0]
    y = np.empty((B, rows.size), np.float64)
    a = np.empty((B, rows.size), np.float64)
    _check(_load().oracle_q8_0_gemv_rows(_ptr(w), N, K, _ptr(x), B, _ptr(rows), rows.size,
                                         _ptr(y), _ptr(a)), "q8_0_gemv")
    return y, a


def swiglu(g, u) -> np.ndarray:
    g = np.ascontiguousarray(np.asarray(g, dtype=np.float64))
    u = np.ascontiguousarray(np.asarray(u, dtype=np.float64))
    if g.shape != u.shape:
        raise ValueError("g and u must have the same shape")
    out = np.empty_like(g)
    _load().oracle_swiglu(_ptr(g), _ptr(u), g.size, _ptr(out))
    return out


def argmax(v) -> int:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float64).reshape(-1))
    return int(_load().oracle_argmax(_ptr(v), v.size))


def split_qg(y, head_dim: int):
    """De-interleave a q-projection-with-gate output (B x N, per head head_dim Q
    values then head_dim gate values) into contiguous Q and G (B x N/2 each);
    Doppler 0.1.8, split_qg.wgsl."""
    y = np.ascontiguousarray(np.asarray(y, dtype=np.float64))
    y2 = y.reshape(-1, y.shape[-1])
    B, N = y2.shape
    q = np.empty((B, N // 2), np.float64)
    g = np.empty((B, N // 2), np.float64)
    _check(_load().oracle_split_qg(_ptr(y2), B, N, head_dim, _ptr(q), _ptr(g)), "split_qg")
    return q, g


# --- W4A16 prefill ------------------------------------------------------------

def float_to_fp16(f) -> np.ndarray:
    """fp32 values -> binary16 bit patterns (uint16), round to nearest even."""
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float32))
    out = np.empty(f.shape, np.uint16)
    _load().oracle_float_to_fp16_array(_ptr(f), f.size, _ptr(out))
    return out


def q4k_dequant_f16(w, N: int, K: int, layout: str = "aos") -> np.ndarray:
    """N x K binary16 bit patterns of the weights rounded to fp32, then to fp16."""
    w = _u8(w)
    out = np.empty((N, K), np.uint16)
    _check(_load().oracle_q4k_dequant_f16(_ptr(w), _layout_flag(layout), N, K, _ptr(out)),
           "q4k_dequant_f16")
    return out


def q4k_prefill(w, N: int, K: int, x16, rows=None, layout: str = "aos"):
    """W4A16 prefill: y, A (each M x nrows, float64) for x16 an M x K array of
    binary16 bit patterns (uint16) or of float16 values; qualiaDB
    qwen3_attention, prefill_weights (W4A16 M128 dispatcher)."""
    w = _u8(w)
    x16 = np.asarray(x16)
    if x16.dtype == np.float16:
        x16 = x16.view(np.uint16)
    if x16.dtype != np.uint16:
        raise TypeError("x16 must hold binary16 bit patterns (uint16) or float16 values")
    x16 = np.ascontiguousarray(x16)
    if x16.ndim == 1:
        x16 = x16.reshape(1, -1)
    if x16.shape[1] != K:
        raise ValueError("x16 must have K columns")
    rows = _rows_arg(rows, N)
    M = x16.shape[0]
    y = np.empty((M, rows.size), np.float64)
    a = np.empty((M, rows.size), np.float64)
    _check(_load().oracle_q4k_prefill_rows(_ptr(w), _layout_flag(layout), N, K, _ptr(x16), M,
                                           _ptr(rows), rows.size, _ptr(y), _ptr(a)),
           "q4k_prefill")
    return y, a


# --- tolerance rules ----------------------------------------------------------

def gemv_tolerance(a):
    """Allowed |y_gpu - y_ref| for a GEMV output: 1e-4 * sum|w*x| + 1e-6."""
    return 1e-4 * np.asarray(a, dtype=np.float64) + 1e-6


def swiglu_tolerance(g, u, a_g, a_u):
    """Allowed |out_gpu - out_ref| for silu(g)*u, propagated from the GEMV rule.

    |d silu/dg| <= 1.0998 everywhere, so an error tol_g in g moves silu(g) by
    at most 1.1*tol_g; the error tol_u in u is scaled by |silu(g)|.  The second
    order term tol_g*tol_u is covered by the constant slack.
    """
    g = np.asarray(g, dtype=np.float64)
    u = np.asarray(u, dtype=np.float64)
    tg = gemv_tolerance(a_g)
    tu = gemv_tolerance(a_u)
    silu = g / (1.0 + np.exp(-g))
    # the last relative term covers the fp32 rounding of silu and of the product
    return 1.1 * np.abs(u) * tg + np.abs(silu) * tu + 1.1 * tg * tu + 1e-6 \
        + 1e-6 * np.abs(silu * u)
