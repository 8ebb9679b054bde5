"""B200-native fused dequantize + GEMV for GGML-style Q8_0 / Q4_K weights.

A thin ctypes binding over ``libdqgemv.so`` (C ABI in ``include/dqgemv.h``).
Every function here only checks and marshals arguments (PyTorch supplies the
device memory and the current CUDA stream); all of the computation runs in the
library's sm_100a kernels.  There is no CPU path: if the shared library is
missing or the call fails, a ``DQError`` is raised.

Entry points (same names as the C ABI):
    q4k_gemv, q4k_swiglu_gemv, q8_0_gemv, q4k_repack_soa,
    q4k_dequant, q8_0_dequant, dq_workspace_bytes, dq_device_error
"""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdqgemv.so")

DQ_LAYOUT_AOS = 0
DQ_LAYOUT_SOA = 1
DQ_OP_Q8_0_GEMV = 0
DQ_OP_Q4K_GEMV = 1
DQ_OP_Q4K_SWIGLU = 2
DQ_OP_Q4K_PREFILL = 3
DQ_OP_Q4K_FFN = 4
MAX_PREFILL_M = 65536

Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES = 256, 144
Q8_0_BLOCK_ELEMS, Q8_0_BLOCK_BYTES = 32, 34

EXPORTED = ("q8_0_gemv", "q4k_gemv", "q4k_swiglu_gemv", "q4k_repack_soa", "dq_workspace_bytes",
            "q8_0_dequant", "q4k_dequant", "dq_status_string", "dq_last_cuda_error",
            "dq_device_error", "q4k_gemv_noalloc", "dq_noalloc_scratch_bytes", "q4k_gemv_split_qg",
            "q4k_gemv_group", "q4k_prefill_gemm", "q4k_gemv_residual", "q4k_ffn_block", "dq_test_lost_copy")


class DQError(RuntimeError):
    """A libdqgemv entry point returned an error status."""

    def __init__(self, func, status, cuda_error=0):
        self.status = status
        self.cuda_error = cuda_error
        msg = "%s failed: %s" % (func, status_string(status))
        if cuda_error:
            msg += " (cudaError %d)" % cuda_error
        super().__init__(msg)


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load libdqgemv.so and declare its signatures.  Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(
                "libdqgemv.so not found at %s: build it with "
                "`python -m dequant_gemv_q4_b200.build` (there is no CPU fallback)" % path)
        lib = ctypes.CDLL(path)
        p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "q8_0_gemv": [p, p, p, i64, i64, i32, p, sz, p],
            "q4k_gemv": [p, i32, p, p, i64, i64, i32, p, p, sz, p],
            "q4k_swiglu_gemv": [p, p, i32, p, p, i64, i64, i32, p, sz, p],
            "q4k_repack_soa": [p, p, i64, i64, p],
            "q8_0_dequant": [p, p, i64, i64, p],
            "q4k_dequant": [p, i32, p, i64, i64, p],
            "dq_device_error": [p, i32, p],
            "q4k_gemv_noalloc": [p, i32, p, p, i64, i64, i32, p, p],
            "q4k_gemv_split_qg": [p, i32, p, p, p, i64, i64, i32, i64, p, sz, p],
            "q4k_gemv_group": [i32, p, p, p, i32, p, i64, p, sz, p],
            "q4k_prefill_gemm": [p, i32, p, p, i64, i64, i64, p, sz, p],
            "q4k_gemv_residual": [p, i32, p, p, p, i64, i64, i32, p, p, sz, p],
            "q4k_ffn_block": [p, p, p, i32, p, p, p, i64, i64, i32, p, sz, p],
            "dq_test_lost_copy": [p, p, p, i64, i64, ctypes.c_uint64, p, sz, p],
        }
        for name, args in sigs.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = i32
        lib.dq_workspace_bytes.argtypes = [i32, i64, i64, i32, i32]
        lib.dq_workspace_bytes.restype = sz
        lib.dq_status_string.argtypes = [i32]
        lib.dq_status_string.restype = ctypes.c_char_p
        lib.dq_noalloc_scratch_bytes.argtypes = []
        lib.dq_noalloc_scratch_bytes.restype = sz
        lib.dq_last_cuda_error.argtypes = []
        lib.dq_last_cuda_error.restype = i32
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().dq_status_string(int(status)).decode()


def _check(func: str, status: int) -> None:
    if status != 0:
        raise DQError(func, status, load_library().dq_last_cuda_error())


# --- argument marshalling ----------------------------------------------------------

def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return ctypes.c_void_p(t.data_ptr())


def _weights(w, name, N, K, elems, bytes_):
    torch = _torch()
    ptr = _dev(w, name, torch.uint8)
    need = N * (K // elems) * bytes_
    if w.numel() != need:
        raise ValueError("%s holds %d bytes, an %dx%d matrix needs %d" % (name, w.numel(), N, K, need))
    return ptr


def _x2d(x, K):
    torch = _torch()
    if x.dim() == 1:
        x = x.view(1, -1)
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError("x must be (K,) or (B, K)")
    _dev(x, "x", torch.float32)
    return x


def _layout(layout) -> int:
    if layout in ("aos", DQ_LAYOUT_AOS):
        return DQ_LAYOUT_AOS
    if layout in ("soa", DQ_LAYOUT_SOA):
        return DQ_LAYOUT_SOA
    raise ValueError("layout must be 'aos' or 'soa'")


def _workspace(ws, need, device):
    torch = _torch()
    if need == 0:
        return ctypes.c_void_p(0), 0, None
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    _dev(ws, "workspace", torch.uint8)
    return ctypes.c_void_p(ws.data_ptr()), ws.numel(), ws


def dq_workspace_bytes(op: int, N: int, K: int, B: int, with_argmax: bool = False) -> int:
    """Scratch bytes a GEMV call needs on the current device (see dqgemv.h)."""
    v = load_library().dq_workspace_bytes(int(op), int(N), int(K), int(B), int(bool(with_argmax)))
    if v == ctypes.c_size_t(-1).value:
        raise ValueError("invalid op or shape for dq_workspace_bytes")
    return int(v)


# --- entry points ------------------------------------------------------------------

def q4k_gemv(w, x, N: int, K: int, layout="aos", y=None, argmax: bool = False, workspace=None,
             stream=None):
    """y = W x for a Q4_K matrix W (N x K).  x: (K,) or (B, K) fp32.

    Returns y of shape (B, N) (or (N,) for 1-D x); with ``argmax=True`` returns
    (y, idx) where idx is a 1-element int64 CUDA tensor holding the argmax of y.
    """
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, K)
    B = x2.shape[0]
    wp = _weights(w, "w", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    yp = _dev(y, "y", torch.float32)
    if y.numel() != B * N:
        raise ValueError("y must hold B*N floats")
    idx = None
    ip = ctypes.c_void_p(0)
    if argmax:
        idx = torch.empty(1, dtype=torch.int64, device=x.device)
        ip = ctypes.c_void_p(idx.data_ptr())
    need = dq_workspace_bytes(DQ_OP_Q4K_GEMV, N, K, B, argmax)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    _check("q4k_gemv", lib.q4k_gemv(wp, _layout(layout), ctypes.c_void_p(x2.data_ptr()), yp, N, K, B,
                                    ip, wsp, wsn, _stream(stream)))
    out = y.view(N) if one_d else y.view(B, N)
    return (out, idx) if argmax else out


def q4k_gemv_residual(w, x, residual, N: int, K: int, layout="aos", y=None, argmax: bool = False,
                      workspace=None, stream=None):
    """y = W x + residual (the FFN block's down projection with its residual add);
    residual has y's shape and may be y itself.  Returns as q4k_gemv."""
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, K)
    B = x2.shape[0]
    wp = _weights(w, "w", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    rp = _dev(residual, "residual", torch.float32)
    if residual.numel() != B * N:
        raise ValueError("residual must hold B*N floats")
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    yp = _dev(y, "y", torch.float32)
    if y.numel() != B * N:
        raise ValueError("y must hold B*N floats")
    idx = None
    ip = ctypes.c_void_p(0)
    if argmax:
        idx = torch.empty(1, dtype=torch.int64, device=x.device)
        ip = ctypes.c_void_p(idx.data_ptr())
    need = dq_workspace_bytes(DQ_OP_Q4K_GEMV, N, K, B, argmax)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    _check("q4k_gemv_residual", lib.q4k_gemv_residual(wp, _layout(layout), ctypes.c_void_p(x2.data_ptr()), rp, yp,
                                                      N, K, B, ip, wsp, wsn, _stream(stream)))
    out = y.view(N) if one_d else y.view(B, N)
    return (out, idx) if argmax else out


def q4k_ffn_block(w_gate, w_up, w_down, x, H: int, F: int, residual=None, layout="aos", y=None,
                  workspace=None, stream=None):
    """A decoder layer's FFN block: y = W_down (silu(W_gate x) * (W_up x)) [+ residual].
    x: (H,) or (B, H) fp32; W_gate, W_up: F x H; W_down: H x F.  residual may be x or y."""
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, H)
    B = x2.shape[0]
    gp = _weights(w_gate, "w_gate", F, H, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    up = _weights(w_up, "w_up", F, H, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    dp = _weights(w_down, "w_down", H, F, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    rp = ctypes.c_void_p(0)
    if residual is not None:
        rp = _dev(residual, "residual", torch.float32)
        if residual.numel() != B * H:
            raise ValueError("residual must hold B*H floats")
    if y is None:
        y = torch.empty((B, H), dtype=torch.float32, device=x.device)
    yp = _dev(y, "y", torch.float32)
    if y.numel() != B * H:
        raise ValueError("y must hold B*H floats")
    need = dq_workspace_bytes(DQ_OP_Q4K_FFN, H, F, B)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    _check("q4k_ffn_block", lib.q4k_ffn_block(gp, up, dp, _layout(layout), ctypes.c_void_p(x2.data_ptr()), rp, yp,
                                              H, F, B, wsp, wsn, _stream(stream)))
    return y.view(H) if one_d else y.view(B, H)


def q4k_gemv_noalloc(w, x, N: int, K: int, layout="aos", y=None, argmax: bool = False, stream=None):
    """q4k_gemv through the entry point that allocates nothing.

    For callers that cannot allocate device memory: the library's own fixed
    scratch array (dq_noalloc_scratch_bytes()) replaces the workspace, so only
    y (and the argmax slot, when asked for) are passed.  Calls sharing that
    array must not overlap on the GPU.
    """
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, K)
    B = x2.shape[0]
    wp = _weights(w, "w", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    yp = _dev(y, "y", torch.float32)
    idx = None
    ip = ctypes.c_void_p(0)
    if argmax:
        idx = torch.empty(1, dtype=torch.int64, device=x.device)
        ip = ctypes.c_void_p(idx.data_ptr())
    _check("q4k_gemv_noalloc", lib.q4k_gemv_noalloc(wp, _layout(layout), ctypes.c_void_p(x2.data_ptr()), yp,
                                                    N, K, B, ip, _stream(stream)))
    out = y.view(N) if one_d else y.view(B, N)
    return (out, idx) if argmax else out


def dq_noalloc_scratch_bytes() -> int:
    return int(load_library().dq_noalloc_scratch_bytes())


def q4k_gemv_split_qg(w, x, N: int, K: int, head_dim: int, layout="aos", q=None, g=None, workspace=None,
                      stream=None):
    """y = W x for a q-projection-with-gate matrix, stored de-interleaved:
    per head, head_dim Q rows then head_dim gate rows of y go to Q and G
    (each (B, N/2), or (N/2,) for 1-D x).  Returns (Q, G)."""
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, K)
    B = x2.shape[0]
    wp = _weights(w, "w", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    half = N // 2
    if q is None:
        q = torch.empty((B, half), dtype=torch.float32, device=x.device)
    if g is None:
        g = torch.empty((B, half), dtype=torch.float32, device=x.device)
    qp = _dev(q, "q", torch.float32)
    gp = _dev(g, "g", torch.float32)
    if q.numel() != B * half or g.numel() != B * half:
        raise ValueError("q and g must hold B*N/2 floats each")
    need = dq_workspace_bytes(DQ_OP_Q4K_GEMV, N, K, B)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    _check("q4k_gemv_split_qg", lib.q4k_gemv_split_qg(wp, _layout(layout), ctypes.c_void_p(x2.data_ptr()), qp, gp,
                                                      N, K, B, head_dim, wsp, wsn, _stream(stream)))
    if one_d:
        return q.view(half), g.view(half)
    return q.view(B, half), g.view(B, half)


def q4k_prefill_gemm(w, x16, N: int, K: int, layout="aos", y=None, workspace=None, stream=None):
    """W4A16 prefill: y (M, N) fp32 = x16 (M, K) binary16 times the binary16
    rounding of the Q4_K matrix w (N x K), transposed, on the tensor cores."""
    torch = _torch()
    lib = load_library()
    if x16.dim() != 2 or x16.shape[1] != K:
        raise ValueError("x16 must be (M, K)")
    M = x16.shape[0]
    xp = _dev(x16, "x16", torch.float16)
    wp = _weights(w, "w", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=x16.device)
    yp = _dev(y, "y", torch.float32)
    if y.numel() != M * N:
        raise ValueError("y must hold M*N floats")
    need = dq_workspace_bytes(DQ_OP_Q4K_PREFILL, N, K, M)
    wsp, wsn, _keep = _workspace(workspace, need, x16.device)
    _check("q4k_prefill_gemm", lib.q4k_prefill_gemm(wp, _layout(layout), xp, yp, N, K, M, wsp, wsn,
                                                    _stream(stream)))
    return y.view(M, N)


MAX_GROUP = 4


def q4k_gemv_group(ws, x, Ns, K: int, layout="aos", ys=None, workspace=None, stream=None):
    """Batch-1 GEMVs of up to four Q4_K matrices sharing x, in one launch.

    ws: list of weight tensors (N_m x K each); Ns: their row counts; x: (K,)
    fp32.  Returns the list of outputs (N_m,) (or fills ``ys``)."""
    torch = _torch()
    lib = load_library()
    count = len(ws)
    if not 1 <= count <= MAX_GROUP or len(Ns) != count:
        raise ValueError("1 to %d matrices, one row count each" % MAX_GROUP)
    x2 = _x2d(x, K)
    if x2.shape[0] != 1:
        raise ValueError("a grouped GEMV takes one activation vector")
    wps = [_weights(w, "w[%d]" % m, int(n), K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES) for m, (w, n) in enumerate(zip(ws, Ns))]
    if ys is None:
        ys = [torch.empty(int(n), dtype=torch.float32, device=x.device) for n in Ns]
    yps = [_dev(yv, "y[%d]" % m, torch.float32) for m, yv in enumerate(ys)]
    for yv, n in zip(ys, Ns):
        if yv.numel() != int(n):
            raise ValueError("each output must hold N[m] floats")
    padded = sum((int(n) + 15) // 16 * 16 for n in Ns)
    need = dq_workspace_bytes(DQ_OP_Q4K_GEMV, padded, K, 1)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    arr_w = (ctypes.c_void_p * count)(*[wp.value for wp in wps])
    arr_n = (ctypes.c_int64 * count)(*[int(n) for n in Ns])
    arr_y = (ctypes.c_void_p * count)(*[yp.value for yp in yps])
    _check("q4k_gemv_group", lib.q4k_gemv_group(count, arr_w, arr_n, arr_y, _layout(layout),
                                                ctypes.c_void_p(x2.data_ptr()), K, wsp, wsn, _stream(stream)))
    return ys


def q4k_swiglu_gemv(w_gate, w_up, x, N: int, K: int, layout="aos", out=None, workspace=None,
                    stream=None):
    """out = silu(W_gate x) * (W_up x) for two Q4_K matrices (N x K)."""
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, K)
    B = x2.shape[0]
    gp = _weights(w_gate, "w_gate", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    up = _weights(w_up, "w_up", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    if out is None:
        out = torch.empty((B, N), dtype=torch.float32, device=x.device)
    op = _dev(out, "out", torch.float32)
    need = dq_workspace_bytes(DQ_OP_Q4K_SWIGLU, N, K, B)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    _check("q4k_swiglu_gemv", lib.q4k_swiglu_gemv(gp, up, _layout(layout), ctypes.c_void_p(x2.data_ptr()),
                                                  op, N, K, B, wsp, wsn, _stream(stream)))
    return out.view(N) if one_d else out.view(B, N)


def q8_0_gemv(w, x, N: int, K: int, y=None, workspace=None, stream=None):
    """y = W x for a Q8_0 matrix W (N x K)."""
    torch = _torch()
    lib = load_library()
    one_d = x.dim() == 1
    x2 = _x2d(x, K)
    B = x2.shape[0]
    wp = _weights(w, "w", N, K, Q8_0_BLOCK_ELEMS, Q8_0_BLOCK_BYTES)
    if y is None:
        y = torch.empty((B, N), dtype=torch.float32, device=x.device)
    yp = _dev(y, "y", torch.float32)
    need = dq_workspace_bytes(DQ_OP_Q8_0_GEMV, N, K, B)
    wsp, wsn, _keep = _workspace(workspace, need, x.device)
    _check("q8_0_gemv", lib.q8_0_gemv(wp, ctypes.c_void_p(x2.data_ptr()), yp, N, K, B, wsp, wsn,
                                      _stream(stream)))
    return y.view(N) if one_d else y.view(B, N)


def q4k_repack_soa(w_aos, N: int, K: int, out=None, stream=None):
    """AoS -> SoA repack of a Q4_K matrix (layout documented in dqgemv.h)."""
    torch = _torch()
    lib = load_library()
    ap = _weights(w_aos, "w_aos", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    if out is None:
        out = torch.empty_like(w_aos)
    op = _weights(out, "w_soa", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    _check("q4k_repack_soa", lib.q4k_repack_soa(ap, op, N, K, _stream(stream)))
    return out


def q4k_dequant(w, N: int, K: int, layout="aos", out=None, stream=None):
    """Debug dequantization of a Q4_K matrix to fp32 (N, K)."""
    torch = _torch()
    lib = load_library()
    wp = _weights(w, "w", N, K, Q4K_BLOCK_ELEMS, Q4K_BLOCK_BYTES)
    if out is None:
        out = torch.empty((N, K), dtype=torch.float32, device=w.device)
    op = _dev(out, "out", torch.float32)
    _check("q4k_dequant", lib.q4k_dequant(wp, _layout(layout), op, N, K, _stream(stream)))
    return out


def q8_0_dequant(w, N: int, K: int, out=None, stream=None):
    """Debug dequantization of a Q8_0 matrix to fp32 (N, K)."""
    torch = _torch()
    lib = load_library()
    wp = _weights(w, "w", N, K, Q8_0_BLOCK_ELEMS, Q8_0_BLOCK_BYTES)
    if out is None:
        out = torch.empty((N, K), dtype=torch.float32, device=w.device)
    op = _dev(out, "out", torch.float32)
    _check("q8_0_dequant", lib.q8_0_dequant(wp, op, N, K, _stream(stream)))
    return out


def dq_device_error(clear: bool = True, stream=None) -> int:
    """Synchronize and return the device error flag (0 = none); see dqgemv.h."""
    lib = load_library()
    flag = ctypes.c_int(0)
    _check("dq_device_error", lib.dq_device_error(ctypes.byref(flag), int(bool(clear)), _stream(stream)))
    return flag.value
