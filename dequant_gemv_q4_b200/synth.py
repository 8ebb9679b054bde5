"""Seeded synthetic inputs: raw Q8_0 / Q4_K block bytes and fp32 activations.

This module only draws random numbers and lays the drawn fields out as bytes;
it holds none of the dequantize / GEMV arithmetic.  Both the CUDA path and the
CPU oracle are fed from it, so that they see the same bytes.

Value distributions (one generator per workload, ``numpy.random.default_rng``):

* Q4_K super-block (144 bytes = d | dmin | 12 scale bytes | 128 quant bytes):
  ``d ~ U[1e-3, 1e-2]`` and ``dmin ~ U[0, 5e-3]``, each rounded to fp16 (round
  to nearest even); 12 uniformly random scale bytes, which makes the 16 packed
  six-bit scale/min fields i.i.d. uniform on [0, 63] because the packing is a
  bijection of the 96 bits; 128 uniformly random quant bytes, which makes every
  4-bit quant uniform on [0, 15].
* Q8_0 block (34 bytes = d | 32 int8): ``d ~ U[1e-3, 1e-2]`` rounded to fp16,
  quants uniform on [-127, 127].
* Activations ``x ~ N(0, 1)`` in fp32, optionally multiplied by a power of two.

Draw order within a workload: matrix fields in the order d, dmin, scales,
quants (gate matrix before up matrix), then x.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

Q8_0_BLOCK_ELEMS = 32
Q8_0_BLOCK_BYTES = 34
Q4K_BLOCK_ELEMS = 256
Q4K_BLOCK_BYTES = 144


def q4k_matrix(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """N x (K/256 * 144) uint8: N rows of GGML-style Q4_K super-blocks."""
    if K % Q4K_BLOCK_ELEMS:
        raise ValueError("K must be a multiple of 256")
    nb = N * (K // Q4K_BLOCK_ELEMS)
    d = rng.uniform(1e-3, 1e-2, nb).astype(np.float16)
    dmin = rng.uniform(0.0, 5e-3, nb).astype(np.float16)
    scales = rng.integers(0, 256, (nb, 12), dtype=np.uint8)
    qs = rng.integers(0, 256, (nb, 128), dtype=np.uint8)
    return q4k_pack(d, dmin, scales, qs).reshape(N, -1)


def q4k_pack(d, dmin, scales, qs) -> np.ndarray:
    """Lay out per-block fields as (nb, 144) bytes: d | dmin | scales | qs."""
    d = np.ascontiguousarray(np.asarray(d, dtype=np.float16).reshape(-1))
    dmin = np.ascontiguousarray(np.asarray(dmin, dtype=np.float16).reshape(-1))
    nb = d.size
    out = np.empty((nb, Q4K_BLOCK_BYTES), np.uint8)
    out[:, 0:2] = d.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 2:4] = dmin.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 4:16] = np.asarray(scales, dtype=np.uint8).reshape(nb, 12)
    out[:, 16:144] = np.asarray(qs, dtype=np.uint8).reshape(nb, 128)
    return out


def q8_0_matrix(rng: np.random.Generator, N: int, K: int) -> np.ndarray:
    """N x (K/32 * 34) uint8: N rows of GGML-style Q8_0 blocks."""
    if K % Q8_0_BLOCK_ELEMS:
        raise ValueError("K must be a multiple of 32")
    nb = N * (K // Q8_0_BLOCK_ELEMS)
    d = rng.uniform(1e-3, 1e-2, nb).astype(np.float16)
    q = rng.integers(-127, 128, (nb, Q8_0_BLOCK_ELEMS), dtype=np.int8)
    return q8_0_pack(d, q).reshape(N, -1)


def q8_0_pack(d, q) -> np.ndarray:
    d = np.ascontiguousarray(np.asarray(d, dtype=np.float16).reshape(-1))
    nb = d.size
    out = np.empty((nb, Q8_0_BLOCK_BYTES), np.uint8)
    out[:, 0:2] = d.astype("<f2").view(np.uint8).reshape(nb, 2)
    out[:, 2:] = np.asarray(q, dtype=np.int8).reshape(nb, Q8_0_BLOCK_ELEMS).view(np.uint8)
    return out


def activations(rng: np.random.Generator, B: int, K: int, scale: float = 1.0) -> np.ndarray:
    """B x K fp32 N(0,1), times `scale` (a power of two keeps the draw exact)."""
    x = rng.standard_normal(B * K, dtype=np.float32).reshape(B, K)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def activations_f16(rng: np.random.Generator, M: int, K: int, scale: float = 1.0) -> np.ndarray:
    """M x K binary16 activations (numpy float16): N(0,1) draws in fp32, times
    `scale`, converted to the nearest binary16 value."""
    return activations(rng, M, K, scale).astype(np.float16)


# ---------------------------------------------------------------------------
# Named workloads: the five decode shapes the library is measured on.
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    name: str
    fmt: str            # "q8_0" or "q4k"
    op: str             # "gemv", "swiglu" or "gemv_argmax"
    N: int
    K: int
    batches: tuple      # batch sizes exercised
    seed: int
    x_scale: float = 1.0
    notes: str = field(default="", compare=False)


WORKLOADS = {
    "q8_0_gemv_1024x1024": Workload("q8_0_gemv_1024x1024", "q8_0", "gemv", 1024, 1024, (1,), 0,
                                    notes="Q8_0 GEMV, batch 1"),
    "q4k_gemv_4096x1024": Workload("q4k_gemv_4096x1024", "q4k", "gemv", 4096, 1024, (1,), 1,
                                   notes="q-projection-with-gate shape of a hidden-1024 model"),
    "q4k_swiglu_12288x4096": Workload("q4k_swiglu_12288x4096", "q4k", "swiglu", 12288, 4096,
                                      (1,), 2, notes="fused gate/up SwiGLU, two matrices"),
    "q4k_down_4096x12288": Workload("q4k_down_4096x12288", "q4k", "gemv", 4096, 12288,
                                    (1, 2, 4, 8), 3, notes="down projection, B in {1,2,4,8}"),
    "q4k_lmhead_248320x4096": Workload("q4k_lmhead_248320x4096", "q4k", "gemv_argmax", 248320,
                                       4096, (1,), 4, x_scale=1.0 / 64,
                                       notes="LM head with argmax, x scaled by 1/64"),
}


def make_inputs(wl: Workload, B: int = 1):
    """Seeded inputs of a workload: dict with 'w' (or 'w_gate','w_up') and 'x' (B x K)."""
    rng = np.random.default_rng(wl.seed)
    gen = q4k_matrix if wl.fmt == "q4k" else q8_0_matrix
    out = {}
    if wl.op == "swiglu":
        out["w_gate"] = gen(rng, wl.N, wl.K)
        out["w_up"] = gen(rng, wl.N, wl.K)
    else:
        out["w"] = gen(rng, wl.N, wl.K)
    out["x"] = activations(rng, B, wl.K, wl.x_scale)
    return out
