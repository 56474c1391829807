"""CPU oracle for fine-grained FP8 quantization and the block-scaled FP8 GEMM.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference legs of ``bench.py`` may import this package.
It shares no code with the CUDA path and never imports it.

Two parts:

* ``liboracle.so`` (``fp8_oracle.c``): the E4M3 codec and the three
  quantizers, written from the definitions (see the C file's header).
* numpy FP64 GEMM: dequantize exactly (``decode(q) * s`` in double) and
  multiply with BLAS ``dgemm``.  The same routine gives
  ``T = sum_k |a_k b_k|``, which sets the tolerance.

The GEMM follows the-good.kr wr_id=2169793 para 1 (per-group scaling
factors along the inner dimension K, applied as dequantization) and
why-be.co.kr wr_id=57820 para 3 (partial results multiplied by the scaling
factors and added in FP32): exactly, the product of the dequantized
operands, summed over K.  FP64 is the "exact" stand-in: every product of two
dequantized values is exact in double, and the sum's rounding error is far
below the acceptance band.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

_lib = None


def lib() -> ctypes.CDLL:
    """Load (building if needed) the C oracle."""
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_scale_from_amax.argtypes = [ctypes.c_float, i32]
        L.orc_scale_from_amax.restype = ctypes.c_float
        L.orc_quant_act_1x128.argtypes = [vp, i64, i64, i64, vp, i64, vp, i64, i32]
        L.orc_quant_act_1x128.restype = None
        L.orc_quant_weight_128x128.argtypes = [vp, i64, i64, i64, vp, i64, vp, i32]
        L.orc_quant_weight_128x128.restype = None
        L.orc_quant_rowwise.argtypes = [vp, i64, i64, i64, vp, i64, vp, i32]
        L.orc_quant_rowwise.restype = None
        L.orc_gemm_triple.argtypes = [vp, vp, i64, vp, vp, i64, i32, i64, i64, i64, vp, vp]
        L.orc_quant_tensorwise.restype = None
        L.orc_quant_tensorwise.argtypes = [vp, i64, i64, i64, vp, i64, vp, i32]
        L.orc_gemm_triple.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ----------------------------------------------------------------------------------
# codec
# ----------------------------------------------------------------------------------

def e4m3_encode(v: float) -> int:
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_decode(code: int) -> float:
    return float(lib().orc_e4m3_decode(int(code) & 0xFF))


_DECODE = None


def decode_table() -> np.ndarray:
    """float64[256]: value of every E4M3 byte (NaN for 0x7F / 0xFF)."""
    global _DECODE
    if _DECODE is None:
        _DECODE = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return _DECODE


def scale_from_amax(amax: float, pow2: bool) -> float:
    return float(lib().orc_scale_from_amax(float(amax), int(bool(pow2))))


# ----------------------------------------------------------------------------------
# quantizers
# ----------------------------------------------------------------------------------

def quant_act_1x128(x_bits: np.ndarray, pow2: bool, ld_s: Optional[int] = None):
    """x_bits: uint16 bf16 bits [M, K].  Returns (q uint8 [M, K], s float32 [K/128, ld_s])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    M, K = x.shape
    assert K % 128 == 0
    ld = M if ld_s is None else ld_s
    q = np.empty((M, K), dtype=np.uint8)
    s = np.zeros((K // 128, ld), dtype=np.float32)
    lib().orc_quant_act_1x128(_ptr(x), M, K, K, _ptr(q), K, _ptr(s), ld, int(bool(pow2)))
    return q, s


def quant_weight_128x128(w_bits: np.ndarray, pow2: bool):
    """w_bits: uint16 bf16 bits [N, K].  Returns (q uint8 [N, K], s float32 [N/128, K/128])."""
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    N, K = w.shape
    assert N % 128 == 0 and K % 128 == 0
    q = np.empty((N, K), dtype=np.uint8)
    s = np.empty((N // 128, K // 128), dtype=np.float32)
    lib().orc_quant_weight_128x128(_ptr(w), N, K, K, _ptr(q), K, _ptr(s), int(bool(pow2)))
    return q, s


def quant_rowwise(x_bits: np.ndarray, pow2: bool = False):
    """One scale per row over all of K.  Returns (q uint8 [M, K], s float32 [M])."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    M, K = x.shape
    q = np.empty((M, K), dtype=np.uint8)
    s = np.empty((M,), dtype=np.float32)
    lib().orc_quant_rowwise(_ptr(x), M, K, K, _ptr(q), K, _ptr(s), int(bool(pow2)))
    return q, s


def quant_tensorwise(x_bits: np.ndarray, pow2: bool = False):
    """One scale for the whole tensor (the coarse baseline of the outlier study).
    Returns (q uint8 [R, C], s float)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    R, C = x.shape
    q = np.empty((R, C), dtype=np.uint8)
    s = np.zeros((1,), dtype=np.float32)
    lib().orc_quant_tensorwise(_ptr(x), R, C, C, _ptr(q), C, _ptr(s), int(bool(pow2)))
    return q, float(s[0])


# ----------------------------------------------------------------------------------
# GEMM
# ----------------------------------------------------------------------------------

def dequant_rows_groupmajor(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """decode(q[m, k]) * s[k // 128, m] in float64.  q [M, K]; s [K/128, >= M]."""
    M, K = q.shape
    d = decode_table()[q]
    sc = np.asarray(s, dtype=np.float64)[:, :M].T          # [M, G]
    return (d.reshape(M, K // 128, 128) * sc[:, :, None]).reshape(M, K)


def dequant_blocks(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """decode(q[n, k]) * s[n // 128, k // 128] in float64.  q [N, K]; s [N/128, K/128]."""
    N, K = q.shape
    d = decode_table()[q]
    sc = np.asarray(s, dtype=np.float64)
    return (d.reshape(N // 128, 128, K // 128, 128) * sc[:, None, :, None]).reshape(N, K)


def dequant_rowwise(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """decode(q[m, k]) * s[m] in float64."""
    return decode_table()[q] * np.asarray(s, dtype=np.float64)[:, None]


def gemm_ref(a_deq: np.ndarray, b_deq: np.ndarray, with_abs: bool = True):
    """C_ref = A B^T and T = |A| |B|^T in float64 (BLAS dgemm)."""
    c = a_deq @ b_deq.T
    t = np.abs(a_deq) @ np.abs(b_deq).T if with_abs else None
    return c, t


def gemm_blockscaled_ref(qa, sa, qb, sb, b_rowwise: bool = False):
    """Oracle of the dense block-scaled GEMM.

    qa [M, K], sa [K/128, >= M] group-major; qb [N, K]; sb [N/128, K/128]
    (128x128 blocks) or, with ``b_rowwise``, [K/128, >= N] group-major (1x128 tiles).
    Returns (C_ref, T) float64 [M, N].
    """
    A = dequant_rows_groupmajor(qa, sa)
    B = dequant_rows_groupmajor(qb, sb) if b_rowwise else dequant_blocks(qb, sb)
    return gemm_ref(A, B)


def gemm_triple(qa, sa, qb, sb, b_rowwise: bool = False):
    """Brute-force triple loop in C (tiny shapes).  Same arguments as gemm_blockscaled_ref."""
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    M, K = qa.shape
    N = qb.shape[0]
    C = np.empty((M, N), dtype=np.float64)
    T = np.empty((M, N), dtype=np.float64)
    ld_sb = sb.shape[1] if b_rowwise else 0
    lib().orc_gemm_triple(_ptr(qa), _ptr(sa), sa.shape[1], _ptr(qb), _ptr(sb), ld_sb,
                          int(bool(b_rowwise)), M, N, K, _ptr(C), _ptr(T))
    return C, T


def gemm_grouped_ref(qa, sa, qw, sw, offsets, rows=None):
    """Oracle of the grouped GEMM: rows offsets[e]..offsets[e+1] of A times W[e]^T.

    qa [sumM, K]; sa [K/128, >= sumM]; qw [E, N, K]; sw [E, N/128, K/128].
    ``rows`` (optional int array) restricts the output to those global rows.
    Returns (C_ref, T) float64 [len(rows) or sumM, N].
    """
    off = np.asarray(offsets, dtype=np.int64)
    E, N, K = qw.shape
    rows = np.arange(off[-1]) if rows is None else np.asarray(rows, dtype=np.int64)
    C = np.zeros((rows.size, N))
    T = np.zeros((rows.size, N))
    expert = np.searchsorted(off, rows, side="right") - 1
    for e in np.unique(expert):
        sel = np.nonzero(expert == e)[0]
        r = rows[sel]
        A = decode_table()[qa[r]] * np.asarray(sa, np.float64)[:, r].T.repeat(128, axis=1)
        B = dequant_blocks(qw[e], sw[e])
        c, t = gemm_ref(A, B)
        C[sel] = c
        T[sel] = t
    return C, T


# ----------------------------------------------------------------------------------
# acceptance
# ----------------------------------------------------------------------------------

FP32_REL = 2e-5
FP32_ABS = 1e-30


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits); the subnormal spacing below 2^-126."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, ex = np.frexp(a)                      # a = f * 2^ex, f in [0.5, 1): a in [2^(ex-1), 2^ex)
    e = np.maximum(ex.astype(np.float64) - 1.0, -126.0)
    return np.where(a > 0, np.exp2(e - 7.0), np.exp2(-133.0))


def check_fp32(C: np.ndarray, C_ref: np.ndarray, T: np.ndarray):
    """Boolean mask of entries that satisfy |C - C_ref| <= 2e-5 T + 1e-30."""
    return np.abs(np.asarray(C, np.float64) - C_ref) <= FP32_REL * T + FP32_ABS


def check_bf16(C: np.ndarray, C_ref: np.ndarray, T: np.ndarray):
    """(ok mask, fallback mask) for bf16 outputs.

    Primary: |C - C_ref| <= 1 bf16 ulp of C_ref.  Fallback where the sum cancels
    (T >> |C_ref|): C is the bf16 rounding of some value inside the fp32 band,
    i.e. |C - C_ref| <= 2e-5 T + ulp_bf16(C) / 2.
    """
    C = np.asarray(C, np.float64)
    d = np.abs(C - C_ref)
    prim = d <= bf16_ulp(C_ref)
    fb = d <= FP32_REL * T + 0.5 * bf16_ulp(C) + FP32_ABS
    return prim | fb, (~prim) & fb
