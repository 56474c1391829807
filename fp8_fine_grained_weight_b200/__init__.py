"""fp8q: fine-grained FP8 (E4M3) quantization and block-scaled FP8 GEMM on B200 (sm_100a).

A thin ctypes binding over ``libfp8q.so`` (the C ABI in ``include/fp8q.h``).  Every
step of the computation runs in the library's CUDA kernels; this module only checks
tensor dtypes/devices, allocates outputs with PyTorch and passes raw device pointers
and the current CUDA stream.  There is no CPU fallback: if the library is missing or
a call fails, an exception is raised.

Layouts (see include/fp8q.h):
  activation scales  group-major fp32 [K/128, ld]   (scale of row m, group g at [g, m])
  weight scales      fp32 [N/128, K/128]
  E4M3 tensors       torch.uint8 (view as torch.float8_e4m3fn if wanted)
"""
from __future__ import annotations

import collections
import contextlib
import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

OUT_BF16, OUT_FP32 = 0, 1
BSCALE_BLOCK, BSCALE_ROW = 0, 1

STATUS = {0: "FP8Q_OK", 1: "FP8Q_ERR_NULL", 2: "FP8Q_ERR_SHAPE", 3: "FP8Q_ERR_ALIGN",
          4: "FP8Q_ERR_UNSUPPORTED", 5: "FP8Q_ERR_CUDA", 6: "FP8Q_ERR_TIMEOUT",
          7: "FP8Q_ERR_SCALE"}

# name -> (restype, argtypes); mirrors include/fp8q.h
_i64, _i32, _vp, _f = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_float
SIGNATURES = {
    "fp8q_quant_act_1x128": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _i32, _vp]),
    "fp8q_quant_weight_128x128": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _i32, _vp]),
    "fp8q_quant_rowwise": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _i32, _vp]),
    "fp8q_transpose_blocks": (_i32, [_vp, _vp, _i64, _i64, _i64, _vp, _vp, _i64, _vp]),
    "fp8q_quant_act_dual": (_i32, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _vp, _i64,
                                   _vp, _i64, _i32, _vp]),
    "fp8_gemm_blockscaled": (_i32, [_vp, _vp, _i64, _vp, _vp, _i64, _i32, _vp, _i32,
                                    _i64, _i64, _i64, _i64, _i64, _i64, _vp]),
    "fp8_gemm_blockscaled_ue8m0": (_i32, [_vp, _vp, _i64, _vp, _vp, _i64, _i32, _vp, _i32,
                                          _i64, _i64, _i64, _i64, _i64, _i64, _vp]),
    "fp8_gemm_blockscaled_quant": (_i32, [_vp, _vp, _i64, _vp, _vp, _i64, _i32, _vp, _i64,
                                          _vp, _i64, _vp, _i64, _i32, _i64, _i64, _i64, _i64,
                                          _i64, _vp]),
    "fp8_gemm_grouped_ue8m0": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _i32, _vp, _i32, _i64, _i64,
                                      _i64, _vp]),
    "fp8_gemm_blockscaled_ws": (_i32, [_vp, _vp, _i64, _vp, _vp, _i64, _i32, _vp, _i32,
                                       _i64, _i64, _i64, _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp]),
    "fp8_gemm_workspace_size": (_i32, [_i64, _i64, _i64, ctypes.POINTER(ctypes.c_size_t)]),
    "fp8_gemm_blockscaled_noalloc": (_i32, [_vp, _vp, _i64, _vp, _vp, _i64, _i32, _vp, _i32,
                                            _i64, _i64, _i64, _i64, _i64, _i64, _vp]),
    "fp8_gemm_grouped": (_i32, [_vp, _vp, _i64, _vp, _vp, _vp, _i32, _vp, _i32,
                                _i64, _i64, _i64, _vp]),
    "fp8_gemm_nopromo": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _i64, _i64, _vp]),
    "fp8q_get_device_error": (_i32, [_vp]),
    "fp8q_selftest_wait_timeout": (_i32, [ctypes.c_uint64, _vp]),
    "fp8q_status_string": (ctypes.c_char_p, [_i32]),
    "fp8q_abi_version": (_i32, []),
}

_lib: Optional[ctypes.CDLL] = None


class Fp8qError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status & 0xFF, status)} "
                         f"({lib().fp8q_status_string(status).decode()}), site {status >> 8}")


def lib() -> ctypes.CDLL:
    """The loaded C library.  Raises if ``libfp8q.so`` has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m fp8_fine_grained_weight_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _call(name: str, *args) -> None:
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise Fp8qError(name, st)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _on(t: torch.Tensor):
    """Make t's device the current one for a library call.  The library sizes grids and
    binds its driver context through the current device, so operands on another GPU must
    not be passed while a different device is current."""
    return torch.cuda.device(t.device) if t.is_cuda else contextlib.nullcontext()


def _require_cuda(t: torch.Tensor, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")


def _need(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None) -> None:
    _require_cuda(t, name)
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if t.dim() and t.stride(-1) != 1:
        raise ValueError(f"{name} must be contiguous in its last dimension")


def _u8(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t


def _same_device(t: torch.Tensor, device: torch.device, name: str) -> None:
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, the other operands on {device}")


def _rows(t: torch.Tensor, dtype, name: str, rows: int, cols: int, device: torch.device) -> None:
    """A 2-D operand the kernels address as [rows, cols] through its row stride: on `device`,
    contiguous in its last dimension and at least rows x cols (the library sees only a
    pointer and the stride, so a smaller tensor would be read or written out of bounds)."""
    _need(t, dtype, name, 2)
    _same_device(t, device, name)
    if t.shape[0] < rows or t.shape[1] < cols:
        raise ValueError(f"{name} must be at least [{rows}, {cols}], got {tuple(t.shape)}")


def _dense(t: torch.Tensor, dtype, name: str, shape, device: torch.device) -> None:
    """An operand the kernels address with an implied row pitch: exactly `shape`, contiguous."""
    _need(t, dtype, name)
    _same_device(t, device, name)
    if tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor of shape {tuple(shape)}, "
                         f"got {tuple(t.shape)} with strides {t.stride()}")


# --------------------------------------------------------------------------------------
# quantization
# --------------------------------------------------------------------------------------

def quant_act_1x128(x: torch.Tensor, pow2: bool = False, ld_scale: Optional[int] = None,
                    out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """1x128 activation tiles: x bf16 [M, K] -> (q uint8 [M, K], s fp32 [K/128, ld_scale])."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    if out is None:
        ld = M if ld_scale is None else int(ld_scale)
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
        s = torch.empty((K // 128 if K % 128 == 0 else 0, ld), dtype=torch.float32, device=x.device)
    else:
        q, s = out
        _rows(_u8(q), torch.uint8, "q", M, K, x.device)
        _rows(s, torch.float32, "s", K // 128, M, x.device)
        ld = s.stride(0)
        if ld_scale is not None and int(ld_scale) != ld:
            raise ValueError(f"ld_scale {ld_scale} disagrees with the row stride {ld} of s")
    with _on(x):
        _call("fp8q_quant_act_1x128", x.data_ptr(), M, K, x.stride(0), _u8(q).data_ptr(),
              _u8(q).stride(0), s.data_ptr(), ld, int(bool(pow2)), _stream(x))
    return q, s


def quant_act_dual(x: torch.Tensor, pow2: bool = False, out=None):
    """Rows and columns from one read: x bf16 [M, K] (M, K multiples of 128) ->
    (q uint8 [M, K], s fp32 [K/128, M], qt uint8 [K, M], st fp32 [M/128, K]), where (q, s)
    is quant_act_1x128(x) and (qt, st) is quant_act_1x128 of x transposed."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    if out is None:
        q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
        s = torch.empty((K // 128, M), dtype=torch.float32, device=x.device)
        qt = torch.empty((K, M), dtype=torch.uint8, device=x.device)
        st = torch.empty((M // 128, K), dtype=torch.float32, device=x.device)
    else:
        q, s, qt, st = out
        _rows(_u8(q), torch.uint8, "q", M, K, x.device)
        _rows(s, torch.float32, "s", K // 128, M, x.device)
        _rows(_u8(qt), torch.uint8, "qt", K, M, x.device)
        _rows(st, torch.float32, "st", M // 128, K, x.device)
    q8, qt8 = _u8(q), _u8(qt)
    with _on(x):
        _call("fp8q_quant_act_dual", x.data_ptr(), M, K, x.stride(0), q8.data_ptr(), q8.stride(0),
              s.data_ptr(), s.stride(0), qt8.data_ptr(), qt8.stride(0), st.data_ptr(), st.stride(0),
              int(bool(pow2)), _stream(x))
    return q, s, qt, st


def transpose_blocks(q: torch.Tensor, s: torch.Tensor, out=None):
    """q uint8 [N, K], s fp32 [N/128, K/128] (128x128 blocks) -> (q^T [K, N], s^T [K/128, N/128]):
    the 128x128 quantization of the transposed matrix."""
    q = _u8(q)
    _need(q, torch.uint8, "q", 2)
    _need(s, torch.float32, "s", 2)
    N, K = q.shape
    _dense(s, torch.float32, "s", (N // 128, K // 128), q.device)
    if out is None:
        qt = torch.empty((K, N), dtype=torch.uint8, device=q.device)
        st = torch.empty((K // 128, N // 128), dtype=torch.float32, device=q.device)
    else:
        qt, st = out
        _rows(_u8(qt), torch.uint8, "qt", K, N, q.device)
        _dense(st, torch.float32, "st", (K // 128, N // 128), q.device)
    with _on(q):
        _call("fp8q_transpose_blocks", q.data_ptr(), s.data_ptr(), N, K, q.stride(0),
              _u8(qt).data_ptr(), st.data_ptr(), _u8(qt).stride(0), _stream(q))
    return qt, st


def quant_weight_128x128(w: torch.Tensor, pow2: bool = False,
                         out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None):
    """128x128 weight blocks: w bf16 [N, K] (or [E, N, K]) -> (q uint8, s fp32 [.., N/128, K/128])."""
    _need(w, torch.bfloat16, "w")
    if w.dim() not in (2, 3):
        raise ValueError("w must be [N, K] or [E, N, K]")
    if not w.is_contiguous():
        raise ValueError("w must be contiguous")
    K = w.shape[-1]
    N_all = w.numel() // K if K else 0
    s_shape = (*w.shape[:-2], w.shape[-2] // 128, K // 128)
    if out is None:
        q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
        s = torch.empty(s_shape, dtype=torch.float32, device=w.device)
    else:
        q, s = out
        _dense(_u8(q), torch.uint8, "q", w.shape, w.device)     # row pitch K implied
        _dense(s, torch.float32, "s", s_shape, w.device)
    with _on(w):
        _call("fp8q_quant_weight_128x128", w.data_ptr(), N_all, K, K, _u8(q).data_ptr(), K,
              s.data_ptr(), int(bool(pow2)), _stream(w))
    return q, s


def quant_rowwise(x: torch.Tensor, pow2: bool = False):
    """One scale per row over all of K: x bf16 [M, K] -> (q uint8 [M, K], s fp32 [M])."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((M,), dtype=torch.float32, device=x.device)
    with _on(x):
        _call("fp8q_quant_rowwise", x.data_ptr(), M, K, x.stride(0), q.data_ptr(), q.stride(0),
              s.data_ptr(), int(bool(pow2)), _stream(x))
    return q, s


# --------------------------------------------------------------------------------------
# GEMM
# --------------------------------------------------------------------------------------

def _out_code(out_dtype) -> int:
    if out_dtype == torch.bfloat16:
        return OUT_BF16
    if out_dtype == torch.float32:
        return OUT_FP32
    raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")


# Split-K workspaces cached per (device, stream), least recently used first.  At most
# _WORKSPACE_MAX are kept (each at most a few tens of MB); a program that cycles through
# more streams than that gets a new buffer when it returns to an evicted one.  A buffer is
# allocated on, and only ever used by, its own stream, so dropping it is safe while GEMMs on
# that stream are still in flight (the caching allocator orders the reuse after them).
# Callers that want no cached buffers pass workspace= themselves.
_WORKSPACE: "collections.OrderedDict" = collections.OrderedDict()
_WORKSPACE_MAX = 8


def workspace_bytes(M: int, N: int, K: int) -> int:
    """Device workspace the dense GEMM can use to split its last wave (0 if none)."""
    n = ctypes.c_size_t(0)
    _call("fp8_gemm_workspace_size", M, N, K, ctypes.byref(n))
    return int(n.value)


def _workspace(device, stream: int, nbytes: int) -> torch.Tensor:
    """A scratch buffer of at least nbytes for one (device, stream), grown on demand
    (never shrunk).  Calls on one stream run in order and share it; GEMMs on different
    streams get different buffers, so they may run concurrently."""
    key = (torch.device(device).index, int(stream))
    ws = _WORKSPACE.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _WORKSPACE[key] = ws
    _WORKSPACE.move_to_end(key)
    while len(_WORKSPACE) > _WORKSPACE_MAX:
        _WORKSPACE.popitem(last=False)
    return ws


def _dense_gemm_operands(qa, sa, qb, sb, b_rowwise: bool, out, out_dtype, alloc: bool = True):
    """Checks of the dense GEMMs' operands; returns (qa, qb, out, M, N, K) (out allocated
    when None and ``alloc``)."""
    qa, qb = _u8(qa), _u8(qb)
    _need(qa, torch.uint8, "qa", 2)
    _need(qb, torch.uint8, "qb", 2)
    dev = qa.device
    _same_device(qb, dev, "qb")
    M, K = qa.shape
    N = qb.shape[0]
    if qb.shape[1] != K:
        raise ValueError("qa and qb disagree on K")
    _rows(sa, torch.float32, "sa", K // 128, M, dev)             # [K/128, >= M]
    if b_rowwise:
        _rows(sb, torch.float32, "sb", K // 128, N, dev)         # [K/128, >= N]
    else:                                                        # [N/128, K/128], pitch implied
        _dense(sb, torch.float32, "sb", (-(-N // 128), K // 128), dev)
    if out is None:
        if alloc:
            out = torch.empty((M, N), dtype=out_dtype, device=dev)
    else:
        _out_code(out.dtype)
        _rows(out, out.dtype, "out", M, N, dev)
    return qa, qb, out, M, N, K


def gemm_blockscaled(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                     out_dtype=torch.bfloat16, b_rowwise: bool = False,
                     out: Optional[torch.Tensor] = None, split_k: bool = True,
                     workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """C = A B^T with per-128-K promotion.

    qa uint8 [M, K]; sa fp32 [K/128, >= M]; qb uint8 [N, K];
    sb fp32 [N/128, K/128] (128x128 blocks) or, with ``b_rowwise``, [K/128, >= N].
    ``split_k``: split the last partial wave of tiles along K (uses a device workspace:
    ``workspace`` if given, else a buffer cached per device and stream).
    """
    qa, qb, out, M, N, K = _dense_gemm_operands(qa, sa, qb, sb, b_rowwise, out, out_dtype)
    ws_ptr, ws_len = None, 0
    with _on(qa):
        if split_k and M > 0:
            need = workspace_bytes(M, N, K)
            if need:
                ws = workspace if workspace is not None else _workspace(qa.device, _stream(qa), need)
                _same_device(ws, qa.device, "workspace")
                if ws.numel() * ws.element_size() >= need:
                    ws_ptr, ws_len = ws.data_ptr(), ws.numel() * ws.element_size()
        _call("fp8_gemm_blockscaled_ws", qa.data_ptr(), sa.data_ptr(), sa.stride(0), qb.data_ptr(),
              sb.data_ptr(), sb.stride(0) if b_rowwise else 0,
              BSCALE_ROW if b_rowwise else BSCALE_BLOCK, out.data_ptr(), _out_code(out.dtype),
              M, N, K, qa.stride(0), qb.stride(0), out.stride(0), ws_ptr, ws_len, _stream(qa))
    return out


def gemm_blockscaled_quant(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                           pow2: bool = False, b_rowwise: bool = False, with_c: bool = True,
                           out=None):
    """bf16 C = A B^T with per-128-K promotion, also quantized 1x128 in the GEMM's epilogue.

    Same operands as ``gemm_blockscaled``.  Returns (C bf16 [M, N] or None without
    ``with_c``, qc uint8 [M, N], sc fp32 [N/128, M]) where (qc, sc) equals
    ``quant_act_1x128(C, pow2)``.  ``out``: (C or None, qc, sc) to write into.
    """
    if out is None:
        qa, qb, c, M, N, K = _dense_gemm_operands(qa, sa, qb, sb, b_rowwise, None, torch.bfloat16,
                                                  alloc=with_c)
        qc = torch.empty((M, N), dtype=torch.uint8, device=qa.device)
        sc = torch.empty((N // 128, M), dtype=torch.float32, device=qa.device)
    else:
        c, qc, sc = out
        if c is not None and c.dtype != torch.bfloat16:
            raise ValueError("C must be bf16")
        qa, qb, c, M, N, K = _dense_gemm_operands(qa, sa, qb, sb, b_rowwise, c, torch.bfloat16,
                                                  alloc=False)
        _rows(_u8(qc), torch.uint8, "qc", M, N, qa.device)
        _rows(sc, torch.float32, "sc", N // 128, M, qa.device)
    with _on(qa):
        _call("fp8_gemm_blockscaled_quant", qa.data_ptr(), sa.data_ptr(), sa.stride(0), qb.data_ptr(),
              sb.data_ptr(), sb.stride(0) if b_rowwise else 0,
              BSCALE_ROW if b_rowwise else BSCALE_BLOCK, c.data_ptr() if c is not None else None,
              c.stride(0) if c is not None else 0, _u8(qc).data_ptr(), _u8(qc).stride(0),
              sc.data_ptr(), sc.stride(0), int(bool(pow2)), M, N, K, qa.stride(0), qb.stride(0),
              _stream(qa))
    return c, qc, sc


def gemm_blockscaled_ue8m0(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                           out_dtype=torch.bfloat16, b_rowwise: bool = False,
                           out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """C = A B^T for power-of-two scales, scaled inside the tensor core (UE8M0 block scales).

    Same operands as ``gemm_blockscaled``; every scale must be a power of two in
    [2^-127, 2^127] (the quantizers' ``pow2`` option).  Other scales are reported through
    ``device_error()`` as (8 << 8) | FP8Q_ERR_SCALE.
    """
    qa, qb, out, M, N, K = _dense_gemm_operands(qa, sa, qb, sb, b_rowwise, out, out_dtype)
    with _on(qa):
        _call("fp8_gemm_blockscaled_ue8m0", qa.data_ptr(), sa.data_ptr(), sa.stride(0), qb.data_ptr(),
              sb.data_ptr(), sb.stride(0) if b_rowwise else 0,
              BSCALE_ROW if b_rowwise else BSCALE_BLOCK, out.data_ptr(), _out_code(out.dtype),
              M, N, K, qa.stride(0), qb.stride(0), out.stride(0), _stream(qa))
    return out


def _gemm_grouped(entry: str, qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                 m_offsets: torch.Tensor, out_dtype=torch.bfloat16,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """MoE grouped GEMM through `entry`: rows m_offsets[e]..m_offsets[e+1] of A times W[e]^T.

    qa uint8 [sumM, K]; sa fp32 [K/128, >= sumM]; qw uint8 [E, N, K]; sw fp32 [E, N/128, K/128];
    m_offsets int32 [E + 1] on the device (read by the kernel, no host sync).
    """
    qa, qw = _u8(qa), _u8(qw)
    _need(qa, torch.uint8, "qa", 2)
    _need(qw, torch.uint8, "qw", 3)
    _need(m_offsets, torch.int32, "m_offsets", 1)
    if not (qa.is_contiguous() and qw.is_contiguous()):
        raise ValueError("qa and qw must be contiguous")
    dev = qa.device
    M, K = qa.shape
    E, N, Kw = qw.shape
    if Kw != K:
        raise ValueError("qa and qw disagree on K")
    _same_device(qw, dev, "qw")
    _same_device(m_offsets, dev, "m_offsets")
    _rows(sa, torch.float32, "sa", K // 128, M, dev)                          # [K/128, >= sumM]
    _dense(sw, torch.float32, "sw", (E, -(-N // 128), K // 128), dev)         # [E, N/128, K/128]
    if m_offsets.numel() != E + 1:
        raise ValueError("m_offsets must have E + 1 entries")
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev)
    else:
        _out_code(out.dtype)
        _rows(out, out.dtype, "out", M, N, dev)
    with _on(qa):
        _call(entry, qa.data_ptr(), sa.data_ptr(), sa.stride(0), qw.data_ptr(),
              sw.data_ptr(), out.data_ptr(), _out_code(out.dtype), m_offsets.data_ptr(), E, M, N, K,
              _stream(qa))
    return out


def gemm_grouped(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                 m_offsets: torch.Tensor, out_dtype=torch.bfloat16,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """MoE grouped GEMM with per-128-K promotion: rows m_offsets[e]..m_offsets[e+1] of A
    times W[e]^T.  qa uint8 [sumM, K]; sa fp32 [K/128, >= sumM]; qw uint8 [E, N, K];
    sw fp32 [E, N/128, K/128]; m_offsets int32 [E + 1] on the device."""
    return _gemm_grouped("fp8_gemm_grouped", qa, sa, qw, sw, m_offsets, out_dtype, out)


def gemm_grouped_ue8m0(qa: torch.Tensor, sa: torch.Tensor, qw: torch.Tensor, sw: torch.Tensor,
                       m_offsets: torch.Tensor, out_dtype=torch.bfloat16,
                       out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """gemm_grouped for power-of-two scales, applied inside the tensor core."""
    return _gemm_grouped("fp8_gemm_grouped_ue8m0", qa, sa, qw, sw, m_offsets, out_dtype, out)


def gemm_nopromo(qa: torch.Tensor, sa: torch.Tensor, qb: torch.Tensor, sb: torch.Tensor,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Accumulation-study variant: one accumulator over all of K, 1xK scales sa [M], sb [N]; fp32 C."""
    qa, qb = _u8(qa), _u8(qb)
    _need(qa, torch.uint8, "qa", 2)
    _need(qb, torch.uint8, "qb", 2)
    _need(sa, torch.float32, "sa", 1)
    _need(sb, torch.float32, "sb", 1)
    dev = qa.device
    M, K = qa.shape
    N = qb.shape[0]
    if qb.shape[1] != K:
        raise ValueError("qa and qb disagree on K")
    for t, name, n in ((qb, "qb", None), (sa, "sa", M), (sb, "sb", N)):
        _same_device(t, dev, name)
        if n is not None and t.shape[0] < n:
            raise ValueError(f"{name} must hold at least {n} scales, got {t.shape[0]}")
    if out is None:
        out = torch.empty((M, N), dtype=torch.float32, device=dev)
    else:
        _rows(out, torch.float32, "out", M, N, dev)
    with _on(qa):
        _call("fp8_gemm_nopromo", qa.data_ptr(), sa.data_ptr(), qb.data_ptr(), sb.data_ptr(),
              out.data_ptr(), M, N, K, qa.stride(0), qb.stride(0), out.stride(0), _stream(qa))
    return out


def device_error(device=None) -> int:
    """Read and clear the library's device error word on `device` (default: the current
    device); synchronizes that device's current stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib().fp8q_get_device_error(torch.cuda.current_stream(dev).cuda_stream))


def status_string(status: int) -> str:
    return lib().fp8q_status_string(int(status)).decode()
