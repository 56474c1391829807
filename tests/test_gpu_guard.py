"""Guard bands around every output of every entry point (the stand-in for a memory checker).

Each output lives inside a larger buffer filled with a sentinel byte: a leading guard, the
columns between the written width and the row pitch, rows past the written rows, and a
trailing guard.  After the call every one of those bytes must still be the sentinel, and
the written region must be finite.  Shapes are ragged (rows not a multiple of the tile
height) so that the tiles' masked edges are exercised; one GEMM case splits its last wave
along K so that the split-K path and its reduction are covered too.
"""
import ctypes

import numpy as np
import pytest

import workloads
from tests._helpers import to_dev_bf16

pytestmark = pytest.mark.gpu

SENTINEL = 0xA5
GUARD = 256          # bytes before and after every buffer (keeps 16-byte alignment)


@pytest.fixture(scope="module")
def fq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp8_fine_grained_weight_b200 as fq
    fq.lib()
    return fq


class Guarded:
    """A [rows, cols] output with row pitch `ld` (elements) inside a sentinel-filled buffer
    with `pad_rows` extra rows and GUARD bytes on both ends."""

    def __init__(self, rows, cols, ld, dtype, pad_rows=3):
        import torch
        self.rows, self.cols, self.ld, self.pad = rows, cols, ld, pad_rows
        self.esz = torch.tensor([], dtype=dtype).element_size()
        body = (rows + pad_rows) * ld * self.esz
        self.raw = torch.full((GUARD + body + GUARD,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.full = self.raw[GUARD:GUARD + body].view(dtype).view(rows + pad_rows, ld)
        self.view = self.full[:rows, :cols]

    def ptr(self):
        return self.view.data_ptr()

    def check(self, name):
        host = self.raw.cpu().numpy()
        must = np.ones(host.size, dtype=bool)
        for r in range(self.rows):
            o = GUARD + r * self.ld * self.esz
            must[o:o + self.cols * self.esz] = False
        bad = np.flatnonzero(must & (host != SENTINEL))
        assert bad.size == 0, (f"{name}: {bad.size} bytes written outside [{self.rows}, {self.cols}] "
                               f"(pitch {self.ld}); first offsets {(bad[:8] - GUARD).tolist()}")
        if self.view.dtype.is_floating_point:
            import torch
            assert torch.isfinite(self.view.float()).all(), f"{name}: non-finite values written"


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def test_quant_act_1x128_guard(fq):
    import torch
    M, K = 200, 384
    x = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(1), (M, K), 1.0, 0.01))
    q = Guarded(M, K, K + 32, torch.uint8)
    s = Guarded(K // 128, M, M + 12, torch.float32)
    fq.quant_act_1x128(x, False, out=(q.view, s.view))
    q.check("quant_act q")
    s.check("quant_act scales")


def test_quant_weight_and_rowwise_guard_through_the_c_abi(fq):
    import torch
    L = fq.lib()
    N, K = 256, 384
    w = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(2), (N, K), 0.02))
    q = Guarded(N, K, K + 64, torch.uint8)
    s = Guarded(N // 128, K // 128, K // 128, torch.float32, pad_rows=0)
    assert L.fp8q_quant_weight_128x128(w.data_ptr(), N, K, K, q.ptr(), K + 64, s.ptr(), 0, _stream()) == 0
    M = 77
    x = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(3), (M, K), 1.0))
    qr = Guarded(M, K, K + 16, torch.uint8)
    sr = Guarded(1, M, M, torch.float32, pad_rows=0)
    assert L.fp8q_quant_rowwise(x.data_ptr(), M, K, K, qr.ptr(), K + 16, sr.ptr(), 0, _stream()) == 0
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    q.check("quant_weight q")
    s.check("quant_weight scales")
    qr.check("quant_rowwise q")
    sr.check("quant_rowwise scales")


def test_quant_dual_and_transpose_guard(fq):
    import torch
    M, K = 256, 384
    x = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(4), (M, K), 1.0, 0.01))
    q = Guarded(M, K, K + 8, torch.uint8)
    s = Guarded(K // 128, M, M + 4, torch.float32)
    qt = Guarded(K, M, M + 16, torch.uint8)
    st = Guarded(M // 128, K, K + 4, torch.float32)
    fq.quant_act_dual(x, False, out=(q.view, s.view, qt.view, st.view))
    for g, name in ((q, "dual q"), (s, "dual s"), (qt, "dual qt"), (st, "dual st")):
        g.check(name)
    wq, ws = fq.quant_weight_128x128(to_dev_bf16(workloads.normal_bf16(np.random.default_rng(5), (M, K), 0.02)))
    tq = Guarded(K, M, M + 32, torch.uint8)
    ts = Guarded(K // 128, M // 128, M // 128, torch.float32, pad_rows=0)
    fq.transpose_blocks(wq, ws, out=(tq.view, ts.view))
    tq.check("transpose_blocks qt")
    ts.check("transpose_blocks st")


def _gemm_operands(fq, M, N, K, seed, pow2=False, rowwise=False):
    rng = np.random.default_rng(seed)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(workloads.normal_bf16(rng, (M, K), 1.0, 0.001)), pow2)
    b = to_dev_bf16(workloads.normal_bf16(rng, (N, K), 0.02 if not rowwise else 1.0))
    qb, sb = fq.quant_act_1x128(b, pow2) if rowwise else fq.quant_weight_128x128(b, pow2)
    return qa, sa, qb, sb


# (300, 384, 512): ragged rows and a partial column tile; (4096, 7168, 1024): its last wave
# is split along K (workspace path and the reduction kernel).
@pytest.mark.parametrize("M,N,K", [(300, 384, 512), (4096, 7168, 1024)])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_gemm_blockscaled_guard(fq, M, N, K, out_fp32):
    import torch
    qa, sa, qb, sb = _gemm_operands(fq, M, N, K, M + N)
    dt = torch.float32 if out_fp32 else torch.bfloat16
    C = Guarded(M, N, N + 64, dt)
    fq.gemm_blockscaled(qa, sa, qb, sb, out=C.view)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    C.check(f"gemm_blockscaled {M}x{N}x{K}")


# M = 300: three row tiles, the last one ragged; M = 77: one partial row tile.
@pytest.mark.parametrize("M", [300, 77])
@pytest.mark.parametrize("rowwise", [False, True])
def test_gemm_ue8m0_and_nopromo_guard(fq, rowwise, M):
    import torch
    N, K = 640, 512                    # 640 = 2.86 tiles of 224 columns: a partial last tile
    qa, sa, qb, sb = _gemm_operands(fq, M, N, K, 11, pow2=True, rowwise=rowwise)
    C = Guarded(M, N, N + 32, torch.bfloat16)
    fq.gemm_blockscaled_ue8m0(qa, sa, qb, sb, b_rowwise=rowwise, out=C.view)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    C.check("gemm_blockscaled_ue8m0")
    if not rowwise:
        x = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(12), (M, K), 1.0))
        y = to_dev_bf16(workloads.normal_bf16(np.random.default_rng(13), (N, K), 1.0))
        qx, sx = fq.quant_rowwise(x)
        qy, sy = fq.quant_rowwise(y)
        Cn = Guarded(M, N, N + 8, torch.float32)
        fq.gemm_nopromo(qx, sx, qy, sy, out=Cn.view)
        torch.cuda.synchronize()
        Cn.check("gemm_nopromo")


@pytest.mark.parametrize("with_c", [True, False])
def test_gemm_quant_out_guard(fq, with_c):
    """The GEMM that also quantizes its output: C (optional), the codes (pitch > N) and the
    group-major scales (pitch > M); N = 384 leaves the last tile's second half outside."""
    import torch
    M, N, K = 300, 384, 512
    qa, sa, qb, sb = _gemm_operands(fq, M, N, K, 41)
    C = Guarded(M, N, N + 64, torch.bfloat16) if with_c else None
    q = Guarded(M, N, N + 48, torch.uint8)
    s = Guarded(N // 128, M, M + 20, torch.float32)
    fq.gemm_blockscaled_quant(qa, sa, qb, sb, out=(C.view if with_c else None, q.view, s.view))
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    if with_c:
        C.check("gemm_blockscaled_quant C")
    q.check("gemm_blockscaled_quant codes")
    s.check("gemm_blockscaled_quant scales")


def test_noalloc_guard(fq):
    import torch
    M, N, K = 300, 1024, 2048          # splits its last wave: the fixed scratch is used
    L = fq.lib()
    need = ctypes.c_size_t(0)
    assert L.fp8_gemm_workspace_size(M, N, K, ctypes.byref(need)) == 0 and need.value > 0
    qa, sa, qb, sb = _gemm_operands(fq, M, N, K, 21)
    C = Guarded(M, N, N + 16, torch.float32)
    assert L.fp8_gemm_blockscaled_noalloc(qa.data_ptr(), sa.data_ptr(), sa.stride(0), qb.data_ptr(),
                                          sb.data_ptr(), 0, 0, C.ptr(), 1, M, N, K, qa.stride(0),
                                          qb.stride(0), N + 16, _stream()) == 0
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    C.check("gemm_blockscaled_noalloc")


@pytest.mark.parametrize("ue8m0", [False, True])
def test_grouped_guard(fq, ue8m0):
    """Grouped C has an implied pitch N: the guard is the rows past the last offset (slack
    of the allocation) and the bytes after the buffer."""
    import torch
    counts = np.array([5, 0, 130, 1, 77])
    off = workloads.offsets_from_counts(counts)
    used, M, N, K = int(off[-1]), 256, 384, 256
    rng = np.random.default_rng(31)
    qa, sa = fq.quant_act_1x128(to_dev_bf16(workloads.normal_bf16(rng, (M, K), 1.0)), ue8m0)
    qw, sw = fq.quant_weight_128x128(to_dev_bf16(workloads.normal_bf16(rng, (len(counts), N, K), 0.02)), ue8m0)
    C = Guarded(used, N, N, torch.bfloat16, pad_rows=M - used)
    gemm = fq.gemm_grouped_ue8m0 if ue8m0 else fq.gemm_grouped
    gemm(qa, sa, qw, sw, torch.from_numpy(off).cuda(), out=C.full)
    torch.cuda.synchronize()
    assert fq.device_error() == 0
    C.check("grouped" + (" ue8m0" if ue8m0 else ""))
