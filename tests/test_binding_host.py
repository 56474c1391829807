"""The Python binding's marshalling, on the CPU: each entry point's operand checks and
the arguments it hands to the C ABI.  The library call is recorded instead of made and
the CUDA-tensor requirement is lifted, so CPU tensors stand in for device buffers; the
shapes are the ones the GPU tests, the bench and the FP8 linear layer use."""
import collections

import pytest
import torch

import fp8_fine_grained_weight_b200 as fq

bf16, u8, f32, i32 = torch.bfloat16, torch.uint8, torch.float32, torch.int32


@pytest.fixture
def calls(monkeypatch):
    log = []
    monkeypatch.setattr(fq, "_require_cuda", lambda t, name: None)
    monkeypatch.setattr(fq, "_stream", lambda t: 0)
    monkeypatch.setattr(fq, "workspace_bytes", lambda M, N, K: 0)
    monkeypatch.setattr(fq, "_call", lambda name, *args: log.append((name, args)))
    return log


def E(*shape, dtype=u8):
    return torch.empty(shape, dtype=dtype)


def test_product_path_still_requires_cuda_tensors():
    with pytest.raises(TypeError, match="CUDA tensor"):
        fq.quant_act_1x128(E(4, 128, dtype=bf16))


def test_quant_act_scale_pitch_is_the_scale_buffers_row_stride(calls):
    x = E(256, 384, dtype=bf16)
    q, s = fq.quant_act_1x128(x)
    assert q.shape == (256, 384) and s.shape == (3, 256) and calls[-1][1][7] == 256
    q2, s2 = fq.quant_act_1x128(x, ld_scale=260)
    assert s2.shape == (3, 260) and calls[-1][1][7] == 260
    fq.quant_act_1x128(x, out=(q, s))                       # the bench's reuse
    assert calls[-1][1][7] == 256
    padded = E(3, 264, dtype=f32)
    fq.quant_act_1x128(x, out=(q, padded))
    assert calls[-1][1][7] == 264                           # the buffer's pitch, not M
    fq.quant_act_1x128(x, out=(q.view(torch.float8_e4m3fn), s))
    with pytest.raises(ValueError, match="ld_scale"):
        fq.quant_act_1x128(x, ld_scale=256, out=(q, padded))
    with pytest.raises(ValueError, match="at least"):
        fq.quant_act_1x128(x, out=(q, E(3, 255, dtype=f32)))
    with pytest.raises(ValueError, match="at least"):
        fq.quant_act_1x128(x, out=(E(255, 384), s))
    with pytest.raises(TypeError):
        fq.quant_act_1x128(x, out=(q, E(3, 256, dtype=bf16)))
    with pytest.raises(ValueError, match="is on"):
        fq.quant_act_1x128(x, out=(q, torch.empty((3, 256), dtype=f32, device="meta")))


def test_quant_dual_outputs(calls):
    x = E(256, 384, dtype=bf16)
    bufs = fq.quant_act_dual(x)
    assert [tuple(t.shape) for t in bufs] == [(256, 384), (3, 256), (384, 256), (2, 384)]
    fq.quant_act_dual(x, out=bufs)
    q, s, qt, st = bufs
    for bad in ((q, s, E(384, 255), st), (q, s, qt, E(1, 384, dtype=f32)),
                (E(256, 383), s, qt, st)):
        with pytest.raises(ValueError):
            fq.quant_act_dual(x, out=bad)


def test_quant_weight_and_transpose_blocks(calls):
    w = E(256, 384, dtype=bf16)
    q, s = fq.quant_weight_128x128(w)
    assert s.shape == (2, 3)
    fq.quant_weight_128x128(w, out=(q, s))
    with pytest.raises(ValueError):                         # row pitch K is implied
        fq.quant_weight_128x128(w, out=(E(256, 512)[:, :384], s))
    q3, s3 = fq.quant_weight_128x128(E(2, 256, 384, dtype=bf16))
    assert s3.shape == (2, 2, 3)
    with pytest.raises(ValueError):
        fq.quant_weight_128x128(E(2, 256, 384, dtype=bf16), out=(q3, s))
    qt, st = fq.transpose_blocks(q, s)
    assert qt.shape == (384, 256) and st.shape == (3, 2)
    fq.transpose_blocks(q, s, out=(qt, st))
    with pytest.raises(ValueError):
        fq.transpose_blocks(q, s.t())                       # not contiguous
    with pytest.raises(ValueError):
        fq.transpose_blocks(q, s, out=(qt, E(2, 3, dtype=f32)))


@pytest.mark.parametrize("gemm", [fq.gemm_blockscaled, fq.gemm_blockscaled_ue8m0])
def test_dense_gemm_operands(calls, gemm):
    qa, sa = E(256, 384), E(3, 256, dtype=f32)
    qb, sb = E(512, 384), E(4, 3, dtype=f32)
    C = gemm(qa, sa, qb, sb)
    assert C.shape == (256, 512) and C.dtype == bf16
    gemm(qa, sa, qb, E(3, 512, dtype=f32), b_rowwise=True)
    gemm(qa, E(3, 260, dtype=f32), qb, sb)                  # padded activation scales
    gemm(qa, sa, qb, sb, out=E(300, 512, dtype=f32))        # more rows than M
    gemm(qa.view(torch.float8_e4m3fn), sa, qb.view(torch.float8_e4m3fn), sb)
    for kw in (dict(sa=E(3, 255, dtype=f32)), dict(sa=E(2, 256, dtype=f32)),
               dict(sb=E(4, 4, dtype=f32)), dict(sb=E(3, 4, dtype=f32)),
               dict(out=E(256, 511, dtype=f32)), dict(qb=E(512, 256))):
        args = dict(qa=qa, sa=sa, qb=qb, sb=sb) | {k: v for k, v in kw.items() if k != "out"}
        with pytest.raises(ValueError):
            gemm(args["qa"], args["sa"], args["qb"], args["sb"], out=kw.get("out"))
    with pytest.raises(ValueError):
        gemm(qa, sa, qb, E(3, 511, dtype=f32), b_rowwise=True)
    with pytest.raises(TypeError):
        gemm(qa, sa, qb, sb, out=E(256, 512, dtype=torch.float16))
    with pytest.raises(ValueError, match="is on"):
        gemm(qa, sa, torch.empty((512, 384), dtype=u8, device="meta"), sb)


@pytest.mark.parametrize("gemm", [fq.gemm_grouped, fq.gemm_grouped_ue8m0])
def test_grouped_gemm_operands(calls, gemm):
    qa, sa = E(300, 256), E(2, 300, dtype=f32)
    qw, sw = E(3, 128, 256), E(3, 1, 2, dtype=f32)
    off = torch.tensor([0, 3, 3, 300], dtype=i32)
    C = gemm(qa, sa, qw, sw, off)
    assert C.shape == (300, 128)
    gemm(qa, sa, qw, sw, off, out_dtype=f32, out=E(340, 128, dtype=f32))   # slack rows
    gemm(E(0, 256), E(2, 0, dtype=f32), qw, sw, torch.zeros(4, dtype=i32))  # no tokens
    for args in ((qa, sa, qw, E(3, 2, 2, dtype=f32), off), (qa, sa, qw, sw, off[:3]),
                 (qa, E(2, 299, dtype=f32), qw, sw, off), (qa, sa, E(3, 128, 384), sw, off)):
        with pytest.raises(ValueError):
            gemm(*args)
    with pytest.raises(ValueError):
        gemm(qa, sa, qw, sw, off, out=E(300, 127, dtype=bf16))


def test_nopromo_operands(calls):
    qa, qb = E(256, 384), E(512, 384)
    C = fq.gemm_nopromo(qa, E(256, dtype=f32), qb, E(512, dtype=f32))
    assert C.shape == (256, 512) and C.dtype == f32
    with pytest.raises(ValueError):
        fq.gemm_nopromo(qa, E(256, dtype=f32), qb, E(511, dtype=f32))
    with pytest.raises(TypeError):                           # the accumulator is written as fp32
        fq.gemm_nopromo(qa, E(256, dtype=f32), qb, E(512, dtype=f32), out=E(256, 512, dtype=bf16))
    with pytest.raises(ValueError):
        fq.gemm_nopromo(qa, E(256, dtype=f32), qb, E(512, dtype=f32), out=E(255, 512, dtype=f32))


@pytest.mark.parametrize("pow2", [False, True])
def test_fp8_linear_wiring(calls, pow2):
    """Forward: the dual quantization of X, the weight quantization and the Fprop GEMM;
    backward: the dual quantization of dY, the transposed weight blocks, Dgrad and Wgrad
    (ROW-mode B scales) -- seven calls whose operands all pass the checks."""
    from fp8_fine_grained_weight_b200.linear import fp8_linear
    T, K, N = 256, 384, 512
    x = torch.zeros(T, K, dtype=bf16, requires_grad=True)
    w = torch.zeros(N, K, dtype=bf16, requires_grad=True)
    y = fp8_linear(x, w, pow2)
    assert y.shape == (T, N)
    y.backward(torch.zeros(T, N, dtype=bf16))
    assert x.grad.shape == (T, K) and w.grad.shape == (N, K)
    gemm = "fp8_gemm_blockscaled_ue8m0" if pow2 else "fp8_gemm_blockscaled_ws"
    assert [c[0] for c in calls] == ["fp8q_quant_act_dual", "fp8q_quant_weight_128x128", gemm,
                                     "fp8q_quant_act_dual", "fp8q_transpose_blocks", gemm, gemm]
    # Wgrad: B scales in ROW mode (mode argument 1) with the transposed copy's pitch K
    assert calls[-1][1][6] == fq.BSCALE_ROW and calls[-1][1][5] == K


def test_split_workspace_is_per_stream(calls, monkeypatch):
    """The cached split-K workspace is keyed by (device, stream): GEMMs on one stream share
    it (they run in order), GEMMs on different streams never do."""
    monkeypatch.setattr(fq, "workspace_bytes", lambda M, N, K: 4096)
    monkeypatch.setattr(fq, "_WORKSPACE", collections.OrderedDict())
    qa, sa, qb, sb = E(256, 384), E(3, 256, dtype=f32), E(512, 384), E(4, 3, dtype=f32)
    ptrs = []
    for stream in (11, 11, 22):
        monkeypatch.setattr(fq, "_stream", lambda t, s=stream: s)
        fq.gemm_blockscaled(qa, sa, qb, sb)
        name, args = calls[-1]
        assert name == "fp8_gemm_blockscaled_ws" and args[-1] == stream and args[-2] >= 4096
        ptrs.append(args[-3])
    assert ptrs[0] == ptrs[1] != ptrs[2]
    own = E(8192)
    fq.gemm_blockscaled(qa, sa, qb, sb, workspace=own)       # a caller's buffer is used as is
    assert calls[-1][1][-3] == own.data_ptr()



def test_split_workspace_cache_is_bounded(calls, monkeypatch):
    """At most _WORKSPACE_MAX per-stream buffers are cached; the least recently used one is
    dropped first, and a stream that comes back gets a fresh buffer."""
    monkeypatch.setattr(fq, "workspace_bytes", lambda M, N, K: 4096)
    monkeypatch.setattr(fq, "_WORKSPACE", collections.OrderedDict())
    monkeypatch.setattr(fq, "_WORKSPACE_MAX", 3)
    qa, sa, qb, sb = E(256, 384), E(3, 256, dtype=f32), E(512, 384), E(4, 3, dtype=f32)

    def on(stream):
        monkeypatch.setattr(fq, "_stream", lambda t, s=stream: s)
        fq.gemm_blockscaled(qa, sa, qb, sb)
        return calls[-1][1][-3]

    first = on(1)
    for stream in (2, 3, 1, 4):            # stream 1 is used again, so 2 is the oldest
        on(stream)
    assert [k[1] for k in fq._WORKSPACE] == [3, 1, 4]
    assert on(1) == first                  # still cached
    on(2)                                  # evicted earlier: a new buffer, 3 drops out
    assert [k[1] for k in fq._WORKSPACE] == [4, 1, 2]
