"""Shared helpers of the GPU parity tests (test infrastructure)."""
import numpy as np

import oracle
import workloads


def to_dev_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return workloads.bf16_bits_to_fp32(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.cpu().numpy()


def assert_bytes_equal(name, got: np.ndarray, want: np.ndarray):
    """Bit-exact comparison with a report of the first mismatches (row, col, got, want)."""
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    if got.dtype == np.float32:
        got, want = got.view(np.uint32), want.view(np.uint32)
    bad = np.argwhere(got != want)
    if bad.size:
        first = [(tuple(int(i) for i in b), hex(int(got[tuple(b)])), hex(int(want[tuple(b)])))
                 for b in bad[:8]]
        raise AssertionError(f"{name}: {len(bad)} mismatches of {got.size}; first {first}")


def assert_gemm_close(name, C: np.ndarray, C_ref: np.ndarray, T: np.ndarray, bf16: bool):
    """The acceptance band: fp32 |C-C_ref| <= 2e-5 T + 1e-30; bf16 1 ulp (cancellation fallback)."""
    C = np.asarray(C, dtype=np.float64)
    if bf16:
        ok, fb = oracle.check_bf16(C, C_ref, T)
    else:
        ok = oracle.check_fp32(C, C_ref, T)
        fb = np.zeros_like(ok)
    if not ok.all():
        bad = np.argwhere(~ok)
        first = [(tuple(int(i) for i in b), float(C[tuple(b)]), float(C_ref[tuple(b)]),
                  float(T[tuple(b)])) for b in bad[:8]]
        raise AssertionError(f"{name}: {len(bad)} of {C.size} outside the band; first "
                             f"(idx, C, C_ref, T) {first}")
    return int(fb.sum())


def rel_err_stats(C, C_ref, T):
    e = np.abs(np.asarray(C, np.float64) - C_ref) / np.maximum(T, 1e-300)
    return float(e.max()), float(np.median(e))
