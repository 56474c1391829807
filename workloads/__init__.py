"""Seeded synthetic inputs for the five fine-grained FP8 workloads.

This module only *draws* inputs: normal samples, outlier positions, MoE
routing counts, and the bf16 bit patterns of those samples.  It holds none
of the quantization or GEMM arithmetic, so both the CPU oracle and the CUDA
path can take their inputs from here without sharing any of the method.

Every array is a numpy array on the host.  bf16 tensors are returned as
``uint16`` bit patterns (round-to-nearest-even from the fp32 samples), which
the caller hands to its own side unchanged.

Workload shapes.  The pages are cited by site and paragraph (paragraph n of
the post): the 1x128 activation tile / 128x128 weight block comes from
the-good.kr wr_id=2169793 para 4; 256 routed experts, 8 active per token and
expert intermediate size 2048 from why-be.co.kr wr_id=57820 para 2; the
at-most-256-token decode batch per expert from pkd.ac.th webboard 78017 para 3.
The widths 7168 / 16384 and the distributions are the workload definitions
of this project, not figures from the pages.

=========  ===============================================================
tiny       A [128, 512] ~N(0,1) + 0.1% outliers x100, B [256, 512] ~N(0,0.02)
dense      A [4096, 7168] ~N(0,1) + outliers, W [7168, 7168] ~N(0,0.006)
prefill    32 experts, W_e [4096, 7168] ~N(0,0.006), Zipf(1.1) top-8/256 routing
decode     64 experts, W_e [7168, 2048] ~N(0,0.006), M_e ~ U{1..256}
wgrad      dY [7168, 16384] ~N(0,1e-3), X [2048, 16384] ~N(0,1)
=========  ===============================================================

The second parameter of N(mu, sigma) is read as the standard deviation.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

SEED_BASE = 1000


def rng_for(config_index: int, stream: int = 0) -> np.random.Generator:
    """A PCG64 generator for workload ``config_index`` (1..5), sub-stream ``stream``."""
    return np.random.Generator(np.random.PCG64([SEED_BASE + config_index, stream]))


def fp32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 samples to bf16 (nearest, ties to even) and return the 16-bit patterns.

    This is input preparation: the synthetic tensors are *defined* as bf16.
    NaN never occurs in the generated data.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_fp32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float, outlier_frac: float = 0.0,
                outlier_mul: float = 100.0, chunk: int = 1 << 24) -> np.ndarray:
    """bf16 bits of N(0, std^2) samples; ``outlier_frac`` of the entries are multiplied by
    ``outlier_mul`` in fp32 before the bf16 rounding.

    Exactly ``round(outlier_frac * numel)`` distinct positions are taken from a seeded
    permutation.  Samples are drawn in fixed-size chunks so that memory stays bounded
    for the multi-GB workloads; the chunking is part of the seeded definition.
    """
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        x = rng.standard_normal(hi - lo, dtype=np.float32)
        x *= np.float32(std)
        out[lo:hi] = fp32_to_bf16_bits(x)
    n_out = int(round(outlier_frac * n))
    if n_out:
        pos = rng.permutation(n)[:n_out] if n <= (1 << 26) else _distinct_positions(rng, n, n_out)
        v = bf16_bits_to_fp32(out[pos]) * np.float32(outlier_mul)
        out[pos] = fp32_to_bf16_bits(v)
    return out.reshape(shape)


def _distinct_positions(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """k distinct positions in [0, n) without materialising a permutation of n."""
    chosen = np.unique(rng.integers(0, n, size=int(k * 1.1) + 16))
    while chosen.size < k:
        chosen = np.unique(np.concatenate([chosen, rng.integers(0, n, size=k)]))
    return rng.permutation(chosen)[:k]


def small_int_e4m3_codes(rng: np.random.Generator, shape, lo: int = -4, hi: int = 4) -> np.ndarray:
    """Uniform integers in [lo, hi] written as E4M3 bytes (the unit-scale tiny variant).

    Small integers are exact in E4M3: |v| <= 8 needs at most 3 mantissa bits.  The
    byte table below is the plain E4M3FN bit layout (sign | exponent+7 | mantissa)
    of each integer, spelled out so that this module needs no codec.
    """
    table = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48, 5: 0x4A, 6: 0x4C, 7: 0x4E, 8: 0x50}
    v = rng.integers(lo, hi + 1, size=shape)
    out = np.empty(v.shape, dtype=np.uint8)
    for k, code in table.items():
        out[v == k] = code
        if k:
            out[v == -k] = code | 0x80
    return out, v.astype(np.int64)


# ----------------------------------------------------------------------------------
# MoE routing counts
# ----------------------------------------------------------------------------------

def zipf_topk_counts(rng: np.random.Generator, tokens: int = 16384, experts: int = 256,
                     topk: int = 8, alpha: float = 1.1, chunk: int = 4096) -> np.ndarray:
    """Per-expert token counts of a top-k-of-E routing with Zipf(alpha) expert popularity.

    Popularity p_i is proportional to (i+1)^-alpha over expert ids in order.  Every token
    draws ``topk`` distinct experts without replacement with probabilities proportional to p
    (Gumbel-top-k).  Returns int64 counts of shape [experts].
    """
    logp = -alpha * np.log(np.arange(1, experts + 1, dtype=np.float64))
    counts = np.zeros(experts, dtype=np.int64)
    for lo in range(0, tokens, chunk):
        n = min(chunk, tokens - lo)
        g = rng.gumbel(size=(n, experts))
        keys = logp[None, :] + g
        top = np.argpartition(-keys, topk - 1, axis=1)[:, :topk]
        counts += np.bincount(top.ravel(), minlength=experts)
    return counts


def offsets_from_counts(counts) -> np.ndarray:
    """int32 prefix offsets [E+1] of per-expert row counts."""
    c = np.asarray(counts, dtype=np.int64)
    off = np.zeros(c.size + 1, dtype=np.int64)
    np.cumsum(c, out=off[1:])
    return off.astype(np.int32)


# ----------------------------------------------------------------------------------
# Workload descriptors
# ----------------------------------------------------------------------------------

@dataclasses.dataclass
class Workload:
    name: str
    index: int
    M: int                       # rows of A (sum over experts for grouped)
    N: int
    K: int
    pow2_a: bool
    pow2_b: bool
    out_fp32: bool
    b_rowwise: bool = False      # B quantized 1x128 along K (wgrad) instead of 128x128
    experts: int = 0             # 0 = dense
    counts: Optional[np.ndarray] = None
    a_std: float = 1.0
    b_std: float = 0.006
    a_outliers: float = 0.0
    draw_K: int = 0              # >0: draw at this K and keep the first K columns

    @property
    def offsets(self) -> Optional[np.ndarray]:
        return None if self.counts is None else offsets_from_counts(self.counts)

    @property
    def gemm_flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def gen_a(self, rows: Optional[int] = None) -> np.ndarray:
        """bf16 bits of A; with ``rows``, a shorter A from the same seeded stream.

        The normal samples of the shorter A are a prefix of the full draw; its outlier
        positions are drawn for its own size.
        """
        r = self.M if rows is None else rows
        kd = self.draw_K or self.K
        a = normal_bf16(rng_for(self.index, 1), (r, kd), self.a_std, self.a_outliers)
        return a if kd == self.K else np.ascontiguousarray(a[:, :self.K])

    def gen_b(self) -> np.ndarray:
        """bf16 bits of B / W: [N, K] dense, [E, N, K] grouped."""
        kd = self.draw_K or self.K
        shape = (self.N, kd) if not self.experts else (self.experts, self.N, kd)
        b = normal_bf16(rng_for(self.index, 2), shape, self.b_std)
        return b if kd == self.K else np.ascontiguousarray(b[..., :self.K])


def tiny() -> Workload:
    return Workload("tiny_128x256x512_fp32", 1, 128, 256, 512, False, False, True,
                    a_std=1.0, b_std=0.02, a_outliers=0.001)


def dense() -> Workload:
    return Workload("dense_4096x7168x7168_pow2_bf16", 2, 4096, 7168, 7168, True, True, False,
                    a_std=1.0, b_std=0.006, a_outliers=0.001)


def prefill_counts() -> np.ndarray:
    """Token counts of experts 0..31 (the 32 most popular ids) under the seeded routing."""
    return zipf_topk_counts(rng_for(3, 0))[:32]


def prefill() -> Workload:
    c = prefill_counts()
    return Workload("moe_prefill_32x4096x7168_bf16", 3, int(c.sum()), 4096, 7168, False, False,
                    False, experts=32, counts=c, a_std=1.0, b_std=0.006, a_outliers=0.001)


def decode_counts() -> np.ndarray:
    return rng_for(4, 0).integers(1, 257, size=64).astype(np.int64)


def decode() -> Workload:
    c = decode_counts()
    return Workload("moe_decode_64x7168x2048_pow2a_bf16", 4, int(c.sum()), 7168, 2048, True, False,
                    False, experts=64, counts=c, a_std=1.0, b_std=0.006)


def wgrad(K: int = 16384) -> Workload:
    """dY [7168, K] as A, X [2048, K] as B; both 1x128 along K; fp32 out.

    The K = 4096 / 8192 prefixes of the accumulation study are the first K columns of
    the K = 16384 tensors (same seeded draw, sliced).
    """
    return Workload(f"wgrad_7168x2048x{K}_fp32", 5, 7168, 2048, K, False, False, True,
                    b_rowwise=True, a_std=1e-3, b_std=1.0, draw_K=16384)


ALL = {"tiny": tiny, "dense": dense, "prefill": prefill, "decode": decode, "wgrad": wgrad}
