"""Outlier study: one scale per tensor against 1x128 / 128x128 scaling, as the outliers grow.

TEST INFRASTRUCTURE (CPU only).  the-good.kr wr_id=2169793 para 4: mapping the whole
tensor's maximum to the FP8 maximum leaves low-precision training very sensitive to
activation outliers; pkd.ac.th webboard 78017 para 1: scaling at a finer grain instead.

A is drawn ~N(0, 1) and 0.1% of its entries (seeded positions) are multiplied by an
outlier factor f before the bf16 rounding (f = 100 is the workloads' recipe; 1 means no
outliers); B is the workload's weight matrix.  C = A B^T is formed in FP64 from the bf16
inputs (exact), from fine-grained codes (A 1x128, B 128x128) and from per-tensor codes.
Per method and f:
  c_rel_frobenius  ||C_q - C||_F / ||C||_F
  bulk_rel_error   ||A_q - A||_F / ||A||_F over the entries that are not outliers
  bulk_zero_share  share of the non-outlier nonzero entries of A whose code is zero
Run:  python -m oracle.outlier_study   (prints a JSON table; under a minute).
"""
import json

import numpy as np

import oracle
import workloads

FACTORS = (1.0, 100.0, 1e3, 1e4, 1e5)


def _with_outliers(rng, shape, factor, frac=0.001):
    x = workloads.bf16_bits_to_fp32(workloads.normal_bf16(rng, shape, 1.0, 0.0)).copy()
    n = int(round(frac * x.size))
    pos = rng.choice(x.size, size=n, replace=False)
    mask = np.zeros(x.size, bool)
    mask[pos] = True
    mask = mask.reshape(shape)
    x[mask] *= np.float32(factor)
    return workloads.fp32_to_bf16_bits(x), mask


def _errors(a_bits, mask, b_bits):
    A = workloads.bf16_bits_to_fp32(a_bits).astype(np.float64)
    B = workloads.bf16_bits_to_fp32(b_bits).astype(np.float64)
    C = A @ B.T
    tab = oracle.decode_table()
    qa, sa = oracle.quant_act_1x128(a_bits, False)
    qb, sb = oracle.quant_weight_128x128(b_bits, False)
    qa_t, s_a = oracle.quant_tensorwise(a_bits)
    qb_t, s_b = oracle.quant_tensorwise(b_bits)
    methods = {"fine": (oracle.dequant_rows_groupmajor(qa, sa), oracle.dequant_blocks(qb, sb), qa),
               "tensor": (tab[qa_t] * s_a, tab[qb_t] * s_b, qa_t)}
    bulk = ~mask
    nz = bulk & (A != 0)
    res = {}
    for name, (Ad, Bd, q) in methods.items():
        res[name] = {
            "c_rel_frobenius": float(np.linalg.norm(Ad @ Bd.T - C) / np.linalg.norm(C)),
            "bulk_rel_error": float(np.linalg.norm((Ad - A)[bulk]) / np.linalg.norm(A[bulk])),
            "bulk_zero_share": float(np.mean(tab[q][nz] == 0)),
        }
    return res


def study(M, b_bits, seed, factors=FACTORS):
    out = {}
    for f in factors:
        a, mask = _with_outliers(np.random.default_rng(seed), (M, b_bits.shape[1]), f)
        out[f"x{f:g}"] = _errors(a, mask, b_bits)
    return out


def study_tiny():
    """A [128, 512] against the tiny workload's B [256, 512]."""
    return study(128, workloads.tiny().gen_b(), 11)


def study_dense(n_rows=64):
    """n_rows x 7168 activations against the dense workload's W [7168, 7168]."""
    return study(n_rows, workloads.dense().gen_b(), 12)


if __name__ == "__main__":
    print(json.dumps({"tiny": study_tiny(), "dense_64_rows": study_dense()}, indent=1))
