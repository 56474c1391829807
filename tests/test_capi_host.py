"""Host-only checks of the C ABI: the library loads, exports every function that
include/fp8q.h declares, and rejects bad arguments before any launch.

No call here reaches a kernel launch or any CUDA call (validation returns first), so
these run on a machine without a GPU.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")


@pytest.fixture(scope="module")
def L():
    from fp8_fine_grained_weight_b200 import build
    build.build()
    import fp8_fine_grained_weight_b200 as fq
    return fq.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:fp8q|fp8)_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    for want in ("fp8q_quant_act_1x128", "fp8q_quant_weight_128x128", "fp8_gemm_blockscaled",
                 "fp8_gemm_grouped", "fp8q_get_device_error", "fp8q_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(L):
    import fp8_fine_grained_weight_b200 as fq
    for name in declared_functions():
        assert hasattr(L, name), name
        assert name in fq.SIGNATURES, f"binding lacks {name}"


def declarations():
    """name -> (return type, [parameter types]) of every function the header declares."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for ret, name, params in re.findall(
            r"((?:const\s+)?[A-Za-z_]\w*\s*\**)\s*\b((?:fp8q|fp8)_[a-z0-9_]+)\s*\(([^)]*)\)\s*;", src):
        ps = [] if params.strip() in ("", "void") else [p.strip() for p in params.split(",")]
        types = [re.sub(r"\s*\b\w+$", "", p) if not p.endswith("*") else p for p in ps]
        out[name] = (ret.strip(), types)
    return out


def _ctype_of(c_type: str):
    c = " ".join(c_type.replace("*", " * ").split())
    if c == "size_t *":
        return ctypes.POINTER(ctypes.c_size_t)
    if c in ("const char *",):
        return ctypes.c_char_p
    if "*" in c:
        return ctypes.c_void_p
    return {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "uint64_t": ctypes.c_uint64,
            "size_t": ctypes.c_size_t, "float": ctypes.c_float}[c]


def test_binding_signatures_match_the_header():
    """Every ctypes signature in the binding has the header's arity and argument widths:
    a mismatch would pass garbage pointers or sizes into the library."""
    import fp8_fine_grained_weight_b200 as fq
    decl = declarations()
    assert set(decl) == set(declared_functions())
    for name, (ret, params) in decl.items():
        res, args = fq.SIGNATURES[name]
        assert res is _ctype_of(ret), (name, ret)
        want = [_ctype_of(p) for p in params]
        assert len(args) == len(want), (name, len(args), len(want))
        for i, (got, w) in enumerate(zip(args, want)):
            same = got is w or (getattr(got, "_type_", None) is getattr(w, "_type_", 0))
            assert same, (name, i, params[i], got, w)


def test_status_strings_and_version(L):
    assert L.fp8q_abi_version() == 1
    assert L.fp8q_status_string(0) == b"ok"
    assert b"timed out" in L.fp8q_status_string(6)
    assert L.fp8q_status_string(6 | (4 << 8)) == L.fp8q_status_string(6)
    assert b"power of two" in L.fp8q_status_string(7)
    assert L.fp8q_status_string(7 | (8 << 8)) == L.fp8q_status_string(7)
    assert L.fp8q_status_string(99) == b"unknown status"


NULL = None
P16 = 0x10000          # a fake, 16-byte aligned "device" address: never dereferenced
P_MIS = 0x10004        # misaligned by 4


def test_quant_act_validation(L):
    f = L.fp8q_quant_act_1x128
    assert f(P16, 0, 128, 128, P16, 128, P16, 0, 0, NULL) == 0          # empty: no-op
    assert f(P16, -1, 128, 128, P16, 128, P16, 1, 0, NULL) == 2
    assert f(NULL, 4, 128, 128, P16, 128, P16, 4, 0, NULL) == 1
    assert f(P16, 4, 100, 128, P16, 128, P16, 4, 0, NULL) == 2          # K % 128
    assert f(P16, 4, 128, 64, P16, 128, P16, 4, 0, NULL) == 2           # ldx < K
    assert f(P16, 4, 128, 128, P16, 128, P16, 3, 0, NULL) == 2          # ld_scale < M
    assert f(P_MIS, 4, 128, 128, P16, 128, P16, 4, 0, NULL) == 3        # x misaligned
    assert f(P16, 4, 128, 132, P16, 128, P16, 4, 0, NULL) == 3          # ldx % 8
    # one block per (64-row block, 128-column group) on a one-dimensional grid of at
    # most 2^31 - 1 blocks
    M = 64 << 30
    assert f(P16, M, 256, 256, P16, 256, P16, M, 0, NULL) == 2         # 2^31 blocks
    M = 64 << 31
    assert f(P16, M, 128, 128, P16, 128, P16, M, 0, NULL) == 2


def test_quant_dual_validation(L):
    f = L.fp8q_quant_act_dual

    def call(M=256, K=256, ldx=256, q=P16, ldq=256, s=P16, ld_s=256, qt=P16, ldqt=256, st=P16,
             ld_st=256, x=P16):
        return f(x, M, K, ldx, q, ldq, s, ld_s, qt, ldqt, st, ld_st, 0, NULL)

    assert call(M=0) == 0                       # empty: no-op
    assert call(M=-1) == 2
    assert call(qt=NULL) == 1
    assert call(M=200, ld_s=256, ldqt=256) == 2  # M % 128: the transposed K
    assert call(K=200) == 2
    assert call(ldqt=128) == 2                  # ldqt < M
    assert call(ld_st=128) == 2                 # ld_st < K
    assert call(ldqt=264) == 3                  # 16-byte row starts of qt
    assert call(qt=P_MIS) == 3
    assert call(x=P_MIS) == 3
    M = 128 << 30                               # 2^30 row tiles x 2 groups = 2^31 blocks
    assert call(M=M, ld_s=M, ldqt=M) == 2


def test_quant_weight_validation(L):
    f = L.fp8q_quant_weight_128x128
    assert f(P16, 0, 128, 128, P16, 128, P16, 0, NULL) == 0
    assert f(P16, 100, 128, 128, P16, 128, P16, 0, NULL) == 2           # N % 128
    assert f(P16, 128, 128, 128, NULL, 128, P16, 0, NULL) == 1
    assert f(P_MIS, 128, 128, 128, P16, 128, P16, 0, NULL) == 3


@pytest.mark.parametrize("entry", ["fp8_gemm_blockscaled", "fp8_gemm_blockscaled_ue8m0"])
def test_gemm_validation(L, entry):
    f = getattr(L, entry)
    ok_args = dict(A=P16, sA=P16, ld_sa=256, B=P16, sB=P16, ld_sb=0, mode=0, C=P16, out=0,
                   M=256, N=256, K=256, lda=256, ldb=256, ldc=256)

    def call(**kw):
        a = dict(ok_args, **kw)
        return f(a["A"], a["sA"], a["ld_sa"], a["B"], a["sB"], a["ld_sb"], a["mode"], a["C"],
                 a["out"], a["M"], a["N"], a["K"], a["lda"], a["ldb"], a["ldc"], NULL)

    assert call(M=0) == 0                      # empty problem: no-op
    assert call(A=NULL) == 1
    assert call(sB=NULL) == 1
    assert call(K=200, lda=256, ldb=256) == 2  # K % 128
    assert call(N=200) == 2                    # N % 128
    assert call(M=-5) == 2
    assert call(lda=128) == 2                  # lda < K
    assert call(ld_sa=100) == 2                # ld_sa < M
    assert call(mode=1, ld_sb=100) == 2        # ROW mode needs ld_sb >= N
    assert call(mode=7) == 4
    assert call(out=3) == 4
    assert call(A=P_MIS) == 3
    assert call(lda=264) == 3                  # not a multiple of 16
    assert call(ldc=260, out=0) == 3           # 520 B row pitch is not a multiple of 16


def test_gemm_quant_validation(L):
    f = L.fp8_gemm_blockscaled_quant
    ok_args = dict(A=P16, sA=P16, ld_sa=256, B=P16, sB=P16, ld_sb=0, mode=0, C=P16, ldc=256,
                   qC=P16, ldq=256, sC=P16, ld_sc=256, pow2=0, M=256, N=256, K=256, lda=256,
                   ldb=256)

    def call(**kw):
        a = dict(ok_args, **kw)
        return f(a["A"], a["sA"], a["ld_sa"], a["B"], a["sB"], a["ld_sb"], a["mode"], a["C"],
                 a["ldc"], a["qC"], a["ldq"], a["sC"], a["ld_sc"], a["pow2"], a["M"], a["N"],
                 a["K"], a["lda"], a["ldb"], NULL)

    assert call(M=0) == 0                      # empty problem: no-op
    assert call(A=NULL) == 1
    assert call(qC=NULL) == 1
    assert call(sC=NULL) == 1
    assert call(C=NULL, qC=NULL) == 1          # the codes are not optional
    assert call(N=200) == 2                    # N % 128
    assert call(ldq=128) == 2                  # ldq < N
    assert call(ld_sc=100) == 2                # ld_sc < M
    assert call(ldc=128) == 2                  # ldc < N (C given)
    assert call(ldq=264) == 3                  # not a multiple of 16
    assert call(qC=P_MIS) == 3
    assert call(ldc=260) == 3                  # 520 B row pitch is not a multiple of 16
    assert call(mode=7) == 4


@pytest.mark.parametrize("entry", ["fp8_gemm_grouped", "fp8_gemm_grouped_ue8m0"])
def test_grouped_validation(L, entry):
    f = getattr(L, entry)
    assert f(P16, P16, 64, P16, P16, P16, 0, P16, 0, 64, 256, 256, NULL) == 4      # no groups
    assert f(P16, P16, 64, P16, P16, P16, 0, P16, 2000, 64, 256, 256, NULL) == 4   # too many
    assert f(P16, P16, 64, P16, P16, P16, 0, P16, 4, 0, 256, 256, NULL) == 0       # empty
    assert f(P16, P16, 64, P16, P16, P16, 0, NULL, 4, 64, 256, 256, NULL) == 1
    assert f(P16, P16, 32, P16, P16, P16, 0, P16, 4, 64, 256, 256, NULL) == 2      # ld_sa
    assert f(P16, P16, 64, P16, P16, P16, 0, P16, 4, 64, 256, 200, NULL) == 2      # K


def test_nopromo_validation(L):
    f = L.fp8_gemm_nopromo
    assert f(P16, P16, P16, P16, P16, 0, 256, 256, 256, 256, 256, NULL) == 0
    assert f(P16, NULL, P16, P16, P16, 4, 256, 256, 256, 256, 256, NULL) == 1
    assert f(P16, P16, P16, P16, P16, 4, 250, 256, 256, 256, 256, NULL) == 2


def test_binding_refuses_cpu_tensors():
    torch = pytest.importorskip("torch")
    import fp8_fine_grained_weight_b200 as fq
    with pytest.raises(TypeError):
        fq.quant_act_1x128(torch.zeros(4, 128, dtype=torch.bfloat16))
