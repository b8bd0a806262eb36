"""The C ABI without a GPU: library loading, exported symbols, size helpers
and host-side argument checks.

No call here reaches a kernel launch: every call with fake device pointers
carries at least one argument the host rejects first.
"""
import ctypes
import os
import re

import pytest

import binary_weight_transformer_b200 as bwt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lowbit.h")
FAKE = 0x10000  # 64 KB-aligned, never dereferenced


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lowbit_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from binary_weight_transformer_b200 import _build
    _build.build()
    return bwt.lib()


def test_library_exports_every_declared_function(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    # and the binding types each of them
    assert set(names) <= set(bwt.ABI)


def test_size_helpers(lib):
    assert bwt.packed_row_bytes(bwt.TERNARY2, 2560) == 640
    assert bwt.packed_row_bytes(bwt.TERNARY2, 17) == 8  # 4 * ceil(17/16)
    assert bwt.packed_row_bytes(bwt.BINARY1, 17) == 3
    assert bwt.packed_row_bytes(bwt.INT4, 9) == 8
    assert bwt.packed_ld(bwt.BINARY1, 17) == 16
    assert bwt.packed_ld(bwt.INT4, 3584) == 1792
    assert bwt.packed_row_bytes(bwt.TERNARY2, 0) == 0
    assert bwt.scale_count(bwt.TERNARY2, 768) == 1
    assert bwt.scale_count(bwt.BINARY1, 768) == 768
    assert bwt.scale_count(bwt.INT4, 0) == 0
    assert bwt.max_k(bwt.TERNARY2) == 2**31 // (128 * 64) - 1
    assert bwt.max_k(bwt.INT4) == (2**31 - 1) // (128 * 16 * 7)
    assert lib.lowbit_pack_workspace_bytes(bwt.TERNARY2, 9728) == 9728 * 8
    assert lib.lowbit_pack_workspace_bytes(bwt.BINARY1, 9728) == 0
    assert lib.lowbit_status_string(7) == b"device pipeline wait timed out"
    assert lib.lowbit_version() >= 100


def _linear(lib, **kw):
    a = dict(q=FAKE, ldq=256, s_x=FAKE, M=4, K=256, packed=FAKE, ldp=64, s_w=FAKE, fmt=bwt.TERNARY2,
             N=8, y=FAKE, ydt=bwt.F32, ldy=8, path=0)
    a.update(kw)
    return lib.lowbit_linear_path(a["q"], a["ldq"], a["s_x"], a["M"], a["K"], a["packed"], a["ldp"], a["s_w"],
                                  a["fmt"], a["N"], a["y"], a["ydt"], a["ldy"], a["path"], None, None)


# (M, N, K, format, path, SMs) -> kernel, worked out by hand from the
# dispatch rules (tiles of 128 tokens x 256 features, K blocks of 128):
# GEMV up to 4 tokens; warp MMAs up to 16; the shared-memory GEMM below 512
# tokens, split over a cluster of C in {2, 4, 8} CTAs (the largest with
# tiles * C <= SMs and 2 K blocks per split) when twice its 128 x 256 tiles
# fit the SMs and K has at least 4 blocks; from 512, SM pairs for ternary
# weights (split-K kept when K >= 2048 and the GEMM splits) and the
# tensor-memory GEMM for the other formats.
DISPATCH = [
    ((1, 9728, 2560, bwt.TERNARY2, 0, 148), "gemv_smem_kernel/gemv_kernel"),
    ((4, 9728, 2560, bwt.TERNARY2, 0, 148), "gemv_smem_kernel/gemv_kernel"),
    ((16, 9728, 2560, bwt.TERNARY2, 0, 148), "skinny_mma_kernel/stream_mma_kernel"),
    ((8, 192, 768, bwt.BINARY1, 0, 148), "skinny_mma_kernel/stream_mma_kernel"),      # 96-byte rows
    ((16, 2560, 9728, bwt.TERNARY2, 0, 148), "skinny_mma_kernel/stream_mma_kernel"),  # 2432-byte rows
    ((17, 2560, 9728, bwt.TERNARY2, 0, 148), "gemm_splitk_kernel"),  # 10 tiles x 8
    ((128, 9728, 2560, bwt.TERNARY2, 0, 148), "gemm_splitk_kernel"),  # 38 tiles x 2
    ((256, 768, 192, bwt.TERNARY2, 0, 148), "gemm_kernel"),  # 2 K blocks: no split
    ((300, 9728, 2560, bwt.TERNARY2, 0, 148), "gemm_kernel"),  # 114 tiles: no split
    ((8192, 9728, 2560, bwt.TERNARY2, 0, 148), "gemm_pair_kernel"),
    ((1024, 2560, 9728, bwt.TERNARY2, 0, 148), "gemm_pair_kernel"),  # 80 tiles: no split
    ((512, 2560, 9728, bwt.TERNARY2, 0, 148), "gemm_splitk_kernel"),  # 40 tiles x 2, deep K
    ((512, 2560, 9728, bwt.TERNARY2, 0, 64), "gemm_pair_kernel"),    # 40 x 2 > 64 SMs: no split
    ((1024, 256, 1024, bwt.TERNARY2, 0, 148), "gemm_pair_kernel"),   # splits, but K < 2048
    ((8192, 1280, 3584, bwt.INT4, 0, 148), "gemm_ts_kernel"),
    ((512, 1280, 3584, bwt.INT4, 0, 148), "gemm_ts_kernel"),  # splits, but not ternary
    ((16384, 192, 768, bwt.BINARY1, 0, 148), "gemm_ts_kernel"),
    # forced paths
    ((300, 9728, 2560, bwt.TERNARY2, 1, 148), "gemv_smem_kernel/gemv_kernel"),
    ((8192, 9728, 2560, bwt.TERNARY2, 2, 148), "gemm_kernel"),
    ((2, 2560, 9728, bwt.TERNARY2, 2, 148), "gemm_splitk_kernel"),
    ((1, 9728, 2560, bwt.INT4, 3, 148), "gemm_ts_kernel"),
    ((64, 9728, 2560, bwt.BINARY1, 4, 148), "gemm_ts_pair_kernel"),
    ((16, 2560, 9728, bwt.TERNARY2, 5, 148), "skinny_mma_kernel/stream_mma_kernel"),
    ((1, 9728, 2560, bwt.TERNARY2, 6, 148), "gemm_pair_kernel"),
]


@pytest.mark.parametrize("args,name", DISPATCH)
def test_linear_kernel_dispatch(lib, args, name):
    assert bwt.linear_kernel(*args) == name


def test_linear_kernel_rejects_bad_arguments(lib):
    k = ctypes.c_int(0)
    q = lib.lowbit_linear_kernel
    assert q(16, 256, 256, bwt.TERNARY2, 7, 148, ctypes.byref(k)) == bwt.ERR_INVALID_ARG   # path
    assert q(17, 256, 256, bwt.TERNARY2, 5, 148, ctypes.byref(k)) == bwt.ERR_INVALID_ARG   # path 5, M > 16
    assert q(0, 256, 256, bwt.TERNARY2, 0, 148, ctypes.byref(k)) == bwt.ERR_INVALID_ARG
    assert q(16, 256, 0, bwt.TERNARY2, 0, 148, ctypes.byref(k)) == bwt.ERR_INVALID_ARG
    assert q(16, 256, 256, 3, 0, 148, ctypes.byref(k)) == bwt.ERR_INVALID_ARG             # format
    assert q(16, 256, 256, bwt.TERNARY2, 0, 148, None) == bwt.ERR_INVALID_ARG
    big = bwt.max_k(bwt.INT4) + 1
    assert q(16, 256, big, bwt.INT4, 0, 148, ctypes.byref(k)) == bwt.ERR_OVERFLOW_BOUND
    assert lib.lowbit_kernel_name(0) == b"unknown"


def test_linear_rejects_bad_arguments(lib):
    assert _linear(lib, q=None) == bwt.ERR_INVALID_ARG
    assert _linear(lib, M=0) == bwt.ERR_INVALID_ARG
    assert _linear(lib, N=-1) == bwt.ERR_INVALID_ARG
    assert _linear(lib, ldq=128) == bwt.ERR_INVALID_ARG          # ldq < K
    assert _linear(lib, ldy=7) == bwt.ERR_INVALID_ARG            # ldy < N
    assert _linear(lib, ldp=48) == bwt.ERR_INVALID_ARG           # ldp < row bytes
    assert _linear(lib, fmt=3) == bwt.ERR_INVALID_ARG
    assert _linear(lib, ydt=7) == bwt.ERR_INVALID_ARG
    assert _linear(lib, path=7) == bwt.ERR_INVALID_ARG
    assert _linear(lib, path=5, M=17) == bwt.ERR_INVALID_ARG   # warp-MMA kernel: M <= 16
    assert _linear(lib, q=FAKE + 8) == bwt.ERR_ALIGNMENT
    assert _linear(lib, ldq=264) == bwt.ERR_ALIGNMENT
    assert _linear(lib, ldp=72) == bwt.ERR_ALIGNMENT
    assert _linear(lib, y=FAKE + 2) == bwt.ERR_ALIGNMENT
    big = bwt.max_k(bwt.TERNARY2) + 1
    assert _linear(lib, K=big, ldq=(big + 15) // 16 * 16,
                   ldp=bwt.packed_ld(bwt.TERNARY2, big)) == bwt.ERR_OVERFLOW_BOUND
    k4 = bwt.max_k(bwt.INT4) + 1
    assert _linear(lib, fmt=bwt.INT4, K=k4, ldq=(k4 + 15) // 16 * 16,
                   ldp=bwt.packed_ld(bwt.INT4, k4)) == bwt.ERR_OVERFLOW_BOUND


def test_linear_ex_rejects_unknown_flags(lib):
    f = lib.lowbit_linear_ex
    args = [FAKE, 256, FAKE, 4, 256, FAKE, 64, FAKE, bwt.TERNARY2, 8, FAKE, bwt.F32, 8, 0]
    for flags in (4, 8, 0x80000000, 0xFFFFFFFF):
        assert f(*args, flags, None, None) == bwt.ERR_INVALID_ARG
    for flags in (bwt.EXCLUSIVE, bwt.WEIGHTS_STABLE | bwt.EXCLUSIVE):  # accepted: the call gets past the checks
        assert f(*args, flags, None, None) != bwt.ERR_INVALID_ARG
    bad = list(args)
    bad[0] = None                                   # q = NULL with a valid flag
    assert f(*bad, bwt.WEIGHTS_STABLE, None, None) == bwt.ERR_INVALID_ARG


def _group(lib, n=2, M=1, fmt=bwt.TERNARY2, ydt=bwt.BF16, flags=0, **item):
    """lowbit_bitlinear_group on fake device pointers (checks run before any
    device work, so nothing is dereferenced); item overrides apply to the
    last layer."""
    items = (bwt.BitlinearItem * max(n, 1))()
    for i in range(max(n, 1)):
        f = dict(x=FAKE, ldx=2560, g=None, packed=FAKE, ldp=640, s_w=FAKE, N=9728, K=2560, y=FAKE, ldy=9728,
                 q=None, ldq=0, s_x=None)
        if i == max(n, 1) - 1:
            f.update(item)
        items[i] = bwt.BitlinearItem(**f)
    return lib.lowbit_bitlinear_group(ctypes.cast(items, ctypes.c_void_p), n, M, bwt.BF16, bwt.NORM_NONE, 1e-5, fmt,
                                      ydt, flags, None, None)


def test_bitlinear_group_rejects_bad_arguments(lib):
    assert lib.lowbit_bitlinear_group(None, 1, 1, bwt.BF16, 0, 1e-5, bwt.TERNARY2, bwt.BF16, 0, None,
                                      None) == bwt.ERR_INVALID_ARG
    assert _group(lib, n=0) == bwt.ERR_INVALID_ARG
    assert _group(lib, n=bwt.GROUP_MAX + 1) == bwt.ERR_INVALID_ARG
    assert _group(lib, M=0) == bwt.ERR_INVALID_ARG
    assert _group(lib, M=5) == bwt.ERR_INVALID_ARG                  # decode only: M <= 4
    assert _group(lib, flags=2) == bwt.ERR_INVALID_ARG
    assert _group(lib, fmt=3) == bwt.ERR_INVALID_ARG
    assert _group(lib, ydt=7) == bwt.ERR_INVALID_ARG
    assert _group(lib, x=None) == bwt.ERR_INVALID_ARG
    assert _group(lib, y=None) == bwt.ERR_INVALID_ARG
    assert _group(lib, ldy=100) == bwt.ERR_INVALID_ARG              # ldy < N
    assert _group(lib, ldp=624) == bwt.ERR_INVALID_ARG              # ldp < row bytes
    assert _group(lib, ldx=2000) == bwt.ERR_INVALID_ARG             # ldx < K
    assert _group(lib, packed=FAKE + 8) == bwt.ERR_ALIGNMENT
    assert _group(lib, y=FAKE + 1) == bwt.ERR_ALIGNMENT
    assert _group(lib, q=FAKE, ldq=2560 + 8) == bwt.ERR_ALIGNMENT
    assert _group(lib, q=FAKE, ldq=16) == bwt.ERR_INVALID_ARG       # ldq < K
    # a layer longer than LOWBIT_FUSED_MAX_K makes the group run its prologue
    # kernel first, which needs every layer's q and s_x
    assert _group(lib) == bwt.ERR_INVALID_ARG
    assert _group(lib, q=FAKE, ldq=2560, s_x=FAKE) == bwt.ERR_INVALID_ARG   # the first layer has none
    # the codes of a layer must fit the kernel's staging: M * K_r <= 98304
    k = bwt.FUSED_MAX_BYTES + 128
    assert _group(lib, K=k, ldx=k, ldp=bwt.packed_ld(bwt.TERNARY2, k)) == bwt.ERR_UNSUPPORTED
    assert _group(lib, M=4, K=24576 + 128, ldx=24704,
                  ldp=bwt.packed_ld(bwt.TERNARY2, 24704)) == bwt.ERR_UNSUPPORTED


def test_act_quant_rejects_bad_arguments(lib):
    f = lib.lowbit_act_quant
    assert f(None, bwt.F32, 4, 64, 64, 0.0, FAKE, 64, FAKE, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, 5, 4, 64, 64, 0.0, FAKE, 64, FAKE, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, bwt.F32, 0, 64, 64, 0.0, FAKE, 64, FAKE, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, bwt.F32, 4, 64, 32, 0.0, FAKE, 64, FAKE, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, bwt.F32, 4, 64, 64, -1.0, FAKE, 64, FAKE, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, bwt.F32, 4, 64, 64, float("nan"), FAKE, 64, FAKE, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE + 2, bwt.F32, 4, 64, 64, 0.0, FAKE, 64, FAKE, None, None) == bwt.ERR_ALIGNMENT
    assert f(FAKE + 1, bwt.BF16, 4, 64, 64, 0.0, FAKE, 64, FAKE, None, None) == bwt.ERR_ALIGNMENT
    assert f(FAKE, bwt.F32, 4, 64, 64, 0.0, FAKE + 8, 64, FAKE, None, None) == bwt.ERR_ALIGNMENT
    assert f(FAKE, bwt.F32, 4, 64, 64, 0.0, FAKE, 72, FAKE, None, None) == bwt.ERR_ALIGNMENT


def test_pack_rejects_bad_arguments(lib):
    f = lib.lowbit_pack
    need = lib.lowbit_pack_workspace_bytes(bwt.TERNARY2, 8)
    ok = dict(w=FAKE, N=8, K=64, ldw=64, fmt=bwt.TERNARY2, eps=1e-5, packed=FAKE, ldp=16, s_w=FAKE,
              ws=FAKE, wsb=need)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return f(a["w"], a["N"], a["K"], a["ldw"], a["fmt"], a["eps"], a["packed"], a["ldp"], a["s_w"],
                 a["ws"], a["wsb"], None, None)
    assert call(w=None) == bwt.ERR_INVALID_ARG
    assert call(ldw=32) == bwt.ERR_INVALID_ARG
    assert call(ldp=8) == bwt.ERR_INVALID_ARG
    assert call(ws=None) == bwt.ERR_INVALID_ARG
    assert call(wsb=need - 1) == bwt.ERR_INVALID_ARG
    assert call(eps=-1e-5) == bwt.ERR_INVALID_ARG
    assert call(ldp=24) == bwt.ERR_ALIGNMENT
    assert call(packed=FAKE + 4) == bwt.ERR_ALIGNMENT


def test_unpack_rejects_bad_arguments(lib):
    f = lib.lowbit_unpack
    assert f(None, 16, 4, 64, bwt.TERNARY2, FAKE, 64, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, 16, 4, 64, bwt.TERNARY2, FAKE, 32, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, 8, 4, 64, bwt.TERNARY2, FAKE, 64, None, None) == bwt.ERR_INVALID_ARG
    assert f(FAKE, 24, 4, 64, bwt.TERNARY2, FAKE, 64, None, None) == bwt.ERR_ALIGNMENT


def test_oracle_and_library_share_no_code():
    # The oracle is a separate C file built by gcc; the CUDA library never
    # includes or links it, and it never includes the library's headers.
    orc = open(os.path.join(ROOT, "oracle", "lowbit_oracle.c")).read()
    includes = re.findall(r"^\s*#\s*include\s*[<\"]([^>\"]+)", orc, flags=re.M)
    assert sorted(includes) == ["math.h", "omp.h", "stdint.h", "stdlib.h", "string.h"]
    csrc = os.path.join(ROOT, "binary_weight_transformer_b200", "csrc")
    for fn in os.listdir(csrc):
        text = open(os.path.join(csrc, fn)).read()
        assert "oracle" not in text.lower(), fn
    pkg = os.path.join(ROOT, "binary_weight_transformer_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            assert "import oracle" not in open(os.path.join(pkg, fn)).read(), fn
