"""lowbit_pack_ternary_noalloc against lowbit_pack (needs a B200).

The no-allocation entry point serves callers that cannot allocate device
memory when they pack weights: runtimes whose device-memory budget is fixed at
start-up, and hosts whose memory belongs to an allocator a C caller cannot
reach.  Its row-sum scratch is a static device array inside the library, so it
must produce exactly what lowbit_pack produces with a caller-provided
workspace, call after call, whatever an earlier call left in that array.

This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU runs deselect -m gpu
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binary_weight_transformer_b200 as bwt  # noqa: E402
from binary_weight_transformer_b200 import workloads as wls  # noqa: E402

DEV = "cuda:0"
MAX_ROWS = 65536  # LOWBIT_NOALLOC_MAX_ROWS in include/lowbit.h


@pytest.fixture(scope="module")
def lib():
    from binary_weight_transformer_b200 import _build
    _build.build()
    return bwt.lib()


def _noalloc(lib, w, eps, ldp):
    """Call the entry point through the C ABI with caller-owned outputs."""
    N, K = w.shape
    packed = torch.full((N, ldp), 0xA5, dtype=torch.uint8, device=DEV)  # stale bytes must be overwritten
    s_w = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    st = lib.lowbit_pack_ternary_noalloc(w.data_ptr(), N, K, w.stride(0), ctypes.c_float(eps), packed.data_ptr(),
                                         ldp, s_w.data_ptr(), status.data_ptr(),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    assert st == bwt.OK, bwt.STATUS_NAMES.get(st, st)
    assert status.item() == 0
    return packed, s_w


def _reference(w, eps, ldp):
    packed, s_w = bwt.lowbit_pack(w, bwt.TERNARY2, eps, ldp=ldp)
    torch.cuda.synchronize()
    return packed, s_w


def test_noalloc_matches_lowbit_pack_on_consecutive_calls(lib):
    # Two calls in a row: a large tensor, then a smaller one, so the second
    # call runs on an array still holding the first call's row sums.  The
    # codes, packed bytes and scale are integer or exact results, so the
    # comparison is bit for bit, the tolerance the other packer tests use.
    cases = [(9728, 2560, 1e-5, 0), (300, 1000, 0.0, 16)]
    for N, K, eps, extra in cases:
        w = torch.from_numpy(wls.normal_weights(N + K, N, K)).to(DEV)
        ldp = bwt.packed_ld(bwt.TERNARY2, K) + extra
        got_p, got_s = _noalloc(lib, w, eps, ldp)
        ref_p, ref_s = _reference(w, eps, ldp)
        assert torch.equal(got_p, ref_p), (N, K)
        assert got_s.cpu().numpy().view(np.uint32)[0] == ref_s.cpu().numpy().view(np.uint32)[0], (N, K)


def test_noalloc_rejects_more_rows_than_its_scratch(lib):
    N, K = MAX_ROWS + 1, 16
    w = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    packed = torch.empty((N, 16), dtype=torch.uint8, device=DEV)
    s_w = torch.empty(1, dtype=torch.float32, device=DEV)
    st = lib.lowbit_pack_ternary_noalloc(w.data_ptr(), N, K, K, ctypes.c_float(1e-5), packed.data_ptr(), 16,
                                         s_w.data_ptr(), None,
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bwt.ERR_INVALID_ARG
    # the largest accepted size still works
    w = torch.from_numpy(wls.normal_weights(7, MAX_ROWS, K)).to(DEV)
    got_p, got_s = _noalloc(lib, w, 1e-5, 16)
    ref_p, ref_s = _reference(w, 1e-5, 16)
    assert torch.equal(got_p, ref_p) and torch.equal(got_s, ref_s)
