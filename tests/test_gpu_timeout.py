"""A pipeline wait that runs out, on a B200 (needs a GPU).

Every mbarrier wait in the tensor-core kernels is bounded.  On expiry the
kernel records LOWBIT_ERR_TIMEOUT in the caller's status word, lets the
copies and MMAs it already issued complete, frees its tensor memory and
returns, so the context stays usable.  Here the bound is lowered to one SM
cycle (lowbit_set_wait_limit): the first wait of the single-CTA shared-memory
GEMM that does not succeed at once runs out.  The test checks the status
word, then restores the bound and checks that a normal launch in the same
context is still bit-exact.  No GPU fault is involved: the kernel returns on
its own.
"""
import numpy as np
import pytest

import oracle
from binary_weight_transformer_b200 import workloads as wls

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - CPU runs deselect -m gpu
    pytest.skip("needs a CUDA device", allow_module_level=True)

import binary_weight_transformer_b200 as bwt  # noqa: E402

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def built():
    from binary_weight_transformer_b200 import _build
    _build.build()
    oracle.build()
    bwt.lib()
    yield
    bwt.set_wait_limit(0)


def test_wait_timeout_is_reported_and_the_context_survives():
    M, N, K = 256, 512, 256  # 4 output tiles, 2 K blocks: the single-CTA GEMM, no split
    fmt = bwt.TERNARY2
    assert bwt.linear_kernel(M, N, K, fmt, path=2) == "gemm_kernel"
    w = wls.normal_weights(6000, N, K)
    x = wls.normal_activations(6001, M, K)
    packed, s_w = bwt.lowbit_pack(torch.from_numpy(w).to(DEV), fmt)
    q, s_x = bwt.lowbit_act_quant(torch.from_numpy(x).to(DEV))
    torch.cuda.synchronize()

    bwt.set_wait_limit(1)
    try:
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        bwt.lowbit_linear(q, s_x, packed, s_w, fmt, N, bwt.I32, K=K, status=st, path=2)
        torch.cuda.synchronize()
        assert bwt.status_flags(st) == [bwt.ERR_TIMEOUT]
    finally:
        bwt.set_wait_limit(0)

    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    y = bwt.lowbit_linear(q, s_x, packed, s_w, fmt, N, bwt.I32, K=K, status=st, path=2)
    torch.cuda.synchronize()
    assert st.item() == 0
    codes, _ = oracle.quantize(w, fmt, 1e-5)
    q_o, _ = oracle.act_quant(x)
    assert np.array_equal(y.cpu().numpy().astype(np.int64), oracle.int_dot(q_o, codes, fmt))
