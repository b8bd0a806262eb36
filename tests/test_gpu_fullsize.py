"""Bit-exact parity of the dispatched kernels at the workloads' full sizes
(needs a B200).

Every point of every workload runs as bench.py launches it: lowbit_bitlinear
(the workload's activation prologue and per-token codes, then the linear
layer with the automatic kernel choice and LOWBIT_LINEAR_WEIGHTS_STABLE; one
fused kernel up to 4 tokens), here with the codes and scales also written
out so that they can be compared.  At these sizes
the persistent GEMMs run several output tiles per CTA (or SM pair), so the
second tensor-memory accumulator buffer and the phase flips of their barriers
are exercised.

Checks per point:
  * packed bytes and weight scales equal the oracle's;
  * int8 codes of every row equal the oracle's, and so do the scales s_x
    (to 1e-6 relative after an RMSNorm, whose fp64 sum of squares is
    reduced in another order);
  * int32 accumulators (LOWBIT_I32 output) of the first and last row of every
    256-token tile plus 32 random rows, over all N columns, equal the oracle's
    add/sub/skip integer dot on those rows;
  * every int32 accumulator equals the exact integer product of the oracle's
    codes, computed as a float64 matrix product: each term is an integer of
    magnitude at most 127 * 7 and every partial sum stays below 2^53, so the
    float64 result is the exact integer whatever the summation order;
  * the workload's own output dtype (fp32 or bf16) equals the oracle's
    rescale of those accumulators with the same scales bit for bit, and the
    oracle's rescale with its own scales within the stated tolerances
    (1e-6 relative for fp32, 1 ulp for bf16).
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
TILE = 256


def bf16_ulps(a_bits, b_bits):
    """Distance in bf16 units in the last place (monotone integer mapping)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


@pytest.fixture(scope="module", autouse=True)
def built():
    from binary_weight_transformer_b200 import _build
    _build.build()
    oracle.build()
    bwt.lib()


def tile_edge_rows(M, n_random=32, seed=0):
    """First and last row of every 256-token tile, plus random rows."""
    rows = set()
    for t0 in range(0, M, TILE):
        rows.add(t0)
        rows.add(min(t0 + TILE, M) - 1)
    rng = np.random.default_rng(seed + M)
    rows |= set(rng.choice(M, size=min(n_random, M), replace=False).tolist())
    return np.array(sorted(rows))


def exact_int_product(q, codes):
    """acc = q @ codes^T as exact integers via float64 (see module doc)."""
    a = torch.from_numpy(q.astype(np.float64))
    b = torch.from_numpy(codes.astype(np.float64))
    return (a @ b.T).numpy()


class Packed:
    """A matrix packed on the GPU with the workload's quantiser, checked
    against the oracle's codes and scales."""

    def __init__(self, wl, mi):
        m = wl.matrices[mi]
        w = wls.workload_weights(wl, mi)
        wt = torch.from_numpy(w).to(DEV)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        if wl.quantizer == "centred":
            self.packed, self.s_w = bwt.lowbit_pack_ex(wt, wl.fmt, bwt.QUANT_BINARY_CENTRED, status=st)
            self.codes, beta, _ = oracle.binary_centred_codes(w)
            self.s_wo = np.full(m.N, beta[0], np.float32)
        else:
            self.packed, self.s_w = bwt.lowbit_pack(wt, wl.fmt, 1e-5, status=st)
            self.codes, self.s_wo = oracle.quantize(w, wl.fmt, 1e-5)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert np.array_equal(self.packed.cpu().numpy(), oracle.pack(self.codes, wl.fmt, self.packed.shape[1]))
        assert np.array_equal(self.s_w.cpu().numpy().view(np.uint32), self.s_wo.view(np.uint32))
        if wl.quantizer == "onebit":
            # OneBit: the per-row scale is the output value vector
            self.s_wo = wls.workload_output_vector(wl, mi)
            self.s_w = torch.from_numpy(self.s_wo).to(DEV)
        g = wls.workload_gain(wl, mi)
        self.g = g
        self.g_dev = None if g is None else torch.from_numpy(g).to(DEV)
        self.m = m


def check_point(wl, mi, pk, M, full_product=True):
    """One point through lowbit_bitlinear (one fused kernel up to 4 tokens,
    else the prologue kernel and the linear kernel), as bench.py runs it."""
    m = pk.m
    bf = wl.x_dtype == wls.BF16
    norm = bwt.NORM_RMS if wl.norm else bwt.NORM_NONE
    x = wls.workload_activations(wl, mi, M)
    if bf:
        xt = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    else:
        xt = torch.from_numpy(x).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    y32, q, s_x = bwt.lowbit_bitlinear(xt, pk.packed, pk.s_w, wl.fmt, m.N, bwt.I32, pk.g_dev, norm, 1e-5,
                                       wl.hadamard, want_codes=True, status=st, weights_stable=True)
    yo = bwt.lowbit_bitlinear(xt, pk.packed, pk.s_w, wl.fmt, m.N, wl.y_dtype, pk.g_dev, norm, 1e-5, wl.hadamard,
                              status=st, weights_stable=True)
    torch.cuda.synchronize()
    assert st.item() == 0, bwt.status_flags(st)

    q_o, s_xo = oracle.act_prologue(x, pk.g, wl.norm, 1e-5, wl.hadamard, bf16_bits=bf)
    q_g = q.cpu().numpy()[:, :m.K]
    assert np.array_equal(q_g, q_o), (wl.name, mi, M)
    s_g = s_x.cpu().numpy()
    if wl.norm:
        # the fp64 sum of squares is reduced in another order: 1e-6 relative
        assert np.max(np.abs(s_g.astype(np.float64) - s_xo) / np.maximum(s_xo, 1e-38)) <= 1e-6
    else:
        assert np.array_equal(s_g.view(np.uint32), s_xo.view(np.uint32)), (wl.name, mi, M)

    acc_g = y32.cpu().numpy().astype(np.int64)
    rows = tile_edge_rows(M, seed=mi)
    acc_o = oracle.int_dot(q_o[rows], pk.codes, wl.fmt, nthreads=oracle.max_threads())
    assert np.array_equal(acc_g[rows], acc_o), (wl.name, mi, M, "sampled rows")
    if full_product:
        exact = exact_int_product(q_o, pk.codes)
        assert np.array_equal(acc_g, exact.astype(np.int64)), (wl.name, mi, M, "all rows")
        acc_all, s_ref = acc_g, s_xo
    else:
        acc_all, s_ref = acc_g[rows], s_xo[rows]
    out = "bf16" if wl.y_dtype == wls.BF16 else "f32"
    # the output is checked against the oracle's rescale of the same
    # accumulators with the GPU's own row scales (bit for bit) and with the
    # oracle's (to the stated tolerance)
    s_gr = s_g if full_product else s_g[rows]
    ref_same = oracle.rescale(acc_all, pk.s_wo, s_gr, out)
    ref = oracle.rescale(acc_all, pk.s_wo, s_ref, out)
    if out == "bf16":
        got = yo.view(torch.int16).cpu().numpy().view(np.uint16)
        got = got if full_product else got[rows]
        assert np.array_equal(got, ref_same), (wl.name, mi, M, out)
        assert bf16_ulps(got, ref).max() <= 1
    else:
        got = yo.cpu().numpy()
        got = got if full_product else got[rows]
        assert np.array_equal(got.view(np.uint32), ref_same.view(np.uint32)), (wl.name, mi, M, out)
        assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)) <= 1e-6


@pytest.mark.parametrize("mi", [0, 1], ids=["2560->9728", "9728->2560"])
def test_ternary_4b_all_points(mi):
    wl = wls.WORKLOADS["ternary_4b"]
    pk = Packed(wl, mi)
    for M in wl.Ms:
        check_point(wl, mi, pk, M)


@pytest.mark.parametrize("mi", [0, 1], ids=["1280->3584", "3584->1280"])
def test_t4nt_int4_all_points(mi):
    wl = wls.WORKLOADS["t4nt_int4"]
    pk = Packed(wl, mi)
    for M in wl.Ms:
        check_point(wl, mi, pk, M)


def test_impeto_binary_all_matrices():
    wl = wls.WORKLOADS["impeto_binary"]
    for mi in range(len(wl.matrices)):
        pk = Packed(wl, mi)
        for M in wl.Ms:
            check_point(wl, mi, pk, M)


def test_atomic_stack_all_matrices():
    wl = wls.WORKLOADS["atomic_stack"]
    for mi in range(len(wl.matrices)):
        pk = Packed(wl, mi)
        for M in wl.Ms:
            check_point(wl, mi, pk, M)


def test_single_ternary():
    wl = wls.WORKLOADS["single_ternary"]
    pk = Packed(wl, 0)
    for M in wl.Ms:
        check_point(wl, 0, pk, M)


@pytest.mark.parametrize("mi", [0, 1], ids=["2560->9728", "9728->2560"])
def test_ternary_4b_rmsnorm_all_points(mi):
    wl = wls.WORKLOADS["ternary_4b_rmsnorm"]
    pk = Packed(wl, mi)
    for M in wl.Ms:
        check_point(wl, mi, pk, M)


def test_bitnet_v1_binary_all_matrices():
    wl = wls.WORKLOADS["bitnet_v1_binary"]
    for mi in range(len(wl.matrices)):
        pk = Packed(wl, mi)
        for M in wl.Ms:
            check_point(wl, mi, pk, M)


def test_onebit_4096_all_points():
    wl = wls.WORKLOADS["onebit_4096"]
    pk = Packed(wl, 0)
    for M in wl.Ms:
        check_point(wl, 0, pk, M)


@pytest.mark.parametrize("mi", [0, 1], ids=["9728->2560", "2560->2560"])
def test_h_bitlinear_4b_all_points(mi):
    wl = wls.WORKLOADS["h_bitlinear_4b"]
    pk = Packed(wl, mi)
    for M in wl.Ms:
        check_point(wl, mi, pk, M)
