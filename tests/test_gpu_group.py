"""The grouped decode launch, lowbit_bitlinear_group, against the oracle
(needs a B200).

One launch computes several independent BitLinear layers on the same M <= 4
tokens.  Per layer, the codes and int32 accumulators must equal the oracle's
bit for bit; the scales and float outputs must too without the RMSNorm, and
within the prologue tests' tolerances with it (1e-6 relative for s_x and
fp32, 1 bf16 ulp), since the fp64 sum of squares is reduced in another
order.  The groups are chosen so that the persistent kernel runs a cluster
over several units and across layer boundaries.
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
FMTS = [bwt.TERNARY2, bwt.BINARY1, bwt.INT4]
FMT_IDS = {bwt.TERNARY2: "ternary", bwt.BINARY1: "binary", bwt.INT4: "int4"}


@pytest.fixture(scope="module", autouse=True)
def built():
    from binary_weight_transformer_b200 import _build
    _build.build()
    oracle.build()
    bwt.lib()


def bf16_ulps(a_bits, b_bits):
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


def to_dev(x, bf16):
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


class Layer:
    """One layer's host data, its packed weights on the device, and the
    oracle's codes."""

    def __init__(self, fmt, N, K, M, seed, bf16, use_g, w=None, x=None, g=None):
        self.fmt, self.N, self.K = fmt, N, K
        self.w = wls.normal_weights(seed, N, K) if w is None else w
        if x is None:
            x = wls.normal_activations(seed + 1, M, K, 0.005, 10.0)
            x = wls.to_bf16_bits(x) if bf16 else x
        self.x, self.bf16 = x, bf16
        self.g = (wls.gain_vector(seed + 2, K) if use_g else None) if g is None else g
        self.codes, self.s_w = oracle.quantize(self.w, fmt, 1e-5)
        self.packed, self.s_w_dev = bwt.lowbit_pack(torch.from_numpy(self.w).to(DEV), fmt, 1e-5)
        assert np.array_equal(self.s_w_dev.cpu().numpy(), self.s_w)
        self.x_dev = to_dev(x, bf16)
        self.g_dev = None if self.g is None else torch.from_numpy(self.g).to(DEV)


def run_group(layers, fmt, out, norm, weights_stable=False):
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    args = ([L.x_dev for L in layers], [L.packed for L in layers], [L.s_w_dev for L in layers], fmt,
            [L.N for L in layers])
    gs = [L.g_dev for L in layers]
    y32, q, s_x = bwt.lowbit_bitlinear_group(*args, bwt.I32, gs, norm, 1e-5, want_codes=True, status=st,
                                             weights_stable=weights_stable)
    y = bwt.lowbit_bitlinear_group(*args, out, gs, norm, 1e-5, status=st, weights_stable=weights_stable)
    torch.cuda.synchronize()
    assert st.item() == 0
    return y32, q, s_x, y


def check_layer(L, norm, out, y32, q, s_x, y, rows=None):
    """Layer L against the oracle; rows: the output rows whose accumulators
    are recomputed by the oracle (all when None)."""
    q_o, s_o = oracle.act_prologue(L.x, L.g, norm == bwt.NORM_RMS, 1e-5, 0, bf16_bits=L.bf16)
    q_g = q.cpu().numpy()[:, :L.K]
    assert np.array_equal(q_g, q_o)
    s_g = s_x.cpu().numpy()
    if norm:
        assert np.max(np.abs(s_g.astype(np.float64) - s_o) / np.maximum(s_o, 1e-38)) <= 1e-6
    else:
        assert np.array_equal(s_g.view(np.uint32), s_o.view(np.uint32))
    codes = L.codes if rows is None else L.codes[rows]
    acc_o = oracle.int_dot(q_o, codes, L.fmt, nthreads=oracle.max_threads())
    acc_g = y32.cpu().numpy().astype(np.int64)
    acc_g = acc_g if rows is None else acc_g[:, rows]
    assert np.array_equal(acc_g, acc_o)
    # the float output from the kernel's own scales is the oracle's rescale
    s_w = L.s_w if (L.fmt == bwt.TERNARY2 or rows is None) else L.s_w[rows]
    y_o = oracle.rescale(acc_o, s_w, s_g, "bf16" if out == bwt.BF16 else "f32")
    if out == bwt.BF16:
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        got = got if rows is None else got[:, rows]
        assert np.array_equal(got, y_o)
    else:
        got = y.cpu().numpy()
        got = got if rows is None else got[:, rows]
        assert np.array_equal(got.view(np.uint32), y_o.view(np.uint32))


# Layers of different widths and depths, as in one decode block: QKV-like
# and FFN-like shapes, a single output row, ragged K and N.
SHAPES = [(9728, 2560), (2560, 9728), (768, 256), (300, 200), (1, 4096), (37, 1000), (4096, 4112)]


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("norm", [bwt.NORM_NONE, bwt.NORM_RMS], ids=["plain", "rmsnorm"])
def test_group_matches_oracle(fmt, M, norm):
    bf16 = M != 2
    shapes = [(N, K) for N, K in SHAPES if M * ((K + 127) // 128 * 128) <= bwt.FUSED_MAX_BYTES]
    layers = [Layer(fmt, N, K, M, 6000 + 31 * i + fmt + 7 * M, bf16, use_g=(i % 2 == 0))
              for i, (N, K) in enumerate(shapes)]
    out = bwt.BF16 if bf16 else bwt.F32
    y32, q, s_x, y = run_group(layers, fmt, out, norm, weights_stable=(M == 1))
    for i, L in enumerate(layers):
        check_layer(L, norm, out, y32[i], q[i], s_x[i], y[i])


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
def test_group_equals_separate_calls(fmt):
    # without the norm every value of a layer is computed the same way alone
    # or in a group, so the outputs are bit-identical
    layers = [Layer(fmt, N, K, 1, 6500 + i, True, use_g=True) for i, (N, K) in enumerate(SHAPES)]
    ys = bwt.lowbit_bitlinear_group([L.x_dev for L in layers], [L.packed for L in layers],
                                    [L.s_w_dev for L in layers], fmt, [L.N for L in layers], bwt.BF16,
                                    [L.g_dev for L in layers])
    for L, y in zip(layers, ys):
        y1 = bwt.lowbit_bitlinear(L.x_dev, L.packed, L.s_w_dev, fmt, L.N, bwt.BF16, L.g_dev)
        assert torch.equal(y, y1)


def test_group_persistent_many_units():
    # 24 layers of 2560 -> 9728 at M = 1: far more units than resident
    # clusters, so every cluster runs several units and crosses layers.  The
    # codes are checked in full against the oracle, the accumulators on the
    # first and last rows of every 64-row unit plus random rows.
    fmt, N, K = bwt.TERNARY2, 9728, 2560
    w = wls.normal_weights(6600, N, K)
    layers = [Layer(fmt, N, K, 1, 6601 + 3 * i, True, use_g=True, w=w) for i in range(24)]
    y32, q, s_x, y = run_group(layers, fmt, bwt.BF16, bwt.NORM_NONE, weights_stable=True)
    rng = np.random.default_rng(6602)
    edges = np.concatenate([np.arange(0, N, 64), np.arange(63, N, 64)])
    rows = np.unique(np.concatenate([edges, rng.choice(N, 256, replace=False)]))
    for i, L in enumerate(layers):
        check_layer(L, bwt.NORM_NONE, bwt.BF16, y32[i], q[i], s_x[i], y[i], rows=rows)


def test_group_atomic_stack_decode():
    # all 25 matrices of the 6-layer stack at one token, in one launch
    wl = wls.WORKLOADS["atomic_stack"]
    layers = []
    for i, m in enumerate(wl.matrices):
        layers.append(Layer(wl.fmt, m.N, m.K, 1, 0, False, use_g=False, w=wls.workload_weights(wl, i),
                            x=wls.workload_activations(wl, i, 1)))
    y32, q, s_x, y = run_group(layers, wl.fmt, bwt.BF16, bwt.NORM_NONE, weights_stable=True)
    for i, L in enumerate(layers):
        check_layer(L, bwt.NORM_NONE, bwt.BF16, y32[i], q[i], s_x[i], y[i])


def test_group_flags_nonfinite_rows():
    fmt, N, K = bwt.TERNARY2, 512, 256
    a = Layer(fmt, N, K, 1, 6700, False, use_g=False)
    x = a.x.copy()
    x[0, 17] = np.inf
    b = Layer(fmt, N, K, 1, 6701, False, use_g=False, x=x)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    bwt.lowbit_bitlinear_group([a.x_dev, b.x_dev], [a.packed, b.packed], [a.s_w_dev, b.s_w_dev], fmt, [N, N],
                               bwt.F32, status=st)
    torch.cuda.synchronize()
    assert bwt.status_flags(st) == [bwt.ERR_NONFINITE]
