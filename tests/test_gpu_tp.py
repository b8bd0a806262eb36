"""The tensor-parallel kernels on one B200 (needs a GPU).

The row-parallel kernels (slice statistics, codes with a given row maximum,
scales from whole-row statistics, the rescale epilogue) are checked against
the oracle and numpy, and a split layer is run for 2 and 4 ranks one rank
after another on the same GPU: the reductions a collective would perform are
done here by torch on the per-rank results (no kernel waits on another), and
the result is compared with the unsplit lowbit_bitlinear.  The collectives
themselves are covered on CPU ranks by tests/test_tp_cpu.py.
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
from binary_weight_transformer_b200 import tp  # noqa: E402

DEV = "cuda:0"
FMTS = [bwt.TERNARY2, bwt.BINARY1, bwt.INT4]


@pytest.fixture(scope="module", autouse=True)
def built():
    from binary_weight_transformer_b200 import _build
    _build.build()
    oracle.build()
    bwt.lib()


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("out", [bwt.F32, bwt.BF16, bwt.I32])
def test_rescale_matches_oracle(fmt, out):
    M, N = 37, 333
    rng = np.random.default_rng(5000 + fmt)
    acc = rng.integers(-2_000_000, 2_000_000, size=(M, N)).astype(np.int32)
    s_x = (rng.random(M) * 0.05).astype(np.float32)
    s_x[3] = 0.0
    s_w = (rng.random(1 if fmt == bwt.TERNARY2 else N) * 0.02).astype(np.float32)
    y = bwt.lowbit_rescale(torch.from_numpy(acc).to(DEV), torch.from_numpy(s_x).to(DEV),
                           torch.from_numpy(s_w).to(DEV), fmt, out).cpu()
    if out == bwt.I32:
        assert np.array_equal(y.numpy(), acc)
    elif out == bwt.F32:
        ref = oracle.rescale(acc.astype(np.int64), s_w, s_x, "f32")
        assert np.array_equal(y.numpy().view(np.uint32), ref.view(np.uint32))
    else:
        ref = oracle.rescale(acc.astype(np.int64), s_w, s_x, "bf16")
        assert np.array_equal(y.view(torch.int16).numpy().view(np.uint16), ref)


@pytest.mark.parametrize("hb", [0, 128])
@pytest.mark.parametrize("use_g", [False, True])
def test_row_stats_and_given_max_codes(hb, use_g):
    M, K = 21, 1024
    x = wls.normal_activations(5100, M, K, 0.01, 8.0)
    x[2] = 0.0
    g = wls.gain_vector(5101, K) if use_g else None
    xt = torch.from_numpy(x).to(DEV)
    gt = None if g is None else torch.from_numpy(g).to(DEV)
    row_max, row_ss = bwt.lowbit_act_row_stats(xt, gt, hb, with_ss=True)
    u = x if g is None else (x * g).astype(np.float32)
    if hb:
        u = oracle.fwht32(u.reshape(M, K // hb, hb)).reshape(M, K)
    assert np.array_equal(row_max.cpu().numpy(), np.abs(u).max(axis=1))
    ss = (x.astype(np.float64) ** 2).sum(axis=1)
    assert np.allclose(row_ss.cpu().numpy(), ss, rtol=1e-13, atol=0)
    # with the slice's own maximum the codes are those of the prologue
    q = bwt.lowbit_act_quant_given_max(xt, row_max, gt, hb)
    q_o, _ = oracle.act_prologue(x, g, False, 1e-5, hb)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    # and the scales from the statistics are the prologue's
    for norm in (bwt.NORM_NONE, bwt.NORM_RMS):
        s_x = bwt.lowbit_act_scales(row_max, row_ss, K, norm, 1e-5, hb).cpu().numpy()
        _, s_o = oracle.act_prologue(x, g, norm == bwt.NORM_RMS, 1e-5, hb)
        assert np.max(np.abs(s_x.astype(np.float64) - s_o) / np.maximum(s_o, 1e-38)) <= 1e-6


def test_given_max_below_the_slice_max_is_reported():
    x = torch.ones((2, 128), dtype=torch.float32, device=DEV)
    row_max = torch.full((2,), 0.5, dtype=torch.float32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    bwt.lowbit_act_quant_given_max(x, row_max, status=st)
    torch.cuda.synchronize()
    assert bwt.status_flags(st) == [bwt.ERR_INVALID_ARG]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("norm,hb,use_g", [(0, 0, False), (1, 0, True), (1, 512, True)])
def test_split_layer_equals_unsplit(fmt, world, norm, hb, use_g):
    M, N, K = 40, 1536, 2048
    w = wls.normal_weights(5200 + fmt, N, K)
    x = wls.to_bf16_bits(wls.normal_activations(5201, M, K, 0.005, 10.0))
    g = wls.gain_vector(5202, K) if use_g else None
    xt = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    gt = None if g is None else torch.from_numpy(g).to(DEV)
    packed, s_w = bwt.lowbit_pack(torch.from_numpy(w).to(DEV), fmt)
    y_ref = bwt.lowbit_bitlinear(xt, packed, s_w, fmt, N, bwt.F32, gt, norm, 1e-5, hb)
    torch.cuda.synchronize()

    # row-parallel, ranks one after another
    spans = [tp.split(K, world, r, tp.feature_granule(hb)) for r in range(world)]
    stats = [bwt.lowbit_act_row_stats(xt[:, k0:k1], None if gt is None else gt[k0:k1], hb, with_ss=bool(norm))
             for k0, k1 in spans]
    row_max = torch.stack([s[0] for s in stats]).amax(dim=0)            # all-reduce MAX
    row_ss = torch.stack([s[1] for s in stats]).sum(dim=0) if norm else None  # all-reduce SUM
    s_x = bwt.lowbit_act_scales(row_max, row_ss, K, norm, 1e-5, hb)
    acc = torch.zeros((M, N), dtype=torch.int32, device=DEV)
    for k0, k1 in spans:
        q = bwt.lowbit_act_quant_given_max(xt[:, k0:k1], row_max, None if gt is None else gt[k0:k1], hb)
        acc += bwt.lowbit_linear(q, s_x, tp.packed_feature_slice(packed, fmt, k0, k1), s_w, fmt, N, bwt.I32,
                                 K=k1 - k0)                             # all-reduce SUM (int32)
    y_row = bwt.lowbit_rescale(acc, s_x, s_w, fmt, bwt.F32)
    # column-parallel, ranks one after another
    cols = []
    for r in range(world):
        n0, n1 = tp.split(N, world, r)
        cols.append(bwt.lowbit_bitlinear(xt, packed[n0:n1], tp.row_scales_slice(s_w, fmt, n0, n1), fmt, n1 - n0,
                                         bwt.F32, gt, norm, 1e-5, hb))
    y_col = torch.cat(cols, dim=1)
    torch.cuda.synchronize()
    a, b, c = y_ref.cpu().numpy(), y_row.cpu().numpy(), y_col.cpu().numpy()
    assert np.array_equal(c.view(np.uint32), a.view(np.uint32))
    if norm:
        assert np.max(np.abs(b - a) / np.maximum(np.abs(a), 1e-30)) <= 1e-6
    else:
        assert np.array_equal(b.view(np.uint32), a.view(np.uint32))
