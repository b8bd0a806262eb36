"""Parity of the activation prologue (gain, RMSNorm, block Hadamard rotation,
per-token codes) and of the whole BitLinear call with the oracle (needs a
B200).

Codes and int32 accumulators must be bit-identical.  Scales and outputs that
do not depend on the RMSNorm's sum of squares are computed by the same
operations on both sides and must be bit-identical too; with the RMSNorm the
fp64 sum of squares is reduced in a different order, so s_x and the float
outputs are held to the stated tolerances: 1e-6 relative for fp32, 1 ulp for
bf16.
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


def status_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def to_dev(x, bf16):
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(DEV).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV)


def gain(K, seed):
    return (1.0 + 0.1 * np.random.default_rng(seed).standard_normal(K)).astype(np.float32)


def check_scales(got, want, norm):
    if norm:
        rel = np.abs(got.astype(np.float64) - want.astype(np.float64)) / np.maximum(np.abs(want), 1e-38)
        assert rel.max() <= 1e-6, rel.max()
    else:
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


OPTIONS = [(False, 0, 0), (True, 0, 0), (False, 1, 0), (True, 1, 0), (False, 0, 64), (True, 1, 512),
           (False, 1, 2)]
OPT_IDS = [f"g{int(g)}-norm{n}-h{h}" for g, n, h in OPTIONS]


@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
@pytest.mark.parametrize("opt", OPTIONS, ids=OPT_IDS)
@pytest.mark.parametrize("M,K", [(1, 2560), (7, 1024), (300, 9728), (2048, 512), (33, 2560), (5, 40960), (1024, 2560),
                                 (3, 16384), (4, 2624)])
def test_act_quant_ex_matches_oracle(M, K, opt, bf16):
    use_g, norm, hb = opt
    if hb and K % hb:
        pytest.skip("block does not divide K")
    x = wls.normal_activations(3000 + M + K, M, K, 0.005, 10.0)
    x[0, :] = 0.0  # zero row: zero codes and scale
    if bf16:
        x = wls.to_bf16_bits(x)
    g = gain(K, 3001) if use_g else None
    st = status_word()
    q, s_x = bwt.lowbit_act_quant_ex(to_dev(x, bf16), None if g is None else torch.from_numpy(g).to(DEV), norm,
                                     1e-5, hb, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    q_o, s_o = oracle.act_prologue(x, g, norm == 1, 1e-5, hb, bf16_bits=bf16)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    check_scales(s_x.cpu().numpy(), s_o, norm)


@pytest.mark.parametrize("opt", OPTIONS, ids=OPT_IDS)
def test_act_quant_ex_unaligned_rows(opt):
    # Rows that do not start on 16-byte boundaries take the staged kernel.
    use_g, norm, hb = opt
    M, K, ldx = 9, 256, 259
    if hb > K:
        pytest.skip("block longer than the row")
    base = wls.normal_activations(3100, M, ldx, 0.01, 8.0)
    x = base[:, :K]
    g = gain(K, 3101) if use_g else None
    xt = torch.from_numpy(base).to(DEV)[:, :K]
    q, s_x = bwt.lowbit_act_quant_ex(xt, None if g is None else torch.from_numpy(g).to(DEV), norm, 1e-5, hb)
    q_o, s_o = oracle.act_prologue(x, g, norm == 1, 1e-5, hb)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    check_scales(s_x.cpu().numpy(), s_o, norm)


def test_act_quant_ex_flags_nonfinite_gain():
    x = np.ones((3, 64), np.float32)
    g = np.ones(64, np.float32)
    g[9] = np.inf
    for hb in (0, 64):
        st = status_word()
        bwt.lowbit_act_quant_ex(to_dev(x, False), torch.from_numpy(g).to(DEV), bwt.NORM_RMS, 1e-5, hb, status=st)
        torch.cuda.synchronize()
        assert bwt.status_flags(st) == [bwt.ERR_NONFINITE]


def test_act_quant_ex_rejects_bad_blocks():
    x = torch.zeros((2, 96), dtype=torch.float32, device=DEV)
    for hb in (3, 1, 64, 128, -4):  # not a power of two, one, not dividing 96, above K
        with pytest.raises(bwt.LowbitError) as e:
            bwt.lowbit_act_quant_ex(x, hadamard=hb)
        assert e.value.status == bwt.ERR_INVALID_ARG
    big = torch.zeros((1, 49152 + 64), dtype=torch.float32, device=DEV)
    with pytest.raises(bwt.LowbitError) as e:
        bwt.lowbit_act_quant_ex(big, norm=bwt.NORM_RMS)
    assert e.value.status == bwt.ERR_UNSUPPORTED


# ---------------------------------------------------------------------------
# the whole BitLinear call
# ---------------------------------------------------------------------------

def oracle_bitlinear(x, w, fmt, g, norm, hb, out, bf16):
    codes, s_w = oracle.quantize(w, fmt, 1e-5)
    q, s_x = oracle.act_prologue(x, g, norm == 1, 1e-5, hb, bf16_bits=bf16)
    acc = oracle.int_dot(q, codes, fmt, nthreads=oracle.max_threads())
    return acc, oracle.rescale(acc, s_w, s_x, out), q, s_x


def run_bitlinear(fmt, M, N, K, opt, bf16, seed, out, path=0):
    use_g, norm, hb = opt
    w = wls.normal_weights(seed, N, K)
    x = wls.normal_activations(seed + 1, M, K, 0.005, 10.0)
    if bf16:
        x = wls.to_bf16_bits(x)
    g = gain(K, seed + 2) if use_g else None
    packed, s_w = bwt.lowbit_pack(torch.from_numpy(w).to(DEV), fmt, 1e-5)
    st = status_word()
    outs = {}
    for ydt in (bwt.I32, out):
        outs[ydt] = bwt.lowbit_bitlinear(to_dev(x, bf16), packed, s_w, fmt, N, ydt,
                                         None if g is None else torch.from_numpy(g).to(DEV), norm, 1e-5, hb,
                                         want_codes=True, status=st, path=path, weights_stable=True)
    torch.cuda.synchronize()
    assert st.item() == 0
    return x, w, g, outs


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("opt", OPTIONS, ids=OPT_IDS)
@pytest.mark.parametrize("M,N,K,bf16", [(1, 9728, 2560, True), (3, 2560, 9728, True), (4, 768, 192, False),
                                        (2, 300, 200, False), (1, 4096, 256, False), (16, 2560, 2560, True),
                                        (300, 1000, 512, False)], ids=str)
def test_bitlinear_matches_oracle(fmt, opt, M, N, K, bf16):
    use_g, norm, hb = opt
    if hb and K % hb:
        pytest.skip("block does not divide K")
    out = bwt.BF16 if bf16 else bwt.F32
    x, w, g, outs = run_bitlinear(fmt, M, N, K, opt, bf16, 4000 + M + N + K + fmt, out)
    acc_o, y_o, q_o, s_o = oracle_bitlinear(x, w, fmt, g, norm, hb, "bf16" if bf16 else "f32", bf16)
    y32, q, s_x = outs[bwt.I32]
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    check_scales(s_x.cpu().numpy(), s_o, norm)
    assert np.array_equal(y32.cpu().numpy().astype(np.int64), acc_o)
    y = outs[out][0]
    if bf16:
        got = y.view(torch.int16).cpu().numpy().view(np.uint16)
        assert bf16_ulps(got, y_o).max() <= 1
        if not norm:
            assert np.array_equal(got, y_o)
    else:
        got = y.cpu().numpy()
        assert np.max(np.abs(got - y_o) / np.maximum(np.abs(y_o), 1e-30)) <= 1e-6
        if not norm:
            assert np.array_equal(got.view(np.uint32), y_o.view(np.uint32))


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,K", [(1, 1024), (2, 1000), (4, 1024), (3, 520), (1, 200)])
def test_fused_decode_equals_two_launches(fmt, M, K):
    # The fused kernel (codes computed in every block; rows of at most
    # FUSED_MAX_K features) and the prologue kernel followed by lowbit_linear
    # give the same codes and accumulators; without the norm also the same
    # scales and outputs, bit for bit.
    N = 2560
    assert bwt.bitlinear_fuses(M, K) and not bwt.bitlinear_fuses(M, bwt.FUSED_MAX_K + 1)
    w = wls.normal_weights(4100 + fmt, N, K)
    x = to_dev(wls.to_bf16_bits(wls.normal_activations(4101, M, K, 0.005, 10.0)), True)
    g = torch.from_numpy(gain(K, 4102)).to(DEV)
    packed, s_w = bwt.lowbit_pack(torch.from_numpy(w).to(DEV), fmt, 1e-5)
    for norm in (bwt.NORM_NONE, bwt.NORM_RMS):
        y1, q1, s1 = bwt.lowbit_bitlinear(x, packed, s_w, fmt, N, bwt.I32, g, norm, want_codes=True)
        q2, s2 = bwt.lowbit_act_quant_ex(x, g, norm)
        y2 = bwt.lowbit_linear(q2, s2, packed, s_w, fmt, N, bwt.I32, K=K, path=1)
        assert torch.equal(y1, y2) and torch.equal(q1[:, :K], q2[:, :K])
        if norm == bwt.NORM_NONE:
            assert torch.equal(s1, s2)
            f1 = bwt.lowbit_bitlinear(x, packed, s_w, fmt, N, bwt.BF16, g, norm)
            f2 = bwt.lowbit_linear(q2, s2, packed, s_w, fmt, N, bwt.BF16, K=K, path=1)
            assert torch.equal(f1, f2)


def test_bitlinear_needs_workspace_when_not_fused():
    x = torch.zeros((8, 256), dtype=torch.float32, device=DEV)
    packed = torch.zeros((64, 64), dtype=torch.uint8, device=DEV)
    s_w = torch.ones(1, dtype=torch.float32, device=DEV)
    y = torch.empty((8, 64), dtype=torch.float32, device=DEV)
    st = bwt.lib().lowbit_bitlinear(x.data_ptr(), bwt.F32, 8, 256, 256, None, 0, 1e-5, 0, packed.data_ptr(), 64,
                                    s_w.data_ptr(), bwt.TERNARY2, 64, y.data_ptr(), bwt.F32, 64, None, 0, None, 0, 0,
                                    None, None)
    assert st == bwt.ERR_INVALID_ARG


# ---------------------------------------------------------------------------
# BitNet v1 centred binary codes (lowbit_pack_ex)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(192, 192), (37, 101), (1, 4096), (2048, 192), (5, 7)])
def test_pack_centred_bit_exact(N, K):
    w = (wls.normal_weights(4200 + N + K, N, K) + np.float32(0.01)).astype(np.float32)
    if N > 2:
        w[1, :] = 0.0  # rows around the mean
    st = status_word()
    packed, s_w = bwt.lowbit_pack_ex(torch.from_numpy(w).to(DEV), bwt.BINARY1, bwt.QUANT_BINARY_CENTRED, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    codes, beta, _ = oracle.binary_centred_codes(w)
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(codes, bwt.BINARY1, packed.shape[1]))
    assert np.array_equal(s_w.cpu().numpy().view(np.uint32), np.full(N, beta[0], np.float32).view(np.uint32))


def test_pack_centred_tie_takes_minus_one():
    # a weight equal to the tensor mean takes -1 (M8.8 0x02E)
    w = np.array([[1.0, 2.0, 3.0], [0.0, 2.0, 4.0]], np.float32)
    packed, s_w = bwt.lowbit_pack_ex(torch.from_numpy(w).to(DEV), bwt.BINARY1, bwt.QUANT_BINARY_CENTRED)
    codes = bwt.lowbit_unpack(packed, 3, bwt.BINARY1).cpu().numpy()
    assert codes.tolist() == [[-1, -1, 1], [-1, -1, 1]]
    assert s_w.cpu().tolist() == [2.0, 2.0]


def test_pack_ex_rejects_centred_for_other_formats():
    w = torch.zeros((4, 32), dtype=torch.float32, device=DEV)
    for fmt in (bwt.TERNARY2, bwt.INT4):
        with pytest.raises(bwt.LowbitError) as e:
            bwt.lowbit_pack_ex(w, fmt, bwt.QUANT_BINARY_CENTRED)
        assert e.value.status == bwt.ERR_INVALID_ARG


def test_pack_ex_default_is_lowbit_pack():
    w = torch.from_numpy(wls.normal_weights(4300, 100, 300)).to(DEV)
    for fmt in FMTS:
        p1, s1 = bwt.lowbit_pack_ex(w, fmt)
        p2, s2 = bwt.lowbit_pack(w, fmt)
        assert torch.equal(p1, p2) and torch.equal(s1, s2)
