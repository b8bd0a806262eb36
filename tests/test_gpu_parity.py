"""Parity of the CUDA path with the oracle (needs a B200).

Both sides get the same seeded inputs (binary_weight_transformer_b200.workloads).
Codes, packed bytes, scales, int8 activations and int32 accumulators must be
bit-identical.  Floating outputs must meet the stated tolerances: fp32 within
1e-6 relative, bf16 within 1 unit in the last place.  Both sides also use the
same operation order, so the float outputs are additionally checked for bit
equality in separate tests.
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


def status_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def ulp_distance_bf16(a_bits, b_bits):
    """Distance in bf16 units in the last place (monotone integer mapping)."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


def gpu_pack(w, fmt, eps=1e-5, extra_ld=0):
    wt = torch.from_numpy(w).to(DEV)
    ldp = bwt.packed_ld(fmt, w.shape[1]) + extra_ld
    st = status_word()
    packed, s_w = bwt.lowbit_pack(wt, fmt, eps, ldp=ldp, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return packed, s_w


def gpu_act(x_np, bf16=False, eps=0.0):
    if bf16:
        xt = torch.from_numpy(x_np.view(np.int16)).to(DEV).view(torch.bfloat16)
    else:
        xt = torch.from_numpy(x_np).to(DEV)
    st = status_word()
    q, s_x = bwt.lowbit_act_quant(xt, eps, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return q, s_x


# ---------------------------------------------------------------------------
# activation quantiser
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
# Shapes cover one thread group per row for every TPR (the 1024-thread group
# of both register builds: 9728, 12288, 16384, 24584), the scalar-load path
# (unaligned rows), rows longer than the register path (65560), many rows of
# 16-byte vectors, and a zero row in each.
@pytest.mark.parametrize("M,K", [(1, 192), (7, 200), (3, 9728), (257, 2560), (5, 13), (64, 3),
                                 (9, 65536 + 24), (300, 9728), (1000, 192), (600, 12288), (256, 24),
                                 (33, 768), (5, 16384), (2, 24584)])
@pytest.mark.parametrize("eps", [0.0, 1e-5])
def test_act_quant_bit_exact(M, K, bf16, eps):
    x = wls.normal_activations(100 + M + K, M, K, 0.01, 8.0)
    x[0, :] = 0.0  # an all-zero row: zero codes and zero scale
    if bf16:
        x = wls.to_bf16_bits(x)
    q, s_x = gpu_act(x, bf16, eps)
    q_o, s_o = oracle.act_quant(x, eps, bf16_bits=bf16)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


# The deep build (five vectors per thread at 1536 resident threads) runs when
# it halves the thread group of the wide build and M x group fills two waves
# of the GPU, or when only it holds the row; each case is sized 10% past that
# bound for its group: bf16 K = 320, 1280, 2560, 5120, 9728, 20480 (groups 8 to
# 512), f32 K = 9728 (512), and rows of 3073 to 5120 vectors (1024, any M).
@pytest.mark.parametrize("K,bf16", [(320, True), (1280, True), (2560, True), (5120, True), (9728, True),
                                    (20480, True), (9728, False), (24584, True), (40960, True), (20480, False)])
def test_act_quant_bit_exact_deep(K, bf16):
    nvec = K // (8 if bf16 else 4)
    groups = (8, 32, 64, 128, 256, 512, 1024)
    tpr_deep = next(g for g in groups if nvec <= 5 * g)
    tpr_wide = next((g for g in groups if nvec <= 3 * g), None)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    M = 3 if tpr_wide is None else (2 * sms * 1536 * 11 // 10 + tpr_deep - 1) // tpr_deep
    x = wls.normal_activations(7 + K, M, K, 0.01, 8.0)
    x[0, :] = 0.0
    if bf16:
        x = wls.to_bf16_bits(x)
    q, s_x = gpu_act(x, bf16, 0.0)
    q_o, s_o = oracle.act_quant(x, 0.0, bf16_bits=bf16)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


# Many rows of the decode and prefill shapes: ragged M, the largest
# workload M at K = 2560, the smallest rows (one 16-byte vector), and zero
# first and last rows.
@pytest.mark.parametrize("bf16", [False, True], ids=["f32", "bf16"])
@pytest.mark.parametrize("M,K", [(512, 2560), (1031, 2048), (8192, 2560), (600, 8), (2000, 1000), (513, 1536)])
@pytest.mark.parametrize("eps", [0.0, 1e-5])
def test_act_quant_many_rows_bit_exact(M, K, bf16, eps):
    x = wls.normal_activations(300 + M + K, M, K, 0.01, 8.0)
    x[0, :] = 0.0
    x[M - 1, :] = 0.0
    if bf16:
        x = wls.to_bf16_bits(x)
    q, s_x = gpu_act(x, bf16, eps)
    q_o, s_o = oracle.act_quant(x, eps, bf16_bits=bf16)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


def edge_rows(seed, M, K, eps):
    """Rows that stress the codes' rounding: by row index mod 4, ordinary
    N(0,1); tiny (max |x| from 1e-44 to 1e-36, subnormals included, where the
    reciprocal of the row max is not a normal fp32); values placed within a few
    ulp of rounding midpoints, 127x/max|x| = k + 1/2; and large (1e30 to 1e35,
    127x still finite).  With a large eps all rows are scaled near 1e36 (and
    clipped to 2e36, where 127x is still finite) so that the codes are not all
    zero."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    for t in range(M):
        kind = t % 4
        if eps > 1.0:
            x[t] = np.clip(x[t] * 10 ** rng.uniform(35.0, 35.7), -2e36, 2e36)
        elif kind == 1:
            x[t] *= 10 ** rng.uniform(-44.0, -36.0)
        elif kind == 2:
            g = 10 ** rng.uniform(-3.0, 3.0)
            k = rng.integers(-127, 127, K)
            x[t] = (k + 0.5) * g / 127.0 * (1.0 + rng.uniform(-3e-7, 3e-7, K))
            x[t, 0] = g
        elif kind == 3:
            x[t] *= 10 ** rng.uniform(30.0, 35.0)
    return x.astype(np.float32)


# eps = 0; 5e37 (d just below 2^126: the fast path); 1e38 (d above it: the
# divide for every value).  Small M takes the wide build, large M the deep one
# (K = 9728) and, at M = 1024, the wide build with many blocks (K = 2560, 2048).
@pytest.mark.parametrize("eps", [0.0, 5e37, 1e38])
@pytest.mark.parametrize("K,bf16,deep", [(2560, True, False), (2560, False, False), (9728, True, True),
                                         (9728, False, True), (2560, True, "many"), (2048, False, "many")])
def test_act_quant_rounding_edges(K, bf16, deep, eps):
    M = 64
    if deep == "many":
        M = 1024
    elif deep:
        nvec = K // (8 if bf16 else 4)
        tpr_deep = next(g for g in (8, 32, 64, 128, 256, 512, 1024) if nvec <= 5 * g)
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        M = (2 * sms * 1536 * 11 // 10 + tpr_deep - 1) // tpr_deep
    x = edge_rows(K + int(eps > 0) + int(eps > 6e37), M, K, eps)
    if bf16:
        x = wls.to_bf16_bits(x)
    q, s_x = gpu_act(x, bf16, eps)
    q_o, s_o = oracle.act_quant(x, eps, bf16_bits=bf16)
    assert np.array_equal(q.cpu().numpy()[:, :K], q_o)
    assert np.array_equal(s_x.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


@pytest.mark.parametrize("M", [4, 300, 700], ids=["regs", "ring", "many"])
def test_act_quant_flags_nonfinite(M):
    x = np.ones((M, 64), np.float32)
    x[2, 5] = np.nan
    x[3, 7] = 1e37  # x * 127 overflows fp32
    xt = torch.from_numpy(x).to(DEV)
    st = status_word()
    q, s_x = bwt.lowbit_act_quant(xt, 0.0, status=st)
    torch.cuda.synchronize()
    assert bwt.status_flags(st) == [bwt.ERR_NONFINITE]
    if M > 4:  # the finite rows are unaffected
        q_o, s_o = oracle.act_quant(x[4:], 0.0)
        assert np.array_equal(q.cpu().numpy()[4:, :64], q_o)


# ---------------------------------------------------------------------------
# packer / unpacker
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("N,K", [(768, 192), (37, 101), (5, 7), (1, 4096), (96, 1000), (300, 33)])
def test_pack_bit_exact(fmt, N, K):
    w = wls.normal_weights(200 + N + K, N, K)
    if fmt == bwt.INT4 and N > 1:
        w[0] = 0.0  # a zero row: zero scale, zero codes
        w[1] *= 100.0  # tanh clipping bends strongly
    packed, s_w = gpu_pack(w, fmt, extra_ld=16)
    codes, s_o = oracle.quantize(w, fmt, 1e-5)
    p_o = oracle.pack(codes, fmt, packed.shape[1])
    assert np.array_equal(packed.cpu().numpy(), p_o)
    assert np.array_equal(s_w.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


@pytest.mark.parametrize("fmt,N,K", [(bwt.TERNARY2, 9728, 2560), (bwt.TERNARY2, 2560, 9728),
                                     (bwt.INT4, 3584, 1280), (bwt.INT4, 1280, 3584),
                                     (bwt.BINARY1, 2048, 192)], ids=str)
def test_pack_full_size_bit_exact(fmt, N, K):
    w = wls.normal_weights(300 + K, N, K)
    packed, s_w = gpu_pack(w, fmt)
    codes, s_o = oracle.quantize(w, fmt, 1e-5)
    assert np.array_equal(packed.cpu().numpy(), oracle.pack(codes, fmt, packed.shape[1]))
    assert np.array_equal(s_w.cpu().numpy().view(np.uint32), s_o.view(np.uint32))


def test_pack_ternary_eps_zero_tie():
    # M8.8 §0x05A tie rule: w/gamma = 0.5 exactly rounds to 0 (nearest even).
    w = np.array([[0.25, -0.75, 0.5, -0.5]], np.float32)
    packed, s_w = gpu_pack(w, bwt.TERNARY2, eps=0.0)
    codes = bwt.lowbit_unpack(packed, 4, bwt.TERNARY2).cpu().numpy()
    assert s_w.item() == 0.5
    assert codes.tolist() == [[0, -1, 1, -1]]


def test_pack_flags_nonfinite():
    w = np.ones((3, 40), np.float32)
    w[1, 3] = np.inf
    for fmt in FMTS:
        wt = torch.from_numpy(w).to(DEV)
        st = status_word()
        bwt.lowbit_pack(wt, fmt, status=st)
        torch.cuda.synchronize()
        assert bwt.status_flags(st) == [bwt.ERR_NONFINITE], fmt


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
def test_unpack_roundtrip_and_reserved(fmt):
    N, K = 50, 77
    w = wls.normal_weights(400 + fmt, N, K)
    packed, _ = gpu_pack(w, fmt)
    codes_o, _ = oracle.quantize(w, fmt)
    st = status_word()
    codes = bwt.lowbit_unpack(packed, K, fmt, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert np.array_equal(codes.cpu().numpy(), codes_o)
    # a non-zero padding byte is rejected
    bad = packed.clone()
    bad[3, -1] = 1
    st.zero_()
    bwt.lowbit_unpack(bad, K, fmt, status=st)
    torch.cuda.synchronize()
    assert bwt.status_flags(st) == [bwt.ERR_RESERVED_CODE]
    if fmt != bwt.BINARY1:
        # a reserved field (10 / 1000) inside the extent is rejected
        bad = packed.clone()
        bad[4, 0] = (bad[4, 0] & ~0x3 if fmt == bwt.TERNARY2 else bad[4, 0] & ~0xF) | \
            (0x2 if fmt == bwt.TERNARY2 else 0x8)
        st.zero_()
        bwt.lowbit_unpack(bad, K, fmt, status=st)
        torch.cuda.synchronize()
        assert bwt.status_flags(st) == [bwt.ERR_RESERVED_CODE]


# ---------------------------------------------------------------------------
# linear: both kernels, every format and output type
# ---------------------------------------------------------------------------

def run_case(fmt, M, N, K, path, out, seed, zero_w=False, x_bf16=False, weights_stable=False):
    if path == 5 and M > 16:
        pytest.skip("the warp-MMA kernel takes at most 16 tokens")
    w = wls.normal_weights(seed, N, K)
    if zero_w:
        w[:] = 0.0
    x = wls.normal_activations(seed + 1, M, K, 0.01, 8.0)
    if x_bf16:
        x = wls.to_bf16_bits(x)
    packed, s_w = gpu_pack(w, fmt)
    q, s_x = gpu_act(x, x_bf16)
    st = status_word()
    y = bwt.lowbit_linear(q, s_x, packed, s_w, fmt, N, out, K=K, status=st, path=path,
                          weights_stable=weights_stable)
    torch.cuda.synchronize()
    assert st.item() == 0
    codes, s_wo = oracle.quantize(w, fmt, 1e-5)
    q_o, s_xo = oracle.act_quant(x, 0.0, bf16_bits=x_bf16)
    acc = oracle.int_dot(q_o, codes, fmt, nthreads=oracle.max_threads())
    return y, acc, s_wo, s_xo


# Includes shapes that take the cluster split-K path of the GEMM (few output
# tiles, deep K): (16, 96, 1000), (300, 768, 1040), (200, 1, 4000),
# (64, 500, 4096), (130, 1000, 2000).
SHAPES = [(1, 768, 192), (3, 257, 200), (16, 96, 1000), (17, 300, 192), (129, 513, 384), (300, 768, 1040),
          (5, 33, 16), (200, 1, 4000), (64, 500, 4096), (130, 1000, 2000)]


@pytest.mark.parametrize("path", [1, 2, 3, 4, 5, 6], ids=["gemv", "gemm", "gemm_ts", "gemm_ts_pair", "skinny", "gemm_pair"])
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,N,K", SHAPES, ids=str)
def test_linear_int32_accumulators_bit_exact(path, fmt, M, N, K):
    y, acc, _, _ = run_case(fmt, M, N, K, path, bwt.I32, 500 + M + N + K)
    assert np.array_equal(y.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("path", [1, 2, 3, 4, 5, 6], ids=["gemv", "gemm", "gemm_ts", "gemm_ts_pair", "skinny", "gemm_pair"])
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,N,K", SHAPES[:6] + SHAPES[8:], ids=str)
def test_linear_f32_within_tolerance(path, fmt, M, N, K):
    y, acc, s_w, s_x = run_case(fmt, M, N, K, path, bwt.F32, 600 + M + N + K)
    ref = oracle.rescale(acc, s_w, s_x, "f32")
    got = y.cpu().numpy()
    denom = np.maximum(np.abs(ref), np.finfo(np.float32).tiny)
    assert np.max(np.abs(got - ref) / denom) <= 1e-6
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("path", [1, 2, 3, 4, 5, 6], ids=["gemv", "gemm", "gemm_ts", "gemm_ts_pair", "skinny", "gemm_pair"])
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,N,K", SHAPES[:6] + SHAPES[8:], ids=str)
def test_linear_bf16_within_one_ulp(path, fmt, M, N, K):
    y, acc, s_w, s_x = run_case(fmt, M, N, K, path, bwt.BF16, 700 + M + N + K, x_bf16=True)
    ref = oracle.rescale(acc, s_w, s_x, "bf16")
    got = bf16_bits(y)
    assert ulp_distance_bf16(got, ref).max() <= 1
    assert np.array_equal(got, ref)


# Split plans of the shared-memory GEMM (path 2): K split over clusters of
# 2, 4 and 8 CTAs, with one or two token tiles and ragged N, K and M.
#   (17, 9728, 2560): 38 tiles x 2        (24, 7168, 2560): 28 tiles x 4
#   (40, 2560, 9728): 10 tiles x 8        (9, 640, 1024): 3 tiles x 4 (8 K blocks)
#   (130, 1000, 2000): 2 x 4 tiles x 8    (64, 500, 4096), (3, 2560, 9728): x 8
SPLIT_SHAPES = [(17, 9728, 2560), (24, 7168, 2560), (40, 2560, 9728), (9, 640, 1024), (130, 1000, 2000),
                (64, 500, 4096), (3, 2560, 9728)]


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES, ids=str)
def test_split_plans_int32_bit_exact(fmt, M, N, K):
    y, acc, _, _ = run_case(fmt, M, N, K, 2, bwt.I32, 950 + M + N + K)
    assert np.array_equal(y.cpu().numpy().astype(np.int64), acc)


# The warp-MMA kernel with rows longer than 512 packed bytes streams weights
# and token codes through a TMA ring (128 bytes of every row per stage) and
# splits K over a cluster of 2 or 4 CTAs when the 32-row tiles are few.
#   (16, 2560, 9728): 80 tiles, 19 stages (ternary) -> 2 CTAs per tile
#   (9, 1000, 4100): 32 tiles, K ragged in the last stage -> 4 (ternary, 4-bit) or 2 (binary)
#   (5, 300, 3000): 10 tiles, 6 ternary stages -> 2;  (16, 9728, 2560): 304 tiles, no split
#   (12, 33, 65536): 2 tiles, 128 ternary stages: the 12-stage ring wraps ten times -> 4
STREAM_SHAPES = [(16, 2560, 9728), (9, 1000, 4100), (5, 300, 3000), (16, 9728, 2560), (12, 33, 65536)]


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,N,K", STREAM_SHAPES, ids=str)
@pytest.mark.parametrize("path", [0, 5], ids=["auto", "skinny"])
def test_stream_and_split_int32_bit_exact(fmt, M, N, K, path):
    y, acc, _, _ = run_case(fmt, M, N, K, path, bwt.I32, 970 + M + N + K)
    assert np.array_equal(y.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
def test_stream_split_bf16_bit_exact(fmt):
    M, N, K = 16, 2560, 9728
    y, acc, s_w, s_x = run_case(fmt, M, N, K, 5, bwt.BF16, 990, x_bf16=True)
    assert np.array_equal(bf16_bits(y), oracle.rescale(acc, s_w, s_x, "bf16"))


# LOWBIT_LINEAR_EXCLUSIVE: when the SM-pair GEMM (path 6) would end on a
# partial round, it shares the K blocks of the remaining tiles evenly over the
# pairs (stream-K) and adds the int32 partial tiles through a device
# workspace.  Schedules on 74 pairs: 17 whole rounds, the tail not shared
# (8192, 9728, 2560: 16 rounds + 32 tiles of 20 K blocks, where sharing does
# not pay); 3 rounds, then 98 tiles of 76 blocks (8192,
# 2560, 9728); 40 tiles of 76 blocks, no whole round (1024, 2560, 9728); one
# round, then 78 tiles of 20 (1024, 9728, 2560); 40 ragged tiles of 76 blocks,
# up to 2 partial tiles added per tile (1000, 2500, 9728); 6 ragged tiles of 32
# blocks, kept whole since 4 partial tiles per tile would cost more (300, 700,
# 4096); 8 tiles of 128 blocks, up to 10 partial tiles per tile (512, 1000,
# 16384); 9 tiles of 6 blocks, no split (768, 768, 768).
# Each launch gets its own activations and output dtype, so that a partial
# tile or flag left by an earlier launch cannot pass for this one's; the
# output must equal the unsplit launch bit for bit, and the oracle on
# sampled rows (every row of the small shapes).
PAIR_SPLIT_SHAPES = [(8192, 9728, 2560), (8192, 2560, 9728), (1024, 2560, 9728), (1024, 9728, 2560),
                     (1000, 2500, 9728), (300, 700, 4096), (512, 1000, 16384), (768, 768, 768)]


@pytest.mark.parametrize("M,N,K,fmt", [s + (bwt.TERNARY2,) for s in PAIR_SPLIT_SHAPES]
                         + [(300, 700, 4096, f) for f in (bwt.BINARY1, bwt.INT4)]
                         + [(1000, 2500, 9728, f) for f in (bwt.BINARY1, bwt.INT4)]
                         + [(1024, 2560, 9728, f) for f in (bwt.BINARY1, bwt.INT4)], ids=str)
def test_pair_stream_k_bit_exact(M, N, K, fmt):
    w = wls.normal_weights(1100 + M + K, N, K)
    packed, s_w = gpu_pack(w, fmt)
    xs = [wls.normal_activations(1101 + M + K + i, M, K, 0.01, 8.0) for i in range(3)]
    acts = [gpu_act(x, False) for x in xs]
    st = status_word()
    outs = [bwt.I32, bwt.BF16, bwt.I32]
    ys = {}
    for exclusive in (False, True, True):  # twice split: the epoch flags must not carry over
        for i, out in enumerate(outs):
            q, s_x = acts[i]
            ys[(exclusive, i)] = bwt.lowbit_linear(q, s_x, packed, s_w, fmt, N, out, K=K, status=st, path=6,
                                                   exclusive=exclusive)
    torch.cuda.synchronize()
    assert st.item() == 0
    for i in range(len(outs)):
        assert torch.equal(ys[(True, i)], ys[(False, i)])
    codes, _ = oracle.quantize(w, fmt, 1e-5)
    rows = np.arange(M)
    if M * N * K > 2e9:  # first and last row of every 256-row tile, and random rows
        rng = np.random.default_rng(1102)
        rows = np.unique(np.concatenate([np.arange(0, M, 256), np.arange(255, M, 256), rng.choice(M, 64)]))
    for i in (0, 2):
        q_o, _ = oracle.act_quant(xs[i], 0.0)
        acc = oracle.int_dot(q_o[rows], codes, fmt, nthreads=oracle.max_threads())
        assert np.array_equal(ys[(True, i)].cpu().numpy()[rows].astype(np.int64), acc)


# LOWBIT_LINEAR_WEIGHTS_STABLE: weight reads start before the wait for the
# preceding kernel (here the act quant that produced q, launched just before
# on the same stream); the results must not change.  Shapes cover the GEMV
# (one and several token groups), the cluster split-K GEMM, the persistent
# GEMM, and the tensor-memory GEMM with more tiles than SMs.
@pytest.mark.parametrize("path", [0, 1, 2, 3, 5, 6], ids=["auto", "gemv", "gemm", "gemm_ts", "skinny", "gemm_pair"])
@pytest.mark.parametrize("fmt", FMTS, ids=FMT_IDS.get)
@pytest.mark.parametrize("M,N,K", [(1, 2560, 768), (9, 300, 1000), (16, 2600, 2600), (130, 1000, 2000),
                                   (600, 4000, 640)], ids=str)
def test_linear_weights_stable_bit_exact(path, fmt, M, N, K):
    if path == 1 and M > 16:
        pytest.skip("GEMV path kept to decode sizes")
    y, acc, _, _ = run_case(fmt, M, N, K, path, bwt.I32, 900 + M + N + K, weights_stable=True)
    assert np.array_equal(y.cpu().numpy().astype(np.int64), acc)


@pytest.mark.parametrize("path", [1, 2, 3, 4, 5, 6], ids=["gemv", "gemm", "gemm_ts", "gemm_ts_pair", "skinny", "gemm_pair"])
def test_linear_degenerate_weights(path):
    # all-zero weights: gamma = 0, every code 0, y = 0
    y, acc, _, _ = run_case(bwt.TERNARY2, 16 if path == 5 else 20, 64, 256, path, bwt.F32, 800, zero_w=True)
    assert not acc.any()
    assert not y.cpu().numpy().any()


@pytest.mark.parametrize("path", [1, 2, 3, 4, 5, 6], ids=["gemv", "gemm", "gemm_ts", "gemm_ts_pair", "skinny", "gemm_pair"])
def test_linear_all_plus_one_gives_row_sums(path):
    # ternary codes all +1: acc[t, n] = sum_k q[t, k] (add/sub/skip rule)
    M, N, K = (16 if path == 5 else 19), 40, 320
    w = np.full((N, K), 0.5, np.float32)
    x = wls.normal_activations(801, M, K)
    packed, s_w = gpu_pack(w, bwt.TERNARY2)
    q, s_x = gpu_act(x)
    y = bwt.lowbit_linear(q, s_x, packed, s_w, bwt.TERNARY2, N, bwt.I32, K=K, path=path)
    rows = q.cpu().numpy()[:, :K].astype(np.int64).sum(axis=1)
    assert np.array_equal(y.cpu().numpy(), np.repeat(rows[:, None], N, axis=1))


def test_linear_ignores_bytes_of_q_past_k():
    # K = 202: the last 4-byte activation word is partly past K (ldq = 208)
    N, K = 70, 202
    for path in (1, 2, 3, 5):
        M = 16 if path == 5 else 40
        for fmt in FMTS:
            w = wls.normal_weights(810 + fmt, N, K)
            x = wls.normal_activations(811, M, K)
            packed, s_w = gpu_pack(w, fmt)
            q, s_x = gpu_act(x)
            ref = bwt.lowbit_linear(q, s_x, packed, s_w, fmt, N, bwt.I32, K=K, path=path).cpu()
            q2 = q.clone()
            q2[:, K:] = 77  # garbage in the stride padding
            got = bwt.lowbit_linear(q2, s_x, packed, s_w, fmt, N, bwt.I32, K=K, path=path).cpu()
            assert torch.equal(got, ref)


# ---------------------------------------------------------------------------
# the workloads at full size, in the configuration bench.py times
# ---------------------------------------------------------------------------

def test_single_ternary_full():
    wl = wls.WORKLOADS["single_ternary"]
    m = wl.matrices[0]
    M = wl.Ms[0]
    w = wls.workload_weights(wl, 0)
    x = wls.workload_activations(wl, 0, M)
    packed, s_w = gpu_pack(w, wl.fmt)
    q, s_x = gpu_act(x)
    y = bwt.lowbit_linear(q, s_x, packed, s_w, wl.fmt, m.N, bwt.F32, K=m.K)
    codes, s_wo = oracle.quantize(w, wl.fmt, 1e-5)
    q_o, s_xo = oracle.act_quant(x)
    ref, _ = oracle.linear(q_o, s_xo, oracle.pack(codes, wl.fmt), s_wo, wl.fmt, m.K)
    got = y.cpu().numpy()
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)) <= 1e-6


def _sampled_rows(M, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows |= {0, M - 1}
    return np.array(sorted(rows))


@pytest.mark.parametrize("name", ["ternary_4b", "t4nt_int4"])
def test_sweep_workloads_sampled(name):
    wl = wls.WORKLOADS[name]
    for mi, m in enumerate(wl.matrices):
        w = wls.workload_weights(wl, mi)
        packed, s_w = gpu_pack(w, wl.fmt)
        codes, s_wo = oracle.quantize(w, wl.fmt, 1e-5)
        assert np.array_equal(s_w.cpu().numpy().view(np.uint32), s_wo.view(np.uint32))
        bf = wl.x_dtype == wls.BF16
        for M in wl.Ms:
            x = wls.workload_activations(wl, mi, M)
            q, s_x = gpu_act(x, bf)
            y = bwt.lowbit_linear(q, s_x, packed, s_w, wl.fmt, m.N, bwt.BF16, K=m.K)
            rows = _sampled_rows(M)
            q_o, s_xo = oracle.act_quant(x[rows], 0.0, bf16_bits=bf)
            assert np.array_equal(q.cpu().numpy()[rows, :m.K], q_o)
            acc = oracle.int_dot(q_o, codes, wl.fmt, nthreads=oracle.max_threads())
            ref = oracle.rescale(acc, s_wo, s_xo, "bf16")
            got = bf16_bits(y)[rows]
            assert ulp_distance_bf16(got, ref).max() <= 1, (name, mi, M)


def test_impeto_binary_stack_sampled():
    wl = wls.WORKLOADS["impeto_binary"]
    M = wl.Ms[0]
    for mi in (0, 1, 4, 6, len(wl.matrices) - 1):  # q, k, gate, down, head
        m = wl.matrices[mi]
        w = wls.workload_weights(wl, mi)
        x = wls.workload_activations(wl, mi, M)
        packed, s_w = gpu_pack(w, wl.fmt)
        q, s_x = gpu_act(x)
        y = bwt.lowbit_linear(q, s_x, packed, s_w, wl.fmt, m.N, bwt.F32, K=m.K)
        rows = _sampled_rows(M, 64, mi)
        codes, s_wo = oracle.quantize(w, wl.fmt, 1e-5)
        q_o, s_xo = oracle.act_quant(x[rows])
        acc = oracle.int_dot(q_o, codes, wl.fmt, nthreads=oracle.max_threads())
        ref = oracle.rescale(acc, s_wo, s_xo, "f32")
        got = y.cpu().numpy()[rows]
        assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)) <= 1e-6


def test_atomic_stack_full():
    wl = wls.WORKLOADS["atomic_stack"]
    for mi in (0, 1, 2, 3, len(wl.matrices) - 1):
        m = wl.matrices[mi]
        w = wls.workload_weights(wl, mi)
        packed, s_w = gpu_pack(w, wl.fmt)
        codes, s_wo = oracle.quantize(w, wl.fmt, 1e-5)
        for M in wl.Ms:
            x = wls.workload_activations(wl, mi, M)
            q, s_x = gpu_act(x)
            y = bwt.lowbit_linear(q, s_x, packed, s_w, wl.fmt, m.N, bwt.BF16, K=m.K)
            q_o, s_xo = oracle.act_quant(x)
            acc = oracle.int_dot(q_o, codes, wl.fmt, nthreads=oracle.max_threads())
            ref = oracle.rescale(acc, s_wo, s_xo, "bf16")
            assert ulp_distance_bf16(bf16_bits(y), ref).max() <= 1
