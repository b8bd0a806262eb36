// gemv.cu -- packed-weight GEMV for few tokens (decode).
//
// "M8.8 - Native Binary and Ternary Transformers" 0x09B: decode has a small
// token dimension and streams large weight matrices, so the kernel is bound
// by the bytes of packed weights it reads.  The integer dot is the
// add/subtract/skip rule ("Atomic-1Bit" README; M8.8 0x05D) executed four
// codes at a time: each packed word is expanded in registers into int8x4
// words holding (c << S) (no table, one shift and one mask per four ternary
// codes) and multiplied with dp4a, which for c in {-1,0,+1} is exactly the
// add / subtract / skip of the activation.
//
// Layout of the work: one warp per output row; lane l streams the row's
// 16-byte chunks l, l+32, ... with non-allocating loads (each weight byte is
// read once), multiplies them with the matching int8 activation bytes (small,
// re-read from L1/L2 by every warp), and the 32 partial sums are combined with
// warp shuffles.  The epilogue (M8.8 0x02D) is fused: y = float(acc) *
// (s_w * s_x) in fp32, optionally rounded to bf16.
#include "lowbit_internal.cuh"

namespace lowbit {
namespace {

constexpr int kWarps = 8;

// 16 activation bytes starting at k (a multiple of 16), bytes at k' >= K zero.
__device__ __forceinline__ uint4 load_q16(const int8_t *qrow, int64_t k, int64_t K)
{
    if (k + 16 <= K) return __ldg(reinterpret_cast<const uint4 *>(qrow + k));
    uint4 v = make_uint4(0, 0, 0, 0);
    if (k < K) {
        v = __ldg(reinterpret_cast<const uint4 *>(qrow + k));
        const int valid = static_cast<int>(K - k);  // 1..15
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int lo = 4 * i;
            uint32_t m;
            if (valid >= lo + 4) m = 0xffffffffu;
            else if (valid <= lo) m = 0u;
            else m = (1u << (8 * (valid - lo))) - 1u;
            (&v.x)[i] &= m;
        }
    }
    return v;
}

template <int FMT>
__device__ __forceinline__ int32_t chunk_dot(const uint4 &wv, const int8_t *qrow, int64_t k0, int64_t K,
                                             int32_t acc)
{
    if constexpr (FMT == kT2) {
        // 64 codes: word j holds codes 16j..16j+15 of the chunk.
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 qv = load_q16(qrow, k0 + 16 * j, K);
            const uint32_t w = (&wv.x)[j];
#pragma unroll
            for (int g = 0; g < 4; ++g)
                acc = __dp4a(static_cast<int>(t2_expand(w, g)), static_cast<int>((&qv.x)[g]), acc);
        }
    } else if constexpr (FMT == kI4) {
        // 32 codes: word j holds codes 8j..8j+7.
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const uint4 qv = load_q16(qrow, k0 + 16 * p, K);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w = (&wv.x)[2 * p + h];
                acc = __dp4a(static_cast<int>(i4_expand(w, 0)), static_cast<int>((&qv.x)[2 * h]), acc);
                acc = __dp4a(static_cast<int>(i4_expand(w, 1)), static_cast<int>((&qv.x)[2 * h + 1]), acc);
            }
        }
    } else {
        // 128 codes: word j holds codes 32j..32j+31, bit b = code 32j+b.
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w = (&wv.x)[j];
#pragma unroll
            for (int p = 0; p < 2; ++p) {
                const uint4 qv = load_q16(qrow, k0 + 32 * j + 16 * p, K);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t nib = (w >> (16 * p + 4 * m)) & 0xFu;
                    acc = __dp4a(static_cast<int>(b1_expand_nibble(nib)), static_cast<int>((&qv.x)[m]), acc);
                }
            }
        }
    }
    return acc;
}

template <int OUT>
__device__ __forceinline__ void store_out(void *y, int64_t idx, int32_t acc, float sw, float sx)
{
    if constexpr (OUT == LOWBIT_I32) {
        static_cast<int32_t *>(y)[idx] = acc;
    } else if constexpr (OUT == LOWBIT_F32) {
        static_cast<float *>(y)[idx] = rescale(acc, sw, sx);
    } else {
        static_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(rescale(acc, sw, sx));
    }
}

// Each warp takes R consecutive rows and U 16-byte chunks per lane of each:
// all R*U weight loads are issued before any of them is used, so a batch of
// rows costs one DRAM round trip, and the grid is sized to run in one wave.
template <int FMT, int MT, int U, int R, int OUT>
__global__ void __launch_bounds__(kWarps * 32)
gemv_kernel(const int8_t *__restrict__ q, int64_t ldq, const float *__restrict__ s_x, int M, int64_t K,
            const uint8_t *__restrict__ packed, int64_t ldp, int64_t nchunks, const float *__restrict__ s_w,
            int64_t N, void *__restrict__ y, int64_t ldy)
{
    using F = Fmt<FMT>;
    constexpr int kCodesPerChunk = 4 * F::kCodesPerWord;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    for (int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * R; row0 < N;
         row0 += static_cast<int64_t>(gridDim.x) * kWarps * R) {
        int32_t acc[R][MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[r][t] = 0;
        for (int64_t c0 = 0; c0 < nchunks; c0 += 32 * U) {
            uint4 wv[R][U];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int64_t c = c0 + lane + 32 * u;
                    wv[r][u] = (c < nchunks && row0 + r < N) ? ld_stream_u4(packed + (row0 + r) * ldp + c * 16)
                                                             : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t c = c0 + lane + 32 * u;
                if (c < nchunks) {
#pragma unroll
                    for (int r = 0; r < R; ++r)
#pragma unroll
                        for (int t = 0; t < MT; ++t)
                            if (t < M)
                                acc[r][t] = chunk_dot<FMT>(wv[r][u], q + t * ldq, c * kCodesPerChunk, K, acc[r][t]);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t row = row0 + r;
            const float sw = (row < N) ? s_w[FMT == kT2 ? 0 : row] : 0.0f;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                int32_t v = acc[r][t];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == t && t < M && row < N) store_out<OUT>(y, t * ldy + row, v >> F::kShift, sw, s_x[t]);
            }
        }
    }
}

template <int FMT, int MT, int U, int R>
lowbit_status launch_mt(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                        const uint8_t *packed, int64_t ldp, int64_t nchunks, const float *s_w, int64_t N,
                        void *y, lowbit_dtype ydt, int64_t ldy, cudaStream_t st)
{
    int64_t blocks = (N + kWarps * R - 1) / (kWarps * R);
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (blocks > cap) blocks = cap;
    const dim3 grid(static_cast<unsigned>(blocks)), block(kWarps * 32);
    if (ydt == LOWBIT_F32)
        gemv_kernel<FMT, MT, U, R, LOWBIT_F32><<<grid, block, 0, st>>>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ldy);
    else if (ydt == LOWBIT_BF16)
        gemv_kernel<FMT, MT, U, R, LOWBIT_BF16><<<grid, block, 0, st>>>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ldy);
    else
        gemv_kernel<FMT, MT, U, R, LOWBIT_I32><<<grid, block, 0, st>>>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ldy);
    return launch_status();
}

// Pick U (chunks per lane in flight) from the row length and R (rows per
// warp) so that the grid fills the GPU in about one wave of 2 blocks per SM.
template <int FMT, int MT>
lowbit_status launch_u(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                       const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N,
                       void *y, lowbit_dtype ydt, int64_t ldy, cudaStream_t st)
{
    const int64_t nchunks = (row_bytes + 15) / 16;
    const int64_t slots = static_cast<int64_t>(device_sm_count()) * 2 * kWarps;  // warps in one wave
    if (nchunks <= 64) {
        if (MT == 1 && N >= 4 * slots)
            return launch_mt<FMT, MT, 2, 4>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, st);
        if (MT <= 4 && N >= 2 * slots)
            return launch_mt<FMT, MT, 2, 2>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, st);
        return launch_mt<FMT, MT, 2, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, st);
    }
    return launch_mt<FMT, MT, 8, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, st);
}

template <int FMT>
lowbit_status launch_fmt(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                         const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N,
                         void *y, lowbit_dtype ydt, int64_t ldy, cudaStream_t st)
{
    if (M <= 1) return launch_u<FMT, 1>(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, st);
    if (M <= 4) return launch_u<FMT, 4>(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, st);
    return launch_u<FMT, 16>(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, st);
}

}  // namespace

// Token rows are processed 16 at a time; each group is one launch.
lowbit_status gemv_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                          const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                          lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, cudaStream_t st)
{
    const int64_t esz = (ydt == LOWBIT_BF16) ? 2 : 4;
    for (int64_t t0 = 0; t0 < M; t0 += 16) {
        const int m = static_cast<int>(M - t0 < 16 ? M - t0 : 16);
        const int8_t *qg = q + t0 * ldq;
        const float *sg = s_x + t0;
        void *yg = static_cast<char *>(y) + t0 * ldy * esz;
        lowbit_status s;
        if (f == LOWBIT_TERNARY2) s = launch_fmt<kT2>(qg, ldq, sg, m, K, packed, ldp, row_bytes, s_w, N, yg, ydt, ldy, st);
        else if (f == LOWBIT_BINARY1) s = launch_fmt<kB1>(qg, ldq, sg, m, K, packed, ldp, row_bytes, s_w, N, yg, ydt, ldy, st);
        else s = launch_fmt<kI4>(qg, ldq, sg, m, K, packed, ldp, row_bytes, s_w, N, yg, ydt, ldy, st);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

}  // namespace lowbit
