// gemv_impl.cuh -- packed-weight GEMV for few tokens (decode).
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
#pragma once

#include "lowbit_internal.cuh"

namespace lowbit {
namespace gemv_detail {

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
            int64_t N, void *__restrict__ y, int64_t ldy, int prefetch)
{
    using F = Fmt<FMT>;
    constexpr int kCodesPerChunk = 4 * F::kCodesPerWord;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // With prefetch the first weight loads are issued before the wait for the
    // previous kernel (the caller vouches that it does not write the weights).
    bool waited = prefetch == 0;
    if (waited) pdl_wait();
    pdl_trigger();
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
            if (!waited) {
                pdl_wait();
                waited = true;
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

// Activation bytes a 16-byte weight chunk needs, in 16-byte pieces.
template <int FMT> struct QPieces { static constexpr int value = 4 * Fmt<FMT>::kCodesPerWord / 16; };

// chunk_dot with the chunk's activation pieces already in registers.
template <int FMT>
__device__ __forceinline__ int32_t chunk_dot_regs(const uint4 &wv, const uint4 *qv, int32_t acc)
{
    if constexpr (FMT == kT2) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w = (&wv.x)[j];
#pragma unroll
            for (int g = 0; g < 4; ++g)
                acc = __dp4a(static_cast<int>(t2_expand(w, g)), static_cast<int>((&qv[j].x)[g]), acc);
        }
    } else if constexpr (FMT == kI4) {
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t w = (&wv.x)[2 * p + h];
                acc = __dp4a(static_cast<int>(i4_expand(w, 0)), static_cast<int>((&qv[p].x)[2 * h]), acc);
                acc = __dp4a(static_cast<int>(i4_expand(w, 1)), static_cast<int>((&qv[p].x)[2 * h + 1]), acc);
            }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w = (&wv.x)[j];
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t nib = (w >> (16 * p + 4 * m)) & 0xFu;
                    acc = __dp4a(static_cast<int>(b1_expand_nibble(nib)), static_cast<int>((&qv[2 * j + p].x)[m]), acc);
                }
        }
    }
    return acc;
}

// The token codes are staged once per block into shared memory (zero past K)
// after the block's weight loads are in flight, so their latency overlaps the
// DRAM round trip; each lane then reads a chunk's activation bytes once and
// applies them to all R rows it holds.
template <int FMT, int MT, int U, int R, int OUT>
__global__ void __launch_bounds__(kWarps * 32)
gemv_smem_kernel(const int8_t *__restrict__ q, int64_t ldq, const float *__restrict__ s_x, int M, int64_t K,
                 const uint8_t *__restrict__ packed, int64_t ldp, int64_t nchunks, const float *__restrict__ s_w,
                 int64_t N, void *__restrict__ y, int64_t ldy, int prefetch)
{
    using F = Fmt<FMT>;
    constexpr int QP = QPieces<FMT>::value;
    extern __shared__ uint4 qs[];  // [M][QP][nchunks]: piece-major, so lanes read consecutive pieces
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * R;
    const int64_t qpieces = nchunks * QP;
    // With prefetch the first weight loads are issued before the wait for the
    // previous kernel (the caller vouches that it does not write the weights).
    if (prefetch == 0) pdl_wait();
    pdl_trigger();

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
        if (c0 == 0) {
            if (prefetch != 0) pdl_wait();
            for (int64_t i = threadIdx.x; i < M * qpieces; i += blockDim.x) {
                const int64_t t = i / qpieces, j = i % qpieces;   // j = chunk * QP + piece
                qs[t * qpieces + (j % QP) * nchunks + j / QP] = load_q16(q + t * ldq, j * 16, K);
            }
            __syncthreads();
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t c = c0 + lane + 32 * u;
            if (c < nchunks) {
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                    if (t < M) {
                        uint4 qv[QP];
#pragma unroll
                        for (int p = 0; p < QP; ++p) qv[p] = qs[t * qpieces + p * nchunks + c];
#pragma unroll
                        for (int r = 0; r < R; ++r) acc[r][t] = chunk_dot_regs<FMT>(wv[r][u], qv, acc[r][t]);
                    }
                }
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

constexpr int64_t kGemvSmemMax = 96 * 1024;

template <int FMT, int MT, int U, int R>
lowbit_status launch_smem(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K, const uint8_t *packed,
                          int64_t ldp, int64_t nchunks, const float *s_w, int64_t N, void *y, lowbit_dtype ydt,
                          int64_t ldy, size_t smem, int prefetch, cudaStream_t st)
{
    static PerDevice configured;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            const int lim = static_cast<int>(kGemvSmemMax);
            return (cudaFuncSetAttribute(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_F32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess &&
                    cudaFuncSetAttribute(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess &&
                    cudaFuncSetAttribute(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_I32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess) ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    const int64_t blocks = (N + kWarps * R - 1) / (kWarps * R);
    const dim3 g(static_cast<unsigned>(blocks)), b(kWarps * 32);
    if (ydt == LOWBIT_F32)
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_F32>, g, b, smem, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
    else if (ydt == LOWBIT_BF16)
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_BF16>, g, b, smem, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
    else
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_I32>, g, b, smem, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
}

// Long rows whose activations do not fit the shared-memory staging: the
// activation bytes are read through L1 instead (persistent grid).
template <int FMT, int MT>
lowbit_status launch_global(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                            const uint8_t *packed, int64_t ldp, int64_t nchunks, const float *s_w, int64_t N,
                            void *y, lowbit_dtype ydt, int64_t ldy, int prefetch, cudaStream_t st)
{
    int64_t blocks = (N + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (blocks > cap) blocks = cap;
    const dim3 grid(static_cast<unsigned>(blocks)), block(kWarps * 32);
    if (ydt == LOWBIT_F32)
        return launch_pdl(gemv_kernel<FMT, MT, 8, 1, LOWBIT_F32>, grid, block, 0, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
    else if (ydt == LOWBIT_BF16)
        return launch_pdl(gemv_kernel<FMT, MT, 8, 1, LOWBIT_BF16>, grid, block, 0, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
    else
        return launch_pdl(gemv_kernel<FMT, MT, 8, 1, LOWBIT_I32>, grid, block, 0, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
}

// One launch for up to 4 tokens.  U (16-byte chunks per lane in flight) comes
// from the row length and R (rows per warp) is raised for short rows so the
// grid stays near one wave of two blocks per SM.
template <int FMT, int MT>
lowbit_status launch_tokens(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                            const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N,
                            void *y, lowbit_dtype ydt, int64_t ldy, int prefetch, cudaStream_t st)
{
    const int64_t nchunks = (row_bytes + 15) / 16;
    const int64_t smem_i = static_cast<int64_t>(M) * nchunks * QPieces<FMT>::value * 16;
    if (smem_i > kGemvSmemMax)
        return launch_global<FMT, MT>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, prefetch, st);
    const size_t smem = static_cast<size_t>(smem_i);
    const int64_t slots = static_cast<int64_t>(device_sm_count()) * 2 * kWarps;  // warps in one wave
    if (nchunks <= 64) {
        if constexpr (MT == 1) {
            if (N >= 4 * slots)
                return launch_smem<FMT, MT, 2, 4>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, st);
        }
        if (N >= 2 * slots)
            return launch_smem<FMT, MT, 2, 2>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, st);
        return launch_smem<FMT, MT, 2, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, st);
    }
    if (nchunks <= 160)
        return launch_smem<FMT, MT, 5, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, st);
    return launch_smem<FMT, MT, 8, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, st);
}

// Tokens are processed in groups of up to 4, one launch per group.
template <int FMT>
lowbit_status gemv_launch_fmt(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                              const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N,
                              void *y, lowbit_dtype ydt, int64_t ldy, int prefetch, cudaStream_t st)
{
    const int64_t esz = (ydt == LOWBIT_BF16) ? 2 : 4;
    for (int64_t t0 = 0; t0 < M; t0 += 4) {
        const int m = static_cast<int>(M - t0 < 4 ? M - t0 : 4);
        const int8_t *qg = q + t0 * ldq;
        const float *sg = s_x + t0;
        void *yg = static_cast<char *>(y) + t0 * ldy * esz;
        const lowbit_status s = (m == 1)
            ? launch_tokens<FMT, 1>(qg, ldq, sg, m, K, packed, ldp, row_bytes, s_w, N, yg, ydt, ldy, prefetch, st)
            : launch_tokens<FMT, 4>(qg, ldq, sg, m, K, packed, ldp, row_bytes, s_w, N, yg, ydt, ldy, prefetch, st);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

}  // namespace gemv_detail
}  // namespace lowbit
