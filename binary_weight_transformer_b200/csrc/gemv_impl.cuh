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

#include "quant_rule.cuh"

namespace lowbit {
namespace gemv_detail {

constexpr int kWarps = 8;

// 16 activation bytes starting at k (a multiple of 16), bytes at k' >= K zero.
__device__ __forceinline__ uint4 load_q16(const int8_t *qrow, int64_t k, int64_t K)
{
    if (k + 16 <= K) return ld_act_u4(qrow + k);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (k < K) {
        v = ld_act_u4(qrow + k);
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
                if (lane == t && t < M && row < N) store_out<OUT>(y, t * ldy + row, v >> F::kShift, sw, ld_act_f32(s_x + t));
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

// The R rows of one warp starting at row0, U 16-byte chunks per lane per
// step, against activation codes staged in shared memory as qs[M][QP][nchunks]
// (piece-major, so the lanes read consecutive pieces).  stage() runs once,
// after the first weight loads of the warp are issued and before qs is read,
// so the staging latency overlaps the DRAM round trip of the weights; it is
// called by every thread of the block.
template <int FMT, int MT, int U, int R, class Stage>
__device__ __forceinline__ void rows_dot(const uint8_t *__restrict__ packed, int64_t ldp, int64_t nchunks, int64_t N,
                                         int64_t row0, int M, const uint4 *qs, Stage &&stage, int32_t (&acc)[R][MT])
{
    constexpr int QP = QPieces<FMT>::value;
    const int lane = threadIdx.x & 31;
    const int64_t qpieces = nchunks * QP;
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
        if (c0 == 0) stage();
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
}

// The warp's R rows of y: lane t writes token t after a shuffle reduction.
template <int FMT, int MT, int R, int OUT>
__device__ __forceinline__ void rows_store(const int32_t (&acc)[R][MT], int64_t row0, int64_t N, int M,
                                           const float *__restrict__ s_w, void *__restrict__ y, int64_t ldy,
                                           const float (&sxr)[MT])
{
    using F = Fmt<FMT>;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t row = row0 + r;
        const float sw = (row < N) ? s_w[FMT == kT2 ? 0 : row] : 0.0f;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            int32_t v = acc[r][t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == t && t < M && row < N) store_out<OUT>(y, t * ldy + row, v >> F::kShift, sw, sxr[t]);
        }
    }
}

// The token codes are staged once per block into shared memory (zero past K)
// after the block's weight loads are in flight; each lane then reads a
// chunk's activation bytes once and applies them to all R rows it holds.
template <int FMT, int MT, int U, int R, int OUT>
__global__ void __launch_bounds__(kWarps * 32)
gemv_smem_kernel(const int8_t *__restrict__ q, int64_t ldq, const float *__restrict__ s_x, int M, int64_t K,
                 const uint8_t *__restrict__ packed, int64_t ldp, int64_t nchunks, const float *__restrict__ s_w,
                 int64_t N, void *__restrict__ y, int64_t ldy, int prefetch)
{
    constexpr int QP = QPieces<FMT>::value;
    extern __shared__ uint4 qs[];
    const int warp = threadIdx.x >> 5;
    const int64_t row0 = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * R;
    const int64_t qpieces = nchunks * QP;
    // With prefetch the first weight loads are issued before the wait for the
    // previous kernel (the caller vouches that it does not write the weights).
    if (prefetch == 0) pdl_wait();
    pdl_trigger();
    float sxr[MT];  // the token scales, read once, not in the epilogue
    int32_t acc[R][MT];
    rows_dot<FMT, MT, U, R>(packed, ldp, nchunks, N, row0, M, qs, [&] {
        if (prefetch != 0) pdl_wait();
#pragma unroll
        for (int t = 0; t < MT; ++t) sxr[t] = t < M ? ld_act_f32(s_x + t) : 0.0f;
        for (int64_t i = threadIdx.x; i < M * qpieces; i += blockDim.x) {
            const int64_t t = i / qpieces, j = i % qpieces;   // j = chunk * QP + piece
            qs[t * qpieces + (j % QP) * nchunks + j / QP] = load_q16(q + t * ldq, j * 16, K);
        }
        __syncthreads();
    }, acc);
    rows_store<FMT, MT, R, OUT>(acc, row0, N, M, s_w, y, ldy, sxr);
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
    const dim3 g(static_cast<unsigned>((N + kWarps * R - 1) / (kWarps * R))), b(kWarps * 32);
    if (ydt == LOWBIT_F32)
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_F32>, g, b, smem, st, 0, q, ldq, s_x, M, K, packed,
                          ldp, nchunks, s_w, N, y, ldy, prefetch);
    else if (ydt == LOWBIT_BF16)
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_BF16>, g, b, smem, st, 0, q, ldq, s_x, M, K, packed,
                          ldp, nchunks, s_w, N, y, ldy, prefetch);
    else
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_I32>, g, b, smem, st, 0, q, ldq, s_x, M, K, packed,
                          ldp, nchunks, s_w, N, y, ldy, prefetch);
}

// ---------------------------------------------------------------------------
// Grouped fused decode: one launch computes up to kGroupMax BitLinear layers
// on M <= 4 token rows each, with the activation prologue in the kernel.
//
// The rows of every layer are cut into units of one block (8 warps x R
// rows); block b of the grid takes a contiguous range of units whose packed
// bytes are about 1/blocks of the group's (persistent: the grid holds at
// most as many blocks as are resident at once).  A block first issues the
// weight loads of its first unit and L2 prefetches for its other units,
// then computes the codes and scales of the layers of its range itself
// (every block repeats the prologue of the layers it touches: a few thousand
// features of arithmetic, cheaper than the barriers and round trips of
// sharing it), then streams its units against the staged codes.  The layers
// are independent: no layer may read what another writes.
struct GroupItem {
    const void *x;         // [M, ldx] token rows
    const float *g;        // [K] gain or nullptr
    int8_t *q_out;         // optional codes [M, ldq_out]
    float *s_x_out;        // optional scales [M]
    const uint8_t *packed; // [N, ldp]
    const float *s_w;
    void *y;               // [M, ldy]
    int64_t ldx, ldq_out, ldp, ldy;
    int64_t cost0;         // sum of units x nchunks over the layers before this one
    int32_t N, K, nchunks;
    int32_t unit0, units;  // this layer's units: [unit0, unit0 + units)
};
constexpr int kGroupMax = 32;
struct GroupArgs {
    GroupItem item[kGroupMax];
    int64_t cost_total;
    int32_t *status;
    float eps_norm;
    int n_items, units, M, xbf16, norm, prefetch;
};
static_assert(sizeof(GroupArgs) <= 4000, "the group must fit the 4 KB kernel parameter space");

// Smallest unit whose cost offset is >= target (the number of units if none).
__device__ __forceinline__ int first_unit_at(const GroupArgs &a, int64_t target)
{
    for (int i = 0; i < a.n_items; ++i) {
        const GroupItem &I = a.item[i];
        if (target <= I.cost0) return I.unit0;
        const int64_t steps = (target - I.cost0 + I.nchunks - 1) / I.nchunks;
        if (steps < I.units) return I.unit0 + static_cast<int>(steps);
    }
    return a.units;
}

// The layer that unit u belongs to, searching up from layer i.
__device__ __forceinline__ int item_of(const GroupArgs &a, int u, int i)
{
    while (i + 1 < a.n_items && a.item[i + 1].unit0 <= u) ++i;
    return i;
}

// Prefetch `bytes` (a multiple of 16) at a 16-byte aligned address into L2.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// L1-allocating loads of activation-side data, issued after the wait for
// the previous kernel (asm volatile keeps them there): the prologue reads
// every row twice, for the statistics and for the codes.
__device__ __forceinline__ uint2 ld_ca_u2(const void *p)
{
    uint2 v;
    asm volatile("ld.global.ca.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint4 ld_ca_u4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.ca.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p)
                 : "memory");
    return v;
}

// Features k0..k0+3 of token row xr (bf16 when xbf16, else fp32), 0 past K.
__device__ __forceinline__ void quad_x(int xbf16, const char *xr, int64_t k0, int64_t K, float (&f)[4])
{
    const bool full = k0 + 4 <= K;
    if (xbf16) {
        const char *p = xr + 2 * k0;
        if (full && (reinterpret_cast<uintptr_t>(p) & 7u) == 0) {
            const uint2 w = ld_ca_u2(p);
            f[0] = __uint_as_float(w.x << 16);
            f[1] = __uint_as_float(w.x & 0xffff0000u);
            f[2] = __uint_as_float(w.y << 16);
            f[3] = __uint_as_float(w.y & 0xffff0000u);
            return;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] = k0 + e < K ? qrule::In<__nv_bfloat16>::scalar(xr, k0 + e) : 0.0f;
    } else {
        const char *p = xr + 4 * k0;
        if (full && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
            const uint4 w = ld_ca_u4(p);
            f[0] = __uint_as_float(w.x);
            f[1] = __uint_as_float(w.y);
            f[2] = __uint_as_float(w.z);
            f[3] = __uint_as_float(w.w);
            return;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) f[e] = k0 + e < K ? qrule::In<float>::scalar(xr, k0 + e) : 0.0f;
    }
}

// f *= g[k0..k0+3] (features past K keep their zero).
__device__ __forceinline__ void quad_gain(const float *g, int64_t k0, int64_t K, float (&f)[4])
{
    if (k0 + 4 <= K && (reinterpret_cast<uintptr_t>(g + k0) & 15u) == 0) {
        const uint4 w = ld_ca_u4(g + k0);
        f[0] = __fmul_rn(f[0], __uint_as_float(w.x));
        f[1] = __fmul_rn(f[1], __uint_as_float(w.y));
        f[2] = __fmul_rn(f[2], __uint_as_float(w.z));
        f[3] = __fmul_rn(f[3], __uint_as_float(w.w));
        return;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
        if (k0 + e < K) f[e] = __fmul_rn(f[e], ld_act_f32(g + k0 + e));
}

// Pass 1 of one 16-feature piece p of token t of layer I: max |x * g| bits
// into amax and, with norm, the fp64 sum of x^2 (before the gain) into ss,
// value by value in feature order.
__device__ __forceinline__ void piece_partial(const GroupItem &I, int xbf16, bool norm, int t, int64_t p,
                                              uint32_t &amax, double &ss)
{
    const char *xr = static_cast<const char *>(I.x) + t * I.ldx * (xbf16 ? 2 : 4);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float f[4];
        quad_x(xbf16, xr, 16 * p + 4 * e, I.K, f);
        if (norm) {
#pragma unroll
            for (int v = 0; v < 4; ++v) ss = __fma_rn(static_cast<double>(f[v]), static_cast<double>(f[v]), ss);
        }
        if (I.g != nullptr) quad_gain(I.g, 16 * p + 4 * e, I.K, f);
#pragma unroll
        for (int v = 0; v < 4; ++v) amax = max(amax, __float_as_uint(f[v]) & 0x7fffffffu);
    }
}

// s_x of a row from max |x * g| bits m and the sum of squares q2.
__device__ __forceinline__ float row_scale_of(uint32_t m, double q2, bool norm, int64_t K, float eps_norm)
{
    if (m == 0) return 0.0f;
    const float gm = __uint_as_float(m);
    if (!norm) return __fdiv_rn(gm, 127.0f);
    const double sc = __ddiv_rn(static_cast<double>(gm),
                                __dsqrt_rn(__dadd_rn(__ddiv_rn(q2, static_cast<double>(K)), static_cast<double>(eps_norm))));
    return __double2float_rn(__ddiv_rn(sc, 127.0));
}

// The 16 codes of piece p of token t of layer I for the row maximum bits m
// (zero past K and for an all-zero row).
__device__ __forceinline__ uint4 piece_codes(const GroupItem &I, int xbf16, int t, int64_t p, uint32_t m)
{
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    if (16 * p < I.K && m != 0) {
        const char *xr = static_cast<const char *>(I.x) + t * I.ldx * (xbf16 ? 2 : 4);
        const float gm = __uint_as_float(m);
        const float c = __fmul_rn(127.0f, __frcp_rn(gm));
        const bool slow = !(gm >= 0x1p-121f && gm < 0x1p126f);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float f[4];
            quad_x(xbf16, xr, 16 * p + 4 * e, I.K, f);
            if (I.g != nullptr) quad_gain(I.g, 16 * p + 4 * e, I.K, f);
            bool near = slow;
            w[e] = qrule::quant4(f[0], f[1], f[2], f[3], c, near);
            if (near) w[e] = qrule::quant4_exact(f[0], f[1], f[2], f[3], gm);
        }
        const int64_t valid = static_cast<int64_t>(I.K) - 16 * p;
        if (valid < 16) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int lo = 4 * e;
                uint32_t mk;
                if (valid >= lo + 4) mk = 0xffffffffu;
                else if (valid <= lo) mk = 0u;
                else mk = (1u << (8 * (valid - lo))) - 1u;
                w[e] &= mk;
            }
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Stores piece p's codes into row t of q_out (only the bytes below K).
__device__ __forceinline__ void store_codes(const GroupItem &I, int t, int64_t p, const uint4 &out)
{
    int8_t *dst = I.q_out + t * I.ldq_out + 16 * p;
    if (16 * p + 16 <= I.K) {
        *reinterpret_cast<uint4 *>(dst) = out;
    } else {
        const uint8_t *bytes = reinterpret_cast<const uint8_t *>(&out);
        for (int64_t e = 0; 16 * p + e < I.K; ++e) dst[e] = static_cast<int8_t>(bytes[e]);
    }
}

// The row statistics of every thread's pieces tid, tid + 256, ... reduced in
// a fixed order -- a shuffle tree, then the 8 warps in order -- so every
// block that computes a row gets the same maximum and scale.  Partials are
// exchanged through red_max / red_ss ([kWarps][MT]); the caller reads them
// after the block barrier this function ends with.
template <int MT>
__device__ __forceinline__ void reduce_rows(uint32_t (&amax)[MT], double (&ss)[MT], uint32_t (*red_max)[MT],
                                            double (*red_ss)[MT])
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            amax[t] = max(amax[t], __shfl_xor_sync(0xffffffffu, amax[t], o));
            ss[t] = __dadd_rn(ss[t], __shfl_xor_sync(0xffffffffu, ss[t], o));
        }
        if (lane == 0) {
            red_max[warp][t] = amax[t];
            red_ss[warp][t] = ss[t];
        }
    }
    __syncthreads();
}

template <int MT>
__device__ __forceinline__ void combine_row(const uint32_t (*red_max)[MT], const double (*red_ss)[MT], int t,
                                            uint32_t &m, double &q2)
{
    m = red_max[0][t];
    q2 = red_ss[0][t];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) {
        m = max(m, red_max[w][t]);
        q2 = __dadd_rn(q2, red_ss[w][t]);
    }
}

// The codes and scales of layers i0..i1 of the group, computed in this block
// from x: codes into qs (layer i at qoff[i - i0], [M][QP][nchunks]
// piece-major as the GEMV reads them, zero past K) and scales into
// sx_s[(i - i0) * MT + t].  Pass 1 reduces max |x*g| and, with the norm, the
// fp64 sum of x^2 over each row (reduce_rows: a fixed order, so every block
// gets the same scale), pass 2 reads the row again (L1) and writes the
// codes.  The block whose range holds the layer's first unit (`writer`) also
// stores them to q_out / s_x_out and reports non-finite rows.  Called by
// every thread of the block.
template <int QP, int MT>
__device__ void stage_block(const GroupArgs &a, int i0, int i1, int u_begin, int u_end, const int32_t *qoff,
                            uint4 *qs, float *sx_s)
{
    __shared__ uint32_t red_max[kWarps][MT];
    __shared__ double red_ss[kWarps][MT];
    __shared__ uint32_t gm_s[MT];
    const bool norm = a.norm != 0;
    for (int i = i0; i <= i1; ++i) {
        const GroupItem &I = a.item[i];
        const int64_t qp = static_cast<int64_t>(I.nchunks) * QP;  // code pieces per token row
        const int64_t np = (static_cast<int64_t>(I.K) + 15) / 16;  // pieces holding features
        uint4 *qi = qs + qoff[i - i0];
        const bool writer = u_begin <= I.unit0 && I.unit0 < u_end;
        uint32_t amax[MT];
        double ss[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            amax[t] = 0;
            ss[t] = 0.0;
        }
        for (int64_t p = threadIdx.x; p < np; p += blockDim.x) {
#pragma unroll
            for (int t = 0; t < MT; ++t)
                if (t < a.M) piece_partial(I, a.xbf16, norm, t, p, amax[t], ss[t]);
        }
        reduce_rows<MT>(amax, ss, red_max, red_ss);
        if (threadIdx.x < a.M) {
            const int t = threadIdx.x;
            uint32_t m;
            double q2;
            combine_row<MT>(red_max, red_ss, t, m, q2);
            const float sx = row_scale_of(m, q2, norm, I.K, a.eps_norm);
            gm_s[t] = m;
            sx_s[(i - i0) * MT + t] = sx;
            if (writer) {
                if (!finite_bits(m) || !finite_bits(__float_as_uint(__fmul_rn(__uint_as_float(m), 127.0f))))
                    report(a.status, LOWBIT_ERR_NONFINITE);
                if (I.s_x_out != nullptr) I.s_x_out[t] = sx;
            }
        }
        __syncthreads();
        for (int64_t p = threadIdx.x; p < qp; p += blockDim.x) {
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t >= a.M) continue;
                const uint4 out = piece_codes(I, a.xbf16, t, p, p < np ? gm_s[t] : 0u);
                qi[t * qp + (p % QP) * I.nchunks + p / QP] = out;
                if (writer && I.q_out != nullptr && p < np) store_codes(I, t, p, out);
            }
        }
    }
    __syncthreads();
}

// Held to three blocks per SM (at most 85 registers a thread).
template <int FMT, int MT, int U, int R, int OUT>
__global__ void __launch_bounds__(kWarps * 32, 3) gemv_group_kernel(const __grid_constant__ GroupArgs a)
{
    constexpr int QP = QPieces<FMT>::value;
    extern __shared__ uint4 qs[];
    __shared__ float sx_s[kGroupMax * MT];
    __shared__ int32_t qoff_s[kGroupMax];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t blocks = gridDim.x;
    const int u_begin = first_unit_at(a, static_cast<int64_t>(blockIdx.x) * a.cost_total / blocks);
    const int u_end = first_unit_at(a, (static_cast<int64_t>(blockIdx.x) + 1) * a.cost_total / blocks);
    const int i0 = item_of(a, u_begin, 0);
    const int i1 = u_end > u_begin ? item_of(a, u_end - 1, i0) : i0;
    auto row_of = [&](const GroupItem &I, int u) {
        return (static_cast<int64_t>(u - I.unit0) * kWarps + warp) * R;
    };
    // With prefetch the weight loads and prefetches are issued before the
    // wait for the previous kernel (the caller vouches that it does not
    // write the weights).
    bool waited = a.prefetch == 0;
    if (waited) pdl_wait();
    pdl_trigger();
    // L2 prefetch of the rows of this warp's units (the first unit's first
    // chunks are also loaded into registers right away; its later chunks and
    // the later units then come from L2)
    for (int u = u_begin, it = i0; u < u_end; ++u) {
        it = item_of(a, u, it);
        const GroupItem &I = a.item[it];
        const int64_t row = row_of(I, u) + lane;
        if (lane < R && row < I.N) prefetch_l2(I.packed + row * I.ldp, static_cast<uint32_t>(I.nchunks) * 16u);
    }
    if (threadIdx.x == 0) {
        int32_t off = 0;
        for (int i = i0; i <= i1; ++i) {
            qoff_s[i - i0] = off;
            off += a.M * a.item[i].nchunks * QP;
        }
    }
    __syncthreads();

    int it = i0;
    bool staged = false;
    float sxr[MT];
    for (int u = u_begin; u < u_end; ++u) {
        it = item_of(a, u, it);
        const GroupItem &I = a.item[it];
        const int64_t row0 = row_of(I, u);
        int32_t acc[R][MT];
        rows_dot<FMT, MT, U, R>(I.packed, I.ldp, I.nchunks, I.N, row0, a.M, qs + qoff_s[it - i0], [&] {
            if (!staged) {
                if (!waited) {
                    pdl_wait();
                    waited = true;
                }
                stage_block<QP, MT>(a, i0, i1, u_begin, u_end, qoff_s, qs, sx_s);
                staged = true;
            }
#pragma unroll
            for (int t = 0; t < MT; ++t) sxr[t] = sx_s[(it - i0) * MT + t];
        }, acc);
        rows_store<FMT, MT, R, OUT>(acc, row0, I.N, a.M, I.s_w, I.y, I.ldy, sxr);
    }
    if (!waited) pdl_wait();
}

// Resident blocks with `smem` bytes of codes, per device (cached; 0 when the
// query fails).
template <int FMT, int MT, int U, int R, int OUT>
int group_resident_blocks(size_t smem)
{
    struct Entry { int dev; size_t smem; int blocks; };
    static std::mutex mu;
    static Entry cache[64];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].smem == smem) return cache[i].blocks;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_group_kernel<FMT, MT, U, R, OUT>, kWarps * 32,
                                                      smem) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    const int blocks = per_sm * device_sm_count();
    if (blocks > 0 && used < 64) cache[used++] = Entry{dev, smem, blocks};
    return blocks;
}

template <int FMT, int MT, int U, int R, int OUT>
lowbit_status launch_group_out(GroupArgs &a, size_t smem, cudaStream_t st)
{
    const int resident = group_resident_blocks<FMT, MT, U, R, OUT>(smem);
    if (resident <= 0) return LOWBIT_ERR_CUDA;
    const int64_t blocks = a.units < resident ? a.units : resident;
    return launch_pdl(gemv_group_kernel<FMT, MT, U, R, OUT>, dim3(static_cast<unsigned>(blocks)), dim3(kWarps * 32),
                      smem, st, 0, a);
}

template <int FMT, int MT, int U, int R>
lowbit_status launch_group(GroupArgs &a, lowbit_dtype ydt, size_t smem, cudaStream_t st)
{
    static PerDevice configured;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            const int lim = static_cast<int>(kGemvSmemMax);
            return (cudaFuncSetAttribute(gemv_group_kernel<FMT, MT, U, R, LOWBIT_F32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess &&
                    cudaFuncSetAttribute(gemv_group_kernel<FMT, MT, U, R, LOWBIT_BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess &&
                    cudaFuncSetAttribute(gemv_group_kernel<FMT, MT, U, R, LOWBIT_I32>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess) ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    const int64_t rows_per_block = kWarps * R;
    int64_t units = 0, cost = 0;
    for (int i = 0; i < a.n_items; ++i) {
        GroupItem &I = a.item[i];
        I.unit0 = static_cast<int32_t>(units);
        I.units = static_cast<int32_t>((I.N + rows_per_block - 1) / rows_per_block);
        I.cost0 = cost;
        units += I.units;
        cost += static_cast<int64_t>(I.units) * I.nchunks;
    }
    if (units > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    a.units = static_cast<int>(units);
    a.cost_total = cost;
    if (ydt == LOWBIT_F32) return launch_group_out<FMT, MT, U, R, LOWBIT_F32>(a, smem, st);
    if (ydt == LOWBIT_BF16) return launch_group_out<FMT, MT, U, R, LOWBIT_BF16>(a, smem, st);
    return launch_group_out<FMT, MT, U, R, LOWBIT_I32>(a, smem, st);
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
    const int64_t qpieces = nchunks * QPieces<FMT>::value;
    const int64_t smem_i = static_cast<int64_t>(M) * qpieces * 16;
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

// U and R for a group: R (rows per warp) so that the units about fill the
// resident blocks (three per SM) once, with U = 2 chunks per lane; a group
// of few rows takes R = 1 and U from its longest rows, as the plain GEMV.
template <int FMT, int MT>
lowbit_status launch_group_tokens(GroupArgs &a, int64_t max_nchunks, int64_t rows, lowbit_dtype ydt, size_t smem,
                                  cudaStream_t st)
{
    const int64_t warps = static_cast<int64_t>(device_sm_count()) * 3 * kWarps;  // resident warps
    if constexpr (MT == 1) {
        if (rows >= 2 * warps) return launch_group<FMT, MT, 2, 4>(a, ydt, smem, st);
    }
    if (rows >= warps) return launch_group<FMT, MT, 2, 2>(a, ydt, smem, st);
    if (max_nchunks <= 64) return launch_group<FMT, MT, 2, 1>(a, ydt, smem, st);
    // (eight chunks per lane do not fit the registers with four tokens)
    if constexpr (MT == 1) {
        if (max_nchunks > 160) return launch_group<FMT, MT, 8, 1>(a, ydt, smem, st);
    }
    return launch_group<FMT, MT, 5, 1>(a, ydt, smem, st);
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

// The grouped fused decode call (nchunks of every item set by the caller).
// The codes of all layers of a launch are staged in shared memory at once,
// so consecutive layers are launched together while their codes fit
// kGemvSmemMax (every single layer fits: the caller checks it).
template <int FMT>
lowbit_status gemv_group_launch_fmt(const GroupArgs &all, lowbit_dtype ydt, cudaStream_t st)
{
    constexpr int QP = QPieces<FMT>::value;
    int first = 0;
    while (first < all.n_items) {
        GroupArgs a = all;
        int64_t bytes = 0, max_nchunks = 0, rows = 0;
        int n = 0;
        while (first + n < all.n_items) {
            const GroupItem &I = all.item[first + n];
            const int64_t b = static_cast<int64_t>(all.M) * I.nchunks * QP * 16;
            if (n > 0 && bytes + b > kGemvSmemMax) break;
            if (b > kGemvSmemMax) return LOWBIT_ERR_INVALID_ARG;
            a.item[n] = I;
            bytes += b;
            max_nchunks = I.nchunks > max_nchunks ? I.nchunks : max_nchunks;
            rows += I.N;
            ++n;
        }
        a.n_items = n;
        const size_t smem = static_cast<size_t>(bytes);
        const lowbit_status s = all.M == 1 ? launch_group_tokens<FMT, 1>(a, max_nchunks, rows, ydt, smem, st)
                                           : launch_group_tokens<FMT, 4>(a, max_nchunks, rows, ydt, smem, st);
        if (s != LOWBIT_OK) return s;
        first += n;
    }
    return LOWBIT_OK;
}

}  // namespace gemv_detail

}  // namespace lowbit
