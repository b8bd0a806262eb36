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

// Activation side of a fused decode call (lowbit_bitlinear): the token rows
// x [M, ldx] (fp32 or bf16) with an optional gain g and RMSNorm, from which
// every block computes the int8 codes and scales itself (the per-token rule
// of quant_rule.cuh; the RMSNorm factor enters only the scale).  Block 0
// also writes the codes and scales to q_out / s_x_out when they are given.
struct Prologue {
    const void *x;
    int64_t ldx;
    const float *g;
    int8_t *q_out;
    int64_t ldq_out;
    float *s_x_out;
    int32_t *status;
    float eps_norm;
    int xbf16;
    int norm;
};

// Element k of token row xr as fp32 (0 past K).
__device__ __forceinline__ float x_at(const Prologue &p, const char *xr, int64_t k, int64_t K)
{
    if (k >= K) return 0.0f;
    return p.xbf16 ? qrule::In<__nv_bfloat16>::scalar(xr, k) : qrule::In<float>::scalar(xr, k);
}

// Raw data of one 16-feature piece of a token row: 16 bf16 values in words
// 0-7, or 16 fp32 values in words 0-15 (f32 set), zero past K.
struct Piece {
    uint32_t w[16];
    bool f32;
};

__device__ __forceinline__ void put4(uint32_t (&w)[16], int at, const uint4 &v)
{
    w[at] = v.x;
    w[at + 1] = v.y;
    w[at + 2] = v.z;
    w[at + 3] = v.w;
}

// Issues the loads of piece j of token row xr (16-byte vector loads when the
// piece is whole and aligned, else element loads as fp32).
__device__ __forceinline__ void load_piece(const Prologue &p, const char *xr, int64_t j, int64_t K, Piece &pc)
{
    const int64_t k0 = 16 * j;
    pc.f32 = !p.xbf16;
    if (k0 >= K) {
#pragma unroll
        for (int i = 0; i < 16; ++i) pc.w[i] = 0u;
        pc.f32 = true;
        return;
    }
    const bool vec = k0 + 16 <= K && (reinterpret_cast<uintptr_t>(xr) & 15u) == 0;
    if (vec && p.xbf16) {
        put4(pc.w, 0, ld_act_u4(xr + k0 * 2));
        put4(pc.w, 4, ld_act_u4(xr + k0 * 2 + 16));
    } else if (vec) {
#pragma unroll
        for (int i = 0; i < 4; ++i) put4(pc.w, 4 * i, ld_act_u4(xr + k0 * 4 + 16 * i));
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) pc.w[i] = __float_as_uint(x_at(p, xr, k0 + i, K));
        pc.f32 = true;
    }
}

__device__ __forceinline__ float piece_value(const Piece &pc, int i)
{
    if (pc.f32) return __uint_as_float(pc.w[i]);
    const uint32_t w = pc.w[i >> 1];
    return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
}

// Codes and scales of the M <= MT token rows, staged into qs (piece-major, as
// the q staging of gemv_smem_kernel) and sx_s[M].  Called by every thread of
// the block.  Each thread takes pieces threadIdx.x + blockDim.x * i; the
// loads of a batch of PB pieces of every token are all issued before any is
// used (one L2 round trip per batch), and when the row fits one batch it
// stays in registers for the code pass.
template <int QP, int MT>
__device__ void stage_codes_from_x(const Prologue &p, int M, int64_t K, int64_t nchunks, uint4 *qs, float *sx_s)
{
    constexpr int PB = MT == 1 ? 4 : 1;
    __shared__ uint32_t red_max[kWarps][MT];
    __shared__ double red_ss[kWarps][MT];
    const int64_t qpieces = nchunks * QP;
    const int64_t npieces = (K + 15) / 16;
    const int64_t per_batch = static_cast<int64_t>(blockDim.x) * PB;
    const bool single = npieces <= per_batch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t xsz = p.xbf16 ? 2 : 4;
    uint32_t amax[MT];
    double ss[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        amax[t] = 0;
        ss[t] = 0.0;
    }
    Piece pc[PB][MT];
    auto load_batch = [&](int64_t b0) {
#pragma unroll
        for (int b = 0; b < PB; ++b)
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                const int64_t j = b0 + threadIdx.x + static_cast<int64_t>(blockDim.x) * b;
                if (t < M) load_piece(p, static_cast<const char *>(p.x) + t * p.ldx * xsz, j, K, pc[b][t]);
            }
    };
    // pass 1: max |x*g| and sum of x^2 per token
    for (int64_t b0 = 0; b0 < npieces; b0 += per_batch) {
        load_batch(b0);
#pragma unroll
        for (int b = 0; b < PB; ++b) {
            const int64_t j = b0 + threadIdx.x + static_cast<int64_t>(blockDim.x) * b;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t < M && 16 * j < K) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float v = piece_value(pc[b][t], i);
                        if (p.norm) ss[t] = __fma_rn(static_cast<double>(v), static_cast<double>(v), ss[t]);
                        const float u = (p.g != nullptr && 16 * j + i < K) ? __fmul_rn(v, p.g[16 * j + i]) : v;
                        amax[t] = max(amax[t], __float_as_uint(u) & 0x7fffffffu);
                    }
                }
            }
        }
    }
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
    float gm[MT], c[MT];
    bool slow[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        uint32_t a = red_max[0][t];
        double q2 = red_ss[0][t];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            a = max(a, red_max[w][t]);
            q2 = __dadd_rn(q2, red_ss[w][t]);
        }
        amax[t] = a;
        gm[t] = __uint_as_float(a);
        c[t] = __fmul_rn(127.0f, __frcp_rn(gm[t]));
        slow[t] = !(gm[t] >= 0x1p-121f && gm[t] < 0x1p126f);
        if (threadIdx.x == 0 && t < M) {
            float sx = 0.0f;
            if (a != 0) {
                if (p.norm) {
                    double s = __ddiv_rn(static_cast<double>(gm[t]),
                                         __dsqrt_rn(__dadd_rn(__ddiv_rn(q2, static_cast<double>(K)),
                                                              static_cast<double>(p.eps_norm))));
                    sx = __double2float_rn(__ddiv_rn(s, 127.0));
                } else {
                    sx = __fdiv_rn(gm[t], 127.0f);
                }
            }
            sx_s[t] = sx;
            const bool bad = !finite_bits(a) || !finite_bits(__float_as_uint(__fmul_rn(gm[t], 127.0f)));
            if (blockIdx.x == 0) {
                if (bad) report(p.status, LOWBIT_ERR_NONFINITE);
                if (p.s_x_out != nullptr) p.s_x_out[t] = sx;
            }
        }
    }
    // pass 2: codes, 16 per piece (pieces past K are zero codes)
    for (int64_t b0 = 0; b0 < qpieces; b0 += per_batch) {
        if (!(single && b0 == 0)) load_batch(b0);
#pragma unroll
        for (int b = 0; b < PB; ++b) {
            const int64_t j = b0 + threadIdx.x + static_cast<int64_t>(blockDim.x) * b;
            if (j >= qpieces) continue;
#pragma unroll
            for (int t = 0; t < MT; ++t) {
                if (t < M) {
                    uint4 out = make_uint4(0, 0, 0, 0);
                    if (16 * j < K && amax[t] != 0) {
                        float u[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float v = piece_value(pc[b][t], i);
                            u[i] = (p.g != nullptr && 16 * j + i < K) ? __fmul_rn(v, p.g[16 * j + i]) : v;
                        }
                        bool near = slow[t];
                        uint32_t w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            w[i] = qrule::quant4(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3], c[t], near);
                        if (near) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                w[i] = qrule::quant4_exact(u[4 * i], u[4 * i + 1], u[4 * i + 2], u[4 * i + 3], gm[t]);
                        }
                        // features past K are zero codes
                        const int64_t valid = K - 16 * j;
                        if (valid < 16) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int lo = 4 * i;
                                uint32_t m;
                                if (valid >= lo + 4) m = 0xffffffffu;
                                else if (valid <= lo) m = 0u;
                                else m = (1u << (8 * (valid - lo))) - 1u;
                                w[i] &= m;
                            }
                        }
                        out = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                    qs[t * qpieces + (j % QP) * nchunks + j / QP] = out;
                    if (blockIdx.x == 0 && p.q_out != nullptr && 16 * j < K) {
                        int8_t *dst = p.q_out + t * p.ldq_out + 16 * j;
                        if (16 * j + 16 <= K) {
                            *reinterpret_cast<uint4 *>(dst) = out;
                        } else {
                            const uint8_t *bytes = reinterpret_cast<const uint8_t *>(&out);
                            for (int64_t i = 0; 16 * j + i < K; ++i) dst[i] = static_cast<int8_t>(bytes[i]);
                        }
                    }
                }
            }
        }
    }
}

// The token codes are staged once per block into shared memory (zero past K)
// after the block's weight loads are in flight, so their latency overlaps the
// DRAM round trip; each lane then reads a chunk's activation bytes once and
// applies them to all R rows it holds.
// With PRO the codes are computed in the block from the token rows instead
// (see Prologue); q and s_x are then unused.
template <int FMT, int MT, int U, int R, int OUT, bool PRO = false>
__global__ void __launch_bounds__(kWarps * 32)
gemv_smem_kernel(const int8_t *__restrict__ q, int64_t ldq, const float *__restrict__ s_x, int M, int64_t K,
                 const uint8_t *__restrict__ packed, int64_t ldp, int64_t nchunks, const float *__restrict__ s_w,
                 int64_t N, void *__restrict__ y, int64_t ldy, int prefetch, Prologue pro)
{
    using F = Fmt<FMT>;
    constexpr int QP = QPieces<FMT>::value;
    extern __shared__ uint4 qs[];  // [M][QP][nchunks]: piece-major, so lanes read consecutive pieces
    __shared__ float sx_s[PRO ? MT : 1];
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
    float sxr[MT];  // the token scales, read once

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
            if constexpr (PRO) {
                stage_codes_from_x<QP, MT>(pro, M, K, nchunks, qs, sx_s);
            } else {
                // token scales first, then the codes in batches whose loads are
                // all issued before the shared-memory stores (one L2 round trip
                // per batch)
#pragma unroll
                for (int t = 0; t < MT; ++t) sxr[t] = t < M ? ld_act_f32(s_x + t) : 0.0f;
                constexpr int kBatch = 4;
                for (int64_t i0 = threadIdx.x; i0 < M * qpieces; i0 += static_cast<int64_t>(blockDim.x) * kBatch) {
                    uint4 v[kBatch];
#pragma unroll
                    for (int b = 0; b < kBatch; ++b) {
                        const int64_t i = i0 + static_cast<int64_t>(blockDim.x) * b;
                        if (i < M * qpieces) v[b] = load_q16(q + (i / qpieces) * ldq, (i % qpieces) * 16, K);
                    }
#pragma unroll
                    for (int b = 0; b < kBatch; ++b) {
                        const int64_t i = i0 + static_cast<int64_t>(blockDim.x) * b;
                        if (i < M * qpieces) {
                            const int64_t t = i / qpieces, j = i % qpieces;   // j = chunk * QP + piece
                            qs[t * qpieces + (j % QP) * nchunks + j / QP] = v[b];
                        }
                    }
                }
            }
            __syncthreads();
            if constexpr (PRO) {
#pragma unroll
                for (int t = 0; t < MT; ++t) sxr[t] = sx_s[t];
            }
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
            if (lane == t && t < M && row < N)
                store_out<OUT>(y, t * ldy + row, v >> F::kShift, sw, sxr[t]);
        }
    }
}

constexpr int64_t kGemvSmemMax = 96 * 1024;

template <int FMT, int MT, int U, int R, bool PRO>
lowbit_status launch_smem_t(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                            const uint8_t *packed, int64_t ldp, int64_t nchunks, const float *s_w, int64_t N, void *y,
                            lowbit_dtype ydt, int64_t ldy, size_t smem, int prefetch, const Prologue &pro,
                            cudaStream_t st)
{
    static PerDevice configured;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            const int lim = static_cast<int>(kGemvSmemMax);
            return (cudaFuncSetAttribute(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_F32, PRO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess &&
                    cudaFuncSetAttribute(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_BF16, PRO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess &&
                    cudaFuncSetAttribute(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_I32, PRO>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, lim) == cudaSuccess) ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    const int64_t blocks = (N + kWarps * R - 1) / (kWarps * R);
    const dim3 g(static_cast<unsigned>(blocks)), b(kWarps * 32);
    if (ydt == LOWBIT_F32)
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_F32, PRO>, g, b, smem, st, 0, q, ldq, s_x, M, K,
                          packed, ldp, nchunks, s_w, N, y, ldy, prefetch, pro);
    else if (ydt == LOWBIT_BF16)
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_BF16, PRO>, g, b, smem, st, 0, q, ldq, s_x, M, K,
                          packed, ldp, nchunks, s_w, N, y, ldy, prefetch, pro);
    else
        return launch_pdl(gemv_smem_kernel<FMT, MT, U, R, LOWBIT_I32, PRO>, g, b, smem, st, 0, q, ldq, s_x, M, K,
                          packed, ldp, nchunks, s_w, N, y, ldy, prefetch, pro);
}

template <int FMT, int MT, int U, int R>
lowbit_status launch_smem(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K, const uint8_t *packed,
                          int64_t ldp, int64_t nchunks, const float *s_w, int64_t N, void *y, lowbit_dtype ydt,
                          int64_t ldy, size_t smem, int prefetch, const Prologue *pro, cudaStream_t st)
{
    if (pro != nullptr)
        return launch_smem_t<FMT, MT, U, R, true>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem,
                                                  prefetch, *pro, st);
    return launch_smem_t<FMT, MT, U, R, false>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem,
                                               prefetch, Prologue{}, st);
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
// grid stays near one wave of two blocks per SM.  With `pro` the block
// computes the codes from the token rows itself (the staging must then fit
// shared memory; the caller checks gemv_fused_fits).
template <int FMT, int MT>
lowbit_status launch_tokens(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                            const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N,
                            void *y, lowbit_dtype ydt, int64_t ldy, int prefetch, cudaStream_t st,
                            const Prologue *pro = nullptr)
{
    const int64_t nchunks = (row_bytes + 15) / 16;
    const int64_t smem_i = static_cast<int64_t>(M) * nchunks * QPieces<FMT>::value * 16;
    if (smem_i > kGemvSmemMax) {
        if (pro != nullptr) return LOWBIT_ERR_INVALID_ARG;
        return launch_global<FMT, MT>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, prefetch, st);
    }
    const size_t smem = static_cast<size_t>(smem_i);
    const int64_t slots = static_cast<int64_t>(device_sm_count()) * 2 * kWarps;  // warps in one wave
    if (nchunks <= 64) {
        if constexpr (MT == 1) {
            if (N >= 4 * slots)
                return launch_smem<FMT, MT, 2, 4>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, pro, st);
        }
        if (N >= 2 * slots)
            return launch_smem<FMT, MT, 2, 2>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, pro, st);
        return launch_smem<FMT, MT, 2, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, pro, st);
    }
    if (nchunks <= 160)
        return launch_smem<FMT, MT, 5, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, pro, st);
    return launch_smem<FMT, MT, 8, 1>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ydt, ldy, smem, prefetch, pro, st);
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

// The fused decode call: M <= 4 token rows, codes computed in every block.
template <int FMT>
lowbit_status gemv_fused_launch_fmt(const Prologue &pro, int64_t M, int64_t K, const uint8_t *packed, int64_t ldp,
                                    int64_t row_bytes, const float *s_w, int64_t N, void *y, lowbit_dtype ydt,
                                    int64_t ldy, int prefetch, cudaStream_t st)
{
    const int m = static_cast<int>(M);
    if (m == 1)
        return launch_tokens<FMT, 1>(nullptr, 0, nullptr, m, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch,
                                     st, &pro);
    return launch_tokens<FMT, 4>(nullptr, 0, nullptr, m, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st,
                                 &pro);
}

}  // namespace gemv_detail

// True when the fused decode GEMV can stage the codes of M tokens of K
// features (format f) in shared memory.
inline bool gemv_fused_fits(int64_t M, int64_t K, int64_t row_bytes, lowbit_format f)
{
    if (M < 1 || M > 4) return false;
    const int64_t nchunks = (row_bytes + 15) / 16;
    const int64_t qp = f == LOWBIT_TERNARY2 ? 4 : (f == LOWBIT_BINARY1 ? 8 : 2);
    (void)K;
    return M * nchunks * qp * 16 <= gemv_detail::kGemvSmemMax;
}

}  // namespace lowbit
