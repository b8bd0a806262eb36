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

// Activation side of one layer of a fused decode call (lowbit_bitlinear,
// lowbit_bitlinear_group): the token rows x [M, ldx] (fp32 or bf16) with an
// optional gain g and RMSNorm, from which the blocks of a cluster compute the
// int8 codes and scales themselves (the per-token rule of quant_rule.cuh; the
// RMSNorm factor enters only the scale), and to which one cluster also writes
// the codes and scales (q_out / s_x_out) when they are given.
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

// Thread-block cluster helpers of the fused decode GEMV.
__device__ __forceinline__ uint32_t cl_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cl_size()
{
    uint32_t n;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
    return n;
}
__device__ __forceinline__ void cl_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of `local` in block `rank` of the cluster
__device__ __forceinline__ uint32_t cl_map(const void *local, uint32_t rank)
{
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(a)
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(local))), "r"(rank));
    return a;
}
__device__ __forceinline__ void cl_st128(uint32_t addr, const uint4 &v)
{
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ uint32_t cl_ld32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ double cl_ld64(uint32_t addr)
{
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
    return v;
}

// The 16 values of piece j (features 16j..16j+15) of token row xr, 0 past K.
__device__ __forceinline__ void piece_values(const Prologue &p, const char *xr, int64_t j, int64_t K, float (&u)[16])
{
    const int64_t k0 = 16 * j;
    const bool vec = k0 + 16 <= K && (reinterpret_cast<uintptr_t>(xr) & 15u) == 0;
    if (vec && p.xbf16) {
        const uint4 a = ld_act_u4(xr + k0 * 2);
        const uint4 b = ld_act_u4(xr + k0 * 2 + 16);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            u[e] = qrule::In<__nv_bfloat16>::get(a, e);
            u[8 + e] = qrule::In<__nv_bfloat16>::get(b, e);
        }
    } else if (vec) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 a = ld_act_u4(xr + k0 * 4 + 16 * i);
            u[4 * i] = __uint_as_float(a.x);
            u[4 * i + 1] = __uint_as_float(a.y);
            u[4 * i + 2] = __uint_as_float(a.z);
            u[4 * i + 3] = __uint_as_float(a.w);
        }
    } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int64_t k = k0 + e;
            u[e] = k >= K ? 0.0f
                          : (p.xbf16 ? qrule::In<__nv_bfloat16>::scalar(xr, k) : qrule::In<float>::scalar(xr, k));
        }
    }
}

// Codes and scales of the M <= MT token rows, staged into qs (piece-major, as
// the q staging of gemv_smem_kernel) and sx_s[M] of every block of the
// cluster.  The blocks of a cluster share the work: block r of C takes code
// pieces [r P / C, (r + 1) P / C) of every token.  Each block reduces its
// share's max |x*g| and sum of squares, the C partials are read over
// distributed shared memory and combined in rank order (so every block gets
// the same row maximum and scale), then each block quantises its share and
// writes each 16-code piece into the code buffer of every block of the
// cluster.  The blocks of one cluster per layer (`writer`) also store the
// codes and scales to q_out / s_x_out and report non-finite rows.  Called by
// every thread of every block of the cluster.
template <int QP, int MT, bool KEEP>
__device__ void stage_codes_from_x(const Prologue &p, int M, int64_t K, int64_t nchunks, uint4 *qs, float *sx_s,
                                   bool writer)
{
    __shared__ uint32_t red_max[kWarps][MT];
    __shared__ double red_ss[kWarps][MT];
    __shared__ uint32_t part_max[MT];
    __shared__ double part_ss[MT];
    const uint32_t C = cl_size(), rank = cl_rank();
    const int64_t qpieces = nchunks * QP;
    const int64_t j0 = static_cast<int64_t>(rank) * qpieces / C, j1 = static_cast<int64_t>(rank + 1) * qpieces / C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t xsz = p.xbf16 ? 2 : 4;

    // pass 1: this block's share, max |x*g| and sum of x^2 per token.  With
    // KEEP (one token) and a share of at most one piece per thread, the piece
    // stays in registers for the code pass.
    constexpr bool kKeep = KEEP && MT == 1;
    const bool keep = kKeep && (j1 - j0) <= static_cast<int64_t>(blockDim.x);
    float held[16];
    uint32_t amax[MT];
    double ss[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        amax[t] = 0;
        ss[t] = 0.0;
    }
    for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
        if (16 * j >= K) continue;
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (t < M) {
                float u[16];
                piece_values(p, static_cast<const char *>(p.x) + t * p.ldx * xsz, j, K, u);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    if (p.norm) ss[t] = __fma_rn(static_cast<double>(u[e]), static_cast<double>(u[e]), ss[t]);
                    if (p.g != nullptr && 16 * j + e < K) u[e] = __fmul_rn(u[e], p.g[16 * j + e]);
                    amax[t] = max(amax[t], __float_as_uint(u[e]) & 0x7fffffffu);
                }
                if constexpr (kKeep) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) held[e] = u[e];
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
    if (threadIdx.x < MT) {
        const int t = threadIdx.x;
        uint32_t a = red_max[0][t];
        double q2 = red_ss[0][t];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) {
            a = max(a, red_max[w][t]);
            q2 = __dadd_rn(q2, red_ss[w][t]);
        }
        part_max[t] = a;
        part_ss[t] = q2;
    }
    cl_sync();  // every block's partials are visible in the cluster
    // one thread per (peer, token) fetches that partial into this block
    __shared__ uint32_t all_max[8][MT];
    __shared__ double all_ss[8][MT];
    if (threadIdx.x < C * MT) {
        const uint32_t s = threadIdx.x / MT, t = threadIdx.x % MT;
        all_max[s][t] = cl_ld32(cl_map(&part_max[t], s));
        all_ss[s][t] = cl_ld64(cl_map(&part_ss[t], s));
    }
    __syncthreads();

    // the whole rows' statistics, combined in rank order
    float gm[MT], c[MT];
    bool slow[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
        uint32_t a = 0;
        double q2 = 0.0;
        for (uint32_t s = 0; s < C; ++s) {
            a = max(a, all_max[s][t]);
            q2 = __dadd_rn(q2, all_ss[s][t]);
        }
        amax[t] = a;
        gm[t] = __uint_as_float(a);
        c[t] = __fmul_rn(127.0f, __frcp_rn(gm[t]));
        slow[t] = !(gm[t] >= 0x1p-121f && gm[t] < 0x1p126f);
        if (threadIdx.x == 0 && t < M) {
            float sx = 0.0f;
            if (a != 0) {
                if (p.norm) {
                    double sc = __ddiv_rn(static_cast<double>(gm[t]),
                                          __dsqrt_rn(__dadd_rn(__ddiv_rn(q2, static_cast<double>(K)),
                                                               static_cast<double>(p.eps_norm))));
                    sx = __double2float_rn(__ddiv_rn(sc, 127.0));
                } else {
                    sx = __fdiv_rn(gm[t], 127.0f);
                }
            }
            sx_s[t] = sx;
            const bool bad = !finite_bits(a) || !finite_bits(__float_as_uint(__fmul_rn(gm[t], 127.0f)));
            if (writer && rank == 0) {
                if (bad) report(p.status, LOWBIT_ERR_NONFINITE);
                if (p.s_x_out != nullptr) p.s_x_out[t] = sx;
            }
        }
    }
    // pass 2: codes of this block's share (pieces past K are zero codes),
    // written to every block of the cluster
    for (int64_t j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
            if (t < M) {
                uint4 out = make_uint4(0, 0, 0, 0);
                if (16 * j < K && amax[t] != 0) {
                    float u[16];
                    if (keep) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) u[e] = held[e];
                    } else {
                        piece_values(p, static_cast<const char *>(p.x) + t * p.ldx * xsz, j, K, u);
                        if (p.g != nullptr) {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                if (16 * j + e < K) u[e] = __fmul_rn(u[e], p.g[16 * j + e]);
                        }
                    }
                    bool near = slow[t];
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        w[e] = qrule::quant4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3], c[t], near);
                    if (near) {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = qrule::quant4_exact(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3], gm[t]);
                    }
                    const int64_t valid = K - 16 * j;
                    if (valid < 16) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int lo = 4 * e;
                            uint32_t m;
                            if (valid >= lo + 4) m = 0xffffffffu;
                            else if (valid <= lo) m = 0u;
                            else m = (1u << (8 * (valid - lo))) - 1u;
                            w[e] &= m;
                        }
                    }
                    out = make_uint4(w[0], w[1], w[2], w[3]);
                }
                const uint4 *slot = &qs[t * qpieces + (j % QP) * nchunks + j / QP];
                for (uint32_t s = 0; s < C; ++s) cl_st128(cl_map(slot, s), out);
                if (writer && p.q_out != nullptr && 16 * j < K) {
                    int8_t *dst = p.q_out + t * p.ldq_out + 16 * j;
                    if (16 * j + 16 <= K) {
                        *reinterpret_cast<uint4 *>(dst) = out;
                    } else {
                        const uint8_t *bytes = reinterpret_cast<const uint8_t *>(&out);
                        for (int64_t e = 0; 16 * j + e < K; ++e) dst[e] = static_cast<int8_t>(bytes[e]);
                    }
                }
            }
        }
    }
    cl_sync();  // every code piece has reached every block
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
// The work is cut into units of C blocks x 8 warps x R rows of one layer;
// cluster c of the grid (C blocks, C <= 8) takes a contiguous range of units
// whose packed bytes are about 1/clusters of the group's (persistent: the
// grid holds at most as many clusters as are resident at once).  Whenever a
// cluster reaches a unit of the next layer, its blocks compute that layer's
// codes together (stage_codes_from_x) while the unit's first weight loads
// are in flight.  The layers are independent: no layer may read what another
// writes.
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

// Held to three blocks per SM (at most 85 registers a thread).
template <int FMT, int MT, int U, int R, int OUT>
__global__ void __launch_bounds__(kWarps * 32, 3) gemv_group_kernel(const __grid_constant__ GroupArgs a)
{
    constexpr int QP = QPieces<FMT>::value;
    extern __shared__ uint4 qs[];
    __shared__ float sx_s[MT];
    const int warp = threadIdx.x >> 5;
    const uint32_t C = cl_size(), rank = cl_rank();
    const int64_t clusters = gridDim.x / C, cl = blockIdx.x / C;
    const int u_begin = first_unit_at(a, cl * a.cost_total / clusters);
    const int u_end = first_unit_at(a, (cl + 1) * a.cost_total / clusters);
    // With prefetch the first weight loads are issued before the wait for the
    // previous kernel (the caller vouches that it does not write the weights).
    bool waited = a.prefetch == 0;
    if (waited) pdl_wait();
    pdl_trigger();
    int it = 0, cur = -1;
    float sxr[MT];
    for (int u = u_begin; u < u_end; ++u) {
        while (it + 1 < a.n_items && a.item[it + 1].unit0 <= u) ++it;
        const GroupItem &I = a.item[it];
        const int64_t row0 = ((static_cast<int64_t>(u - I.unit0) * C + rank) * kWarps + warp) * R;
        int32_t acc[R][MT];
        rows_dot<FMT, MT, U, R>(I.packed, I.ldp, I.nchunks, I.N, row0, a.M, qs, [&] {
            if (it == cur) return;  // the same layer's codes are staged already
            if (!waited) {
                pdl_wait();
                waited = true;
            }
            if (cur >= 0) cl_sync();  // every block of the cluster is done with the previous codes
            Prologue p;
            p.x = I.x;
            p.ldx = I.ldx;
            p.g = I.g;
            p.q_out = I.q_out;
            p.ldq_out = I.ldq_out;
            p.s_x_out = I.s_x_out;
            p.status = a.status;
            p.eps_norm = a.eps_norm;
            p.xbf16 = a.xbf16;
            p.norm = a.norm;
            stage_codes_from_x<QP, MT, (U * R <= 5)>(p, a.M, I.K, I.nchunks, qs, sx_s, u == I.unit0);
            __syncthreads();
#pragma unroll
            for (int t = 0; t < MT; ++t) sxr[t] = sx_s[t];
            cur = it;
        }, acc);
        rows_store<FMT, MT, R, OUT>(acc, row0, I.N, a.M, I.s_w, I.y, I.ldy, sxr);
    }
}

// Resident clusters of C blocks with `smem` bytes of codes each, per device
// (cached; 0 when the query fails).
template <int FMT, int MT, int U, int R, int OUT>
int group_resident_clusters(unsigned C, size_t smem)
{
    struct Entry { int dev; unsigned C; size_t smem; int clusters; };
    static std::mutex mu;
    static Entry cache[64];
    static int used = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].dev == dev && cache[i].C == C && cache[i].smem == smem) return cache[i].clusters;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = C;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemv_group_kernel<FMT, MT, U, R, OUT>, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    if (clusters > 0 && used < 64) cache[used++] = Entry{dev, C, smem, clusters};
    return clusters;
}

template <int FMT, int MT, int U, int R, int OUT>
lowbit_status launch_group_out(GroupArgs &a, unsigned C, size_t smem, cudaStream_t st)
{
    const int resident = group_resident_clusters<FMT, MT, U, R, OUT>(C, smem);
    if (resident <= 0) return LOWBIT_ERR_CUDA;
    const int64_t clusters = a.units < resident ? a.units : resident;
    return launch_pdl(gemv_group_kernel<FMT, MT, U, R, OUT>, dim3(static_cast<unsigned>(clusters * C)),
                      dim3(kWarps * 32), smem, st, C, a);
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
    // units of C blocks; C = 8 unless every layer has fewer row blocks
    const int64_t rows_per_block = kWarps * R;
    int64_t max_blocks = 1;
    for (int i = 0; i < a.n_items; ++i) {
        const int64_t blocks = (a.item[i].N + rows_per_block - 1) / rows_per_block;
        max_blocks = blocks > max_blocks ? blocks : max_blocks;
    }
    const unsigned C = static_cast<unsigned>(max_blocks < 8 ? max_blocks : 8);
    int64_t units = 0, cost = 0;
    for (int i = 0; i < a.n_items; ++i) {
        GroupItem &I = a.item[i];
        const int64_t blocks = (I.N + rows_per_block - 1) / rows_per_block;
        I.unit0 = static_cast<int32_t>(units);
        I.units = static_cast<int32_t>((blocks + C - 1) / C);
        I.cost0 = cost;
        units += I.units;
        cost += static_cast<int64_t>(I.units) * I.nchunks;
    }
    if (units > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    a.units = static_cast<int>(units);
    a.cost_total = cost;
    if (ydt == LOWBIT_F32) return launch_group_out<FMT, MT, U, R, LOWBIT_F32>(a, C, smem, st);
    if (ydt == LOWBIT_BF16) return launch_group_out<FMT, MT, U, R, LOWBIT_BF16>(a, C, smem, st);
    return launch_group_out<FMT, MT, U, R, LOWBIT_I32>(a, C, smem, st);
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

// The same choice of U and R for a group, from its longest rows and its
// total rows (the persistent grid spreads the rows over the resident blocks).
template <int FMT, int MT>
lowbit_status launch_group_tokens(GroupArgs &a, int64_t max_nchunks, int64_t rows, lowbit_dtype ydt, size_t smem,
                                  cudaStream_t st)
{
    const int64_t slots = static_cast<int64_t>(device_sm_count()) * 2 * kWarps;
    if (max_nchunks <= 64) {
        if constexpr (MT == 1) {
            if (rows >= 4 * slots) return launch_group<FMT, MT, 2, 4>(a, ydt, smem, st);
        }
        if (rows >= 2 * slots) return launch_group<FMT, MT, 2, 2>(a, ydt, smem, st);
        return launch_group<FMT, MT, 2, 1>(a, ydt, smem, st);
    }
    if (max_nchunks <= 160) return launch_group<FMT, MT, 5, 1>(a, ydt, smem, st);
    return launch_group<FMT, MT, 8, 1>(a, ydt, smem, st);
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

// The grouped fused decode call (nchunks of every item set by the caller):
// the codes of all M tokens of the longest layer must fit the staging.
template <int FMT>
lowbit_status gemv_group_launch_fmt(GroupArgs &a, lowbit_dtype ydt, cudaStream_t st)
{
    int64_t max_nchunks = 0, rows = 0;
    for (int i = 0; i < a.n_items; ++i) {
        max_nchunks = a.item[i].nchunks > max_nchunks ? a.item[i].nchunks : max_nchunks;
        rows += a.item[i].N;
    }
    const int64_t smem = static_cast<int64_t>(a.M) * max_nchunks * QPieces<FMT>::value * 16;
    if (smem > kGemvSmemMax) return LOWBIT_ERR_INVALID_ARG;
    if (a.M == 1) return launch_group_tokens<FMT, 1>(a, max_nchunks, rows, ydt, static_cast<size_t>(smem), st);
    return launch_group_tokens<FMT, 4>(a, max_nchunks, rows, ydt, static_cast<size_t>(smem), st);
}

}  // namespace gemv_detail

}  // namespace lowbit
