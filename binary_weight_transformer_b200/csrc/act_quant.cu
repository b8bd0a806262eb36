// act_quant.cu -- per-token absmax int8 activation codes, with the optional
// activation prologue of a BitLinear layer in the same pass.
//
// "M8.8 - Native Binary and Ternary Transformers", section 0x05C (signed
// per-token A8: gamma_t = max|x_t|, reconstruction scale gamma_t/127, an
// all-zero row has zero codes and zero scale) and section 0x02C/0x02E (round
// to nearest, ties to even).  Per element: q = clip(rint((x*127) /
// (gamma_t + eps)), -128, 127) with one fp32 multiply and one IEEE fp32
// divide.
//
// Prologue options (the same page, 0x02E and 0x03: the activation is
// normalised before its codes are taken; 0x06A: OneBit's input value vector;
// 0x07C: H-BitLinear's online Hadamard transform):
//   gain g      u_k = RN32(x_k * g_k) replaces x_k;
//   RMSNorm     the row factor 1/sqrt(mean_k x_k^2 + eps_norm);
//   Hadamard    an unnormalised fp32 fast Walsh-Hadamard transform of every
//               block of hb consecutive features (radix 2, stages h = 1, 2,
//               4, ...), with the factor 1/sqrt(hb).
// Both row factors are positive, so they cancel in absmax codes: the codes
// are taken from u by the rule above (eps = 0) and the factors multiply only
// the scale, s_x = max|u| / sqrt(hb) / rms / 127, evaluated in fp64 (the
// sum of squares in fp64) and rounded once to fp32.
//
// One HBM pass: a group of TPR threads owns a row, loads it into registers
// with 16-byte non-allocating loads, reduces the row's absmax with warp
// shuffles (plus shared memory across warps when TPR > 32), then quantises
// from registers.  The max is taken on the fp32 bit pattern of |x|, which
// orders non-negative floats exactly and puts Inf/NaN above every finite
// value, so one test of gamma_t detects a non-finite row.
//
// Throughput is set by the bytes each SM has in flight while rows load, i.e.
// by resident threads x vectors per thread, and the registers that hold the
// vectors bound both.  Two builds of the kernel: "deep", up to five 16-byte
// vectors per thread at 1536 resident threads (40 registers), for grids of
// at least two full waves; "wide", up to three vectors at 2048 threads (32
// registers), which spreads a row over more threads when rows are few.
// Measured for bf16 rows on B200: 8192 x 9728 in 49 us deep, 58 us wide, 64 us
// with the compiler's own register choice; 1024 x 2560 in 4.1 us wide, 4.8 us
// deep.  The Hadamard rotation needs whole blocks of a row at once and runs
// in a separate kernel that stages the row in shared memory.
#include "quant_rule.cuh"

namespace lowbit {
namespace {

using namespace qrule;

// Max of a uint32 over the TPR threads that own one row.
template <int TPR>
__device__ __forceinline__ uint32_t row_max(uint32_t v, uint32_t *red)
{
#pragma unroll
    for (int o = (TPR < 32 ? TPR : 32) / 2; o > 0; o >>= 1)
        v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (TPR > 32) {
        constexpr int kWarps = TPR / 32;
        const int lane = threadIdx.x & 31;
        const int warp_in_row = (threadIdx.x % TPR) / 32;
        const int row_slot = threadIdx.x / TPR;
        if (lane == 0) red[row_slot * kWarps + warp_in_row] = v;
        __syncthreads();
        v = red[row_slot * kWarps];
#pragma unroll
        for (int i = 1; i < kWarps; ++i) v = max(v, red[row_slot * kWarps + i]);
    }
    return v;
}

// Sum of a double over the TPR threads that own one row (fixed tree order).
template <int TPR>
__device__ __forceinline__ double row_sum(double v, double *red)
{
#pragma unroll
    for (int o = (TPR < 32 ? TPR : 32) / 2; o > 0; o >>= 1)
        v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (TPR > 32) {
        constexpr int kWarps = TPR / 32;
        const int lane = threadIdx.x & 31;
        const int warp_in_row = (threadIdx.x % TPR) / 32;
        const int row_slot = threadIdx.x / TPR;
        if (lane == 0) red[row_slot * kWarps + warp_in_row] = v;
        __syncthreads();
        v = red[row_slot * kWarps];
#pragma unroll
        for (int i = 1; i < kWarps; ++i) v = __dadd_rn(v, red[row_slot * kWarps + i]);
    }
    return v;
}

__host__ __device__ constexpr int block_threads(int tpr) { return tpr > 256 ? tpr : 256; }

// The two builds: vectors per thread and resident threads per SM.
constexpr int kWideVPT = 3, kWideThreads = 2048;
constexpr int kDeepVPT = 5, kDeepThreads = 1536;

// Option bits of the register kernel.
constexpr int kOptGain = 1;
constexpr int kOptNorm = 2;

// Resident threads of a build.  With the gain, rows keep x g as fp32 between
// the passes (twice the registers of a 16-bit row), so both builds run 1024
// threads (64 registers).
template <typename T, int OPT>
__host__ __device__ constexpr int build_threads(bool deep)
{
    return (OPT & kOptGain) != 0 ? 1024 : (deep ? kDeepThreads : kWideThreads);
}

// Element i of a 16-byte vector of x, times the gain when GAIN.
template <typename T, bool GAIN>
__device__ __forceinline__ float elem(const uint4 &b, const float *gv, int i)
{
    const float v = In<T>::get(b, i);
    if constexpr (GAIN) return __fmul_rn(v, gv[i]);
    else return v;
}

// The E gains of vector v (E = 4 or 8 floats, one or two 16-byte loads,
// through L1: every row of the grid reads the same gains).
template <int E>
__device__ __forceinline__ void load_gain(const float *g, int64_t v, float (&gv)[8])
{
    const uint4 a = ld_act_ca_u4(g + v * E);
    gv[0] = __uint_as_float(a.x); gv[1] = __uint_as_float(a.y);
    gv[2] = __uint_as_float(a.z); gv[3] = __uint_as_float(a.w);
    if constexpr (E == 8) {
        const uint4 b = ld_act_ca_u4(g + v * E + 4);
        gv[4] = __uint_as_float(b.x); gv[5] = __uint_as_float(b.y);
        gv[6] = __uint_as_float(b.z); gv[7] = __uint_as_float(b.w);
    }
}

// s_x of a row from max|u| (nonzero): gamma/127 in fp32 with neither the
// norm nor the rotation (equal to the fp64 quotient rounded once), else
// gamma / sqrt(hb) / rms / 127 in fp64, rounded once to fp32.
__device__ __forceinline__ float row_scale(float gmax, bool norm, double ss, int64_t K, float eps_norm, int hb)
{
    if (!norm && hb <= 1) return __fdiv_rn(gmax, 127.0f);
    double s = static_cast<double>(gmax);
    if (hb > 1) s = __ddiv_rn(s, __dsqrt_rn(static_cast<double>(hb)));
    if (norm)
        s = __ddiv_rn(s, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(K)), static_cast<double>(eps_norm))));
    return __double2float_rn(__ddiv_rn(s, 127.0));
}

// Rows whose 16-byte vectors fit TPR*VPT registers: one global read.
// OPT = 0 is the plain per-token quantiser; kOptGain multiplies x by g
// (g 16-byte aligned), kOptNorm applies the RMSNorm factor to the scale
// (eps must be 0 with options).
template <typename T, int TPR, int VPT, int SM_THREADS, int OPT>
__global__ void __launch_bounds__(block_threads(TPR), SM_THREADS / block_threads(TPR))
act_quant_regs(const void *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
               int8_t *__restrict__ q, int64_t ldq, float *__restrict__ s_x, int32_t *status,
               const float *__restrict__ g, float eps_norm)
{
    constexpr bool GAIN = (OPT & kOptGain) != 0;
    constexpr bool NORM = (OPT & kOptNorm) != 0;
    constexpr int kThreads = block_threads(TPR);
    constexpr int kRows = kThreads / TPR;
    constexpr int E = In<T>::kPerVec;
    __shared__ uint32_t red[kThreads / 32];
    __shared__ double red_ss[NORM ? kThreads / 32 : 1];
    pdl_wait();
    pdl_trigger();

    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRows + threadIdx.x / TPR;
    const int r = threadIdx.x % TPR;
    const bool live = row < M;
    const int64_t nvec = K / E;
    const char *xrow = static_cast<const char *>(x) + (live ? row : 0) * ldx * sizeof(T);

    uint4 buf[VPT];
    // With the gain, u = x g is kept from the first pass for the second, so
    // the gains are read once (the L1 reads of the gains, twice per element,
    // bounded the kernel).
    float uf[GAIN ? VPT : 1][GAIN ? E : 1];
    uint32_t amax = 0;
    double ss = 0.0;
    float gv[8];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t v = r + static_cast<int64_t>(i) * TPR;
        if (live && v < nvec) {
            buf[i] = ld_act_u4(xrow + v * 16);
            if constexpr (GAIN || NORM) {
                if constexpr (GAIN) load_gain<E>(g, v, gv);
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float u = elem<T, GAIN>(buf[i], gv, e);
                    if constexpr (GAIN) uf[i][e] = u;
                    amax = max(amax, __float_as_uint(u) & 0x7fffffffu);
                    if constexpr (NORM) {
                        const double xd = static_cast<double>(In<T>::get(buf[i], e));
                        ss = __fma_rn(xd, xd, ss);
                    }
                }
            } else {
                amax = max(amax, In<T>::absmax_bits(buf[i]));
            }
        }
    }
    // Tail elements past the last whole vector, one per thread.
    const int64_t tail0 = nvec * E;
    float tail_x = 0.0f;
    const bool has_tail = live && (tail0 + r < K) && r < E;
    if (has_tail) {
        tail_x = In<T>::scalar(xrow, tail0 + r);
        if constexpr (NORM) ss = __fma_rn(static_cast<double>(tail_x), static_cast<double>(tail_x), ss);
        if constexpr (GAIN) tail_x = __fmul_rn(tail_x, g[tail0 + r]);
        amax = max(amax, __float_as_uint(tail_x) & 0x7fffffffu);
    }
    amax = row_max<TPR>(amax, red);
    if constexpr (NORM) ss = row_sum<TPR>(ss, red_ss);
    if (!live) return;

    const float gm = __uint_as_float(amax);
    const bool bad = !finite_bits(amax) || !finite_bits(__float_as_uint(__fmul_rn(gm, 127.0f)));
    if (bad && r == 0) report(status, LOWBIT_ERR_NONFINITE);
    const float d = __fadd_rn(gm, eps);
    const float c = __fmul_rn(127.0f, __frcp_rn(d));
    // Rows with max|x| below about 3.7e-37, or an eps near the fp32 maximum.
    const bool slow = !(d >= 0x1p-121f && d < 0x1p126f);
    int8_t *qrow = q + row * ldq;

#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t v = r + static_cast<int64_t>(i) * TPR;
        if (v < nvec) {
            const uint4 &b = buf[i];
            // u_e: element e of this vector (times its gain)
            auto ue = [&](int e) {
                if constexpr (GAIN) return uf[i][e];
                else return elem<T, false>(b, gv, e);
            };
            if constexpr (E == 4) {
                bool near = slow;
                const float u0 = ue(0), u1 = ue(1);
                const float u2 = ue(2), u3 = ue(3);
                uint32_t out = quant4(u0, u1, u2, u3, c, near);
                if (near) out = quant4_exact(u0, u1, u2, u3, d);
                if (amax == 0) out = 0;
                *reinterpret_cast<uint32_t *>(qrow + v * 4) = out;
            } else {
                bool near = slow;
                uint32_t lo = quant4(ue(0), ue(1), ue(2), ue(3), c, near);
                uint32_t hi = quant4(ue(4), ue(5), ue(6), ue(7), c, near);
                if (near) {
                    lo = quant4_exact(ue(0), ue(1), ue(2), ue(3), d);
                    hi = quant4_exact(ue(4), ue(5), ue(6), ue(7), d);
                }
                if (amax == 0) lo = hi = 0;
                *reinterpret_cast<uint2 *>(qrow + v * 8) = make_uint2(lo, hi);
            }
        }
    }
    if (has_tail) qrow[tail0 + r] = amax != 0 ? quant_one(tail_x, d) : 0;
    if (r == 0) {
        if constexpr (OPT == 0) s_x[row] = amax != 0 ? __fdiv_rn(gm, 127.0f) : 0.0f;
        else s_x[row] = amax != 0 ? row_scale(gm, NORM, ss, K, eps_norm, 0) : 0.0f;
    }
}

// Rows too long for registers, or rows without 16-byte alignment: a max
// pass, then a quantise pass (the second read mostly hits L2), with scalar
// loads.  One 256-thread block per row.
template <typename T>
__global__ void __launch_bounds__(256)
act_quant_long(const void *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
               int8_t *__restrict__ q, int64_t ldq, float *__restrict__ s_x, int32_t *status)
{
    __shared__ uint32_t red[8];
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const char *xrow = static_cast<const char *>(x) + row * ldx * sizeof(T);
    uint32_t amax = 0;
    for (int64_t k = threadIdx.x; k < K; k += 256)
        amax = max(amax, __float_as_uint(In<T>::scalar(xrow, k)) & 0x7fffffffu);
    amax = row_max<256>(amax, red);
    const float g = __uint_as_float(amax);
    const bool bad = !finite_bits(amax) || !finite_bits(__float_as_uint(__fmul_rn(g, 127.0f)));
    if (bad && threadIdx.x == 0) report(status, LOWBIT_ERR_NONFINITE);
    const float d = __fadd_rn(g, eps);
    int8_t *qrow = q + row * ldq;
    for (int64_t k = threadIdx.x; k < K; k += 256)
        qrow[k] = amax != 0 ? quant_one(In<T>::scalar(xrow, k), d) : 0;
    if (threadIdx.x == 0) s_x[row] = amax != 0 ? __fdiv_rn(g, 127.0f) : 0.0f;
}

// The prologue with the row staged in shared memory as fp32: gain, sum of
// squares, block Hadamard transform (one __syncthreads per stage), absmax,
// codes.  Any alignment; K * 4 bytes of dynamic shared memory.  One block of
// 256 threads per row.
constexpr int kStagedThreads = 256;

//
// Modes for a row split over ranks (the input dimension of a row-parallel
// layer), where the per-token statistics are reduced across ranks before the
// codes are taken: kStagedFull computes codes and scale from this slice
// alone; kStagedStats writes only the slice's max|u| (stat_max) and sum of
// squares (stat_ss, when not NULL); kStagedCodes takes the codes with the
// given row maximum stat_max[t] (the maximum over the whole row).
constexpr int kStagedFull = 0;
constexpr int kStagedStats = 1;
constexpr int kStagedCodes = 2;

template <typename T>
__global__ void __launch_bounds__(kStagedThreads)
act_prologue_staged(const void *__restrict__ x, int64_t M, int64_t K, int64_t ldx,
                    const float *__restrict__ g, int norm, float eps_norm, int hb,
                    int8_t *__restrict__ q, int64_t ldq, float *__restrict__ s_x, int32_t *status,
                    int mode = kStagedFull, float *__restrict__ stat_max = nullptr,
                    double *__restrict__ stat_ss = nullptr)
{
    extern __shared__ float su[];
    __shared__ uint32_t red[kStagedThreads / 32];
    __shared__ double red_ss[kStagedThreads / 32];
    pdl_wait();
    pdl_trigger();
    const int64_t row = blockIdx.x;
    const char *xrow = static_cast<const char *>(x) + row * ldx * sizeof(T);
    double ss = 0.0;
    for (int64_t k = threadIdx.x; k < K; k += kStagedThreads) {
        const float v = In<T>::scalar(xrow, k);
        if (norm) ss = __fma_rn(static_cast<double>(v), static_cast<double>(v), ss);
        su[k] = g != nullptr ? __fmul_rn(v, g[k]) : v;
    }
    // the block's sum of squares (fixed tree order)
    if (norm) {
        ss = row_sum<kStagedThreads>(ss, red_ss);
    }
    __syncthreads();
    if (hb > 1) {
        const int64_t half = K / 2;
        for (int h = 1; h < hb; h <<= 1) {
            for (int64_t p = threadIdx.x; p < half; p += kStagedThreads) {
                const int64_t j = (p / h) * 2 * h + (p % h);
                const float a = su[j], b = su[j + h];
                su[j] = __fadd_rn(a, b);
                su[j + h] = __fsub_rn(a, b);
            }
            __syncthreads();
        }
    }
    uint32_t amax = 0;
    for (int64_t k = threadIdx.x; k < K; k += kStagedThreads)
        amax = max(amax, __float_as_uint(su[k]) & 0x7fffffffu);
    amax = row_max<kStagedThreads>(amax, red);
    if (mode == kStagedStats) {
        if (!finite_bits(amax) && threadIdx.x == 0) report(status, LOWBIT_ERR_NONFINITE);
        if (threadIdx.x == 0) {
            stat_max[row] = __uint_as_float(amax);
            if (stat_ss != nullptr) stat_ss[row] = ss;
        }
        return;
    }
    if (mode == kStagedCodes) {
        // this slice's values may not exceed the row maximum it was given
        const uint32_t given = ld_act_u32(stat_max + row) & 0x7fffffffu;
        if (amax > given && threadIdx.x == 0) report(status, LOWBIT_ERR_INVALID_ARG);
        amax = given;
    }
    const float gm = __uint_as_float(amax);
    const bool bad = !finite_bits(amax) || !finite_bits(__float_as_uint(__fmul_rn(gm, 127.0f)));
    if (bad && threadIdx.x == 0) report(status, LOWBIT_ERR_NONFINITE);
    int8_t *qrow = q + row * ldq;
    for (int64_t k = threadIdx.x; k < K; k += kStagedThreads)
        qrow[k] = amax != 0 ? quant_one(su[k], gm) : 0;
    if (threadIdx.x == 0 && mode == kStagedFull)
        s_x[row] = amax != 0 ? row_scale(gm, norm != 0, ss, K, eps_norm, hb) : 0.0f;
}

// The Hadamard prologue in registers, for blocks of at most 512 features and
// rows of at most kFwhtMaxK features: one block per token row with one warp
// per 512-feature chunk (ceil(K / 512) warps); lane l holds features
// 16l..16l+15 of its warp's chunk.  Every hb-feature block lies inside one
// chunk (512 / hb is whole), so the stages h < 16 of its transform run
// within a lane; for the stages 16 <= h < hb the chunk is transposed through
// the warp's 2 KB of dynamic shared memory, leaving one stage across lanes.
// The staged kernel's fp32 additions and subtractions run in the same order:
// bit-identical values, with no barrier per stage.  Then the row maximum
// (and the sum of squares) over the block, the codes from registers (the
// fast rule of quant_rule.cuh) and the scale; `mode` as act_prologue_staged.
// One chunk per warp keeps the registers low (about 40 warps resident per SM
// at 4B-class rows; the earlier build with up to three chunks per warp of 8
// ran 24).
constexpr int kFwhtMaxWarps = 32;
constexpr int64_t kFwhtMaxK = static_cast<int64_t>(kFwhtMaxWarps) * 512;
// Rows of at most 20 chunks take a build bounded to two 640-thread blocks per
// SM (48 registers): 38 warps resident at K = 9728 instead of 19.
constexpr int kFwhtWarpsTwo = 20;
constexpr int kFwhtWarpFloats = 512 + 16;  // a chunk with one float of padding per 32

template <typename T, int MAXW>
__global__ void __launch_bounds__(MAXW * 32, MAXW <= kFwhtWarpsTwo ? 2 : 1)
act_prologue_fwht(const void *__restrict__ x, int64_t M, int64_t K, int64_t ldx, const float *__restrict__ g,
                  int norm, float eps_norm, int hb, int8_t *__restrict__ q, int64_t ldq, float *__restrict__ s_x,
                  int32_t *status, int mode, float *__restrict__ stat_max, double *__restrict__ stat_ss)
{
    __shared__ uint32_t red[kFwhtMaxWarps];
    __shared__ double red_ss[kFwhtMaxWarps];
    extern __shared__ float fwht_sm[];  // kFwhtWarpFloats per warp
    pdl_wait();
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nw = static_cast<int>(blockDim.x >> 5);
    const int64_t row = blockIdx.x;
    const char *xrow = static_cast<const char *>(x) + row * ldx * static_cast<int64_t>(sizeof(T));
    const bool xvec = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (ldx * static_cast<int64_t>(sizeof(T))) % 16 == 0;
    const bool gvec = g == nullptr || (reinterpret_cast<uintptr_t>(g) & 15u) == 0;
    float u[16];
    double ss = 0.0;
    uint32_t amax = 0;
    const int64_t chunk = warp;
    const int64_t k0 = (chunk * 32 + lane) * 16;
    {
        // the gains are requested before x, so their round trip overlaps
        // x's instead of following the first use of x
        const bool gv = g != nullptr && gvec && k0 + 16 <= K;
        uint4 gw[4];
        if (gv) {
#pragma unroll
            for (int v = 0; v < 4; ++v) gw[v] = ld_act_ca_u4(g + k0 + 4 * v);
        }
        if (xvec && k0 + 16 <= K) {
            if constexpr (sizeof(T) == 2) {
#pragma unroll
                for (int v = 0; v < 2; ++v) {
                    const uint4 w = ld_act_u4(xrow + 2 * (k0 + 8 * v));
#pragma unroll
                    for (int e = 0; e < 8; ++e) u[8 * v + e] = In<T>::get(w, e);
                }
            } else {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 w = ld_act_u4(xrow + 4 * (k0 + 4 * v));
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[4 * v + e] = In<T>::get(w, e);
                }
            }
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) u[e] = k0 + e < K ? In<T>::scalar(xrow, k0 + e) : 0.0f;
        }
        if (norm) {
#pragma unroll
            for (int e = 0; e < 16; ++e) ss = __fma_rn(static_cast<double>(u[e]), static_cast<double>(u[e]), ss);
        }
        if (g != nullptr) {
            if (gv) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const uint4 w = gw[v];
                    u[4 * v] = __fmul_rn(u[4 * v], __uint_as_float(w.x));
                    u[4 * v + 1] = __fmul_rn(u[4 * v + 1], __uint_as_float(w.y));
                    u[4 * v + 2] = __fmul_rn(u[4 * v + 2], __uint_as_float(w.z));
                    u[4 * v + 3] = __fmul_rn(u[4 * v + 3], __uint_as_float(w.w));
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (k0 + e < K) u[e] = __fmul_rn(u[e], ld_act_f32(g + k0 + e));
            }
        }
        // the transform of every hb-feature block: stages h < 16 in the lane
#pragma unroll
        for (int h = 1; h < 16; h <<= 1) {
            if (h >= hb) break;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                if (e & h) continue;
                const float a = u[e], b = u[e + h];
                u[e] = __fadd_rn(a, b);
                u[e + h] = __fsub_rn(a, b);
            }
        }
        // stages 16 <= h < hb: the chunk moves through shared memory so that
        // lane l holds features 32 j + l (j = 0..15).  Stage 16 then pairs
        // lane l with lane l ^ 16 (the lane with bit 16 clear holds a, its
        // partner b; (a, b) -> (a + b, a - b)), and stages 32.. pair t[j]
        // with t[j ^ h/32] inside the lane; the chunk moves back for the
        // codes.  Feature f is stored at f + f / 32 (one float of padding per
        // 32): the row-wise writes (16 l + e) and the column-wise reads
        // (32 j + l) are both free of bank conflicts, and both address a
        // per-lane base plus a constant.
        if (hb > 16) {
            float *sw = fwht_sm + warp * kFwhtWarpFloats;
            float *wr = sw + 16 * lane + (lane >> 1);  // feature 16 lane + e at wr[e]
            float *rd = sw + lane;                     // feature 32 j + lane at rd[33 j]
            __syncwarp();  // the previous chunk's reads are done
#pragma unroll
            for (int e = 0; e < 16; ++e) wr[e] = u[e];
            __syncwarp();
            float t[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) t[j] = rd[33 * j];
            // a + b in the lower lane, a - b = b * -1 + a in the upper one: one
            // fused multiply-add by +-1 is exact before its single rounding
            const float sgn = (lane & 16) != 0 ? -1.0f : 1.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float other = __shfl_xor_sync(0xffffffffu, t[j], 16);
                t[j] = __fmaf_rn(sgn, t[j], other);
            }
#pragma unroll
            for (int h = 32; h < 512; h <<= 1) {
                if (h >= hb) break;
                const int jm = h >> 5;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    if (j & jm) continue;
                    const float a = t[j], b = t[j + jm];
                    t[j] = __fadd_rn(a, b);
                    t[j + jm] = __fsub_rn(a, b);
                }
            }
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 16; ++j) rd[33 * j] = t[j];
            __syncwarp();
#pragma unroll
            for (int e = 0; e < 16; ++e) u[e] = wr[e];
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) amax = max(amax, __float_as_uint(u[e]) & 0x7fffffffu);
    }
    // the row's maximum and sum of squares over the block (fixed tree order)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (norm) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    }
    if (lane == 0) {
        red[warp] = amax;
        red_ss[warp] = ss;
    }
    __syncthreads();
    // every warp reduces the warps' partials with the same shuffle tree (lane
    // w holds warp w's), so all threads get the same maximum and sum
    amax = lane < nw ? red[lane] : 0u;
    ss = lane < nw ? red_ss[lane] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (norm) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    }
    if (mode == kStagedStats) {
        if (threadIdx.x == 0) {
            if (!finite_bits(amax)) report(status, LOWBIT_ERR_NONFINITE);
            stat_max[row] = __uint_as_float(amax);
            if (stat_ss != nullptr) stat_ss[row] = ss;
        }
        return;
    }
    if (mode == kStagedCodes) {
        // this slice's values may not exceed the row maximum it was given
        const uint32_t given = ld_act_u32(stat_max + row) & 0x7fffffffu;
        if (amax > given && threadIdx.x == 0) report(status, LOWBIT_ERR_INVALID_ARG);
        amax = given;
    }
    const float gm = __uint_as_float(amax);
    const bool bad = !finite_bits(amax) || !finite_bits(__float_as_uint(__fmul_rn(gm, 127.0f)));
    if (bad && threadIdx.x == 0) report(status, LOWBIT_ERR_NONFINITE);
    const float c127 = __fmul_rn(127.0f, __frcp_rn(gm));
    const bool slow = !(gm >= 0x1p-121f && gm < 0x1p126f);
    int8_t *qrow = q + row * ldq;
    if (k0 < K) {
        uint32_t wq[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            bool near = slow;
            wq[e] = quant4(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3], c127, near);
            if (near) wq[e] = quant4_exact(u[4 * e], u[4 * e + 1], u[4 * e + 2], u[4 * e + 3], gm);
            if (amax == 0) wq[e] = 0;
        }
        if (k0 + 16 <= K) {
            *reinterpret_cast<uint4 *>(qrow + k0) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
        } else {
            const uint8_t *bytes = reinterpret_cast<const uint8_t *>(wq);
            for (int64_t e = 0; k0 + e < K; ++e) qrow[k0 + e] = static_cast<int8_t>(bytes[e]);
        }
    }
    if (threadIdx.x == 0 && mode == kStagedFull)
        s_x[row] = amax != 0 ? row_scale(gm, norm != 0, ss, K, eps_norm, hb) : 0.0f;
}

// s_x of rows whose statistics were reduced over a split row: max|u| over
// the whole row, the sum of squares over the whole row (norm), K_total
// features.
__global__ void row_scales_from_stats(const float *__restrict__ row_max, const double *__restrict__ row_ss, int64_t M,
                                      int64_t K_total, int norm, float eps_norm, int hb, float *__restrict__ s_x,
                                      int32_t *status)
{
    pdl_wait();
    pdl_trigger();
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= M) return;
    const float gm = ld_act_f32(row_max + t);
    const uint32_t bits = __float_as_uint(gm) & 0x7fffffffu;
    if (!finite_bits(bits) || !finite_bits(__float_as_uint(__fmul_rn(gm, 127.0f)))) report(status, LOWBIT_ERR_NONFINITE);
    s_x[t] = bits != 0 ? row_scale(__uint_as_float(bits), norm != 0, norm ? ld_act_f64(row_ss + t) : 0.0, K_total, eps_norm, hb)
                       : 0.0f;
}

// Largest row the staged prologue kernel holds in shared memory.
constexpr int64_t kMaxStagedK = 48 * 1024;

template <typename T>
lowbit_status launch_staged(const void *x, int64_t M, int64_t K, int64_t ldx, const float *g, int norm,
                            float eps_norm, int hb, int8_t *q, int64_t ldq, float *s_x, int32_t *status,
                            cudaStream_t st, int mode = kStagedFull, float *row_max = nullptr,
                            double *row_ss = nullptr)
{
    // blocks of at most 512 features in rows of at most kFwhtMaxK: registers
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (hb >= 2 && hb <= 512 && K <= kFwhtMaxK) {
        const int warps = static_cast<int>((K + 511) / 512);
        if (warps <= kFwhtWarpsTwo)
            return launch_pdl(act_prologue_fwht<T, kFwhtWarpsTwo>, dim3(static_cast<unsigned>(M)), dim3(32 * warps),
                              static_cast<size_t>(warps) * kFwhtWarpFloats * 4, st, 0, x, M, K, ldx, g, norm, eps_norm, hb, q,
                              ldq, s_x, status, mode, row_max, row_ss);
        static PerDevice fwht_configured;  // up to 64 KB of dynamic shared memory
        if (fwht_configured.get(dev, [&] {
                return cudaFuncSetAttribute(act_prologue_fwht<T, kFwhtMaxWarps>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kFwhtMaxWarps * kFwhtWarpFloats * 4) == cudaSuccess ? 1 : 0;
            }) <= 0)
            return LOWBIT_ERR_CUDA;
        return launch_pdl(act_prologue_fwht<T, kFwhtMaxWarps>, dim3(static_cast<unsigned>(M)), dim3(32 * warps),
                          static_cast<size_t>(warps) * kFwhtWarpFloats * 4, st, 0, x, M, K, ldx, g, norm, eps_norm, hb, q, ldq,
                          s_x, status, mode, row_max, row_ss);
    }
    static PerDevice configured;  // the shared-memory limit is raised once per device
    if (configured.get(dev, [&] {
            return cudaFuncSetAttribute(act_prologue_staged<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kMaxStagedK * 4)) == cudaSuccess ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    return launch_pdl(act_prologue_staged<T>, dim3(static_cast<unsigned>(M)), dim3(kStagedThreads),
                      static_cast<size_t>(K) * 4, st, 0, x, M, K, ldx, g, norm, eps_norm, hb, q, ldq, s_x, status,
                      mode, row_max, row_ss);
}

template <typename T>
lowbit_status launch(const void *x, int64_t M, int64_t K, int64_t ldx, float eps, int8_t *q,
                     int64_t ldq, float *s_x, int32_t *status, cudaStream_t st, const float *g, int opt,
                     float eps_norm)
{
    constexpr int E = In<T>::kPerVec;
    const int64_t nvec = K / E;
    // 16-byte vector loads need a 16-byte aligned base and row stride (and a
    // 16-byte aligned gain); any other layout takes a scalar-load kernel.
    const bool vec_ok = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 &&
                        (ldx * static_cast<int64_t>(sizeof(T))) % 16 == 0 &&
                        (g == nullptr || (reinterpret_cast<uintptr_t>(g) & 15u) == 0);
    auto staged = [&]() {
        return launch_staged<T>(x, M, K, ldx, g, (opt & kOptNorm) ? 1 : 0, eps_norm, 0, q, ldq, s_x, status, st);
    };
    if (!vec_ok) {
        if (opt != 0) return staged();
        return launch_pdl(act_quant_long<T>, dim3(static_cast<unsigned>(M)), dim3(256), 0, st, 0, x, M, K, ldx, eps,
                          q, ldq, s_x, status);
    }
    // Smallest thread group per row whose registers hold the row.
    auto group_for = [&](int vpt) {
        for (int tpr : {8, 32, 64, 128, 256, 512, 1024})
            if (nvec <= static_cast<int64_t>(tpr) * vpt) return tpr;
        return 0;
    };
    // Deep when the wide build cannot hold the row, or when it halves the
    // group (more vectors per thread) and the grid still fills two waves.
    const int tpr_wide = group_for(kWideVPT), tpr_deep = group_for(kDeepVPT);
    const bool deep = tpr_deep != 0 &&
                      (tpr_wide == 0 || (tpr_deep < tpr_wide &&
                                         M * tpr_deep >= 2 * static_cast<int64_t>(device_sm_count()) * kDeepThreads));
    const int tpr = deep ? tpr_deep : tpr_wide;
    if (tpr == 0) {  // longer than either register build holds
        if (opt != 0) return staged();
        return launch_pdl(act_quant_long<T>, dim3(static_cast<unsigned>(M)), dim3(256), 0, st, 0, x, M, K, ldx, eps,
                          q, ldq, s_x, status);
    }
    const int rows_per_block = block_threads(tpr) / tpr;
    const unsigned grid = static_cast<unsigned>((M + rows_per_block - 1) / rows_per_block);
#define LOWBIT_AQ_OPT(TPR, OPT)                                                                                  \
    if (opt == OPT) {                                                                                            \
        if (deep)                                                                                                \
            return launch_pdl(act_quant_regs<T, TPR, kDeepVPT, build_threads<T, OPT>(true), OPT>, dim3(grid),    \
                              dim3(block_threads(TPR)), 0, st, 0, x, M, K, ldx, eps, q, ldq, s_x, status, g,     \
                              eps_norm);                                                                         \
        return launch_pdl(act_quant_regs<T, TPR, kWideVPT, build_threads<T, OPT>(false), OPT>, dim3(grid),       \
                          dim3(block_threads(TPR)), 0, st, 0, x, M, K, ldx, eps, q, ldq, s_x, status, g, eps_norm); \
    }
#define LOWBIT_AQ(TPR)                                                                                           \
    if (tpr == TPR) {                                                                                            \
        LOWBIT_AQ_OPT(TPR, 0)                                                                                    \
        LOWBIT_AQ_OPT(TPR, kOptGain)                                                                             \
        LOWBIT_AQ_OPT(TPR, kOptNorm)                                                                             \
        LOWBIT_AQ_OPT(TPR, kOptGain | kOptNorm)                                                                  \
    }
    LOWBIT_AQ(8)
    LOWBIT_AQ(32)
    LOWBIT_AQ(64)
    LOWBIT_AQ(128)
    LOWBIT_AQ(256)
    LOWBIT_AQ(512)
    LOWBIT_AQ(1024)
#undef LOWBIT_AQ
#undef LOWBIT_AQ_OPT
    return LOWBIT_ERR_INVALID_ARG;
}

}  // namespace

lowbit_status act_quant_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                               float eps, int8_t *q, int64_t ldq, float *s_x, int32_t *status,
                               cudaStream_t st)
{
    if (xdt == LOWBIT_F32) return launch<float>(x, M, K, ldx, eps, q, ldq, s_x, status, st, nullptr, 0, 0.0f);
    return launch<__nv_bfloat16>(x, M, K, ldx, eps, q, ldq, s_x, status, st, nullptr, 0, 0.0f);
}

int64_t act_prologue_max_staged_k() { return kMaxStagedK; }

lowbit_status act_prologue_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                  const float *g, int norm, float eps_norm, int hb, int8_t *q, int64_t ldq,
                                  float *s_x, int32_t *status, cudaStream_t st)
{
    if (hb > 1) {
        if (xdt == LOWBIT_F32)
            return launch_staged<float>(x, M, K, ldx, g, norm, eps_norm, hb, q, ldq, s_x, status, st);
        return launch_staged<__nv_bfloat16>(x, M, K, ldx, g, norm, eps_norm, hb, q, ldq, s_x, status, st);
    }
    const int opt = (g != nullptr ? kOptGain : 0) | (norm ? kOptNorm : 0);
    if (xdt == LOWBIT_F32) return launch<float>(x, M, K, ldx, 0.0f, q, ldq, s_x, status, st, g, opt, eps_norm);
    return launch<__nv_bfloat16>(x, M, K, ldx, 0.0f, q, ldq, s_x, status, st, g, opt, eps_norm);
}

// Per-token statistics of a row slice (split-row mode): max|u| after the
// gain and rotation, and the fp64 sum of squares of x when row_ss is given.
lowbit_status act_row_stats_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                   const float *g, int hb, float *row_max, double *row_ss, int32_t *status,
                                   cudaStream_t st)
{
    const int norm = row_ss != nullptr ? 1 : 0;
    if (xdt == LOWBIT_F32)
        return launch_staged<float>(x, M, K, ldx, g, norm, 0.0f, hb, nullptr, 0, nullptr, status, st, kStagedStats,
                                    row_max, row_ss);
    return launch_staged<__nv_bfloat16>(x, M, K, ldx, g, norm, 0.0f, hb, nullptr, 0, nullptr, status, st,
                                        kStagedStats, row_max, row_ss);
}

// Codes of a row slice with the given whole-row maximum (split-row mode).
lowbit_status act_codes_given_max_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                         const float *g, int hb, const float *row_max, int8_t *q, int64_t ldq,
                                         int32_t *status, cudaStream_t st)
{
    float *rm = const_cast<float *>(row_max);  // read only in this mode
    if (xdt == LOWBIT_F32)
        return launch_staged<float>(x, M, K, ldx, g, 0, 0.0f, hb, q, ldq, nullptr, status, st, kStagedCodes, rm,
                                    nullptr);
    return launch_staged<__nv_bfloat16>(x, M, K, ldx, g, 0, 0.0f, hb, q, ldq, nullptr, status, st, kStagedCodes, rm,
                                        nullptr);
}

lowbit_status act_scales_launch(const float *row_max, const double *row_ss, int64_t M, int64_t K_total, int norm,
                                float eps_norm, int hb, float *s_x, int32_t *status, cudaStream_t st)
{
    return launch_pdl(row_scales_from_stats, dim3(static_cast<unsigned>((M + 255) / 256)), dim3(256), 0, st, 0,
                      row_max, row_ss, M, K_total, norm, eps_norm, hb, s_x, status);
}

}  // namespace lowbit
