// act_quant.cu -- per-token absmax int8 activation codes.
//
// "M8.8 - Native Binary and Ternary Transformers", section 0x05C (signed
// per-token A8: gamma_t = max|x_t|, reconstruction scale gamma_t/127, an
// all-zero row has zero codes and zero scale) and section 0x02C/0x02E (round
// to nearest, ties to even).  Per element: q = clip(rint((x*127) /
// (gamma_t + eps)), -128, 127) with one fp32 multiply and one IEEE fp32
// divide.
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
// deep.
#include "lowbit_internal.cuh"

namespace lowbit {
namespace {

template <typename T> struct In;
template <> struct In<float> {
    static constexpr int kPerVec = 4;
    __device__ static float get(const uint4 &v, int i) { return __uint_as_float((&v.x)[i]); }
    __device__ static float scalar(const void *p, int64_t i) { return static_cast<const float *>(p)[i]; }
    // max of |x| bits over one vector (a non-finite value sorts above all finite ones)
    __device__ static uint32_t absmax_bits(const uint4 &v)
    {
        return max(max(v.x & 0x7fffffffu, v.y & 0x7fffffffu), max(v.z & 0x7fffffffu, v.w & 0x7fffffffu));
    }
};
template <> struct In<__nv_bfloat16> {
    static constexpr int kPerVec = 8;
    __device__ static float get(const uint4 &v, int i)
    {
        const uint32_t w = (&v.x)[i >> 1];
        return __uint_as_float((i & 1) ? (w & 0xffff0000u) : (w << 16));
    }
    __device__ static float scalar(const void *p, int64_t i)
    {
        const uint16_t h = static_cast<const uint16_t *>(p)[i];
        return __uint_as_float(static_cast<uint32_t>(h) << 16);
    }
    // 16-bit lane-wise max of the |x| bit patterns, then the larger half
    __device__ static uint32_t absmax_bits(const uint4 &v)
    {
        const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                                    __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
        return max(m << 16, m & 0xffff0000u);
    }
};

__device__ __forceinline__ int8_t quant_one(float x, float d)
{
    float t = rintf(__fdiv_rn(__fmul_rn(x, 127.0f), d));
    t = fminf(fmaxf(t, -128.0f), 127.0f);
    return static_cast<int8_t>(static_cast<int>(t));
}

// Codes for four values without a divide or a conversion instruction each.
// The exact code is rint(z), z = RN(t/d), t = RN(127x).  With c = RN(127 *
// RN(1/d)) and u = RN(x*c), |u - t/d| <= (127|x|/d) * 4 * 2^-24 < 3.1e-5 and
// |z - t/d| <= 2^-18 < 3.9e-6 (|z| < 128), so |u - z| < 3.5e-5: u and z round
// to the same integer unless u lies within that distance of a midpoint
// k + 1/2.  Rounding uses the IEEE nearest-even addition v = u + 1.5*2^23,
// exact to the unit for |u| < 2^22: v - 1.5*2^23 is rint(u) and the low byte
// of v's bit pattern is the code in two's complement.  A value within 1e-4
// of a midpoint (about 2 in 10^4) sets `near`; the caller then redoes the
// four values with the IEEE divide.  |u| <= 127.0001, so no clamp is needed.
// The relative bounds need RN(1/d) and c normal and finite, i.e. d in
// [2^-121, 2^126); outside it the caller takes the divide for every value.
__device__ __forceinline__ uint32_t quant4(float x0, float x1, float x2, float x3, float c, bool &near)
{
    constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
    const float u0 = __fmul_rn(x0, c), u1 = __fmul_rn(x1, c), u2 = __fmul_rn(x2, c), u3 = __fmul_rn(x3, c);
    const float v0 = __fadd_rn(u0, kMagic), v1 = __fadd_rn(u1, kMagic);
    const float v2 = __fadd_rn(u2, kMagic), v3 = __fadd_rn(u3, kMagic);
    near |= fabsf(__fsub_rn(u0, __fsub_rn(v0, kMagic))) > 0.4999f;
    near |= fabsf(__fsub_rn(u1, __fsub_rn(v1, kMagic))) > 0.4999f;
    near |= fabsf(__fsub_rn(u2, __fsub_rn(v2, kMagic))) > 0.4999f;
    near |= fabsf(__fsub_rn(u3, __fsub_rn(v3, kMagic))) > 0.4999f;
    const uint32_t lo = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x0040);
    const uint32_t hi = __byte_perm(__float_as_uint(v2), __float_as_uint(v3), 0x0040);
    return __byte_perm(lo, hi, 0x5410);
}

__device__ __forceinline__ uint32_t quant4_exact(float x0, float x1, float x2, float x3, float d)
{
    return static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x0, d))) |
           (static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x1, d))) << 8) |
           (static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x2, d))) << 16) |
           (static_cast<uint32_t>(static_cast<uint8_t>(quant_one(x3, d))) << 24);
}

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

__host__ __device__ constexpr int block_threads(int tpr) { return tpr > 256 ? tpr : 256; }

// The two builds: vectors per thread and resident threads per SM.
constexpr int kWideVPT = 3, kWideThreads = 2048;
constexpr int kDeepVPT = 5, kDeepThreads = 1536;

// Rows whose 16-byte vectors fit TPR*VPT registers: one global read.
template <typename T, int TPR, int VPT, int SM_THREADS>
__global__ void __launch_bounds__(block_threads(TPR), SM_THREADS / block_threads(TPR))
act_quant_regs(const void *__restrict__ x, int64_t M, int64_t K, int64_t ldx, float eps,
               int8_t *__restrict__ q, int64_t ldq, float *__restrict__ s_x, int32_t *status)
{
    constexpr int kThreads = block_threads(TPR);
    constexpr int kRows = kThreads / TPR;
    constexpr int E = In<T>::kPerVec;
    __shared__ uint32_t red[kThreads / 32];
    pdl_wait();
    pdl_trigger();

    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRows + threadIdx.x / TPR;
    const int r = threadIdx.x % TPR;
    const bool live = row < M;
    const int64_t nvec = K / E;
    const char *xrow = static_cast<const char *>(x) + (live ? row : 0) * ldx * sizeof(T);

    uint4 buf[VPT];
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t v = r + static_cast<int64_t>(i) * TPR;
        if (live && v < nvec) {
            buf[i] = ld_stream_u4(xrow + v * 16);
            amax = max(amax, In<T>::absmax_bits(buf[i]));
        }
    }
    // Tail elements past the last whole vector, one per thread.
    const int64_t tail0 = nvec * E;
    float tail_x = 0.0f;
    const bool has_tail = live && (tail0 + r < K) && r < E;
    if (has_tail) {
        tail_x = In<T>::scalar(xrow, tail0 + r);
        amax = max(amax, __float_as_uint(tail_x) & 0x7fffffffu);
    }
    amax = row_max<TPR>(amax, red);
    if (!live) return;

    const float g = __uint_as_float(amax);
    const bool bad = !finite_bits(amax) || !finite_bits(__float_as_uint(__fmul_rn(g, 127.0f)));
    if (bad && r == 0) report(status, LOWBIT_ERR_NONFINITE);
    const float d = __fadd_rn(g, eps);
    const float c = __fmul_rn(127.0f, __frcp_rn(d));
    // Rows with max|x| below about 3.7e-37, or an eps near the fp32 maximum.
    const bool slow = !(d >= 0x1p-121f && d < 0x1p126f);
    int8_t *qrow = q + row * ldq;

#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int64_t v = r + static_cast<int64_t>(i) * TPR;
        if (v < nvec) {
            const uint4 &b = buf[i];
            if constexpr (E == 4) {
                bool near = slow;
                uint32_t out = quant4(In<T>::get(b, 0), In<T>::get(b, 1), In<T>::get(b, 2), In<T>::get(b, 3), c, near);
                if (near) out = quant4_exact(In<T>::get(b, 0), In<T>::get(b, 1), In<T>::get(b, 2), In<T>::get(b, 3), d);
                if (amax == 0) out = 0;
                *reinterpret_cast<uint32_t *>(qrow + v * 4) = out;
            } else {
                bool near = slow;
                uint32_t lo = quant4(In<T>::get(b, 0), In<T>::get(b, 1), In<T>::get(b, 2), In<T>::get(b, 3), c, near);
                uint32_t hi = quant4(In<T>::get(b, 4), In<T>::get(b, 5), In<T>::get(b, 6), In<T>::get(b, 7), c, near);
                if (near) {
                    lo = quant4_exact(In<T>::get(b, 0), In<T>::get(b, 1), In<T>::get(b, 2), In<T>::get(b, 3), d);
                    hi = quant4_exact(In<T>::get(b, 4), In<T>::get(b, 5), In<T>::get(b, 6), In<T>::get(b, 7), d);
                }
                if (amax == 0) lo = hi = 0;
                *reinterpret_cast<uint2 *>(qrow + v * 8) = make_uint2(lo, hi);
            }
        }
    }
    if (has_tail) qrow[tail0 + r] = amax != 0 ? quant_one(tail_x, d) : 0;
    if (r == 0) s_x[row] = amax != 0 ? __fdiv_rn(g, 127.0f) : 0.0f;
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

template <typename T>
lowbit_status launch(const void *x, int64_t M, int64_t K, int64_t ldx, float eps, int8_t *q,
                     int64_t ldq, float *s_x, int32_t *status, cudaStream_t st)
{
    constexpr int E = In<T>::kPerVec;
    const int64_t nvec = K / E;
    // 16-byte vector loads need a 16-byte aligned base and row stride; any
    // other layout takes the scalar-load kernel.
    const bool vec_ok = (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (ldx * static_cast<int64_t>(sizeof(T))) % 16 == 0;
    if (!vec_ok) {
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
    if (tpr == 0)  // longer than either register build holds
        return launch_pdl(act_quant_long<T>, dim3(static_cast<unsigned>(M)), dim3(256), 0, st, 0, x, M, K, ldx, eps,
                          q, ldq, s_x, status);
    const int rows_per_block = block_threads(tpr) / tpr;
    const unsigned grid = static_cast<unsigned>((M + rows_per_block - 1) / rows_per_block);
#define LOWBIT_AQ(TPR)                                                                                          \
    if (tpr == TPR) {                                                                                           \
        if (deep)                                                                                               \
            return launch_pdl(act_quant_regs<T, TPR, kDeepVPT, kDeepThreads>, dim3(grid), dim3(block_threads(TPR)), \
                              0, st, 0, x, M, K, ldx, eps, q, ldq, s_x, status);                                \
        return launch_pdl(act_quant_regs<T, TPR, kWideVPT, kWideThreads>, dim3(grid), dim3(block_threads(TPR)),    \
                          0, st, 0, x, M, K, ldx, eps, q, ldq, s_x, status);                                    \
    }
    LOWBIT_AQ(8)
    LOWBIT_AQ(32)
    LOWBIT_AQ(64)
    LOWBIT_AQ(128)
    LOWBIT_AQ(256)
    LOWBIT_AQ(512)
    LOWBIT_AQ(1024)
#undef LOWBIT_AQ
    return launch_pdl(act_quant_long<T>, dim3(static_cast<unsigned>(M)), dim3(256), 0, st, 0, x, M, K, ldx, eps, q,
                      ldq, s_x, status);
}

}  // namespace

lowbit_status act_quant_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                               float eps, int8_t *q, int64_t ldq, float *s_x, int32_t *status,
                               cudaStream_t st)
{
    if (xdt == LOWBIT_F32) return launch<float>(x, M, K, ldx, eps, q, ldq, s_x, status, st);
    return launch<__nv_bfloat16>(x, M, K, ldx, eps, q, ldq, s_x, status, st);
}

}  // namespace lowbit
