// pack.cu -- weight quantisers and packers (offline, once per weight).
//
// Built with -fmad=false and written with explicit _rn intrinsics: every
// floating-point step is one IEEE operation in the stated order, so the codes
// and scales are reproducible bit for bit.
//
//   Ternary, "M8.8 - Native Binary and Ternary Transformers" 0x05A-0x05B:
//     gamma = mean|W| over the tensor.  The sum is fp64 in a fixed order (each
//     row k-ascending by one thread, then the row sums n-ascending by one
//     thread), rounded once to fp32; codes clip(rint(w/(gamma+eps)), -1, 1).
//   Binary, same page 0x06E (+1 if w >= 0, both zeros) with the per-row
//     mean-absolute scale of 0x02B.
//   4-bit, "T4NT-0.5B" model card: w_c = 3*tanh(w/3), per-row scale
//     max|w_c|/7, 15 levels.  tanh is evaluated here in fp64 by a fixed
//     sequence (see tanh_fixed) rather than by a library call, so the result
//     does not depend on a math library's last bit.
#include <mutex>

#include "lowbit_internal.cuh"

namespace lowbit {
namespace {

// ---------------------------------------------------------------------------
// tanh in fp64 by a fixed operation sequence.
//   tanh(a) = e / (e + 2) with e = expm1(2a) for a >= 0 (sign restored);
//   expm1(u) for u <= ln2/2: Taylor series u*(1 + u/2*(1 + u/3*(... u/16))),
//   else Cody-Waite: k = rint(u/ln2), r = (u - k*L_hi) - k*L_lo with ln 2
//   split into a 32-bit-mantissa head and a tail, expm1(u) = 2^k(1+expm1(r))-1;
//   a > 20 gives 1.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double expm1_taylor(double r)
{
    double p = 1.0;
#pragma unroll
    for (int n = 16; n >= 2; --n) p = __dadd_rn(1.0, __ddiv_rn(__dmul_rn(r, p), static_cast<double>(n)));
    return __dmul_rn(r, p);
}

__device__ double tanh_fixed(double z)
{
    const double kLn2Head = 0x1.62e42fee00000p-1;
    const double kLn2Tail = 0x1.a39ef35793c76p-33;
    const double kHalfLn2 = 0x1.62e42fefa39efp-2;
    if (z != z) return z;
    const double a = fabs(z);
    double t;
    if (a > 20.0) {
        t = 1.0;
    } else {
        const double u = __dmul_rn(2.0, a);
        double e;
        if (u <= kHalfLn2) {
            e = expm1_taylor(u);
        } else {
            const double k = rint(__ddiv_rn(u, __dadd_rn(kLn2Head, kLn2Tail)));
            const double r = __dsub_rn(__dsub_rn(u, __dmul_rn(k, kLn2Head)), __dmul_rn(k, kLn2Tail));
            const double p = expm1_taylor(r);
            e = __dsub_rn(scalbn(__dadd_rn(1.0, p), static_cast<int>(k)), 1.0);
        }
        t = __ddiv_rn(e, __dadd_rn(e, 2.0));
    }
    return z < 0 ? -t : t;
}

__device__ __forceinline__ float clip_tanh(float w)
{
    const double z = __ddiv_rn(static_cast<double>(w), 3.0);
    return __double2float_rn(__dmul_rn(3.0, tanh_fixed(z)));
}

// ---------------------------------------------------------------------------
// Per-row reductions: one thread per row, k ascending.
// ---------------------------------------------------------------------------
// mode 0: ternary, write the fp64 row sum of |w| to rows[n].
// mode 1: binary, write s_w[n] = fp32(sum / K).
// mode 2: 4-bit, write s_w[n] = max_k |clip_tanh(w)| / 7.
// mode 3: centred binary, write the fp64 row sums of w to rows[n] and of |w|
//         to rows[N + n].
__global__ void row_reduce(const float *__restrict__ w, int64_t N, int64_t K, int64_t ldw, int mode,
                           double *__restrict__ rows, float *__restrict__ s_w, int32_t *status)
{
    const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (n >= N) return;
    const float *wr = w + n * ldw;
    bool bad = false;
    if (mode == 2) {
        float m = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            const float v = wr[k];
            bad |= !finite_bits(__float_as_uint(v));
            m = fmaxf(m, fabsf(clip_tanh(v)));
        }
        s_w[n] = __fdiv_rn(m, 7.0f);
    } else if (mode == 3) {
        double r = 0.0, ra = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const float v = wr[k];
            bad |= !finite_bits(__float_as_uint(v));
            r = __dadd_rn(r, static_cast<double>(v));
            ra = __dadd_rn(ra, fabs(static_cast<double>(v)));
        }
        rows[n] = r;
        rows[N + n] = ra;
    } else {
        double r = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const float v = wr[k];
            bad |= !finite_bits(__float_as_uint(v));
            r = __dadd_rn(r, fabs(static_cast<double>(v)));
        }
        if (mode == 0) rows[n] = r;
        else s_w[n] = __double2float_rn(__ddiv_rn(r, static_cast<double>(K)));
    }
    if (bad) report(status, LOWBIT_ERR_NONFINITE);
}

// Ternary gamma: the row sums added in order n = 0..N-1.  One warp: the
// lanes load 32 consecutive row sums at a time and every lane adds them in
// order from shuffles (the same additions in the same order in every lane),
// so the loads are not serialised behind the additions.
__global__ void ternary_gamma(const double *__restrict__ rows, int64_t N, int64_t K, float *s_w)
{
    if (blockIdx.x != 0 || threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    double S = 0.0;
    for (int64_t n0 = 0; n0 < N; n0 += 32) {
        const double v = n0 + lane < N ? rows[n0 + lane] : 0.0;
        const int cnt = N - n0 < 32 ? static_cast<int>(N - n0) : 32;
        for (int i = 0; i < cnt; ++i) S = __dadd_rn(S, __shfl_sync(0xffffffffu, v, i));
    }
    if (lane == 0) s_w[0] = __double2float_rn(__ddiv_rn(S, static_cast<double>(N) * static_cast<double>(K)));
}

// Centred binary scalars: the row sums added in order n = 0..N-1 (one warp,
// as ternary_gamma); alpha = mean(W) and beta = mean|W|, each the fp64 mean
// rounded once to fp32, stored as two floats after the 2N row sums.
__global__ void centred_scalars(double *__restrict__ rows, int64_t N, int64_t K)
{
    if (blockIdx.x != 0 || threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    double S = 0.0, A = 0.0;
    for (int64_t n0 = 0; n0 < N; n0 += 32) {
        const bool in = n0 + lane < N;
        const double v = in ? rows[n0 + lane] : 0.0;
        const double a = in ? rows[N + n0 + lane] : 0.0;
        const int cnt = N - n0 < 32 ? static_cast<int>(N - n0) : 32;
        for (int i = 0; i < cnt; ++i) {
            S = __dadd_rn(S, __shfl_sync(0xffffffffu, v, i));
            A = __dadd_rn(A, __shfl_sync(0xffffffffu, a, i));
        }
    }
    __syncwarp();  // every lane has read its row sums before lane 0 writes after them
    if (lane == 0) {
        const double nk = static_cast<double>(N) * static_cast<double>(K);
        float *out = reinterpret_cast<float *>(rows + 2 * N);
        out[0] = __double2float_rn(__ddiv_rn(S, nk));
        out[1] = __double2float_rn(__ddiv_rn(A, nk));
    }
}

// BitNet v1 centred codes in the binary layout: bit 0 (+1) where w > alpha,
// bit 1 (-1) otherwise (a weight equal to the mean takes -1); the thread of
// word 0 of each row also writes that row's scale s_w[n] = beta.
__global__ void pack_centred_words(const float *__restrict__ w, int64_t N, int64_t K, int64_t ldw,
                                   const float *__restrict__ ab, uint8_t *__restrict__ packed, int64_t ldp,
                                   float *__restrict__ s_w)
{
    const int64_t words_per_row = ldp / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= N * words_per_row) return;
    const int64_t n = idx / words_per_row;
    const int64_t wi = idx % words_per_row;
    const float alpha = ab[0];
    const float *wr = w + n * ldw;
    uint32_t word = 0;
    const int64_t k0 = wi * 32;
    for (int kk = 0; kk < 32; ++kk) {
        const int64_t k = k0 + kk;
        if (k >= K) break;
        word |= (wr[k] > alpha ? 0u : 1u) << kk;
    }
    reinterpret_cast<uint32_t *>(packed + n * ldp)[wi] = word;
    if (wi == 0) s_w[n] = ab[1];
}

// ---------------------------------------------------------------------------
// Packing: one thread per 32-bit word of the output row (words past the row's
// logical extent are written zero).
// ---------------------------------------------------------------------------
template <int FMT>
__device__ __forceinline__ uint32_t code_field(float v, float scale_or_d)
{
    if constexpr (FMT == kT2) {
        if (scale_or_d == 0.0f) return 0u;
        float t = rintf(__fdiv_rn(v, scale_or_d));
        t = fminf(fmaxf(t, -1.0f), 1.0f);
        return static_cast<uint32_t>(static_cast<int>(t)) & 3u;
    } else if constexpr (FMT == kI4) {
        if (scale_or_d == 0.0f) return 0u;
        float t = rintf(__fdiv_rn(clip_tanh(v), scale_or_d));
        t = fminf(fmaxf(t, -7.0f), 7.0f);
        return static_cast<uint32_t>(static_cast<int>(t)) & 15u;
    } else {
        return v >= 0.0f ? 0u : 1u;
    }
}

template <int FMT>
__global__ void pack_words(const float *__restrict__ w, int64_t N, int64_t K, int64_t ldw, float eps,
                           const float *__restrict__ s_w, uint8_t *__restrict__ packed, int64_t ldp)
{
    using F = Fmt<FMT>;
    const int64_t words_per_row = ldp / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= N * words_per_row) return;
    const int64_t n = idx / words_per_row;
    const int64_t wi = idx % words_per_row;
    const float *wr = w + n * ldw;
    float s = 0.0f;
    if constexpr (FMT == kT2) s = __fadd_rn(s_w[0], eps);
    if constexpr (FMT == kI4) s = s_w[n];
    uint32_t word = 0;
    const int64_t k0 = wi * F::kCodesPerWord;
#pragma unroll 4
    for (int kk = 0; kk < F::kCodesPerWord; ++kk) {
        const int64_t k = k0 + kk;
        if (k >= K) break;
        const uint32_t f = code_field<FMT>(wr[k], s);
        int bit;
        if constexpr (FMT == kB1) bit = kk;
        else bit = 8 * (kk % 4) + F::kBits * (kk / 4);
        word |= f << bit;
    }
    reinterpret_cast<uint32_t *>(packed + n * ldp)[wi] = word;
}

// ---------------------------------------------------------------------------
// Unpacking with validation: one thread per 32-bit word.
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void unpack_words(const uint8_t *__restrict__ packed, int64_t ldp, int64_t N, int64_t K,
                             int8_t *__restrict__ codes, int64_t ldc, int32_t *status)
{
    using F = Fmt<FMT>;
    const int64_t words_per_row = ldp / 4;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= N * words_per_row) return;
    const int64_t n = idx / words_per_row;
    const int64_t wi = idx % words_per_row;
    const uint32_t word = reinterpret_cast<const uint32_t *>(packed + n * ldp)[wi];
    const int64_t k0 = wi * F::kCodesPerWord;
    uint32_t owned = 0;
    bool reserved = false;
    for (int kk = 0; kk < F::kCodesPerWord; ++kk) {
        const int64_t k = k0 + kk;
        if (k >= K) break;
        int bit;
        if constexpr (FMT == kB1) bit = kk;
        else bit = 8 * (kk % 4) + F::kBits * (kk / 4);
        const uint32_t mask = (1u << F::kBits) - 1u;
        const uint32_t f = (word >> bit) & mask;
        owned |= mask << bit;
        int c;
        if constexpr (FMT == kB1) {
            c = f ? -1 : 1;
        } else {
            constexpr uint32_t kTop = 1u << (F::kBits - 1);
            if (f == kTop) { reserved = true; c = 0; }
            else c = (f & kTop) ? static_cast<int>(f) - (1 << F::kBits) : static_cast<int>(f);
        }
        codes[n * ldc + k] = static_cast<int8_t>(c);
    }
    if (reserved || (word & ~owned) != 0u) report(status, LOWBIT_ERR_RESERVED_CODE);
}

unsigned blocks_for(int64_t n, int threads) { return static_cast<unsigned>((n + threads - 1) / threads); }

}  // namespace

lowbit_status pack_launch(const float *w, int64_t N, int64_t K, int64_t ldw, lowbit_format f, float eps,
                          uint8_t *packed, int64_t ldp, float *s_w, void *workspace,
                          int32_t *status, cudaStream_t st)
{
    const int64_t nwords = N * (ldp / 4);
    switch (f) {
    case LOWBIT_TERNARY2: {
        double *rows = static_cast<double *>(workspace);
        row_reduce<<<blocks_for(N, 128), 128, 0, st>>>(w, N, K, ldw, 0, rows, s_w, status);
        ternary_gamma<<<1, 32, 0, st>>>(rows, N, K, s_w);
        pack_words<kT2><<<blocks_for(nwords, 256), 256, 0, st>>>(w, N, K, ldw, eps, s_w, packed, ldp);
        break;
    }
    case LOWBIT_BINARY1:
        row_reduce<<<blocks_for(N, 128), 128, 0, st>>>(w, N, K, ldw, 1, nullptr, s_w, status);
        pack_words<kB1><<<blocks_for(nwords, 256), 256, 0, st>>>(w, N, K, ldw, eps, s_w, packed, ldp);
        break;
    default:
        row_reduce<<<blocks_for(N, 128), 128, 0, st>>>(w, N, K, ldw, 2, nullptr, s_w, status);
        pack_words<kI4><<<blocks_for(nwords, 256), 256, 0, st>>>(w, N, K, ldw, eps, s_w, packed, ldp);
        break;
    }
    return launch_status();
}

lowbit_status pack_centred_launch(const float *w, int64_t N, int64_t K, int64_t ldw, uint8_t *packed, int64_t ldp,
                                  float *s_w, void *workspace, int32_t *status, cudaStream_t st)
{
    double *rows = static_cast<double *>(workspace);
    const int64_t nwords = N * (ldp / 4);
    row_reduce<<<blocks_for(N, 128), 128, 0, st>>>(w, N, K, ldw, 3, rows, s_w, status);
    centred_scalars<<<1, 32, 0, st>>>(rows, N, K);
    pack_centred_words<<<blocks_for(nwords, 256), 256, 0, st>>>(w, N, K, ldw, reinterpret_cast<const float *>(rows + 2 * N),
                                                                 packed, ldp, s_w);
    return launch_status();
}

lowbit_status unpack_launch(const uint8_t *packed, int64_t ldp, int64_t N, int64_t K, lowbit_format f,
                            int8_t *codes, int64_t ldc, int32_t *status, cudaStream_t st)
{
    const int64_t nwords = N * (ldp / 4);
    const unsigned g = blocks_for(nwords, 256);
    if (f == LOWBIT_TERNARY2) unpack_words<kT2><<<g, 256, 0, st>>>(packed, ldp, N, K, codes, ldc, status);
    else if (f == LOWBIT_BINARY1) unpack_words<kB1><<<g, 256, 0, st>>>(packed, ldp, N, K, codes, ldc, status);
    else unpack_words<kI4><<<g, 256, 0, st>>>(packed, ldp, N, K, codes, ldc, status);
    return launch_status();
}

}  // namespace lowbit

// ---------------------------------------------------------------------------
// Ternary packing without a caller-provided workspace.
//
// Some callers cannot allocate device memory when they pack: runtimes that fix
// their device-memory budget at start-up and forbid allocation afterwards, and
// hosts whose device memory belongs to another allocator that a plain C caller
// cannot reach (a cudaFree would also synchronise the whole device, stalling
// their other streams).  For them the fixed-order row sums that the ternary
// scale needs live in a file-scope device array instead of a workspace.
// The array is at most kNoAllocMaxRows fp64 values (512 KB) and every GPU
// that loads the library keeps it until the process exits.
// ---------------------------------------------------------------------------
namespace lowbit {
namespace {

constexpr int64_t kNoAllocMaxRows = LOWBIT_NOALLOC_MAX_ROWS;
static __device__ __align__(256) double g_noalloc_row_sums[kNoAllocMaxRows];

// Device address of g_noalloc_row_sums, looked up once per device with that
// device current.  In host code the array's name is only a host-side stand-in,
// so the kernels must be given this address, never the name.
double *noalloc_scratch(int dev)
{
    static std::mutex mu;
    static double *addr[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_row_sums) != cudaSuccess || p == nullptr) return nullptr;
        addr[dev] = static_cast<double *>(p);
    }
    return addr[dev];
}

}  // namespace
}  // namespace lowbit

extern "C" lowbit_status lowbit_pack_ternary_noalloc(const float *w, int64_t N, int64_t K, int64_t ldw, float eps,
                                                     uint8_t *packed, int64_t ldp, float *s_w,
                                                     int32_t *status_dev, void *stream)
{
    using namespace lowbit;
    if (w == nullptr || packed == nullptr || s_w == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || ldw < K || !(eps >= 0.0f) || eps > 3.0e38f) return LOWBIT_ERR_INVALID_ARG;
    if (N > kNoAllocMaxRows || K > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    if (ldp < static_cast<int64_t>(4 * ((K + 15) / 16))) return LOWBIT_ERR_INVALID_ARG;
    if (ldp % 16 != 0 || (reinterpret_cast<uintptr_t>(packed) & 15u) != 0 ||
        (reinterpret_cast<uintptr_t>(w) & 3u) != 0 || (reinterpret_cast<uintptr_t>(s_w) & 3u) != 0)
        return LOWBIT_ERR_ALIGNMENT;
    // The device check reads a per-device cache filled on the first call.
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LOWBIT_ERR_CUDA;
    double *rows = noalloc_scratch(dev);
    if (rows == nullptr) return LOWBIT_ERR_CUDA;
    // Every row sum the call reads (rows 0..N-1) is written earlier in the
    // same call, so nothing left by a previous call is ever read and the
    // array needs no clearing.
    const TraceRange trace("lowbit_pack_ternary_noalloc");
    return pack_launch(w, N, K, ldw, LOWBIT_TERNARY2, eps, packed, ldp, s_w, rows, status_dev,
                       static_cast<cudaStream_t>(stream));
}
