// abi.cu -- the C ABI: argument checks on the host, then kernel dispatch.
//
// Every check here runs before any launch, so a rejected call launches
// nothing.  The operator definitions are stated in include/lowbit.h.
#include <climits>
#include <cstdio>

#include "lowbit_internal.cuh"

namespace lowbit {

lowbit_status act_quant_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx, float eps,
                               int8_t *q, int64_t ldq, float *s_x, int32_t *status, cudaStream_t st);
lowbit_status pack_launch(const float *w, int64_t N, int64_t K, int64_t ldw, lowbit_format f, float eps,
                          uint8_t *packed, int64_t ldp, float *s_w, void *workspace, int32_t *status,
                          cudaStream_t st);
lowbit_status pack_centred_launch(const float *w, int64_t N, int64_t K, int64_t ldw, uint8_t *packed, int64_t ldp,
                                  float *s_w, void *workspace, int32_t *status, cudaStream_t st);
lowbit_status unpack_launch(const uint8_t *packed, int64_t ldp, int64_t N, int64_t K, lowbit_format f,
                            int8_t *codes, int64_t ldc, int32_t *status, cudaStream_t st);
lowbit_status gemv_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                          const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                          lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                          cudaStream_t st);
lowbit_status gemm_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                          const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                          lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                          int32_t *status, cudaStream_t st);

// True when the shared-memory GEMM would split K over a cluster on a GPU
// with `sms` SMs (few output tiles, deep K).
bool gemm_splits_k(lowbit_format f, int64_t M, int64_t N, int64_t K, int64_t sms);

lowbit_status gemm_ts_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                             const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                             lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                             int32_t *status, cudaStream_t st);

lowbit_status skinny_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                            const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                            lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                            int32_t *status, cudaStream_t st);

lowbit_status gemm_pair_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                               const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                               lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                               int exclusive, int32_t *status, cudaStream_t st);

lowbit_status gemm_ts_pair_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                                  const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                                  lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy,
                                  int32_t *status, cudaStream_t st);

lowbit_status act_prologue_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                  const float *g, int norm, float eps_norm, int hb, int8_t *q, int64_t ldq,
                                  float *s_x, int32_t *status, cudaStream_t st);
lowbit_status gemv_group_launch(const lowbit_bitlinear_item *items, int n, int64_t M, lowbit_dtype xdt, int norm,
                                float eps_norm, lowbit_format f, lowbit_dtype ydt, int prefetch, int32_t *status,
                                cudaStream_t st);

lowbit_status act_row_stats_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                   const float *g, int hb, float *row_max, double *row_ss, int32_t *status,
                                   cudaStream_t st);
lowbit_status act_codes_given_max_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                         const float *g, int hb, const float *row_max, int8_t *q, int64_t ldq,
                                         int32_t *status, cudaStream_t st);
lowbit_status act_scales_launch(const float *row_max, const double *row_ss, int64_t M, int64_t K_total, int norm,
                                float eps_norm, int hb, float *s_x, int32_t *status, cudaStream_t st);
lowbit_status rescale_launch(const int32_t *acc, int64_t ldacc, int64_t M, int64_t N, const float *s_x,
                             const float *s_w, int per_row, void *y, lowbit_dtype ydt, int64_t ldy, cudaStream_t st);

lowbit_status set_wait_limit_gemm(long long cycles);
lowbit_status set_wait_limit_gemm_ts(long long cycles);
lowbit_status set_wait_limit_skinny(long long cycles);

lowbit_status launch_status()
{
    return cudaGetLastError() == cudaSuccess ? LOWBIT_OK : LOWBIT_ERR_CUDA;
}

namespace {

struct DeviceInfo {
    int sms = 0;
    int major = 0;
    int minor = 0;
    bool ok = false;
};

// Queried once per device; SM count and compute capability are published
// together as one int (SMs in the low 16 bits, major and minor above).
DeviceInfo device_info()
{
    static PerDevice cache;
    DeviceInfo d;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return d;
    const int packed = cache.get(dev, [&] {
        cudaDeviceProp p;
        if (cudaGetDeviceProperties(&p, dev) != cudaSuccess || p.multiProcessorCount <= 0 ||
            p.multiProcessorCount > 0xffff || p.major < 0 || p.major > 0x7f || p.minor < 0 || p.minor > 0xff)
            return 0;
        return p.multiProcessorCount | (p.minor << 16) | (p.major << 24);
    });
    if (packed <= 0) return d;
    d.sms = packed & 0xffff;
    d.minor = (packed >> 16) & 0xff;
    d.major = (packed >> 24) & 0x7f;
    d.ok = true;
    return d;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_format(lowbit_format f) { return f == LOWBIT_TERNARY2 || f == LOWBIT_BINARY1 || f == LOWBIT_INT4; }

// The kernel lowbit_linear_path launches for a valid problem; rb = packed
// row bytes, sms = SMs of the GPU it runs on.
lowbit_kernel choose_kernel(int64_t M, int64_t N, int64_t K, lowbit_format f, int64_t rb, int path, int64_t sms)
{
    // Up to 4 tokens the dp4a GEMV streams weights fastest; from 5 on its
    // int8 MACs outgrow the CUDA cores and tensor-core MMAs win.
    if (path == 1 || (path == 0 && M <= 4)) return LOWBIT_KERNEL_GEMV;
    // 5 to 16 tokens: warp-level tensor-core MMAs, with long rows streamed
    // (weights and token codes) through a TMA ring and K split over a
    // cluster when the output rows are few; measured faster than the split-K
    // GEMM on every decode shape of the workloads (e.g. 9728->2560 at M = 16:
    // 11.0 vs 12.4 us before the cluster split; 3584->1280 at M = 8: 6.7 vs
    // 10.0 us).
    (void)rb;
    if (path == 5 || (path == 0 && M <= 16)) return LOWBIT_KERNEL_WARP_MMA;
    if (path == 6) return LOWBIT_KERNEL_GEMM_PAIR;
    if (path == 4) return LOWBIT_KERNEL_GEMM_TMEM_PAIR;
    // Below 512 tokens the shared-memory variant, which splits K over a
    // cluster when tiles are few, wins.  From 512 tokens ternary weights run
    // on SM pairs with the expanded tile in shared memory (measured fastest
    // for them), except for deep K (>= 2048) with output tiles too few to
    // fill the GPU: there the split-K shared-memory kernel stays faster
    // (9728->2560 at M = 512: 28.6 us vs 32.8 us; for 1024->256 at M = 1024
    // the pair kernel is ahead, 9.2 us vs 9.6 us).  4-bit and binary weights
    // take the tensor-memory variant from 512 tokens (the split-K kernel
    // measured faster for some of their shapes and slower for others).
    const bool splits = gemm_splits_k(f, M, N, K, sms);
    if (path == 0 && M >= 512 && f == LOWBIT_TERNARY2)
        return (K >= 2048 && splits) ? LOWBIT_KERNEL_GEMM_SPLITK : LOWBIT_KERNEL_GEMM_PAIR;
    if (path == 3 || (path == 0 && M >= 512)) return LOWBIT_KERNEL_GEMM_TMEM;
    return splits ? LOWBIT_KERNEL_GEMM_SPLITK : LOWBIT_KERNEL_GEMM;
}

// Checks shared by lowbit_linear_ex and lowbit_linear_kernel that depend on
// the problem's shape only.
lowbit_status check_linear_shape(int64_t M, int64_t N, int64_t K, lowbit_format f, int path)
{
    if (!valid_format(f) || path < 0 || path > 6) return LOWBIT_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || M > INT32_MAX || N > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    if (path == 5 && M > 16) return LOWBIT_ERR_INVALID_ARG;
    if (K > lowbit_max_k(f)) return LOWBIT_ERR_OVERFLOW_BOUND;
    return LOWBIT_OK;
}

}  // namespace

// The kernels are built for sm_100a only.
lowbit_status check_device()
{
    const DeviceInfo d = device_info();
    if (!d.ok) return LOWBIT_ERR_CUDA;
    if (d.major != 10 || d.minor != 0) return LOWBIT_ERR_UNSUPPORTED;
    return LOWBIT_OK;
}

int device_sm_count()
{
    const DeviceInfo d = device_info();
    return d.ok ? d.sms : 148;
}

}  // namespace lowbit

using namespace lowbit;

extern "C" {

size_t lowbit_packed_row_bytes(lowbit_format f, int64_t K)
{
    if (K <= 0) return 0;
    switch (f) {
    case LOWBIT_TERNARY2: return static_cast<size_t>(4 * ((K + 15) / 16));
    case LOWBIT_BINARY1: return static_cast<size_t>((K + 7) / 8);
    case LOWBIT_INT4: return static_cast<size_t>(4 * ((K + 7) / 8));
    default: return 0;
    }
}

size_t lowbit_packed_ld(lowbit_format f, int64_t K)
{
    const size_t rb = lowbit_packed_row_bytes(f, K);
    return (rb + 15) / 16 * 16;
}

int64_t lowbit_scale_count(lowbit_format f, int64_t N)
{
    if (N <= 0 || !valid_format(f)) return 0;
    return f == LOWBIT_TERNARY2 ? 1 : N;
}

int64_t lowbit_max_k(lowbit_format f)
{
    // The kernels accumulate (c << S) * q: 2^31 / (128 * 64) - 1 for ternary
    // and binary, 2^31 / (128 * 16 * 7) for 4-bit codes.
    switch (f) {
    case LOWBIT_TERNARY2:
    case LOWBIT_BINARY1: return (static_cast<int64_t>(INT32_MAX) / (128 * 64));
    case LOWBIT_INT4: return (static_cast<int64_t>(INT32_MAX) / (128 * 16 * 7));
    default: return 0;
    }
}

size_t lowbit_pack_workspace_bytes(lowbit_format f, int64_t N)
{
    if (f != LOWBIT_TERNARY2 || N <= 0) return 0;
    return (static_cast<size_t>(N) * 8 + 255) / 256 * 256;
}

lowbit_status lowbit_pack(const float *w, int64_t N, int64_t K, int64_t ldw, lowbit_format f, float eps,
                          uint8_t *packed, int64_t ldp, float *s_w, void *workspace, size_t workspace_bytes,
                          int32_t *status_dev, void *stream)
{
    if (!valid_format(f) || w == nullptr || packed == nullptr || s_w == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || ldw < K || !(eps >= 0.0f) || eps > 3.0e38f) return LOWBIT_ERR_INVALID_ARG;
    if (ldp < static_cast<int64_t>(lowbit_packed_row_bytes(f, K))) return LOWBIT_ERR_INVALID_ARG;
    if (N > INT32_MAX || K > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    if (ldp % 16 != 0 || !aligned(packed, 16) || !aligned(w, 4) || !aligned(s_w, 4)) return LOWBIT_ERR_ALIGNMENT;
    const size_t need = lowbit_pack_workspace_bytes(f, N);
    if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return LOWBIT_ERR_INVALID_ARG;
    if (need > 0 && !aligned(workspace, 8)) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_pack");
    return pack_launch(w, N, K, ldw, f, eps, packed, ldp, s_w, workspace, status_dev,
                       static_cast<cudaStream_t>(stream));
}

size_t lowbit_pack_ex_workspace_bytes(lowbit_format f, int quantizer, int64_t N)
{
    if (N <= 0 || !valid_format(f)) return 0;
    if (quantizer == LOWBIT_QUANT_DEFAULT) return lowbit_pack_workspace_bytes(f, N);
    if (quantizer == LOWBIT_QUANT_BINARY_CENTRED && f == LOWBIT_BINARY1)
        return (static_cast<size_t>(N) * 16 + 16 + 255) / 256 * 256;
    return 0;
}

lowbit_status lowbit_pack_ex(const float *w, int64_t N, int64_t K, int64_t ldw, lowbit_format f, int quantizer,
                             float eps, uint8_t *packed, int64_t ldp, float *s_w, void *workspace,
                             size_t workspace_bytes, int32_t *status_dev, void *stream)
{
    if (quantizer == LOWBIT_QUANT_DEFAULT)
        return lowbit_pack(w, N, K, ldw, f, eps, packed, ldp, s_w, workspace, workspace_bytes, status_dev, stream);
    if (quantizer != LOWBIT_QUANT_BINARY_CENTRED || f != LOWBIT_BINARY1) return LOWBIT_ERR_INVALID_ARG;
    if (w == nullptr || packed == nullptr || s_w == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || ldw < K || N > INT32_MAX || K > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    if (ldp < static_cast<int64_t>(lowbit_packed_row_bytes(f, K))) return LOWBIT_ERR_INVALID_ARG;
    if (ldp % 16 != 0 || !aligned(packed, 16) || !aligned(w, 4) || !aligned(s_w, 4)) return LOWBIT_ERR_ALIGNMENT;
    const size_t need = lowbit_pack_ex_workspace_bytes(f, quantizer, N);
    if (workspace == nullptr || workspace_bytes < need) return LOWBIT_ERR_INVALID_ARG;
    if (!aligned(workspace, 8)) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_pack_ex");
    return pack_centred_launch(w, N, K, ldw, packed, ldp, s_w, workspace, status_dev,
                               static_cast<cudaStream_t>(stream));
}

lowbit_status lowbit_unpack(const uint8_t *packed, int64_t ldp, int64_t N, int64_t K, lowbit_format f,
                            int8_t *codes, int64_t ldc, int32_t *status_dev, void *stream)
{
    if (!valid_format(f) || packed == nullptr || codes == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0 || ldc < K || ldp < static_cast<int64_t>(lowbit_packed_row_bytes(f, K)))
        return LOWBIT_ERR_INVALID_ARG;
    if (ldp % 16 != 0 || !aligned(packed, 16)) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_unpack");
    return unpack_launch(packed, ldp, N, K, f, codes, ldc, status_dev, static_cast<cudaStream_t>(stream));
}

lowbit_status lowbit_act_quant(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx, float eps,
                               int8_t *q, int64_t ldq, float *s_x, int32_t *status_dev, void *stream)
{
    if (x == nullptr || q == nullptr || s_x == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (xdt != LOWBIT_F32 && xdt != LOWBIT_BF16) return LOWBIT_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0 || ldx < K || ldq < K || !(eps >= 0.0f) || eps > 3.0e38f) return LOWBIT_ERR_INVALID_ARG;
    if (M > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    const int64_t esz = xdt == LOWBIT_F32 ? 4 : 2;
    if (!aligned(x, static_cast<uintptr_t>(esz)) || !aligned(q, 16) || ldq % 16 != 0 || !aligned(s_x, 4))
        return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_act_quant");
    return act_quant_launch(x, xdt, M, K, ldx, eps, q, ldq, s_x, status_dev, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Checks of the activation-side arguments shared by lowbit_act_quant_ex and
// lowbit_bitlinear (q and s_x checked by the caller, who may allow NULL).
lowbit_status check_prologue_args(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                  const float *g, int norm, float eps_norm, int hadamard)
{
    if (x == nullptr || (xdt != LOWBIT_F32 && xdt != LOWBIT_BF16)) return LOWBIT_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0 || ldx < K || M > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    if (norm != LOWBIT_NORM_NONE && norm != LOWBIT_NORM_RMS) return LOWBIT_ERR_INVALID_ARG;
    if (!(eps_norm >= 0.0f) || eps_norm > 3.0e38f) return LOWBIT_ERR_INVALID_ARG;
    if (hadamard < 0 || hadamard == 1 || (hadamard > 0 && ((hadamard & (hadamard - 1)) != 0 ||
                                                             hadamard > K || K % hadamard != 0)))
        return LOWBIT_ERR_INVALID_ARG;
    const int64_t esz = xdt == LOWBIT_F32 ? 4 : 2;
    if (!aligned(x, static_cast<uintptr_t>(esz)) || (g != nullptr && !aligned(g, 4))) return LOWBIT_ERR_ALIGNMENT;
    const bool options = g != nullptr || norm != LOWBIT_NORM_NONE || hadamard > 0;
    if (options && K > LOWBIT_PROLOGUE_MAX_K) return LOWBIT_ERR_UNSUPPORTED;
    return LOWBIT_OK;
}

// Decode shapes the GEMV can take from activations: M <= 4 rows whose codes
// fit its shared memory.
bool decode_from_x(int64_t M, int64_t K, int hadamard, int path)
{
    return M <= 4 && hadamard == 0 && (path == 0 || path == 1) && M * ((K + 127) / 128 * 128) <= LOWBIT_FUSED_MAX_BYTES;
}

// ... of which the fused kernel (codes computed in every block) takes the
// short rows.
bool fused_decode(int64_t M, int64_t K, int hadamard, int path)
{
    return decode_from_x(M, K, hadamard, path) && K <= LOWBIT_FUSED_MAX_K;
}

}  // namespace

extern "C" {

lowbit_status lowbit_act_quant_ex(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                  const float *g, int norm, float eps_norm, int hadamard,
                                  int8_t *q, int64_t ldq, float *s_x, int32_t *status_dev, void *stream)
{
    const lowbit_status a = check_prologue_args(x, xdt, M, K, ldx, g, norm, eps_norm, hadamard);
    if (a != LOWBIT_OK) return a;
    if (q == nullptr || s_x == nullptr || ldq < K) return LOWBIT_ERR_INVALID_ARG;
    if (!aligned(q, 16) || ldq % 16 != 0 || !aligned(s_x, 4)) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_act_quant_ex");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (g == nullptr && norm == LOWBIT_NORM_NONE && hadamard == 0)
        return act_quant_launch(x, xdt, M, K, ldx, 0.0f, q, ldq, s_x, status_dev, st);
    return act_prologue_launch(x, xdt, M, K, ldx, g, norm, eps_norm, hadamard, q, ldq, s_x, status_dev, st);
}

lowbit_status lowbit_bitlinear(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                               const float *g, int norm, float eps_norm, int hadamard,
                               const uint8_t *packed, int64_t ldp, const float *s_w, lowbit_format f, int64_t N,
                               void *y, lowbit_dtype ydt, int64_t ldy,
                               int8_t *q, int64_t ldq, float *s_x,
                               int path, unsigned flags, int32_t *status_dev, void *stream)
{
    const lowbit_status a = check_prologue_args(x, xdt, M, K, ldx, g, norm, eps_norm, hadamard);
    if (a != LOWBIT_OK) return a;
    if ((flags & ~(LOWBIT_LINEAR_WEIGHTS_STABLE | LOWBIT_LINEAR_EXCLUSIVE)) != 0) return LOWBIT_ERR_INVALID_ARG;
    if (!valid_format(f) || packed == nullptr || s_w == nullptr || y == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (ydt != LOWBIT_F32 && ydt != LOWBIT_BF16 && ydt != LOWBIT_I32) return LOWBIT_ERR_INVALID_ARG;
    if (N <= 0 || ldy < N) return LOWBIT_ERR_INVALID_ARG;
    const lowbit_status shape = check_linear_shape(M, N, K, f, path);
    if (shape != LOWBIT_OK) return shape;
    const int64_t rb = static_cast<int64_t>(lowbit_packed_row_bytes(f, K));
    if (ldp < rb) return LOWBIT_ERR_INVALID_ARG;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    if (!aligned(packed, 16) || ldp % 16 != 0 || !aligned(s_w, 4) || !aligned(y, static_cast<uintptr_t>(esz)))
        return LOWBIT_ERR_ALIGNMENT;
    const bool fused = fused_decode(M, K, hadamard, path);
    if (!fused && (q == nullptr || s_x == nullptr)) return LOWBIT_ERR_INVALID_ARG;
    if (q != nullptr) {
        if (ldq < K) return LOWBIT_ERR_INVALID_ARG;
        if (!aligned(q, 16) || ldq % 16 != 0) return LOWBIT_ERR_ALIGNMENT;
    }
    if (s_x != nullptr && !aligned(s_x, 4)) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int prefetch = (flags & LOWBIT_LINEAR_WEIGHTS_STABLE) != 0 ? 1 : 0;
    if (fused) {
        const TraceRange trace("lowbit_bitlinear");
        const lowbit_bitlinear_item item = {x, ldx, g, packed, ldp, s_w, N, K, y, ldy, q, ldq, s_x};
        return gemv_group_launch(&item, 1, M, xdt, norm, eps_norm, f, ydt, prefetch, status_dev, st);
    }
    const lowbit_status s1 = lowbit_act_quant_ex(x, xdt, M, K, ldx, g, norm, eps_norm, hadamard, q, ldq, s_x,
                                                 status_dev, stream);
    if (s1 != LOWBIT_OK) return s1;
    // the prologue kernel just before writes q and s_x, never the weights
    return lowbit_linear_ex(q, ldq, s_x, M, K, packed, ldp, s_w, f, N, y, ydt, ldy, path, flags, status_dev, stream);
}

lowbit_status lowbit_bitlinear_group(const lowbit_bitlinear_item *items, int n_items, int64_t M,
                                     lowbit_dtype xdt, int norm, float eps_norm, lowbit_format f,
                                     lowbit_dtype ydt, unsigned flags, int32_t *status_dev, void *stream)
{
    if (items == nullptr || n_items < 1 || n_items > LOWBIT_GROUP_MAX || M < 1 || M > 4)
        return LOWBIT_ERR_INVALID_ARG;
    if ((flags & ~(LOWBIT_LINEAR_WEIGHTS_STABLE | LOWBIT_LINEAR_EXCLUSIVE)) != 0) return LOWBIT_ERR_INVALID_ARG;
    if (!valid_format(f) || (ydt != LOWBIT_F32 && ydt != LOWBIT_BF16 && ydt != LOWBIT_I32))
        return LOWBIT_ERR_INVALID_ARG;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    for (int i = 0; i < n_items; ++i) {
        const lowbit_bitlinear_item &it = items[i];
        const lowbit_status a = check_prologue_args(it.x, xdt, M, it.K, it.ldx, it.g, norm, eps_norm, 0);
        if (a != LOWBIT_OK) return a;
        if (it.packed == nullptr || it.s_w == nullptr || it.y == nullptr) return LOWBIT_ERR_INVALID_ARG;
        if (it.N <= 0 || it.ldy < it.N) return LOWBIT_ERR_INVALID_ARG;
        const lowbit_status shape = check_linear_shape(M, it.N, it.K, f, 0);
        if (shape != LOWBIT_OK) return shape;
        if (!decode_from_x(M, it.K, 0, 0)) return LOWBIT_ERR_UNSUPPORTED;
        if (it.ldp < static_cast<int64_t>(lowbit_packed_row_bytes(f, it.K))) return LOWBIT_ERR_INVALID_ARG;
        if (!aligned(it.packed, 16) || it.ldp % 16 != 0 || !aligned(it.s_w, 4) ||
            !aligned(it.y, static_cast<uintptr_t>(esz)))
            return LOWBIT_ERR_ALIGNMENT;
        if (it.q != nullptr) {
            if (it.ldq < it.K) return LOWBIT_ERR_INVALID_ARG;
            if (!aligned(it.q, 16) || it.ldq % 16 != 0) return LOWBIT_ERR_ALIGNMENT;
        }
        if (it.s_x != nullptr && !aligned(it.s_x, 4)) return LOWBIT_ERR_ALIGNMENT;
    }
    // layers longer than LOWBIT_FUSED_MAX_K run as lowbit_bitlinear does for
    // them (prologue kernel, then the GEMV): their q and s_x are required
    lowbit_bitlinear_item short_items[LOWBIT_GROUP_MAX];
    int n_short = 0;
    for (int i = 0; i < n_items; ++i) {
        if (items[i].K <= LOWBIT_FUSED_MAX_K) short_items[n_short++] = items[i];
        else if (items[i].q == nullptr || items[i].s_x == nullptr) return LOWBIT_ERR_INVALID_ARG;
    }
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_bitlinear_group");
    const int prefetch = (flags & LOWBIT_LINEAR_WEIGHTS_STABLE) != 0 ? 1 : 0;
    if (n_short > 0) {
        const lowbit_status s = gemv_group_launch(short_items, n_short, M, xdt, norm, eps_norm, f, ydt, prefetch,
                                                  status_dev, static_cast<cudaStream_t>(stream));
        if (s != LOWBIT_OK) return s;
    }
    for (int i = 0; i < n_items; ++i) {
        const lowbit_bitlinear_item &it = items[i];
        if (it.K <= LOWBIT_FUSED_MAX_K) continue;
        const lowbit_status s = lowbit_bitlinear(it.x, xdt, M, it.K, it.ldx, it.g, norm, eps_norm, 0, it.packed, it.ldp,
                                                 it.s_w, f, it.N, it.y, ydt, it.ldy, it.q, it.ldq, it.s_x, 0, flags,
                                                 status_dev, stream);
        if (s != LOWBIT_OK) return s;
    }
    return LOWBIT_OK;
}

lowbit_status lowbit_act_row_stats(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                   const float *g, int hadamard, float *row_max, double *row_ss,
                                   int32_t *status_dev, void *stream)
{
    const lowbit_status a = check_prologue_args(x, xdt, M, K, ldx, g, LOWBIT_NORM_NONE, 0.0f, hadamard);
    if (a != LOWBIT_OK) return a;
    if (row_max == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (K > LOWBIT_PROLOGUE_MAX_K) return LOWBIT_ERR_UNSUPPORTED;
    if (!aligned(row_max, 4) || (row_ss != nullptr && !aligned(row_ss, 8))) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_act_row_stats");
    return act_row_stats_launch(x, xdt, M, K, ldx, g, hadamard, row_max, row_ss, status_dev,
                                static_cast<cudaStream_t>(stream));
}

lowbit_status lowbit_act_quant_given_max(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                         const float *g, int hadamard, const float *row_max,
                                         int8_t *q, int64_t ldq, int32_t *status_dev, void *stream)
{
    const lowbit_status a = check_prologue_args(x, xdt, M, K, ldx, g, LOWBIT_NORM_NONE, 0.0f, hadamard);
    if (a != LOWBIT_OK) return a;
    if (row_max == nullptr || q == nullptr || ldq < K) return LOWBIT_ERR_INVALID_ARG;
    if (K > LOWBIT_PROLOGUE_MAX_K) return LOWBIT_ERR_UNSUPPORTED;
    if (!aligned(row_max, 4) || !aligned(q, 16) || ldq % 16 != 0) return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_act_quant_given_max");
    return act_codes_given_max_launch(x, xdt, M, K, ldx, g, hadamard, row_max, q, ldq, status_dev,
                                      static_cast<cudaStream_t>(stream));
}

lowbit_status lowbit_act_scales(const float *row_max, const double *row_ss, int64_t M, int64_t K_total, int norm,
                                float eps_norm, int hadamard, float *s_x, int32_t *status_dev, void *stream)
{
    if (row_max == nullptr || s_x == nullptr || M <= 0 || K_total <= 0 || M > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    if (norm != LOWBIT_NORM_NONE && norm != LOWBIT_NORM_RMS) return LOWBIT_ERR_INVALID_ARG;
    if (norm == LOWBIT_NORM_RMS && row_ss == nullptr) return LOWBIT_ERR_INVALID_ARG;
    if (!(eps_norm >= 0.0f) || eps_norm > 3.0e38f) return LOWBIT_ERR_INVALID_ARG;
    if (hadamard < 0 || hadamard == 1 || (hadamard > 0 && ((hadamard & (hadamard - 1)) != 0 || hadamard > K_total)))
        return LOWBIT_ERR_INVALID_ARG;
    if (!aligned(row_max, 4) || !aligned(s_x, 4) || (row_ss != nullptr && !aligned(row_ss, 8)))
        return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_act_scales");
    return act_scales_launch(row_max, row_ss, M, K_total, norm, eps_norm, hadamard, s_x, status_dev,
                             static_cast<cudaStream_t>(stream));
}

lowbit_status lowbit_rescale(const int32_t *acc, int64_t ldacc, int64_t M, int64_t N, const float *s_x,
                             const float *s_w, lowbit_format f, void *y, lowbit_dtype ydt, int64_t ldy,
                             int32_t *status_dev, void *stream)
{
    (void)status_dev;
    if (acc == nullptr || s_x == nullptr || s_w == nullptr || y == nullptr || !valid_format(f))
        return LOWBIT_ERR_INVALID_ARG;
    if (ydt != LOWBIT_F32 && ydt != LOWBIT_BF16 && ydt != LOWBIT_I32) return LOWBIT_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || ldacc < N || ldy < N || M > INT32_MAX || N > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    if (!aligned(acc, 4) || !aligned(s_x, 4) || !aligned(s_w, 4) || !aligned(y, static_cast<uintptr_t>(esz)))
        return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const TraceRange trace("lowbit_rescale");
    return rescale_launch(acc, ldacc, M, N, s_x, s_w, f == LOWBIT_TERNARY2 ? 0 : 1, y, ydt, ldy,
                          static_cast<cudaStream_t>(stream));
}

lowbit_status lowbit_linear_ex(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                               const uint8_t *packed, int64_t ldp, const float *s_w, lowbit_format f, int64_t N,
                               void *y, lowbit_dtype ydt, int64_t ldy, int path, unsigned flags,
                               int32_t *status_dev, void *stream)
{
    if ((flags & ~(LOWBIT_LINEAR_WEIGHTS_STABLE | LOWBIT_LINEAR_EXCLUSIVE)) != 0) return LOWBIT_ERR_INVALID_ARG;
    const int prefetch = (flags & LOWBIT_LINEAR_WEIGHTS_STABLE) != 0 ? 1 : 0;
    if (!valid_format(f) || q == nullptr || s_x == nullptr || packed == nullptr || s_w == nullptr || y == nullptr)
        return LOWBIT_ERR_INVALID_ARG;
    if (ydt != LOWBIT_F32 && ydt != LOWBIT_BF16 && ydt != LOWBIT_I32) return LOWBIT_ERR_INVALID_ARG;
    if (path < 0 || path > 6) return LOWBIT_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0 || ldq < K || ldy < N) return LOWBIT_ERR_INVALID_ARG;
    if (path == 5 && M > 16) return LOWBIT_ERR_INVALID_ARG;
    if (M > INT32_MAX || N > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
    const int64_t rb = static_cast<int64_t>(lowbit_packed_row_bytes(f, K));
    if (ldp < rb) return LOWBIT_ERR_INVALID_ARG;
    const lowbit_status shape = check_linear_shape(M, N, K, f, path);
    if (shape != LOWBIT_OK) return shape;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    if (!aligned(q, 16) || ldq % 16 != 0 || !aligned(packed, 16) || ldp % 16 != 0 || !aligned(s_x, 4) ||
        !aligned(s_w, 4) || !aligned(y, static_cast<uintptr_t>(esz)))
        return LOWBIT_ERR_ALIGNMENT;
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const TraceRange trace("lowbit_linear");
    switch (choose_kernel(M, N, K, f, rb, path, device_sm_count())) {
    case LOWBIT_KERNEL_GEMV:
        return gemv_launch(q, ldq, s_x, M, K, packed, ldp, rb, s_w, f, N, y, ydt, ldy, prefetch, st);
    case LOWBIT_KERNEL_WARP_MMA:
        return skinny_launch(q, ldq, s_x, M, K, packed, ldp, rb, s_w, f, N, y, ydt, ldy, prefetch, status_dev, st);
    case LOWBIT_KERNEL_GEMM_PAIR:
        return gemm_pair_launch(q, ldq, s_x, M, K, packed, ldp, rb, s_w, f, N, y, ydt, ldy, prefetch,
                                (flags & LOWBIT_LINEAR_EXCLUSIVE) != 0 ? 1 : 0, status_dev, st);
    case LOWBIT_KERNEL_GEMM_TMEM_PAIR:
        return gemm_ts_pair_launch(q, ldq, s_x, M, K, packed, ldp, rb, s_w, f, N, y, ydt, ldy, status_dev, st);
    case LOWBIT_KERNEL_GEMM_TMEM:
        return gemm_ts_launch(q, ldq, s_x, M, K, packed, ldp, rb, s_w, f, N, y, ydt, ldy, prefetch, status_dev, st);
    default:  // LOWBIT_KERNEL_GEMM or LOWBIT_KERNEL_GEMM_SPLITK: the launcher splits by the same rule
        return gemm_launch(q, ldq, s_x, M, K, packed, ldp, rb, s_w, f, N, y, ydt, ldy, prefetch, status_dev, st);
    }
}

lowbit_status lowbit_linear_kernel(int64_t M, int64_t N, int64_t K, lowbit_format f, int path, int sm_count,
                                   lowbit_kernel *kernel)
{
    if (kernel == nullptr) return LOWBIT_ERR_INVALID_ARG;
    const lowbit_status shape = check_linear_shape(M, N, K, f, path);
    if (shape != LOWBIT_OK) return shape;
    int64_t sms = sm_count;
    if (sms <= 0) {
        const lowbit_status d = check_device();
        if (d != LOWBIT_OK) return d;
        sms = device_sm_count();
    }
    *kernel = choose_kernel(M, N, K, f, static_cast<int64_t>(lowbit_packed_row_bytes(f, K)), path, sms);
    return LOWBIT_OK;
}

const char *lowbit_kernel_name(lowbit_kernel k)
{
    switch (k) {
    case LOWBIT_KERNEL_GEMV: return "gemv_smem_kernel/gemv_kernel";
    case LOWBIT_KERNEL_WARP_MMA: return "skinny_mma_kernel/stream_mma_kernel";
    case LOWBIT_KERNEL_GEMM: return "gemm_kernel";
    case LOWBIT_KERNEL_GEMM_SPLITK: return "gemm_splitk_kernel";
    case LOWBIT_KERNEL_GEMM_PAIR: return "gemm_pair_kernel";
    case LOWBIT_KERNEL_GEMM_TMEM: return "gemm_ts_kernel";
    case LOWBIT_KERNEL_GEMM_TMEM_PAIR: return "gemm_ts_pair_kernel";
    default: return "unknown";
    }
}

lowbit_status lowbit_linear_path(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                                 const uint8_t *packed, int64_t ldp, const float *s_w, lowbit_format f, int64_t N,
                                 void *y, lowbit_dtype ydt, int64_t ldy, int path, int32_t *status_dev,
                                 void *stream)
{
    return lowbit_linear_ex(q, ldq, s_x, M, K, packed, ldp, s_w, f, N, y, ydt, ldy, path, 0u, status_dev, stream);
}

lowbit_status lowbit_linear(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                            const uint8_t *packed, int64_t ldp, const float *s_w, lowbit_format f, int64_t N,
                            void *y, lowbit_dtype ydt, int64_t ldy, int32_t *status_dev, void *stream)
{
    return lowbit_linear_path(q, ldq, s_x, M, K, packed, ldp, s_w, f, N, y, ydt, ldy, 0, status_dev, stream);
}

lowbit_status lowbit_set_wait_limit(int64_t cycles)
{
    const lowbit_status d = check_device();
    if (d != LOWBIT_OK) return d;
    const long long c = cycles > 0 ? static_cast<long long>(cycles) : 0;
    lowbit_status s = set_wait_limit_gemm(c);
    if (s == LOWBIT_OK) s = set_wait_limit_gemm_ts(c);
    if (s == LOWBIT_OK) s = set_wait_limit_skinny(c);
    return s;
}

const char *lowbit_status_string(lowbit_status s)
{
    switch (s) {
    case LOWBIT_OK: return "ok";
    case LOWBIT_ERR_INVALID_ARG: return "invalid argument";
    case LOWBIT_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case LOWBIT_ERR_UNSUPPORTED: return "unsupported (needs an sm_100 device)";
    case LOWBIT_ERR_OVERFLOW_BOUND: return "K exceeds the int32 accumulator bound";
    case LOWBIT_ERR_NONFINITE: return "non-finite input";
    case LOWBIT_ERR_RESERVED_CODE: return "reserved code pattern or non-zero unowned bit";
    case LOWBIT_ERR_TIMEOUT: return "device pipeline wait timed out";
    case LOWBIT_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
    }
}

int lowbit_version(void) { return 100; }

}  // extern "C"
