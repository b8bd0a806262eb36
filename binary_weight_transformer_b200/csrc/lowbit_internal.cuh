// lowbit_internal.cuh -- device helpers shared by the library's kernels.
//
// Code expansion.  Every kernel turns packed weight codes into int8x4 words
// that hold (c << S) for four consecutive codes, S = 6 for ternary and binary
// and S = 4 for 4-bit codes.  Shifting the field to the top of its byte makes
// the sign extension free; the integer dot then carries a factor 2^S that the
// epilogue removes with an exact arithmetic shift (the sum is a multiple of
// 2^S).  The int32 bound becomes |acc| * 2^S < 2^31, which is why
// lowbit_max_k is 2^31 / (128 * 64) - 1 for ternary and binary and
// 2^31 / (128 * 16 * 7) for 4-bit codes.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>

#include "lowbit.h"
#include "host_once.h"

namespace lowbit {

// A named range on the NVTX timeline (Nsight Systems, ncu's NVTX filters)
// around the launches of one ABI call.  With no tool attached the push and
// the pop return at once.
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};

constexpr int kT2 = LOWBIT_TERNARY2;
constexpr int kB1 = LOWBIT_BINARY1;
constexpr int kI4 = LOWBIT_INT4;

template <int FMT> struct Fmt;
// Ternary: 16 codes per 32-bit word, plane order (byte (k%16)%4, field (k%16)/4).
template <> struct Fmt<kT2> {
    static constexpr int kBits = 2;
    static constexpr int kShift = 6;
    static constexpr int kCodesPerWord = 16;
};
// Binary: 32 codes per word, bit k (little-bit-first bytes), 1 = -1.
template <> struct Fmt<kB1> {
    static constexpr int kBits = 1;
    static constexpr int kShift = 6;
    static constexpr int kCodesPerWord = 32;
};
// 4-bit: 8 codes per word, plane order (byte (k%8)%4, nibble (k%8)/4).
template <> struct Fmt<kI4> {
    static constexpr int kBits = 4;
    static constexpr int kShift = 4;
    static constexpr int kCodesPerWord = 8;
};

// Four ternary codes 4j..4j+3 of word w as int8 (64*c): move field j of each
// byte to bits 7..6 of that byte.
__device__ __forceinline__ uint32_t t2_expand(uint32_t w, int j)
{
    return (w << (6 - 2 * j)) & 0xC0C0C0C0u;
}

// Four 4-bit codes 4h..4h+3 of word w as int8 (16*c): nibble h of each byte
// moved to the high nibble.
__device__ __forceinline__ uint32_t i4_expand(uint32_t w, int h)
{
    return h == 0 ? ((w << 4) & 0xF0F0F0F0u) : (w & 0xF0F0F0F0u);
}

// Four binary codes from the low 4 bits of `nib`: bit m goes to bit 7 of byte
// m (one multiply by 2^7 + 2^14 + 2^21 + 2^28 spreads the four bits without
// carries), then bit 6 is set in every byte: 0x40 = +64, 0xC0 = -64.
__device__ __forceinline__ uint32_t b1_expand_nibble(uint32_t nib)
{
    return ((nib * 0x10204080u) & 0x80808080u) | 0x40404040u;
}

__device__ __forceinline__ void report(int32_t *status, int code)
{
    if (status != nullptr) atomicOr(status, 1 << code);
}

__device__ __forceinline__ bool finite_bits(uint32_t u) { return (u & 0x7f800000u) != 0x7f800000u; }

// 16-byte streaming load that does not allocate in L1 (weights are read once
// per launch).  It takes the non-coherent read-only path, so it is only for
// data that no kernel writes while the reader is resident: the packed
// weights (see LOWBIT_LINEAR_WEIGHTS_STABLE).
__device__ __forceinline__ uint4 ld_stream_u4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Loads of activation-side data (x, codes, scales).  The kernels are
// launched with programmatic stream serialization, so a kernel can be
// resident while the kernel before it still writes these arrays; after
// griddepcontrol.wait the writes are visible to coherent loads, but the
// read-only (.nc) path is defined only for data constant over the reader's
// lifetime.  These loads are cached in L2 only (.cg), which is coherent and
// does not allocate in L1.
__device__ __forceinline__ uint4 ld_act_u4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// The same for activation-side data that every row of a kernel re-reads (a
// gain vector): L1-allocating (.ca), still issued after griddepcontrol.wait
// by the asm volatile.
__device__ __forceinline__ uint4 ld_act_ca_u4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.ca.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_act_u32(const void *p)
{
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint16_t ld_act_u16(const void *p)
{
    uint16_t v;
    asm volatile("ld.global.cg.u16 %0, [%1];" : "=h"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ float ld_act_f32(const float *p) { return __uint_as_float(ld_act_u32(p)); }

__device__ __forceinline__ double ld_act_f64(const double *p)
{
    double v;
    asm volatile("ld.global.cg.f64 %0, [%1];" : "=d"(v) : "l"(p) : "memory");
    return v;
}

// Output conversion shared by the epilogues: y = float(acc) * (s_w * s_x)
// with the two scales multiplied first, each product one fp32 rounding.
__device__ __forceinline__ float rescale(int32_t acc, float sw, float sx)
{
    return __fmul_rn(__int2float_rn(acc), __fmul_rn(sw, sx));
}

// Programmatic dependent launch.  The hot-path kernels are launched with
// programmatic stream serialization, so a kernel may start while the one
// before it on the stream is still running.  pdl_wait() blocks until that
// kernel has completed and its memory operations are visible; every kernel
// calls it before its first global-memory access (activations, weights,
// outputs, status word), so the order of memory effects is exactly the
// stream order and only the launch and the prologue (barrier set-up, tensor
// memory allocation) overlap the previous kernel.  pdl_trigger() allows the
// next kernel to be launched.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace lowbit

// Host-side launch helpers (defined in abi.cu and pack.cu).
namespace lowbit {
lowbit_status launch_status();
// LOWBIT_OK on a B200 (sm_100); LOWBIT_ERR_UNSUPPORTED on another device,
// LOWBIT_ERR_CUDA when the device cannot be queried.  Cached per device.
lowbit_status check_device();
int device_sm_count();

// Launch with programmatic stream serialization (see pdl_wait); cluster_x > 0
// also sets the cluster size for kernels without compiled-in cluster dims.
template <typename... KArgs, typename... Args>
inline lowbit_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                unsigned cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    unsigned n = 1;
    if (cluster_x > 0) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster_x;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        n = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) return LOWBIT_ERR_CUDA;
    return launch_status();
}
lowbit_status pack_launch(const float *w, int64_t N, int64_t K, int64_t ldw, lowbit_format f, float eps,
                          uint8_t *packed, int64_t ldp, float *s_w, void *workspace, int32_t *status,
                          cudaStream_t st);
}
