// epilogue.cu -- the rescale of int32 accumulators as a kernel of its own.
//
// "M8.8 - Native Binary and Ternary Transformers" 0x02D: y = float(acc) *
// (s_w * s_x), the two scales multiplied first.  The linear kernels fuse this
// step; it runs separately where the accumulators of one output are summed
// across ranks first (a row-parallel layer, 0x08B-0x08C: the int32 partial
// sums are all-reduced before the epilogue, which keeps the result identical
// to the unsplit layer).  One thread per four outputs of a row; HBM-bound.
#include "lowbit_internal.cuh"

namespace lowbit {
namespace {

template <int OUT>
__device__ __forceinline__ void put(void *y, int64_t idx, int32_t a, float sw, float sx)
{
    if constexpr (OUT == LOWBIT_F32) static_cast<float *>(y)[idx] = rescale(a, sw, sx);
    else if constexpr (OUT == LOWBIT_BF16) static_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(rescale(a, sw, sx));
    else static_cast<int32_t *>(y)[idx] = a;
}

template <int OUT>
__global__ void __launch_bounds__(256)
rescale_kernel(const int32_t *__restrict__ acc, int64_t ldacc, int64_t M, int64_t N, const float *__restrict__ s_x,
               const float *__restrict__ s_w, int per_row, void *__restrict__ y, int64_t ldy)
{
    pdl_wait();
    pdl_trigger();
    const int64_t quads = (N + 3) / 4;
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= M * quads) return;
    const int64_t t = i / quads;
    const int64_t n0 = (i % quads) * 4;
    const float sx = ld_act_f32(s_x + t);
    for (int j = 0; j < 4; ++j) {
        const int64_t n = n0 + j;
        if (n < N) put<OUT>(y, t * ldy + n, static_cast<int32_t>(ld_act_u32(acc + t * ldacc + n)), s_w[per_row ? n : 0], sx);
    }
}

}  // namespace

lowbit_status rescale_launch(const int32_t *acc, int64_t ldacc, int64_t M, int64_t N, const float *s_x,
                             const float *s_w, int per_row, void *y, lowbit_dtype ydt, int64_t ldy, cudaStream_t st)
{
    const int64_t threads = M * ((N + 3) / 4);
    const dim3 grid(static_cast<unsigned>((threads + 255) / 256)), block(256);
    if (ydt == LOWBIT_F32)
        return launch_pdl(rescale_kernel<LOWBIT_F32>, grid, block, 0, st, 0, acc, ldacc, M, N, s_x, s_w, per_row, y, ldy);
    if (ydt == LOWBIT_BF16)
        return launch_pdl(rescale_kernel<LOWBIT_BF16>, grid, block, 0, st, 0, acc, ldacc, M, N, s_x, s_w, per_row, y,
                          ldy);
    return launch_pdl(rescale_kernel<LOWBIT_I32>, grid, block, 0, st, 0, acc, ldacc, M, N, s_x, s_w, per_row, y, ldy);
}

}  // namespace lowbit
