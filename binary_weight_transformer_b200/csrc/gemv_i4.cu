// gemv_i4.cu -- GEMV instantiations for one weight format (the template
// code is in gemv_impl.cuh; one file per format keeps builds parallel).
#include "gemv_impl.cuh"

namespace lowbit {
lowbit_status gemv_launch_i4(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                              const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N,
                              void *y, lowbit_dtype ydt, int64_t ldy, int prefetch, cudaStream_t st)
{
    return gemv_detail::gemv_launch_fmt<kI4>(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
}

lowbit_status gemv_group_launch_i4(const gemv_detail::GroupArgs &a, lowbit_dtype ydt, cudaStream_t st)
{
    return gemv_detail::gemv_group_launch_fmt<kI4>(a, ydt, st);
}
}  // namespace lowbit
