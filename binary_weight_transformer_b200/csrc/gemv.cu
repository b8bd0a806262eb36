// gemv.cu -- dispatch of the packed-weight GEMV over the weight formats.
#include "lowbit_internal.cuh"

namespace lowbit {
lowbit_status gemv_launch_t2(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_launch_b1(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_launch_i4(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);

lowbit_status gemv_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                          const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                          lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                          cudaStream_t st)
{
    if (f == LOWBIT_TERNARY2) return gemv_launch_t2(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
    if (f == LOWBIT_BINARY1) return gemv_launch_b1(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
    return gemv_launch_i4(q, ldq, s_x, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
}
}  // namespace lowbit
