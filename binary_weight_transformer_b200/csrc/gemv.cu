// gemv.cu -- dispatch of the packed-weight GEMV over the weight formats.
#include "gemv_impl.cuh"

namespace lowbit {
lowbit_status gemv_launch_t2(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_launch_b1(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_launch_i4(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);

lowbit_status gemv_fused_launch_t2(const gemv_detail::Prologue &, int64_t, int64_t, const uint8_t *, int64_t, int64_t,
                                   const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_fused_launch_b1(const gemv_detail::Prologue &, int64_t, int64_t, const uint8_t *, int64_t, int64_t,
                                   const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_fused_launch_i4(const gemv_detail::Prologue &, int64_t, int64_t, const uint8_t *, int64_t, int64_t,
                                   const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);

// The fused decode call of lowbit_bitlinear: x -> codes in every block -> GEMV.
lowbit_status gemv_fused_launch(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx, const float *g,
                                int norm, float eps_norm, const uint8_t *packed, int64_t ldp, int64_t row_bytes,
                                const float *s_w, lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy,
                                int8_t *q_out, int64_t ldq, float *s_x_out, int prefetch, int32_t *status,
                                cudaStream_t st)
{
    gemv_detail::Prologue pro;
    pro.x = x;
    pro.ldx = ldx;
    pro.g = g;
    pro.q_out = q_out;
    pro.ldq_out = ldq;
    pro.s_x_out = s_x_out;
    pro.status = status;
    pro.eps_norm = eps_norm;
    pro.xbf16 = xdt == LOWBIT_BF16 ? 1 : 0;
    pro.norm = norm;
    if (f == LOWBIT_TERNARY2) return gemv_fused_launch_t2(pro, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
    if (f == LOWBIT_BINARY1) return gemv_fused_launch_b1(pro, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
    return gemv_fused_launch_i4(pro, M, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, st);
}

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
