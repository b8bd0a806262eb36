// gemv.cu -- dispatch of the packed-weight GEMV over the weight formats.
#include "gemv_impl.cuh"

namespace lowbit {
lowbit_status gemv_launch_t2(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_launch_b1(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);
lowbit_status gemv_launch_i4(const int8_t *, int64_t, const float *, int64_t, int64_t, const uint8_t *, int64_t,
                             int64_t, const float *, int64_t, void *, lowbit_dtype, int64_t, int, cudaStream_t);

lowbit_status gemv_group_launch_t2(const gemv_detail::GroupArgs &, lowbit_dtype, cudaStream_t);
lowbit_status gemv_group_launch_b1(const gemv_detail::GroupArgs &, lowbit_dtype, cudaStream_t);
lowbit_status gemv_group_launch_i4(const gemv_detail::GroupArgs &, lowbit_dtype, cudaStream_t);

// The grouped fused decode call of lowbit_bitlinear_group (and of
// lowbit_bitlinear with one item): x -> codes in the kernel -> GEMV, for
// every item.  The arguments are checked by the caller.
lowbit_status gemv_group_launch(const lowbit_bitlinear_item *items, int n, int64_t M, lowbit_dtype xdt, int norm,
                                float eps_norm, lowbit_format f, lowbit_dtype ydt, int prefetch, int32_t *status,
                                cudaStream_t st)
{
    if (n < 1 || n > gemv_detail::kGroupMax || M < 1 || M > 4) return LOWBIT_ERR_INVALID_ARG;
    gemv_detail::GroupArgs a = {};
    a.n_items = n;
    a.M = static_cast<int>(M);
    a.xbf16 = xdt == LOWBIT_BF16 ? 1 : 0;
    a.norm = norm;
    a.eps_norm = eps_norm;
    a.status = status;
    a.prefetch = prefetch;
    for (int i = 0; i < n; ++i) {
        const lowbit_bitlinear_item &in = items[i];
        gemv_detail::GroupItem &I = a.item[i];
        if (in.N > INT32_MAX || in.K > INT32_MAX) return LOWBIT_ERR_INVALID_ARG;
        I.x = in.x;
        I.g = in.g;
        I.q_out = in.q;
        I.s_x_out = in.s_x;
        I.packed = in.packed;
        I.s_w = in.s_w;
        I.y = in.y;
        I.ldx = in.ldx;
        I.ldq_out = in.ldq;
        I.ldp = in.ldp;
        I.ldy = in.ldy;
        I.N = static_cast<int32_t>(in.N);
        I.K = static_cast<int32_t>(in.K);
        I.nchunks = static_cast<int32_t>((lowbit_packed_row_bytes(f, in.K) + 15) / 16);
    }
    if (f == LOWBIT_TERNARY2) return gemv_group_launch_t2(a, ydt, st);
    if (f == LOWBIT_BINARY1) return gemv_group_launch_b1(a, ydt, st);
    return gemv_group_launch_i4(a, ydt, st);
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
