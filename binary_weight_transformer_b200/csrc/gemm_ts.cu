// gemm_ts.cu -- tensor-core GEMM with the weight operand in tensor memory.
//
// Same operator as gemm_sm100.cu ("M8.8 - Native Binary and Ternary
// Transformers" 0x02D, 0x09A-0x09B): acc = sum_k q[t,k] c[n,k] on the
// 5th-generation tensor cores, the packed artifact consumed directly.  Here
// the operands are swapped: the MMA's A operand is a 128-row tile of weight
// codes and B is a tile of up to 224 tokens, so that
//
//   D[n, t] (TMEM, s32) += A[n, k] (TMEM, int8) * B[t, k] (smem, int8).
//
// Expander warps read their row's packed codes from the TMA-staged tile,
// expand them in registers and write them straight into tensor memory with
// tcgen05.st (one 32-column store per row and K step): the expanded operand
// never passes through shared memory, which leaves shared-memory bandwidth
// to the TMA and the MMA's reads of the token tile.
//
// Warp roles: 0 TMA producer; 1 TMEM allocation and MMA issue; 2-5 expanders
// (warp w owns TMEM lanes 32*(w%4)..+31 = weight rows); 6-9 epilogue.
// TMEM columns: two accumulator buffers of 224 and two A stages of 32.
// Every mbarrier wait is bounded (see tc_common.cuh).
#include "tc_common.cuh"

namespace lowbit {
namespace ts {

using namespace tc;

constexpr int BW = 128;         // weight rows per tile (MMA M)
constexpr int BT = 224;         // largest token tile (MMA N)
constexpr int BK = 128;         // K per stage
constexpr int kThreads = 320;
constexpr int kACols = BK / 4;  // TMEM columns per A stage (4 int8 per column)
constexpr int kAStages = 2;
constexpr int kDCols = BT;
constexpr uint32_t kTmemCols = 512;
constexpr int kStages = 5;      // TMA stages: token tile + packed tile

template <int FMT> __host__ __device__ constexpr int packed_row_kblock() { return BK * Fmt<FMT>::kBits / 8; }
constexpr int Q_BYTES = BT * BK;  // largest token tile
template <int FMT> __host__ __device__ constexpr int p_bytes() { return BW * packed_row_kblock<FMT>(); }
template <int OUT> __host__ __device__ constexpr int stage_row_bytes() { return OUT == LOWBIT_BF16 ? 80 : 144; }
template <int OUT> __host__ __device__ constexpr int stage_warp_bytes() { return 32 * stage_row_bytes<OUT>(); }

template <int FMT, int OUT>
__host__ __device__ constexpr size_t smem_bytes()
{
    return 1024 + static_cast<size_t>(kStages) * (Q_BYTES + p_bytes<FMT>()) + 4 * stage_warp_bytes<OUT>() +
           8 * (2 * kStages + 2 * kAStages + 8);
}

__device__ __forceinline__ void tmem_st_32cols(uint32_t taddr, const uint32_t (&v)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
          "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
          "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
          "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// D (TMEM) += A (TMEM) * B (smem descriptor)^T, s8 x s8 -> s32.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor: s32 accumulate, s8 x s8, both K-major, M = 128, N = nt.
__device__ __forceinline__ uint32_t idesc_for(int nt)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nt >> 3) << 17) |
           (static_cast<uint32_t>(BW >> 4) << 24);
}

// One weight row's 128 codes of one K step, expanded to 32 int8x4 words of
// (c << S) in K order.
template <int FMT>
__device__ __forceinline__ void expand_row(uint32_t prow, uint32_t (&w)[32])
{
    if constexpr (FMT == kT2) {
        // 32 packed bytes = 8 words of 16 codes.
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint4 p = lds128(prow + h * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int g = 0; g < 4; ++g) w[16 * h + 4 * j + g] = t2_expand((&p.x)[j], g);
        }
    } else if constexpr (FMT == kI4) {
        // 64 packed bytes = 16 words of 8 codes.
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint4 p = lds128(prow + h * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                w[8 * h + 2 * j] = i4_expand((&p.x)[j], 0);
                w[8 * h + 2 * j + 1] = i4_expand((&p.x)[j], 1);
            }
        }
    } else {
        // 16 packed bytes = 4 words of 32 codes.
        const uint4 p = lds128(prow);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int m = 0; m < 8; ++m) w[8 * j + m] = b1_expand_nibble(((&p.x)[j] >> (4 * m)) & 0xFu);
    }
}

// Epilogue of one 32-token chunk for this warp's 32 weight rows.  v[i] is the
// accumulator of (row n = this lane, token t0 + i).  The values go through a
// per-warp staging tile (token-major, rows padded by 16 bytes) so that the
// global stores are 64-byte (bf16) or 128-byte (fp32, int32) row segments.
template <int OUT>
__device__ __forceinline__ void store_chunk(const uint32_t (&v)[32], float sw, const float *__restrict__ s_x,
                                            int shift, void *__restrict__ y, int64_t ldy, int64_t t0, int64_t M,
                                            int64_t n0, int64_t N, bool vec_ok, uint32_t stage, int lane)
{
    constexpr int kEsz = OUT == LOWBIT_BF16 ? 2 : 4;
    constexpr int RS = stage_row_bytes<OUT>();
    const int64_t n = n0 + lane;
    if (vec_ok && n0 + 32 <= N) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int32_t a = static_cast<int32_t>(v[i]) >> shift;
            const uint32_t addr = stage + i * RS + lane * kEsz;
            if constexpr (OUT == LOWBIT_I32) {
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
            } else {
                const float sx = (t0 + i < M) ? ld_act_f32(s_x + t0 + i) : 0.0f;
                const float f = rescale(a, sw, sx);
                if constexpr (OUT == LOWBIT_F32) {
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(__float_as_uint(f)) : "memory");
                } else {
                    const __nv_bfloat16 b = __float2bfloat16_rn(f);
                    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(*reinterpret_cast<const uint16_t *>(&b))
                                 : "memory");
                }
            }
        }
        __syncwarp();
        constexpr int kPieces = 32 * kEsz / 16;     // 16-byte pieces per token row
        constexpr int kRowsPerPass = 32 / kPieces;
#pragma unroll
        for (int pass = 0; pass < kPieces; ++pass) {
            const int r = pass * kRowsPerPass + lane / kPieces;
            const int piece = lane % kPieces;
            const uint4 val = lds128(stage + r * RS + piece * 16);
            if (t0 + r < M) {
                char *dst = static_cast<char *>(y) + ((t0 + r) * ldy + n0) * kEsz + piece * 16;
                *reinterpret_cast<uint4 *>(dst) = val;
            }
        }
        __syncwarp();
    } else if (n < N) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (t0 + i < M) {
                const int32_t a = static_cast<int32_t>(v[i]) >> shift;
                const int64_t idx = (t0 + i) * ldy + n;
                if constexpr (OUT == LOWBIT_I32) {
                    static_cast<int32_t *>(y)[idx] = a;
                } else if constexpr (OUT == LOWBIT_F32) {
                    static_cast<float *>(y)[idx] = rescale(a, sw, ld_act_f32(s_x + t0 + i));
                } else {
                    static_cast<__nv_bfloat16 *>(y)[idx] = __float2bfloat16_rn(rescale(a, sw, ld_act_f32(s_x + t0 + i)));
                }
            }
        }
    }
}

template <int FMT, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_ts_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_p,
               const float *__restrict__ s_x, const float *__restrict__ s_w, int64_t M, int64_t N, int64_t K,
               void *__restrict__ y, int64_t ldy, int vec_ok, int nt, int prefetch, int32_t *status)
{
    constexpr int PB = packed_row_kblock<FMT>();
    constexpr int P_BYTES = p_bytes<FMT>();
    constexpr int kShift = Fmt<FMT>::kShift;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                          // kStages x 28 KB, 1024-aligned
    uint8_t *sP = sQ + kStages * Q_BYTES;        // kStages x P_BYTES
    uint8_t *sStage = sP + kStages * P_BYTES;    // 4 x epilogue staging
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + 4 * stage_warp_bytes<OUT>());
    // full_tma[s]: the TMA stage's token and packed tiles have landed.
    // full_a[s2]: A stage s2 holds the expanded weights of a K step, and the
    //   expanders saw that step's TMA stage complete, so one wait on full_a
    //   orders the MMA after both (release/acquire through the expanders).
    // mma_done[s]: the MMAs of the K step that used TMA stage s are complete;
    //   it frees that TMA stage and, two K steps later, the A stage.
    uint64_t *full_tma = bars;
    uint64_t *mma_done = bars + kStages;
    uint64_t *full_a = bars + 2 * kStages;
    uint64_t *acc_full = full_a + 2 * kAStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_full + 4;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(acc_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acc_full + 6);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < kAStages; ++s) mbar_init(&full_a[s], 128);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_p)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(const_cast<uint32_t *>(tmem_slot))), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Global memory is touched only after the previous kernel on the stream
    // has completed (programmatic dependent launch, see pdl_wait).  With
    // prefetch the TMA thread first starts the packed-weight half of its
    // first stages (the caller vouches that the previous kernel does not
    // write the weights) and waits after that.
    if (prefetch == 0 || threadIdx.x != 0) pdl_wait();
    pdl_trigger();
    const uint32_t a_col0 = 2 * kDCols;          // first A stage column

    const int64_t num_w = (N + BW - 1) / BW;
    const int64_t num_t = (M + nt - 1) / nt;
    const int64_t num_tiles = num_w * num_t;
    const int nkb = static_cast<int>((K + BK - 1) / BK);
    const uint32_t q_bytes = static_cast<uint32_t>(nt) * BK;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            uint32_t npre = 0;  // stages whose weight half was started before the wait
            if (prefetch != 0) {
                if (blockIdx.x < num_tiles) {
                    const int w0 = static_cast<int>((blockIdx.x % num_w) * BW);
                    npre = static_cast<uint32_t>(nkb < kStages ? nkb : kStages);
                    for (uint32_t i = 0; i < npre; ++i) {
                        mbar_arrive_expect_tx(&full_tma[i], q_bytes + P_BYTES);
                        tma_load_2d(sP + i * P_BYTES, &map_p, &full_tma[i], static_cast<int>(i) * PB, w0);
                    }
                }
                pdl_wait();
            }
            for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int w0 = static_cast<int>((tile % num_w) * BW);
                const int t0 = static_cast<int>((tile / num_w) * nt);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % kStages;
                    if (g < npre) {
                        tma_load_2d(sQ + s * Q_BYTES, &map_q, &full_tma[s], kb * BK, t0);
                        continue;
                    }
                    if (!wait_bar(&mma_done[s], ((g / kStages) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full_tma[s], q_bytes + P_BYTES);
                    tma_load_2d(sQ + s * Q_BYTES, &map_q, &full_tma[s], kb * BK, t0);
                    tma_load_2d(sP + s * P_BYTES, &map_p, &full_tma[s], kb * PB, w0);
                }
            }
            if (!ok) {
                for (uint32_t i = 0; i < kStages && i < g; ++i) {
                    const uint32_t gi = g - 1 - i;
                    drain_bar(&full_tma[gi % kStages], (gi / kStages) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idesc = idesc_for(nt);
            // K-major SW128 descriptor of TMA stage 0; stage s and K slice kk
            // add (s * Q_BYTES + kk * 32) / 16 to its start-address field.
            const uint64_t qdesc0 = sw128_desc(smem_u32(sQ));
            uint32_t g = 0;
            uint32_t t = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
                const int b = t & 1;
                if (!wait_bar(&acc_empty[b], ((t >> 1) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kDCols);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s1 = g % kStages, s2 = g % kAStages;
                    if (!wait_bar(&full_a[s2], (g / kAStages) & 1u, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t qdesc = qdesc0 + static_cast<uint64_t>((s1 * Q_BYTES) >> 4);
                    const uint32_t a_tmem = tmem_base + a_col0 + static_cast<uint32_t>(s2 * kACols);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        tc_mma_i8_ts(d_tmem, a_tmem + kk * (UMMA_K / 4), qdesc + static_cast<uint64_t>(kk * (UMMA_K >> 4)),
                                     idesc, (kb | kk) != 0 ? 1u : 0u);
                    tc_commit(&mma_done[s1]);
                }
                if (!ok) break;
                tc_commit(&acc_full[b]);
            }
            tc_commit(drain);
            drain_bar(drain, 0);
        }
    } else if (warp < 6) {
        // ---------------- expanders: packed -> TMEM ----------------
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;             // weight row within the tile
        const uint32_t p_base = smem_u32(sP);
        uint32_t g = 0;
        bool ok = true;
        for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int s1 = g % kStages, s2 = g % kAStages;
                int ready = 0;
                if (lane == 0) ready = wait_bar(&full_tma[s1], (g / kStages) & 1u, abort_flag, status) ? 1 : 0;
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (!ready) { ok = false; break; }
                // Expand in registers first: only the TMEM store waits for the
                // A stage, which is free once the MMAs of K step g - kAStages
                // are complete (mma_done of that step's TMA stage).
                uint32_t w[32];
                expand_row<FMT>(p_base + s1 * P_BYTES + r * PB, w);
                if (lane == 0 && g >= static_cast<uint32_t>(kAStages)) {
                    const uint32_t gp = g - kAStages;
                    ready = wait_bar(&mma_done[gp % kStages], (gp / kStages) & 1u, abort_flag, status) ? 1 : 0;
                }
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (!ready) { ok = false; break; }
                tc_fence_after();
                tmem_st_32cols(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a_col0 +
                                   static_cast<uint32_t>(s2 * kACols), w);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&full_a[s2]);
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int quarter = warp & 3;
        const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>((warp - 6) * stage_warp_bytes<OUT>());
        uint32_t t = 0;
        for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
            const int b = t & 1;
            int ready = 0;
            if (lane == 0) ready = wait_bar(&acc_full[b], (t >> 1) & 1u, abort_flag, status) ? 1 : 0;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            tc_fence_after();
            const int64_t n0 = (tile % num_w) * BW + quarter * 32;
            const int64_t t0 = (tile / num_w) * nt;
            const int64_t n = n0 + lane;
            const float sw = (n < N) ? s_w[FMT == kT2 ? 0 : n] : 0.0f;
#pragma unroll 1
            for (int cc = 0; cc < nt / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(b * kDCols + cc * 32), v);
                const int64_t tc0 = t0 + cc * 32;
                if (tc0 < M && n0 < N)
                    store_chunk<OUT>(v, sw, s_x, kShift, y, ldy, tc0, M, n0, N, vec_ok != 0, stage, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

template <int FMT, int OUT>
lowbit_status launch_t(const CUtensorMap &mq, const CUtensorMap &mp, const float *s_x, const float *s_w, int64_t M,
                       int64_t N, int64_t K, void *y, int64_t ldy, int vec_ok, int nt, int prefetch, int32_t *status,
                       cudaStream_t st)
{
    constexpr size_t smem = smem_bytes<FMT, OUT>();
    static_assert(smem <= 232448, "shared memory budget");
    static PerDevice configured;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            return cudaFuncSetAttribute(gemm_ts_kernel<FMT, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(smem)) == cudaSuccess ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    const int64_t tiles = ((N + BW - 1) / BW) * ((M + nt - 1) / nt);
    const int64_t sms = device_sm_count();
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    return launch_pdl(gemm_ts_kernel<FMT, OUT>, dim3(grid), dim3(kThreads), smem, st, 0, mq, mp, s_x, s_w, M, N, K,
                      y, ldy, vec_ok, nt, prefetch, status);
}

template <int FMT>
lowbit_status launch_fmt(const CUtensorMap &mq, const CUtensorMap &mp, const float *s_x, const float *s_w,
                         int64_t M, int64_t N, int64_t K, void *y, lowbit_dtype ydt, int64_t ldy, int vec_ok,
                         int nt, int prefetch, int32_t *status, cudaStream_t st)
{
    if (ydt == LOWBIT_F32)
        return launch_t<FMT, LOWBIT_F32>(mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, prefetch, status, st);
    if (ydt == LOWBIT_BF16)
        return launch_t<FMT, LOWBIT_BF16>(mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, prefetch, status, st);
    return launch_t<FMT, LOWBIT_I32>(mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, prefetch, status, st);
}


// ---------------------------------------------------------------------------
// SM-pair variant (tcgen05 cta_group::2).
//
// A cluster of two CTAs computes a 256-row weight tile: each CTA expands its
// 128 rows into its own tensor memory, and the MMA (issued by the even CTA
// for both) has M = 256.  The token tile's N columns are split between the
// two CTAs' shared memory, N/2 each, so that each SM stages and reads half the
// token bytes of the single-CTA kernel per MAC; the L2 -> SM traffic per MAC
// drops the same way.  Each CTA's tensor memory holds the accumulators of its
// own 128 weight rows for all N tokens, and each CTA runs its own epilogue.
//
// Barriers (every CTA holds all of them; the even CTA's full_a and acc_empty
// collect the arrivals of both):
//   full_tma[s]   local TMA completion (token half + packed rows)
//   full_a[s2]    even CTA: 4 expander warps x 2 CTAs wrote A stage s2 and saw
//                 their TMA stage complete
//   mma_done[s]   both CTAs, multicast commit: the MMAs of the K step that used
//                 TMA stage s are done (frees the TMA stage, and two K steps
//                 later the A stage)
//   acc_full[b]   both CTAs, multicast commit: accumulator buffer b is final
//   acc_empty[b]  even CTA: 4 epilogue warps x 2 CTAs have drained buffer b
// ---------------------------------------------------------------------------
constexpr int kPairStages = 8;
constexpr int QH_BYTES = (BT / 2) * BK;  // largest token half tile

template <int FMT, int OUT>
__host__ __device__ constexpr size_t smem_bytes_pair()
{
    return 1024 + static_cast<size_t>(kPairStages) * (QH_BYTES + p_bytes<FMT>()) + 4 * stage_warp_bytes<OUT>() +
           8 * (2 * kPairStages + kAStages + 8);
}

__device__ __forceinline__ void tc_mma_i8_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the barrier at this shared-memory offset in both CTAs of the pair
// once the pair's MMAs issued so far are complete.
__device__ __forceinline__ void tc_commit_pair_both(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(smem_u32(bar)), "h"(static_cast<uint16_t>(0x3)) : "memory");
}

__device__ __forceinline__ void tc_commit_pair_self(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint32_t idesc_pair(int nt)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nt >> 3) << 17) |
           (static_cast<uint32_t>((2 * BW) >> 4) << 24);
}

template <int FMT, int OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_ts_pair_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_p,
                    const float *__restrict__ s_x, const float *__restrict__ s_w, int64_t M, int64_t N, int64_t K,
                    void *__restrict__ y, int64_t ldy, int vec_ok, int nt, int32_t *status)
{
    constexpr int PB = packed_row_kblock<FMT>();
    constexpr int P_BYTES = p_bytes<FMT>();
    constexpr int kShift = Fmt<FMT>::kShift;
    constexpr int S = kPairStages;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                      // S x 14 KB token halves, 1024-aligned
    uint8_t *sP = sQ + S * QH_BYTES;         // S x P_BYTES packed rows
    uint8_t *sStage = sP + S * P_BYTES;      // 4 x epilogue staging
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + 4 * stage_warp_bytes<OUT>());
    uint64_t *full_tma = bars;
    uint64_t *mma_done = bars + S;
    uint64_t *full_a = bars + 2 * S;
    uint64_t *acc_full = full_a + kAStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_full + 4;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(acc_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acc_full + 6);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < kAStages; ++s) mbar_init(&full_a[s], 8);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_p)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(const_cast<uint32_t *>(tmem_slot))), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Global memory is touched only after the previous kernel on the stream
    // has completed (programmatic dependent launch, see pdl_wait).
    pdl_wait();
    pdl_trigger();
    const uint32_t a_col0 = 2 * kDCols;

    const int64_t num_w = (N + 2 * BW - 1) / (2 * BW);  // 256-row weight tiles
    const int64_t num_t = (M + nt - 1) / nt;
    const int64_t num_tiles = num_w * num_t;
    const int64_t pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int nkb = static_cast<int>((K + BK - 1) / BK);
    const int half = nt / 2;
    const uint32_t qh_bytes = static_cast<uint32_t>(half) * BK;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int64_t tile = pair; tile < num_tiles && ok; tile += num_pairs) {
                const int w0 = static_cast<int>((tile % num_w) * 2 * BW + rank * BW);
                const int t0 = static_cast<int>((tile / num_w) * nt + rank * half);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % S;
                    if (!wait_bar(&mma_done[s], ((g / S) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full_tma[s], qh_bytes + P_BYTES);
                    tma_load_2d(sQ + s * QH_BYTES, &map_q, &full_tma[s], kb * BK, t0);
                    tma_load_2d(sP + s * P_BYTES, &map_p, &full_tma[s], kb * PB, w0);
                }
            }
            if (!ok) {
                for (uint32_t i = 0; i < static_cast<uint32_t>(S) && i < g; ++i) {
                    const uint32_t gi = g - 1 - i;
                    drain_bar(&full_tma[gi % S], (gi / S) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (even CTA) ----------------
        if (leader && lane == 0) {
            const uint32_t idesc = idesc_pair(nt);
            const uint64_t qdesc0 = sw128_desc(smem_u32(sQ));
            uint32_t g = 0;
            uint32_t t = 0;
            bool ok = true;
            for (int64_t tile = pair; tile < num_tiles && ok; tile += num_pairs, ++t) {
                const int b = t & 1;
                if (!wait_bar(&acc_empty[b], ((t >> 1) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * kDCols);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s1 = g % S, s2 = g % kAStages;
                    if (!wait_bar(&full_a[s2], (g / kAStages) & 1u, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t qdesc = qdesc0 + static_cast<uint64_t>((s1 * QH_BYTES) >> 4);
                    const uint32_t a_tmem = tmem_base + a_col0 + static_cast<uint32_t>(s2 * kACols);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        tc_mma_i8_ts_pair(d_tmem, a_tmem + kk * (UMMA_K / 4),
                                          qdesc + static_cast<uint64_t>(kk * (UMMA_K >> 4)), idesc,
                                          (kb | kk) != 0 ? 1u : 0u);
                    tc_commit_pair_both(&mma_done[s1]);
                }
                if (!ok) break;
                tc_commit_pair_both(&acc_full[b]);
            }
            tc_commit_pair_self(drain);
            drain_bar(drain, 0);
        }
    } else if (warp < 6) {
        // ---------------- expanders: packed -> own TMEM ----------------
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t p_base = smem_u32(sP);
        const uint32_t full_a_leader = map_to_peer(smem_u32(full_a), 0);
        uint32_t g = 0;
        bool ok = true;
        for (int64_t tile = pair; tile < num_tiles && ok; tile += num_pairs) {
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int s1 = g % S, s2 = g % kAStages;
                int ready = 0;
                if (lane == 0) ready = wait_bar(&full_tma[s1], (g / S) & 1u, abort_flag, status) ? 1 : 0;
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (!ready) { ok = false; break; }
                uint32_t w[32];
                expand_row<FMT>(p_base + s1 * P_BYTES + r * PB, w);
                if (lane == 0 && g >= static_cast<uint32_t>(kAStages)) {
                    const uint32_t gp = g - kAStages;
                    ready = wait_bar(&mma_done[gp % S], (gp / S) & 1u, abort_flag, status) ? 1 : 0;
                }
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (!ready) { ok = false; break; }
                tc_fence_after();
                tmem_st_32cols(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a_col0 +
                                   static_cast<uint32_t>(s2 * kACols), w);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(full_a_leader + static_cast<uint32_t>(s2 * 8));
            }
        }
    } else {
        // ---------------- epilogue: own 128 weight rows ----------------
        const int quarter = warp & 3;
        const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>((warp - 6) * stage_warp_bytes<OUT>());
        const uint32_t acc_empty_leader = map_to_peer(smem_u32(acc_empty), 0);
        uint32_t t = 0;
        for (int64_t tile = pair; tile < num_tiles; tile += num_pairs, ++t) {
            const int b = t & 1;
            int ready = 0;
            if (lane == 0) ready = wait_bar(&acc_full[b], (t >> 1) & 1u, abort_flag, status) ? 1 : 0;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            tc_fence_after();
            const int64_t n0 = (tile % num_w) * 2 * BW + rank * BW + quarter * 32;
            const int64_t t0 = (tile / num_w) * nt;
            const int64_t n = n0 + lane;
            const float sw = (n < N) ? s_w[FMT == kT2 ? 0 : n] : 0.0f;
#pragma unroll 1
            for (int cc = 0; cc < nt / 32; ++cc) {
                uint32_t v[32];
                tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(b * kDCols + cc * 32), v);
                const int64_t tc0 = t0 + cc * 32;
                if (tc0 < M && n0 < N)
                    store_chunk<OUT>(v, sw, s_x, kShift, y, ldy, tc0, M, n0, N, vec_ok != 0, stage, lane);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acc_empty_leader + static_cast<uint32_t>(b * 8));
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the pair's MMAs and remote arrivals are over
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

template <int FMT, int OUT>
lowbit_status launch_pair_t(const CUtensorMap &mq, const CUtensorMap &mp, const float *s_x, const float *s_w,
                            int64_t M, int64_t N, int64_t K, void *y, int64_t ldy, int vec_ok, int nt,
                            int32_t *status, cudaStream_t st)
{
    constexpr size_t smem = smem_bytes_pair<FMT, OUT>();
    static_assert(smem <= 232448, "shared memory budget");
    static PerDevice max_pairs;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    // Pairs that can be resident at once (the GPCs decide how many SM pairs
    // exist), found with the shared-memory attribute set on the first launch
    // on each device; the persistent grid never exceeds it.
    const int resident = max_pairs.get(dev, [&] {
        if (cudaFuncSetAttribute(gemm_ts_pair_kernel<FMT, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * static_cast<unsigned>(device_sm_count() / 2));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        int n = 0;
        return cudaOccupancyMaxActiveClusters(&n, gemm_ts_pair_kernel<FMT, OUT>, &cfg) == cudaSuccess ? n : 0;
    });
    if (resident <= 0) return LOWBIT_ERR_CUDA;
    const int64_t tiles = ((N + 2 * BW - 1) / (2 * BW)) * ((M + nt - 1) / nt);
    const int64_t pairs = tiles < resident ? tiles : resident;
    return launch_pdl(gemm_ts_pair_kernel<FMT, OUT>, dim3(static_cast<unsigned>(2 * pairs)), dim3(kThreads), smem,
                      st, 0, mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, status);
}

template <int FMT>
lowbit_status launch_pair_fmt(const CUtensorMap &mq, const CUtensorMap &mp, const float *s_x, const float *s_w,
                              int64_t M, int64_t N, int64_t K, void *y, lowbit_dtype ydt, int64_t ldy, int vec_ok,
                              int nt, int32_t *status, cudaStream_t st)
{
    if (ydt == LOWBIT_F32)
        return launch_pair_t<FMT, LOWBIT_F32>(mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, status, st);
    if (ydt == LOWBIT_BF16)
        return launch_pair_t<FMT, LOWBIT_BF16>(mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, status, st);
    return launch_pair_t<FMT, LOWBIT_I32>(mq, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, nt, status, st);
}

}  // namespace ts

// Token tile: 224 for many tokens, else M rounded up to a multiple of 32.
lowbit_status gemm_ts_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                             const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                             lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                             int32_t *status, cudaStream_t st)
{
    using namespace ts;
    const int nt = M >= BT ? BT : static_cast<int>((M + 31) / 32 * 32);
    CUtensorMap mq, mp;
    if (!make_map_2d(&mq, q, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ldq), BK,
                     static_cast<uint32_t>(nt), CU_TENSOR_MAP_SWIZZLE_128B))
        return LOWBIT_ERR_CUDA;
    const uint32_t pb = f == LOWBIT_TERNARY2 ? packed_row_kblock<kT2>()
                        : f == LOWBIT_BINARY1 ? packed_row_kblock<kB1>()
                                              : packed_row_kblock<kI4>();
    if (!make_map_2d(&mp, packed, static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(N),
                     static_cast<uint64_t>(ldp), pb, BW, CU_TENSOR_MAP_SWIZZLE_NONE))
        return LOWBIT_ERR_CUDA;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    const int vec_ok = ((reinterpret_cast<uintptr_t>(y) & 15u) == 0 && (ldy * esz) % 16 == 0) ? 1 : 0;
    if (f == LOWBIT_TERNARY2) return launch_fmt<kT2>(mq, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, nt, prefetch, status, st);
    if (f == LOWBIT_BINARY1) return launch_fmt<kB1>(mq, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, nt, prefetch, status, st);
    return launch_fmt<kI4>(mq, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, nt, prefetch, status, st);
}

}  // namespace lowbit

namespace lowbit {
// SM-pair variant: token tile as above (224, or M rounded up to 32), each CTA
// of the pair staging half of it.
lowbit_status gemm_ts_pair_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                                  const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                                  lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy,
                                  int32_t *status, cudaStream_t st)
{
    using namespace ts;
    const int nt = M >= BT ? BT : static_cast<int>((M + 31) / 32 * 32);
    CUtensorMap mq, mp;
    if (!make_map_2d(&mq, q, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ldq), BK,
                     static_cast<uint32_t>(nt / 2), CU_TENSOR_MAP_SWIZZLE_128B))
        return LOWBIT_ERR_CUDA;
    const uint32_t pb = f == LOWBIT_TERNARY2 ? packed_row_kblock<kT2>()
                        : f == LOWBIT_BINARY1 ? packed_row_kblock<kB1>()
                                              : packed_row_kblock<kI4>();
    if (!make_map_2d(&mp, packed, static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(N),
                     static_cast<uint64_t>(ldp), pb, BW, CU_TENSOR_MAP_SWIZZLE_NONE))
        return LOWBIT_ERR_CUDA;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    const int vec_ok = ((reinterpret_cast<uintptr_t>(y) & 15u) == 0 && (ldy * esz) % 16 == 0) ? 1 : 0;
    if (f == LOWBIT_TERNARY2)
        return launch_pair_fmt<kT2>(mq, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, nt, status, st);
    if (f == LOWBIT_BINARY1)
        return launch_pair_fmt<kB1>(mq, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, nt, status, st);
    return launch_pair_fmt<kI4>(mq, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, nt, status, st);
}
}  // namespace lowbit

namespace lowbit {
// This file's copy of the pipeline wait bound (see lowbit_set_wait_limit).
lowbit_status set_wait_limit_gemm_ts(long long cycles) { return tc::set_wait_limit_here(cycles); }
}  // namespace lowbit
