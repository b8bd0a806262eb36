// gemm_sm100.cu -- tensor-core GEMM for many tokens (prefill), sm_100a.
//
// "M8.8 - Native Binary and Ternary Transformers" 0x09B: prefill has a large
// token dimension and is a dense contraction, so the integer dot runs on the
// 5th-generation tensor cores (tcgen05.mma kind::i8, s8 x s8 -> s32 in tensor
// memory).  0x09A: unpacking to bytes and calling a generic GEMM would not
// execute the intended operator, so the kernel consumes the packed artifact
// directly: packed weight tiles arrive in shared memory by TMA and are
// expanded there, tile by tile, into the int8 operand the MMA reads; the
// unpacked matrix never exists in global memory.
//
// CTA tile 128 tokens x 256 output features, K step 128.  Warp roles:
//   warp 0      TMA producer: activation tile (128x128 int8, 128B swizzle)
//               and packed weight tile (256 rows x 128 codes) per stage;
//   warp 1      TMEM allocation and the MMA issuer (one thread);
//   warps 2-5   expanders: packed codes -> int8 (c << S) in the UMMA
//               K-major 128B-swizzled layout;
//   warps 6-9   epilogue: tcgen05.ld of the s32 accumulators, acc >> S,
//               y = float(acc) * (s_w * s_x), fp32 / bf16 / int32 stores.
// Accumulators are double-buffered in tensor memory (2 x 256 columns) so the
// epilogue of one tile overlaps the MMAs of the next; CTAs are persistent.
// Every mbarrier wait is bounded in time; on expiry the CTA records
// LOWBIT_ERR_TIMEOUT, drains its copies and MMAs, frees tensor memory and
// returns.
#include "tc_common.cuh"
#include <atomic>

namespace lowbit {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int A_BYTES = BM * BK;
constexpr int E_BYTES = BN * BK;
constexpr int kThreads = 320;
constexpr int kExpThreads = 128;
constexpr uint32_t kTmemCols = 512;

template <int FMT> __host__ __device__ constexpr int packed_bytes_per_kblock() { return BK * Fmt<FMT>::kBits / 8; }

// How the shared-memory GEMM covers a problem whose 128 x 256 output tiles
// leave most SMs idle: K split over a cluster of c CTAs (1..8) and output
// tiles tbn = 256 or 128 features wide.
struct SplitPlan {
    int tbn;
    int c;
};

// Pipeline buffers of the split-K kernel (TMA and expansion rings), which
// hold the partial slices during the reduction: c * ceil(tbn/32 / c) slots
// of 16 KB must fit.
inline int64_t splitk_region_bytes(int stages, int tbn, int packed_bytes_per_kb)
{
    return static_cast<int64_t>(stages) * (BM * BK + tbn * packed_bytes_per_kb) + 2LL * tbn * BK;
}

// The split: 256-feature tiles and the largest cluster c in {2, 4, 8} with
// tiles * c <= SMs and at least 2 K blocks per split, considered when a
// factor 2 fits the SMs; otherwise {256, 1}, the unsplit kernel.  (The kernel
// template also takes 128-feature tiles and any c up to 8, whose reduction
// divides the columns unevenly; on the decode shapes those measured slower
// than this rule: 9728 -> 2560 at 128 tokens took 25.9 us as 20 tiles x 7 against
// 18 us as 10 x 8, and 2560 -> 9728 took 14.9 us as 38 x 3 against 14.2 us as
// 38 x 2, so the planner keeps to the even splits.)
inline SplitPlan splitk_plan(int64_t M, int64_t N, int64_t K, int64_t sms, int stages, int pb)
{
    const int64_t m_tiles = (M + BM - 1) / BM;
    const int64_t nkb = (K + BK - 1) / BK;
    const int64_t tiles = m_tiles * ((N + BN - 1) / BN);
    SplitPlan best{BN, 1};
    if (tiles * 2 > sms || nkb < 4) return best;
    for (int c : {2, 4, 8}) {
        if (tiles * c > sms || nkb < 2 * c) continue;
        if (static_cast<int64_t>(c) * ((BN / 32 + c - 1) / c) * 16 * 1024 > splitk_region_bytes(stages, BN, pb))
            continue;
        best = SplitPlan{BN, c};
    }
    return best;
}

// Ring depths: TMA stages (activation tile + packed tile) and expanded-tile
// stages, chosen to fit 227 KB of shared memory with the epilogue staging.
template <int FMT> __host__ __device__ constexpr int tma_stages() { return FMT == kI4 ? 4 : (FMT == kT2 ? 5 : 6); }
constexpr int kExpStages = 2;
// An expansion stage is freed by the MMA-completion barrier of the TMA stage
// its K step used, so there must be more TMA stages than expansion stages.
static_assert(kExpStages < 4, "fewer expansion stages than TMA stages (4 to 6)");
// Epilogue staging: per epilogue warp, 32 rows of one 32-column chunk, rows
// padded by 16 bytes so the row-wise writes and the column-wise reads are
// free of bank conflicts.
template <int OUT> __host__ __device__ constexpr int stage_row_bytes() { return OUT == LOWBIT_BF16 ? 80 : 144; }
template <int OUT> __host__ __device__ constexpr int stage_warp_bytes() { return 32 * stage_row_bytes<OUT>(); }

// Instruction descriptor: s32 accumulate, s8 x s8, both K-major, M=128, N=n.
__host__ __device__ constexpr uint32_t idesc_m128(int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(BM >> 4) << 24);
}
constexpr uint32_t kIdesc = idesc_m128(BN);

// ---------------------------------------------------------------------------
// Expansion of one stage: ROWS (256, or 128 per CTA of a pair) rows x 128 codes.  Each thread loads 16 bytes of
// packed codes at a time (ld.shared.v4) and writes whole 16-code chunks of the
// int8 tile (st.shared.v4); chunk c of row r goes to r*128 + ((c ^ (r%8))*16),
// the 128B-swizzle pattern the TMA uses for the activation tile.  Within every
// group of 8 lanes the loads cover 128 contiguous bytes and the stores hit 8
// distinct 16-byte bank groups, so neither conflicts.
// ---------------------------------------------------------------------------
template <int FMT, int ROWS = BN>
__device__ __forceinline__ void expand_stage(uint32_t P, uint32_t E, int et)
{
    if constexpr (FMT == kT2) {
        // 32 packed bytes per row: item = (row, half), half = 4 chunks.
#pragma unroll
        for (int j = 0; j < (ROWS * 2) / kExpThreads; ++j) {
            const int i = et + kExpThreads * j;
            const int r = i >> 1, h = i & 1;
            const uint4 w = lds128(P + r * 32 + h * 16);
            const uint32_t rowE = E + r * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t wk = (&w.x)[k];
                const int c = 4 * h + k;
                sts128(rowE + ((c ^ (r & 7)) << 4),
                       make_uint4(t2_expand(wk, 0), t2_expand(wk, 1), t2_expand(wk, 2), t2_expand(wk, 3)));
            }
        }
    } else if constexpr (FMT == kI4) {
        // 64 packed bytes per row: item = (row, quarter), quarter = 2 chunks.
#pragma unroll
        for (int j = 0; j < (ROWS * 4) / kExpThreads; ++j) {
            const int i = et + kExpThreads * j;
            const int r = i >> 2, qd = i & 3;
            const uint4 w = lds128(P + r * 64 + qd * 16);
            const uint32_t rowE = E + r * 128;
            sts128(rowE + (((2 * qd) ^ (r & 7)) << 4),
                   make_uint4(i4_expand(w.x, 0), i4_expand(w.x, 1), i4_expand(w.y, 0), i4_expand(w.y, 1)));
            sts128(rowE + (((2 * qd + 1) ^ (r & 7)) << 4),
                   make_uint4(i4_expand(w.z, 0), i4_expand(w.z, 1), i4_expand(w.w, 0), i4_expand(w.w, 1)));
        }
    } else {
        // 16 packed bytes per row: item = row, 8 chunks of 16 codes (16 bits).
#pragma unroll
        for (int j = 0; j < ROWS / kExpThreads; ++j) {
            const int r = et + kExpThreads * j;
            const uint4 w = lds128(P + r * 16);
            const uint32_t rowE = E + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t h = (&w.x)[c >> 1] >> (16 * (c & 1));
                sts128(rowE + ((c ^ (r & 7)) << 4),
                       make_uint4(b1_expand_nibble(h & 0xFu), b1_expand_nibble((h >> 4) & 0xFu),
                                  b1_expand_nibble((h >> 8) & 0xFu), b1_expand_nibble((h >> 12) & 0xFu)));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Epilogue for one 32-column chunk of one warp's 32 rows.
// v[i] is the accumulator of (row = this lane, column nc + i).
// ---------------------------------------------------------------------------
template <int OUT>
__device__ __forceinline__ uint32_t out_word(const uint32_t (&v)[32], const float (&sw)[32], float sx, int shift,
                                             int j)
{
    if constexpr (OUT == LOWBIT_I32) {
        return static_cast<uint32_t>(static_cast<int32_t>(v[j]) >> shift);
    } else if constexpr (OUT == LOWBIT_F32) {
        return __float_as_uint(rescale(static_cast<int32_t>(v[j]) >> shift, sw[j], sx));
    } else {
        const float a = rescale(static_cast<int32_t>(v[2 * j]) >> shift, sw[2 * j], sx);
        const float b = rescale(static_cast<int32_t>(v[2 * j + 1]) >> shift, sw[2 * j + 1], sx);
        const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t *>(&p);
    }
}

template <int OUT>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&v)[32], const float (&sw)[32], float sx, int shift,
                                               void *__restrict__ y, int64_t ldy, int64_t row0, int64_t M,
                                               int64_t nc, int64_t N, bool vec_ok, uint32_t stage, int lane)
{
    constexpr int kWords = OUT == LOWBIT_BF16 ? 16 : 32;   // 32-bit words per row of the chunk
    constexpr int kEsz = OUT == LOWBIT_BF16 ? 2 : 4;
    constexpr int RS = stage_row_bytes<OUT>();
    const int64_t row = row0 + lane;
    if (vec_ok && nc + 32 <= N) {
        // rows -> staging (row-wise), then staging -> global (column pieces)
#pragma unroll
        for (int p = 0; p < kWords / 4; ++p)
            sts128(stage + lane * RS + p * 16,
                   make_uint4(out_word<OUT>(v, sw, sx, shift, 4 * p), out_word<OUT>(v, sw, sx, shift, 4 * p + 1),
                              out_word<OUT>(v, sw, sx, shift, 4 * p + 2), out_word<OUT>(v, sw, sx, shift, 4 * p + 3)));
        __syncwarp();
        constexpr int kPieces = kWords / 4;        // 16-byte pieces per row
        constexpr int kRowsPerPass = 32 / kPieces;
#pragma unroll
        for (int pass = 0; pass < kPieces; ++pass) {
            const int r = pass * kRowsPerPass + lane / kPieces;
            const int piece = lane % kPieces;
            const uint4 val = lds128(stage + r * RS + piece * 16);
            if (row0 + r < M) {
                char *dst = static_cast<char *>(y) + ((row0 + r) * ldy + nc) * kEsz + piece * 16;
                *reinterpret_cast<uint4 *>(dst) = val;
            }
        }
        __syncwarp();
    } else if (row < M) {
        // ragged column tail or unaligned output: element stores
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            if (nc + i < N) {
                const int32_t a = static_cast<int32_t>(v[i]) >> shift;
                if constexpr (OUT == LOWBIT_I32) {
                    static_cast<int32_t *>(y)[row * ldy + nc + i] = a;
                } else if constexpr (OUT == LOWBIT_F32) {
                    static_cast<float *>(y)[row * ldy + nc + i] = rescale(a, sw[i], sx);
                } else {
                    static_cast<__nv_bfloat16 *>(y)[row * ldy + nc + i] = __float2bfloat16_rn(rescale(a, sw[i], sx));
                }
            }
        }
    }
}

template <int FMT, int OUT, int TBN>
__host__ __device__ constexpr size_t splitk_smem_bytes()
{
    return 1024 + static_cast<size_t>(tma_stages<FMT>()) * (A_BYTES + TBN * packed_bytes_per_kblock<FMT>()) +
           static_cast<size_t>(kExpStages) * TBN * BK + 4 * stage_warp_bytes<OUT>() +
           8 * (2 * tma_stages<FMT>() + 2 * kExpStages + 8);
}

template <int FMT, int OUT>
__host__ __device__ constexpr size_t smem_bytes()
{
    return 1024 + static_cast<size_t>(tma_stages<FMT>()) * (A_BYTES + BN * packed_bytes_per_kblock<FMT>()) +
           static_cast<size_t>(kExpStages) * E_BYTES + 4 * stage_warp_bytes<OUT>() +
           8 * (2 * tma_stages<FMT>() + 2 * kExpStages + 8);
}

template <int FMT, int OUT>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_p,
            const float *__restrict__ s_x, const float *__restrict__ s_w, int64_t M, int64_t N, int64_t K,
            void *__restrict__ y, int64_t ldy, int vec_ok, int prefetch, int32_t *status)
{
    constexpr int ST = tma_stages<FMT>();
    constexpr int SE = kExpStages;
    constexpr int PB = packed_bytes_per_kblock<FMT>();
    constexpr int P_BYTES = BN * PB;
    constexpr int kShift = Fmt<FMT>::kShift;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;                        // ST x 16 KB, 1024-aligned
    uint8_t *sE = sA + ST * A_BYTES;           // SE x 32 KB, 1024-aligned
    uint8_t *sP = sE + SE * E_BYTES;           // ST x P_BYTES
    uint8_t *sStage = sP + ST * P_BYTES;       // 4 x epilogue staging
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + 4 * stage_warp_bytes<OUT>());
    uint64_t *full_tma = bars;
    uint64_t *mma_done = bars + ST;   // MMAs of the step that used TMA stage s are complete
    uint64_t *full_exp = bars + 2 * ST;
    uint64_t *empty_exp = bars + 2 * ST + SE;
    uint64_t *acc_full = bars + 2 * ST + 2 * SE;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_full + 4;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(acc_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acc_full + 6);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < SE; ++s) {
            mbar_init(&full_exp[s], kExpThreads);
            mbar_init(&empty_exp[s], 1);  // unused: the expansion stage is freed by mma_done
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
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

    const int64_t num_m = (M + BM - 1) / BM;
    const int64_t num_n = (N + BN - 1) / BN;
    const int64_t num_tiles = num_m * num_n;
    const int nkb = static_cast<int>((K + BK - 1) / BK);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t g = 0;  // global k-block counter
            bool ok = true;
            uint32_t npre = 0;  // stages whose weight half was started before the wait
            if (prefetch != 0) {
                if (blockIdx.x < num_tiles) {
                    const int n0 = static_cast<int>((blockIdx.x / num_m) * BN);
                    npre = static_cast<uint32_t>(nkb < ST ? nkb : ST);
                    for (uint32_t i = 0; i < npre; ++i) {
                        mbar_arrive_expect_tx(&full_tma[i], A_BYTES + P_BYTES);
                        tma_load_2d(sP + i * P_BYTES, &map_p, &full_tma[i], static_cast<int>(i) * PB, n0);
                    }
                }
                pdl_wait();
            }
            for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = static_cast<int>((tile % num_m) * BM);
                const int n0 = static_cast<int>((tile / num_m) * BN);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s = g % ST;
                    const uint32_t ph = (g / ST) & 1u;
                    if (g < npre) {
                        tma_load_2d(sA + s * A_BYTES, &map_a, &full_tma[s], kb * BK, m0);
                        continue;
                    }
                    if (!wait_bar(&mma_done[s], ph ^ 1u, abort_flag, status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full_tma[s], A_BYTES + P_BYTES);
                    tma_load_2d(sA + s * A_BYTES, &map_a, &full_tma[s], kb * BK, m0);
                    tma_load_2d(sP + s * P_BYTES, &map_p, &full_tma[s], kb * PB, n0);
                }
            }
            if (!ok) {
                // Let copies already issued land before the CTA leaves.
                for (uint32_t i = 0; i < ST && i < g; ++i) {
                    const uint32_t gi = g - 1 - i;
                    drain_bar(&full_tma[gi % ST], (gi / ST) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            uint32_t g = 0;
            uint32_t t = 0;
            bool ok = true;
            for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
                const int b = t & 1;
                const uint32_t aph = (t >> 1) & 1u;
                if (!wait_bar(&acc_empty[b], aph ^ 1u, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * BN);
                for (int kb = 0; kb < nkb; ++kb, ++g) {
                    const int s1 = g % ST, s2 = g % SE;
                    // the expanders saw the TMA stage complete before arriving on
                    // full_exp, so one wait orders the MMA after both
                    if (!wait_bar(&full_exp[s2], (g / SE) & 1u, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + s1 * A_BYTES);
                    const uint32_t e_addr = smem_u32(sE + s2 * E_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        tc_mma_i8(d_tmem, sw128_desc(a_addr + kk * UMMA_K), sw128_desc(e_addr + kk * UMMA_K),
                                  kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    tc_commit(&mma_done[s1]);
                }
                if (!ok) break;
                tc_commit(&acc_full[b]);
            }
            // All MMAs this thread issued are complete once `drain` flips.
            tc_commit(drain);
            drain_bar(drain, 0);
        }
    } else if (warp < 6) {
        // ---------------- expanders ----------------
        const int et = threadIdx.x - 64;
        const uint32_t p_base = smem_u32(sP);
        const uint32_t e_base = smem_u32(sE);
        uint32_t g = 0;
        bool ok = true;
        for (int64_t tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < nkb; ++kb, ++g) {
                const int s1 = g % ST, s2 = g % SE;
                // expansion stage s2 is free once the MMAs of step g - SE are
                // complete (mma_done of that step's TMA stage)
                if (!wait_bar(&full_tma[s1], (g / ST) & 1u, abort_flag, status)) { ok = false; break; }
                if (g >= static_cast<uint32_t>(SE)) {
                    const uint32_t gp = g - SE;
                    if (!wait_bar(&mma_done[gp % ST], (gp / ST) & 1u, abort_flag, status)) { ok = false; break; }
                }
                expand_stage<FMT>(p_base + s1 * P_BYTES, e_base + s2 * E_BYTES, et);
                // Each writer orders its generic-proxy stores before the
                // tensor core's async-proxy reads, then arrives.
                fence_proxy_async_smem();
                mbar_arrive(&full_exp[s2]);
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
        const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>((warp - 6) * stage_warp_bytes<OUT>());
        const float sw_tensor = (FMT == kT2) ? s_w[0] : 0.0f;
        uint32_t t = 0;
        for (int64_t tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
            const int b = t & 1;
            const uint32_t aph = (t >> 1) & 1u;
            // One lane waits and the warp follows its verdict, so the
            // .sync.aligned TMEM loads below always run converged.
            int ready = 0;
            if (lane == 0) ready = wait_bar(&acc_full[b], aph, abort_flag, status) ? 1 : 0;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            tc_fence_after();
            const int64_t m0 = (tile % num_m) * BM;
            const int64_t n0 = (tile / num_m) * BN;
            const int64_t row0 = m0 + quarter * 32;
            const float sx = (row0 + lane < M) ? ld_act_f32(s_x + row0 + lane) : 0.0f;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                const int64_t nc = n0 + cc * 32;
                uint32_t v[32];
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       static_cast<uint32_t>(b * BN + cc * 32);
                tmem_ld_32cols(taddr, v);
                if (nc < N) {
                    float sw[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        sw[i] = (FMT == kT2) ? sw_tensor : ((nc + i < N) ? __ldg(s_w + nc + i) : 0.0f);
                    epilogue_chunk<OUT>(v, sw, sx, kShift, y, ldy, row0, M, nc, N, vec_ok != 0, stage, lane);
                }
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

// ---------------------------------------------------------------------------
// Split-K over a thread-block cluster, for problems with fewer output tiles
// than SMs (few tokens, or few output features).  Tiles are 128 tokens x TBN
// features (256 or 128).  The C CTAs of a cluster (1..8) share one output
// tile; CTA s accumulates k-blocks [s*nkb/C, (s+1)*nkb/C) into tensor memory.
// The partial tiles are then reduce-scattered through distributed shared
// memory: the tile's 32-column chunks are divided among the CTAs (CTA j owns
// chunks [j*NCH/C, (j+1)*NCH/C), NCH = TBN/32), every CTA sends each owner
// its partial sums of the owner's chunks, and each owner adds them (int32
// addition is exact, so the result equals the unsplit accumulation bit for
// bit) and runs the epilogue for its chunks.  No global scratch memory is used.
// ---------------------------------------------------------------------------
template <int FMT, int OUT, int TBN = BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_splitk_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_p,
                   const float *__restrict__ s_x, const float *__restrict__ s_w, int64_t M, int64_t N, int64_t K,
                   void *__restrict__ y, int64_t ldy, int vec_ok, int C, int prefetch, int32_t *status)
{
    constexpr int ST = tma_stages<FMT>();
    constexpr int SE = kExpStages;
    constexpr int PB = packed_bytes_per_kblock<FMT>();
    constexpr int P_BYTES = TBN * PB;
    constexpr int TE_BYTES = TBN * BK;
    constexpr int kShift = Fmt<FMT>::kShift;
    constexpr uint32_t kTileIdesc = idesc_m128(TBN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;
    uint8_t *sE = sA + ST * A_BYTES;
    uint8_t *sP = sE + SE * TE_BYTES;
    uint8_t *sStage = sP + ST * P_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + 4 * stage_warp_bytes<OUT>());
    uint64_t *full_tma = bars;
    uint64_t *mma_done = bars + ST;   // MMAs of the step that used TMA stage s are complete
    uint64_t *full_exp = bars + 2 * ST;
    uint64_t *empty_exp = bars + 2 * ST + SE;
    uint64_t *acc_full = bars + 2 * ST + 2 * SE;
    uint64_t *drain = acc_full + 4;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(acc_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acc_full + 6);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t srank = cluster_rank();

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < SE; ++s) {
            mbar_init(&full_exp[s], kExpThreads);
            mbar_init(&empty_exp[s], 1);  // unused: the expansion stage is freed by mma_done
        }
        mbar_init(&acc_full[0], 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
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

    const int64_t num_m = (M + BM - 1) / BM;
    const int64_t tile = blockIdx.x / C;
    const int m0 = static_cast<int>((tile % num_m) * BM);
    const int n0 = static_cast<int>((tile / num_m) * TBN);
    const int nkb = static_cast<int>((K + BK - 1) / BK);
    const int kb_begin = static_cast<int>((static_cast<int64_t>(srank) * nkb) / C);
    const int kb_end = static_cast<int>((static_cast<int64_t>(srank + 1) * nkb) / C);

    if (warp == 0) {
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            uint32_t npre = 0;  // stages whose weight half was started before the wait
            if (prefetch != 0) {
                const int nloc = kb_end - kb_begin;
                npre = static_cast<uint32_t>(nloc < ST ? nloc : ST);
                for (uint32_t i = 0; i < npre; ++i) {
                    mbar_arrive_expect_tx(&full_tma[i], A_BYTES + P_BYTES);
                    tma_load_2d(sP + i * P_BYTES, &map_p, &full_tma[i], (kb_begin + static_cast<int>(i)) * PB, n0);
                }
                pdl_wait();
            }
            for (int kb = kb_begin; kb < kb_end; ++kb, ++g) {
                const int s = g % ST;
                if (g < npre) {
                    tma_load_2d(sA + s * A_BYTES, &map_a, &full_tma[s], kb * BK, m0);
                    continue;
                }
                if (!wait_bar(&mma_done[s], ((g / ST) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                mbar_arrive_expect_tx(&full_tma[s], A_BYTES + P_BYTES);
                tma_load_2d(sA + s * A_BYTES, &map_a, &full_tma[s], kb * BK, m0);
                tma_load_2d(sP + s * P_BYTES, &map_p, &full_tma[s], kb * PB, n0);
            }
            if (!ok) {
                for (uint32_t i = 0; i < ST && i < g; ++i) {
                    const uint32_t gi = g - 1 - i;
                    drain_bar(&full_tma[gi % ST], (gi / ST) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            for (int kb = kb_begin; kb < kb_end; ++kb, ++g) {
                const int s1 = g % ST, s2 = g % SE;
                if (!wait_bar(&full_exp[s2], (g / SE) & 1u, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t a_addr = smem_u32(sA + s1 * A_BYTES);
                const uint32_t e_addr = smem_u32(sE + s2 * TE_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / UMMA_K; ++kk)
                    tc_mma_i8(tmem_base, sw128_desc(a_addr + kk * UMMA_K), sw128_desc(e_addr + kk * UMMA_K),
                              kTileIdesc, (g | kk) != 0 ? 1u : 0u);
                tc_commit(&mma_done[s1]);
            }
            if (ok) tc_commit(&acc_full[0]);
            tc_commit(drain);
            drain_bar(drain, 0);
        }
    } else if (warp < 6) {
        const int et = threadIdx.x - 64;
        const uint32_t p_base = smem_u32(sP);
        const uint32_t e_base = smem_u32(sE);
        uint32_t g = 0;
        for (int kb = kb_begin; kb < kb_end; ++kb, ++g) {
            const int s1 = g % ST, s2 = g % SE;
            if (!wait_bar(&full_tma[s1], (g / ST) & 1u, abort_flag, status)) break;
            if (g >= static_cast<uint32_t>(SE)) {
                const uint32_t gp = g - SE;
                if (!wait_bar(&mma_done[gp % ST], (gp / ST) & 1u, abort_flag, status)) break;
            }
            expand_stage<FMT, TBN>(p_base + s1 * P_BYTES, e_base + s2 * TE_BYTES, et);
            fence_proxy_async_smem();
            mbar_arrive(&full_exp[s2]);
        }
    }
    int ready = 1;
    if (warp >= 6) {
        int r = 0;
        if (lane == 0) r = wait_bar(&acc_full[0], 0, abort_flag, status) ? 1 : 0;
        ready = __shfl_sync(0xffffffffu, r, 0);
        tc_fence_after();
    }
    __syncwarp();

    // Every CTA of the cluster is done with its pipeline buffers: from here
    // they hold the received partial tiles, piece-major: 16-byte piece p
    // (4 columns) of the owner's lc-th chunk from source rank s sits at
    // ((s * MAXC + lc) * 8 + p) * BM + r, so that the 32 lanes (rows) of one
    // remote store instruction write 512 contiguous bytes.
    constexpr int NCH = TBN / 32;               // 32-column chunks of a tile
    const int MAXC = (NCH + C - 1) / C;         // most chunks one CTA owns
    auto chunk_begin = [&](int j) { return j * NCH / C; };
    const uint32_t recv = smem_u32(sA);
    cluster_sync_all();
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const int64_t row = m0 + row_in_tile;
    if (warp >= 6) {
        for (int j = 0; j < C; ++j) {
            for (int cc = chunk_begin(j); cc < chunk_begin(j + 1); ++cc) {
                uint32_t v[32];
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       static_cast<uint32_t>(cc * 32);
                tmem_ld_32cols(taddr, v);
                if (!ready) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0;
                }
                if (row < M) {
                    const int lc = cc - chunk_begin(j);
                    const uint32_t dst = map_to_peer(
                        recv + static_cast<uint32_t>(((static_cast<int>(srank) * MAXC + lc) * 8 * BM + row_in_tile) * 16),
                        static_cast<uint32_t>(j));
#pragma unroll
                    for (int p = 0; p < 8; ++p)
                        st_cluster128(dst + static_cast<uint32_t>(p * BM * 16), v[4 * p], v[4 * p + 1], v[4 * p + 2],
                                      v[4 * p + 3]);
                }
            }
        }
    }
    cluster_sync_all();
    if (warp >= 6) {
        const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>((warp - 6) * stage_warp_bytes<OUT>());
        const float sx = row < M ? ld_act_f32(s_x + row) : 0.0f;
        const float sw_tensor = (FMT == kT2) ? s_w[0] : 0.0f;
        const int own0 = chunk_begin(static_cast<int>(srank));
        const int own = chunk_begin(static_cast<int>(srank) + 1) - own0;
        for (int lc = 0; lc < own; ++lc) {
            uint32_t v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0;
            if (row < M) {
                for (int s = 0; s < C; ++s) {
                    const uint32_t src = recv + static_cast<uint32_t>(((s * MAXC + lc) * 8 * BM + row_in_tile) * 16);
#pragma unroll
                    for (int p = 0; p < 8; ++p) {
                        const uint4 a = lds128(src + static_cast<uint32_t>(p * BM * 16));
                        v[4 * p] += a.x;
                        v[4 * p + 1] += a.y;
                        v[4 * p + 2] += a.z;
                        v[4 * p + 3] += a.w;
                    }
                }
            }
            const int64_t nc = n0 + static_cast<int64_t>(own0 + lc) * 32;
            if (nc < N) {
                float sw[32];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    sw[i] = (FMT == kT2) ? sw_tensor : ((nc + i < N) ? __ldg(s_w + nc + i) : 0.0f);
                epilogue_chunk<OUT>(v, sw, sx, kShift, y, ldy, m0 + quarter * 32, M, nc, N, vec_ok != 0, stage, lane);
            }
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

// ---------------------------------------------------------------------------
// SM-pair variant (tcgen05 cta_group::2): a cluster of two CTAs computes a
// 256-token x 256-feature tile with M = 256 MMAs issued by the even CTA.  CTA r
// stages tokens m0 + 128r (the MMA's A rows it owns) and expands features
// n0 + 128r (its half of the B operand) into its own shared memory; each CTA's
// tensor memory holds its 128 tokens x all 256 features, and each CTA runs the
// epilogue for them.  Per SM and K step this stages half the expanded weights
// of the single-CTA kernel and issues no MMAs on the odd CTA.
//
// Barriers (all in both CTAs; the even CTA's full_exp and acc_empty collect
// the arrivals of both): full_tma[s] local TMA completion; full_exp[s2] 4
// expander warps x 2 CTAs wrote expansion stage s2 and saw their TMA stage
// complete; mma_done[s] (multicast commit) the MMAs of the K step that used
// TMA stage s are done; acc_full[b] (multicast commit) accumulator b is final;
// acc_empty[b] 4 epilogue warps x 2 CTAs drained accumulator b.
// ---------------------------------------------------------------------------
constexpr int PBM = 128;                      // tokens per CTA (the pair's MMA has M = 256)
constexpr int PBN = 128;                      // features expanded per CTA (the pair's N = 256)
constexpr int PE_BYTES = PBN * BK;
template <int FMT, int OUT> __host__ __device__ constexpr int pair_tma_stages() { return FMT == kI4 ? 7 : 8; }
template <int FMT, int OUT> __host__ __device__ constexpr int pair_exp_stages() { return kExpStages; }
// A pair CTA has EW epilogue warps (warps 6..): one per TMEM lane quarter
// (EW = 4), or two converting half of the columns each (EW = 8).  A warp's
// 32-column chunks run as one dependent chain, so EW = 8 halves a tile's
// epilogue; it pays where that epilogue is exposed (few tiles per pair) and
// costs where it overlaps the next tile's mainloop (measured, bf16 out, 74
// pairs: 9728 -> 2560 at M = 1024 34.3 -> 31.1 us, 2560 -> 9728 30.4 -> 28.4;
// at M = 8192 135.5 -> 139.1 and 143.7 -> 151.6).
template <int EW> __host__ __device__ constexpr int pair_threads() { return (6 + EW) * 32; }
constexpr uint32_t kPairIdesc = (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>((2 * PBN) >> 3) << 17) |
                                (static_cast<uint32_t>((2 * PBM) >> 4) << 24);

template <int FMT, int OUT, int EW = 4>
__host__ __device__ constexpr size_t pair_smem_bytes()
{
    return 1024 + static_cast<size_t>(pair_tma_stages<FMT, OUT>()) * (A_BYTES + PBN * packed_bytes_per_kblock<FMT>()) +
           static_cast<size_t>(pair_exp_stages<FMT, OUT>()) * PE_BYTES + static_cast<size_t>(EW) * stage_warp_bytes<OUT>() +
           8 * (2 * pair_tma_stages<FMT, OUT>() + pair_exp_stages<FMT, OUT>() + 8);
}

__device__ __forceinline__ void tc_mma_i8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

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

// ---------------------------------------------------------------------------
// Stream-K tail of the SM-pair GEMM.  The tiles run round by round (tile
// p + r P on pair p of P) while every pair has a whole tile to take; when the
// last round would be partial, the K blocks of the tiles left after the
// whole rounds (the partial round plus one whole round, or every tile when
// there are fewer tiles than pairs) are shared evenly: pair p takes the
// blocks [p W / P, (p + 1) W / P) of the W = tiles_left x nkb blocks laid out
// tile after tile.  A pair's range is one or more pieces of tiles; only the
// first piece can start inside a tile (kb0 > 0), and only the last can end
// inside one.  A piece that starts inside a tile stores its int32 partial
// tile in the workspace slot of its pair and publishes an epoch flag per
// epilogue warp (32 token rows).  The piece that starts the tile (kb0 = 0)
// and ends inside it is the pair's last; it waits (bounded) for the flags of
// the following pairs that hold the rest of the tile, adds their partial
// tiles (integer addition: the sum is the unsplit accumulation bit for bit)
// and runs the epilogue.  Those pairs start with their pieces, so the wait is
// short.  The workspace is shared by all launches on the device, so the
// split runs only for callers that exclude concurrent SM-pair GEMMs
// (LOWBIT_LINEAR_EXCLUSIVE).
// ---------------------------------------------------------------------------
constexpr int kPairSkMinKb = 8;                           // K blocks of 128 per pair's share, at least
constexpr int kPairSkFixupKb = 12;                       // cost of the tail, in K blocks of MMA time
constexpr int kPairSkExtraKb = 11;                        // and of each partial tile after the first
constexpr int kPairWsSlots = 96;                          // partial tiles held at once (one per pair)
constexpr int kPairWsWords = 2 * PBM * 2 * PBN;  // one 256 x 256 int32 tile (both CTAs)
constexpr int kWsWarpVecs = 32 * 2 * PBN / 4;     // one epilogue warp's 32 rows x 256 int32, in uint4
__device__ uint4 g_pair_ws[kPairWsSlots][kPairWsWords / 4];
__device__ uint32_t g_pair_flag[kPairWsSlots][2][8];  // per pair (slot), CTA and epilogue warp
// One epoch per launch, shared by every instantiation of the kernel (they
// share the flags), so no launch can take another launch's flag for its own.
static std::atomic<uint32_t> g_pair_epoch{0};

// The schedule of a launch: P pairs, the first dp_tiles tiles in whole
// rounds (a multiple of P, or every tile), the rest shared by K block.  The
// shared tail is taken when its estimated time, in K blocks per pair plus
// kPairSkFixupKb, beats the whole-round schedule (ceil(tiles / P) rounds of
// nkb).  The fix-up estimate is measured: a partial tile's store, the
// finisher's staging and its longer epilogue, and the pieces' shorter
// pipelines cost about 12 K blocks of MMA time, and each further partial
// tile added from L2 about 11 more (9728 -> 2560 at M = 128, forced onto
// pairs: 10 K blocks per pair, up to 8 partial tiles per tile, 44 us against
// 19 on the split-K GEMM) (4B-class shapes, 74 pairs,
// bf16 out: 9728 -> 2560 at M = 8192, 4 rounds + 24 tiles of 76 blocks, 145.8
// -> 137.6 us; at M = 1024, 40 tiles of 76, 37.3 -> 33.1 us; 2560 -> 9728 at
// M = 8192, 16 rounds + 32 tiles of 20, 147.0 -> 150.8 us, so that shape keeps
// whole rounds: 300 + 29 + 12 >= 340).
inline void pair_plan(int64_t tiles, int64_t resident, int64_t nkb, int64_t &dp_tiles, int64_t &P_out)
{
    P_out = tiles < resident ? tiles : resident;
    dp_tiles = tiles;
    if (resident <= 0 || tiles <= 0 || resident > kPairWsSlots || tiles % resident == 0) return;
    const int64_t whole = (tiles + P_out - 1) / P_out * nkb;
    const int64_t rounds = tiles / resident;
    const int64_t dp = rounds > 0 ? (rounds - 1) * resident : 0;
    const int64_t W = (tiles - dp) * nkb;
    int64_t P = resident;
    if (rounds == 0 && W / P < kPairSkMinKb) P = W / kPairSkMinKb;
    if (P <= 1 || (rounds == 0 && P <= tiles)) return;
    // a tile is shared by up to ceil(nkb / share) + 1 pairs, so its finisher
    // adds up to ceil(nkb / share) partial tiles; after the first, which is
    // staged in shared memory, each costs about 8 L2 round trips
    const int64_t share = W / P > 0 ? W / P : 1;
    const int64_t partials = (nkb + share - 1) / share;
    const int64_t shared = dp / P * nkb + (W + P - 1) / P + kPairSkFixupKb +
                           kPairSkExtraKb * (partials > 1 ? partials - 1 : 0);
    if (shared >= whole) return;
    dp_tiles = dp;
    P_out = P;
}

// 16-byte copy global -> shared by this thread (L2 only), and the wait for
// all of the thread's copies.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// One unit of work of a pair: K blocks [kb0, kb1) of `tile`.  kb0 > 0: the
// unit's partial tile goes to the pair's workspace slot.  last >= 0: the
// unit starts the tile and ends inside it, and the partial tiles of pairs
// p + 1 .. last are added to it.
struct PairUnit {
    int64_t tile;
    int kb0, kb1, last;
};

// The units of pair p in order: the whole rounds (tiles p, p + P, ... below
// dp_tiles), then the pair's share of the tail.  The divisions run once, when
// the schedule is made, so a unit boundary costs the MMA issuer no more than a
// few integer operations.
struct PairSched {
    int64_t next_dp, dp_tiles, P, W;
    int64_t t, left;  // tail: current tile (from dp_tiles on), K blocks left
    int kb, nkb;      // first K block of the next tail piece

    __device__ __forceinline__ PairSched(int64_t p, int64_t P_, int64_t num_tiles, int nkb_, int64_t dp_tiles_)
        : next_dp(p), dp_tiles(dp_tiles_), P(P_), W(0), t(0), left(0), kb(0), nkb(nkb_)
    {
        if (dp_tiles < num_tiles) {
            W = (num_tiles - dp_tiles) * nkb;
            const int64_t s = p * W / P, e = (p + 1) * W / P;
            t = s / nkb;
            kb = static_cast<int>(s - t * nkb);
            left = e - s;
        }
    }

    // The next unit (false past the pair's last one).
    __device__ __forceinline__ bool next(PairUnit &u)
    {
        if (next_dp < dp_tiles) {
            u = PairUnit{next_dp, 0, nkb, -1};
            next_dp += P;
            return true;
        }
        if (left <= 0) return false;
        const int n = static_cast<int>(left < nkb - kb ? left : nkb - kb);
        u.tile = dp_tiles + t;
        u.kb0 = kb;
        u.kb1 = kb + n;
        // a piece that starts its tile and ends inside it: the pair holding
        // the tile's last K block is the max q with q W / P <= end - 1
        u.last = (kb == 0 && n < nkb) ? static_cast<int>(((t + 1) * nkb * P - 1) / W) : -1;
        left -= n;
        kb = 0;
        ++t;
        return true;
    }
};

// Waits (bounded by the pipeline wait limit) until flag == epoch, with
// acquire order for the reads that follow.  False on timeout (reported).
__device__ inline bool wait_flag(const uint32_t *flag, uint32_t epoch, volatile int *abort_flag, int32_t *status)
{
    const long long t0 = clock64();
    for (uint32_t i = 1;; ++i) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
        if (v == epoch) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - t0 > g_wait_limit_cycles) {
                *abort_flag = 1;
                report(status, LOWBIT_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// Runs f(v, cc) on the 32-column chunks c0 .. c0 + nch - 1 of this warp's
// accumulator rows in order.  (Keeping the next chunk's TMEM load in flight
// while the current one is stored measured no faster.)
template <typename F>
__device__ __forceinline__ void pair_chunks(uint32_t tacc, int c0, int nch, F &&f)
{
#pragma unroll 1
    for (int cc = c0; cc < c0 + nch; ++cc) {
        uint32_t v[32];
        tmem_ld_32cols(tacc + static_cast<uint32_t>(cc * 32), v);
        f(v, cc);
    }
}

template <int FMT, int OUT, int EW>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads<EW>(), 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_p,
                 const float *__restrict__ s_x, const float *__restrict__ s_w, int64_t M, int64_t N, int64_t K,
                 void *__restrict__ y, int64_t ldy, int vec_ok, int prefetch, int32_t *status, int64_t dp_tiles,
                 uint32_t epoch)
{
    constexpr int ST = pair_tma_stages<FMT, OUT>();
    constexpr int SE = pair_exp_stages<FMT, OUT>();
    constexpr int PB = packed_bytes_per_kblock<FMT>();
    constexpr int P_BYTES = PBN * PB;
    constexpr int kShift = Fmt<FMT>::kShift;
    static_assert(SE < ST, "an expansion stage is freed through the MMA barrier of an older TMA stage");
    static_assert(ST * A_BYTES + SE * PE_BYTES >= 4 * kWsWarpVecs * 16, "a partial tile is staged in the rings");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;                        // ST x 16 KB, 1024-aligned
    uint8_t *sE = sA + ST * A_BYTES;           // SE x 16 KB, 1024-aligned
    uint8_t *sP = sE + SE * PE_BYTES;          // ST x P_BYTES
    uint8_t *sStage = sP + ST * P_BYTES;       // 4 x epilogue staging
    uint64_t *bars = reinterpret_cast<uint64_t *>(sStage + EW * stage_warp_bytes<OUT>());
    uint64_t *full_tma = bars;
    uint64_t *mma_done = bars + ST;
    uint64_t *full_exp = bars + 2 * ST;
    uint64_t *acc_full = full_exp + SE;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_full + 4;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(acc_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(acc_full + 6);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < SE; ++s) mbar_init(&full_exp[s], 8);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * EW);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
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
    // has completed (programmatic dependent launch, see pdl_wait); with
    // prefetch the TMA thread starts the weight half of its first stages first.
    if (prefetch == 0 || threadIdx.x != 0) pdl_wait();
    pdl_trigger();

    const int64_t num_m = (M + 2 * PBM - 1) / (2 * PBM);
    const int64_t num_n = (N + 2 * PBN - 1) / (2 * PBN);
    const int64_t num_tiles = num_m * num_n;
    const int64_t pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int nkb = static_cast<int>((K + BK - 1) / BK);
    // Tile t covers tokens (t / num_n) and features (t % num_n): the pairs of
    // one round sweep the features of a few token tiles, so a round's
    // activation rows (the large operand) stay in L2 while the packed weights
    // (2 bits per code) are shared by all rounds.  (With the token tile
    // varying fastest, 9728->2560 at M = 8192 read the 80 MB of codes from
    // HBM about four times: 311 MB per launch in ncu.)

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            uint32_t g = 0;
            bool ok = true;
            uint32_t npre = 0;
            PairUnit u;
            PairSched sched(pair, num_pairs, num_tiles, nkb, dp_tiles);
            if (prefetch != 0) {
                PairSched first = sched;
                if (first.next(u)) {
                    const int n0 = static_cast<int>((u.tile % num_n) * 2 * PBN + rank * PBN);
                    const int nloc = u.kb1 - u.kb0;
                    npre = static_cast<uint32_t>(nloc < ST ? nloc : ST);
                    for (uint32_t i = 0; i < npre; ++i) {
                        mbar_arrive_expect_tx(&full_tma[i], A_BYTES + P_BYTES);
                        tma_load_2d(sP + i * P_BYTES, &map_p, &full_tma[i], (u.kb0 + static_cast<int>(i)) * PB, n0);
                    }
                }
                pdl_wait();
            }
            while (ok && sched.next(u)) {
                const int m0 = static_cast<int>((u.tile / num_n) * 2 * PBM + rank * PBM);
                const int n0 = static_cast<int>((u.tile % num_n) * 2 * PBN + rank * PBN);
                for (int kb = u.kb0; kb < u.kb1; ++kb, ++g) {
                    const int s = g % ST;
                    if (g < npre) {
                        tma_load_2d(sA + s * A_BYTES, &map_a, &full_tma[s], kb * BK, m0);
                        continue;
                    }
                    if (!wait_bar(&mma_done[s], ((g / ST) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full_tma[s], A_BYTES + P_BYTES);
                    tma_load_2d(sA + s * A_BYTES, &map_a, &full_tma[s], kb * BK, m0);
                    tma_load_2d(sP + s * P_BYTES, &map_p, &full_tma[s], kb * PB, n0);
                }
            }
            if (!ok) {
                for (uint32_t i = 0; i < ST && i < g; ++i) {
                    const uint32_t gi = g - 1 - i;
                    drain_bar(&full_tma[gi % ST], (gi / ST) & 1u);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (even CTA) ----------------
        if (leader && lane == 0) {
            uint32_t g = 0;
            uint32_t t = 0;
            bool ok = true;
            PairUnit u;
            PairSched sched(pair, num_pairs, num_tiles, nkb, dp_tiles);
            for (; ok && sched.next(u); ++t) {
                const int b = t & 1;
                if (!wait_bar(&acc_empty[b], ((t >> 1) & 1u) ^ 1u, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * 2 * PBN);
                for (int kb = u.kb0; kb < u.kb1; ++kb, ++g) {
                    const int s1 = g % ST, s2 = g % SE;
                    if (!wait_bar(&full_exp[s2], (g / SE) & 1u, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + s1 * A_BYTES);
                    const uint32_t e_addr = smem_u32(sE + s2 * PE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk)
                        tc_mma_i8_pair(d_tmem, sw128_desc(a_addr + kk * UMMA_K), sw128_desc(e_addr + kk * UMMA_K),
                                       kPairIdesc, (kb != u.kb0 || kk != 0) ? 1u : 0u);
                    tc_commit_pair_both(&mma_done[s1]);
                }
                if (!ok) break;
                tc_commit_pair_both(&acc_full[b]);
            }
            tc_commit_pair_self(drain);
            drain_bar(drain, 0);
        }
    } else if (warp < 6) {
        // ---------------- expanders: own 128 features ----------------
        const int et = threadIdx.x - 64;
        const uint32_t p_base = smem_u32(sP);
        const uint32_t e_base = smem_u32(sE);
        const uint32_t full_exp_leader = map_to_peer(smem_u32(full_exp), 0);
        uint32_t g = 0;
        bool ok = true;
        PairUnit u;
        PairSched sched(pair, num_pairs, num_tiles, nkb, dp_tiles);
        while (ok && sched.next(u)) {
            for (int kb = u.kb0; kb < u.kb1; ++kb, ++g) {
                const int s1 = g % ST, s2 = g % SE;
                if (!wait_bar(&full_tma[s1], (g / ST) & 1u, abort_flag, status)) { ok = false; break; }
                if (g >= static_cast<uint32_t>(SE)) {
                    const uint32_t gp = g - SE;
                    if (!wait_bar(&mma_done[gp % ST], (gp / ST) & 1u, abort_flag, status)) { ok = false; break; }
                }
                expand_stage<FMT, PBN>(p_base + s1 * P_BYTES, e_base + s2 * PE_BYTES, et);
                // each writer orders its stores before the async proxy's reads;
                // one arrival per warp on the even CTA's barrier
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(full_exp_leader + static_cast<uint32_t>(s2 * 8));
            }
        }
    } else {
        // ---------------- epilogue: own 128 tokens x 256 features ----------------
        const int quarter = warp & 3;
        constexpr int kChunksPerWarp = 8 * 4 / EW;             // of the 8 32-column chunks
        const int c0 = ((warp - 6) >> 2) * kChunksPerWarp;     // this warp's first chunk
        const int flag = quarter * 2 + ((warp - 6) >> 2);      // this warp's flag (rows and columns)
        const uint32_t stage = smem_u32(sStage) + static_cast<uint32_t>((warp - 6) * stage_warp_bytes<OUT>());
        const uint32_t acc_empty_leader = map_to_peer(smem_u32(acc_empty), 0);
        const float sw_tensor = (FMT == kT2) ? s_w[0] : 0.0f;
        uint32_t t = 0;
        PairUnit u;
        PairSched sched(pair, num_pairs, num_tiles, nkb, dp_tiles);
        for (; sched.next(u); ++t) {
            const int b = t & 1;
            int ready = 0;
            if (lane == 0) ready = wait_bar(&acc_full[b], (t >> 1) & 1u, abort_flag, status) ? 1 : 0;
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            tc_fence_after();
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * 2 * PBN);
            if (u.kb0 > 0) {
                // a piece that starts inside its tile: publish the partial
                // tile in this pair's slot.  Workspace layout per CTA:
                // [epilogue warp][chunk][4-column group][row], so the 32 lanes
                // (rows) of one store write 512 contiguous bytes and each
                // warp's rows are one contiguous 32 KB block.
                uint4 *ws = g_pair_ws[pair] + rank * (PBM * 2 * PBN / 4) + quarter * kWsWarpVecs;
                pair_chunks(tacc, c0, kChunksPerWarp, [=](const uint32_t(&v)[32], int cc) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        ws[(cc * 8 + j) * 32 + lane] = make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                });
                __threadfence();
                __syncwarp();  // this warp's 32 rows and columns are stored
                if (lane == 0)
                    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(&g_pair_flag[pair][rank][flag]),
                                 "r"(epoch)
                                 : "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(acc_empty_leader + static_cast<uint32_t>(b * 8));
                continue;
            }
            // a piece that starts its tile and ends inside it: the partial
            // tiles of the pairs after this one complete it.  It is the
            // pair's last unit, so its MMAs are complete and nothing else
            // uses the TMA and expansion rings: the first partial tile is
            // staged there with all of a warp's copies in flight at once
            // (one round trip instead of one per chunk); further ones are
            // added from global memory chunk by chunk.
            const int nsum = u.last >= 0 ? u.last - static_cast<int>(pair) : 0;
            bool have = true;  // every lane acquires the flags of its warp's rows itself
            for (int p = 1; p <= nsum; ++p)
                have = have && wait_flag(&g_pair_flag[pair + p][rank][flag], epoch, abort_flag, status);
            const uint32_t staged = smem_u32(sA) + static_cast<uint32_t>(quarter * kWsWarpVecs * 16);
            if (nsum > 0 && have) {
                const uint4 *ws = g_pair_ws[pair + 1] + rank * (PBM * 2 * PBN / 4) + quarter * kWsWarpVecs;
#pragma unroll 8
                for (int i = c0 * 8; i < (c0 + kChunksPerWarp) * 8; ++i)  // this warp's chunks
                    cp_async_16(staged + static_cast<uint32_t>((i * 32 + lane) * 16), ws + i * 32 + lane);
                cp_async_wait_all();
            }
            const int64_t m0 = (u.tile / num_n) * 2 * PBM + rank * PBM;
            const int64_t n0 = (u.tile % num_n) * 2 * PBN;
            const int64_t row0 = m0 + quarter * 32;
            const float sx = (row0 + lane < M) ? ld_act_f32(s_x + row0 + lane) : 0.0f;
            pair_chunks(tacc, c0, kChunksPerWarp, [=](uint32_t(&v)[32], int cc) {
                const int64_t nc = n0 + cc * 32;
                if (nsum > 0 && have) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 a = lds128(staged + static_cast<uint32_t>(((cc * 8 + j) * 32 + lane) * 16));
                        v[4 * j] += a.x;
                        v[4 * j + 1] += a.y;
                        v[4 * j + 2] += a.z;
                        v[4 * j + 3] += a.w;
                    }
                }
                for (int p = 2; p <= nsum && have; ++p) {
                    const uint4 *ws = g_pair_ws[pair + p] + rank * (PBM * 2 * PBN / 4) + quarter * kWsWarpVecs;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 a = ld_act_u4(ws + (cc * 8 + j) * 32 + lane);
                        v[4 * j] += a.x;
                        v[4 * j + 1] += a.y;
                        v[4 * j + 2] += a.z;
                        v[4 * j + 3] += a.w;
                    }
                }
                if (nc < N) {
                    float sw[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        sw[i] = (FMT == kT2) ? sw_tensor : ((nc + i < N) ? __ldg(s_w + nc + i) : 0.0f);
                    epilogue_chunk<OUT>(v, sw, sx, kShift, y, ldy, row0, M, nc, N, vec_ok != 0, stage, lane);
                }
            });
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

// Pairs of one instantiation that can be resident at once, found (with the
// shared-memory attribute set) on the first launch on each device.
template <int FMT, int OUT, int EW>
int pair_resident(int dev)
{
    constexpr size_t smem = pair_smem_bytes<FMT, OUT, EW>();
    static_assert(smem <= 232448, "shared memory budget");
    static PerDevice max_pairs;
    return max_pairs.get(dev, [&] {
        if (cudaFuncSetAttribute(gemm_pair_kernel<FMT, OUT, EW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem)) != cudaSuccess)
            return 0;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * static_cast<unsigned>(device_sm_count() / 2));
        cfg.blockDim = dim3(pair_threads<EW>());
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        return cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<FMT, OUT, EW>, &cfg) == cudaSuccess ? n : 0;
    });
}

template <int FMT, int OUT, int EW>
lowbit_status launch_pair_ew(const CUtensorMap &ma, const CUtensorMap &mp, const float *s_x, const float *s_w,
                             int64_t M, int64_t N, int64_t K, void *y, int64_t ldy, int vec_ok, int prefetch,
                             int exclusive, int32_t *status, int resident, cudaStream_t st)
{
    const int64_t tiles = ((M + 2 * PBM - 1) / (2 * PBM)) * ((N + 2 * PBN - 1) / (2 * PBN));
    int64_t pairs = tiles < resident ? tiles : resident;
    int64_t dp_tiles = tiles;
    if (exclusive) pair_plan(tiles, resident, (K + BK - 1) / BK, dp_tiles, pairs);
    uint32_t epoch = g_pair_epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    if (epoch == 0) epoch = g_pair_epoch.fetch_add(1, std::memory_order_relaxed) + 1;  // 0 is the flags' initial value
    return launch_pdl(gemm_pair_kernel<FMT, OUT, EW>, dim3(static_cast<unsigned>(2 * pairs)),
                      dim3(pair_threads<EW>()), pair_smem_bytes<FMT, OUT, EW>(), st, 0, ma, mp, s_x, s_w, M, N, K,
                      y, ldy, vec_ok, prefetch, status, dp_tiles, epoch);
}

// Eight epilogue warps where a tile's epilogue is mostly exposed (at most
// three tiles per pair) and their staging fits shared memory (bf16 out);
// four otherwise.
template <int FMT, int OUT>
lowbit_status launch_pair_t(const CUtensorMap &ma, const CUtensorMap &mp, const float *s_x, const float *s_w,
                            int64_t M, int64_t N, int64_t K, void *y, int64_t ldy, int vec_ok, int prefetch,
                            int exclusive, int32_t *status, cudaStream_t st)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    const int64_t tiles = ((M + 2 * PBM - 1) / (2 * PBM)) * ((N + 2 * PBN - 1) / (2 * PBN));
    if constexpr (OUT == LOWBIT_BF16) {
        const int resident = pair_resident<FMT, OUT, 8>(dev);
        if (resident <= 0) return LOWBIT_ERR_CUDA;
        if (tiles <= 3 * static_cast<int64_t>(resident))
            return launch_pair_ew<FMT, OUT, 8>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, exclusive,
                                                status, resident, st);
    }
    const int resident = pair_resident<FMT, OUT, 4>(dev);
    if (resident <= 0) return LOWBIT_ERR_CUDA;
    return launch_pair_ew<FMT, OUT, 4>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, exclusive, status,
                                       resident, st);
}

template <int FMT>
lowbit_status launch_pair_fmt(const CUtensorMap &ma, const CUtensorMap &mp, const float *s_x, const float *s_w,
                              int64_t M, int64_t N, int64_t K, void *y, lowbit_dtype ydt, int64_t ldy, int vec_ok,
                              int prefetch, int exclusive, int32_t *status, cudaStream_t st)
{
    if (ydt == LOWBIT_F32)
        return launch_pair_t<FMT, LOWBIT_F32>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, exclusive, status,
                                              st);
    if (ydt == LOWBIT_BF16)
        return launch_pair_t<FMT, LOWBIT_BF16>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, exclusive, status,
                                               st);
    return launch_pair_t<FMT, LOWBIT_I32>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, exclusive, status, st);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int FMT, int OUT, int TBN>
lowbit_status launch_splitk(const CUtensorMap &ma, const CUtensorMap &mp, const float *s_x, const float *s_w,
                            int64_t M, int64_t N, int64_t K, void *y, int64_t ldy, int vec_ok, int C, int prefetch,
                            int32_t *status, cudaStream_t st)
{
    constexpr size_t smem = splitk_smem_bytes<FMT, OUT, TBN>();
    static_assert(smem <= 232448, "shared memory budget");
    static PerDevice configured;  // the attribute is set once per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            return cudaFuncSetAttribute(gemm_splitk_kernel<FMT, OUT, TBN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(smem)) == cudaSuccess ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + TBN - 1) / TBN);
    return launch_pdl(gemm_splitk_kernel<FMT, OUT, TBN>, dim3(static_cast<unsigned>(tiles * C)), dim3(kThreads), smem,
                      st, static_cast<unsigned>(C), ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, C, prefetch, status);
}

template <int FMT, int OUT>
lowbit_status launch_t(const CUtensorMap &ma, const CUtensorMap &mp, const float *s_x, const float *s_w,
                       int64_t M, int64_t N, int64_t K, void *y, int64_t ldy, int vec_ok, int prefetch,
                       int32_t *status, SplitPlan plan, cudaStream_t st)
{
    if (plan.c > 1)
        return launch_splitk<FMT, OUT, 256>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, plan.c, prefetch, status, st);
    constexpr size_t smem = smem_bytes<FMT, OUT>();
    static_assert(smem <= 232448, "shared memory budget");
    static PerDevice configured;  // the attribute is set once per device
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            return cudaFuncSetAttribute(gemm_kernel<FMT, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(smem)) == cudaSuccess ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int64_t sms = device_sm_count();
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    return launch_pdl(gemm_kernel<FMT, OUT>, dim3(grid), dim3(kThreads), smem, st, 0, ma, mp, s_x, s_w, M, N, K, y,
                      ldy, vec_ok, prefetch, status);
}

template <int FMT>
lowbit_status launch_fmt(const CUtensorMap &ma, const CUtensorMap &mp, const float *s_x, const float *s_w,
                         int64_t M, int64_t N, int64_t K, void *y, lowbit_dtype ydt, int64_t ldy, int vec_ok,
                         int prefetch, int32_t *status, SplitPlan plan, cudaStream_t st)
{
    if (ydt == LOWBIT_F32)
        return launch_t<FMT, LOWBIT_F32>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, status, plan, st);
    if (ydt == LOWBIT_BF16)
        return launch_t<FMT, LOWBIT_BF16>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, status, plan, st);
    return launch_t<FMT, LOWBIT_I32>(ma, mp, s_x, s_w, M, N, K, y, ldy, vec_ok, prefetch, status, plan, st);
}

// The split plan of a format: its TMA ring depth and packed bytes per K block.
inline SplitPlan plan_for(lowbit_format f, int64_t M, int64_t N, int64_t K, int64_t sms)
{
    if (f == LOWBIT_TERNARY2) return splitk_plan(M, N, K, sms, tma_stages<kT2>(), packed_bytes_per_kblock<kT2>());
    if (f == LOWBIT_BINARY1) return splitk_plan(M, N, K, sms, tma_stages<kB1>(), packed_bytes_per_kblock<kB1>());
    return splitk_plan(M, N, K, sms, tma_stages<kI4>(), packed_bytes_per_kblock<kI4>());
}

}  // namespace tc

bool gemm_splits_k(lowbit_format f, int64_t M, int64_t N, int64_t K, int64_t sms)
{
    const tc::SplitPlan p = tc::plan_for(f, M, N, K, sms);
    return p.c > 1 || p.tbn != tc::BN;
}

lowbit_status gemm_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                          const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                          lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                          int32_t *status, cudaStream_t st)
{
    using namespace tc;
    CUtensorMap ma, mp;
    if (!make_map_2d(&ma, q, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ldq), BK,
                     BM, CU_TENSOR_MAP_SWIZZLE_128B))
        return LOWBIT_ERR_CUDA;
    const uint32_t pb = f == LOWBIT_TERNARY2 ? packed_bytes_per_kblock<kT2>()
                        : f == LOWBIT_BINARY1 ? packed_bytes_per_kblock<kB1>()
                                              : packed_bytes_per_kblock<kI4>();
    const SplitPlan plan = plan_for(f, M, N, K, device_sm_count());
    if (!make_map_2d(&mp, packed, static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(N),
                     static_cast<uint64_t>(ldp), pb, static_cast<uint32_t>(plan.tbn), CU_TENSOR_MAP_SWIZZLE_NONE))
        return LOWBIT_ERR_CUDA;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    const int vec_ok = ((reinterpret_cast<uintptr_t>(y) & 15u) == 0 && (ldy * esz) % 16 == 0) ? 1 : 0;
    if (f == LOWBIT_TERNARY2)
        return launch_fmt<kT2>(ma, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, prefetch, status, plan, st);
    if (f == LOWBIT_BINARY1)
        return launch_fmt<kB1>(ma, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, prefetch, status, plan, st);
    return launch_fmt<kI4>(ma, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, prefetch, status, plan, st);
}

}  // namespace lowbit

namespace lowbit {
// SM-pair variant: 128-token activation boxes and 128-row packed boxes per CTA.
lowbit_status gemm_pair_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                               const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                               lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                               int exclusive, int32_t *status, cudaStream_t st)
{
    using namespace tc;
    CUtensorMap ma, mp;
    if (!make_map_2d(&ma, q, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ldq), BK,
                     PBM, CU_TENSOR_MAP_SWIZZLE_128B))
        return LOWBIT_ERR_CUDA;
    const uint32_t pb = f == LOWBIT_TERNARY2 ? packed_bytes_per_kblock<kT2>()
                        : f == LOWBIT_BINARY1 ? packed_bytes_per_kblock<kB1>()
                                              : packed_bytes_per_kblock<kI4>();
    if (!make_map_2d(&mp, packed, static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(N),
                     static_cast<uint64_t>(ldp), pb, PBN, CU_TENSOR_MAP_SWIZZLE_NONE))
        return LOWBIT_ERR_CUDA;
    const int64_t esz = ydt == LOWBIT_BF16 ? 2 : 4;
    const int vec_ok = ((reinterpret_cast<uintptr_t>(y) & 15u) == 0 && (ldy * esz) % 16 == 0) ? 1 : 0;
    if (f == LOWBIT_TERNARY2)
        return launch_pair_fmt<kT2>(ma, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, prefetch, exclusive, status,
                                     st);
    if (f == LOWBIT_BINARY1)
        return launch_pair_fmt<kB1>(ma, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, prefetch, exclusive, status,
                                     st);
    return launch_pair_fmt<kI4>(ma, mp, s_x, s_w, M, N, K, y, ydt, ldy, vec_ok, prefetch, exclusive, status,
                                     st);
}
}  // namespace lowbit

namespace lowbit {
// This file's copy of the pipeline wait bound (see lowbit_set_wait_limit).
lowbit_status set_wait_limit_gemm(long long cycles) { return tc::set_wait_limit_here(cycles); }
}  // namespace lowbit
