// skinny_mma.cu -- the integer dot for a few tokens (M <= 16) on the warp-level
// tensor-core instruction mma.sync m16n8k32 (s8 x s8 -> s32).
//
// Same operator as the GEMV and the GEMMs ("M8.8 - Native Binary and Ternary
// Transformers" 0x05D, 0x09A-0x09B; the add/subtract/skip rule of the
// "Atomic-1Bit" README): acc[t, n] = sum_k q[t, k] c[n, k], int32, then the
// fused rescale y = float(acc) * (s_w * s_x) (M8.8 0x02D).
//
// Decode streams packed weights, so the kernel is laid out like the GEMV: every
// weight load of a warp is issued before any of them is used, and nothing
// waits on another warp until the final reduction.  The contraction runs on
// the tensor cores through register fragments instead of dp4a:
//
//   * A (16 x 32, row-major) = 16 weight rows x 32 codes.  Fragment register
//     a0 of lane (g, t) holds codes 4t..4t+3 of row g: with the plane-ordered
//     packing that is exactly one shift-and-mask of one packed word (the same
//     expansion the other kernels use), so the packed words go straight from
//     the load registers into the fragments;
//   * B (32 x 8) = 32 codes x 8 tokens, read from q (L1/L2 resident);
//   * C (16 x 8) = int32 accumulators in registers.
//
// A block of 8 warps owns 32 weight rows (two 16-row slabs) and splits K over
// its warps (16-byte weight chunks c = warp, warp + 8, ...); the 8 partial
// tiles are summed through shared memory and the epilogue writes y.
#include "tc_common.cuh"

namespace lowbit {
namespace skinny {

constexpr int kWarps = 8;
constexpr int kSlabs = 2;              // 16-row slabs per block
constexpr int kRows = 16 * kSlabs;     // weight rows per block
constexpr int kUnroll = 4;             // 16-byte chunks per row in flight per lane

// Codes in one 16-byte chunk of a packed row, and K steps of 32 in it.
template <int FMT> __host__ __device__ constexpr int chunk_codes() { return 4 * Fmt<FMT>::kCodesPerWord; }
template <int FMT> __host__ __device__ constexpr int chunk_steps() { return chunk_codes<FMT>() / 32; }

__device__ __forceinline__ void mma_s8(int32_t (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four activation codes q[token, k..k+3] (k a multiple of 4), zero past K
// and for tokens >= M.
__device__ __forceinline__ uint32_t q_word(const int8_t *__restrict__ q, int64_t ldq, int token, int M, int64_t k,
                                           int64_t K)
{
    if (token >= M || k >= K) return 0u;
    // L1-cached: every warp of every block reads the same few KB of codes.
    // The asm keeps the load after griddepcontrol.wait (see ld_act_u4).
    uint32_t v;
    asm volatile("ld.global.ca.u32 %0, [%1];" : "=r"(v) : "l"(q + token * ldq + k) : "memory");
    const int64_t valid = K - k;
    if (valid < 4) v &= (1u << (8 * valid)) - 1u;
    return v;
}

// A fragment of K step j of a chunk: rows g (wa) and g + 8 (wb), columns
// 4t..4t+3 and 16+4t..16+4t+3 of the step, each as int8 (c << S).
template <int FMT, int J>
__device__ __forceinline__ void a_fragment(const uint4 &wa, const uint4 &wb, int t, uint32_t (&a)[4])
{
    if constexpr (FMT == kT2) {
        // word 2J: codes 0..15 of the step, word 2J+1: codes 16..31; field t
        const uint32_t sh = static_cast<uint32_t>(6 - 2 * t);
        const uint32_t alo = J == 0 ? wa.x : wa.z, ahi = J == 0 ? wa.y : wa.w;
        const uint32_t blo = J == 0 ? wb.x : wb.z, bhi = J == 0 ? wb.y : wb.w;
        a[0] = (alo << sh) & 0xC0C0C0C0u;
        a[1] = (blo << sh) & 0xC0C0C0C0u;
        a[2] = (ahi << sh) & 0xC0C0C0C0u;
        a[3] = (bhi << sh) & 0xC0C0C0C0u;
    } else if constexpr (FMT == kI4) {
        // one step per chunk; codes 4t..4t+3 are nibble (t & 1) of word t >> 1
        const bool hi = (t >> 1) != 0;
        const uint32_t sh = (t & 1) ? 0u : 4u;
        const uint32_t alo = hi ? wa.y : wa.x, ahi = hi ? wa.w : wa.z;
        const uint32_t blo = hi ? wb.y : wb.x, bhi = hi ? wb.w : wb.z;
        a[0] = (alo << sh) & 0xF0F0F0F0u;
        a[1] = (blo << sh) & 0xF0F0F0F0u;
        a[2] = (ahi << sh) & 0xF0F0F0F0u;
        a[3] = (bhi << sh) & 0xF0F0F0F0u;
    } else {
        // word J holds the step's 32 codes, bit b = code b
        const uint32_t aw = J == 0 ? wa.x : J == 1 ? wa.y : J == 2 ? wa.z : wa.w;
        const uint32_t bw = J == 0 ? wb.x : J == 1 ? wb.y : J == 2 ? wb.z : wb.w;
        const uint32_t sh = static_cast<uint32_t>(4 * t);
        a[0] = b1_expand_nibble((aw >> sh) & 0xFu);
        a[1] = b1_expand_nibble((bw >> sh) & 0xFu);
        a[2] = b1_expand_nibble((aw >> (sh + 16)) & 0xFu);
        a[3] = b1_expand_nibble((bw >> (sh + 16)) & 0xFu);
    }
}

// B fragments of the chunk's K steps (codes k0 .. k0 + chunk_codes - 1).
template <int FMT, int NT>
__device__ __forceinline__ void load_b(const int8_t *__restrict__ q, int64_t ldq, int M, int64_t K, int64_t k0, int g,
                                       int t, uint32_t (&b)[chunk_steps<FMT>()][NT][2])
{
#pragma unroll
    for (int j = 0; j < chunk_steps<FMT>(); ++j)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            b[j][nt][0] = q_word(q, ldq, 8 * nt + g, M, k0 + 32 * j + 4 * t, K);
            b[j][nt][1] = q_word(q, ldq, 8 * nt + g, M, k0 + 32 * j + 16 + 4 * t, K);
        }
}

template <int FMT, int NT>
__device__ __forceinline__ void chunk_mma(const uint4 (&wa)[kSlabs], const uint4 (&wb)[kSlabs],
                                          const uint32_t (&b)[chunk_steps<FMT>()][NT][2], int t,
                                          int32_t (&acc)[kSlabs][NT][4])
{
#pragma unroll
    for (int j = 0; j < chunk_steps<FMT>(); ++j) {
#pragma unroll
        for (int s = 0; s < kSlabs; ++s) {
            uint32_t a[4];
            if (j == 0) a_fragment<FMT, 0>(wa[s], wb[s], t, a);
            else if (j == 1) a_fragment<FMT, 1>(wa[s], wb[s], t, a);
            else if (j == 2) a_fragment<FMT, 2>(wa[s], wb[s], t, a);
            else a_fragment<FMT, 3>(wa[s], wb[s], t, a);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_s8(acc[s][nt], a, b[j][nt][0], b[j][nt][1]);
        }
    }
}

template <int FMT, int OUT, int NT>
__global__ void __launch_bounds__(kWarps * 32)
skinny_mma_kernel(const int8_t *__restrict__ q, int64_t ldq, const float *__restrict__ s_x, int M, int64_t K,
                  const uint8_t *__restrict__ packed, int64_t ldp, int64_t nchunks, const float *__restrict__ s_w,
                  int64_t N, void *__restrict__ y, int64_t ldy, int prefetch)
{
    __shared__ int32_t red[kWarps][kSlabs * NT * 4][32];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t n_base = static_cast<int64_t>(blockIdx.x) * kRows;

    // With prefetch the first weight loads are issued before the wait for the
    // previous kernel (the caller vouches that it does not write the weights).
    bool waited = prefetch == 0;
    if (waited) pdl_wait();
    pdl_trigger();

    int32_t acc[kSlabs][NT][4];
#pragma unroll
    for (int s = 0; s < kSlabs; ++s)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[s][nt][i] = 0;

    const uint8_t *rowa[kSlabs], *rowb[kSlabs];
    bool oka[kSlabs], okb[kSlabs];
#pragma unroll
    for (int s = 0; s < kSlabs; ++s) {
        const int64_t ra = n_base + 16 * s + g, rb = ra + 8;
        oka[s] = ra < N;
        okb[s] = rb < N;
        rowa[s] = packed + (oka[s] ? ra : 0) * ldp;
        rowb[s] = packed + (okb[s] ? rb : 0) * ldp;
    }

    for (int64_t c0 = warp; c0 < nchunks; c0 += kWarps * kUnroll) {
        uint4 wa[kUnroll][kSlabs], wb[kUnroll][kSlabs];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t c = c0 + kWarps * u;
#pragma unroll
            for (int s = 0; s < kSlabs; ++s) {
                wa[u][s] = (c < nchunks && oka[s]) ? ld_stream_u4(rowa[s] + c * 16) : make_uint4(0, 0, 0, 0);
                wb[u][s] = (c < nchunks && okb[s]) ? ld_stream_u4(rowb[s] + c * 16) : make_uint4(0, 0, 0, 0);
            }
        }
        if (!waited) {
            pdl_wait();
            waited = true;
        }
        // all activation words of this round before any MMA: one L2 round trip
        uint32_t b[kUnroll][chunk_steps<FMT>()][NT][2];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) load_b<FMT, NT>(q, ldq, M, K, (c0 + kWarps * u) * chunk_codes<FMT>(), g, t, b[u]);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t c = c0 + kWarps * u;
            if (c < nchunks) chunk_mma<FMT, NT>(wa[u], wb[u], b[u], t, acc);
        }
    }
    if (!waited) pdl_wait();

#pragma unroll
    for (int s = 0; s < kSlabs; ++s)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) red[warp][(s * NT + nt) * 4 + i][lane] = acc[s][nt][i];
    __syncthreads();

    // C fragment element i of lane (g, t): row g + 8 * (i >> 1), token 2t + (i & 1).
    constexpr int kElems = kSlabs * NT * 4 * 32;
    for (int idx = threadIdx.x; idx < kElems; idx += kWarps * 32) {
        const int e = idx >> 5, ln = idx & 31;
        int32_t v = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) v += red[w][e][ln];
        const int s = e / (NT * 4), nt = (e >> 2) % NT, i = e & 3;
        const int64_t n = n_base + 16 * s + (ln >> 2) + 8 * (i >> 1);
        const int token = 8 * nt + 2 * (ln & 3) + (i & 1);
        if (n < N && token < M) {
            const int32_t a = v >> Fmt<FMT>::kShift;
            const int64_t idy = static_cast<int64_t>(token) * ldy + n;
            if constexpr (OUT == LOWBIT_I32) {
                static_cast<int32_t *>(y)[idy] = a;
            } else {
                const float f = rescale(a, s_w[FMT == kT2 ? 0 : n], ld_act_f32(s_x + token));
                if constexpr (OUT == LOWBIT_F32) static_cast<float *>(y)[idy] = f;
                else static_cast<__nv_bfloat16 *>(y)[idy] = __float2bfloat16_rn(f);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Streaming variant for long rows.  The register kernel above keeps its
// weight bytes in flight in registers, four lanes per 16-byte word (the
// fragment layout gives the same word to the four lanes of a group), so a
// long row needs several dependent load rounds.  Here one thread streams
// 32-row x 128-byte boxes of the packed artifact, and the token codes of the
// same K range (boxes of 128 codes x 8 or 16 tokens), into a ring of
// shared-memory stages with TMA (128-byte swizzle, so the 8 rows one
// ld.shared reads hit 8 different bank groups); four consumer warps take two
// 16-byte chunks of every row of a stage each and read both fragments from
// shared memory.
// ---------------------------------------------------------------------------
constexpr int kSRows = 32;                       // rows per block (two 16-row slabs)
constexpr int kSBox = 128;                       // bytes of each row per stage
constexpr int kSStageBytes = kSRows * kSBox;     // 4 KB of packed weights per stage
constexpr int kSStages = 12;                     // deepest ring
constexpr int kSRingBytes = 200 * 1024;          // ring budget (one block per SM at the deepest)
constexpr int kSConsumers = 4;                   // consumer warps; warp 4 is the producer

// Codes one stage covers (128 bytes of a packed row), the token-code boxes of
// 128 codes that hold them, and a stage's bytes with NT 8-token tiles.
template <int FMT> __host__ __device__ constexpr int stage_codes() { return 8 * chunk_codes<FMT>(); }
template <int FMT> __host__ __device__ constexpr int q_boxes() { return stage_codes<FMT>() / 128; }
template <int FMT, int NT> __host__ __device__ constexpr int s_stage_bytes()
{
    return kSStageBytes + q_boxes<FMT>() * 8 * NT * 128;
}
template <int FMT, int NT> __host__ __device__ constexpr int s_max_stages()
{
    return kSRingBytes / s_stage_bytes<FMT, NT>() < kSStages ? kSRingBytes / s_stage_bytes<FMT, NT>() : kSStages;
}

__device__ __forceinline__ uint32_t swz128(int row, int chunk)
{
    return static_cast<uint32_t>(row * kSBox + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Four token codes of token row n (of 8 * NT) at code offset o of a stage,
// from its swizzled q boxes at qbase.
template <int NT>
__device__ __forceinline__ uint32_t q_frag(uint32_t qbase, int n, int o)
{
    const int within = o & 127;
    return lds32(qbase + static_cast<uint32_t>((o >> 7) * (8 * NT * 128)) + swz128(n, within >> 4) +
                 static_cast<uint32_t>(within & 15));
}

// With ksplit > 1 the blocks run in clusters of ksplit that share 32 output
// rows: CTA r of a cluster takes stages [r S / ksplit, (r + 1) S / ksplit) of
// the S stages of a row, the CTAs r > 0 store their int32 partial tile into
// CTA 0's shared memory, and CTA 0 adds them (exact) and writes y.
constexpr int kSplitMax = 4;

template <int FMT, int OUT, int NT>
__global__ void __launch_bounds__((kSConsumers + 1) * 32)
stream_mma_kernel(const __grid_constant__ CUtensorMap map_p, const __grid_constant__ CUtensorMap map_q,
                  const float *__restrict__ s_x, int M, int64_t K, const float *__restrict__ s_w, int64_t N,
                  void *__restrict__ y, int64_t ldy, int nstages_all, int ksplit, int depth, int prefetch,
                  int32_t *status)
{
    constexpr int SB = s_stage_bytes<FMT, NT>();
    constexpr int QB = q_boxes<FMT>();
    constexpr int QBOX = 8 * NT * 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[kSStages], empty[kSStages];
    constexpr int kElems = kSlabs * NT * 4 * 32;
    __shared__ int32_t red[kSConsumers][kSlabs * NT * 4][32];
    __shared__ int abort_word;
    volatile int *abort_flag = &abort_word;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = ksplit > 1 ? static_cast<int>(tc::cluster_rank()) : 0;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x / ksplit) * kSRows;
    // this CTA's stages [st0, st0 + nstages) of the row
    const int st0 = static_cast<int>(static_cast<int64_t>(rank) * nstages_all / ksplit);
    const int nstages = static_cast<int>(static_cast<int64_t>(rank + 1) * nstages_all / ksplit) - st0;
    // with ksplit > 1: CTA 0's slots for the partial tiles of CTAs 1.. after the ring
    int32_t (*part)[kElems] = reinterpret_cast<int32_t (*)[kElems]>(ring + depth * SB);

    if (threadIdx.x == 0) {
        for (int i = 0; i < depth; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], kSConsumers);
        }
        abort_word = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_p)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_q)) : "memory");
    }
    __syncthreads();
    // Only the producer may touch global memory before the wait, and only the
    // weights (with prefetch; the caller vouches that the previous kernel does
    // not write them).
    const bool producer = warp == kSConsumers;
    if (!(producer && prefetch != 0)) pdl_wait();
    pdl_trigger();

    if (producer) {
        if (lane == 0) {
            auto load_q = [&](int st, int s) {
#pragma unroll
                for (int b = 0; b < QB; ++b)
                    tc::tma_load_2d(ring + s * SB + kSStageBytes + b * QBOX, &map_q, &full[s],
                                    (st0 + st) * stage_codes<FMT>() + 128 * b, 0);
            };
            // the first `depth` stages need no slot: their weight boxes go
            // out first (before the wait for the previous kernel with
            // prefetch), then their token codes
            const int first = nstages < depth ? nstages : depth;
            for (int st = 0; st < first; ++st) {
                tc::mbar_arrive_expect_tx(&full[st], SB);
                tc::tma_load_2d(ring + st * SB, &map_p, &full[st], (st0 + st) * kSBox, static_cast<int>(n0));
            }
            if (prefetch != 0) pdl_wait();
            for (int st = 0; st < first; ++st) load_q(st, st);
            int issued = first;
            for (int st = first; st < nstages; ++st) {
                const int s = st % depth;
                if (!tc::wait_bar(&empty[s], ((st / depth) & 1u) ^ 1u, abort_flag, status)) break;
                tc::mbar_arrive_expect_tx(&full[s], SB);
                tc::tma_load_2d(ring + s * SB, &map_p, &full[s], (st0 + st) * kSBox, static_cast<int>(n0));
                load_q(st, s);
                issued = st + 1;
            }
            // Every copy issued lands before the block leaves, also when the
            // consumers gave up on a wait (the last `depth` stages; earlier
            // ones were consumed before their slot was reissued).
            for (int i = 0; i < depth && i < issued; ++i) {
                const int st = issued - 1 - i;
                tc::drain_bar(&full[st % depth], (st / depth) & 1u);
            }
        }
        // every lane of this warp takes part in the epilogue below
        if (prefetch != 0) pdl_wait();
    } else {
        const int g = lane >> 2, t = lane & 3;
        int32_t acc[kSlabs][NT][4];
#pragma unroll
        for (int s = 0; s < kSlabs; ++s)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[s][nt][i] = 0;
        const uint32_t ring_base = tc::smem_u32(ring);
        for (int st = 0; st < nstages; ++st) {
            const int s = st % depth;
            int ok = 0;
            if (lane == 0) ok = tc::wait_bar(&full[s], (st / depth) & 1u, abort_flag, status) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const uint32_t stage = ring_base + static_cast<uint32_t>(s * SB);
            const uint32_t qbase = stage + kSStageBytes;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int chunk = 2 * warp + h;            // 16-byte chunk of each row in this stage
                uint4 wa[kSlabs], wb[kSlabs];
#pragma unroll
                for (int sl = 0; sl < kSlabs; ++sl) {
                    wa[sl] = tc::lds128(stage + swz128(16 * sl + g, chunk));
                    wb[sl] = tc::lds128(stage + swz128(16 * sl + g + 8, chunk));
                }
                uint32_t b[chunk_steps<FMT>()][NT][2];
#pragma unroll
                for (int j = 0; j < chunk_steps<FMT>(); ++j)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const int o = chunk * chunk_codes<FMT>() + 32 * j + 4 * t;
                        b[j][nt][0] = q_frag<NT>(qbase, 8 * nt + g, o);
                        b[j][nt][1] = q_frag<NT>(qbase, 8 * nt + g, o + 16);
                    }
                chunk_mma<FMT, NT>(wa, wb, b, t, acc);
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&empty[s]);
        }
#pragma unroll
        for (int sl = 0; sl < kSlabs; ++sl)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[warp][(sl * NT + nt) * 4 + i][lane] = acc[sl][nt][i];
    }
    __syncthreads();

    // this CTA's partial tile, element idx = (fragment element e, lane)
    constexpr int kThreadsS = (kSConsumers + 1) * 32;
    constexpr int kPer = (kElems + kThreadsS - 1) / kThreadsS;
    int32_t vsum[kPer];
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
        const int idx = threadIdx.x + r * kThreadsS;
        int32_t v = 0;
        if (idx < kElems) {
#pragma unroll
            for (int w = 0; w < kSConsumers; ++w) v += red[w][idx >> 5][idx & 31];
        }
        vsum[r] = v;
    }
    if (ksplit > 1) {
        if (rank != 0) {
#pragma unroll
            for (int r = 0; r < kPer; ++r) {
                const int idx = threadIdx.x + r * kThreadsS;
                if (idx < kElems) {
                    const uint32_t dst = tc::map_to_peer(tc::smem_u32(&part[rank - 1][idx]), 0);
                    asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(dst), "r"(vsum[r]) : "memory");
                }
            }
        }
        tc::cluster_sync_all();  // the partial tiles are in CTA 0; no CTA reads another after this
        if (rank != 0) return;
#pragma unroll
        for (int r = 0; r < kPer; ++r) {
            const int idx = threadIdx.x + r * kThreadsS;
            if (idx < kElems)
                for (int p = 0; p + 1 < ksplit; ++p) vsum[r] += part[p][idx];
        }
    }

#pragma unroll
    for (int r = 0; r < kPer; ++r) {
        const int idx = threadIdx.x + r * kThreadsS;
        if (idx >= kElems) continue;
        const int e = idx >> 5, ln = idx & 31;
        const int32_t v = vsum[r];
        const int sl = e / (NT * 4), nt = (e >> 2) % NT, i = e & 3;
        const int64_t n = n0 + 16 * sl + (ln >> 2) + 8 * (i >> 1);
        const int token = 8 * nt + 2 * (ln & 3) + (i & 1);
        if (n < N && token < M) {
            const int32_t a = v >> Fmt<FMT>::kShift;
            const int64_t idy = static_cast<int64_t>(token) * ldy + n;
            if constexpr (OUT == LOWBIT_I32) {
                static_cast<int32_t *>(y)[idy] = a;
            } else {
                const float f = rescale(a, s_w[FMT == kT2 ? 0 : n], ld_act_f32(s_x + token));
                if constexpr (OUT == LOWBIT_F32) static_cast<float *>(y)[idy] = f;
                else static_cast<__nv_bfloat16 *>(y)[idy] = __float2bfloat16_rn(f);
            }
        }
    }
}

template <int FMT, int OUT, int NT>
lowbit_status launch_stream_nt(const CUtensorMap &mp, const int8_t *q, int64_t ldq, const float *s_x, int M,
                               int64_t K, const float *s_w, int64_t N, void *y, int64_t ldy, int nstages, int prefetch,
                               int32_t *status, cudaStream_t st)
{
    constexpr int kMax = s_max_stages<FMT, NT>();
    constexpr size_t kMaxSmem = 1024 + static_cast<size_t>(kMax) * s_stage_bytes<FMT, NT>() +
                                (kSplitMax - 1) * kSlabs * NT * 4 * 32 * sizeof(int32_t);
    static PerDevice configured;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LOWBIT_ERR_CUDA;
    if (configured.get(dev, [&] {
            return cudaFuncSetAttribute(stream_mma_kernel<FMT, OUT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kMaxSmem)) == cudaSuccess ? 1 : 0;
        }) <= 0)
        return LOWBIT_ERR_CUDA;
    CUtensorMap mq;
    if (!tc::make_map_2d(&mq, q, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(ldq), 128,
                         8 * NT, CU_TENSOR_MAP_SWIZZLE_128B))
        return LOWBIT_ERR_CUDA;
    // K split over a cluster of ksplit CTAs: the largest of 4, 2, 1 whose
    // grid runs in one wave at no more than 3 blocks per SM with a ring of at
    // least min(its share of the stages, 4), each CTA keeping 2 stages or
    // more.  The ring is then as deep as the share and the blocks per SM
    // allow (short rows keep several blocks per SM).
    constexpr int64_t kSmSmem = 228 * 1024;   // shared memory per SM
    constexpr int64_t kStatic = 1024 + sizeof(int32_t) * kSConsumers * kSlabs * NT * 4 * 32 + 512;
    constexpr int kElemsH = kSlabs * NT * 4 * 32;
    const int64_t tiles = (N + kSRows - 1) / kSRows;
    const int64_t sms = device_sm_count();
    int ksplit = 1, depth = 1;
    for (int ks : {4, 2, 1}) {
        const int64_t per_sm = (tiles * ks + sms - 1) / sms;
        const int share = (nstages + ks - 1) / ks;
        if (ks > 1 && (per_sm > 3 || nstages < 2 * ks)) continue;
        const int64_t budget = kSmSmem / (per_sm < 1 ? 1 : per_sm) - kStatic - 1024 -
                               (ks > 1 ? (ks - 1) * kElemsH * 4 : 0);
        const int fit = static_cast<int>(budget / s_stage_bytes<FMT, NT>());
        const int want = share < 4 ? share : 4;
        if (ks > 1 && fit < want) continue;
        ksplit = ks;
        depth = share < kMax ? share : kMax;
        if (fit < depth) depth = fit < 1 ? 1 : fit;
        break;
    }
    const size_t smem = 1024 + static_cast<size_t>(depth) * s_stage_bytes<FMT, NT>() +
                        (ksplit > 1 ? static_cast<size_t>(ksplit - 1) * kElemsH * 4 : 0);
    const dim3 grid(static_cast<unsigned>(tiles * ksplit)), block((kSConsumers + 1) * 32);
    return launch_pdl(stream_mma_kernel<FMT, OUT, NT>, grid, block, smem, st, ksplit > 1 ? ksplit : 0, mp, mq, s_x, M,
                      K, s_w, N, y, ldy, nstages, ksplit, depth, prefetch, status);
}

template <int FMT, int OUT>
lowbit_status launch_stream(const CUtensorMap &mp, const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K,
                            const float *s_w, int64_t N, void *y, int64_t ldy, int nstages, int prefetch,
                            int32_t *status, cudaStream_t st)
{
    if (M <= 8)
        return launch_stream_nt<FMT, OUT, 1>(mp, q, ldq, s_x, M, K, s_w, N, y, ldy, nstages, prefetch, status, st);
    return launch_stream_nt<FMT, OUT, 2>(mp, q, ldq, s_x, M, K, s_w, N, y, ldy, nstages, prefetch, status, st);
}

template <int FMT, int OUT>
lowbit_status launch_out(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K, const uint8_t *packed,
                         int64_t ldp, int64_t nchunks, const float *s_w, int64_t N, void *y, int64_t ldy,
                         int prefetch, cudaStream_t st)
{
    const dim3 grid(static_cast<unsigned>((N + kRows - 1) / kRows)), block(kWarps * 32);
    if (M <= 8)
        return launch_pdl(skinny_mma_kernel<FMT, OUT, 1>, grid, block, 0, st, 0, q, ldq, s_x, M, K, packed, ldp,
                          nchunks, s_w, N, y, ldy, prefetch);
    return launch_pdl(skinny_mma_kernel<FMT, OUT, 2>, grid, block, 0, st, 0, q, ldq, s_x, M, K, packed, ldp, nchunks,
                      s_w, N, y, ldy, prefetch);
}

template <int FMT>
lowbit_status launch_fmt(const int8_t *q, int64_t ldq, const float *s_x, int M, int64_t K, const uint8_t *packed,
                         int64_t ldp, int64_t row_bytes, const float *s_w, int64_t N, void *y, lowbit_dtype ydt,
                         int64_t ldy, int prefetch, int32_t *status, cudaStream_t st)
{
    const int64_t nchunks = (row_bytes + 15) / 16;
    // Rows longer than one round of the register kernel (8 warps x 4 chunks)
    // stream through shared memory.
    if (nchunks > kWarps * kUnroll) {
        CUtensorMap mp;
        if (!tc::make_map_2d(&mp, packed, static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(N),
                             static_cast<uint64_t>(ldp), kSBox, kSRows, CU_TENSOR_MAP_SWIZZLE_128B))
            return LOWBIT_ERR_CUDA;
        const int nstages = static_cast<int>((row_bytes + kSBox - 1) / kSBox);
        if (ydt == LOWBIT_F32)
            return launch_stream<FMT, LOWBIT_F32>(mp, q, ldq, s_x, M, K, s_w, N, y, ldy, nstages, prefetch, status, st);
        if (ydt == LOWBIT_BF16)
            return launch_stream<FMT, LOWBIT_BF16>(mp, q, ldq, s_x, M, K, s_w, N, y, ldy, nstages, prefetch, status, st);
        return launch_stream<FMT, LOWBIT_I32>(mp, q, ldq, s_x, M, K, s_w, N, y, ldy, nstages, prefetch, status, st);
    }
    if (ydt == LOWBIT_F32)
        return launch_out<FMT, LOWBIT_F32>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ldy, prefetch, st);
    if (ydt == LOWBIT_BF16)
        return launch_out<FMT, LOWBIT_BF16>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ldy, prefetch, st);
    return launch_out<FMT, LOWBIT_I32>(q, ldq, s_x, M, K, packed, ldp, nchunks, s_w, N, y, ldy, prefetch, st);
}

}  // namespace skinny

// Up to 16 tokens in one launch.
lowbit_status skinny_launch(const int8_t *q, int64_t ldq, const float *s_x, int64_t M, int64_t K,
                            const uint8_t *packed, int64_t ldp, int64_t row_bytes, const float *s_w,
                            lowbit_format f, int64_t N, void *y, lowbit_dtype ydt, int64_t ldy, int prefetch,
                            int32_t *status, cudaStream_t st)
{
    const int m = static_cast<int>(M);
    if (f == LOWBIT_TERNARY2)
        return skinny::launch_fmt<kT2>(q, ldq, s_x, m, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, status, st);
    if (f == LOWBIT_BINARY1)
        return skinny::launch_fmt<kB1>(q, ldq, s_x, m, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, status, st);
    return skinny::launch_fmt<kI4>(q, ldq, s_x, m, K, packed, ldp, row_bytes, s_w, N, y, ydt, ldy, prefetch, status, st);
}

}  // namespace lowbit

namespace lowbit {
// This file's copy of the pipeline wait bound (see lowbit_set_wait_limit).
lowbit_status set_wait_limit_skinny(long long cycles) { return tc::set_wait_limit_here(cycles); }
}  // namespace lowbit
