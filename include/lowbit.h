/*
 * lowbit.h -- C ABI of the B200 (sm_100a) low-bit-weight linear layer.
 *
 * The operator is the BitLinear forward of a BitNet-style transformer,
 *
 *     acc[t,n] = sum_k q[t,k] * c[n,k]            (int32)
 *     y[t,n]   = float(acc[t,n]) * (s_w[n] * s_x[t])
 *
 * with weight codes c ternary {-1,0,+1}, binary {-1,+1} or 4-bit {-7..+7}
 * and per-token int8 activation codes q.  Sources, by page title and section:
 *
 *   "M8.8 - Native Binary and Ternary Transformers": 0x02C-0x02E (activation
 *     codes, integer accumulation, rescale), 0x05A-0x05D (absmean ternary
 *     codes, per-token A8 codes, the add/subtract kernel), 0x06E (binary sign
 *     rule and little-bit-first packing), 0x09A-0x09C (operation ledger,
 *     decode vs prefill, the INT32 bound, the reference decoder).
 *   "Atomic-1Bit" README: the add/sub/skip rule; four ternary codes per byte.
 *   "T4NT-0.5B" model card: tanh(w/3)*3 clipping, 15 symmetric levels.
 *
 * Conventions for every call below
 *   - All array pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing and keeps no per-call state.
 *   - Sizes are elements unless named *_bytes; leading dimensions (ld*) are
 *     the distance between consecutive rows, row-major, K contiguous.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call is asynchronous on that stream; nothing synchronises the host.
 *   - Argument errors are found on the host before any launch and returned
 *     as a lowbit_status; nothing is launched then.
 *   - Data errors found on the device (a non-finite input, a reserved code, a
 *     pipeline wait that ran out) are OR-ed into `*status_dev` as the bit
 *     (1u << status) when `status_dev` is not NULL (a device int32 the caller
 *     zeroes and reads back).  With NULL they are not reported.
 */
#ifndef LOWBIT_H
#define LOWBIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Weight code formats.  Packed layouts (row n starts at byte n*ldp; every bit
 * that no code owns must be zero):
 *   LOWBIT_TERNARY2  2-bit two's-complement fields 00 = 0, 01 = +1, 11 = -1,
 *                    10 reserved; four codes per byte.  Inside each
 *                    little-endian 32-bit word of 16 codes, code k sits in
 *                    byte (k%16)%4, field (k%16)/4 (bits 8*byte + 2*field).
 *                    One scale per tensor.
 *   LOWBIT_BINARY1   bit k%8 of byte k/8 is 1 for -1 and 0 for +1
 *                    (little-bit-first, M8.8 0x06E).  One scale per row.
 *   LOWBIT_INT4      4-bit two's-complement fields, 1000 reserved; inside each
 *                    32-bit word of 8 codes, code k sits in byte (k%8)%4,
 *                    nibble (k%8)/4.  One scale per row. */
typedef enum lowbit_format {
    LOWBIT_TERNARY2 = 0,
    LOWBIT_BINARY1 = 1,
    LOWBIT_INT4 = 2
} lowbit_format;

typedef enum lowbit_dtype {
    LOWBIT_F32 = 0,  /* IEEE fp32 */
    LOWBIT_BF16 = 1, /* bfloat16, fp32 rounded to nearest even */
    LOWBIT_I32 = 2   /* raw int32 accumulators (outputs only) */
} lowbit_dtype;

typedef enum lowbit_status {
    LOWBIT_OK = 0,
    LOWBIT_ERR_INVALID_ARG = 1,     /* null pointer, size <= 0, ld too small, bad enum */
    LOWBIT_ERR_ALIGNMENT = 2,       /* pointer or leading dimension misaligned */
    LOWBIT_ERR_UNSUPPORTED = 3,     /* valid but not implemented (e.g. no sm_100 device) */
    LOWBIT_ERR_OVERFLOW_BOUND = 4,  /* K beyond the int32 accumulator bound */
    LOWBIT_ERR_NONFINITE = 5,       /* device: NaN/Inf input (or x*127 overflow) */
    LOWBIT_ERR_RESERVED_CODE = 6,   /* device: reserved pattern or non-zero unowned bit */
    LOWBIT_ERR_TIMEOUT = 7,         /* device: a pipeline wait gave up */
    LOWBIT_ERR_CUDA = 8             /* a CUDA runtime call or launch failed */
} lowbit_status;

/* Bytes a packed row needs (its logical extent): TERNARY2 4*ceil(K/16),
 * BINARY1 ceil(K/8), INT4 4*ceil(K/8).  0 for a bad format or K <= 0. */
size_t lowbit_packed_row_bytes(lowbit_format f, int64_t K);

/* Smallest valid row stride for packed weights: the row bytes rounded up to
 * a multiple of 16. */
size_t lowbit_packed_ld(lowbit_format f, int64_t K);

/* Number of fp32 weight scales: 1 for TERNARY2 (per tensor, M8.8 0x05A),
 * N for BINARY1 and INT4 (per output row).  0 for bad arguments. */
int64_t lowbit_scale_count(lowbit_format f, int64_t N);

/* Largest K lowbit_linear accepts for a format: the worst case
 * |acc| = 128 * max|c| * K must stay inside int32 (M8.8 0x09C). */
int64_t lowbit_max_k(lowbit_format f);

/* Device workspace lowbit_pack needs: 8*N bytes (rounded to 256) for
 * TERNARY2, whose per-tensor scale is a two-stage fixed-order sum; 0 for the
 * other formats. */
size_t lowbit_pack_workspace_bytes(lowbit_format f, int64_t N);

/* lowbit_pack -- quantise fp32 weights W[N,K] (row stride ldw elements) into
 * codes and pack them (done once per weight, off the hot path; M8.8 0x04D:
 * export freezes codes and scales).
 *   TERNARY2 (M8.8 0x05A-0x05B): gamma = mean|W| over the tensor, summed in
 *     fp64 row by row (k ascending) then over rows (n ascending), rounded once
 *     to fp32; c = clip(rint(w / (gamma + eps)), -1, 1) with an fp32 divide
 *     and nearest-even rounding; s_w[0] = gamma.  eps >= 0 (1e-5 in M8.8).
 *   BINARY1 (M8.8 0x06E, 0x02B): c = +1 if w >= 0 (both zeros) else -1;
 *     s_w[n] = mean_k |W[n,k]| (fp64 sum, k ascending, rounded once).
 *     eps is ignored.
 *   INT4 (T4NT-0.5B): w_c = 3*tanh(w/3) evaluated in fp64 by a fixed operation
 *     sequence (Taylor series of expm1 with a Cody-Waite split of ln 2) and
 *     rounded once to fp32; s_w[n] = max_k |w_c| / 7; c = clip(rint(w_c /
 *     s_w[n]), -7, 7); a zero row gives s_w = 0 and zero codes.  eps ignored.
 * Outputs: packed[N, ldp] bytes (ldp >= lowbit_packed_row_bytes, multiple of
 * 16, 16-byte aligned base; unowned bits written zero), s_w[lowbit_scale_count]
 * fp32.  `workspace` must hold lowbit_pack_workspace_bytes(f, N) bytes of
 * device memory (may be NULL when that is 0).  A non-finite weight sets
 * LOWBIT_ERR_NONFINITE in *status_dev; the artifact is then unspecified. */
lowbit_status lowbit_pack(const float *w, int64_t N, int64_t K, int64_t ldw,
                          lowbit_format f, float eps,
                          uint8_t *packed, int64_t ldp, float *s_w,
                          void *workspace, size_t workspace_bytes,
                          int32_t *status_dev, void *stream);

/* Weight quantisers of lowbit_pack_ex. */
#define LOWBIT_QUANT_DEFAULT 0          /* the format's quantiser of lowbit_pack */
#define LOWBIT_QUANT_BINARY_CENTRED 1   /* BitNet v1 centred sign, LOWBIT_BINARY1 only */

/* Device workspace lowbit_pack_ex needs: lowbit_pack_workspace_bytes for
 * LOWBIT_QUANT_DEFAULT; 16*N + 16 bytes (rounded up to 256) for
 * LOWBIT_QUANT_BINARY_CENTRED.  0 for bad arguments. */
size_t lowbit_pack_ex_workspace_bytes(lowbit_format f, int quantizer, int64_t N);

/* lowbit_pack_ex -- lowbit_pack with a choice of quantiser.
 *   LOWBIT_QUANT_DEFAULT: exactly lowbit_pack.
 *   LOWBIT_QUANT_BINARY_CENTRED (f must be LOWBIT_BINARY1), the original
 *     BitNet's binarisation (M8.8 0x02B, 0x02E): alpha = mean(W) and
 *     beta = mean|W| over the whole tensor, each an fp64 sum in the ternary
 *     scale's fixed order (k ascending within a row, then rows ascending)
 *     divided by N*K and rounded once to fp32; c = +1 where w > alpha and -1
 *     otherwise (a weight equal to the mean takes -1, the page's tie), packed
 *     in the LOWBIT_BINARY1 layout.  The scale is one per tensor; it is written
 *     to all N entries of s_w so that lowbit_linear with LOWBIT_BINARY1 (one
 *     scale per row) applies it unchanged.  eps is ignored.
 * Other arguments, outputs and errors as lowbit_pack; `workspace` must hold
 * lowbit_pack_ex_workspace_bytes(f, quantizer, N) bytes (8-byte aligned). */
lowbit_status lowbit_pack_ex(const float *w, int64_t N, int64_t K, int64_t ldw,
                             lowbit_format f, int quantizer, float eps,
                             uint8_t *packed, int64_t ldp, float *s_w,
                             void *workspace, size_t workspace_bytes,
                             int32_t *status_dev, void *stream);

/* Largest N lowbit_pack_ternary_noalloc accepts. */
#define LOWBIT_NOALLOC_MAX_ROWS 65536

/* lowbit_pack_ternary_noalloc -- lowbit_pack for LOWBIT_TERNARY2 that
 * allocates nothing and takes no workspace.  (The pages have no counterpart:
 * this is a deployment variant of the same packer.)  It is for callers that
 * cannot allocate device memory at packing time: runtimes whose device-memory
 * budget is fixed at start-up, and hosts whose device memory belongs to an
 * allocator a C caller cannot reach (a cudaFree would also synchronise the
 * device and stall their other streams).  The per-row sums of the ternary
 * scale go to a static device array of LOWBIT_NOALLOC_MAX_ROWS doubles
 * (512 KB) that every GPU loading the library keeps until exit.
 *   - N > LOWBIT_NOALLOC_MAX_ROWS returns LOWBIT_ERR_INVALID_ARG; other
 *     arguments, outputs and errors are exactly those of lowbit_pack.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.
 *   - All calls share the one array: calls that may overlap on the GPU (on
 *     different streams, or from several host threads) race and must be
 *     serialised by the caller.  Each call writes every entry it reads, so
 *     the contents left by an earlier call never matter. */
lowbit_status lowbit_pack_ternary_noalloc(const float *w, int64_t N, int64_t K, int64_t ldw,
                                          float eps, uint8_t *packed, int64_t ldp, float *s_w,
                                          int32_t *status_dev, void *stream);

/* lowbit_unpack -- decode packed[N, ldp] into int8 codes[N, ldc] (ldc >= K).
 * A reserved field or a non-zero unowned bit sets LOWBIT_ERR_RESERVED_CODE in
 * *status_dev (M8.8 0x0BB: reserved patterns reject); such a code decodes as
 * 0.  Used by tests and tools, not by the hot path. */
lowbit_status lowbit_unpack(const uint8_t *packed, int64_t ldp, int64_t N, int64_t K,
                            lowbit_format f, int8_t *codes, int64_t ldc,
                            int32_t *status_dev, void *stream);

/* lowbit_act_quant -- per-token absmax int8 quantisation (M8.8 0x05C):
 *   gamma_t = max_k |x[t,k]|;
 *   gamma_t == 0:  q[t,:] = 0, s_x[t] = 0;
 *   else           q = clip(rint((x * 127) / (gamma_t + eps)), -128, 127)
 *                  (fp32 multiply, fp32 IEEE divide, nearest even),
 *                  s_x[t] = gamma_t / 127.
 * x is fp32 or bf16 (xdt = LOWBIT_F32 | LOWBIT_BF16), [M, K] with row stride
 * ldx elements, aligned to its element size (rows that start on 16-byte
 * boundaries take the one-pass vector kernel, others a two-pass scalar one).
 * q is int8 [M, ldq], 16-byte aligned, ldq a multiple of 16, ldq >= K; bytes
 * of q past K are left untouched.  s_x is fp32 [M].  eps >= 0 (0 in the
 * configurations this library is measured on).  A non-finite x, or an x*127
 * that overflows fp32, sets LOWBIT_ERR_NONFINITE; that row is unspecified. */
lowbit_status lowbit_act_quant(const void *x, lowbit_dtype xdt, int64_t M, int64_t K,
                               int64_t ldx, float eps, int8_t *q, int64_t ldq, float *s_x,
                               int32_t *status_dev, void *stream);

/* Activation prologue options of lowbit_act_quant_ex and lowbit_bitlinear. */
#define LOWBIT_NORM_NONE 0 /* no normalisation */
#define LOWBIT_NORM_RMS 1  /* RMSNorm: the row factor 1/sqrt(mean_k x_k^2 + eps_norm) */

/* Largest K the prologue accepts with a gain, RMSNorm or Hadamard option. */
#define LOWBIT_PROLOGUE_MAX_K 49152

/* lowbit_act_quant_ex -- the activation side of a BitLinear layer in one pass
 * over x: an optional RMSNorm with gain (M8.8 0x02E and 0x03: the activation
 * is normalised before its codes are taken; b1.58 and the T4NT model card use
 * RMSNorm), an optional input value vector (the gain alone, OneBit's x * g of
 * M8.8 0x06A), an optional block Hadamard rotation (H-BitLinear, M8.8 0x07C),
 * then the per-token absmax int8 codes of lowbit_act_quant with eps = 0:
 *   u_k   = x_k * g_k                        (fp32 product; g NULL: u = x)
 *   u     = FWHT_hb(u) on every block of `hadamard` consecutive features:
 *           the unnormalised radix-2 fast Walsh-Hadamard transform in fp32,
 *           stages h = 1, 2, 4, ..., each pair (a, b) -> (a + b, a - b)
 *   q     = clip(rint((u * 127) / max_k |u_k|), -128, 127)   (lowbit_act_quant)
 *   s_x   = max|u| / sqrt(hadamard) / rms / 127, rms = sqrt(mean_k x_k^2 +
 *           eps_norm) with LOWBIT_NORM_RMS (1 otherwise), evaluated in fp64
 *           (the sum of squares in fp64) and rounded once to fp32.
 * The RMSNorm output is x * g / rms and the normalised rotation is H/sqrt(hb);
 * both row factors are positive, so they cancel in absmax codes and only the
 * scale carries them: y = q * s_x reconstructs the normalised, rotated row.
 * An all-zero u gives zero codes and s_x = 0.
 * Arguments: x, xdt, M, K, ldx, q, ldq, s_x as lowbit_act_quant.  g: NULL or
 * a device array of K fp32 gains (4-byte aligned; 16-byte aligned for the
 * one-pass vector kernel).  norm: LOWBIT_NORM_NONE or LOWBIT_NORM_RMS.
 * eps_norm >= 0 and finite (ignored without the norm).  hadamard: 0 (none)
 * or a power of two >= 2 that divides K.  With any option K must be at most
 * LOWBIT_PROLOGUE_MAX_K (else LOWBIT_ERR_UNSUPPORTED).  With g NULL, no norm
 * and no rotation the call is exactly lowbit_act_quant with eps = 0.  A
 * non-finite x or g, or a non-finite product or transform, sets
 * LOWBIT_ERR_NONFINITE; that row is then unspecified. */
lowbit_status lowbit_act_quant_ex(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                  const float *g, int norm, float eps_norm, int hadamard,
                                  int8_t *q, int64_t ldq, float *s_x, int32_t *status_dev, void *stream);

/* lowbit_linear -- the low-bit linear layer on int8 activation codes:
 *   acc[t,n] = sum_{k<K} q[t,k] * c[n,k]  (exact int32: add/sub/skip for
 *              ternary and binary codes, Atomic-1Bit README, M8.8 0x05D)
 *   y[t,n]   = acc[t,n]                          (ydt = LOWBIT_I32)
 *            = float(acc) * (s_w[n or 0] * s_x[t]) (LOWBIT_F32; the two scales
 *              are multiplied first, both products fp32, M8.8 0x02D)
 *            = that fp32 value rounded to bf16, nearest even (LOWBIT_BF16).
 * Inputs: q int8 [M, ldq] and packed [N, ldp] as above (16-byte aligned bases,
 * ldq and ldp multiples of 16), s_x fp32 [M], s_w fp32 [lowbit_scale_count].
 * Output y [M, ldy], ldy >= N, aligned to its element size.  Bytes of q past
 * K are ignored.  K <= lowbit_max_k(f), else LOWBIT_ERR_OVERFLOW_BOUND.
 * M <= 4 runs the packed-weight GEMV kernel (dp4a); 5 <= M <= 16 runs
 * warp-level tensor-core MMAs (mma.sync, int8) on weight fragments expanded
 * in registers when rows are short (<= 512 packed bytes) or N >= 3200;
 * otherwise, and for 17 <= M < 512, a tcgen05 tensor-core GEMM (int8 MMA,
 * accumulators in tensor memory) with the expanded weight tile in shared
 * memory and K split over a cluster when the output tiles are few; from
 * M = 512 a tcgen05 GEMM on pairs of SMs (cta_group::2, 256 x 256 tiles,
 * expanded weights in shared memory) for ternary weights, except for
 * K >= 2048 when the shared-memory GEMM would split K (that case keeps it),
 * and the tcgen05 GEMM with the weight tile in tensor memory for 4-bit and
 * binary weights. */
lowbit_status lowbit_linear(const int8_t *q, int64_t ldq, const float *s_x,
                            int64_t M, int64_t K,
                            const uint8_t *packed, int64_t ldp, const float *s_w,
                            lowbit_format f, int64_t N,
                            void *y, lowbit_dtype ydt, int64_t ldy,
                            int32_t *status_dev, void *stream);

/* Same operator with the kernel chosen by the caller: path 0 = automatic (as
 * lowbit_linear), 1 = packed-weight GEMV (any M), 2 = tensor-core GEMM with
 * the expanded weight tile in shared memory (any M), 3 = tensor-core GEMM
 * with the expanded weight tile in tensor memory (any M), 4 = the same on
 * pairs of SMs (one MMA covers 256 weight rows; any M), 5 = warp-level
 * tensor-core MMAs on register fragments (M <= 16), 6 = tensor-core GEMM on
 * pairs of SMs with the expanded weight tile in shared memory (any M).  Other
 * values, and path 5 with M > 16, return LOWBIT_ERR_INVALID_ARG.  Lets tests and benchmarks reach every kernel at
 * every size. */
lowbit_status lowbit_linear_path(const int8_t *q, int64_t ldq, const float *s_x,
                                 int64_t M, int64_t K,
                                 const uint8_t *packed, int64_t ldp, const float *s_w,
                                 lowbit_format f, int64_t N,
                                 void *y, lowbit_dtype ydt, int64_t ldy,
                                 int path, int32_t *status_dev, void *stream);

/* Flag for lowbit_linear_ex: the caller guarantees that the packed artifact
 * and s_w are not written by the kernel that immediately precedes this call
 * on `stream` (nor concurrently by any other stream).  The library launches
 * its kernels so that they may start while the preceding kernel is still
 * running, and every kernel waits for that kernel to finish before touching
 * activations, outputs or the status word.  With this flag the weight bytes,
 * which do not depend on it, are requested before that wait, which hides the
 * memory latency of the first weight tiles behind the previous kernel.  In
 * a decode or prefill loop the preceding kernel is lowbit_act_quant or
 * another linear layer, so the guarantee holds; directly after lowbit_pack of
 * the same weights it does not. */
#define LOWBIT_LINEAR_WEIGHTS_STABLE 1u

/* Flag for lowbit_linear_ex: the caller guarantees that no other SM-pair GEMM
 * of this library runs on the device while this call's kernels run (for
 * example: all linear layers are issued on one stream).  The SM-pair GEMM
 * (ternary weights from 512 tokens) may then share the K blocks of the
 * tiles of its last, partial round (plus one whole round) evenly over all
 * SM pairs (stream-K): a pair whose piece starts inside a tile stores its
 * int32 partial tile in a workspace shared by the device (24 MB of static
 * device memory), and the pair holding the tile's first K blocks adds the
 * partial tiles (exact) before the epilogue.  Concurrent GEMMs would share
 * that workspace, hence the flag.  Results are identical with and without
 * it. */
#define LOWBIT_LINEAR_EXCLUSIVE 2u

/* lowbit_linear_path with launch flags (0 or any of LOWBIT_LINEAR_WEIGHTS_STABLE,
 * LOWBIT_LINEAR_EXCLUSIVE); other flag bits return LOWBIT_ERR_INVALID_ARG.
 * Results are identical for every flag value. */
lowbit_status lowbit_linear_ex(const int8_t *q, int64_t ldq, const float *s_x,
                               int64_t M, int64_t K,
                               const uint8_t *packed, int64_t ldp, const float *s_w,
                               lowbit_format f, int64_t N,
                               void *y, lowbit_dtype ydt, int64_t ldy,
                               int path, unsigned flags,
                               int32_t *status_dev, void *stream);

/* lowbit_bitlinear runs one fused decode kernel when K <= LOWBIT_FUSED_MAX_K
 * and M * K_r <= LOWBIT_FUSED_MAX_BYTES, K_r = K rounded up to a multiple of
 * 128 (the codes of the M tokens are held in shared memory).  Every block
 * of the fused kernel computes the codes it needs; for longer rows that
 * repeated prologue costs more than a separate prologue kernel, measured on
 * B200 (K = 9728, M = 1: 12.4 us fused against 7.1 us for the prologue
 * kernel followed by the GEMV). */
#define LOWBIT_FUSED_MAX_K 1024
#define LOWBIT_FUSED_MAX_BYTES 98304

/* lowbit_bitlinear -- the whole BitLinear forward of M8.8 0x02E on activations
 * x: the prologue of lowbit_act_quant_ex (gain, RMSNorm, Hadamard rotation,
 * per-token codes) followed by lowbit_linear_ex with the given path and
 * flags.  y is identical to calling those two functions in turn.
 *   - Decode: with M <= 4, hadamard == 0, path 0 or 1, K <=
 *     LOWBIT_FUSED_MAX_K and the bound of LOWBIT_FUSED_MAX_BYTES, one fused
 *     kernel runs: while its first weight loads are in flight, every block
 *     computes the codes and scales of the M token rows itself into shared
 *     memory, then streams its packed weight rows (one launch instead of
 *     two, and the codes never go through global memory).  q and s_x may
 *     then be NULL; when given, they receive the codes and scales.
 *   - Otherwise the prologue kernel writes q [M, ldq] and s_x [M] (both
 *     required: device workspace owned by the caller, ldq a multiple of 16,
 *     ldq >= K, q 16-byte aligned), and the linear kernel reads them.
 * Arguments and errors as lowbit_act_quant_ex and lowbit_linear_ex.  With
 * LOWBIT_LINEAR_WEIGHTS_STABLE the packed weights and s_w must not be written
 * by the kernel that precedes this call on the stream. */
lowbit_status lowbit_bitlinear(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                               const float *g, int norm, float eps_norm, int hadamard,
                               const uint8_t *packed, int64_t ldp, const float *s_w, lowbit_format f, int64_t N,
                               void *y, lowbit_dtype ydt, int64_t ldy,
                               int8_t *q, int64_t ldq, float *s_x,
                               int path, unsigned flags, int32_t *status_dev, void *stream);

/* One layer of a grouped decode call (lowbit_bitlinear_group).  Device
 * pointers, all owned by the caller:
 *   x       [M, ldx] token rows of the call's xdt (aligned to its size)
 *   g       [K] fp32 gain or NULL (4-byte aligned)
 *   packed  [N, ldp] packed weights of the call's format (16-byte aligned,
 *           ldp a multiple of 16, ldp >= lowbit_packed_row_bytes(f, K))
 *   s_w     weight scales (lowbit_scale_count(f, N) fp32)
 *   y       [M, ldy] output of the call's ydt, ldy >= N
 *   q, s_x  NULL, or [M, ldq] codes (ldq >= K, multiple of 16, 16-byte
 *           aligned) and [M] fp32 scales that receive the layer's codes. */
typedef struct lowbit_bitlinear_item {
    const void *x;
    int64_t ldx;
    const float *g;
    const uint8_t *packed;
    int64_t ldp;
    const float *s_w;
    int64_t N;
    int64_t K;
    void *y;
    int64_t ldy;
    int8_t *q;
    int64_t ldq;
    float *s_x;
} lowbit_bitlinear_item;

/* Most layers in one lowbit_bitlinear_group call. */
#define LOWBIT_GROUP_MAX 32

/* lowbit_bitlinear_group -- several independent decode BitLinear layers in
 * one persistent GEMV launch (M8.8 0x09B: decode streams whole weight
 * matrices for a few tokens, so the cost of a layer is its packed bytes plus
 * a fixed launch and dependency latency; several layers that read the same
 * or different token rows -- the q, k, v projections, or gate and up, of one
 * block -- share that fixed cost when they run as one kernel).  Each item is
 * computed exactly as lowbit_bitlinear with hadamard = 0 on that item's
 * arguments: codes, scales, int32 sums and outputs are identical to separate
 * calls (the RMSNorm's sum of squares is reduced in the same order).  The
 * layers with K <= LOWBIT_FUSED_MAX_K run in one persistent fused GEMV
 * launch: their rows are cut into units of one block, each resident block
 * takes a contiguous range of units of about equal packed bytes, computes
 * the codes of the layers it touches and streams its units (consecutive
 * layers share a launch while their codes fit 96 KB of shared memory, M *
 * sum of K_r).  Each longer layer runs as lowbit_bitlinear runs it, the
 * prologue kernel then the GEMV (measured faster on B200 than any grouped
 * form for such layers); its q and s_x are then required.
 * items: HOST array of n_items descriptors (read during the call only),
 * 1 <= n_items <= LOWBIT_GROUP_MAX.  M: tokens, 1..4, the same for all items.
 * xdt, norm, eps_norm, f, ydt, flags: shared by all items, with the meanings
 * of lowbit_bitlinear.  Every item needs M * K_r <= LOWBIT_FUSED_MAX_BYTES
 * (K_r = K rounded up to 128) and K <= LOWBIT_PROLOGUE_MAX_K when it has a
 * gain or the norm is on.  The items must be independent: no item's y, q or
 * s_x may overlap another item's inputs or outputs (they are written
 * concurrently).  Errors: invalid or misaligned arguments of any item are
 * reported before anything runs (LOWBIT_ERR_INVALID_ARG,
 * LOWBIT_ERR_ALIGNMENT, LOWBIT_ERR_UNSUPPORTED); device-side conditions
 * (non-finite activations) set bits in *status_dev as lowbit_bitlinear. */
lowbit_status lowbit_bitlinear_group(const lowbit_bitlinear_item *items, int n_items, int64_t M,
                                     lowbit_dtype xdt, int norm, float eps_norm, lowbit_format f,
                                     lowbit_dtype ydt, unsigned flags, int32_t *status_dev, void *stream);

/* Row-parallel layers (M8.8 0x08A-0x08C).  When the input dimension of a
 * layer is split over ranks, each rank holds a slice x[:, k0:k1] of every
 * token row and the packed weights of the same K slice.  The per-token
 * statistics the codes need (max|u| and, with an RMSNorm, the sum of
 * squares) span the whole row, so they are reduced across ranks first; the
 * codes of every slice are then taken with the whole row's maximum, the
 * int32 partial accumulators of the slices are summed (an all-reduce), and
 * one epilogue rescales the sum.  Every value is then identical to the
 * unsplit layer.  The three calls below are the per-rank kernels of that
 * sequence; the collectives in between belong to the caller.  Slice
 * boundaries must be multiples of 128 features and of the Hadamard block. */

/* lowbit_act_row_stats -- per token row of the slice: row_max[t] = max_k |u|
 * (u = x * g, rotated in Hadamard blocks when hadamard > 0, as in
 * lowbit_act_quant_ex) as fp32, and, when row_ss is not NULL, row_ss[t] =
 * sum_k x_k^2 in fp64 (the RMSNorm's sum of squares).  row_max: device fp32
 * [M]; row_ss: device fp64 [M] or NULL.  K <= LOWBIT_PROLOGUE_MAX_K.  A
 * non-finite u sets LOWBIT_ERR_NONFINITE. */
lowbit_status lowbit_act_row_stats(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                   const float *g, int hadamard, float *row_max, double *row_ss,
                                   int32_t *status_dev, void *stream);

/* lowbit_act_quant_given_max -- the int8 codes of a row slice with the whole
 * row's maximum: q = clip(rint((u * 127) / row_max[t]), -128, 127) (fp32
 * multiply and IEEE divide, nearest even; row_max[t] == 0 gives zero codes).
 * A slice value above the maximum it was given sets LOWBIT_ERR_INVALID_ARG in
 * *status_dev. */
lowbit_status lowbit_act_quant_given_max(const void *x, lowbit_dtype xdt, int64_t M, int64_t K, int64_t ldx,
                                         const float *g, int hadamard, const float *row_max,
                                         int8_t *q, int64_t ldq, int32_t *status_dev, void *stream);

/* lowbit_act_scales -- s_x of lowbit_act_quant_ex from whole-row statistics:
 * s_x[t] = row_max[t] / sqrt(hadamard) / rms / 127 (fp64, rounded once),
 * rms = sqrt(row_ss[t] / K_total + eps_norm) with LOWBIT_NORM_RMS (row_ss
 * then required), 1 otherwise; row_max[t] == 0 gives 0. */
lowbit_status lowbit_act_scales(const float *row_max, const double *row_ss, int64_t M, int64_t K_total, int norm,
                                float eps_norm, int hadamard, float *s_x, int32_t *status_dev, void *stream);

/* lowbit_rescale -- the epilogue of lowbit_linear on given int32
 * accumulators acc [M, ldacc]: y = float(acc) * (s_w[n or 0] * s_x[t]) in
 * fp32, or rounded to bf16, or acc itself (LOWBIT_I32); s_w holds
 * lowbit_scale_count(f, N) values.  y [M, ldy], ldy >= N. */
lowbit_status lowbit_rescale(const int32_t *acc, int64_t ldacc, int64_t M, int64_t N, const float *s_x,
                             const float *s_w, lowbit_format f, void *y, lowbit_dtype ydt, int64_t ldy,
                             int32_t *status_dev, void *stream);

/* The kernels lowbit_linear_path can launch. */
typedef enum {
    LOWBIT_KERNEL_GEMV = 1,           /* packed-weight GEMV (dp4a), groups of up to 4 tokens */
    LOWBIT_KERNEL_WARP_MMA = 2,       /* warp-level mma.sync on register weight fragments */
    LOWBIT_KERNEL_GEMM = 3,           /* tcgen05 GEMM, expanded weight tile in shared memory */
    LOWBIT_KERNEL_GEMM_SPLITK = 4,    /* the same with K split over a cluster of 2, 4 or 8 CTAs */
    LOWBIT_KERNEL_GEMM_PAIR = 5,      /* tcgen05 GEMM on SM pairs, tile in shared memory */
    LOWBIT_KERNEL_GEMM_TMEM = 6,      /* tcgen05 GEMM, expanded weight tile in tensor memory */
    LOWBIT_KERNEL_GEMM_TMEM_PAIR = 7  /* the same on SM pairs */
} lowbit_kernel;

/* The kernel lowbit_linear_path(..., path, ...) launches for an M x K by
 * K -> N problem in format f, on a GPU with sm_count SMs (sm_count <= 0: the
 * current device, which must be a B200).  Host only: no launch and no device
 * memory, so with sm_count > 0 it needs no GPU.  `kernel` is a HOST pointer
 * (the one exception to the device-pointer convention above).  Writes *kernel
 * and returns
 * LOWBIT_OK; returns the status lowbit_linear_path would return for the
 * shape (LOWBIT_ERR_INVALID_ARG for M, N or K <= 0, a path outside 0..6, path
 * 5 with M > 16 or a null kernel; LOWBIT_ERR_OVERFLOW_BOUND for K above
 * lowbit_max_k), or LOWBIT_ERR_CUDA / LOWBIT_ERR_UNSUPPORTED when sm_count <= 0
 * and the device cannot be queried or is not a B200. */
lowbit_status lowbit_linear_kernel(int64_t M, int64_t N, int64_t K, lowbit_format f, int path,
                                   int sm_count, lowbit_kernel *kernel);

/* Name of the kernel function(s) behind a lowbit_kernel value, as in a
 * profiler's launch list (static string; "unknown" for other values). */
const char *lowbit_kernel_name(lowbit_kernel k);

/* lowbit_set_wait_limit -- the bound, in SM clock cycles, of every pipeline
 * wait in the tensor-core kernels on the current device (the default,
 * restored by cycles <= 0, is 4e9 cycles, about 2 s).  When a wait runs past
 * it, the kernel sets LOWBIT_ERR_TIMEOUT in *status_dev, lets the copies and
 * tensor-core operations it already issued complete, frees its tensor
 * memory and returns; that launch's output is unspecified and the context
 * stays usable.  Failure-detection tests lower the bound to make a wait run
 * out.  Synchronous (a copy to device memory); call it with no kernel of this
 * library in flight on the device. */
lowbit_status lowbit_set_wait_limit(int64_t cycles);

/* Human-readable name of a status value (static string). */
const char *lowbit_status_string(lowbit_status s);

/* Library version as major*10000 + minor*100 + patch. */
int lowbit_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOWBIT_H */
