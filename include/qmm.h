/*
 * qmm.h -- C ABI of the block-quantized weight matmul library (libqmm.so).
 *
 * The library runs LLM inference matmuls directly on ggml-style block-quantized
 * weights on an NVIDIA B200 (sm_100a). Weights are never dequantized to a
 * separate buffer: each kernel decodes the blocks as it streams them.
 *
 * ---------------------------------------------------------------------------
 * Block formats (ggml style; weights stay in this layout end to end --
 * "Lumen v0.2.0 -- Q8-native decode", section "Phase 7.D -- Q8-native fused
 * matmul"):
 *
 *   Q8_0 (34 bytes / 32 weights): uint16 d (IEEE fp16 bits, little-endian),
 *        then int8 qs[32]. Weight j = qs[j] * d.
 *   Q4_0 (18 bytes / 32 weights): uint16 d (fp16 bits), then uint8 qs[16].
 *        Weight j (j < 16) = ((qs[j] & 15) - 8) * d,
 *        weight j+16      = ((qs[j] >> 4) - 8) * d.
 *
 * A weight matrix W holds N rows (output features) of K/32 blocks each,
 * row-major, K contiguous: block b of row n starts at byte
 * (n * (K/32) + b) * block_bytes. There is no padding between rows.
 *
 * Dense operands are row-major: X[m][k] at X + m*K + k, Y[m][n] at Y + m*N + n.
 * Every matmul computes Y[m][n] = sum_k X[m][k] * W[n][k].
 *
 * ---------------------------------------------------------------------------
 * Conventions shared by every entry point:
 *   - All buffer pointers are DEVICE pointers owned by the caller. The library
 *     allocates no memory and frees none.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; nothing synchronises the host.
 *   - Arguments are validated on the host before any CUDA call. A call that
 *     returns an error has launched nothing and written nothing.
 *   - `block` must be 32 (QMM_ERR_BLOCK otherwise).
 *   - Sizes are int64_t. Negative sizes are QMM_ERR_SHAPE. M == 0 or N == 0 is
 *     a valid empty call that launches nothing. K must be a multiple of 32;
 *     K == 0 makes every output an empty sum (written as 0; the gate/up
 *     output is silu(0) * 0 = 0).
 *   - A pointer may be NULL only if the buffer it names is empty.
 *   - W, Wg, Wu, X and QX must be 16-byte aligned; Y and DX 4-byte aligned
 *     (QMM_ERR_ALIGN). torch / cudaMalloc allocations satisfy both.
 *   - Inputs are assumed finite; NaN / Inf propagation is unspecified.
 *   - The device must be compute capability 10.0 (B200 class); otherwise
 *     QMM_ERR_DEVICE.
 *   - Launch failures are returned as QMM_ERR_CUDA with the CUDA error text in
 *     qmm_last_error_string().
 *   - A kernel that waits too long on one of its own pipeline barriers (about
 *     two seconds) stops, records the fact in a device status word and returns
 *     instead of hanging; qmm_device_status() reads and clears that word.
 *   - Calls are thread-safe. What persists between calls is a once-per-device
 *     kernel attribute set-up and the device status words that
 *     qmm_device_status() reads and clears; no call's result depends on them.
 *
 * Tolerances the library is tested to (per output, S = sum_k |w_k * x_k|):
 *   fp32-accumulated paths: |y - exact| <= 1e-5 * S;
 *   bf16 tensor-core prefill above 32 tokens: |y - exact| <= 4e-3 * S
 *   (up to 32 tokens the prefill path is held to 1e-5 * S);
 *   activation codes and int32 block dots: bit-exact.
 */
#ifndef QMM_H
#define QMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define QMM_API __attribute__((visibility("default")))
#else
#define QMM_API
#endif

struct CUstream_st; /* cudaStream_t == struct CUstream_st * */
typedef struct CUstream_st *qmm_stream_t;

typedef enum {
  QMM_OK = 0,
  QMM_ERR_NULL = 1,         /* required pointer is NULL                       */
  QMM_ERR_SHAPE = 2,        /* negative size, K % 32 != 0, M or K too large  */
  QMM_ERR_BLOCK = 3,        /* block != 32                                    */
  QMM_ERR_ALIGN = 4,        /* pointer not aligned as documented              */
  QMM_ERR_DTYPE = 5,        /* unknown weight type                            */
  QMM_ERR_DEVICE = 6,       /* current device is not compute capability 10.x  */
  QMM_ERR_CUDA = 7,         /* a CUDA runtime call failed                      */
  QMM_ERR_DEVICE_CHECK = 8  /* a kernel recorded a device-side failure         */
} qmm_status;

typedef enum { QMM_Q8_0 = 0, QMM_Q4_0 = 1 } qmm_wtype;

#define QMM_BLOCK 32
#define QMM_Q8_0_BLOCK_BYTES 34
#define QMM_Q4_0_BLOCK_BYTES 18
/* Largest M of the decode entry points (qmm_q8_gemv, qmm_q8q8_gemv,
 * qmm_q4_swiglu_gateup). */
#define QMM_MAX_DECODE_M 8
/* Largest K of every entry point. */
#define QMM_MAX_K 32768
/* Most projections per qmm_q8_gemv_multi call. */
#define QMM_MAX_PROJ 4

/* Option of the *_ex entry points: start streaming the weight blocks before
 * the preceding kernel in the stream has finished (programmatic dependent
 * launch; activations are still read only after it has finished). Only valid
 * when that preceding kernel does not write the weight buffer -- true for
 * model weights, which are written once at load time. */
#define QMM_FLAG_EARLY_WEIGHTS 1u

/*
 * qmm_q8_gemv -- decode GEMV / small-M matmul on Q8_0 weights, fp32 activations.
 *
 * Defined by "Lumen v0.2.0 -- Q8-native decode", section "Phase 7.D --
 * Q8-native fused matmul": the per-block fp16 scale d is broadcast over its 32
 * weights, the K direction is reduced block by block and one output per row is
 * written; there is no load-time dequantisation.
 *
 *   Y[m][n] = sum_b d[n][b] * sum_j qs[n][b][j] * X[m][32b + j]   (fp32 accumulation)
 *
 *   M      1 .. QMM_MAX_DECODE_M tokens (0 = empty call)
 *   N      output features (rows of W), >= 0
 *   K      reduction length, multiple of 32, <= QMM_MAX_K
 *   W      N * K/32 Q8_0 blocks (device, read only, 16-byte aligned)
 *   X      M x K fp32 (device, read only, 16-byte aligned)
 *   Y      M x N fp32 (device, written)
 */
QMM_API qmm_status qmm_q8_gemv(int64_t M, int64_t N, int64_t K, int block, const void *W,
                               const float *X, float *Y, qmm_stream_t stream);

/* qmm_q8_gemv with options: flags is 0 or QMM_FLAG_EARLY_WEIGHTS (unknown bits
 * are QMM_ERR_SHAPE). qmm_q8_gemv(...) == qmm_q8_gemv_ex(..., 0, stream). */
QMM_API qmm_status qmm_q8_gemv_ex(int64_t M, int64_t N, int64_t K, int block, const void *W,
                                  const float *X, float *Y, uint32_t flags, qmm_stream_t stream);

/*
 * qmm_quantize_act_q8_0 -- quantise fp32 activations into ggml Q8_0 blocks
 * (34 bytes: fp16 scale d, then 32 int8 codes), the block format of the
 * weights, so that quantised activations interchange with ggml's.
 *
 * The activation-quantisation step of "Lumen v0.4.0", section "Phase 7.M --
 * Q8xQ8 AVX2 int dot", with the scale kept at fp16 and ggml's reference rule
 * for the codes: amax = max_j |x_j|; d = amax / 127; id = 1 / d (0 when d ==
 * 0); q_j = round-half-away-from-zero(x_j * id); each an IEEE binary32
 * operation; the block stores binary16(d), rounded to nearest even (scales
 * above 65504 become infinity, as in an fp16 conversion). Codes and scales are
 * bit-exact functions of X. This differs from qmm_quantize_act_q8, which keeps
 * d in fp32 and divides x_j / d.
 *
 *   M, K   rows and row length (K multiple of 32); M >= 0
 *   X      M x K fp32 (device, 16-byte aligned)
 *   XB     M x K/32 Q8_0 blocks, M * (K/32) * 34 bytes (device, 16-byte aligned, written)
 */
QMM_API qmm_status qmm_quantize_act_q8_0(int64_t M, int64_t K, int block, const float *X, void *XB,
                                         qmm_stream_t stream);

/*
 * qmm_q8q8_gemv_q8_0 -- qmm_q8q8_gemv with the activations as Q8_0 blocks
 * (fp16 scales), e.g. from qmm_quantize_act_q8_0 or from ggml:
 *
 *   Y[m][n] = sum_b (d[n][b] * dx[m][b]) * sum_j qs[n][b][j] * qx[m][b][j]   (exact int32 dots)
 *
 *   M      1 .. QMM_MAX_DECODE_M (0 = empty call)
 *   W      N * K/32 Q8_0 blocks (16-byte aligned)
 *   XB     M * K/32 Q8_0 blocks (16-byte aligned)
 *   Y      M x N fp32 (written)
 *   flags  0 or QMM_FLAG_EARLY_WEIGHTS
 */
QMM_API qmm_status qmm_q8q8_gemv_q8_0(int64_t M, int64_t N, int64_t K, int block, const void *W, const void *XB,
                                      float *Y, uint32_t flags, qmm_stream_t stream);

/*
 * qmm_q8_gemv_auto -- the per-K choice between the fp32-activation GEMV and
 * the Q8xQ8 GEMV ("Lumen v0.4.0", section "Phase 7.P -- per-shape hybrid
 * dispatch": short-K matmuls on the quantised-activation integer path, long-K
 * ones on the fp32 path). Opt-in: the result depends on K.
 *
 * At M = 1 with K/32 <= 64 blocks, when each CTA's weight slice fits on chip,
 * this is qmm_q8q8_gemv_fused (Y is the Q8xQ8 product of the activations
 * quantised per 32-block, and QX / DX receive their codes and scales);
 * otherwise it is qmm_q8_gemv_ex (fp32 activations; QX / DX untouched). The
 * rule was measured on B200 in chains of dependent launches: 896 -> 4864
 * takes 2.09 us as Q8xQ8 and 2.81 us as fp32; 4864 -> 896 takes 3.56 us and
 * 3.39 us.
 *
 *   M, N, K, block, W, X, Y, flags   as qmm_q8_gemv_ex
 *   QX, DX   M x K int8 (16-byte aligned) and M x K/32 fp32, caller-owned
 *            (always required; written only by the Q8xQ8 form)
 */
QMM_API qmm_status qmm_q8_gemv_auto(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                                    float *Y, int8_t *QX, float *DX, uint32_t flags, qmm_stream_t stream);

/*
 * qmm_q8_gemv_multi -- several Q8_0 projections of the same activations in
 * one launch: Y_i = X . dequant(W_i)^T for i < nproj, each the qmm_q8_gemv
 * product of its matrix (same formula, same tolerance).
 *
 * "LSE v0.4.15", section "Changes" (several projections fed by one shared
 * activation producer in one launch, instead of one launch per projection).
 * At M = 1 and K <= 2048 the row chunks of all matrices form one work list
 * of a single launch of the integer tensor-core streaming kernel; otherwise
 * the call issues one qmm_q8_gemv launch per projection.
 *
 *   M         1 .. QMM_MAX_DECODE_M (0 = empty call)
 *   K         shared row length (multiple of 32)
 *   nproj     1 .. QMM_MAX_PROJ
 *   N, W, Y   HOST arrays of nproj entries: rows of projection i, its
 *             N[i] * K/32 Q8_0 blocks (device, 16-byte aligned) and its
 *             M x N[i] fp32 output (device); N[i] = 0 skips projection i
 *   X         M x K fp32 (device, 16-byte aligned)
 *   flags     0 or QMM_FLAG_EARLY_WEIGHTS
 */
QMM_API qmm_status qmm_q8_gemv_multi(int64_t M, int64_t K, int block, int nproj, const int64_t *N,
                                     const void *const *W, const float *X, float *const *Y, uint32_t flags,
                                     qmm_stream_t stream);

/*
 * qmm_quantize_act_q8 -- quantise fp32 activations to Q8 codes per 32-block.
 *
 * The activation-quantisation step of the Q8xQ8 path ("Lumen v0.4.0 --
 * shape-aware VNNI/fp32 hybrid dispatch", section "Phase 7.M -- Q8xQ8 AVX2 int
 * dot"). For every block of 32 consecutive activations of a row:
 *   amax = max_j |x_j|;  d = amax / 127  (IEEE binary32 division, round to nearest even);
 *   q_j  = round_half_away_from_zero(x_j / d)  (binary32 division), clamped to [-127, 127];
 *   if d == 0, every q_j = 0.
 *
 *   M, K   rows and row length (K multiple of 32, <= QMM_MAX_K); M >= 0
 *   X      M x K fp32 (device, read only, 16-byte aligned)
 *   QX     M x K int8 codes (device, written, 16-byte aligned)
 *   DX     M x K/32 fp32 scales d (device, written)
 * The codes and scales are bit-exact functions of X.
 */
QMM_API qmm_status qmm_quantize_act_q8(int64_t M, int64_t K, int block, const float *X, int8_t *QX,
                               float *DX, qmm_stream_t stream);

/*
 * qmm_q8q8_gemv -- Q8_0 weights times Q8-quantised activations.
 *
 * "Lumen v0.4.0", section "Phase 7.M -- Q8xQ8 AVX2 int dot": each block's dot
 * product of int8 weight codes and int8 activation codes is an exact int32,
 * which is then scaled by both block scales and accumulated in fp32:
 *
 *   isum[m][n][b] = sum_j qs[n][b][j] * QX[m][32b + j]           (exact int32)
 *   Y[m][n]       = sum_b (d[n][b] * DX[m][b]) * isum[m][n][b]   (fp32)
 *
 *   M      1 .. QMM_MAX_DECODE_M (0 = empty call)
 *   W      N * K/32 Q8_0 blocks (16-byte aligned); QX M x K int8 (16-byte
 *          aligned); DX M x K/32 fp32 -- as written by qmm_quantize_act_q8
 *   Y      M x N fp32 (written)
 */
QMM_API qmm_status qmm_q8q8_gemv(int64_t M, int64_t N, int64_t K, int block, const void *W,
                         const int8_t *QX, const float *DX, float *Y, qmm_stream_t stream);

/* qmm_q8q8_gemv with options (0 or QMM_FLAG_EARLY_WEIGHTS). */
QMM_API qmm_status qmm_q8q8_gemv_ex(int64_t M, int64_t N, int64_t K, int block, const void *W,
                                    const int8_t *QX, const float *DX, float *Y, uint32_t flags,
                                    qmm_stream_t stream);

/*
 * qmm_q8q8_gemv_fused -- qmm_quantize_act_q8 followed by qmm_q8q8_gemv as one
 * call: the per-block activation quantisation of "Lumen v0.4.0", section
 * "Phase 7.M -- Q8xQ8 AVX2 int dot", done inside the GEMV (at M = 1, when each
 * CTA's weight slice fits on chip, every CTA quantises X itself; otherwise a
 * quantisation launch precedes the streaming Q8xQ8 launch).
 *
 *   M       1 .. QMM_MAX_DECODE_M (0 = empty call)
 *   W       N * K/32 Q8_0 blocks (16-byte aligned)
 *   X       M x K fp32 (16-byte aligned, read only)
 *   QX, DX  M x K int8 (16-byte aligned) and M x K/32 fp32, written with the
 *           codes and scales qmm_quantize_act_q8 writes for X (bit for bit),
 *           so other Q8xQ8 calls on the same X can reuse them; caller-owned,
 *           the call allocates nothing
 *   Y       M x N fp32 (written), the qmm_q8q8_gemv formula
 *   flags   0 or QMM_FLAG_EARLY_WEIGHTS
 */
QMM_API qmm_status qmm_q8q8_gemv_fused(int64_t M, int64_t N, int64_t K, int block, const void *W,
                                       const float *X, int8_t *QX, float *DX, float *Y, uint32_t flags,
                                       qmm_stream_t stream);

/*
 * qmm_q4_swiglu_gateup -- fused gate/up projection with SwiGLU on Q4_0 weights.
 *
 * "LSE v0.4.16", section "Combined M8 Q4 gate/up execution": one launch reads
 * one shared activation panel X, accumulates the gate and up projections in
 * independent fp32 accumulators and writes only
 *
 *   Y[m][n] = silu(g) * u,  g = sum_k X[m][k] Wg[n][k],  u = sum_k X[m][k] Wu[n][k],
 *   silu(g) = g / (1 + exp(-g)).
 *
 * No gate (or up) temporary is written to memory.
 *
 *   M       1 .. QMM_MAX_DECODE_M (0 = empty call)
 *   Wg, Wu  N * K/32 Q4_0 blocks each (16-byte aligned)
 *   X       M x K fp32 (16-byte aligned)
 *   Y       M x N fp32 (written)
 */
QMM_API qmm_status qmm_q4_swiglu_gateup(int64_t M, int64_t N, int64_t K, int block, const void *Wg,
                                const void *Wu, const float *X, float *Y, qmm_stream_t stream);

/* qmm_q4_swiglu_gateup with options (0 or QMM_FLAG_EARLY_WEIGHTS). */
QMM_API qmm_status qmm_q4_swiglu_gateup_ex(int64_t M, int64_t N, int64_t K, int block, const void *Wg,
                                           const void *Wu, const float *X, float *Y, uint32_t flags,
                                           qmm_stream_t stream);

/*
 * qmm_q4_gemv -- decode GEMV / small-M matmul on Q4_0 weights, fp32 activations.
 *
 * The Q4_0 counterpart of qmm_q8_gemv, for the rest of a Q4 model's matmul
 * set: the M8 Q4 down projection that "LSE v0.4.16" keeps on its matrix
 * cores (section "Retained optimizations and compatibility") and the Q4-native
 * matmul that "Lumen v0.5.0" lists in its section "What's next":
 *
 *   Y[m][n] = sum_b d[n][b] * sum_j (q[n][b][j] - 8) * X[m][32b + j]   (fp32 accumulation)
 *
 * For M >= 2 (and M = 1 with K not a multiple of 256, or K > 7680) it runs the
 * fused gate/up kernel with one matrix, so each output equals the
 * corresponding gate (or up) projection of qmm_q4_swiglu_gateup's unfused form
 * bit for bit. M = 1 otherwise runs the integer tensor-core GEMV on the raw
 * codes (the activations as base-256 digits, as in qmm_q8_gemv's lm_head
 * form); the result is within the same fp32 tolerance, not bit-equal to the
 * gate/up kernel's.
 *
 *   M      1 .. QMM_MAX_DECODE_M (0 = empty call)
 *   W      N * K/32 Q4_0 blocks (16-byte aligned)
 *   X      M x K fp32 (16-byte aligned)
 *   Y      M x N fp32 (written)
 *   flags  0 or QMM_FLAG_EARLY_WEIGHTS
 */
QMM_API qmm_status qmm_q4_gemv(int64_t M, int64_t N, int64_t K, int block, const void *W, const float *X,
                               float *Y, uint32_t flags, qmm_stream_t stream);

/*
 * qmm_quant_matmul_prefill -- prefill panel Y = X . W^T on the tensor cores.
 *
 * "LSE v0.4.16", section "Retained optimizations and compatibility" (M1024
 * prefill panels): a many-token matmul against block-quantized weights.
 * Above 32 tokens the blocks are decoded to bf16 (w = q*d rounded to nearest
 * even) and multiplied by the bf16 activations with fp32 accumulation on the
 * tcgen05 tensor cores (|y - exact| <= 4e-3 * S). Up to 32 tokens a small-M
 * kernel multiplies the exact integer codes by the activations (mma.sync,
 * fp32 accumulation) and applies each block's d in fp32, so no decoded weight
 * is rounded (|y - exact| <= 1e-5 * S). qmm_prefill_plan tells which runs.
 *
 *   wtype   QMM_Q8_0 or QMM_Q4_0 (QMM_ERR_DTYPE otherwise)
 *   M       tokens, >= 0
 *   W       N * K/32 blocks of `wtype` (16-byte aligned)
 *   X       M x K bf16 bit patterns (uint16_t, 16-byte aligned)
 *   Y       M x N fp32 (written)
 */
QMM_API qmm_status qmm_quant_matmul_prefill(int wtype, int64_t M, int64_t N, int64_t K, int block,
                                    const void *W, const uint16_t *X, float *Y,
                                    qmm_stream_t stream);

/* qmm_quant_matmul_prefill with options (0 or QMM_FLAG_EARLY_WEIGHTS: the
 * weight blocks are streamed and decoded before the preceding kernel in the
 * stream has finished; X is loaded and Y written only after it). */
QMM_API qmm_status qmm_quant_matmul_prefill_ex(int wtype, int64_t M, int64_t N, int64_t K, int block,
                                               const void *W, const uint16_t *X, float *Y, uint32_t flags,
                                               qmm_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Test and utility exports (not on the hot path).                           */

/*
 * qmm_q8q8_block_dots -- the exact int32 block dots of qmm_q8q8_gemv, written
 * out: isum[(m*N + n)*(K/32) + b] (M x N x K/32 int32, device, written).
 * Computed by the same device code as qmm_q8q8_gemv; used to test the integer
 * part bit-exactly.
 */
QMM_API qmm_status qmm_q8q8_block_dots(int64_t M, int64_t N, int64_t K, int block, const void *W,
                               const int8_t *QX, int32_t *isum, qmm_stream_t stream);

/*
 * qmm_q8q8_gemv_fused_dots -- qmm_q8q8_gemv_fused with its exact int32 block
 * dots written out as well: isum[n*(K/32) + b] for M = 1, in general
 * isum[(m*N + n)*(K/32) + b] (M x N x K/32 int32, device, written). The
 * kernel choice is qmm_q8q8_gemv_fused's; where that is the resident kernel,
 * its dump instance runs (the same arithmetic plus the store of each dot), so
 * the per-block integer part of the fused path ("Lumen v0.4.0", section
 * "Phase 7.M -- Q8xQ8 AVX2 int dot") can be tested bit for bit. Y, QX and DX
 * are written exactly as by qmm_q8q8_gemv_fused. No options (no early
 * weights).
 */
QMM_API qmm_status qmm_q8q8_gemv_fused_dots(int64_t M, int64_t N, int64_t K, int block, const void *W,
                                            const float *X, int8_t *QX, float *DX, float *Y, int32_t *isum,
                                            qmm_stream_t stream);

/*
 * qmm_q8q8_block_dots_q8_0 -- the exact int32 block dots of
 * qmm_q8q8_gemv_q8_0 (activations as Q8_0 blocks XB), written out as
 * isum[(m*N + n)*(K/32) + b]; the same device code as that entry point's.
 */
QMM_API qmm_status qmm_q8q8_block_dots_q8_0(int64_t M, int64_t N, int64_t K, int block, const void *W,
                                            const void *XB, int32_t *isum, qmm_stream_t stream);

/*
 * qmm_test_withheld_copy -- exercises the bounded-wait failure path (the
 * "guards" of "LSE v0.4.15", section "Qualification and measurements") without
 * any fault: one kernel launch in which CTA 0 never issues one of its copies,
 * so its waits on that copy give up after wait_ns nanoseconds (1e3 .. 2e9).
 *   kernel 0: the streaming Q8_0 GEMV (M 1..8, X fp32); the first weight
 *             stage of CTA 0 is withheld.
 *   kernel 1: the small-M prefill kernel on Q8_0 weights (M 1..32, X bf16;
 *             QMM_ERR_SHAPE unless qmm_prefill_plan reports that kernel);
 *             the whole weight copy of CTA 0 (cluster rank 0) is withheld, and
 *             with split K the other ranks still meet it at the cluster
 *             barrier.
 * The starved CTA records kDevTimeout bits in the device status word,
 * finishes without touching the withheld buffer and returns; the outputs it
 * owns are left unwritten or undefined, the others are computed as usual.
 * qmm_device_status() then reports the bits (QMM_ERR_DEVICE_CHECK) and clears
 * them; later calls are unaffected. Not for production use.
 */
QMM_API qmm_status qmm_test_withheld_copy(int kernel, int64_t M, int64_t N, int64_t K, int block, const void *W,
                                          const void *X, float *Y, uint64_t wait_ns, qmm_stream_t stream);

/*
 * qmm_q4_gateup_unfused -- the unfused counterpart of qmm_q4_swiglu_gateup:
 * writes the gate and up projections G, U (M x N fp32 each) with two separate
 * projection launches, then Y = silu(G) * U with a third launch. Each
 * projection uses the same accumulation code and order as the fused kernel,
 * so Y matches qmm_q4_swiglu_gateup bit for bit ("LSE v0.4.16", section
 * "Combined M8 Q4 gate/up execution": exact outputs preserved).
 */
QMM_API qmm_status qmm_q4_gateup_unfused(int64_t M, int64_t N, int64_t K, int block, const void *Wg,
                                 const void *Wu, const float *X, float *G, float *U, float *Y,
                                 qmm_stream_t stream);

/*
 * qmm_prefill_plan -- the tiling qmm_quant_matmul_prefill would launch on the
 * current device for this problem, without launching anything:
 * plan[0] = tokens per output tile (MT; above 256 each k step takes two
 * MMAs), plan[1] = K ranges per tile (thread-block cluster size, 1 = no
 * split), plan[2] = MMA stages in flight (0 for the small-M kernel),
 * plan[3] = CTAs of the launch, plan[4] = the kernel: 0 = tcgen05 tiles with
 * the A operand in tensor memory, 1 = the small-M kernel (M <= 32: each CTA's
 * weight share and X slice in shared memory, mma.sync bf16).
 * Host memory `plan` (5 int32, written). Needs an sm_100 device
 * (QMM_ERR_DEVICE otherwise); M, N >= 1, K >= 32 (QMM_ERR_SHAPE).
 */
QMM_API qmm_status qmm_prefill_plan(int wtype, int64_t M, int64_t N, int64_t K, int block, int32_t *plan);

/* Text of the last error raised on the calling host thread ("" if none). */
QMM_API const char *qmm_last_error_string(void);

/* Library version string, e.g. "qmm 0.1.0 sm_100a". */
QMM_API const char *qmm_version(void);

/*
 * qmm_device_status -- synchronises the current device, then reads and clears
 * the device-side status words that kernels set when a bounded wait gives up.
 * *bits receives their OR (0 = no failure recorded; 1 = a copy or stage never
 * arrived, 2 = a copy in flight could not be drained on the error path, 4 = a
 * tensor-core commit never arrived). Returns QMM_OK when *bits == 0,
 * QMM_ERR_DEVICE_CHECK when a failure was recorded, or QMM_ERR_CUDA if the
 * synchronisation itself failed.
 */
QMM_API qmm_status qmm_device_status(uint32_t *bits);

#ifdef __cplusplus
}
#endif

#endif /* QMM_H */
