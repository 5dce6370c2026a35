/*
 * rbd.h -- C ABI of the rotated low-bit quantized linear layer (B200, sm_100a).
 *
 * The layer (as described on the Krea-2 model cards):
 *   - bf16 activations are rotated online, group-wise, by a 256-wide regular
 *     Hadamard matrix and quantised per token inside the kernel
 *     ("Krea-2 Turbo -- INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)",
 *     header paragraph);
 *   - weights are rotated the same way and packed offline to signed INT4, or
 *     kept as per-row INT8 for the protected ff.down layers
 *     ("Krea 2 Turbo OrbitQuant W4A4", sections "Fused transformer" and
 *     "What is quantized");
 *   - the low-bit GEMM accumulates in int32; scales, bias, an optional
 *     SVDQuant-style low-rank branch and a sigmoid gate or gated residual are
 *     applied in the epilogue ("Fused transformer"; "Krea-2-SVDQuant-ComfyUI",
 *     sections "Why this exists" and "LoRA");
 *   - group-64 scales follow "Krea 2 Turbo Nunchaku Lite INT4 r32", header.
 *
 * Conventions for every entry point:
 *   - Pointers named x, w, codes, scales, y, ... are DEVICE pointers owned by
 *     the caller; the library allocates no device memory and never frees.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued asynchronously on it; no call synchronises the host except
 *     rbd_check().
 *   - bf16 tensors are passed as `const void*` holding IEEE bfloat16 bits.
 *   - All matrices are row-major.  ld* arguments are row strides in elements.
 *   - Arguments are validated on the host before anything is launched.  An
 *     invalid call returns a non-zero rbd_status and launches nothing.  There
 *     is no fallback path: an unsupported shape or mode is an error.
 *   - A kernel whose bounded wait expires records RBD_ERR_DEVICE_TIMEOUT in a
 *     device status word; rbd_check() reports (and clears) it.
 */
#ifndef RBD_H_
#define RBD_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rbd_status {
  RBD_OK = 0,
  RBD_ERR_INVALID_ARG = 1,    /* null pointer, bad size or inconsistent arguments */
  RBD_ERR_UNSUPPORTED = 2,    /* valid request this library does not implement   */
  RBD_ERR_ALIGNMENT = 3,      /* pointer or stride not 16-byte aligned           */
  RBD_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed               */
  RBD_ERR_DEVICE_TIMEOUT = 5  /* a device-side bounded wait expired              */
} rbd_status;

/* How activation codes are stored, one code per byte either way.  The codes
 * themselves (the integers) are the same; only the byte that holds one differs.
 *   RBD_CODES_INT8  the code as a two's-complement int8.
 *   RBD_CODES_E4M3  the code as the E4M3 (8-bit float, 4 exponent and 3
 *                   mantissa bits, bias 7) value equal to it; every INT4 code
 *                   is exact in E4M3.  4-bit codes only.  rbd_w4a4_linear
 *                   with group-64 scales runs these on the FP8 tensor-core
 *                   path (fp32 group partials, exact for 64-wide groups).    */
typedef enum rbd_code_format {
  RBD_CODES_INT8 = 0,
  RBD_CODES_E4M3 = 1
} rbd_code_format;

/* Quantisation configuration.
 *   bits        4 (signed INT4, codes in [-8,7], produced range [-7,7]) or
 *               8 (signed INT8, produced range [-127,127]).
 *   rot_group   256: rotate every 256-wide K block by R = H/16, H the regular
 *               Hadamard matrix (J4 - 2 I4) Kronecker-powered four times;
 *               0: no rotation.
 *   scale_group 0: one scale per row (per token for activations, per output
 *               channel for weights); 64: one scale per 64-wide K block of a
 *               row (group-64 scales).
 *   code_format an rbd_code_format: how activation codes are stored (written
 *               by the quantisers, read by the linears).  Weight packers take
 *               RBD_CODES_INT8 only.  RBD_CODES_E4M3 needs bits == 4 (else
 *               RBD_ERR_UNSUPPORTED); the linears take it with group-64 scales
 *               only.  Zero-initialising the struct selects RBD_CODES_INT8.  */
typedef struct rbd_qcfg {
  int32_t bits;
  int32_t rot_group;
  int32_t scale_group;
  int32_t code_format;
} rbd_qcfg;

/* Online activation rotate + dynamic quantise (INT4 tensorwise card, header:
 * the activation rotation happens at run time and the quantisation scales are
 * computed by the kernel itself).
 *   x       bf16 [M, ldx], first K columns used.  ldx >= K, ldx % 8 == 0,
 *           x 16-byte aligned.
 *   M       >= 0 (M == 0 is a no-op).   K: multiple of 256 (rotation) or of 64,
 *           K <= 16384.
 *   codes   [M, K], one code per byte in cfg.code_format (two's-complement
 *           int8, or the equal E4M3 value for 4-bit codes), 16-byte aligned.
 *   scales  float32 [M] (scale_group 0) or [M, K/64] (scale_group 64);
 *           dequantised value = code * scale.
 * Per row (or per 64 block): amax = max |xr|, scale = amax/qmax,
 * code = clamp(rint_even(xr * (qmax/amax))), all float32 IEEE operations, xr the
 * exact rotated value rounded once to float32.  An all-zero row or block gets
 * scale 0 and codes 0.                                                         */
rbd_status rbd_rot_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, rbd_qcfg cfg,
                             int8_t* codes, float* scales, void* stream);

/* RMSNorm and adaLN-style modulation fused ahead of rbd_rot_quant_act
 * (Krea 2 Turbo OrbitQuant W4A4, "Fused transformer": the norm and the
 * modulation are folded into the kernels that quantise activations).  Per row:
 *   r = 1 / sqrt(sum_k x_k^2 / K + eps), float64 IEEE operations on the exact
 *       squares, rounded once to float32 (r = 0 when the radicand is 0);
 *   per element, single float32 operations in this order:
 *       u = x * r;  u = u * gamma[k];  u = u * (1 + scale[k]);  u = u + shift[k];
 *   u is rounded to bf16, then rotated and quantised exactly as
 *   rbd_rot_quant_act does.
 *   gamma, shift, scale  bf16 [K], 16-byte aligned, or NULL (the step is then
 *           skipped); one modulation vector for all rows (batch 1).
 *   eps     finite, >= 0 (RBD_ERR_INVALID_ARG otherwise).
 * The float64 sum is exact when the squares of a row span fewer than about
 * 53 - 16 - log2(K) binades; outside that the device's summation order can
 * differ from the exact sum in the last float64 bit, which changes r only when
 * r lies within that distance of a float32 rounding boundary.
 * Other arguments, layouts and errors as rbd_rot_quant_act.                  */
rbd_status rbd_norm_rot_quant_act(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                  const void* shift, const void* scale, float eps, rbd_qcfg cfg,
                                  int8_t* codes, float* scales, void* stream);

/* rbd_rot_quant_act plus the first factor of the low-rank branch on the
 * UNROTATED input: ld = X L1 (Krea-2-SVDQuant-ComfyUI, "LoRA": the branch is a
 * parallel linear, (W + L1 L2)-style, W x + L2 (L1 x)).
 *   l1t     bf16 [r, K] row-major: L1 stored output-major, which is the
 *           nn.Linear weight layout of the down projection.  r in {16, 32, 64}.
 *   ld      bf16 [M, r] row-major (float32 accumulation, rounded once).
 * With group-64 scales (cfg.scale_group == 64) one kernel reads X once and
 * writes codes, scales and ld; with row scales it enqueues two kernels
 * (rotate/quantise, then the down product).  Codes and scales are identical
 * to rbd_rot_quant_act's in both cases.                                     */
rbd_status rbd_lowrank_fused(const void* x, int64_t M, int64_t K, int64_t ldx, rbd_qcfg cfg,
                             int8_t* codes, float* scales, const void* l1t, int32_t r, void* ld,
                             void* stream);

/* The low-rank branch's first factor alone, ld = X L1 on the unrotated input
 * (Krea-2-SVDQuant-ComfyUI, "LoRA"), for paths whose quantiser is not
 * rbd_lowrank_fused (the NVFP4 variant).
 *   x       bf16 [M, ldx], 16-byte aligned, ldx % 8 == 0; K % 128 == 0, K <= 16384.
 *   l1t     bf16 [r, K] row-major (L1 stored output-major), r in {16, 32, 64}.
 *   ld      bf16 [M, r] row-major (float32 accumulation, a fixed-order
 *           reduction, rounded once).                                          */
rbd_status rbd_lowrank_down(const void* x, int64_t M, int64_t K, int64_t ldx, const void* l1t,
                            int32_t r, void* ld, void* stream);

/* Offline weight rotate + quantise + pack to signed INT4 (INT4 tensorwise card,
 * header: the weights are signed four-bit codes, rotated in groups of 256).
 * Each output row of W is rotated and quantised exactly like a token.
 *   w       bf16 [N, K] row-major, 16-byte aligned.    cfg.bits must be 4.
 *   packed  uint8 [N, K/2]: byte k/2 of row n holds code k (even k) in the low
 *           nibble and code k+1 in the high nibble, two's complement.
 *   scales  float32 [N] or [N, K/64].                                          */
rbd_status rbd_pack_weights_int4(const void* w, int64_t N, int64_t K, rbd_qcfg cfg,
                                 uint8_t* packed, float* scales, void* stream);

/* Offline per-row INT8 weights for the protected ff.down layers (OrbitQuant
 * card, "What is quantized": those 28 projections keep eight-bit weights with
 * one scale per output row and run as W8A8).
 *   w8      int8 [N, K].  cfg.bits must be 8.                                  */
rbd_status rbd_pack_weights_int8(const void* w, int64_t N, int64_t K, rbd_qcfg cfg,
                                 int8_t* w8, float* scales, void* stream);

/* Epilogue options of the linear calls ("Fused transformer": the Q|K|V|gate
 * GEMM applies the sigmoid gate on its way out, and the residual adds with
 * their gates are done by the GEMMs' epilogues as well;
 * "What is quantized": biases are not 4-bit tensors).
 *   bias      bf16 [N] or NULL.
 *   ld, l2t   low-rank branch: ld bf16 [M, r] (from rbd_lowrank_fused) and the
 *             second factor stored output-major, l2t bf16 [N, r] (the
 *             nn.Linear layout of the up projection; the branch adds
 *             ld @ l2t^T).  r in {16, 32, 64}; r = 0 disables the branch.
 *   gate_mode 0: none.  1: sigmoid on output columns [gate_col0, gate_col1).
 *             2: out = residual + gate[n] * y (gated residual).
 *   gate      bf16 [N] (gate_mode 2).   residual bf16 [M, ldr] (gate_mode 2).
 *   acc_debug NULL, or int32 receiving the exact integer accumulators:
 *             [M, N] with scale_group 0, [K/64, M, N] with scale_group 64.
 *             Meant for small checks; it adds a full int32 write per output.
 * Order: y = dequant(acc) + bias + ld l2t^T, then the gate, one round to bf16. */
typedef struct rbd_epilogue {
  const void* bias;
  const void* ld;
  const void* l2t;
  int32_t r;
  int32_t gate_mode;
  int64_t gate_col0;
  int64_t gate_col1;
  const void* gate;
  const void* residual;
  int64_t ldr;
  int32_t* acc_debug;
} rbd_epilogue;

/* W4A4 linear: INT4 activation codes (from rbd_rot_quant_act with bits 4)
 * times packed INT4 weights (rbd_pack_weights_int4), then the epilogue.
 *   cfg.code_format RBD_CODES_INT8: int32 accumulation on the tcgen05 INT8
 *           tensor path.  RBD_CODES_E4M3 (group-64 scales only): the weight
 *           nibbles are widened to E4M3 and each 64-wide group partial is
 *           accumulated in float32 on the FP8 tensor path, exactly (every
 *           partial is an integer of magnitude <= 4096).  Both give the same
 *           integer partials; the E4M3 path promotes them with two float32
 *           operations per element and group instead of three.
 *   codes   [M, K] one code per byte in cfg.code_format, sx float32 [M] or
 *           [M, K/64].
 *   w_packed uint8 [N, K/2], sw float32 [N] or [N, K/64].
 *   K % 128 == 0, N % 128 == 0, M >= 1 (ragged M is handled).  A shape whose
 *   per-tile scale table does not fit in shared memory (group scales with a
 *   very large K) returns RBD_ERR_UNSUPPORTED.
 *   epi     may be NULL (no bias, branch or gate).
 *   y       bf16 [M, ldy], ldy >= N, ldy % 8 == 0.
 * Up to 64 tokens run on a weight-streaming kernel (16 output features per
 * block, K split across its warps, warp-level MMAs) instead of the tiled
 * one; results follow the same contract.  That kernel is launched with
 * programmatic stream serialisation: it may start while the preceding
 * kernel on the stream is still running, but before that kernel has
 * completed it only prefetches w_packed into L2 (never stale: L2 is the
 * point of coherence) and reads nothing else.                               */
rbd_status rbd_w4a4_linear(const int8_t* codes, const float* sx, const uint8_t* w_packed,
                           const float* sw, int64_t M, int64_t N, int64_t K, rbd_qcfg cfg,
                           const rbd_epilogue* epi, void* y, int64_t ldy, void* stream);

/* W8A8 linear (per-row INT8 ff.down): INT8 codes times INT8 weights.
 * Same contract as rbd_w4a4_linear with w8 int8 [N, K] and cfg.bits == 8,
 * including the weight-streaming kernel for up to 64 tokens.               */
rbd_status rbd_w8a8_linear(const int8_t* codes, const float* sx, const int8_t* w8,
                           const float* sw, int64_t M, int64_t N, int64_t K, rbd_qcfg cfg,
                           const rbd_epilogue* epi, void* y, int64_t ldy, void* stream);

/* ---- NVFP4 variant ------------------------------------------------------
 * The same rotated layer with FP4 operands on the block-scaled tensor cores
 * ("Krea 2 Turbo Nunchaku Lite INT4 r32", Benchmark: the NVFP4 build).  Each
 * tensor (activations per call, weights once) is quantised in two levels:
 *   gs = amax(rotated tensor) / (6 * 448)                      float32
 *   bs = E4M3_RN_satfinite(amax(block of 16) / (6 * gs))       one per 16 elements
 *   q  = E2M1_RN_satfinite(x / (bs * gs))
 * (every quotient and product an IEEE float32 operation) and the GEMM computes
 * y = gs_x * gs_w * sum_k (q_x bs_x)(q_w bs_w) with float32 accumulation.
 *
 * Block-scale layout ("tile-interleaved", the layout the MMA's scale operand
 * is loaded from): rows in tiles of 128, scale columns (one per 16 elements
 * of K) in steps of 4; byte offset of (row, col) =
 *   ((row/128 * (K/64) + col/4) * 32 + row%32) * 16 + (row%128)/32 * 4 + col%4.
 * A buffer holds rbd_nvfp4_scale_bytes(rows, K) bytes (rows rounded up to 128).
 *
 * Returns the block-scale buffer size in bytes, or -1 for invalid sizes.      */
int64_t rbd_nvfp4_scale_bytes(int64_t rows, int64_t K);

/* Rotates (rot_group 256, or 0 for none) and quantises x bf16 [M, ldx] to NVFP4.
 *   codes        uint8 [M, K/2]: two E2M1 codes per byte, element k (even) in
 *                the low nibble; 8-byte aligned.
 *   block_scales uint8, tile-interleaved E4M3 (see above), 16-byte aligned;
 *                rows past M in the last tile are left untouched.
 *   tensor_scale one float32 (device): gs.
 *   work         4 bytes of device scratch holding the running tensor amax
 *                between the two passes; overwritten, so calls sharing it must
 *                not run concurrently.
 *   K % 256 == 0, K <= 16384.  Two passes over x (amax, then quantisation).    */
rbd_status rbd_nvfp4_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int32_t rot_group,
                           uint8_t* codes, uint8_t* block_scales, float* tensor_scale,
                           uint32_t* work, void* stream);

/* rbd_nvfp4_quant without a caller-provided scratch buffer; the method on the
 * pages has no counterpart to this call: it only changes where the scratch
 * lives.  For callers that cannot allocate device memory for the library
 * (plain C hosts without a device allocator, serving loops that must not
 * allocate between steps).  The quantiser's one scratch word (the running
 * tensor amax) lives in a library-owned 256-byte array per device; a call
 * needing more than that array returns RBD_ERR_UNSUPPORTED.  The first call on
 * a device looks the array up with cudaGetSymbolAddress (do it before any
 * stream capture).  The word is cleared at the start of every call.  All calls
 * on a device share the array, so calls that overlap in time (other streams,
 * other host threads) race and give wrong results.  Allocates nothing.
 * The looked-up address is kept for the life of the process: a device reset
 * (cudaDeviceReset, or another library resetting the primary context) after
 * the first call on that device is not supported, since the kept address then
 * points into freed memory.
 * Arguments and results as rbd_nvfp4_quant.                                   */
rbd_status rbd_nvfp4_quant_noalloc(const void* x, int64_t M, int64_t K, int64_t ldx, int32_t rot_group,
                                   uint8_t* codes, uint8_t* block_scales, float* tensor_scale,
                                   void* stream);

/* NVFP4 linear: y = gs_x gs_w (Q_x . Q_w^T) + epilogue.
 *   xq uint8 [M, K/2], xbs tile-interleaved scales of the M token rows, xgs the
 *   activation tensor scale (device float); wq uint8 [N, K/2], wbs, wgs
 *   likewise for the weights (rbd_nvfp4_quant of W [N, K]).
 *   K % 256 == 0, N % 128 == 0; all code and scale buffers 16-byte aligned.
 *   epi: bias, low-rank branch and gate modes as for rbd_w4a4_linear
 *   (Krea-2-SVDQuant-ComfyUI, "LoRA": the same parallel branch beside the
 *   FP4 product): y = gs_x gs_w acc + bias + (ld l2)[m, n], the branch
 *   computed by a bf16 MMA with float32 accumulation (ld from
 *   rbd_lowrank_down, r in {16, 32, 64}); acc_debug is not supported here
 *   (RBD_ERR_UNSUPPORTED).
 *   y bf16 [M, ldy], ldy >= N, ldy % 8 == 0.                                  */
rbd_status rbd_nvfp4_linear(const uint8_t* xq, const uint8_t* xbs, const float* xgs,
                            const uint8_t* wq, const uint8_t* wbs, const float* wgs,
                            int64_t M, int64_t N, int64_t K, const rbd_epilogue* epi,
                            void* y, int64_t ldy, void* stream);

/* INT4 KV-cache codec ("lab", Study 6, "The cache becomes the model":
 * four-bit codes, two to a byte, with a scale for each (token, head, rotary
 * band); the rotary bands of a head are channels 0-43, 44-85 and 86-127;
 * finer scale groups stay inside one band; a read unpacks and rescales in a
 * single pass).
 *   groups_per_band n in {1, 2, 4}: 3, 6 or 12 groups per head; a band of b
 *           channels is cut into n contiguous runs whose sizes differ by at
 *           most one, longer runs first.
 *   Per group, float32 IEEE: amax, s = amax / 7, inv = 7 / amax,
 *   q = clamp(rint_even(x * inv), -8, 7); an all-zero group gets s = 0.
 *   The cache is a ring of `capacity` token slots: input token t (0 <= t < T)
 *   is slot (slot0 + t) mod capacity; T <= capacity, 0 <= slot0 < capacity.
 *   codes   uint8 [capacity, H, 64], 16-byte aligned: byte i of a head holds
 *           channel 2i in the low nibble, 2i + 1 in the high nibble.
 *   scales  float32 [capacity, H, 3n].
 *   x / y   bf16 [T, ldt] row-major, one row per token holding H heads of 128
 *           channels (head h at h * 128); ldt >= 128 H, ldt % 8 == 0,
 *           16-byte aligned.
 * Encode writes the T slots; decode reads them back as RN_bf16(q * s).       */
rbd_status rbd_kv4_encode(const void* x, int64_t T, int64_t H, int64_t ldt, int32_t groups_per_band,
                          uint8_t* codes, float* scales, int64_t capacity, int64_t slot0, void* stream);
rbd_status rbd_kv4_decode(const uint8_t* codes, const float* scales, int64_t capacity, int64_t slot0,
                          int64_t T, int64_t H, int32_t groups_per_band, void* y, int64_t ldt,
                          void* stream);

/* Q/K RMSNorm + RoPE ("Krea 2 Turbo OrbitQuant W4A4", "Fused transformer":
 * a Q/K RMSNorm + RoPE kernel follows the Q|K|V|gate GEMM in every block;
 * "lab", Study 6: rotary bands of 44 (time), 42 (height), 42 (width) channels).
 * Per token t and head h of 128 channels:
 *   r = 1 / sqrt(sum(x^2) / 128 + eps) in float64, rounded to float32
 *   (r = 0 when that radicand is 0); then in float32 u = x r gamma,
 *   (y[2i], y[2i+1]) = (u[2i] c - u[2i+1] s, u[2i] s + u[2i+1] c),
 *   c = cos_t[t][i], s = sin_t[t][i]; y rounded once to bf16.
 *   x, y    bf16 [T, ldx] / [T, ldy] row-major, H heads of 128 channels per
 *           row (head h at h * 128); ld >= 128 H, ld % 8 == 0, 16-byte
 *           aligned; y == x (in place) is allowed.
 *   gamma   bf16 [128] shared by the heads, 16-byte aligned, or NULL (ones).
 *   cos_t, sin_t  float32 [T, 64], 16-byte aligned (rbd_rope_tables).
 *   eps     finite, >= 0.
 * Returns RBD_ERR_INVALID_ARG / RBD_ERR_ALIGNMENT for bad arguments, and
 * RBD_ERR_UNSUPPORTED when T * H exceeds 2^30.                               */
rbd_status rbd_qk_norm_rope(const void* x, int64_t T, int64_t H, int64_t ldx, const void* gamma,
                            const float* cos_t, const float* sin_t, float eps, void* y, int64_t ldy,
                            void* stream);

/* Rotary angle tables for rbd_qk_norm_rope.  pos int32 [T, 3] (time, height,
 * width) on the device, 4-byte aligned.  Pair i of a head lies in the band
 * holding channels 2i and 2i + 1 (pairs 0-21 time, 22-42 height, 43-63
 * width); with j its index inside a band of w channels it turns by
 * pos[t][band] * base^(-2j / w), formed in float64; cos_t / sin_t float32
 * [T, 64] (16-byte aligned) receive the rounded cosine and sine.  base > 0,
 * finite (10000 is the usual value).                                         */
rbd_status rbd_rope_tables(const int32_t* pos, int64_t T, double base, float* cos_t, float* sin_t,
                           void* stream);

/* ---- INT8 attention (SageAttention v1 scheme) ------------------------------
 * "Krea 2 Turbo OrbitQuant W4A4", "Fused transformer": attention takes Q.K^T in
 * INT8 and P.V in FP16.  Two calls: rbd_attn_quant prepares the operands,
 * rbd_attn_int8 runs the attention.  Heads are 128 channels wide.
 *
 * Bytes of device scratch rbd_attn_quant needs for Tk keys and H heads (the
 * float64 partial column sums of K and the key mean); -1 for bad sizes.     */
int64_t rbd_attn_workspace_bytes(int64_t Tk, int64_t H);

/* Operand preparation.
 *   q bf16 [Tq, ldq], k bf16 [Tk, ldk], v bf16 [Tk, ldv]: head h at columns
 *     h*128 .. h*128+127 (the layout of the Q|K|V|gate GEMM output after
 *     rbd_qk_norm_rope); ld* >= H*128, ld* % 8 == 0, 16-byte aligned.
 *   Keys are smoothed: per head and channel the mean over the Tk tokens is
 *   taken in float64 (exact sum while a column spans <= 31 binades) and
 *   subtracted in float64, the result rounded once to float32.  Q and the
 *   smoothed K are quantised per (token, head) over the 128 channels:
 *   amax, s = amax/127, inv = 127/amax (IEEE float32 divisions),
 *   code = clamp(rint_even(x * inv), -128, 127); an all-zero head gets s = 0.
 *   qc int8 [H, Tq, 128], sq float32 [H, Tq];
 *   kc int8 [H, Tk, 128], sk float32 [H, tkp] (entries Tk.. unused);
 *   vt fp16 [H, 128, tkp]: V transposed per head, each value rounded to fp16
 *     (nearest even), tokens Tk .. tkp-1 written as zeros;
 *   tkp >= Tk, tkp % 8 == 0 (the row pitch of sk and vt);
 *   work: rbd_attn_workspace_bytes(Tk, H) bytes of device scratch, 16-byte
 *     aligned, overwritten (calls sharing it must not overlap).
 *   Tk == 0 with Tq > 0 is invalid (RBD_ERR_INVALID_ARG); Tq == Tk == 0 is a
 *   no-op.  All outputs 16-byte aligned (sq 4-byte).                         */
rbd_status rbd_attn_quant(const void* q, int64_t ldq, const void* k, int64_t ldk, const void* v, int64_t ldv,
                          int64_t Tq, int64_t Tk, int64_t H, int8_t* qc, float* sq, int8_t* kc, float* sk,
                          void* vt, int64_t tkp, void* work, void* stream);

/* Attention on the prepared operands: for every head and query,
 *   S[key] = (qc . kc[key]) * sq * sk[key] / sqrt(128)  (exact int32 dot product),
 *   P = softmax over the Tk keys, o = P . V with P rounded to fp16 after the
 *   running row maximum is subtracted and V in fp16, float32 accumulation.
 * o bf16 [Tq, ldo], head h at columns h*128; ldo >= H*128, ldo % 8 == 0.
 * Arguments otherwise as rbd_attn_quant produced them (same Tq, Tk, H, tkp).  */
rbd_status rbd_attn_int8(const int8_t* qc, const float* sq, const int8_t* kc, const float* sk, const void* vt,
                         int64_t Tq, int64_t Tk, int64_t H, int64_t tkp, void* o, int64_t ldo, void* stream);

/* ---- Offline SVDQuant fit of the low-rank branch --------------------------
 * "Krea-2-SVDQuant-ComfyUI", "Low-rank refinement, and what the objective
 * actually is" and "Activation-aware branch".  Minimises
 * ||(W - (deq(Q) + L)) diag(d)||_F over a rank-r branch L and codes Q in the
 * layer's own rotated format (cfg: bits 4 or 8, rot_group, scale_group;
 * code_format RBD_CODES_INT8): iterate 1 splits W by a randomized SVD of
 * W diag(d) (test matrix omega_1, one power iteration, QR after every
 * product); each later iterate re-fits the branch to (W - deq(Q)) diag(d) with
 * its own test matrix and quantises bf16(W - L) again; the iterate with the
 * smallest error is kept.  d = act_rms / mean(act_rms), floored at 0.05, or
 * all ones when act_rms is NULL.
 *
 * Bytes of device scratch for an N x K weight, rank r and oversampling p
 * (-1 for an unsupported configuration).                                    */
int64_t rbd_svdquant_workspace_bytes(int64_t N, int64_t K, int32_t rank, int32_t oversample, rbd_qcfg cfg);

/* The fit.  SYNCHRONOUS: it waits for the device between steps (the thin QR
 * factorisations and the (r+p) x K SVD run on the host in float64; the
 * products with W, the requantisation, dequantisation and error run on the
 * device in float64).
 *   w        bf16 [N, K] device, 16-byte aligned; K a multiple of 256 with
 *            rotation (of 64 without), K <= 16384.
 *   omegas   HOST float64 [iters][K][rank + oversample]: the Gaussian test
 *            matrices (inputs, one per iterate).
 *   act_rms  HOST float64 [K] or NULL.
 *   q, scales  device: the kept iterate's codes (packed INT4 [N, K/2] or INT8
 *            [N, K], as rbd_pack_weights_*) and scales.
 *   l1       HOST float64 [K][rank] = (V / d) sqrt(S); l2 HOST float64
 *            [rank][N] = sqrt(S) U^T, so that the branch adds (x l1) l2.
 *   errs     HOST float64 [iters]: the objective after every iterate;
 *   best     HOST int32 (may be NULL): index of the kept iterate.
 *   work     rbd_svdquant_workspace_bytes(...) bytes of device scratch,
 *            16-byte aligned.
 * rank + oversample <= min(N, K, 256).                                       */
rbd_status rbd_svdquant_fit(const void* w, int64_t N, int64_t K, rbd_qcfg cfg, int32_t rank, int32_t oversample,
                            int32_t iters, const double* omegas, const double* act_rms, void* q, float* scales,
                            double* l1, double* l2, double* errs, int32_t* best, void* work, void* stream);

/* Synchronises `stream`, then reports the first device-side error recorded
 * since the last rbd_check (RBD_ERR_DEVICE_TIMEOUT) or a CUDA error, and
 * clears the device status word.                                              */
rbd_status rbd_check(void* stream);

/* Launches a single-thread kernel that waits on an mbarrier nobody signals,
 * bounded by timeout_ns, then records RBD_ERR_DEVICE_TIMEOUT.  It exercises
 * the device-side timeout path without hanging or faulting the GPU; follow it
 * with rbd_check().                                                           */
rbd_status rbd_debug_timeout_probe(int64_t timeout_ns, void* stream);

/* Human-readable name of a status code (static storage).                     */
const char* rbd_status_string(rbd_status s);

/* Library version string (static storage).                                  */
const char* rbd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RBD_H_ */
