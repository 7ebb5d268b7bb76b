/*
 * qlora_nf4.h -- C ABI of the QLoRA NF4 frozen-base linear layer for NVIDIA B200 (sm_100a).
 *
 * The method (QLoRA, Dettmers et al., arXiv:2305.14314), as the source pages state it:
 *   - a frozen base weight W (h x o) is stored as 4-bit NormalFloat codes in blocks of 64
 *     weights, each block with an absmax scale ("QLoRA in LLMs", tensortonic.com, section 3
 *     "How LoRA and Quantization Fit Together" and section 5 "NF4"; "QLoRA: Efficient
 *     Finetuning of Quantized LLMs", mchromiak.github.io, "1. NormalFloat");
 *   - the block scales are themselves quantized to 8 bits, with one higher-precision scale
 *     per 256 of them ("2. Double quantization: Compress the scales too"; "A worked memory
 *     budget for 65 billion weights"; "QLoRA in LLMs" section 6);
 *   - for compute, blocks are dequantized on the fly to bf16 and contracted with the
 *     activations ("QLoRA: the paper that put large-model fine-tuning on a desk",
 *     goodomens.studio, "The core move"), and a trainable low-rank adapter is added:
 *     Y = X.W + s.X.L1.L2 ("The algebra: How two small matrices change a layer"; s = alpha/r,
 *     "QLoRA in LLMs" section 3);
 *   - gradients reach the adapters through the frozen base, which receives none ("One
 *     training step, from input to update"; "QLoRA in LLMs" section 4).
 *
 * Storage layout used throughout (the readings of the pages are stated in the design notes):
 *   Wt      the weight stored transposed, o x h row-major ("out x in"); W' = Wt^T.
 *   block   64 consecutive elements of Wt's flat row-major order (so h % 64 == 0).
 *   codes   n/2 bytes; element 2j of the flat order is the high nibble of byte j.
 *   q8      n/64 bytes: the 8-bit first-level scale of each block.
 *   s2      ceil(n/16384) floats: one fp32 second-level scale per 256 blocks.
 *   w'      bf16_rn( level[code] * (float(q8[b]) * s2[b/256]) ), two fp32 multiplies.
 *   bf16    passed as uint16_t bit patterns.
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers owned by the caller, each aligned to 16 bytes, unless
 *     a parameter says otherwise. The library never allocates, frees or synchronises device
 *     memory except where stated (qlora_get_last_status synchronises its stream).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *   - Outputs are overwritten, never accumulated into. Inputs are not modified.
 *   - Return value: 0 on success; a negative QLORA_ERR_* code when the host-side checks
 *     reject the arguments or a launch fails, in which case nothing was launched (for
 *     argument errors) or the launch error is returned. Faults the kernels detect while
 *     running (non-finite weights, an internal wait that timed out) are OR-ed into a device
 *     status word, read and cleared by qlora_get_last_status.
 *   - The device must be an sm_100 GPU (B200); any other device gives
 *     QLORA_ERR_UNSUPPORTED_DEVICE.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle, layout-compatible with cudaStream_t. */
typedef struct CUstream_st *qlora_stream_t;

/* Host-side status codes (negative) returned by every call. */
enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = -1,       /* null pointer, bad rank r, t < 1, bad scalar           */
  QLORA_ERR_BAD_SHAPE = -2,         /* h % 64 != 0, o % 64 != 0, size overflow               */
  QLORA_ERR_MISALIGNED = -3,        /* a pointer is not 16-byte aligned                      */
  QLORA_ERR_WORKSPACE = -4,         /* workspace pointer NULL or smaller than required       */
  QLORA_ERR_CUDA = -5,              /* a CUDA runtime call or kernel launch failed           */
  QLORA_ERR_UNSUPPORTED_DEVICE = -6, /* the current device is not sm_100                     */
  QLORA_ERR_SCRATCH_LIMIT = -7      /* qlora_linear_fwd_noalloc: the shape needs more scratch
                                       than QLORA_STATIC_SCRATCH_BYTES                        */
};

/* Device-side fault bits (positive), OR-ed into the status word by the kernels. */
enum {
  QLORA_DEV_NONFINITE = 1,          /* nf4_quantize met a NaN or infinite weight             */
  QLORA_DEV_TIMEOUT = 2,            /* a kernel's bounded internal wait expired; outputs of
                                       that call are unspecified                              */
  QLORA_DEV_LAUNCH = 4              /* a kernel found its launch unusable (e.g. too little
                                       shared memory) and did no work                         */
};

/* A packed NF4 weight: caller-owned device buffers plus the logical shape.
 * Block size 64 and scale-group size 256 are fixed by the method. */
typedef struct nf4_weight {
  uint8_t *codes;        /* n/2 bytes, n = out_features * in_features                        */
  uint8_t *absmax_q8;    /* n/64 bytes                                                        */
  float *absmax_s2;      /* ceil(n/16384) floats                                             */
  int64_t out_features;  /* o: rows of Wt                                                     */
  int64_t in_features;   /* h: columns of Wt, h % 64 == 0                                     */
} nf4_weight;

/* The 16 NF4 levels (ascending fp32, exact zero at index 7, ends -1 and +1), as this library
 * derives them from standard-normal quantiles ("QLoRA in LLMs" section 5; "Idea one: NF4" on
 * goodomens.studio). Host call, no device needed. levels: host array of 16 floats;
 * midpoints: host array of 15 floats (decision thresholds) or NULL. Returns 0 or
 * QLORA_ERR_INVALID_ARG when levels is NULL. */
QLORA_API int qlora_nf4_codebook(float *levels, float *midpoints);

/* nf4_quantize -- blockwise NF4 quantization with double-quantized scales.
 * Follows "QLoRA in LLMs" section 2 (absmax scale, normalise, round to the nearest
 * representable value), section 5 (NF4 levels) and section 6 (double quantization), and
 * "2. Double quantization" on mchromiak.github.io.
 *   Wt  device, fp32, o x h row-major (o = q->out_features, h = q->in_features), read only.
 *   q   host pointer to a descriptor whose device buffers receive codes, q8 and s2.
 * Per block: c1 = max|w|; x = w / c1 (fp32, round to nearest); code = number of midpoints
 * strictly below x (a block with c1 == 0 takes code 7). Per group of 256 blocks (the last may
 * be shorter): s2 = max(c1) / 255; q8 = clamp(round_half_even(c1 / s2), 0, 255) (0 when s2
 * is 0). The codes use the exact c1, not the 8-bit scale. A non-finite weight sets
 * QLORA_DEV_NONFINITE; the outputs for its group are then unspecified.
 * Errors: INVALID_ARG (NULL), BAD_SHAPE (h % 64 != 0, o < 1), MISALIGNED. */
QLORA_API int nf4_quantize(const float *Wt, const nf4_weight *q, qlora_stream_t stream);

/* nf4_dequantize -- reconstruct the bf16 weight Wt' (o x h row-major) from a packed weight.
 * "QLoRA in LLMs" section 3 (dequantized into BF16 for a calculation); "1. NormalFloat" on
 * mchromiak.github.io. Wt_out: device, bf16 bits, o*h elements. Bit-exact definition:
 * w' = bf16_rn(level[code] * (float(q8) * s2)). Errors: INVALID_ARG, BAD_SHAPE, MISALIGNED. */
QLORA_API int nf4_dequantize(const nf4_weight *q, uint16_t *Wt_out, qlora_stream_t stream);

/* qlora_linear_fwd -- Y = X.W' + s.X.L1.L2 for one adapted linear layer.
 * "The algebra" (mchromiak.github.io): X is t x h, W is h x o, L1 is h x r, L2 is r x o,
 * scalar s; "QLoRA in LLMs" section 3-4; the base block is dequantized on the fly and
 * discarded ("The core move" on goodomens.studio).
 *   X        device bf16, t x h row-major.          t >= 1.
 *   W        host pointer to the packed weight (o x h stored); h % 64 == 0, o % 64 == 0.
 *   L1       device bf16, h x r row-major.          16 <= r <= 256, r % 16 == 0.
 *   L2       device bf16, r x o row-major.
 *   s        the adapter scale (alpha / r); any finite value.
 *   Y        device bf16, t x o row-major (output).
 *   sT_out   device bf16, t x r (output, bf16(s . X.L1), kept for the backward) or NULL.
 *   workspace, ws_bytes: device scratch of at least qlora_fwd_workspace_bytes(t, h, o, r)
 *            bytes, caller-owned; contents on entry are ignored.
 * Compute: bf16 operands, fp32 accumulation; the LoRA term uses the bf16-rounded
 * sT = bf16(s . X.L1), folded into the same accumulator as X.W'. */
QLORA_API int qlora_linear_fwd(const uint16_t *X, int64_t t, const nf4_weight *W,
                     const uint16_t *L1, const uint16_t *L2, int64_t r, float s,
                     uint16_t *Y, uint16_t *sT_out,
                     void *workspace, size_t ws_bytes, qlora_stream_t stream);

/* qlora_linear_bwd -- gradients of the adapted linear; the frozen W gets none.
 * "One training step, from input to update" (mchromiak.github.io); "QLoRA in LLMs" section 4.
 *   dY       device bf16, t x o (upstream gradient).     X: device bf16, t x h.
 *   W, L1, L2, r, s: as in qlora_linear_fwd.
 *   sT_saved device bf16, t x r = bf16(s . X.L1) from the forward, or NULL to recompute it.
 *   dX       device bf16, t x h (output) = dY.W'^T + sU.L1^T with sU = bf16(s . dY.L2^T).
 *   dL1      device fp32, h x r (output) = X^T . sU.
 *   dL2      device fp32, r x o (output) = sT^T . dY.
 *   workspace, ws_bytes: at least qlora_bwd_workspace_bytes(t, h, o, r) bytes. */
QLORA_API int qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, int64_t t, const nf4_weight *W,
                     const uint16_t *L1, const uint16_t *L2, int64_t r, float s,
                     const uint16_t *sT_saved, uint16_t *dX, float *dL1, float *dL2,
                     void *workspace, size_t ws_bytes, qlora_stream_t stream);

/* qlora_linear_fwd_noalloc -- the same forward as qlora_linear_fwd, for callers that cannot
 * allocate device memory. There is no counterpart in the QLoRA method: this is a deployment
 * convenience. Some callers are handed only their input and output buffers (a plugin slot in
 * a host framework, a serving loop whose memory budget is fixed at start-up) and have no way
 * to obtain a workspace, and cudaMalloc/cudaFree may synchronise the whole device, which a
 * latency-bound caller cannot afford.
 * Instead of a caller workspace this call uses a scratch array of QLORA_STATIC_SCRATCH_BYTES
 * that lives in the library's device image: every GPU that loads the library holds it until
 * the process exits. The call allocates nothing and calls no allocating routine.
 *   - Arguments and results: exactly those of qlora_linear_fwd without workspace/ws_bytes.
 *   - Limit: shapes with qlora_fwd_workspace_bytes(t, h, o, r) > QLORA_STATIC_SCRATCH_BYTES
 *     are rejected with QLORA_ERR_SCRATCH_LIMIT before anything is launched.
 *   - The first call on a device looks up the array's device address (with that device
 *     current) and keeps it for later calls; make that first call before any stream capture
 *     begins. A lookup that fails returns QLORA_ERR_CUDA and is tried again by the next call.
 *   - All calls share the one array, and it keeps whatever the previous call left there (the
 *     call clears the parts that must start at zero itself). Two calls whose kernels overlap on
 *     the GPU, for example on two streams, race on the array: serialise them. */
#define QLORA_STATIC_SCRATCH_BYTES (8u << 20)
QLORA_API int qlora_linear_fwd_noalloc(const uint16_t *X, int64_t t, const nf4_weight *W,
                                       const uint16_t *L1, const uint16_t *L2, int64_t r, float s,
                                       uint16_t *Y, uint16_t *sT_out, qlora_stream_t stream);

/* Workspace sizes in bytes for the two linear calls (host functions, no device needed).
 * Return 0 for shapes the calls would reject. */
QLORA_API size_t qlora_fwd_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r);
QLORA_API size_t qlora_bwd_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r);

/* LoRA dropout on the adapter input ("QLoRA in LLMs" section 12, "Minimal QLoRA Setup with
 * Hugging Face": the example configuration uses a LoRA dropout of 0.05). The pages do not say
 * where it acts; these calls take the adapter branch's input, with inverted scaling:
 *   Y = X.W' + s.((X (.) M / (1 - p)).L1).L2,
 * and the matching gradients dX = dY.W'^T + M (.) (s / (1 - p)).(dY.L2^T).L1^T,
 * dL1 = s.(X (.) M / (1 - p))^T.(dY.L2^T), dL2 = s.((X (.) M / (1 - p)).L1)^T.dY.
 * M (t x h) is drawn, not stored: element e = i*h + j takes word e mod 4 of Philox4x32-10
 * (Salmon et al., "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11) at counter
 * (lo32(e / 4), hi32(e / 4), 0, 0) under key (lo32(seed), hi32(seed)), and is kept when that
 * word is >= floor(p * 2^32). The forward and the backward of one step must get the same
 * (p, seed); a new seed per step and per layer gives fresh masks.
 *   p     dropout probability, 0 <= p < 1 (else INVALID_ARG); p = 0 (or any p below 2^-32) is
 *         exactly the plain layer.
 *   seed  any 64-bit value.
 *   mask_out    (forward) device, t*h/8 bytes, 16-byte aligned, or NULL: receives M as bits,
 *               bit e mod 8 of byte e / 8 = keep bit of element e.
 *   mask_saved  (backward) the forward's mask_out for the same (p, seed), or NULL to draw M
 *               again; with it the backward makes no generator calls.
 * Every other argument is that of qlora_linear_fwd / qlora_linear_bwd, except the workspace,
 * which is larger (it holds X (.) M, and in the backward also the mask as bits and then the
 * masked adapter term of dX):
 * qlora_fwd_dropout_workspace_bytes and qlora_bwd_dropout_workspace_bytes. The rounded
 * s / (1 - p) (fp32) is the scale of sT and sU; sT_out / sT_saved carry
 * bf16(s / (1 - p) . (X (.) M).L1). In the backward the masked term
 * E = bf16(M (.) sU.L1^T) is added to the fp32 accumulator of dY.W'^T before dX's one
 * rounding to bf16. */
QLORA_API int qlora_linear_fwd_dropout(const uint16_t *X, int64_t t, const nf4_weight *W,
                                       const uint16_t *L1, const uint16_t *L2, int64_t r, float s,
                                       float p, uint64_t seed, uint16_t *Y, uint16_t *sT_out,
                                       uint8_t *mask_out, void *workspace, size_t ws_bytes,
                                       qlora_stream_t stream);
QLORA_API int qlora_linear_bwd_dropout(const uint16_t *dY, const uint16_t *X, int64_t t,
                                       const nf4_weight *W, const uint16_t *L1, const uint16_t *L2,
                                       int64_t r, float s, float p, uint64_t seed,
                                       const uint16_t *sT_saved, const uint8_t *mask_saved,
                                       uint16_t *dX, float *dL1, float *dL2, void *workspace,
                                       size_t ws_bytes, qlora_stream_t stream);
QLORA_API size_t qlora_fwd_dropout_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r);
QLORA_API size_t qlora_bwd_dropout_workspace_bytes(int64_t t, int64_t h, int64_t o, int64_t r);

/* qlora_dropout_apply -- Xd = X (.) M for the mask above (dropped elements become +0; no
 * 1 / (1 - p) scaling), so that the mask can be inspected on its own.
 *   X, Xd  device bf16, t x h row-major; Xd == X works in place, any other overlap is
 *          rejected.  h % 64 == 0.
 * Errors: INVALID_ARG (NULL, p outside [0, 1), partial overlap), BAD_SHAPE, MISALIGNED. */
QLORA_API int qlora_dropout_apply(const uint16_t *X, int64_t t, int64_t h, float p, uint64_t seed,
                                  uint16_t *Xd, qlora_stream_t stream);

/* Synchronise `stream`, then return and clear the device status word of the current device:
 * 0, or an OR of QLORA_DEV_* bits, or QLORA_ERR_CUDA if the synchronisation failed. */
QLORA_API int qlora_get_last_status(qlora_stream_t stream);

/* Kernel timing (measurement support, not part of the method). While a profile is open on
 * the current device, the library records a pair of CUDA events around each of its kernel
 * launches, on the launching stream. qlora_profile_begin(capacity) opens a profile for up to
 * `capacity` launches (events are created once and reused; no device memory is allocated).
 * qlora_profile_end synchronises the last recorded event, closes the profile and writes, for
 * each kernel kind k < nkinds, the summed device time in milliseconds (ms[k]) and the number
 * of launches (launches[k]); it returns the number of launches recorded, or QLORA_ERR_CUDA,
 * or QLORA_ERR_INVALID_ARG if the profile overflowed its capacity. Kinds are numbered
 * 0 .. QLORA_KERNEL_KINDS-1 and named by qlora_kernel_name. Not thread-safe across
 * concurrent calls into the library while open. */
#define QLORA_KERNEL_KINDS 8
QLORA_API int qlora_profile_begin(int capacity);
QLORA_API int qlora_profile_end(double *ms, int64_t *launches, int nkinds);
QLORA_API const char *qlora_kernel_name(int kind);

/* Other 4-bit codebooks, for the format comparison the pages draw (NF4 against FP4 and INT4:
 * "QLoRA in LLMs" section 5; "Idea one: NF4", goodomens.studio). Same 64-weight blocks,
 * packing and double-quantized scales as nf4_quantize / nf4_dequantize; only the 16 levels
 * (and the code of the zero level, taken by all-zero blocks) differ. codebook_id:
 *   QLORA_CODEBOOK_NF4 (0)   the NF4 levels (nf4_quantize / nf4_dequantize use these)
 *   QLORA_CODEBOOK_FP4 (1)   FP4 E2M1: {0, .5, 1, 1.5, 2, 3, 4, 6} with both signs, over 6,
 *                            -0 and +0 both kept (codes 7 and 8); zero code 7
 *   QLORA_CODEBOOK_INT4 (2)  absmax INT4: k / 7 for k = -8 .. 7; zero code 8
 * A weight packed with one codebook must be dequantized with the same one (the packed
 * format does not record it); only NF4-packed weights may be passed to the linear calls.
 * qlora_codebook writes that codebook's 16 levels (and 15 midpoints if non-NULL).
 * Errors: QLORA_ERR_INVALID_ARG for an unknown id, else as nf4_quantize / nf4_dequantize. */
#define QLORA_CODEBOOK_NF4 0
#define QLORA_CODEBOOK_FP4 1
#define QLORA_CODEBOOK_INT4 2
QLORA_API int qlora_codebook(int codebook_id, float *levels, float *midpoints);
QLORA_API int qlora_quantize_codebook(const float *Wt, const nf4_weight *q, int codebook_id,
                                      qlora_stream_t stream);
QLORA_API int qlora_dequantize_codebook(const nf4_weight *q, int codebook_id, uint16_t *Wt_out,
                                        qlora_stream_t stream);

/* Other 8-bit formats for the double-quantized block scales ("QLoRA in LLMs" section 1, "FP32,
 * FP16, BF16, and FP8": E4M3 has 4 exponent and 3 fraction bits; section 2, "Choose a scale,
 * then round": symmetric absmax to the integers -127 .. 127). The second level is one fp32
 * scale s2 per 256 blocks in every format; c1 is a block's absmax, c2 its group's largest c1:
 *   QLORA_SCALES_U8 (0)    s2 = c2 / 255, q8 = clamp(rint(c1 / s2), 0, 255)  (nf4_quantize's)
 *   QLORA_SCALES_S8 (1)    s2 = c2 / 127, q8 = clamp(rint(c1 / s2), -127, 127), stored as the
 *                          two's-complement byte (the textbook signed scheme; codes < 0 unused)
 *   QLORA_SCALES_E4M3 (2)  s2 = c2 / 448, q8 = the FP8 E4M3 code (bias 7, no infinities, 0x7F
 *                          NaN) of c1 / s2 rounded to nearest even, saturating at 448
 * Dequantization: w' = bf16_rn(level[code] * (value(q8) * s2)). The 4-bit codes do not depend
 * on the scale format. A weight must be dequantized with the codebook and scale format it was
 * packed with; only NF4 with QLORA_SCALES_U8 may be passed to the linear calls. The
 * _codebook calls are these with QLORA_SCALES_U8.
 * Errors: QLORA_ERR_INVALID_ARG for an unknown id or format, else as nf4_quantize /
 * nf4_dequantize. */
#define QLORA_SCALES_U8 0
#define QLORA_SCALES_S8 1
#define QLORA_SCALES_E4M3 2
QLORA_API int qlora_quantize_format(const float *Wt, const nf4_weight *q, int codebook_id,
                                    int scale_format, qlora_stream_t stream);
QLORA_API int qlora_dequantize_format(const nf4_weight *q, int codebook_id, int scale_format,
                                      uint16_t *Wt_out, qlora_stream_t stream);

/* Adapter merge ("QLoRA in LLMs" section 11, "Saving, Loading, and Merging QLoRA Adapters":
 * dequantize the base into a wider precision, add the LoRA update, optionally quantize the
 * result again): Wt_merged = W'^T + s . (L1 . L2)^T, i.e. W_m = W' + s.L1.L2 in the stored
 * orientation, in fp32:
 *   Wt_merged[j][k] = W'[k][j] + s * sum_c L1[k][c] * L2[c][j]    (o x h, row-major)
 * where W'[k][j] is the nf4_dequantize value (exact bf16) of the packed weight. The rank-r
 * sum is formed from the exact bf16 products in fp32; each element is within
 * (r + 2) * 2^-23 * (|W'| + |s| * sum_c |L1 L2|) of the exact merge. Re-quantize the result
 * with nf4_quantize to obtain a merged packed weight.
 *   W: packed weight (out_features o, in_features h: h % 64 == 0, o % 64 == 0).
 *   L1 (h x r), L2 (r x o): bf16 row-major, 16 <= r <= 256, r % 16 == 0.
 *   Wt_merged: caller-owned device buffer of o * h fp32, 16-byte aligned; overwritten.
 * Errors: QLORA_ERR_INVALID_ARG / _BAD_SHAPE / _MISALIGNED / _CUDA, nothing launched. */
QLORA_API int qlora_merge_adapters(const nf4_weight *W, const uint16_t *L1, const uint16_t *L2,
                                   int64_t r, float s, float *Wt_merged, qlora_stream_t stream);

/* Adapter update with a paged optimizer ("QLoRA in LLMs" sections 4 and 7; "Idea three: paged
 * optimizers", goodomens.studio): one fused AdamW step over n fp32 parameters (an adapter,
 * e.g. L1 with n = h * r, using its dL1 as grad), with decoupled weight decay and bias-corrected
 * moments at 1-based step t:
 *   p <- p (1 - lr wd);  m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2;
 *   p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * and, if param_bf16 is non-NULL, its bf16 copy (round to nearest even) for the next forward.
 * The pages name the optimizer state but not the rule; AdamW is the reading. Any buffer may be
 * unified (cudaMallocManaged) memory, as the pages' paged optimizer keeps its state: the kernel
 * then reads it wherever the driver has placed it (pages on the host migrate on first touch),
 * and with flags = QLORA_ADAMW_PREFETCH each unified buffer is first prefetched to the current
 * device on `stream` (bulk migration; on pages already resident the prefetch still costs
 * driver time). The driver may move the state back to host memory under memory pressure.
 * param, grad, m, v: 16-byte aligned, caller-owned, n % 4 == 0; param, m, v, param_bf16 are
 * updated in place. Hyper-parameters are used as the fp32 values given.
 * Errors: QLORA_ERR_INVALID_ARG (null, n, step < 1, eps <= 0, betas outside [0, 1), unknown
 * flags), QLORA_ERR_MISALIGNED, QLORA_ERR_CUDA; nothing is launched on an error. */
#define QLORA_ADAMW_PREFETCH 1u
QLORA_API int qlora_adamw_step(float *param, uint16_t *param_bf16, const float *grad, float *m,
                               float *v, int64_t n, float lr, float beta1, float beta2,
                               float eps, float weight_decay, int64_t step, unsigned flags,
                               qlora_stream_t stream);

/* The same AdamW step over several tensors (e.g. all adapters of a layer or a model) in one
 * launch: tensor k has counts[k] parameters (counts[k] % 4 == 0) at params[k], grads[k], m[k],
 * v[k] and, if params_bf16 is non-NULL and params_bf16[k] is non-NULL, its bf16 copy at
 * params_bf16[k]. The pointer arrays and counts are HOST arrays of ntensors entries
 * (1 <= ntensors <= 64), read before the call returns; the buffers they point to follow the
 * rules of qlora_adamw_step. Every parameter is updated exactly as qlora_adamw_step updates it
 * (bit-identical results). Errors as qlora_adamw_step; nothing is launched on an error. */
QLORA_API int qlora_adamw_step_multi(int ntensors, float *const *params, uint16_t *const *params_bf16,
                                     const float *const *grads, float *const *m, float *const *v,
                                     const int64_t *counts, float lr, float beta1, float beta2,
                                     float eps, float weight_decay, int64_t step, unsigned flags,
                                     qlora_stream_t stream);

/* Launch shape of the decode GEMV (t <= 16), a scheduling knob with no counterpart in the
 * method. By default the GEMV runs one CTA of 16 warps per SM and splits its units (32 rows x
 * 128 inputs) evenly over all their warps. qlora_set_gemv_max_ctas(n) caps that CTA count at
 * n for later calls on every device (n <= 0 restores the default), e.g. to leave SMs to work
 * on another stream; results do not depend on it beyond fp32 summation order. Returns the
 * previous cap (0 = none). Process-wide; not ordered with calls in flight on other threads. */
QLORA_API int qlora_set_gemv_max_ctas(int n);

/* Self-test of failure detection, with no counterpart in the method and no GPU fault: launches
 * one kernel whose single thread waits on a barrier that nothing will complete, through the
 * same bounded wait every pipelined kernel uses, with the limit shortened to limit_ns
 * (1 us .. 2 s). When the limit passes, the wait gives up and QLORA_DEV_TIMEOUT is OR-ed into
 * the status word, which qlora_get_last_status then returns; the context stays usable.
 * Returns QLORA_ERR_INVALID_ARG for a limit outside that range. */
QLORA_API int qlora_selftest_wait_timeout(int64_t limit_ns, qlora_stream_t stream);

/* A static, human-readable name for any QLORA_* code (never NULL). */
QLORA_API const char *qlora_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
