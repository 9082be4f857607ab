/*
 * ptpc.h - C ABI of the PTPC-FP8 library for NVIDIA B200 (sm_100a).
 *
 * PTPC-FP8 = per-token activation, per-channel weight FP8 quantisation
 * ("PTPC-FP8: boosting vLLM performance on AMD ROCm", vLLM blog, sections
 * "What is PTPC-FP8" and "Per-Token Activation + Per-Channel Weight
 * Quantization").  The activation X is T x Ci (T tokens, Ci input channels),
 * the weight W is Ci x Co (Co output channels); X gets one scale per token
 * (Delta_X[T x 1]) and W one scale per output column (Delta_W[1 x Co]).  The
 * GEMM applies token_scale[t] * channel_scale[o] inside its epilogue, before
 * the single store of the result (section "The challenge: two-step vs fused":
 * the fused call that hands both scale vectors to the FP8 GEMM).
 *
 * Number formats (the page names none; these are this library's readings):
 *   - FP8 codes are OCP E4M3 ("e4m3fn", bias 7, max 448, no infinities).
 *   - scale = amax / 448 as an IEEE fp32 division, round-to-nearest-even;
 *     an all-zero row/column gets scale 1.0f and all codes 0x00.
 *   - code = saturating round-half-to-even E4M3 of the fp32 quotient x / scale.
 *   - out[t][o] = bf16_RNE((acc[t][o] * x_scale[t]) * w_scale[o]), acc the
 *     fp32 tensor-core sum of the decoded code products.
 *
 * Conventions shared by every entry point:
 *   - Pointers named *_dev are device pointers; every buffer is owned by the
 *     caller.  Apart from the 4 KiB static scratch array that
 *     ptpc_scaled_mm_static_scratch uses (held by every GPU that loads the
 *     library), the library never allocates or frees device memory.
 *   - Layouts are dense row-major.  bf16 tensors are passed as raw 16-bit
 *     patterns (void*).
 *   - Alignment: every device pointer must be 16-byte aligned
 *     (PTPC_ERR_MISALIGNED otherwise); so must every row of X (ldx % 8 == 0).
 *   - Shapes: T >= 0 (T == 0 is a no-op returning PTPC_OK); Ci and Co must be
 *     positive multiples of 16 (PTPC_ERR_UNSUPPORTED_SHAPE otherwise), and
 *     T, Ci, Co must each fit in 31 bits.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns; none synchronises, except
 *     ptpc_get_device_status and ptpc_static_scratch_status.
 *   - Errors: the return value is a ptpc_status.  All argument checks run
 *     before any launch; a failed check launches nothing.  A failed launch
 *     returns PTPC_ERR_CUDA.  No C++ exception crosses this boundary.
 *   - Workspace: entry points that take (ws_dev, ws_bytes) need at least
 *     ptpc_workspace_size(op, T, Ci, Co) bytes, zero-filled before its first
 *     use.  Each successful call leaves the workspace's control words zero
 *     again, so a workspace is zero-filled only once.  Calls that share a
 *     workspace must not overlap on the GPU.
 *   - Inputs are assumed finite.  Non-finite inputs do not fault but give
 *     unspecified codes.  The GEMM epilogue multiplies in the order
 *     (acc * x_scale) * w_scale in fp32; outputs are specified where that
 *     intermediate product is finite (|acc * x_scale| < 2^128).  Since
 *     |acc| <= Ci * 448^2 and x_scale = amax / 448, that holds whenever a
 *     token's amax is below 2^128 / (448 * Ci): within 2^24 of the bf16
 *     maximum at Ci = 28672, 2^26 at Ci = 2^17.
 */
#ifndef PTPC_H_
#define PTPC_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PTPC_API __attribute__((visibility("default")))
#else
#define PTPC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PTPC_OK = 0,
    PTPC_ERR_INVALID_ARG = 1,          /* null pointer, negative size, unknown op */
    PTPC_ERR_MISALIGNED = 2,           /* a pointer is not 16-byte aligned */
    PTPC_ERR_UNSUPPORTED_SHAPE = 3,    /* Ci or Co not a positive multiple of 16, or too large */
    PTPC_ERR_WORKSPACE_TOO_SMALL = 4,  /* ws_bytes < ptpc_workspace_size(...) */
    PTPC_ERR_UNSUPPORTED_DEVICE = 5,   /* current device is not compute capability 10.0 */
    PTPC_ERR_CUDA = 6,                 /* a CUDA runtime/driver call failed */
    PTPC_ERR_DEVICE_TIMEOUT = 7,       /* a kernel's bounded wait ran out (device status word) */
    PTPC_ERR_NOT_IMPLEMENTED = 8       /* reserved: no entry point returns it at present */
} ptpc_status;

/* Weight formats.  E4M3 is the PTPC-FP8 format of the entry points above;
 * the others are the sub-byte formats of FP4-FP7 runtime weight quantisation
 * (the llminfo.tech summary "Running LLMs at custom floating-points
 * (near-lossless FP6)": FP6-LLM extended to FP4-FP7 with per-channel
 * quantisation), taken as the OCP MX element types that the tensor cores
 * read natively.  Every format keeps one fp32 scale per output channel,
 * amax / (largest value of the format), and per-token FP8 activations. */
typedef enum {
    PTPC_WFMT_E4M3 = 0,   /* FP8, 1 byte a code, max 448 */
    PTPC_WFMT_E2M1 = 1,   /* FP4, max 6; two codes a byte, even K position in the low nibble */
    PTPC_WFMT_E2M3 = 2,   /* FP6, max 7.5; 16 codes in 12 bytes, code j at bits [6j, 6j+6) little-endian */
    PTPC_WFMT_E3M2 = 3    /* FP6, max 28; packed like E2M3 */
} ptpc_weight_format;

/* Operation ids for ptpc_workspace_size. */
typedef enum {
    PTPC_OP_QUANTIZE_WEIGHTS = 1,
    PTPC_OP_SCALED_MM = 2,
    PTPC_OP_LINEAR = 3,
    PTPC_OP_BENCH_PER_TENSOR = 4,      /* per-tensor quantisers (measurement only) */
    PTPC_OP_BENCH_UNSCALED_MM = 5      /* unscaled fp32 GEMM (measurement only) */
} ptpc_op;

/* Per-token activation quantisation (the page's Delta_X[T x 1]).
 *   X_dev       bf16 [T, Ci] row-major with row pitch ldx elements, read only
 *               (ldx >= Ci, ldx % 8 == 0: e.g. a column slice of a wider
 *               tensor; ldx == Ci for a dense tensor).
 *   Xq_dev      u8   [T, Ci] row-major, written: E4M3 codes of row t with
 *               scale x_scale[t] (the K-major A operand of the GEMM).
 *   x_scale_dev fp32 [T], written: amax(|X[t, :]|) / 448 (1.0f if amax == 0).
 * Codes and scales are bit-exact functions of X (see the conventions above). */
PTPC_API int ptpc_quantize_activations(const void *X_dev, int64_t T, int64_t Ci, int64_t ldx,
                              uint8_t *Xq_dev, float *x_scale_dev, void *stream);

/* Tensor parallelism with the input channels split over ranks (a
 * row-parallel linear, as in the page's TP = 2 evaluation setup in its
 * benchmark section): a rank holds a column slice X_r [T, Ci_r] of every
 * token, but the token's scale comes from the whole row.  The ranks combine
 * their slice maxima (maximum over ranks, exact in any order) and quantise
 * their slice with the combined maxima; the codes and scales are then exactly
 * those ptpc_quantize_activations gives the whole row.
 *
 * ptpc_act_row_amax: amax_dev fp32 [T] = max_k |X[t, k]| of the slice (exact;
 * 0 for an all-zero row).  X as for ptpc_quantize_activations. */
PTPC_API int ptpc_act_row_amax(const void *X_dev, int64_t T, int64_t Ci, int64_t ldx, float *amax_dev,
                               void *stream);

/* ptpc_quantize_activations with the row maxima given: x_scale[t] =
 * amax[t] / 448 (1.0f and all codes 0x00 when amax[t] == 0), codes of the
 * slice with that scale.  amax_dev fp32 [T] must hold maxima of bf16
 * magnitudes that are at least the slice's own (the combined maxima from
 * ptpc_act_row_amax). */
PTPC_API int ptpc_quantize_activations_amax(const void *X_dev, int64_t T, int64_t Ci, int64_t ldx,
                                            const float *amax_dev, uint8_t *Xq_dev, float *x_scale_dev,
                                            void *stream);

/* Per-output-channel weight quantisation (the page's Delta_W[1 x Co]); run
 * once per weight, e.g. when a bf16 checkpoint is loaded.
 *   W_dev       bf16 [Ci, Co] row-major, read only.
 *   Wq_t_dev    u8   [Co, Ci] row-major, written: codes of column o of W,
 *               transposed so that each output channel's codes are
 *               contiguous along Ci (the K-major B operand of the GEMM).
 *   w_scale_dev fp32 [Co], written: amax(|W[:, o]|) / 448 (1.0f if 0).
 *   ws_dev      workspace of ptpc_workspace_size(PTPC_OP_QUANTIZE_WEIGHTS, 0, Ci, Co)
 *               bytes (column maxima). */
PTPC_API int ptpc_quantize_weights(const void *W_dev, int64_t Ci, int64_t Co,
                          uint8_t *Wq_t_dev, float *w_scale_dev,
                          void *ws_dev, size_t ws_bytes, void *stream);

/* Fused row-wise-scaled FP8 GEMM (the page's fused path: the token scales
 * scale the rows of the product, the channel scales its columns):
 *   out[t][o] = bf16_RNE((sum_k dec(Xq[t][k]) * dec(Wq_t[o][k]) * x_scale[t]) * w_scale[o])
 *   Xq_dev      u8 [T, Ci], x_scale_dev fp32 [T]   (from ptpc_quantize_activations)
 *   Wq_t_dev    u8 [Co, Ci], w_scale_dev fp32 [Co] (from ptpc_quantize_weights)
 *   out_dev     bf16 [T, Co] row-major, written once (no intermediate array).
 *   ws_dev      ptpc_workspace_size(PTPC_OP_SCALED_MM, T, Ci, Co) bytes: the
 *               device status word and, for prefill-sized T, room for the
 *               split tail (below), about 19 MB.
 * The sum over k is an fp32 tensor-core accumulation; its order is not
 * specified.  For T <= 192 and few output tiles, K is split over a cluster of
 * 2, 4 or 8 CTAs (see ptpc_gemm_ksplit) whose fp32 partial sums are added in
 * a fixed order.  For prefill-sized T with a long K (at least 16384) whose
 * last wave of output tiles would keep at most half the SMs busy, those
 * tiles are split along K over the whole GPU (see ptpc_gemm_tail_split):
 * their fp32 partial sums go through the workspace and are added in a fixed
 * order.  Ragged prefill T may run with the operands swapped (see
 * ptpc_gemm_swap_tokens); the products and their accumulation are the same
 * kind, only the tiling differs.  Results are deterministic for a given
 * shape and workspace size.  With a smaller workspace (at least the status
 * word) every tile is computed whole. */
PTPC_API int ptpc_scaled_mm(const uint8_t *Xq_dev, const float *x_scale_dev,
                   const uint8_t *Wq_t_dev, const float *w_scale_dev,
                   int64_t T, int64_t Ci, int64_t Co, void *out_dev,
                   void *ws_dev, size_t ws_bytes, void *stream);

/* Fused quantise + GEMM: ptpc_quantize_activations of X into the workspace,
 * then ptpc_scaled_mm, on one stream (the GEMM is launched as a programmatic
 * dependent of the quantiser).  The page's dynamic path, in which activations
 * are quantised on every call rather than ahead of time: the bf16 activation
 * goes in, the bf16 output comes out.
 *   X_dev bf16 [T, Ci] with row pitch ldx (as for ptpc_quantize_activations);
 *   Wq_t_dev / w_scale_dev as for ptpc_scaled_mm;
 *   out_dev bf16 [T, Co];
 *   ws_dev ptpc_workspace_size(PTPC_OP_LINEAR, T, Ci, Co) bytes (holds Xq and
 *   x_scale as well as the GEMM's workspace). */
PTPC_API int ptpc_linear(const void *X_dev, int64_t ldx, const uint8_t *Wq_t_dev, const float *w_scale_dev,
                int64_t T, int64_t Ci, int64_t Co, void *out_dev,
                void *ws_dev, size_t ws_bytes, void *stream);

/* Bytes of workspace an entry point needs for the given shape (0 on invalid
 * arguments).  The value is a multiple of 256. */
PTPC_API size_t ptpc_workspace_size(int op, int64_t T, int64_t Ci, int64_t Co);

/* Synchronises `stream`, reads the device status word at the start of ws_dev
 * (written by kernels whose bounded waits ran out), clears it and returns
 * PTPC_OK or PTPC_ERR_DEVICE_TIMEOUT (PTPC_ERR_CUDA if the read fails). */
PTPC_API int ptpc_get_device_status(void *ws_dev, void *stream);

/* Self-test of the failure path: launches on `stream` one thread that waits,
 * with the same bounded wait the GEMM kernels use, on an mbarrier that
 * nothing arrives at.  The wait runs out after its limit (about 2 s of GPU
 * time), the kernel sets a bit in the status word at the start of ws_dev
 * (256-byte aligned workspace of at least 256 bytes) and returns; nothing
 * faults or hangs and the context stays usable.  A following
 * ptpc_get_device_status(ws_dev, stream) returns PTPC_ERR_DEVICE_TIMEOUT and
 * clears the word.  No counterpart on the page. */
PTPC_API int ptpc_selftest_wait_timeout(void *ws_dev, void *stream);

/* Static, human-readable name of a status code. */
PTPC_API const char *ptpc_status_string(int status);

/* How ptpc_scaled_mm / ptpc_linear run a shape on the current device: the
 * number of CTAs that share each output tile (1: every tile whole; 2, 4 or 8:
 * K split over a cluster of that many CTAs, decode-sized T only).  0 on
 * invalid arguments, T == 0 or an unsupported device.  Launches nothing. */
PTPC_API int ptpc_gemm_ksplit(int64_t T, int64_t Ci, int64_t Co);

/* Bytes of a quantised weight of format fmt: Co * Ci * bits / 8 (0 on
 * invalid arguments; the sub-byte formats need Ci % 128 == 0). */
PTPC_API size_t ptpc_weight_bytes(int fmt, int64_t Ci, int64_t Co);

/* Per-output-channel weight quantisation to format fmt (ptpc_weight_format):
 * w_scale[o] = amax(|W[:, o]|) / max_format (1.0f for an all-zero column),
 * code = saturating round-half-to-even of the fp32 quotient W[k][o] / w_scale[o]
 * in the format (sign kept), written transposed and packed along Ci:
 *   Wq_dev  u8 [Co, ptpc_weight_bytes(fmt, Ci, Co) / Co], row o = channel o's
 *           Ci codes in K order (E4M3: exactly ptpc_quantize_weights' Wq_t).
 * Sub-byte formats need Ci % 128 == 0 (PTPC_ERR_UNSUPPORTED_SHAPE) and a
 * 32-byte aligned Wq_dev (PTPC_ERR_MISALIGNED), as TMA reads them.
 * ws_dev: ptpc_workspace_size(PTPC_OP_QUANTIZE_WEIGHTS, 0, Ci, Co) bytes. */
PTPC_API int ptpc_quantize_weights_fmt(const void *W_dev, int64_t Ci, int64_t Co, int fmt,
                                       uint8_t *Wq_dev, float *w_scale_dev,
                                       void *ws_dev, size_t ws_bytes, void *stream);

/* ptpc_scaled_mm with weights of format fmt (from ptpc_quantize_weights_fmt):
 *   out[t][o] = bf16_RNE((sum_k dec_e4m3(Xq[t][k]) * dec_fmt(Wq[o][k]) * x_scale[t]) * w_scale[o]).
 * The tensor cores read the packed FP4/FP6 codes directly (mixed-format
 * kind::f8f6f4 MMA), so decode-sized T streams 1/2 (FP4) or 3/4 (FP6) of the
 * FP8 weight bytes.  Same plans, workspace and conventions as ptpc_scaled_mm. */
PTPC_API int ptpc_scaled_mm_fmt(const uint8_t *Xq_dev, const float *x_scale_dev,
                                const uint8_t *Wq_dev, const float *w_scale_dev, int fmt,
                                int64_t T, int64_t Ci, int64_t Co, void *out_dev,
                                void *ws_dev, size_t ws_bytes, void *stream);

/* ptpc_linear with weights of format fmt: per-token FP8 quantisation of X,
 * then ptpc_scaled_mm_fmt, on one stream; workspace as for ptpc_linear. */
PTPC_API int ptpc_linear_fmt(const void *X_dev, int64_t ldx, const uint8_t *Wq_dev, const float *w_scale_dev,
                             int fmt, int64_t T, int64_t Ci, int64_t Co, void *out_dev,
                             void *ws_dev, size_t ws_bytes, void *stream);

/* Re-reads the GEMM's tuning overrides from the environment.  They are
 * otherwise read once, at the first GEMM call of the process, so that no call
 * pays for environment lookups:
 *   PTPC_FORCE_KERNEL  = pair | decode   which GEMM kernel runs a shape,
 *   PTPC_FORCE_PAIR_BN = 128 | 256       tile width of the prefill kernel,
 *   PTPC_FORCE_KSPLIT  = 1 | 2 | 4 | 8   CTAs per tile of the decode kernel,
 *   PTPC_FORCE_SPLIT_TAIL = 0 | 1        the prefill kernel's split tail off,
 *                                        or on wherever the workspace allows,
 *   PTPC_FORCE_SWAP    = 0 | 1           the prefill kernel's swapped operands
 *                                        (weights as the 256-row operand,
 *                                        tokens as the tile's columns) off, or
 *                                        on for every prefill-kernel shape,
 *   PTPC_FORCE_GROUP_M = 1 .. 63         tile rows the prefill kernel visits
 *                                        together (their activation tiles
 *                                        kept in L2 while the columns sweep),
 *   PTPC_FORCE_ATTN_CHUNK = 512 | 1024 | 2048 | 4096  context positions a
 *                                        CTA of ptpc_decode_attention takes
 *                                        (4096 only on the tensor-memory
 *                                        kernel; the other takes at most 2048),
 *   PTPC_FORCE_ATTN_KERNEL = mma | tc    which decode-attention kernel runs
 *                                        (tc only where it applies).
 * Each is honoured only where the forced choice is feasible for the shape;
 * results stay within the GEMM's tolerance under every choice.  For tuning
 * and tests, not for production.  Not thread-safe with concurrent GEMM calls
 * that should see a consistent setting.  No counterpart on the page. */
PTPC_API int ptpc_reload_tuning_overrides(void);

/* The split-tail plan of ptpc_scaled_mm / ptpc_linear for a shape on the
 * current device with ws_bytes of GEMM workspace: 0 if every output tile is
 * computed whole, else the number of CTA pairs that share each tile of the
 * last wave (split along K).  Launches nothing.  No counterpart on the page. */
PTPC_API int ptpc_gemm_tail_split(int64_t T, int64_t Ci, int64_t Co, size_t ws_bytes);

/* The operand order of the prefill GEMM's plan for a shape on the current
 * device with ws_bytes of GEMM workspace: 0 if its tiles are 256 tokens x
 * 128 or 256 channels (or the decode kernel runs the shape), else the number
 * of tokens a tile holds when the operands are swapped (256 channels x that
 * many tokens; a multiple of 32, at most 256, chosen so that the token tiles
 * divide T evenly, e.g. 160 for T = 300).  Launches nothing.  No counterpart
 * on the page. */
PTPC_API int ptpc_gemm_swap_tokens(int64_t T, int64_t Ci, int64_t Co, size_t ws_bytes);

/* ptpc_scaled_mm without a caller-provided workspace.  The page has no
 * counterpart: this exists for callers that cannot allocate device memory
 * when they call the GEMM (an engine that partitions all device memory at
 * start-up and forbids allocation on its serving path, or an integration that
 * only hands over input and output buffers).  Same arguments, layouts and
 * results as ptpc_scaled_mm minus (ws_dev, ws_bytes).
 *   Scratch: a file-scope 4 KiB device array inside the library, held by
 *   every GPU that loads the library until the process exits; the GEMM uses
 *   its first 256 bytes (the device status word).  The array has no room
 *   for the split tail, so every output tile is computed whole; results are
 *   bit-identical to ptpc_scaled_mm's wherever that plan has no split tail
 *   (ptpc_gemm_tail_split), and within the GEMM's tolerance of them elsewhere.
 *   The first call on a device looks up the array's device address once
 *   (cudaGetSymbolAddress; its failure returns PTPC_ERR_CUDA).
 *   Nothing is allocated and nothing is cleared per call: the status word is
 *   zero when the library is loaded, the GEMM only sets timeout bits in it,
 *   and those stay set until ptpc_static_scratch_status reads and clears
 *   them.  All calls share the one array: calls that overlap on the GPU
 *   (different streams, or different host threads) race on it, and a timeout
 *   of one of them cannot be told apart from the other's. */
PTPC_API int ptpc_scaled_mm_static_scratch(const uint8_t *Xq_dev, const float *x_scale_dev,
                                           const uint8_t *Wq_t_dev, const float *w_scale_dev,
                                           int64_t T, int64_t Ci, int64_t Co, void *out_dev, void *stream);

/* Device status of ptpc_scaled_mm_static_scratch on the current device: like
 * ptpc_get_device_status, synchronises `stream`, reads the status word of the
 * static scratch array, clears it and returns PTPC_OK or
 * PTPC_ERR_DEVICE_TIMEOUT (a bounded wait of some static-scratch GEMM since the
 * last read ran out; its output is then incomplete).  Allocates nothing.
 * No counterpart on the page. */
PTPC_API int ptpc_static_scratch_status(void *stream);

/* ------------------------------------------------------------------------- */
/* FP8 (E4M3) KV cache.  The PTPC page runs every evaluation with            */
/* kv_cache_dtype=fp8_e4m3 (its lm-evaluation-harness commands).  The page    */
/* gives no scale rule; this library applies the PTPC per-token rule to       */
/* every (token, KV head) vector of D values: scale = amax / 448, codes       */
/* E4M3_satRNE(x / scale), exactly as ptpc_quantize_activations on the rows   */
/* of a [T * H, D] view.  The cache is paged and slot-major:                  */
/*   codes  cache[(slot * H + h) * D + d]  (u8),  scale  scales[slot * H + h], */
/*   slot = block * block_size + offset.                                      */
/* ------------------------------------------------------------------------- */

/* Appends T tokens: K_dev, V_dev bf16 [T, H, D]; slots_dev int64 [T] (a
 * negative slot skips the token, as does a slot >= num_blocks * block_size);
 * k_cache / v_cache u8 [num_blocks * block_size, H, D]; k_scale / v_scale
 * fp32 [num_blocks * block_size, H].  D is 64 or 128; block_size >= 8.
 * Tokens with equal slots race. */
PTPC_API int ptpc_kv_cache_append(const void *K_dev, const void *V_dev, const int64_t *slots_dev, int64_t T,
                                  int64_t H, int64_t D, int64_t block_size, int64_t num_blocks,
                                  uint8_t *k_cache_dev, uint8_t *v_cache_dev, float *k_scale_dev,
                                  float *v_scale_dev, void *stream);

/* Workspace bytes of ptpc_decode_attention (0 on invalid arguments): the
 * device status word (first 256 bytes) and the chunks' partial results. */
PTPC_API size_t ptpc_decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t D, int64_t max_context);

/* Decode attention (one query per sequence) over the FP8 cache:
 *   q_dev bf16 [B, Hq, D], query head h reads KV head h / (Hq / Hkv)
 *   (Hq / Hkv <= 16); the cache holds fewer than 2^31 slots
 *   (num_blocks * block_size; PTPC_ERR_UNSUPPORTED_SHAPE otherwise);
 *   block_tables_dev int32 [B, max_blocks]: the cache blocks of each
 *   sequence in order; context_lens_dev int32 [B]: positions to attend to
 *   (<= max_context; positions whose block-table entry is missing, negative
 *   or past the cache are left out);
 *   out[b][h][d] = bf16_RNE(sum_l p_l * v_scale_l * dec(V_l[d])),
 *   p = softmax_l(softmax_scale * k_scale_l * sum_d q[d] * dec(K_l[d]))
 *   (0 for a sequence with no position), computed in fp32: q K^T from
 *   E4M3 tensor-core products of the K codes with q written as two E4M3
 *   terms (exact for every bf16 q whose scaled value is at least E4M3's
 *   smallest normal 2^-6, see the kernel), P V from tensor-core products of the V codes with P written
 *   as three E4M3 terms (or, in the warp-level kernel, f16 P times the
 *   exactly decoded V codes; see ptpc_decode_attention_kernel).
 *   out_dev bf16 [B, Hq, D].
 *   ws_dev: ptpc_decode_attention_workspace_size(B, Hq, D, max_context)
 *   bytes (the context is split into chunks of 512 to 2048 positions, 4096
 *   with the tensor-memory kernel, chosen per launch to fill the GPU, whose
 *   partial results are combined by a second kernel; when one chunk covers
 *   every context the attention kernel writes the output itself).  It starts with the device status word: the
 *   tensor-memory kernel (see ptpc_decode_attention_kernel) sets a bit there
 *   when one of its bounded waits runs out, which ptpc_get_device_status
 *   reports; the word must be zero before the first call (a zeroed
 *   workspace). */
PTPC_API int ptpc_decode_attention(const void *q_dev, const uint8_t *k_cache_dev, const uint8_t *v_cache_dev,
                                   const float *k_scale_dev, const float *v_scale_dev,
                                   const int32_t *block_tables_dev, const int32_t *context_lens_dev, int64_t B,
                                   int64_t Hq, int64_t Hkv, int64_t D, int64_t block_size, int64_t num_blocks,
                                   int64_t max_blocks, int64_t max_context, float softmax_scale, void *out_dev,
                                   void *ws_dev, size_t ws_bytes, void *stream);

/* Which decode-attention kernel ptpc_decode_attention runs for a shape on
 * this library: 2 the kernel on the fifth-generation tensor cores (tcgen05
 * MMAs into tensor memory, TMA loads), for D = 128 and block sizes that are
 * multiples of 8 (groups of 9 to 16 query heads take two CTAs a KV head);
 * 1 the warp-level kernel (mma.sync tensor-core tiles) for every other
 * supported shape.  PTPC_FORCE_ATTN_KERNEL=mma forces kernel 1 and =tc asks for
 * kernel 2 where it applies (read at the first launch or by
 * ptpc_reload_tuning_overrides; tuning and tests only).  Both compute the
 * same function; the tensor-memory kernel multiplies P, written as three
 * E4M3 terms (about 12 significant bits), by the E4M3 V codes, where the
 * warp-level kernel uses f16 P (11).  0 on invalid arguments. */
PTPC_API int ptpc_decode_attention_kernel(int64_t Hq, int64_t Hkv, int64_t D, int64_t block_size);

/* ------------------------------------------------------------------------- */
/* Measurement-only entry points: the comparison paths the page describes.  */
/* ------------------------------------------------------------------------- */

/* Naive two-step path, step 1 (section "The challenge: two-step vs fused":
 * the FP8 GEMM called without scales): the unscaled FP8 GEMM written out as
 * an fp32 intermediate y_dev [T, Co] row-major.  Same mainloop as
 * ptpc_scaled_mm, so y is bit-identical to that kernel's accumulator.
 * ws_dev: ptpc_workspace_size(PTPC_OP_BENCH_UNSCALED_MM, T, Ci, Co) bytes. */
PTPC_API int ptpc_bench_unscaled_mm_f32(const uint8_t *Xq_dev, const uint8_t *Wq_t_dev,
                               int64_t T, int64_t Ci, int64_t Co, float *y_dev,
                               void *ws_dev, size_t ws_bytes, void *stream);

/* Host-side tensor-map cache of the GEMM entry points: how many maps were
 * taken from the cache (*hits) and how many were encoded (*misses) since the
 * library was loaded.  A GEMM call needs two or three maps, keyed by pointer,
 * shape, tile box and element type; repeated calls on the same buffers hit.
 * No counterpart on the page. */
PTPC_API int ptpc_bench_map_cache_stats(uint64_t *hits, uint64_t *misses);

/* Self-test of the tensor-map cache's logic on a private instance with a
 * stand-in encoder (no GPU needed): hits, misses for another pointer or shape,
 * emptying at capacity, failed encodes not stored.  PTPC_OK if every check
 * holds.  No counterpart on the page. */
PTPC_API int ptpc_bench_map_cache_selftest(void);

/* Effective SM clock during a measurement: one sleeping thread on one SM
 * writes (globaltimer ns, clock64 cycles) pairs to records_dev
 * (uint64 [max_records][2], 8-byte aligned) about every period_ns (>= 1000)
 * until duration_ns (<= 120 s) have passed or max_records (>= 2) are
 * written, and the number written to *count_dev.  Launched on `stream`,
 * typically a side stream that runs alongside the kernels being timed; it
 * uses no shared memory.  Clock = cycles / ns between records.  Every wait
 * inside is bounded.  No counterpart on the page. */
PTPC_API int ptpc_bench_clock_probe(uint64_t *records_dev, int max_records, uint64_t period_ns,
                                    uint64_t duration_ns, int *count_dev, void *stream);

/* Naive two-step path, step 2 (same section: the rank-1 rescale of the
 * intermediate by the token scales, then the channel scales): reads y_dev
 * fp32 [T, Co] and writes
 * out_dev[t][o] = bf16_RNE((y[t][o] * x_scale[t]) * w_scale[o]). */
PTPC_API int ptpc_bench_apply_scales(const float *y_dev, const float *x_scale_dev,
                            const float *w_scale_dev, int64_t T, int64_t Co,
                            void *out_dev, void *stream);

/* Per-tensor ("standard FP8", the page's Delta_X[1] / Delta_W[1]) activation
 * quantisation: one scale for all of X.  Writes the codes to Xq_dev [T, Ci]
 * and that one scale to every entry of x_scale_dev [T], so ptpc_scaled_mm can
 * consume the result unchanged.  ws_dev: ptpc_workspace_size(
 * PTPC_OP_BENCH_PER_TENSOR, T, Ci, 0) bytes. */
PTPC_API int ptpc_bench_quantize_activations_per_tensor(const void *X_dev, int64_t T, int64_t Ci, int64_t ldx,
                                               uint8_t *Xq_dev, float *x_scale_dev,
                                               void *ws_dev, size_t ws_bytes, void *stream);

/* Per-tensor weight quantisation: one scale for all of W (Ci x Co), codes
 * transposed to Wq_t_dev [Co, Ci], the scale written to every entry of
 * w_scale_dev [Co].  ws_dev as for ptpc_quantize_weights. */
PTPC_API int ptpc_bench_quantize_weights_per_tensor(const void *W_dev, int64_t Ci, int64_t Co,
                                           uint8_t *Wq_t_dev, float *w_scale_dev,
                                           void *ws_dev, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PTPC_H_ */
