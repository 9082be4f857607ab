// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace ptpc {

// Quantisers (quant.cu).
// ldx: row pitch of X in elements (>= Ci, multiple of 8).
cudaError_t launch_quant_act(const void *X, int T, int Ci, int64_t ldx, uint8_t *Xq, float *xs, cudaStream_t st);
// Row split over tensor-parallel ranks: the slice's row maxima (fp32 [T]),
// and the quantisation of the slice with given (combined) row maxima.
cudaError_t launch_row_amax(const void *X, int T, int Ci, int64_t ldx, float *amax, cudaStream_t st);
cudaError_t launch_quant_act_amax(const void *X, int T, int Ci, int64_t ldx, const float *amax, uint8_t *Xq,
                                  float *xs, cudaStream_t st);
cudaError_t launch_quant_act_per_tensor(const void *X, int T, int Ci, int64_t ldx, uint8_t *Xq, float *xs,
                                        uint32_t *amax_slot, cudaStream_t st);
// col_amax: Co + 1 32-bit words of scratch.
cudaError_t launch_quant_weight(const void *W, int Ci, int Co, uint8_t *Wq_t, float *w_scale, uint32_t *col_amax,
                                bool per_tensor, cudaStream_t st);
// Sub-byte per-output-channel weight quantisation: fmt 1 = E2M1 (FP4),
// 2 = E2M3, 3 = E3M2 (FP6); Wp [Co, Ci * bits / 8] packed along K; Ci % 128 == 0.
cudaError_t launch_quant_weight_sub(const void *W, int Ci, int Co, int fmt, uint8_t *Wp, float *w_scale,
                                    uint32_t *col_amax, cudaStream_t st);
// FP8 KV cache (quant.cu, attention.cu): append K/V [T, H, D] bf16 rows to
// slot-major caches ([num_slots, H, D] codes, [num_slots, H] scales), and
// decode attention over them (workspace attn_workspace_bytes).
cudaError_t launch_kv_append(const void *K, const void *V, const int64_t *slots, int T, int H, int D,
                             int64_t num_slots, uint8_t *kc, uint8_t *vc, float *ks, float *vs, cudaStream_t st);
size_t attn_workspace_bytes(int B, int Hq, int D, int max_context);
cudaError_t launch_decode_attention(const void *q, const uint8_t *kc, const uint8_t *vc, const float *ks,
                                    const float *vs, const int32_t *block_tables, const int32_t *context_lens,
                                    int B, int Hq, int Hkv, int D, int block_size, int max_blocks,
                                    int64_t num_slots, int max_context, float softmax_scale, void *out, void *ws,
                                    cudaStream_t st);
cudaError_t launch_apply_scales(const float *y, const float *xs, const float *ws, int T, int Co, void *out,
                                cudaStream_t st);

// Scaled GEMM (gemm.cu).  Its workspace holds the device status word and,
// for shapes whose last wave of prefill tiles is split along K, the split's
// counters and fp32 partial accumulators (gemm_workspace_bytes).
struct GemmProblem {
  const uint8_t *Xq;      // [T, Ci]
  const float *xs;        // [T]   (unused for f32 output)
  const uint8_t *Wq_t;    // [Co, Ci]
  const float *ws;        // [Co]  (unused for f32 output)
  int T, Ci, Co;
  void *out;              // bf16 [T, Co] or fp32 [T, Co]
  bool f32_out;           // unscaled fp32 output (naive step 1)
  uint32_t *status;       // device status word
  bool pdl;               // launch as a programmatic dependent of the previous kernel
  int wfmt;               // weight format: 0 E4M3, 1 E2M1, 2 E2M3, 3 E3M2 (packed along Ci)
  size_t ws_bytes;        // workspace at `status` (the split tail needs gemm_workspace_bytes)
};

cudaError_t launch_scaled_gemm(const GemmProblem &p, cudaStream_t st);

// CTAs per tile the decode kernel uses for a shape (1: whole tiles; larger:
// K split over a cluster of that many CTAs).  For tests and reports.
int gemm_ksplit(int T, int Ci, int Co);

// Tail tiles' split of the pair kernel for a shape with ws_bytes of
// workspace (0: every tile whole).  For tests and reports.
int gemm_tail_split(int T, int Ci, int Co, size_t ws_bytes);

// Tokens a tile of the pair kernel's swapped-operand plan holds for a shape
// (0: the plan is not swapped).  For tests and reports.
int gemm_swap_tokens(int T, int Ci, int Co, size_t ws_bytes);

// Workspace bytes of a GEMM call (a multiple of 256).
size_t gemm_workspace_bytes(int T, int Ci, int Co);

int num_sms();

// Re-reads the PTPC_FORCE_* tuning overrides from the environment (they are
// otherwise read once, at the first GEMM call).
void reload_tuning();
void attn_reload_tuning();

// Tensor-map cache counters since the library was loaded.
void map_cache_stats(uint64_t *hits, uint64_t *misses);

// The cache's own logic on a private instance with a stand-in encoder (no
// GPU needed): number of failed checks, 0 when it behaves.
int map_cache_selftest();

}  // namespace ptpc
