// Decode attention on the fifth-generation tensor cores (attention_tc.cu):
// head size 128, GQA groups of up to 16 heads, cache blocks of a multiple of
// 8 positions.  attention.cu chooses between it and the warp-level kernel and
// runs the combine kernel after either.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace ptpc {

bool attn_tc_supported(int D, int G, int block_size);
// The kernel decode attention runs for this shape: 1 the warp-level kernel,
// 2 the tensor-memory kernel (attention.cu, after the tuning override).
int attn_kernel_choice(int D, int G, int block_size);
// CTAs of the kernel that can be resident at once on this device.
int attn_tc_resident();
size_t attn_tc_smem_bytes(int chunk);
// One CTA per (chunk of `chunk` positions, KV head and group of up to 8 of
// its query heads, sequence): partial
// results into part_ml [B, Hq, splits, 2] and part_acc [B, Hq, splits, 128],
// or, with splits == 1 and out non-null, the bf16 output [B, Hq, 128]
// directly (the combine kernel's arithmetic for one chunk); a bounded wait
// that runs out sets a bit in *status.  chunk: a multiple of 128, at most
// 4096.
cudaError_t launch_attn_tc(const void *q, const uint8_t *kc, const uint8_t *vc, const float *ks, const float *vs,
                           const int32_t *block_tables, const int32_t *context_lens, int B, int Hq, int Hkv,
                           int block_size, int max_blocks, int64_t num_slots, uint64_t bs_magic, int chunk,
                           int splits, float scale_log2, float *part_ml, float *part_acc, void *out,
                           uint32_t *status, cudaStream_t st);

}  // namespace ptpc
