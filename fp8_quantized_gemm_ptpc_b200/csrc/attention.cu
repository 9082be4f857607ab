// Decode attention over an FP8 (E4M3) paged KV cache, for sm_100a.
//
// The PTPC page ("PTPC-FP8: boosting vLLM performance on AMD ROCm") runs
// every evaluation with kv_cache_dtype=fp8_e4m3 next to PTPC weights and
// activations.  The cache here holds E4M3 codes with one fp32 scale per
// (token, KV head), the PTPC per-token rule on every head's D-vector
// (kv_append_kernel in quant.cu writes it):
//   codes  cache[(slot * Hkv + g) * D + d],  scale  scales[slot * Hkv + g],
//   slot = block_tables[b][pos / block_size] * block_size + pos % block_size.
// For query head h of sequence b (KV head g = h / (Hq / Hkv)):
//   s_l = softmax_scale * k_scale[l] * sum_d q[h, d] * dec(K[l, d]),
//   out[h, d] = sum_l softmax(s)_l * v_scale[l] * dec(V[l, d]).
//
// Decode is bound by the bytes of the cache it streams (one byte per code).
// A CTA takes one (sequence, KV head) and a chunk of 512 context positions,
// whose block-table entries it first reads into shared memory; its four warps
// take 16-position tiles in turn.  A warp gathers a tile's K and V codes and
// scales with asynchronous copies (cp.async, 16 bytes per copy, zero-filled
// for positions that are not read) into one of two shared-memory stages, so
// the next tile's bytes are in flight while it decodes this one exactly to
// f16 (cvt e4m3x2 -> f16x2; every E4M3 value is an f16 value) and runs
// FlashAttention-style tensor-core MMAs (mma.sync m16n8k16, f16 inputs, fp32
// accumulation) with the GQA group's query heads as the 16 rows: S = Q K^T,
// an online softmax in base 2, O += P V.  The key scales multiply the scores;
// the value scales enter P relative to the tile's largest one (so P stays in
// [0, 1] in f16), and the accumulator is kept in units of that value scale
// (moved between tiles with the softmax's own rescale).  The warps' states
// are combined in shared memory and every CTA writes (max, sum, accumulator)
// for its chunk; a second kernel combines the chunks and rounds to bf16.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace ptpc {

namespace {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = 32 * kAttnWarps;

struct AttnParams {
  const __nv_bfloat16 *q;      // [B, Hq, D]
  const uint8_t *kc, *vc;      // [num_slots, Hkv, D] codes
  const float *ks, *vs;        // [num_slots, Hkv] scales
  const int32_t *block_tables; // [B, max_blocks]
  const int32_t *context_lens; // [B]
  int Hq, Hkv, G, block_size, max_blocks, splits;
  int64_t num_slots;           // cache slots (num_blocks * block_size): larger slots are skipped
  float scale_log2;            // softmax_scale * log2(e)
  float *part_ml;              // [B, Hq, splits, 2]: running max (base-2 units), sum
  float *part_acc;             // [B, Hq, splits, D]
};

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }

// Two bf16 (low half first) -> two f16: exact for magnitudes in f16's range.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w));
  return h2_bits(__floats2half2_rn(f.x, f.y));
}

// Two E4M3 codes (low byte first) -> two f16 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two_codes, __NV_E4M3);
  return (uint32_t)r.x | ((uint32_t)r.y << 16);
}

// 16 codes -> 16 f16 at dst (32 bytes, 16-byte aligned).
__device__ __forceinline__ void decode16(uint4 c, __half *dst) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
  #pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = e4m3x2_to_f16x2(w[i] & 0xFFFFu);
    o[2 * i + 1] = e4m3x2_to_f16x2(w[i] >> 16);
  }
  reinterpret_cast<uint4 *>(dst)[0] = make_uint4(o[0], o[1], o[2], o[3]);
  reinterpret_cast<uint4 *>(dst)[1] = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ void ldsm_x2(uint32_t &r0, uint32_t &r1, const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t &r0, uint32_t &r1, const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

// D (16x8 fp32) += A (16x16 f16, row) * B (16x8 f16, col).
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Cache slot of position pos of sequence b, or -1 where the block table has
// no entry for it or names a block outside the cache (such positions are
// masked instead of read).
__device__ __forceinline__ int64_t kv_slot(const AttnParams &p, int b, int pos) {
  const int bi = pos / p.block_size;
  if (bi >= p.max_blocks) return -1;
  const int blk = __ldg(p.block_tables + (int64_t)b * p.max_blocks + bi);
  const int64_t slot = (int64_t)blk * p.block_size + pos % p.block_size;
  return (blk < 0 || slot >= p.num_slots) ? -1 : slot;
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kMinBlockSize = 8;   // the chunk's block-table entries fit in shared memory

// Shared memory of one CTA: every warp's two code stages (K and V codes and
// scales of 16 positions) and its decoded f16 K and V tiles, which at the end
// double as the warps' accumulators; the chunk's block-table entries.
template <int D, int CHUNK>
struct AttnSmem {
  static constexpr int PITCH = D + 8;                                   // f16 per decoded row
  static constexpr int CODE_STAGE = 2 * 16 * D;                         // bytes: K and V codes
  static constexpr int CODES = kAttnWarps * 2 * CODE_STAGE;
  static constexpr int TILES = kAttnWarps * 2 * 16 * PITCH * 2;         // bytes: decoded K and V
  static constexpr int SCALES = kAttnWarps * 2 * 2 * 16 * 4;            // bytes: k and v scales
  static constexpr int BLOCKS = (CHUNK / kMinBlockSize + 2) * 4;
  static constexpr size_t BYTES = (size_t)CODES + TILES + SCALES + BLOCKS;
  static_assert(kAttnWarps * 16 * D * 4 <= TILES, "combine buffer");
};

template <int D, int CHUNK>
__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(const AttnParams p) {
  using SM = AttnSmem<D, CHUNK>;
  constexpr int KS = D / 16;        // 16-wide K steps of S = Q K^T
  constexpr int NT = D / 8;         // 8-wide column tiles of O
  constexpr int PITCH = SM::PITCH;
  constexpr int CB = D / 2;         // code bytes a lane moves per tile row (two lanes per position)
  extern __shared__ __align__(16) uint8_t dsmem[];
  uint8_t *s_codes = dsmem;
  uint8_t *s_tiles = dsmem + SM::CODES;
  float *s_scl = reinterpret_cast<float *>(dsmem + SM::CODES + SM::TILES);
  int *s_blk = reinterpret_cast<int *>(dsmem + SM::CODES + SM::TILES + SM::SCALES);
  __shared__ float s_ml[kAttnWarps][16][2];
  __shared__ float s_unit[kAttnWarps];

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = __ldg(p.context_lens + b);
  const int c0 = split * CHUNK;
  const int c1 = min(c0 + CHUNK, L);

  // the chunk's block-table entries (-1 where there is none)
  const int bi0 = c0 / p.block_size;
  const int nbi = c1 > c0 ? (c1 - 1) / p.block_size - bi0 + 1 : 0;
  for (int i = threadIdx.x; i < nbi; i += kAttnThreads) {
    const int bi = bi0 + i;
    s_blk[i] = bi < p.max_blocks ? __ldg(p.block_tables + (int64_t)b * p.max_blocks + bi) : -1;
  }
  __syncthreads();
  auto slot_of = [&](int pos) -> int64_t {
    if (pos >= c1) return -1;
    const int blk = s_blk[pos / p.block_size - bi0];
    const int64_t slot = (int64_t)blk * p.block_size + pos % p.block_size;
    return (blk < 0 || slot >= p.num_slots) ? -1 : slot;
  };

  __half *sK = reinterpret_cast<__half *>(s_tiles) + warp * 2 * 16 * PITCH;
  __half *sV = sK + 16 * PITCH;
  uint8_t *wcodes = s_codes + warp * 2 * SM::CODE_STAGE;
  float *wscl = s_scl + warp * 2 * 2 * 16;

  // issue the copies of the tile at `base` into code stage `st`
  auto prefetch = [&](int base, int st) {
    const int kk = lane >> 1, half = lane & 1;
    const int64_t slot = slot_of(base + kk);
    const bool valid = slot >= 0;
    const int64_t off = (valid ? slot * p.Hkv + g : 0) * D + half * CB;
    uint8_t *dk = wcodes + st * SM::CODE_STAGE + kk * D + half * CB;
    uint8_t *dv = dk + 16 * D;
    #pragma unroll
    for (int i = 0; i < CB / 16; ++i) {
      cp_async16(dk + 16 * i, p.kc + off + 16 * i, valid);
      cp_async16(dv + 16 * i, p.vc + off + 16 * i, valid);
    }
    if (half == 0) {
      const int64_t si = valid ? slot * p.Hkv + g : 0;
      cp_async4(wscl + (st * 2 + 0) * 16 + kk, p.ks + si, valid);
      cp_async4(wscl + (st * 2 + 1) * 16 + kk, p.vs + si, valid);
    }
  };

  // query fragments (A operand; rows = the group's heads, padded to 16)
  const int r0 = lane >> 2, cq = (lane & 3) * 2;
  uint32_t qa[KS][4];
  {
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(p.q);
    const int64_t hrow0 = (int64_t)b * p.Hq + (int64_t)g * p.G;
    #pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = r0 + ((i & 1) ? 8 : 0);
        const int col = kk * 16 + cq + ((i & 2) ? 8 : 0);
        qa[kk][i] = row < p.G ? bf16x2_to_f16x2(__ldg(q32 + ((hrow0 + row) * D + col) / 2)) : 0u;
      }
    }
  }

  // the accumulator is kept in units of `unit` (a value scale): O = acc * unit
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.0f, 0.0f}, unit = 1.0f;
  float acc[NT][4];
  #pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

  int st = 0;
  int base = c0 + warp * 16;
  if (base < c1) prefetch(base, 0);
  cp_async_commit();
  for (; base < c1; base += kAttnWarps * 16, st ^= 1) {
    const int next = base + kAttnWarps * 16;
    if (next < c1) prefetch(next, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();     // this tile's copies have landed (the next tile's may not)
    __syncwarp();
    // decode this lane's codes to f16
    {
      const int kk = lane >> 1, half = lane & 1;
      const uint8_t *ck = wcodes + st * SM::CODE_STAGE + kk * D + half * CB;
      #pragma unroll
      for (int i = 0; i < CB / 16; ++i) {
        decode16(*reinterpret_cast<const uint4 *>(ck + 16 * i), sK + kk * PITCH + half * CB + i * 16);
        decode16(*reinterpret_cast<const uint4 *>(ck + 16 * D + 16 * i), sV + kk * PITCH + half * CB + i * 16);
      }
    }
    const float *ksc = wscl + (st * 2 + 0) * 16;
    const float *vsc = wscl + (st * 2 + 1) * 16;
    // the tile's readable positions and its largest value scale
    uint32_t vbits = 0;
    float vmax = 0.0f;
    {
      const int pos = base + (lane & 15);
      const bool valid = slot_of(pos) >= 0;
      vbits = __ballot_sync(0xffffffffu, valid && lane < 16);
      vmax = valid ? vsc[lane & 15] : 0.0f;
      #pragma unroll
      for (int o = 8; o >= 1; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    }
    __syncwarp();

    // S = Q K^T: two 8-position column tiles
    float s[2][4];
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
      #pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        uint32_t b0, b1;
        const int l8 = lane & 7, m = (lane >> 3) & 1;
        ldsm_x2(b0, b1, sK + (j * 8 + l8) * PITCH + kk * 16 + m * 8);
        mma_f16(s[j], qa[kk], b0, b1);
      }
    }
    // key scales, masking, online softmax (rows r0 and r0 + 8)
    float mx[2] = {-INFINITY, -INFINITY};
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kp = j * 8 + cq + e;
        const bool valid = (vbits >> kp) & 1u;
        const float k2 = ksc[kp] * p.scale_log2;
        s[j][e] = valid ? s[j][e] * k2 : -INFINITY;
        s[j][2 + e] = valid ? s[j][2 + e] * k2 : -INFINITY;
        mx[0] = fmaxf(mx[0], s[j][e]);
        mx[1] = fmaxf(mx[1], s[j][2 + e]);
      }
    }
    const float inv_vmax = vmax > 0.0f ? 1.0f / vmax : 0.0f;
    float alpha[2], psum[2] = {0.0f, 0.0f};
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_r[r], mx[r]);
      // a tile with no readable position leaves the state as it is
      alpha[r] = m_new == -INFINITY ? 1.0f : exp2f(m_r[r] - m_new);
      m_r[r] = m_new;
    }
    uint32_t pa[4];
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      float pv[4];
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float vr = vsc[j * 8 + cq + e] * inv_vmax;   // this position's value scale / the tile's largest
        const float p0 = m_r[0] == -INFINITY ? 0.0f : exp2f(s[j][e] - m_r[0]);
        const float p1 = m_r[1] == -INFINITY ? 0.0f : exp2f(s[j][2 + e] - m_r[1]);
        psum[0] += p0;
        psum[1] += p1;
        pv[e] = p0 * vr;
        pv[2 + e] = p1 * vr;
      }
      pa[2 * j] = h2_bits(__floats2half2_rn(pv[0], pv[1]));       // row r0, positions j*8 + cq, +1
      pa[2 * j + 1] = h2_bits(__floats2half2_rn(pv[2], pv[3]));   // row r0 + 8
    }
    // move the accumulator to this tile's units (vmax), with the softmax factor
    const float to_tile = vmax > 0.0f ? unit * inv_vmax : 1.0f;
    if (vmax > 0.0f) unit = vmax;
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 1);
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 2);
      l_r[r] = l_r[r] * alpha[r] + psum[r];
      alpha[r] *= to_tile;
    }
    #pragma unroll
    for (int n = 0; n < NT; ++n) {
      acc[n][0] *= alpha[0];
      acc[n][1] *= alpha[0];
      acc[n][2] *= alpha[1];
      acc[n][3] *= alpha[1];
    }
    // O += P V (A = P: rows r0 / r0 + 8, positions cq.. and cq + 8..)
    const uint32_t a[4] = {pa[0], pa[1], pa[2], pa[3]};
    #pragma unroll
    for (int n = 0; n < NT; ++n) {
      uint32_t b0, b1;
      const int l8 = lane & 7, m = (lane >> 3) & 1;
      ldsm_x2_trans(b0, b1, sV + (m * 8 + l8) * PITCH + n * 8);
      mma_f16(acc[n], a, b0, b1);
    }
    __syncwarp();  // the next tile overwrites this warp's tiles
  }
  cp_async_wait<0>();

  // combine the four warps' states (each accumulator times its unit)
  if ((lane & 3) == 0) {
    s_ml[warp][r0][0] = m_r[0];
    s_ml[warp][r0][1] = l_r[0];
    s_ml[warp][r0 + 8][0] = m_r[1];
    s_ml[warp][r0 + 8][1] = l_r[1];
  }
  if (lane == 0) s_unit[warp] = unit;
  __syncthreads();  // every warp has finished with its tiles: the buffer is free
  float *s_acc = reinterpret_cast<float *>(s_tiles);   // [warp][16][D]
  #pragma unroll
  for (int n = 0; n < NT; ++n) {
    float *row0 = s_acc + ((size_t)warp * 16 + r0) * D + n * 8 + cq;
    float *row1 = s_acc + ((size_t)warp * 16 + r0 + 8) * D + n * 8 + cq;
    row0[0] = acc[n][0] * unit;
    row0[1] = acc[n][1] * unit;
    row1[0] = acc[n][2] * unit;
    row1[1] = acc[n][3] * unit;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < p.G * D; i += kAttnThreads) {
    const int h = i / D, d = i - h * D;
    float m = -INFINITY;
    #pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) m = fmaxf(m, s_ml[w][h][0]);
    float l = 0.0f, o = 0.0f;
    if (m != -INFINITY) {
      #pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float f = exp2f(s_ml[w][h][0] - m);   // 0 for a warp that saw no position
        l += s_ml[w][h][1] * f;
        o += s_acc[((size_t)w * 16 + h) * D + d] * f;
      }
    }
    const int64_t idx = (((int64_t)b * p.Hq + (int64_t)g * p.G + h) * p.splits + split);
    p.part_acc[idx * D + d] = o;
    if (d == 0) {
      p.part_ml[idx * 2] = m;
      p.part_ml[idx * 2 + 1] = l;
    }
  }
}

// out[b, h, :] = sum_s acc_s * 2^(m_s - m) / sum_s l_s * 2^(m_s - m), bf16.
template <int D>
__global__ void __launch_bounds__(D) decode_attn_combine_kernel(const float *__restrict__ part_ml,
                                                                const float *__restrict__ part_acc, int splits,
                                                                __nv_bfloat16 *__restrict__ out) {
  griddep_wait();
  const int64_t bh = blockIdx.x;
  const int d = threadIdx.x;
  float m = -INFINITY;
  for (int s = 0; s < splits; ++s) m = fmaxf(m, part_ml[(bh * splits + s) * 2]);
  float l = 0.0f, o = 0.0f;
  if (m != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float f = exp2f(part_ml[(bh * splits + s) * 2] - m);
      l += part_ml[(bh * splits + s) * 2 + 1] * f;
      o += part_acc[(bh * splits + s) * D + d] * f;
    }
  }
  out[bh * D + d] = __float2bfloat16_rn(l > 0.0f ? o / l : 0.0f);
}

constexpr int kAttnChunk = 512;

template <int D>
cudaError_t launch_attn(const AttnParams &p, int B, __nv_bfloat16 *out, cudaStream_t st) {
  const size_t smem = AttnSmem<D, kAttnChunk>::BYTES;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    cudaError_t a = cudaFuncSetAttribute(decode_attn_kernel<D, kAttnChunk>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (a != cudaSuccess) return a;
    attr_set[dev] = true;
  }
  decode_attn_kernel<D, kAttnChunk><<<dim3(p.splits, p.Hkv, B), kAttnThreads, smem, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B * p.Hq);
  cfg.blockDim = dim3(D);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_attn_combine_kernel<D>, (const float *)p.part_ml,
                            (const float *)p.part_acc, p.splits, out);
}

}  // namespace

int attn_splits(int max_context) { return max_context <= 0 ? 1 : (max_context + kAttnChunk - 1) / kAttnChunk; }

size_t attn_workspace_bytes(int B, int Hq, int D, int max_context) {
  const size_t n = (size_t)B * Hq * attn_splits(max_context);
  return n * 2 * sizeof(float) + n * D * sizeof(float);
}

cudaError_t launch_decode_attention(const void *q, const uint8_t *kc, const uint8_t *vc, const float *ks,
                                    const float *vs, const int32_t *block_tables, const int32_t *context_lens,
                                    int B, int Hq, int Hkv, int D, int block_size, int max_blocks,
                                    int64_t num_slots, int max_context, float softmax_scale, void *out, void *ws,
                                    cudaStream_t st) {
  AttnParams p = {};
  p.num_slots = num_slots;
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.kc = kc;
  p.vc = vc;
  p.ks = ks;
  p.vs = vs;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.block_size = block_size;
  p.max_blocks = max_blocks;
  p.splits = attn_splits(max_context);
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  const size_t n = (size_t)B * Hq * p.splits;
  p.part_ml = static_cast<float *>(ws);
  p.part_acc = static_cast<float *>(ws) + n * 2;
  __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
  if (D == 64) return launch_attn<64>(p, B, o, st);
  if (D == 128) return launch_attn<128>(p, B, o, st);
  return cudaErrorInvalidValue;
}

}  // namespace ptpc
