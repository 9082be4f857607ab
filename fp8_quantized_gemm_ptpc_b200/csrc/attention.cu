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
// Decode is bound by the bytes of the cache it streams (one byte per code),
// so the kernel spends as few instructions per code byte as it can.  A CTA
// takes one (sequence, KV head) and a chunk of 512 context positions, whose
// block-table entries it first reads into shared memory; its four warps take
// 16-position tiles in turn.  A warp gathers a tile's K and V codes and scales
// with asynchronous copies (cp.async, 16 bytes per copy, zero-filled for
// positions that are not read) into a ring of three shared-memory stages, so
// two tiles' bytes are in flight while it computes on a third.  The codes go
// from shared memory straight into the registers of tensor-core MMAs
// (mma.sync m16n8k16, f16 inputs, fp32 accumulation), converted exactly to
// f16 on the way (cvt e4m3x2 -> f16x2: every E4M3 value is an f16 value).
// Both products are taken transposed, S^T = K Q^T and O^T += V^T P^T, so the
// GQA group's 8 query heads are the MMAs' N = 8 operand and no tensor work is
// spent on padding rows; P moves between them by a register transpose.  The
// contraction over d runs in a permuted order (the same for Q and K) in
// which each lane's K codes of a position are contiguous, and the rows of O^T
// are ordered so that each lane's V codes of a position are contiguous too.
// Online softmax in base 2; the key scales multiply the scores; the value
// scales enter P relative to the largest value scale seen so far (so P stays
// in [0, 1] in f16), and the accumulator is kept in units of it.  The warps'
// states are combined in shared memory and every CTA writes (max, sum,
// accumulator) for its chunk; a second kernel combines the chunks and rounds
// to bf16.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <string>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "attention_tc.h"
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
  uint64_t bs_magic;           // floor(2^64 / block_size) + 1: pos / block_size = umul64hi(pos, bs_magic)
  int64_t num_slots;           // cache slots (num_blocks * block_size): larger slots are skipped
  float scale_log2;            // softmax_scale * log2(e)
  float *part_ml;              // [B, Hq, splits, 2]: running max (base-2 units), sum
  float *part_acc;             // [B, Hq, splits, D]
};

__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }

// Two E4M3 codes (low byte first) -> two f16 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two_codes, __NV_E4M3);
  return (uint32_t)r.x | ((uint32_t)r.y << 16);
}

// D (16x8 fp32) += A (16x16 f16, row) * B (16x8 f16, col).
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D (16x8 fp32) += A (16x32 e4m3, row) * B (32x8 e4m3, col); four codes a register.
__device__ __forceinline__ void mma_e4m3(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats -> two E4M3 codes (low byte first), round to nearest even, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t two_codes) {
  const uint32_t h = e4m3x2_to_f16x2(two_codes);
  return __half22float2(*reinterpret_cast<const __half2 *>(&h));
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

constexpr int kAttnStages = 3;     // code stages a warp keeps in flight (two tiles ahead)

// Shared memory of one CTA: every warp's ring of code stages (K and V codes of
// 16 positions, their scales and the tile's validity mask), which at the end
// doubles as the warps' accumulators, and the chunk's block-table entries
// (blocks hold at least 8 positions).
// A position's D code bytes are stored as D/16 16-byte chunks, chunk i at
// chunk index i ^ (position mod D/16), so that the fragment loads below hit
// distinct shared-memory banks.
template <int D, int CHUNK>
struct AttnSmem {
  static constexpr int CODES_TILE = 2 * 16 * D;                       // K then V codes
  static constexpr int STAGE = CODES_TILE + 2 * 16 * 4 + 16;          // + k, v scales + validity mask
  static constexpr int RING = kAttnStages * STAGE;
  static constexpr int CODES = kAttnWarps * RING;
  static constexpr int BLOCKS = (CHUNK / 8 + 2) * 4;
  static constexpr size_t BYTES = (size_t)CODES + BLOCKS;
  static_assert(kAttnWarps * 16 * D * 4 <= CODES, "combine buffer");
  static_assert(STAGE % 16 == 0, "stage alignment");
};

// Byte offset of 16-byte chunk i of tile-local position pos in a code tile.
template <int D>
__device__ __forceinline__ int code_off(int pos, int i) {
  return pos * D + ((i ^ (pos & (D / 16 - 1))) << 4);
}

__device__ __forceinline__ uint32_t lo16(uint32_t w) { return w & 0xFFFFu; }
__device__ __forceinline__ uint32_t hi16(uint32_t w) { return w >> 16; }

// Transpose of an 8x8 b16 matrix held as the warp's m8n8 fragment (lane i:
// row i/4, columns 2(i%4), 2(i%4)+1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// The warp computes, per 16-position tile, S^T = K Q^T (M = 16 positions, N =
// 8 query heads a head tile, K = d) and O^T += V^T P^T (M = 16 values of d,
// N = 8 heads, K = 16 positions): with the GQA group's 8 heads as the N = 8
// operand neither product carries padding rows.  S^T is an E4M3 x E4M3 MMA
// (m16n8k32) that takes the K codes as they are, with no conversion: each
// head's q is scaled by a power of two sigma (the largest with max |q| sigma
// <= 448) and written as two E4M3 terms, q sigma = hi + lo / 16 (hi rounded
// to nearest, lo the rounded remainder times 16); a bf16 q has 8 significant
// bits and each term 4, so the pair holds it exactly wherever |q sigma| is at
// least E4M3's smallest normal 2^-6 (below it, within 2^-14), and S^T = (K hi + (K lo) / 16) / sigma with each product exact and
// fp32 accumulation.  O^T stays an f16 MMA (P needs more than 4 bits).  Lane (g, c) = (lane / 4,
// lane % 4).  In S^T it holds positions g and g + 8 for heads 2c, 2c+1, the
// same heads whose columns it holds in O^T, so the softmax state and the
// accumulator rescale stay in the lane; P goes from the S^T layout to the B
// operand of O^T by one register transpose (movmatrix) per 8 x 8 block.
// Orders that make every lane's code loads contiguous:
//  * contraction over d in S^T: 32-deep K step s, lane column c holds d =
//    c*KB + 8s + {0..3} (k = 4c .. 4c+3) and c*KB + 8s + {4..7} (k = 16+4c ..
//    16+4c+3): a lane's K codes of a position are the KB bytes [c*KB,
//    (c+1)*KB), four codes a register;
//  * rows of O^T: row tile t, row g holds d = VB*g + 2t, row g + 8 holds
//    d = VB*g + 2t + 1: a lane's V codes of a position are the VB bytes
//    [VB*g, VB*(g+1)), and the two positions a register pairs are joined by
//    one byte permute.
// NH: head tiles of 8 (2 for groups of 9 to 16 heads).
template <int D, int CHUNK, int NH>
__global__ void __launch_bounds__(kAttnThreads, NH == 1 ? 4 : 2) decode_attn_kernel(const AttnParams p) {
  using SM = AttnSmem<D, CHUNK>;
  constexpr int KS = D / 32;        // 32-deep K steps of S^T
  constexpr int MT = D / 16;        // 16-row tiles of O^T
  constexpr int KB = D / 4;         // K code bytes a lane holds per position
  constexpr int VB = D / 8;         // V code bytes a lane holds per position
  extern __shared__ __align__(16) uint8_t dsmem[];
  int *s_blk = reinterpret_cast<int *>(dsmem + SM::CODES);
  __shared__ float s_ml[kAttnWarps][16][2];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int L = __ldg(p.context_lens + b);
  const int c0 = split * CHUNK;
  const int c1 = min(c0 + CHUNK, L);

  // the chunk's block-table entries (-1 where there is none)
  const int bi0 = (int)__umul64hi((uint64_t)c0, p.bs_magic);
  const int nbi = c1 > c0 ? (int)__umul64hi((uint64_t)(c1 - 1), p.bs_magic) - bi0 + 1 : 0;
  for (int i = threadIdx.x; i < nbi; i += kAttnThreads) {
    const int bi = bi0 + i;
    s_blk[i] = bi < p.max_blocks ? __ldg(p.block_tables + (int64_t)b * p.max_blocks + bi) : -1;
  }
  __syncthreads();

  uint8_t *ring = dsmem + warp * SM::RING;

  // Copies of the tile at `base` into stage `st`: lane pair (2 kk, 2 kk + 1)
  // takes position kk, each lane half of its K and V codes; even lanes the
  // scales; the tile's validity mask by lane 0.  Positions that are not read
  // (past the context, no block-table entry, block outside the cache) are
  // zero-filled and masked.
  auto prefetch = [&](int base, int st) {
    const int kk = lane >> 1, half = lane & 1;
    const int pos = base + kk;
    int64_t slot = -1;
    if (pos < c1) {
      const int bi = (int)__umul64hi((uint64_t)pos, p.bs_magic);   // pos / block_size, exactly
      const int blk = s_blk[bi - bi0];
      slot = (int64_t)blk * p.block_size + (pos - bi * p.block_size);
      if (blk < 0 || slot >= p.num_slots) slot = -1;
    }
    const bool valid = slot >= 0;
    const int64_t row = valid ? slot * p.Hkv + kvh : 0;
    uint8_t *sk = ring + st * SM::STAGE;
    uint8_t *sv = sk + 16 * D;
    const uint8_t *gk = p.kc + row * D;
    const uint8_t *gv = p.vc + row * D;
    #pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int ci = half * (D / 32) + i;
      cp_async16(sk + code_off<D>(kk, ci), gk + 16 * ci, valid);
      cp_async16(sv + code_off<D>(kk, ci), gv + 16 * ci, valid);
    }
    float *sc = reinterpret_cast<float *>(sk + SM::CODES_TILE);
    if (half == 0) {
      cp_async4(sc + kk, p.ks + row, valid);
      cp_async4(sc + 16 + kk, p.vs + row, valid);
    }
    const uint32_t m = __ballot_sync(0xffffffffu, valid);   // bit 2 kk (and 2 kk + 1): position kk
    if (lane == 0) *reinterpret_cast<uint32_t *>(sc + 32) = m;
  };

  // Q^T fragments (B operand of S^T) as two E4M3 terms: head tile j, head
  // 8j + g, K step s, registers b0 (d = c*KB + 8s + 0..3) and b1 (+ 4..7).
  // inv_sig[j][e]: 1 / sigma of head 8j + 2c + e (the heads of this lane's
  // S^T columns).
  uint32_t qh[NH][KS][2], ql[NH][KS][2];
  float inv_sig[NH][2];
  {
    const uint2 *q64 = reinterpret_cast<const uint2 *>(p.q);   // 4 bf16 a load
    const int64_t hrow0 = (int64_t)b * p.Hq + (int64_t)kvh * p.G;
    #pragma unroll
    for (int j = 0; j < NH; ++j) {
      const int h = 8 * j + g;
      float qv[KS][8];
      float amax = 0.0f;
      #pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        #pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint2 w = make_uint2(0u, 0u);
          if (h < p.G) w = __ldg(q64 + ((hrow0 + h) * D + c * KB + 8 * ks + 4 * i) / 4);
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.y));
          qv[ks][4 * i] = f0.x;
          qv[ks][4 * i + 1] = f0.y;
          qv[ks][4 * i + 2] = f1.x;
          qv[ks][4 * i + 3] = f1.y;
          amax = fmaxf(amax, fmaxf(fmaxf(fabsf(f0.x), fabsf(f0.y)), fmaxf(fabsf(f1.x), fabsf(f1.y))));
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // sigma: 448 / amax with the mantissa cleared (a power of two, so that
      // amax * sigma <= 448), at most 2^126 (a head of subnormal values); 1
      // for an all-zero head
      const float sig = amax > 0.0f ? fminf(__uint_as_float(__float_as_uint(448.0f / amax) & 0x7F800000u),
                                            __uint_as_float(253u << 23))
                                    : 1.0f;
      const float isig = 1.0f / sig;
      #pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        #pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint32_t hi = 0, lo = 0;
          #pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x0 = qv[ks][4 * i + 2 * e] * sig, x1 = qv[ks][4 * i + 2 * e + 1] * sig;
            const uint32_t h2 = f32x2_to_e4m3x2(x0, x1);
            const float2 d = e4m3x2_to_f32x2(h2);
            const uint32_t l2 = f32x2_to_e4m3x2((x0 - d.x) * 16.0f, (x1 - d.y) * 16.0f);
            hi |= h2 << (16 * e);
            lo |= l2 << (16 * e);
          }
          qh[j][ks][i] = hi;
          ql[j][ks][i] = lo;
        }
      }
      inv_sig[j][0] = __shfl_sync(0xffffffffu, isig, 4 * (2 * c));
      inv_sig[j][1] = __shfl_sync(0xffffffffu, isig, 4 * (2 * c + 1));
    }
  }

  // Softmax state of heads 8j + 2c + e (e = 0, 1), and the accumulator, kept
  // in units of `unit`, the largest value scale seen so far (O = acc * unit).
  float m_h[NH][2], l_h[NH][2];
  float acc[NH][MT][4];
  #pragma unroll
  for (int j = 0; j < NH; ++j) {
    m_h[j][0] = m_h[j][1] = -INFINITY;
    l_h[j][0] = l_h[j][1] = 0.0f;
    #pragma unroll
    for (int t = 0; t < MT; ++t) acc[j][t][0] = acc[j][t][1] = acc[j][t][2] = acc[j][t][3] = 0.0f;
  }
  float unit = 0.0f;

  constexpr int STEP = kAttnWarps * 16;
  const int first = c0 + warp * 16;
  #pragma unroll
  for (int i = 0; i < kAttnStages - 1; ++i) {
    if (first + i * STEP < c1) prefetch(first + i * STEP, i);
    cp_async_commit();
  }
  int st = 0;
  for (int base = first; base < c1; base += STEP) {
    {
      const int ahead = base + (kAttnStages - 1) * STEP;
      int st_ahead = st + kAttnStages - 1;
      if (st_ahead >= kAttnStages) st_ahead -= kAttnStages;
      if (ahead < c1) prefetch(ahead, st_ahead);
      cp_async_commit();
    }
    cp_async_wait<kAttnStages - 1>();   // this tile's copies have landed
    __syncwarp();
    const uint8_t *sk = ring + st * SM::STAGE;
    const uint8_t *sv = sk + 16 * D;
    const float *ksc = reinterpret_cast<const float *>(sk + SM::CODES_TILE);
    const float *vsc = ksc + 16;
    const uint32_t vmask = *reinterpret_cast<const uint32_t *>(ksc + 32);

    // S^T = K Q^T (A = K: rows g, g + 8 = positions)
    uint32_t kw[2][KB / 4];
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int pos = g + 8 * r;
      #pragma unroll
      for (int i = 0; i < KB / 16; ++i) {
        const uint4 v = *reinterpret_cast<const uint4 *>(sk + code_off<D>(pos, c * (KB / 16) + i));
        kw[r][4 * i] = v.x;
        kw[r][4 * i + 1] = v.y;
        kw[r][4 * i + 2] = v.z;
        kw[r][4 * i + 3] = v.w;
      }
    }
    float s[NH][4], sl[NH][4];
    #pragma unroll
    for (int j = 0; j < NH; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = sl[j][0] = sl[j][1] = sl[j][2] = sl[j][3] = 0.0f;
    #pragma unroll
    for (int k = 0; k < KS; ++k) {
      const uint32_t a[4] = {kw[0][2 * k], kw[1][2 * k], kw[0][2 * k + 1], kw[1][2 * k + 1]};
      #pragma unroll
      for (int j = 0; j < NH; ++j) {
        mma_e4m3(s[j], a, qh[j][k][0], qh[j][k][1]);
        mma_e4m3(sl[j], a, ql[j][k][0], ql[j][k][1]);
      }
    }
    #pragma unroll
    for (int j = 0; j < NH; ++j) {
      #pragma unroll
      for (int e = 0; e < 4; ++e) s[j][e] = fmaf(sl[j][e], 0.0625f, s[j][e]);
    }

    // this lane's positions g (s[.][0..1]) and g + 8 (s[.][2..3])
    const bool ok0 = (vmask >> (2 * g)) & 1u, ok8 = (vmask >> (2 * (g + 8))) & 1u;
    const float k0 = ksc[g] * p.scale_log2, k8 = ksc[g + 8] * p.scale_log2;
    const float v0 = ok0 ? vsc[g] : 0.0f, v8 = ok8 ? vsc[g + 8] : 0.0f;
    float vmax = fmaxf(v0, v8);
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 4));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 8));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 16));
    // the unit grows to this tile's largest value scale where that is larger
    const float new_unit = fmaxf(unit, vmax);
    const float to_unit = new_unit > unit && unit > 0.0f ? __fdividef(unit, new_unit) : 1.0f;
    unit = new_unit;
    const float inv_unit = unit > 0.0f ? __fdividef(1.0f, unit) : 0.0f;
    const float vr0 = v0 * inv_unit, vr8 = v8 * inv_unit;

    uint32_t pb[NH][2];
    bool rescale = false;
    float alpha[NH][2];
    #pragma unroll
    for (int j = 0; j < NH; ++j) {
      // key scales and masking
      // the key scale and the query's 1 / sigma multiplied first: each may be
      // far from 1 (a huge query has a tiny 1 / sigma), their product is not
      const float k0h0 = k0 * inv_sig[j][0], k0h1 = k0 * inv_sig[j][1];
      const float k8h0 = k8 * inv_sig[j][0], k8h1 = k8 * inv_sig[j][1];
      s[j][0] = ok0 ? s[j][0] * k0h0 : -INFINITY;
      s[j][1] = ok0 ? s[j][1] * k0h1 : -INFINITY;
      s[j][2] = ok8 ? s[j][2] * k8h0 : -INFINITY;
      s[j][3] = ok8 ? s[j][3] * k8h1 : -INFINITY;
      float pv[4];
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        // head 8j + 2c + e: its largest score of the tile over the 16 positions
        float mx = fmaxf(s[j][e], s[j][2 + e]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m_h[j][e], mx);
        // a tile with no readable position leaves the state as it is
        alpha[j][e] = m_new == -INFINITY ? 1.0f : exp2f(m_h[j][e] - m_new);
        m_h[j][e] = m_new;
        const float p0 = m_new == -INFINITY ? 0.0f : exp2f(s[j][e] - m_new);
        const float p8 = m_new == -INFINITY ? 0.0f : exp2f(s[j][2 + e] - m_new);
        float ps = p0 + p8;
        ps += __shfl_xor_sync(0xffffffffu, ps, 4);
        ps += __shfl_xor_sync(0xffffffffu, ps, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
        l_h[j][e] = l_h[j][e] * alpha[j][e] + ps;
        alpha[j][e] *= to_unit;
        rescale |= alpha[j][e] != 1.0f;
        pv[e] = p0 * vr0;
        pv[2 + e] = p8 * vr8;
      }
      // P' of positions 0..7 and 8..15 as 8 x 8 blocks (row = position,
      // columns = heads 2c, 2c+1), transposed into the B operand of O^T
      // (k = positions 2c, 2c+1 and 2c+8, 2c+9, n = head g)
      pb[j][0] = movmatrix_trans(h2_bits(__floats2half2_rn(pv[0], pv[1])));
      pb[j][1] = movmatrix_trans(h2_bits(__floats2half2_rn(pv[2], pv[3])));
    }
    // rescale the accumulator only where a factor differs from one
    if (__any_sync(0xffffffffu, rescale)) {
      #pragma unroll
      for (int j = 0; j < NH; ++j) {
        #pragma unroll
        for (int t = 0; t < MT; ++t) {
          acc[j][t][0] *= alpha[j][0];
          acc[j][t][1] *= alpha[j][1];
          acc[j][t][2] *= alpha[j][0];
          acc[j][t][3] *= alpha[j][1];
        }
      }
    }

    // O^T += V^T P'^T (A = V^T: rows = d, k = positions 2c, 2c+1, 2c+8, 2c+9)
    uint32_t vw[4][VB / 4];
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int pos = 2 * c + (q & 1) + ((q & 2) ? 8 : 0);
      if constexpr (VB == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(sv + code_off<D>(pos, g));
        vw[q][0] = v.x;
        vw[q][1] = v.y;
        vw[q][2] = v.z;
        vw[q][3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(sv + code_off<D>(pos, g >> 1) + 8 * (g & 1));
        vw[q][0] = v.x;
        vw[q][1] = v.y;
      }
    }
    #pragma unroll
    for (int t = 0; t < MT; ++t) {
      // bytes 2t (row g) and 2t + 1 (row g + 8) of the lane's run
      const uint32_t sel = (t & 1) ? 0x7362u : 0x5140u;
      const uint32_t x01 = __byte_perm(vw[0][t >> 1], vw[1][t >> 1], sel);   // positions 2c, 2c+1
      const uint32_t x89 = __byte_perm(vw[2][t >> 1], vw[3][t >> 1], sel);   // positions 2c+8, 2c+9
      const uint32_t a[4] = {e4m3x2_to_f16x2(lo16(x01)), e4m3x2_to_f16x2(hi16(x01)),
                             e4m3x2_to_f16x2(lo16(x89)), e4m3x2_to_f16x2(hi16(x89))};
      #pragma unroll
      for (int j = 0; j < NH; ++j) mma_f16(acc[j][t], a, pb[j][0], pb[j][1]);
    }
    __syncwarp();  // this stage is refilled two tiles later
    if (++st == kAttnStages) st = 0;
  }
  cp_async_wait<0>();

  // combine the four warps' states (each accumulator times its unit)
  if (g == 0) {
    #pragma unroll
    for (int j = 0; j < NH; ++j) {
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        s_ml[warp][8 * j + 2 * c + e][0] = m_h[j][e];
        s_ml[warp][8 * j + 2 * c + e][1] = l_h[j][e];
      }
    }
  }
  __syncthreads();  // every warp has finished with its ring: the buffer is free
  float *s_acc = reinterpret_cast<float *>(dsmem);   // [warp][16 heads][D]
  #pragma unroll
  for (int j = 0; j < NH; ++j) {
    #pragma unroll
    for (int t = 0; t < MT; ++t) {
      const int d0 = VB * g + 2 * t, d8 = d0 + 1;
      float *h0 = s_acc + ((size_t)warp * 16 + 8 * j + 2 * c) * D;
      float *h1 = h0 + D;
      h0[d0] = acc[j][t][0] * unit;
      h1[d0] = acc[j][t][1] * unit;
      h0[d8] = acc[j][t][2] * unit;
      h1[d8] = acc[j][t][3] * unit;
    }
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
    const int64_t idx = (((int64_t)b * p.Hq + (int64_t)kvh * p.G + h) * p.splits + split);
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

// Context chunk of a CTA: 512, 1024 or 2048 positions (up to 4096 for the
// tensor-memory kernel).  Larger chunks pay the
// CTA's start (block table, query terms) and end (the warps' combine) over
// more tiles but leave fewer CTAs to fill the GPU; the launch takes the chunk
// with the fewest rounds of resident CTAs times (positions a CTA — at most the
// longest context — + `fixed`, the CTA's start and end counted in positions)
// (ties: the larger chunk).
constexpr int kAttnChunkMin = 512;

template <int D, int CHUNK, int NH>
cudaError_t launch_attn_chunk(const AttnParams &p, int B, cudaStream_t st) {
  const size_t smem = AttnSmem<D, CHUNK>::BYTES;
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t a = cudaFuncSetAttribute(decode_attn_kernel<D, CHUNK, NH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (a != cudaSuccess) return a;
    attr_set[dev].store(true, std::memory_order_release);
  }
  decode_attn_kernel<D, CHUNK, NH><<<dim3(p.splits, p.Hkv, B), kAttnThreads, smem, st>>>(p);
  return cudaGetLastError();
}

// CTAs of the attention kernel that can be resident at once on this device.
template <int D, int NH>
int attn_resident() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 148, per_sm = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaFuncSetAttribute(decode_attn_kernel<D, 2048, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)AttnSmem<D, 2048>::BYTES);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_attn_kernel<D, 2048, NH>, kAttnThreads,
                                                    AttnSmem<D, 2048>::BYTES) != cudaSuccess || per_sm <= 0)
    per_sm = 1;
  cudaGetLastError();
  const int n = std::max(1, sms * per_sm);
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// PTPC_FORCE_ATTN_CHUNK = 512 | 1024 | 2048 | 4096 (tuning and tests only;
// 4096 only for the tensor-memory kernel, the other takes 2048): read at
// the first launch, or again by attn_reload_tuning.
std::atomic<int> g_attn_chunk{-1};

int read_attn_chunk() {
  const char *v = std::getenv("PTPC_FORCE_ATTN_CHUNK");
  if (v == nullptr) return 0;
  const int c = std::atoi(v);
  return c == 512 || c == 1024 || c == 2048 || c == 4096 ? c : 0;
}

int attn_chunk(int pairs, int max_context, int resident, int fixed = 0, int max_chunk = 2048) {
  int forced = g_attn_chunk.load(std::memory_order_relaxed);
  if (forced < 0) {
    forced = read_attn_chunk();
    g_attn_chunk.store(forced, std::memory_order_relaxed);
  }
  if (forced > 0) return std::min(forced, max_chunk);
  int best = kAttnChunkMin;
  long long best_cost = -1;
  for (int chunk = kAttnChunkMin; chunk <= max_chunk; chunk *= 2) {
    const long long ctas = (long long)pairs * ((std::max(max_context, 1) + chunk - 1) / chunk);
    const long long cost = (ctas + resident - 1) / resident * (std::min(chunk, std::max(max_context, 1)) + fixed);
    if (best_cost < 0 || cost <= best_cost) {
      best = chunk;
      best_cost = cost;
    }
  }
  return best;
}

// Decode attention runs the tensor-memory kernel of attention_tc.cu where it
// applies (D = 128, blocks of a multiple of 8 positions) and the warp-level
// kernel above otherwise.
// PTPC_FORCE_ATTN_KERNEL = mma | tc (tuning and tests only) forces one (tc
// only where it applies).  Read at the first launch, or again by
// attn_reload_tuning.
constexpr int kAttnKernelAuto = 0, kAttnKernelMma = 1, kAttnKernelTc = 2;
std::atomic<int> g_attn_kernel{-1};

int read_attn_kernel() {
  const char *v = std::getenv("PTPC_FORCE_ATTN_KERNEL");
  if (v == nullptr) return kAttnKernelAuto;
  const std::string s(v);
  return s == "mma" ? kAttnKernelMma : s == "tc" ? kAttnKernelTc : kAttnKernelAuto;
}

bool attn_use_tc(int D, int G, int block_size) {
  int k = g_attn_kernel.load(std::memory_order_relaxed);
  if (k < 0) {
    k = read_attn_kernel();
    g_attn_kernel.store(k, std::memory_order_relaxed);
  }
  if (!attn_tc_supported(D, G, block_size)) return false;
  return k != kAttnKernelMma;
}

template <int D>
cudaError_t launch_attn_combine(const AttnParams &p, int B, __nv_bfloat16 *out, cudaStream_t st) {
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

template <int D, int NH>
cudaError_t launch_attn(AttnParams p, int B, int max_context, __nv_bfloat16 *out, cudaStream_t st) {
  const int chunk = attn_chunk(B * p.Hkv, max_context, attn_resident<D, NH>());
  p.splits = (std::max(max_context, 1) + chunk - 1) / chunk;
  cudaError_t e = chunk == 2048   ? launch_attn_chunk<D, 2048, NH>(p, B, st)
                  : chunk == 1024 ? launch_attn_chunk<D, 1024, NH>(p, B, st)
                                  : launch_attn_chunk<D, 512, NH>(p, B, st);
  if (e != cudaSuccess) return e;
  return launch_attn_combine<D>(p, B, out, st);
}

cudaError_t launch_attn_tc_and_combine(AttnParams p, int B, int max_context, uint32_t *status, __nv_bfloat16 *out,
                                       cudaStream_t st) {
  // the tensor-memory kernel's start (barriers, tensor memory, the first
  // tiles' load latency) costs about three 128-position tiles
  const int chunk = attn_chunk(B * p.Hkv * ((p.G + 7) / 8), max_context, attn_tc_resident(), 384, 4096);
  p.splits = (std::max(max_context, 1) + chunk - 1) / chunk;
  // one chunk covers every context: the kernel writes the output itself
  const bool single = p.splits == 1;
  cudaError_t e = launch_attn_tc(p.q, p.kc, p.vc, p.ks, p.vs, p.block_tables, p.context_lens, B, p.Hq, p.Hkv,
                                 p.block_size, p.max_blocks, p.num_slots, p.bs_magic, chunk, p.splits, p.scale_log2,
                                 p.part_ml, p.part_acc, single ? out : nullptr, status, st);
  if (e != cudaSuccess || single) return e;
  return launch_attn_combine<128>(p, B, out, st);
}

}  // namespace

int attn_kernel_choice(int D, int G, int block_size) { return attn_use_tc(D, G, block_size) ? 2 : 1; }

void attn_reload_tuning() {
  g_attn_chunk.store(read_attn_chunk(), std::memory_order_relaxed);
  g_attn_kernel.store(read_attn_kernel(), std::memory_order_relaxed);
}

// The most chunks a launch can split a context into (the workspace bound).
int attn_splits(int max_context) { return max_context <= 0 ? 1 : (max_context + kAttnChunkMin - 1) / kAttnChunkMin; }

// The device status word (256 bytes reserved), then the partial results.
constexpr size_t kAttnStatusBytes = 256;

size_t attn_workspace_bytes(int B, int Hq, int D, int max_context) {
  const size_t n = (size_t)B * Hq * attn_splits(max_context);
  return kAttnStatusBytes + n * 2 * sizeof(float) + n * D * sizeof(float);
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
  // ceil(2^64 / block_size): pos * bs_magic / 2^64 is pos / block_size plus less than 2^-32 for
  // pos < 2^32, and the fractional part of pos / block_size is at most 1 - 1 / block_size,
  // so the high word is the exact quotient
  p.bs_magic = ~0ull / (uint64_t)block_size + 1;
  p.max_blocks = max_blocks;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  // partial results of up to attn_splits(max_context) chunks a head
  const size_t n = (size_t)B * Hq * attn_splits(max_context);
  uint32_t *status = static_cast<uint32_t *>(ws);
  p.part_ml = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kAttnStatusBytes);
  p.part_acc = p.part_ml + n * 2;
  __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
  if (attn_use_tc(D, p.G, block_size)) return launch_attn_tc_and_combine(p, B, max_context, status, o, st);
  if (D == 64) return p.G > 8 ? launch_attn<64, 2>(p, B, max_context, o, st) : launch_attn<64, 1>(p, B, max_context, o, st);
  if (D == 128) return p.G > 8 ? launch_attn<128, 2>(p, B, max_context, o, st) : launch_attn<128, 1>(p, B, max_context, o, st);
  return cudaErrorInvalidValue;
}

}  // namespace ptpc
