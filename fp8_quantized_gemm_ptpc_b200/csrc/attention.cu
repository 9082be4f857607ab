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
// from shared memory straight into the registers of FlashAttention-style
// tensor-core MMAs (mma.sync m16n8k16, f16 inputs, fp32 accumulation; the
// GQA group's query heads are the 16 rows), converted exactly to f16 on the
// way (cvt e4m3x2 -> f16x2: every E4M3 value is an f16 value).  To make that
// possible the contraction over d in S = Q K^T runs in a permuted order (the
// same for Q and K) in which each lane's codes of a position are contiguous,
// and O's columns are ordered so that each lane's V codes of a position are
// contiguous too; the two positions a V register pairs are joined by one byte
// permute.  Online softmax in base 2; the key scales multiply the scores; the
// value scales enter P relative to the largest value scale seen so far (so P
// stays in [0, 1] in f16), and the accumulator is kept in units of it.  The
// warps' states are combined in shared memory and every CTA writes (max, sum,
// accumulator) for its chunk; a second kernel combines the chunks and rounds
// to bf16.
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

// D (16x8 fp32) += A (16x16 f16, row) * B (16x8 f16, col).
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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
constexpr int kAttnStages = 3;     // code stages a warp keeps in flight (two tiles ahead)

// Shared memory of one CTA: every warp's ring of code stages (K and V codes of
// 16 positions, their scales and the tile's validity mask), which at the end
// doubles as the warps' accumulators, and the chunk's block-table entries.
// A position's D code bytes are stored as D/16 16-byte chunks, chunk i at
// chunk index i ^ (position mod D/16), so that the fragment loads below hit
// distinct shared-memory banks.
template <int D, int CHUNK>
struct AttnSmem {
  static constexpr int CODES_TILE = 2 * 16 * D;                       // K then V codes
  static constexpr int STAGE = CODES_TILE + 2 * 16 * 4 + 16;          // + k, v scales + validity mask
  static constexpr int RING = kAttnStages * STAGE;
  static constexpr int CODES = kAttnWarps * RING;
  static constexpr int BLOCKS = (CHUNK / kMinBlockSize + 2) * 4;
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

template <int D, int CHUNK>
__global__ void __launch_bounds__(kAttnThreads, 3) decode_attn_kernel(const AttnParams p) {
  using SM = AttnSmem<D, CHUNK>;
  constexpr int KS = D / 16;        // 16-deep K steps of S = Q K^T
  constexpr int NT = D / 8;         // 8-wide column tiles of O
  constexpr int KB = D / 4;         // K code bytes a lane holds per position (its share of D)
  constexpr int VB = D / 8;         // V code bytes a lane holds per position
  extern __shared__ __align__(16) uint8_t dsmem[];
  int *s_blk = reinterpret_cast<int *>(dsmem + SM::CODES);
  __shared__ float s_ml[kAttnWarps][16][2];

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
      const int blk = s_blk[pos / p.block_size - bi0];
      slot = (int64_t)blk * p.block_size + pos % p.block_size;
      if (blk < 0 || slot >= p.num_slots) slot = -1;
    }
    const bool valid = slot >= 0;
    const int64_t row = valid ? slot * p.Hkv + g : 0;
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

  // Query fragments (A operand of S = Q K^T; rows = the group's heads, padded
  // to 16).  The contraction over d is taken in a permuted order: in K step
  // s, lane column c (lane & 3) holds d = c*KB + 4s + {0, 1} (logical k =
  // 2c, 2c+1) and c*KB + 4s + {2, 3} (logical 2c+8, 2c+9), so that a lane's K
  // codes for a position are the KB contiguous bytes [c*KB, (c+1)*KB).
  const int r0 = lane >> 2, cq = lane & 3;
  uint32_t qa[KS][4];
  {
    const uint32_t *q32 = reinterpret_cast<const uint32_t *>(p.q);
    const int64_t hrow0 = (int64_t)b * p.Hq + (int64_t)g * p.G;
    #pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = r0 + ((i & 1) ? 8 : 0);
        const int col = cq * KB + 4 * kk + ((i & 2) ? 2 : 0);
        qa[kk][i] = row < p.G ? bf16x2_to_f16x2(__ldg(q32 + ((hrow0 + row) * D + col) / 2)) : 0u;
      }
    }
  }

  // The accumulator is kept in units of `unit`, the largest value scale seen
  // so far (O = acc * unit); column tile n, columns 2cq, 2cq+1 hold
  // d = VB*(2cq) + n and VB*(2cq+1) + n (the V operand's d order: lane row r0
  // holds d = VB*r0 + n, so its V codes for a position are the VB contiguous
  // bytes [VB*r0, VB*(r0+1))).
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.0f, 0.0f}, unit = 0.0f;
  float acc[NT][4];
  #pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;

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

    // S = Q K^T: column tile j holds positions 8j .. 8j+7 (B operand: lane
    // row r0 = position 8j + r0, its KB code bytes)
    float s[2][4];
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int pos = 8 * j + r0;
      uint32_t kw[KB / 4];
      #pragma unroll
      for (int i = 0; i < KB / 16; ++i) {
        const uint4 v = *reinterpret_cast<const uint4 *>(sk + code_off<D>(pos, cq * (KB / 16) + i));
        kw[4 * i] = v.x;
        kw[4 * i + 1] = v.y;
        kw[4 * i + 2] = v.z;
        kw[4 * i + 3] = v.w;
      }
      s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.0f;
      #pragma unroll
      for (int kk = 0; kk < KS; ++kk)
        mma_f16(s[j], qa[kk], e4m3x2_to_f16x2(lo16(kw[kk])), e4m3x2_to_f16x2(hi16(kw[kk])));
    }

    // this lane's positions: 2cq, 2cq+1 (column tile 0) and 2cq+8, 2cq+9 (tile 1)
    const float2 ks01 = *reinterpret_cast<const float2 *>(ksc + 2 * cq);
    const float2 ks89 = *reinterpret_cast<const float2 *>(ksc + 2 * cq + 8);
    const float2 vs01 = *reinterpret_cast<const float2 *>(vsc + 2 * cq);
    const float2 vs89 = *reinterpret_cast<const float2 *>(vsc + 2 * cq + 8);
    const float kscl[2][2] = {{ks01.x, ks01.y}, {ks89.x, ks89.y}};
    const float vscl[2][2] = {{vs01.x, vs01.y}, {vs89.x, vs89.y}};
    bool ok[2][2];
    float vmax = 0.0f;
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        ok[j][e] = (vmask >> (2 * (8 * j + 2 * cq + e))) & 1u;
        if (ok[j][e]) vmax = fmaxf(vmax, vscl[j][e]);
      }
    }
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 1));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, 2));

    // key scales, masking, online softmax (rows r0 and r0 + 8)
    float mx[2] = {-INFINITY, -INFINITY};
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float k2 = kscl[j][e] * p.scale_log2;
        s[j][e] = ok[j][e] ? s[j][e] * k2 : -INFINITY;
        s[j][2 + e] = ok[j][e] ? s[j][2 + e] * k2 : -INFINITY;
        mx[0] = fmaxf(mx[0], s[j][e]);
        mx[1] = fmaxf(mx[1], s[j][2 + e]);
      }
    }
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
    // the unit grows to this tile's largest value scale where that is larger
    const float new_unit = fmaxf(unit, vmax);
    const float to_unit = new_unit > unit && unit > 0.0f ? __fdividef(unit, new_unit) : 1.0f;
    unit = new_unit;
    const float inv_unit = unit > 0.0f ? __fdividef(1.0f, unit) : 0.0f;
    uint32_t pa[4];
    #pragma unroll
    for (int j = 0; j < 2; ++j) {
      float pv[4];
      #pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float vr = vscl[j][e] * inv_unit;   // this position's value scale / the unit
        const float p0 = m_r[0] == -INFINITY ? 0.0f : exp2f(s[j][e] - m_r[0]);
        const float p1 = m_r[1] == -INFINITY ? 0.0f : exp2f(s[j][2 + e] - m_r[1]);
        psum[0] += p0;
        psum[1] += p1;
        pv[e] = p0 * vr;
        pv[2 + e] = p1 * vr;
      }
      pa[2 * j] = h2_bits(__floats2half2_rn(pv[0], pv[1]));       // row r0, positions 8j + 2cq, +1
      pa[2 * j + 1] = h2_bits(__floats2half2_rn(pv[2], pv[3]));   // row r0 + 8
    }
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 1);
      psum[r] += __shfl_xor_sync(0xffffffffu, psum[r], 2);
      l_r[r] = l_r[r] * alpha[r] + psum[r];
      alpha[r] *= to_unit;
    }
    // rescale the accumulator only where a factor differs from one
    if (__any_sync(0xffffffffu, alpha[0] != 1.0f || alpha[1] != 1.0f)) {
      #pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] *= alpha[0];
        acc[n][1] *= alpha[0];
        acc[n][2] *= alpha[1];
        acc[n][3] *= alpha[1];
      }
    }

    // O += P V.  A = P (rows r0 / r0 + 8; k = positions 2cq, 2cq+1 and
    // 2cq+8, 2cq+9); B = V (k = those positions, n = d of column tile n):
    // lane row r0 holds d = VB*r0 + n, so the two codes of a B register (two
    // positions, one d) are byte n of two positions' VB-byte runs, paired
    // with a byte permute before the conversion.
    const uint32_t a[4] = {pa[0], pa[1], pa[2], pa[3]};
    uint32_t vw[4][VB / 4];
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int pos = 2 * cq + (q & 1) + ((q & 2) ? 8 : 0);
      if constexpr (VB == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(sv + code_off<D>(pos, r0));
        vw[q][0] = v.x;
        vw[q][1] = v.y;
        vw[q][2] = v.z;
        vw[q][3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2 *>(sv + code_off<D>(pos, r0 >> 1) + 8 * (r0 & 1));
        vw[q][0] = v.x;
        vw[q][1] = v.y;
      }
    }
    #pragma unroll
    for (int n = 0; n < NT; n += 2) {
      const uint32_t sel = (n & 2) ? 0x7362u : 0x5140u;
      const uint32_t x01 = __byte_perm(vw[0][n >> 2], vw[1][n >> 2], sel);   // positions 2cq, 2cq+1
      const uint32_t x89 = __byte_perm(vw[2][n >> 2], vw[3][n >> 2], sel);   // positions 2cq+8, 2cq+9
      mma_f16(acc[n], a, e4m3x2_to_f16x2(lo16(x01)), e4m3x2_to_f16x2(lo16(x89)));
      mma_f16(acc[n + 1], a, e4m3x2_to_f16x2(hi16(x01)), e4m3x2_to_f16x2(hi16(x89)));
    }
    __syncwarp();  // this stage is refilled two tiles later
    if (++st == kAttnStages) st = 0;
  }
  cp_async_wait<0>();

  // combine the four warps' states (each accumulator times its unit)
  if (cq == 0) {
    s_ml[warp][r0][0] = m_r[0];
    s_ml[warp][r0][1] = l_r[0];
    s_ml[warp][r0 + 8][0] = m_r[1];
    s_ml[warp][r0 + 8][1] = l_r[1];
  }
  __syncthreads();  // every warp has finished with its ring: the buffer is free
  float *s_acc = reinterpret_cast<float *>(dsmem);   // [warp][16][D]
  #pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int d0 = VB * (2 * cq) + n, d1 = VB * (2 * cq + 1) + n;
    float *row0 = s_acc + ((size_t)warp * 16 + r0) * D;
    float *row1 = s_acc + ((size_t)warp * 16 + r0 + 8) * D;
    row0[d0] = acc[n][0] * unit;
    row0[d1] = acc[n][1] * unit;
    row1[d0] = acc[n][2] * unit;
    row1[d1] = acc[n][3] * unit;
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
