// PTPC-FP8 scaled GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// out[t][o] = bf16_RNE((acc[t][o] * x_scale[t]) * w_scale[o]),
// acc[t][o] = sum_k dec(Xq[t][k]) * dec(Wq_t[o][k]),
// the fused row-wise-scaled FP8 GEMM of "PTPC-FP8: boosting vLLM performance
// on AMD ROCm" (section "The challenge: two-step vs fused"): the two scale
// vectors are applied to the accumulator on chip, between the tensor-memory
// load and the single store of the output, so no T x Co intermediate is ever
// written.  The page's kernel is AMD's (MI300X); these are written for B200.
//
// Two kernels share the structure below.
//   * ptpc_gemm_pair_kernel (prefill): a cluster of two CTAs on two
//     SMs computes 256 x 256 tiles with tcgen05.mma.cta_group::2.
//   * ptpc_gemm_decode_kernel (decode-sized T, at most 256; see make_plan):
//     one CTA per SM, operands swapped — 128 weight rows are the MMA's M
//     operand and the T tokens (padded to a multiple of 16) its N operand.
// In both, warp 0 (one thread) streams 128-byte-wide K slices of Xq and Wq_t
// with TMA into a shared-memory ring (128-byte swizzle, no multicast); warp 1
// (one thread) issues the MMAs (E4M3 x E4M3 -> fp32, K = 32 each) into one of
// two tensor-memory accumulators and commits every stage back to the
// producer; warps 2-5 read the finished accumulator with tcgen05.ld (each
// warp owns one 32-lane quarter), apply the two scales, round to bf16 and
// store, while the MMA warp fills the other accumulator.
//
// Work schedule: whole tiles, round-robin over the CTAs (CTA pairs), except
// that a decode problem with fewer than half as many tiles as SMs splits K:
// the S CTAs of a thread-block cluster (S = 2, 4 or 8) share one tile, each
// streaming 1/S of its K-blocks, so S times as many SMs stream weights.  Each
// CTA leaves its fp32 partial sums in its own shared memory; after a cluster
// barrier every CTA finishes 128/S of the tile's channels by reading the S
// partial sums over distributed shared memory and adding them in rank order
// (a fixed order: the result does not depend on timing), then applies the
// scales and stores.  No partial sum goes through global memory.
//
// Every wait on an mbarrier is bounded (see mbar_wait); a wait that runs out
// sets a bit in the device status word, and the CTA stops issuing work, lets
// its own copies and MMAs drain, frees its tensor memory and exits.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace ptpc {

namespace {

constexpr int BM = 128;      // token rows per CTA tile (tensor-memory lanes)
constexpr size_t kGemmStatusBytes = 256;  // the workspace's device status word (and its padding)
constexpr int BK = 128;      // K bytes per stage (= one 128-byte swizzle row)
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

// Weight formats: 0 E4M3 (PTPC-FP8), 1 E2M1 (FP4), 2 E2M3 and 3 E3M2 (FP6).
// The sub-byte weights sit packed in global memory and are unpacked by TMA
// into the same one-byte-per-element shared-memory layout as E4M3 (16 codes
// per 16-byte chunk), so only the bytes a stage transfers and the MMA's
// operand format change.
__host__ __device__ constexpr int wf_bits(int wf) { return wf == 0 ? 8 : wf == 1 ? 4 : 6; }
__host__ __device__ constexpr uint32_t wf_mma(int wf) {
  return wf == 0 ? kMmaE4M3 : wf == 1 ? kMmaE2M1 : wf == 2 ? kMmaE2M3 : kMmaE3M2;
}

struct GemmParams {
  int T, Co;
  int num_m, num_n, num_kb;   // tile grid (pair kernel: token tile rows; decode: one row of all tokens)
  // pair kernel, operands swapped: the weights are the MMA's M = 256 operand
  // (256 channels a tile) and nt tokens (a multiple of 32, at most 256) its N
  // operand; swap = 0: 256 tokens x BN channels a tile
  int swap, nt;
  int group_m;                // tile rows visited together (L2 reuse of weights)
  int num_tiles;
  int ksplit;                 // decode kernel: CTAs (one cluster) per tile, 1 = whole tiles
  int np;                     // decode kernel: tokens padded to the MMA's N (multiple of 16)
  int stages;                 // decode kernel: shared-memory ring depth
  int tmem_cols;              // decode kernel: tensor-memory columns allocated (two accumulators)
  // pair kernel, split tail: the last tail_tiles tiles of the raster (the
  // under-filled last wave) are split along K over tail_split CTA pairs each
  int full_tiles;             // tiles done whole (num_tiles - tail_tiles)
  int tail_tiles, tail_split;
  float *partials;            // fp32 [tail_tiles][tail_split][256][BN] partial accumulators
  uint32_t *tail_count;       // [2][tail_tiles]: CTAs that stored their partial / finished reducing
  const float *xs;
  const float *ws;
  void *out;
  uint32_t *status;
};

// One piece of work: K-blocks [kb0, kb1) of tile `tile` (row m, column n).
// split >= 0: a K range of a split tail tile (the partial is reduced later).
struct Unit {
  int tile, m, n, kb0, kb1, split;
};

// The same sequence of units for the producer, the MMA issuer and the
// epilogue of one CTA (pair) `id` out of `count`: tiles id, id + count, ...
// whole, or, when the decode kernel splits K (ksplit > 1), the one tile of
// this CTA's cluster and this CTA's share of its K-blocks.
struct Sched {
  int next_tile, step, kb0, kb1;
  int tail_unit;  // pair kernel: index of this pair's unit in the split tail, -1 if none (or done)

  __device__ __forceinline__ void init(const GemmParams &p, int id, int count) {
    tail_unit = -1;
    if (p.ksplit > 1) {
      const int r = id % p.ksplit;  // == %cluster_ctarank for a 1-D cluster
      next_tile = id / p.ksplit;
      step = p.num_tiles;  // one tile per cluster
      kb0 = r * p.num_kb / p.ksplit;
      kb1 = (r + 1) * p.num_kb / p.ksplit;
    } else {
      next_tile = id;
      step = count;
      kb0 = 0;
      kb1 = p.num_kb;
      if (p.tail_tiles > 0 && id < p.tail_tiles * p.tail_split) tail_unit = id;
    }
  }

  __device__ __forceinline__ void raster(const GemmParams &p, Unit &u) {
    // grouped raster: group_m tile rows, all tile columns, rows fastest
    const int per_group = p.group_m * p.num_n;
    const int g = u.tile / per_group;
    const int first_m = g * p.group_m;
    const int gm = min(p.group_m, p.num_m - first_m);
    const int r = u.tile - g * per_group;
    u.m = first_m + r % gm;
    u.n = r / gm;
  }

  __device__ __forceinline__ bool next(const GemmParams &p, Unit &u) {
    if (next_tile < p.full_tiles) {
      u.tile = next_tile;
      next_tile += step;
      u.kb0 = kb0;
      u.kb1 = kb1;
      u.split = -1;
      raster(p, u);
      return true;
    }
    if (tail_unit >= 0) {
      const int j = tail_unit / p.tail_split;
      const int r = tail_unit - j * p.tail_split;
      tail_unit = -1;
      u.tile = p.full_tiles + j;
      u.kb0 = r * p.num_kb / p.tail_split;
      u.kb1 = (r + 1) * p.num_kb / p.tail_split;
      u.split = r;
      raster(p, u);
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Stages one warp's 32 rows x 128 bytes in 128-byte-swizzled shared memory and
// stores them with TMA at (col, row).  `packed` holds this lane's row.  The
// stored lines are marked evict-first in L2: the kernel never reads them, and
// they must not push out the operand tiles that other CTAs still read.
__device__ __forceinline__ void stage_and_store(const CUtensorMap *tmC, uint8_t *cbuf, const uint32_t (&packed)[32],
                                                int col, int row, int lane, uint64_t pol) {
  // the previous TMA store from this buffer must have finished reading it
  if (lane == 0) bulk_wait_read<0>();
  __syncwarp();
  #pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int pos = j ^ (lane & 7);
    *reinterpret_cast<uint4 *>(cbuf + lane * 128 + pos * 16) =
        make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
  }
  fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d_hint(tmC, cbuf, col, row, pol);
    bulk_commit();
  }
}

// Column scales of a 64-column chunk into this warp's scratch `sc`.
__device__ __forceinline__ void load_col_scales(float *sc, const GemmParams &p, int col0, int lane) {
  __syncwarp();
  sc[lane] = (col0 + lane < p.Co) ? __ldg(p.ws + col0 + lane) : 0.0f;
  sc[lane + 32] = (col0 + 32 + lane < p.Co) ? __ldg(p.ws + col0 + 32 + lane) : 0.0f;
  __syncwarp();
}

// (acc * x_scale) * w_scale for 32 accumulators (raw fp32 bits), packed to
// 16 bf16 pairs at packed[off .. off+15].
__device__ __forceinline__ void scale_pack32(const uint32_t (&r)[32], float xsr, const float *sc,
                                             uint32_t (&packed)[32], int off) {
  #pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 wv = *reinterpret_cast<const float4 *>(sc + 4 * j);
    const float v0 = __fmul_rn(__fmul_rn(__uint_as_float(r[4 * j + 0]), xsr), wv.x);
    const float v1 = __fmul_rn(__fmul_rn(__uint_as_float(r[4 * j + 1]), xsr), wv.y);
    const float v2 = __fmul_rn(__fmul_rn(__uint_as_float(r[4 * j + 2]), xsr), wv.z);
    const float v3 = __fmul_rn(__fmul_rn(__uint_as_float(r[4 * j + 3]), xsr), wv.w);
    packed[off + 2 * j] = pack_bf16x2(v0, v1);
    packed[off + 2 * j + 1] = pack_bf16x2(v2, v3);
  }
}

// Fused epilogue of one accumulator held in tensor memory: 32 token rows (one
// lane quarter; lane i = row store_row0 + i) x BN_T columns from global
// column col_base.  After the last tensor-memory read the accumulator buffer
// is released by one arrival on `release_bar` (a shared::cluster address:
// this CTA's barrier or the pair leader's).
template <int BN_T, bool F32OUT>
__device__ __forceinline__ void epilogue_store_tile(const CUtensorMap *tmC, uint32_t tbase, uint8_t *cbuf,
                                                    float *sc, const GemmParams &p, int col_base,
                                                    int store_row0, float xsr, int lane, uint32_t release_bar,
                                                    uint64_t pol) {
  constexpr int EPI_COLS = F32OUT ? 32 : 64;
  #pragma unroll 1
  for (int c0 = 0; c0 < BN_T; c0 += EPI_COLS) {
    uint32_t packed[32];
    if constexpr (F32OUT) {
      tmem_ld_32x32b_x32(tbase + c0, packed);
      tmem_wait_ld();
    } else {
      load_col_scales(sc, p, col_base + c0, lane);
      uint32_t r[32];
      tmem_ld_32x32b_x32(tbase + c0, r);
      tmem_wait_ld();
      scale_pack32(r, xsr, sc, packed, 0);
      tmem_ld_32x32b_x32(tbase + c0 + 32, r);
      tmem_wait_ld();
      scale_pack32(r, xsr, sc + 32, packed, 16);
    }
    if (c0 + EPI_COLS >= BN_T) {
      // the whole accumulator has been read: hand it back to the MMA issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release_bar);
    }
    stage_and_store(tmC, cbuf, packed, col_base + c0, store_row0, lane, pol);
  }
}

// ----------------------------------------------------------------------------
// Decode kernel (T <= kDecodeMaxT), operands swapped: acc^T = Wq_t . Xq^T.
// The 128 weight rows of a channel tile are the MMA's M = 128 operand and the
// T tokens, padded to NP (a multiple of 16, at most 256), are its N operand.
// A stage then carries 16 KB of weights and only NP x 128 bytes of
// activations, instead of a 128-row activation box that is mostly
// out-of-bounds fill, and the ring is as deep as shared memory allows (12
// stages at NP = 16, 4 at NP = 256).  Tensor-memory lane
// = output channel, column = token: each epilogue thread owns one channel, so
// w_scale is one register and every token's 32 channels of a warp are one
// contiguous store.  With ksplit = S > 1 the grid is made of S-CTA clusters,
// one tile each, and the epilogue leaves the partial sums in shared memory
// for the cluster reduction instead of storing.
// ----------------------------------------------------------------------------
constexpr int kDecodeMaxT = 256;       // largest T the decode kernel takes (MMA N <= 256)
constexpr int kDecodeWholeMaxT = 192;  // above this, the pair kernel (unless forced)
constexpr int kDecMaxStages = 16;
constexpr int kDecWBytes = BM * BK;   // weight tile of one stage
constexpr size_t kDecBarBytes = 512;  // barriers and flags after the ring
constexpr size_t kDecSmemMax = 232448;

__host__ __device__ constexpr size_t dec_smem_bytes(int np, int stages) {
  return 1024 + (size_t)stages * (kDecWBytes + (size_t)np * BK) + kDecBarBytes;
}

// Whole tile: scales applied per (token, channel), one bf16 (or fp32) store
// per token; the accumulator is released after its last tensor-memory read.
template <bool F32OUT>
__device__ __forceinline__ void decode_store_tile(const GemmParams &p, uint32_t tbase, int ch, float wsr,
                                                  int lane, uint32_t release_bar) {
  const bool ch_ok = ch < p.Co;
  #pragma unroll 1
  for (int c0 = 0; c0 < p.np; c0 += 16) {
    uint32_t r[16];
    tmem_ld_32x32b_x16(tbase + c0, r);
    tmem_wait_ld();
    if (c0 + 16 >= p.np) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release_bar);
    }
    if (!ch_ok) continue;
    #pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = c0 + j;
      if (t < p.T) {
        const float acc = __uint_as_float(r[j]);
        if constexpr (F32OUT) {
          static_cast<float *>(p.out)[(size_t)t * p.Co + ch] = acc;
        } else {
          const float v = __fmul_rn(__fmul_rn(acc, __ldg(p.xs + t)), wsr);
          static_cast<__nv_bfloat16 *>(p.out)[(size_t)t * p.Co + ch] = __float2bfloat16_rn(v);
        }
      }
    }
  }
}

// K split over a cluster, step 1: this CTA's partial sums of the tile, from
// tensor memory to red[t][c] (fp32, BM floats per token) in its own shared
// memory.  Each warp writes 32 consecutive floats per token (no bank
// conflicts).
__device__ __forceinline__ void decode_dump_tile(const GemmParams &p, uint32_t tbase, float *red, int q, int lane) {
  float *dst = red + q * 32 + lane;
  #pragma unroll 1
  for (int c0 = 0; c0 < p.np; c0 += 16) {
    uint32_t r[16];
    tmem_ld_32x32b_x16(tbase + c0, r);
    tmem_wait_ld();
    #pragma unroll
    for (int j = 0; j < 16; ++j) dst[(c0 + j) * BM] = __uint_as_float(r[j]);
  }
}

// K split over a cluster, step 2 (after a cluster barrier): this CTA (rank)
// finishes channels [rank * 128/S, (rank + 1) * 128/S) of the tile for every
// token.  Each thread takes 4 consecutive channels of one token, loads them
// from all S CTAs' red arrays over distributed shared memory (16 bytes per
// load; U groups, U * S loads in flight), adds the S partial sums in rank
// order, applies the scales and stores.
template <int S, bool F32OUT>
__device__ __forceinline__ void decode_cluster_reduce(const GemmParams &p, const float *red, int tile,
                                                      uint32_t rank) {
  constexpr int CS = BM / S;                // channels this CTA finishes
  constexpr int G = CS / 4;                 // 4-channel groups per token
  constexpr int U = S >= 8 ? 1 : 8 / S;     // groups per thread in flight
  uint32_t base[S];
  #pragma unroll
  for (int s = 0; s < S; ++s) base[s] = mapa_shared(red, (uint32_t)s);
  const int total = p.T * G;
  const int c_first = (int)rank * CS;
  for (int i0 = threadIdx.x; i0 < total; i0 += U * kThreads) {
    float4 v[U][S];
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      const int idx = i0 + u * kThreads;
      if (idx < total) {
        const int t = idx / G;
        const int c = c_first + (idx - t * G) * 4;
        const uint32_t off = (uint32_t)(t * BM + c) * 4u;
        #pragma unroll
        for (int s = 0; s < S; ++s) v[u][s] = ld_shared_cluster_f32x4(base[s] + off);
      }
    }
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      const int idx = i0 + u * kThreads;
      if (idx >= total) continue;
      const int t = idx / G;
      const int c = c_first + (idx - t * G) * 4;
      const int ch = tile * BM + c;
      if (ch >= p.Co) continue;  // Co % 16 == 0: the 4 channels are valid together
      float4 acc = v[u][0];
      #pragma unroll
      for (int s = 1; s < S; ++s) {
        acc.x = __fadd_rn(acc.x, v[u][s].x);
        acc.y = __fadd_rn(acc.y, v[u][s].y);
        acc.z = __fadd_rn(acc.z, v[u][s].z);
        acc.w = __fadd_rn(acc.w, v[u][s].w);
      }
      if constexpr (F32OUT) {
        *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (size_t)t * p.Co + ch) = acc;
      } else {
        const float a = __ldg(p.xs + t);
        const float4 w = __ldg(reinterpret_cast<const float4 *>(p.ws + ch));
        const uint32_t lo = pack_bf16x2(__fmul_rn(__fmul_rn(acc.x, a), w.x), __fmul_rn(__fmul_rn(acc.y, a), w.y));
        const uint32_t hi = pack_bf16x2(__fmul_rn(__fmul_rn(acc.z, a), w.z), __fmul_rn(__fmul_rn(acc.w, a), w.w));
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) + (size_t)t * p.Co + ch) =
            make_uint2(lo, hi);
      }
    }
  }
}

template <bool F32OUT, int WF>
__global__ void __launch_bounds__(kThreads, 1)
    ptpc_gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                            const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int STAGES = p.stages;
  const int X_BYTES = p.np * BK;
  uint8_t *sW = smem;
  uint8_t *sX = sW + STAGES * kDecWBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(sX + STAGES * X_BYTES);
  uint64_t *empty = full + kDecMaxStages;
  uint64_t *tfull = empty + kDecMaxStages;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  const uint32_t acc_cols = (uint32_t)p.tmem_cols / 2;  // column stride of the two accumulators
  // K split: partial sums of the tile, [NP tokens][BM channels] fp32, in the
  // ring (idle once the accumulator is complete; the weight and activation
  // stages are contiguous, and NP * 512 bytes fit in them: checked by the plan)
  float *red = reinterpret_cast<float *>(sW);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      const uint64_t polW = policy_evict_first();  // every weight byte is read once
      const uint64_t polX = policy_evict_last();   // every CTA reads the activations
      // bytes TMA moves per stage: the weights at their packed size
      const uint32_t stage_tx = (uint32_t)(kDecWBytes * wf_bits(WF) / 8 + X_BYTES);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      Sched sc;
      Unit u;
      // The weights never depend on the kernel launched just before this one:
      // the first stages' weight tiles are requested before waiting for it.
      int pre = 0;
      sc.init(p, blockIdx.x, gridDim.x);
      if (sc.next(p, u)) {
        for (; pre < STAGES && u.kb0 + pre < u.kb1; ++pre) {
          mbar_arrive_expect_tx(&full[pre], stage_tx);
          tma_load_2d(sW + pre * kDecWBytes, &tmW, &full[pre], (u.kb0 + pre) * BK, u.n * BM, polW);
        }
      }
      griddep_wait();  // Xq may come from the kernel launched just before
      int issued = 0;
      sc.init(p, blockIdx.x, gridDim.x);
      while (ok && sc.next(p, u)) {
        for (int kb = u.kb0; kb < u.kb1; ++kb, ++issued) {
          if (issued >= pre) {
            if (!mbar_wait(&empty[stage], phase ^ 1)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], stage_tx);
            tma_load_2d(sW + stage * kDecWBytes, &tmW, &full[stage], kb * BK, u.n * BM, polW);
          }
          tma_load_2d(sX + stage * X_BYTES, &tmX, &full[stage], kb * BK, 0, polX);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      griddep_launch_dependents();
      if (!ok) {
        atomicOr(p.status, kStatusTimeoutProducer);
        for (int s = 0; s < STAGES; ++s) mbar_wait(&full[s], s < stage ? phase : phase ^ 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_f8f6f4_f32(BM, p.np, wf_mma(WF), kMmaE4M3);  // A = weights
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      Sched sc;
      sc.init(p, blockIdx.x, gridDim.x);
      Unit u;
      while (ok && sc.next(p, u)) {
        const int buf = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        ++local;
        if (!mbar_wait(&tempty[buf], aphase ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)buf * acc_cols;
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sW + stage * kDecWBytes));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sX + stage * X_BYTES));
          #pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_f8f6f4(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                     (kb > u.kb0 || kk > 0) ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[buf]);
      }
      if (!ok) atomicOr(p.status, kStatusTimeoutMma);
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // tensor-memory lane quarter = channels q*32 .. q*32+31
    int local = 0;
    bool ok = true;
    griddep_wait();  // x_scale may come from the kernel launched just before
    Sched sc;
    sc.init(p, blockIdx.x, gridDim.x);
    Unit u;
    while (sc.next(p, u)) {
      const int buf = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      ++local;
      const int ch = u.n * BM + q * 32 + lane;
      const float wsr = (!F32OUT && ch < p.Co) ? __ldg(p.ws + ch) : 0.0f;
      // tcgen05.ld is warp-collective: the whole warp stops or none of it
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], aphase))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * acc_cols;
      if (p.ksplit == 1)
        decode_store_tile<F32OUT>(p, tbase, ch, wsr, lane, smem_u32(&tempty[buf]));
      else
        decode_dump_tile(p, tbase, red, q, lane);
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeoutEpilogue);
  }

  if (p.ksplit > 1) {
    // Every CTA of the cluster reaches both barriers on every path (a timed
    // out wait above only skips work), so neither can wait forever.
    __syncwarp();    // warps 0 and 1 arrive from a one-lane branch
    cluster_sync();  // all partial sums of the tile are in shared memory
    const int tile = blockIdx.x / p.ksplit;
    const uint32_t rank = cluster_ctarank();
    if (p.ksplit == 2)
      decode_cluster_reduce<2, F32OUT>(p, red, tile, rank);
    else if (p.ksplit == 4)
      decode_cluster_reduce<4, F32OUT>(p, red, tile, rank);
    else
      decode_cluster_reduce<8, F32OUT>(p, red, tile, rank);
    cluster_sync();  // no CTA reads another's shared memory any more
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
  }
}

// ----------------------------------------------------------------------------
// Split tail of the pair kernel.  The tiles of the last, under-filled wave are
// split along K over tail_split CTA pairs each; every CTA of those pairs
// stores its 128 rows x BN fp32 partial accumulator in the workspace, counts
// itself in, waits (bounded) until the tile's 2 * tail_split CTAs have all
// stored theirs, and then finishes 1 / (2 * tail_split) of the tile: the
// partials added in split order (a fixed order: deterministic), the two
// scales applied, bf16 stored.  The last CTA to finish zeroes the tile's
// counters for the next call.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// This lane's row of the partial accumulator: tensor memory -> global.
template <int BN_T>
__device__ __forceinline__ void dump_partial(uint32_t tbase, float *row_dst, int lane, uint32_t release_bar) {
  #pragma unroll 1
  for (int c0 = 0; c0 < BN_T; c0 += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tbase + c0, r);
    tmem_wait_ld();
    if (c0 + 32 >= BN_T) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release_bar);
    }
    float4 *d = reinterpret_cast<float4 *>(row_dst + c0);
    #pragma unroll
    for (int j = 0; j < 8; ++j)
      __stcg(d + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
  }
}

// Operands swapped: tensor-memory lane = output channel, column = token.
// This warp's 32 channels [ch0, ch0 + 32) of tokens [t0, t0 + nt): each
// chunk of 32 tokens is scaled ((acc * x_scale) * w_scale, the same order as
// the unswapped tile), transposed through shared memory ([32 tokens][32
// channels], unswizzled) and stored by TMA; the output map clips tokens >= T
// and channels >= Co.  The accumulator buffer is released after its last
// tensor-memory read.
template <bool F32OUT>
__device__ __forceinline__ void epilogue_store_swap(const CUtensorMap *tmC, uint32_t tbase, uint8_t *cbuf,
                                                    const GemmParams &p, int ch0, int t0, int lane,
                                                    uint32_t release_bar, uint64_t pol) {
  const int ch = ch0 + lane;
  float wsr = 0.0f;
  if constexpr (!F32OUT) wsr = ch < p.Co ? __ldg(p.ws + ch) : 0.0f;
  #pragma unroll 1
  for (int c0 = 0; c0 < p.nt; c0 += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tbase + c0, r);
    tmem_wait_ld();
    if (c0 + 32 >= p.nt) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release_bar);
    }
    float xsl = 0.0f;  // lane j holds the scale of token t0 + c0 + j
    if constexpr (!F32OUT) {
      const int t = t0 + c0 + lane;
      xsl = t < p.T ? __ldg(p.xs + t) : 0.0f;
    }
    // the previous TMA store from this buffer must have finished reading it
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();
    if constexpr (F32OUT) {
      float *s = reinterpret_cast<float *>(cbuf);
      #pragma unroll
      for (int j = 0; j < 32; ++j) s[j * 32 + lane] = __uint_as_float(r[j]);
    } else {
      __nv_bfloat16 *s = reinterpret_cast<__nv_bfloat16 *>(cbuf);
      #pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float xs = __shfl_sync(0xffffffffu, xsl, j);
        s[j * 32 + lane] = __float2bfloat16_rn(__fmul_rn(__fmul_rn(__uint_as_float(r[j]), xs), wsr));
      }
    }
    fence_async_shared();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d_hint(tmC, cbuf, ch0, t0 + c0, pol);
      bulk_commit();
    }
  }
}

// Operands swapped, split tail: this lane's channel of the partial
// accumulator, stored transposed (partial[token][channel], 256 channels a
// token row) so that the reduction reads and writes whole channel runs.
__device__ __forceinline__ void dump_partial_swap(uint32_t tbase, float *col_dst, int nt, int lane,
                                                  uint32_t release_bar) {
  #pragma unroll 1
  for (int c0 = 0; c0 < nt; c0 += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tbase + c0, r);
    tmem_wait_ld();
    if (c0 + 32 >= nt) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release_bar);
    }
    #pragma unroll
    for (int j = 0; j < 32; ++j) __stcg(col_dst + (size_t)(c0 + j) * 256, __uint_as_float(r[j]));
  }
}

// Reducer `ridx` (0 .. 2 * split - 1) of tail tile j at tile position (m, n):
// groups of 8 output columns, [ridx * G / (2 S), (ridx + 1) * G / (2 S)).
// A partial tile is R token rows x BN_T channels (R = 256, or nt when the
// operands are swapped).
// A thread takes U groups at a time and loads four splits of all of them
// before adding (8 U independent 16-byte loads in flight: the partials come
// from L2, and a load-add chain per split would leave the reduction waiting on
// latency); the additions stay in split order 0, 1, 2, ...
template <int BN_T>
__device__ __forceinline__ void reduce_tail_tile(const GemmParams &p, int j, int m, int n, int ridx, int etid) {
  constexpr int U = 2;
  constexpr int SU = 4;
  const int S = p.tail_split;
  const int R = p.swap ? p.nt : 2 * BM;
  constexpr int G8 = BN_T / 8;
  const int G = R * G8;
  const int g0 = (int)((long long)ridx * G / (2 * S));
  const int g1 = (int)((long long)(ridx + 1) * G / (2 * S));
  const float *base = p.partials + (size_t)j * S * R * BN_T;
  const size_t split_stride = (size_t)R * BN_T;
  for (int gb = g0 + etid; gb < g1; gb += U * 32 * kEpiWarps) {
    float a[U][8];
    size_t off[U];
    bool live[U];
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      const int g = gb + u * 32 * kEpiWarps;
      live[u] = g < g1;
      const int row = live[u] ? g / G8 : 0;
      const int c8 = live[u] ? (g - row * G8) * 8 : 0;
      off[u] = (size_t)row * BN_T + c8;
      #pragma unroll
      for (int i = 0; i < 8; ++i) a[u][i] = 0.0f;
    }
    for (int sp0 = 0; sp0 < S; sp0 += SU) {
      float4 v[SU][U][2];
      #pragma unroll
      for (int k = 0; k < SU; ++k) {
        #pragma unroll
        for (int u = 0; u < U; ++u) {
          if (sp0 + k < S && live[u]) {
            const float4 *src = reinterpret_cast<const float4 *>(base + (size_t)(sp0 + k) * split_stride + off[u]);
            v[k][u][0] = __ldcg(src);
            v[k][u][1] = __ldcg(src + 1);
          } else {
            v[k][u][0] = v[k][u][1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          }
        }
      }
      #pragma unroll
      for (int k = 0; k < SU; ++k) {
        if (sp0 + k >= S) break;
        #pragma unroll
        for (int u = 0; u < U; ++u) {
          const float w[8] = {v[k][u][0].x, v[k][u][0].y, v[k][u][0].z, v[k][u][0].w,
                              v[k][u][1].x, v[k][u][1].y, v[k][u][1].z, v[k][u][1].w};
          #pragma unroll
          for (int i = 0; i < 8; ++i) a[u][i] = (sp0 + k == 0) ? w[i] : __fadd_rn(a[u][i], w[i]);
        }
      }
    }
    #pragma unroll
    for (int u = 0; u < U; ++u) {
      if (!live[u]) continue;
      const int g = gb + u * 32 * kEpiWarps;
      const int row = g / G8;
      const int c8 = (g - row * G8) * 8;
      const int t = m * R + row;
      const int col = n * BN_T + c8;
      if (t >= p.T || col >= p.Co) continue;  // Co % 16 == 0: the 8 columns are valid together
      const float xs = __ldg(p.xs + t);
      const float4 w0 = __ldg(reinterpret_cast<const float4 *>(p.ws + col));
      const float4 w1 = __ldg(reinterpret_cast<const float4 *>(p.ws + col + 4));
      const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
      uint32_t o[4];
      #pragma unroll
      for (int i = 0; i < 4; ++i)
        o[i] = pack_bf16x2(__fmul_rn(__fmul_rn(a[u][2 * i], xs), w[2 * i]),
                           __fmul_rn(__fmul_rn(a[u][2 * i + 1], xs), w[2 * i + 1]));
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + (size_t)t * p.Co + col) =
          make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// ----------------------------------------------------------------------------
// CTA-pair kernel (prefill): a cluster of two CTAs on two SMs computes a
// 256 (tokens) x 256 (channels) tile with tcgen05.mma.cta_group::2 (M = 256,
// N = 256, K = 32).  CTA r of the pair loads token rows [r*128, r*128+128)
// of A and channel rows [r*128, r*128+128) of B into its own shared memory
// (no multicast) and signals the leader's (r = 0) stage barrier; the leader
// issues every MMA, reading both CTAs' shared memory, and its commits arrive
// on the barriers of both CTAs.  Each CTA's tensor memory holds its 128 token
// rows x 256 columns, which its own epilogue warps store.  Per SM this moves
// 32 KB of operands per 128-deep K-block instead of 48 KB for a one-CTA
// 128 x 256 tile, for the same tensor work.
// ----------------------------------------------------------------------------
// BN: tile width (MMA N), 256 or 128; each CTA of the pair loads BN / 2
// weight rows.
//
// Swapped operands (BN = 256 variants, p.swap): for token counts that leave
// most of a 256-row tile empty (e.g. T = 300: 512 rows computed for 300), the
// weights become the M = 256 operand (CTA r loads channel rows [r*128,
// r*128+128) of a 256-channel tile) and nt tokens the N operand (CTA r loads
// nt / 2 token rows), nt a multiple of 32 chosen so that the token tiles
// divide T evenly.  Tensor-memory lane = channel, column = token; the
// epilogue transposes through shared memory.  Same ring, barriers, schedule
// and split tail.
template <int STAGES, bool F32OUT, int BN, int WF = 0>
struct PairCfg {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = (BN / 2) * BK;
  static constexpr int B_TX = B_BYTES * wf_bits(WF) / 8;  // weight bytes TMA moves (packed size)
  static constexpr int EPI_BUF = 32 * 128;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators (a power of two >= 32)
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + kEpiWarps * EPI_BUF +
                                 kEpiWarps * 64 * sizeof(float) + 256;
  static_assert(SMEM <= 232448, "shared memory");
};

template <int STAGES, bool F32OUT, int BN, int WF>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ptpc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  using C = PairCfg<STAGES, F32OUT, BN, WF>;
  constexpr int HALF_N = BN / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + STAGES * C::A_BYTES;
  uint8_t *sC = sB + STAGES * C::B_BYTES;
  float *sScale = reinterpret_cast<float *>(sC + kEpiWarps * C::EPI_BUF);
  uint64_t *full = reinterpret_cast<uint64_t *>(sScale + kEpiWarps * 64);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  uint32_t *tail_flag = tmem_holder + 1;  // split tail: 1 while this CTA's protocol is intact

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (elect_one()) {
      // Activation tiles are read by every column tile of their group of tile
      // rows: kept (evict-last).  Weight tiles are read by the group's tile
      // rows at about the same time: normal priority.  Marked evict-first
      // (as in the decode kernel, where each weight byte is read once) they
      // were pushed out of L2 by the output stream before the other rows
      // read them: 10.8 GB of DRAM reads for the 0.54 GB of operands of the
      // 70B gate+up layer at T = 8192.
      const uint64_t polA = policy_evict_last();
      const uint64_t polB = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      Sched sc;
      Unit u;
      // Which shared-memory slot takes the weight tile and which the token
      // tile: unswapped, tokens are the A operand (128 rows a CTA) and
      // weights B (HALF_N rows); swapped, the weights are A (128 channel rows
      // a CTA) and the tokens B (nt / 2 rows a CTA).
      bool swap = false;
      if constexpr (BN == 256) swap = p.swap != 0;
      uint8_t *const sW = swap ? sA : sB;
      uint8_t *const sX = swap ? sB : sA;
      const int w_stride = swap ? C::A_BYTES : C::B_BYTES;
      const int x_stride = swap ? C::B_BYTES : C::A_BYTES;
      const uint32_t stage_tx = swap ? 2u * (uint32_t)(C::B_TX + (p.nt / 2) * BK) : 2u * (C::A_BYTES + C::B_TX);
      const int x_rows = swap ? p.nt : 2 * BM;
      // weight tiles of the first stages before waiting for the previous kernel
      int pre = 0;
      sc.init(p, cid, ncl);
      if (sc.next(p, u)) {
        const int w_row = u.n * BN + (int)rank * HALF_N;
        for (; pre < STAGES && u.kb0 + pre < u.kb1; ++pre) {
          if (leader) mbar_arrive_expect_tx(&full[pre], stage_tx);
          tma_load_2d_pair(sW + pre * w_stride, &tmB, mapa_shared(&full[pre], 0), (u.kb0 + pre) * BK, w_row,
                           polB);
        }
      }
      griddep_wait();
      int issued = 0;
      sc.init(p, cid, ncl);
      while (ok && sc.next(p, u)) {
        const int x_row = u.m * x_rows + (int)rank * (x_rows / 2);
        const int w_row = u.n * BN + (int)rank * HALF_N;
        for (int kb = u.kb0; kb < u.kb1; ++kb, ++issued) {
          const uint32_t lead_full = mapa_shared(&full[stage], 0);
          if (issued >= pre) {
            if (!mbar_wait(&empty[stage], phase ^ 1)) {
              ok = false;
              break;
            }
            if (leader) mbar_arrive_expect_tx(&full[stage], stage_tx);
            tma_load_2d_pair(sW + stage * w_stride, &tmB, lead_full, kb * BK, w_row, polB);
          }
          tma_load_2d_pair(sX + stage * x_stride, &tmA, lead_full, kb * BK, x_row, polA);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      griddep_launch_dependents();
      if (!ok) {
        atomicOr(p.status, kStatusTimeoutProducer);
        // the leader's stage barriers count both CTAs' bytes: once they have
        // all completed, no copy into either CTA is still in flight
        if (leader)
          for (int s = 0; s < STAGES; ++s) mbar_wait(&full[s], s < stage ? phase : phase ^ 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader && elect_one()) {
      // unswapped: A = tokens, B = weights (N = BN); swapped: A = weights, B = tokens (N = nt)
      uint32_t idesc = idesc_f8f6f4_f32(2 * BM, BN, kMmaE4M3, wf_mma(WF));
      if constexpr (BN == 256)
        if (p.swap) idesc = idesc_f8f6f4_f32(2 * BM, p.nt, wf_mma(WF), kMmaE4M3);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      Sched sc;
      sc.init(p, cid, ncl);
      Unit u;
      while (ok && sc.next(p, u)) {
        const int buf = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        ++local;
        if (!mbar_wait(&tempty[buf], aphase ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        for (int kb = u.kb0; kb < u.kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * C::B_BYTES));
          #pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_f8f6f4_pair(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                          (kb > u.kb0 || kk > 0) ? 1u : 0u);
          mma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(&tfull[buf], 0x3);
      }
      if (!ok) atomicOr(p.status, kStatusTimeoutMma);
      mma_commit_pair_mc(drain, 0x1);
      mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int ew = warp - 2;
    const int etid = threadIdx.x - 64;
    uint8_t *cbuf = sC + ew * C::EPI_BUF;
    float *scl = sScale + ew * 64;
    int local = 0;
    bool ok = true;
    bool swap = false;
    if constexpr (BN == 256) swap = p.swap != 0;
    // a member of the split tail: decided by the schedule alone, so every
    // epilogue warp runs the tail protocol's barriers whatever happens above
    const bool tail_member = p.tail_tiles > 0 && !F32OUT && cid < p.tail_tiles * p.tail_split;
    const uint64_t polC = policy_evict_first();  // output lines: never read here
    int tail_j = 0, tail_m = 0, tail_n = 0, tail_r = 0;
    bool dumped = false;
    if (tail_member) {
      if (etid == 0) *tail_flag = 1u;
      epi_bar();
    }
    griddep_wait();
    Sched sc;
    sc.init(p, cid, ncl);
    Unit u;
    while (sc.next(p, u)) {
      const int buf = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      ++local;
      const int row0 = u.m * (2 * BM) + (int)rank * BM + q * 32;
      const int row = row0 + lane;
      float xsr = 0.0f;
      if (!F32OUT && !swap && row < p.T) xsr = __ldg(p.xs + row);
      // tcgen05.ld is warp-collective: the whole warp stops or none of it
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], aphase))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
      if (swap) {
        if constexpr (BN == 256) {
          // lanes are channels u.n * 256 + rank * 128 + q * 32 + lane, columns tokens
          const int ch0 = u.n * BN + (int)rank * HALF_N + q * 32;
          if (u.split < 0) {
            epilogue_store_swap<F32OUT>(&tmC, tbase, cbuf, p, ch0, u.m * p.nt, lane,
                                        mapa_shared(&tempty[buf], 0), polC);
          } else if constexpr (!F32OUT) {
            tail_j = u.tile - p.full_tiles;
            tail_m = u.m;
            tail_n = u.n;
            tail_r = u.split;
            float *dst = p.partials + (size_t)(tail_j * p.tail_split + u.split) * p.nt * BN +
                         (rank * HALF_N + q * 32 + lane);
            dump_partial_swap(tbase, dst, p.nt, lane, mapa_shared(&tempty[buf], 0));
            dumped = true;
          }
        }
      } else if (u.split < 0) {
        epilogue_store_tile<BN, F32OUT>(&tmC, tbase, cbuf, scl, p, u.n * BN, row0, xsr, lane,
                                        mapa_shared(&tempty[buf], 0), polC);
      } else if constexpr (!F32OUT) {
        tail_j = u.tile - p.full_tiles;
        tail_m = u.m;
        tail_n = u.n;
        tail_r = u.split;
        float *dst = p.partials +
                     ((size_t)(tail_j * p.tail_split + u.split) * (2 * BM) + rank * BM + q * 32 + lane) * BN;
        dump_partial<BN>(tbase, dst, lane, mapa_shared(&tempty[buf], 0));
        dumped = true;
      }
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeoutEpilogue);
    if (lane == 0) bulk_wait<0>();
    if (tail_member) {
      // 1. count this CTA in once all four warps have stored their rows
      __threadfence();
      if (!dumped && lane == 0) atomicAnd(tail_flag, 0u);
      epi_bar();
      uint32_t *arrived = p.tail_count + tail_j;
      uint32_t *finished = p.tail_count + p.tail_tiles + tail_j;
      const uint32_t members = 2u * (uint32_t)p.tail_split;
      if (etid == 0) {
        if (*tail_flag) {
          __threadfence();  // after the barrier: releases every warp's partial stores
          atomicAdd(arrived, 1u);
          // 2. wait (bounded) for every member CTA of the tile
          bool all = ld_acquire_u32(arrived) >= members;
          const uint64_t t0 = global_timer_ns();
          while (!all) {
            __nanosleep(256);
            all = ld_acquire_u32(arrived) >= members;
            if (!all && global_timer_ns() - t0 > kWaitLimitNs) break;
          }
          if (!all) {
            atomicOr(p.status, kStatusTimeoutEpilogue);
            *tail_flag = 0u;
          }
        }
      }
      epi_bar();
      __threadfence();
      // 3. this CTA's share of the tile
      if (*tail_flag) reduce_tail_tile<BN>(p, tail_j, tail_m, tail_n, tail_r * 2 + (int)rank, etid);
      __threadfence();
      epi_bar();
      // 4. the last member to finish leaves the counters zero
      if (etid == 0 && *tail_flag) {
        if (atomicAdd(finished, 1u) == members - 1u) {
          atomicExch(arrived, 0u);
          atomicExch(finished, 0u);
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync();  // the leader's MMAs into both CTAs' tensor memory are complete
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// What a 2-D tensor map encodes.  The encoding depends on nothing else (not
// on the current device or context), so equal keys give identical maps.
struct MapKey {
  const void *base;
  uint64_t inner, outer, row_bytes;
  uint32_t box_inner, box_outer;
  int dt, sw;
  bool operator==(const MapKey &o) const {
    return base == o.base && inner == o.inner && outer == o.outer && row_bytes == o.row_bytes &&
           box_inner == o.box_inner && box_outer == o.box_outer && dt == o.dt && sw == o.sw;
  }
};

struct MapKeyHash {
  size_t operator()(const MapKey &k) const {
    uint64_t h = reinterpret_cast<uintptr_t>(k.base);
    for (uint64_t v : {k.inner, k.outer, k.row_bytes, (uint64_t)k.box_inner << 32 | k.box_outer,
                       (uint64_t)k.dt << 8 | (uint64_t)k.sw})
      h = (h ^ v) * 0x100000001B3ull + (h >> 29);
    return (size_t)h;
  }
};

// Encoded tensor maps, keyed by what they encode.  Layers call the GEMM with
// the same buffers again and again, so after the first call of a layer its
// maps come from here instead of being encoded anew.  Bounded: emptied when
// it reaches `cap` entries.  Thread-safe; the encoder runs outside the lock.
class MapCache {
 public:
  explicit MapCache(size_t cap) : cap_(cap) {}

  template <typename Encoder>
  bool get(CUtensorMap *m, const MapKey &k, Encoder encode) {
    {
      std::lock_guard<std::mutex> lock(mu_);
      auto it = map_.find(k);
      if (it != map_.end()) {
        *m = it->second;
        hits_.fetch_add(1, std::memory_order_relaxed);
        return true;
      }
    }
    if (!encode(m, k)) return false;
    misses_.fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> lock(mu_);
    if (map_.size() >= cap_) map_.clear();
    map_.emplace(k, *m);
    return true;
  }

  uint64_t hits() const { return hits_.load(std::memory_order_relaxed); }
  uint64_t misses() const { return misses_.load(std::memory_order_relaxed); }
  size_t size() {
    std::lock_guard<std::mutex> lock(mu_);
    return map_.size();
  }

 private:
  size_t cap_;
  std::mutex mu_;
  std::unordered_map<MapKey, CUtensorMap, MapKeyHash> map_;
  std::atomic<uint64_t> hits_{0}, misses_{0};
};

constexpr size_t kMapCacheMax = 4096;
MapCache g_maps(kMapCacheMax);   // shared by every device and host thread

bool encode_map_2d(CUtensorMap *m, const MapKey &k) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {k.inner, k.outer};
  cuuint64_t strides[1] = {k.row_bytes};
  cuuint32_t box[2] = {k.box_inner, k.box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, (CUtensorMapDataType)k.dt, 2, const_cast<void *>(k.base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, (CUtensorMapSwizzle)k.sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  const MapKey k{base, inner, outer, row_bytes, box_inner, box_outer, (int)dt, (int)sw};
  return g_maps.get(m, k, encode_map_2d);
}

// Tensor map of the weight codes Wq [Co, Ci]: one byte per code (E4M3), or
// packed 4-bit / 6-bit codes that TMA unpacks into 16-byte chunks of 16 codes
// in shared memory (box inner extent 128 codes, rows 32-byte aligned).
bool make_weight_map(CUtensorMap *m, const GemmProblem &pr, uint32_t rows) {
  if (pr.wfmt == 0)
    return make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Wq_t, pr.Ci, pr.Co, pr.Ci, BK, rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  const CUtensorMapDataType dt =
      pr.wfmt == 1 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_16U6_ALIGN16B;
  return make_map_2d(m, dt, pr.Wq_t, pr.Ci, pr.Co, (uint64_t)pr.Ci * wf_bits(pr.wfmt) / 8, BK, rows,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_maps(const GemmProblem &pr, uint32_t b_rows, CUtensorMap *tmA, CUtensorMap *tmB, CUtensorMap *tmC) {
  if (!make_map_2d(tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Xq, pr.Ci, pr.T, pr.Ci, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_weight_map(tmB, pr, b_rows))
    return false;
  if (pr.f32_out)
    return make_map_2d(tmC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 4, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  return make_map_2d(tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 2, 64, 32,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

// Swapped operands: token tiles of nt / 2 rows a CTA, weight tiles of 128
// rows a CTA, and an output box of 32 channels x 32 tokens, unswizzled (the
// epilogue's transposed staging).
bool make_swap_maps(const GemmProblem &pr, int nt, CUtensorMap *tmA, CUtensorMap *tmB, CUtensorMap *tmC) {
  if (!make_map_2d(tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Xq, pr.Ci, pr.T, pr.Ci, BK, (uint32_t)(nt / 2),
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_weight_map(tmB, pr, BM))
    return false;
  if (pr.f32_out)
    return make_map_2d(tmC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 4, 32, 32,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
  return make_map_2d(tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 2, 32, 32,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Ring depth of the pair kernel per tile width (the stages fill ~192 KB).
template <int BN>
constexpr int pair_stages() {
  return BN == 256 ? 6 : 8;
}

template <bool F32OUT, int BN, int WF = 0>
void set_pair_smem() {
  cudaFuncSetAttribute(ptpc_gemm_pair_kernel<pair_stages<BN>(), F32OUT, BN, WF>,
                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)PairCfg<pair_stages<BN>(), F32OUT, BN, WF>::SMEM);
}

// CTA pairs of the BN-wide pair kernel that can be resident at once.
template <int BN>
int pair_resident(int sms) {
  cudaLaunchConfig_t q = {};
  q.gridDim = dim3(2 * (sms / 2));
  q.blockDim = dim3(kThreads);
  q.dynamicSmemBytes = PairCfg<pair_stages<BN>(), false, BN>::SMEM;
  int ncl = 0;
  if (cudaOccupancyMaxActiveClusters(&ncl, ptpc_gemm_pair_kernel<pair_stages<BN>(), false, BN, 0>, &q) != cudaSuccess ||
      ncl <= 0)
    ncl = sms / 2;
  cudaGetLastError();
  return ncl;
}

// Per device: dynamic shared-memory opt-in of every kernel variant, the SM
// count, and the number of CTA pairs that can be resident at once.
struct DeviceInfo {
  bool ready = false;
  int sms = 148;
  int pair_clusters = 74;     // resident CTA pairs, 256-wide tiles
  int pair_clusters128 = 74;  // resident CTA pairs, 128-wide tiles
  int dec_clusters[9] = {};  // resident decode clusters of 2, 4 and 8 CTAs
};

// Most clusters of `size` CTAs of `kernel` (with `smem` bytes each) that can
// be resident at once; 0 if unknown.
template <typename Kernel>
int max_clusters(Kernel kernel, int sms, int size, size_t smem) {
  cudaLaunchConfig_t q = {};
  q.gridDim = dim3(size * (sms / size));
  q.blockDim = dim3(kThreads);
  q.dynamicSmemBytes = smem;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeClusterDimension;
  a[0].val.clusterDim.x = size;
  a[0].val.clusterDim.y = 1;
  a[0].val.clusterDim.z = 1;
  q.attrs = a;
  q.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &q) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

const DeviceInfo &device_info() {
  static DeviceInfo info[64];
  static std::atomic<bool> ready[64];
  static DeviceInfo fallback;
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return fallback;
  }
  if (ready[dev].load(std::memory_order_acquire)) return info[dev];
  std::lock_guard<std::mutex> lock(mu);  // first use of a device may come from several host threads
  DeviceInfo &d = info[dev];
  if (!ready[dev].load(std::memory_order_relaxed)) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) d.sms = v;
    for (auto k : {ptpc_gemm_decode_kernel<false, 0>, ptpc_gemm_decode_kernel<true, 0>,
                   ptpc_gemm_decode_kernel<false, 1>, ptpc_gemm_decode_kernel<false, 2>,
                   ptpc_gemm_decode_kernel<false, 3>})
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecSmemMax);
    set_pair_smem<false, 256>();
    set_pair_smem<true, 256>();
    set_pair_smem<false, 128>();
    set_pair_smem<true, 128>();
    set_pair_smem<false, 256, 1>();
    set_pair_smem<false, 128, 1>();
    set_pair_smem<false, 256, 2>();
    set_pair_smem<false, 128, 2>();
    set_pair_smem<false, 256, 3>();
    set_pair_smem<false, 128, 3>();
    // the pair kernel's cluster size is compiled in (__cluster_dims__)
    d.pair_clusters = pair_resident<256>(d.sms);
    d.pair_clusters128 = pair_resident<128>(d.sms);
    // the decode kernel takes its cluster size at launch; ask for the largest
    // shared-memory footprint it launches with
    for (int size = 2; size <= 8; size *= 2) {
      const int a = max_clusters(ptpc_gemm_decode_kernel<false, 0>, d.sms, size, kDecSmemMax);
      const int b = max_clusters(ptpc_gemm_decode_kernel<true, 0>, d.sms, size, kDecSmemMax);
      d.dec_clusters[size] = std::min(a, b);
    }
    d.ready = true;
    ready[dev].store(true, std::memory_order_release);
  }
  return d;
}

// The launch plan of one problem.
struct Plan {
  bool pair;
  int tile_rows, bn;
  int num_m, num_n, num_kb, num_tiles;
  int group_m;
  int ctas;     // CTAs (decode kernel) or CTA pairs (pair kernel) launched
  int ksplit;   // decode kernel: CTAs per tile (cluster size), 1 = whole tiles
  int np, stages, tmem_cols;  // decode kernel only
  bool red_fits;              // decode kernel: the K-split buffer fits in the ring
  int tail_tiles, tail_split; // pair kernel: split tail (0: every tile whole)
  bool swap;                  // pair kernel: weights as the M operand, nt tokens a tile
  int nt;
};

// Time of a 128-wide pair tile relative to half a 256-wide one.  Measured on
// B200 from wave counts and times of both widths: 1.05-1.09 where the GEMM is
// short, 1.14-1.18 on longer ones, 1.32 on the 70B gate+up at T = 8192 (more
// operand bytes per FLOP under the power cap).  1.15 picks the faster width
// on every measured shape, e.g. 512 x 8192 -> 10240: 53.7 us (128-wide, 3
// waves) against 68.1 us (256-wide, 2 waves of which the second is 8% full).
constexpr double kPairN128Cost = 1.15;

// Tuning overrides (not for production use), from the environment:
// PTPC_FORCE_KERNEL = pair | decode, PTPC_FORCE_PAIR_BN = 128 | 256,
// PTPC_FORCE_KSPLIT = 1 | 2 | 4 | 8, PTPC_FORCE_SPLIT_TAIL = 0 | 1 (the pair
// kernel's split tail off, or on wherever it is feasible), PTPC_FORCE_SWAP =
// 0 | 1 (the pair kernel's swapped operands off, or on for every pair-kernel
// shape), PTPC_FORCE_GROUP_M = 1 .. 63 (tile rows visited together by the pair
// kernel).  Read once, at the first GEMM call of the process (or again by
// reload_tuning), not on every call.
struct Tuning {
  int kernel;   // 0 automatic, 1 pair, 2 decode
  int pair_bn;  // 0 automatic, 128, 256
  int ksplit;   // 0 automatic, 1, 2, 4, 8
  int streamk;  // 0 automatic, 1 off, 2 on wherever feasible
  int swap;     // 0 automatic, 1 off, 2 on
  int group_m;  // 0 automatic, else tile rows a group (1 .. 63)
};

int env_int(const char *name, int fallback) {
  const char *v = std::getenv(name);
  if (v == nullptr || *v == '\0') return fallback;
  char *end = nullptr;
  const long x = std::strtol(v, &end, 10);
  return (end != nullptr && *end == '\0') ? (int)x : fallback;
}

Tuning read_tuning() {
  Tuning t{0, 0, 0, 0, 0, 0};
  const char *k = std::getenv("PTPC_FORCE_KERNEL");
  if (k != nullptr && std::strcmp(k, "pair") == 0) t.kernel = 1;
  if (k != nullptr && std::strcmp(k, "decode") == 0) t.kernel = 2;
  const int bn = env_int("PTPC_FORCE_PAIR_BN", 0);
  if (bn == 128 || bn == 256) t.pair_bn = bn;
  const int ks = env_int("PTPC_FORCE_KSPLIT", 0);
  if (ks == 1 || ks == 2 || ks == 4 || ks == 8) t.ksplit = ks;
  const int sk = env_int("PTPC_FORCE_SPLIT_TAIL", -1);
  if (sk == 0) t.streamk = 1;
  if (sk == 1) t.streamk = 2;
  const int sw = env_int("PTPC_FORCE_SWAP", -1);
  if (sw == 0) t.swap = 1;
  if (sw == 1) t.swap = 2;
  const int gm = env_int("PTPC_FORCE_GROUP_M", 0);
  if (gm >= 1 && gm <= 63) t.group_m = gm;
  return t;
}

// Packed as kernel | pair_bn / 128 << 2 | ksplit << 4 | streamk << 9 |
// swap << 11 | group_m << 13, plus bit 8 once read.
std::atomic<uint32_t> g_tuning{0};

uint32_t pack_tuning(const Tuning &t) {
  return 0x100u | (uint32_t)t.kernel | (uint32_t)(t.pair_bn / 128) << 2 | (uint32_t)t.ksplit << 4 |
         (uint32_t)t.streamk << 9 | (uint32_t)t.swap << 11 | (uint32_t)t.group_m << 13;
}

Tuning tuning() {
  uint32_t v = g_tuning.load(std::memory_order_relaxed);
  if ((v & 0x100u) == 0) {
    v = pack_tuning(read_tuning());
    g_tuning.store(v, std::memory_order_relaxed);
  }
  return Tuning{(int)(v & 3u), (int)((v >> 2) & 3u) * 128, (int)((v >> 4) & 15u), (int)((v >> 9) & 3u),
                (int)((v >> 11) & 3u), (int)((v >> 13) & 63u)};
}

// Fewest K-blocks a CTA of a K-split cluster streams.
constexpr int kMinSplitKb = 4;

// The decode kernel's plan for T <= kDecodeMaxT: whole 128-channel tiles, or
// K split over a cluster when that puts at least twice as many SMs on the
// weight stream, all tiles in one wave.
Plan decode_plan(int T, int Ci, int Co, const DeviceInfo &d) {
  Plan pl = {};
  pl.pair = false;
  pl.num_kb = (Ci + BK - 1) / BK;
  pl.tile_rows = std::max(T, 1);  // one tile row holds every token
  pl.bn = BM;
  pl.group_m = 1;
  pl.np = std::max(16, (T + 15) / 16 * 16);
  const size_t stage_bytes = kDecWBytes + (size_t)pl.np * BK;
  pl.stages = (int)std::min<size_t>(kDecMaxStages, (kDecSmemMax - dec_smem_bytes(pl.np, 0)) / stage_bytes);
  pl.tmem_cols = 64;  // each accumulator starts on a 32-column boundary
  while (pl.tmem_cols < 2 * pl.np) pl.tmem_cols <<= 1;
  // the K-split reduction buffer must fit in the ring (true for every NP <= 256)
  pl.red_fits = (size_t)pl.np * BM * sizeof(float) <= (size_t)pl.stages * stage_bytes;
  pl.num_m = 1;
  pl.num_n = (Co + BM - 1) / BM;
  pl.num_tiles = pl.num_n;
  pl.ksplit = 1;
  auto feasible = [&](int size) {
    return (long long)pl.num_tiles * size <= d.sms && pl.num_tiles <= d.dec_clusters[size] &&
           pl.num_kb >= size * kMinSplitKb && pl.red_fits;
  };
  for (int size = 8; size >= 2; size /= 2) {
    if (feasible(size)) {
      pl.ksplit = size;
      break;
    }
  }
  // PTPC_FORCE_KSPLIT = 1, 2, 4 or 8 (tuning only; ignored where infeasible)
  const int forced = tuning().ksplit;
  if (forced == 1 || ((forced == 2 || forced == 4 || forced == 8) && feasible(forced))) pl.ksplit = forced;
  pl.ctas = pl.ksplit > 1 ? pl.num_tiles * pl.ksplit : std::max(1, std::min(pl.num_tiles, d.sms));
  return pl;
}

// Tile width of the pair kernel for a shape: 128-wide tiles halve the size of
// the last partial wave but move more operand bytes per FLOP, so they are
// taken only when they finish the waves sooner by a margin.
int choose_pair_bn(int T, int Co, const DeviceInfo &d) {
  const int forced = tuning().pair_bn;  // 128 or 256 (tuning only)
  if (forced != 0) return forced;
  const long long m = (T + 2 * BM - 1) / (2 * BM);
  const long long w256 = (m * ((Co + 255) / 256) + d.pair_clusters - 1) / d.pair_clusters;
  const long long w128 = (m * ((Co + 127) / 128) + d.pair_clusters128 - 1) / d.pair_clusters128;
  // cost in 128-wide tile-times; a 128-wide tile costs kPairN128Cost of half a 256-wide one
  return (double)w128 * kPairN128Cost < (double)(2 * w256) ? 128 : 256;
}

// Split tail of the pair kernel.  With W whole waves and R < pairs tiles
// left, the last wave keeps only R of the pairs busy for a whole tile time.
// Splitting those R tiles along K over S = pairs / R pairs each (S >= 2, at
// least kMinTailKb K-blocks per split) finishes them in about 1/S of a tile
// time plus the partials' round trip through L2 and the distributed
// reduction.  Taken only where the caller's workspace holds the partials.
constexpr int kMinTailKb = 4;
// Measured on B200 (70B layers, T = 256 ... 3001, split on against off): the
// split pays only on long K (down-proj, K = 28672: +8% at T = 2048, +13% at
// T = 3001); at K = 8192 it is within +-2% on gate+up and 1-5% slower on
// the 10240-wide QKV, since a last wave of few tiles already runs at the
// higher clock that the idle rest of the GPU leaves it.
constexpr int kMinTailTotalKb = 128;
constexpr int kMaxTailPairs = 74;      // bound of the workspace size (a B200's 148 SMs in pairs)
constexpr size_t kTailCountBytes = 1024;

size_t tail_workspace(int tail_tiles, int split, int bn) {
  return kTailCountBytes + (size_t)tail_tiles * split * (2 * BM) * bn * sizeof(float);
}

void choose_tail(Plan &pl, size_t ws_bytes) {
  pl.tail_tiles = 0;
  pl.tail_split = 0;
  const int forced = tuning().streamk;          // 0 automatic, 1 off, 2 on
  if (forced == 1 || pl.num_tiles <= pl.ctas) return;
  if (forced != 2 && pl.num_kb < kMinTailTotalKb) return;
  const int rem = pl.num_tiles % pl.ctas;
  if (rem == 0) return;
  const int pairs = std::min(pl.ctas, kMaxTailPairs);
  int split = std::min(pairs / rem, pl.num_kb / kMinTailKb);
  if (split < 2) return;
  // worth it only if the last wave is mostly idle: at most half the pairs busy
  if (forced != 2 && 2 * rem > pl.ctas) return;
  if (kGemmStatusBytes + tail_workspace(rem, split, pl.bn) > ws_bytes) return;
  pl.tail_tiles = rem;
  pl.tail_split = split;
}

// Cost of a swapped pair tile of nt tokens, in unswapped 256 x 256 tile
// times: F + (1 - F) nt / 256.  The tensor work scales with nt, but every
// stage still moves the 16 KB-a-CTA weight tile through shared memory
// (written by TMA, read by the MMA) whatever nt is.  Measured on B200 (70B
// layers, same tile counts both ways): nt = 160 costs 0.74, 192 0.81, 224
// 0.87 of an unswapped tile; F = 0.3 fits the small nt, which matter most.
constexpr double kSwapFixed = 0.3;

double swap_tile_cost(int nt) {
  const double f = nt / 256.0;
  return kSwapFixed + (1.0 - kSwapFixed) * f;
}

// Tile times of `tiles` tiles on `pairs` CTA pairs: whole waves, and a last
// partial wave that costs a whole tile time, or 1/split of one (plus 0.1 for
// the partials' round trip) where the split tail takes it (same conditions
// as choose_tail).
double est_waves(long long tiles, int pairs, int num_kb, size_t ws_bytes, int bn) {
  const long long full = tiles / pairs;
  const long long rem = tiles % pairs;
  if (rem == 0) return (double)full;
  const int forced = tuning().streamk;
  if (full > 0 && forced != 1 && (forced == 2 || num_kb >= kMinTailTotalKb) && (forced == 2 || 2 * rem <= pairs)) {
    const int split = (int)std::min<long long>(std::min(pairs, kMaxTailPairs) / rem, num_kb / kMinTailKb);
    if (split >= 2 && kGemmStatusBytes + tail_workspace((int)rem, split, bn) <= ws_bytes)
      return (double)full + 1.0 / split + 0.1;
  }
  return (double)(full + 1);
}

// The prefill kernel's plan: whole tiles on the CTA pairs, 256 tokens x BN
// channels a tile, or, with the operands swapped, 256 channels x nt tokens
// where that finishes the waves sooner (ragged T: the token tiles divide T
// evenly instead of rounding it up to 256 rows), then the split tail.
// Tile rows visited together: at most kGroupMaxRows, and no more than keep
// kGroupL2Bytes of activation tiles (half the 126 MB L2).  Measured on the
// 70B layers at T = 8192 (32 tile rows; ncu DRAM reads of one launch without
// a cache flush): gate+up (2 MB of activations a row) 2.53 GB with groups of
// 8, 1.41 GB with 16, 3.50 GB with 32; down-proj (7.3 MB a row) 2.07 GB with
// 8, 2.33 GB with 16.
constexpr long long kGroupL2Bytes = 64ll << 20;
constexpr int kGroupMaxRows = 16;

Plan pair_plan(int T, int Ci, int Co, const DeviceInfo &d, size_t ws_bytes) {
  Plan pl = {};
  pl.pair = true;
  pl.ksplit = 1;
  pl.num_kb = (Ci + BK - 1) / BK;
  pl.tile_rows = 2 * BM;
  pl.bn = choose_pair_bn(T, Co, d);
  pl.num_m = (T + pl.tile_rows - 1) / pl.tile_rows;
  pl.num_n = (Co + pl.bn - 1) / pl.bn;
  pl.num_tiles = pl.num_m * pl.num_n;
  const int pairs = pl.bn == 128 ? d.pair_clusters128 : d.pair_clusters;
  // swapped: ceil(T / 256) token tiles of equal size, rounded up to 32
  const int ntt = (T + 2 * BM - 1) / (2 * BM);
  const int nt = ((T + ntt - 1) / ntt + 31) / 32 * 32;
  const long long swap_tiles = (long long)ntt * ((Co + 255) / 256);
  const double cost_plain = est_waves(pl.num_tiles, pairs, pl.num_kb, ws_bytes, pl.bn) *
                            (pl.bn == 128 ? 0.5 * kPairN128Cost : 1.0);
  const double cost_swap = est_waves(swap_tiles, d.pair_clusters, pl.num_kb, ws_bytes, 256) * swap_tile_cost(nt);
  const int forced = tuning().swap;  // 0 automatic, 1 off, 2 on
  pl.swap = forced == 2 || (forced == 0 && cost_swap < cost_plain);
  if (pl.swap) {
    pl.nt = nt;
    pl.tile_rows = nt;
    pl.bn = 256;
    pl.num_m = ntt;
    pl.num_n = (Co + 255) / 256;
    pl.num_tiles = (int)swap_tiles;
  }
  // Tile rows visited together: their activation tiles stay in L2 (loaded
  // evict-last) while the column tiles sweep past, so every weight tile is
  // read from DRAM once per group.
  const long long row_bytes = (long long)pl.tile_rows * Ci;
  pl.group_m = (int)std::max(1LL, std::min<long long>(std::min(pl.num_m, kGroupMaxRows), kGroupL2Bytes / row_bytes));
  if (tuning().group_m > 0) pl.group_m = std::min(pl.num_m, tuning().group_m);
  pl.ctas = std::max(1, std::min(pl.num_tiles, pl.bn == 128 ? d.pair_clusters128 : d.pair_clusters));
  choose_tail(pl, ws_bytes);
  return pl;
}

// Which kernel runs a shape.  Measured on B200 with weights streamed from
// HBM (70B layer shapes): the decode kernel is faster than the pair kernel
// for every T <= 160 and ties at T = 192; above, the pair kernel wins, with a
// K split in the decode kernel too (T = 256, 28672 -> 8192: 53.8 us against
// 66.1 us; 8192 -> 8192: 25.3 against 31.4 us).
// PTPC_FORCE_KERNEL = "pair" or "decode" overrides the choice (tuning only;
// the decode kernel takes T <= 256 only).
Plan make_plan(int T, int Ci, int Co, size_t ws_bytes) {
  const DeviceInfo &d = device_info();
  const int force = tuning().kernel;
  if (force == 1) return pair_plan(T, Ci, Co, d, ws_bytes);
  if (T <= kDecodeMaxT && (force == 2 || T <= kDecodeWholeMaxT)) return decode_plan(T, Ci, Co, d);
  return pair_plan(T, Ci, Co, d, ws_bytes);
}

template <typename Kernel>
cudaError_t launch_decode(Kernel kernel, int grid, int cluster, size_t smem, const CUtensorMap &tmW,
                          const CUtensorMap &tmX, const GemmParams &gp, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tmW, tmX, gp);
}

template <typename Kernel>
cudaError_t launch(Kernel kernel, int grid, size_t smem, const CUtensorMap &tmA, const CUtensorMap &tmB,
                   const CUtensorMap &tmC, const GemmParams &gp, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmC, gp);
}

template <bool F32OUT, int BN, int WF = 0>
cudaError_t launch_pair(int grid, const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmC,
                        const GemmParams &gp, bool pdl, cudaStream_t st) {
  return launch(ptpc_gemm_pair_kernel<pair_stages<BN>(), F32OUT, BN, WF>, grid,
                PairCfg<pair_stages<BN>(), F32OUT, BN, WF>::SMEM, tmA, tmB, tmC, gp, pdl, st);
}

}  // namespace

int num_sms() { return device_info().sms; }

void reload_tuning() { g_tuning.store(pack_tuning(read_tuning()), std::memory_order_relaxed); }

void map_cache_stats(uint64_t *hits, uint64_t *misses) {
  *hits = g_maps.hits();
  *misses = g_maps.misses();
}

int map_cache_selftest() {
  // a private cache of 4 entries and an encoder that only counts its calls
  // and stamps the key's pointer into the map
  MapCache c(4);
  int encodes = 0;
  auto fake = [&](CUtensorMap *m, const MapKey &k) {
    ++encodes;
    std::memset(m, 0, sizeof(*m));
    std::memcpy(m, &k.base, sizeof(k.base));
    return true;
  };
  auto key = [](uintptr_t base, uint64_t rows) {
    return MapKey{reinterpret_cast<const void *>(base), 4096, rows, 4096, 128, 128, 0, 3};
  };
  CUtensorMap m;
  const void *got = nullptr;
  int fails = 0;
  auto check = [&](bool ok) { fails += ok ? 0 : 1; };
  check(c.get(&m, key(0x1000, 64), fake) && encodes == 1 && c.misses() == 1 && c.hits() == 0);
  check(c.get(&m, key(0x1000, 64), fake) && encodes == 1 && c.hits() == 1);          // hit
  std::memcpy(&got, &m, sizeof(got));
  check(got == reinterpret_cast<const void *>(0x1000));
  check(c.get(&m, key(0x2000, 64), fake) && encodes == 2);                           // same shape, other pointer
  std::memcpy(&got, &m, sizeof(got));
  check(got == reinterpret_cast<const void *>(0x2000));
  check(c.get(&m, key(0x1000, 128), fake) && encodes == 3);                          // same pointer, other shape
  check(c.get(&m, key(0x1000, 64), fake) && encodes == 3 && c.hits() == 2);          // still cached
  check(c.size() == 3);
  check(c.get(&m, key(0x3000, 64), fake) && c.size() == 4);
  check(c.get(&m, key(0x4000, 64), fake) && c.size() == 1 && encodes == 5);          // full: emptied, then added
  check(c.get(&m, key(0x1000, 64), fake) && encodes == 6);                           // gone with the rest
  auto failing = [](CUtensorMap *, const MapKey &) { return false; };
  check(!c.get(&m, key(0x5000, 64), failing) && c.size() == 2);                      // a failed encode is not stored
  return fails;
}

int gemm_ksplit(int T, int Ci, int Co) { return make_plan(T, Ci, Co, gemm_workspace_bytes(T, Ci, Co)).ksplit; }

int gemm_tail_split(int T, int Ci, int Co, size_t ws_bytes) { return make_plan(T, Ci, Co, ws_bytes).tail_split; }

int gemm_swap_tokens(int T, int Ci, int Co, size_t ws_bytes) {
  const Plan pl = make_plan(T, Ci, Co, ws_bytes);
  return pl.pair && pl.swap ? pl.nt : 0;
}

size_t gemm_workspace_bytes(int T, int Ci, int Co) {
  // the status word, plus the split tail's counters and partials where the
  // pair kernel could split one (more than one wave, K long enough), sized
  // for kMaxTailPairs pairs of 256-wide tiles
  const int num_kb = (Ci + BK - 1) / BK;
  if (T <= kDecodeWholeMaxT || num_kb < 2 * kMinTailKb) return kGemmStatusBytes;
  return kGemmStatusBytes + tail_workspace(1, kMaxTailPairs, 256);
}

cudaError_t launch_scaled_gemm(const GemmProblem &pr, cudaStream_t st) {
  const Plan pl = make_plan(pr.T, pr.Ci, pr.Co, pr.f32_out ? 0 : pr.ws_bytes);
  GemmParams gp = {};
  gp.T = pr.T;
  gp.Co = pr.Co;
  gp.num_m = pl.num_m;
  gp.num_n = pl.num_n;
  gp.num_kb = pl.num_kb;
  gp.group_m = pl.group_m;
  gp.num_tiles = pl.num_tiles;
  gp.ksplit = pl.ksplit;
  gp.np = pl.np;
  gp.stages = pl.stages;
  gp.tmem_cols = pl.tmem_cols;
  gp.tail_tiles = pl.tail_tiles;
  gp.tail_split = pl.tail_split;
  gp.full_tiles = pl.num_tiles - pl.tail_tiles;
  gp.swap = pl.swap ? 1 : 0;
  gp.nt = pl.nt;
  if (pl.tail_tiles > 0) {
    uint8_t *w = reinterpret_cast<uint8_t *>(pr.status);
    gp.tail_count = reinterpret_cast<uint32_t *>(w + kGemmStatusBytes);
    gp.partials = reinterpret_cast<float *>(w + kGemmStatusBytes + kTailCountBytes);
  }
  gp.xs = pr.xs;
  gp.ws = pr.ws;
  gp.out = pr.out;
  gp.status = pr.status;
  if (pr.f32_out && pr.wfmt != 0) return cudaErrorInvalidValue;  // the naive path is E4M3 only
  if (!pl.pair) {
    CUtensorMap tmW, tmX;
    if (!make_weight_map(&tmW, pr, BM) ||
        !make_map_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Xq, pr.Ci, pr.T, pr.Ci, BK, pl.np,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const size_t smem = dec_smem_bytes(pl.np, pl.stages);
    switch (pr.f32_out ? -1 : pr.wfmt) {
      case -1: return launch_decode(ptpc_gemm_decode_kernel<true, 0>, pl.ctas, pl.ksplit, smem, tmW, tmX, gp, pr.pdl, st);
      case 1: return launch_decode(ptpc_gemm_decode_kernel<false, 1>, pl.ctas, pl.ksplit, smem, tmW, tmX, gp, pr.pdl, st);
      case 2: return launch_decode(ptpc_gemm_decode_kernel<false, 2>, pl.ctas, pl.ksplit, smem, tmW, tmX, gp, pr.pdl, st);
      case 3: return launch_decode(ptpc_gemm_decode_kernel<false, 3>, pl.ctas, pl.ksplit, smem, tmW, tmX, gp, pr.pdl, st);
      default: return launch_decode(ptpc_gemm_decode_kernel<false, 0>, pl.ctas, pl.ksplit, smem, tmW, tmX, gp, pr.pdl, st);
    }
  }
  CUtensorMap tmA, tmB, tmC;
  if (pl.swap) {
    if (!make_swap_maps(pr, pl.nt, &tmA, &tmB, &tmC)) return cudaErrorInvalidValue;
  } else if (!make_maps(pr, pl.bn / 2, &tmA, &tmB, &tmC)) {
    return cudaErrorInvalidValue;
  }
  const int grid = 2 * pl.ctas;
  if (pr.f32_out)
    return pl.bn == 128 ? launch_pair<true, 128>(grid, tmA, tmB, tmC, gp, pr.pdl, st)
                        : launch_pair<true, 256>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
  if (pl.bn == 128) {
    switch (pr.wfmt) {
      case 1: return launch_pair<false, 128, 1>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
      case 2: return launch_pair<false, 128, 2>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
      case 3: return launch_pair<false, 128, 3>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
      default: return launch_pair<false, 128, 0>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
    }
  }
  switch (pr.wfmt) {
    case 1: return launch_pair<false, 256, 1>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
    case 2: return launch_pair<false, 256, 2>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
    case 3: return launch_pair<false, 256, 3>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
    default: return launch_pair<false, 256, 0>(grid, tmA, tmB, tmC, gp, pr.pdl, st);
  }
}

}  // namespace ptpc
