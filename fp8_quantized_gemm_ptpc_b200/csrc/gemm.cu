// PTPC-FP8 scaled GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// out[t][o] = bf16_RNE((acc[t][o] * x_scale[t]) * w_scale[o]),
// acc[t][o] = sum_k dec(Xq[t][k]) * dec(Wq_t[o][k]),
// the fused row-wise-scaled FP8 GEMM of "PTPC-FP8: boosting vLLM performance
// on AMD ROCm" (section "The challenge: two-step vs fused"): the two scale
// vectors are applied to the accumulator on chip, between the tensor-memory
// load and the single store of the output, so no T x Co intermediate is ever
// written.  The page's kernel is AMD's (MI300X); this one is written for B200:
//
//   * persistent CTAs (one per SM) walk output tiles of 128 tokens x BN
//     channels in an L2-friendly grouped order;
//   * warp 0 (one thread) streams 128-byte-wide K slices of Xq and Wq_t with
//     TMA into a STAGES-deep shared-memory ring (128-byte swizzle);
//   * warp 1 (one thread) issues tcgen05.mma kind::f8f6f4 (E4M3 x E4M3 ->
//     fp32, M = 128, N = BN, K = 32) into one of two tensor-memory
//     accumulators, and commits each stage back to the producer;
//   * warps 2-5 read the finished accumulator with tcgen05.ld (each warp owns
//     one 32-lane quarter of tensor memory = 32 token rows), scale, round to
//     bf16, stage the tile in swizzled shared memory and store it with TMA,
//     while the MMA warp already fills the other accumulator.
//   * For decode-sized T (one 128-row block) the K loop can be split over
//     several CTAs (split-K).  Each writes an fp32 partial; the CTA that
//     finishes a tile last (atomic counter, no waiting) sums the partials in
//     split order, scales and stores.  The reduction order is fixed, so the
//     result does not depend on which CTA finishes last.
//
// Every wait on an mbarrier is bounded (see mbar_wait); a wait that runs out
// sets a bit in the device status word, and the CTA stops issuing work, lets
// its own copies and MMAs drain, frees its tensor memory and exits.
#include <algorithm>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace ptpc {

namespace {

constexpr int BM = 128;      // tokens per tile (MMA M, tensor-memory lanes)
constexpr int BK = 128;      // K bytes per stage (= one 128-byte swizzle row)
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;

struct GemmParams {
  int T, Co;
  int num_m, num_n, num_kb;
  int group_m;
  int nsplit;
  int num_units;
  const float *xs;
  const float *ws;
  void *out;
  uint32_t *status;
  uint32_t *counters;
  float *partials;
};

template <int BN, int STAGES, bool F32OUT>
struct Cfg {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int EPI_COLS = F32OUT ? 32 : 64;     // columns in one 128-byte output row chunk
  static constexpr int EPI_BUF = 32 * 128;              // one warp's staging: 32 rows x 128 bytes
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                   : (2 * BN <= 256) ? 256 : 512;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + kEpiWarps * EPI_BUF +
                                 kEpiWarps * 64 * sizeof(float) + 256;
  static_assert(BN % EPI_COLS == 0, "BN must be a multiple of the epilogue chunk");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void unit_coords(const GemmParams &p, int unit, int &m, int &n, int &kb0, int &kb1,
                                            int &tile, int &split) {
  tile = unit / p.nsplit;
  split = unit - tile * p.nsplit;
  const int per_group = p.group_m * p.num_n;
  const int g = tile / per_group;
  const int first_m = g * p.group_m;
  const int gm = min(p.group_m, p.num_m - first_m);
  const int r = tile - g * per_group;
  m = first_m + r % gm;
  n = r / gm;
  kb0 = (int)(((long long)split * p.num_kb) / p.nsplit);
  kb1 = (int)(((long long)(split + 1) * p.num_kb) / p.nsplit);
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&v);
}

// Fused epilogue of one accumulator: 32 token rows (one TMEM lane quarter,
// lane i = row store_row0 + i) x BN_T columns starting at global column
// col_base.  fp32 -> (acc * x_scale) * w_scale -> bf16 (or the raw fp32
// accumulator), staged as 32 x 128-byte chunks in 128-byte-swizzled shared
// memory and written with TMA stores.  After the last tensor-memory read the
// accumulator buffer is released by one arrival on `release_bar` (a
// shared::cluster address: this CTA's barrier or the pair leader's).
template <int BN_T, bool F32OUT>
__device__ __forceinline__ void epilogue_store_tile(const CUtensorMap *tmC, uint32_t tbase, uint8_t *cbuf,
                                                    float *sc, const GemmParams &p, int col_base,
                                                    int store_row0, float xsr, int lane, uint32_t release_bar) {
  constexpr int EPI_COLS = F32OUT ? 32 : 64;
  #pragma unroll 1
  for (int c0 = 0; c0 < BN_T; c0 += EPI_COLS) {
    uint32_t packed[32];
    if constexpr (F32OUT) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tbase + c0, r);
      tmem_wait_ld();
      #pragma unroll
      for (int j = 0; j < 32; ++j) packed[j] = r[j];
    } else {
      __syncwarp();
      const int col0 = col_base + c0;
      sc[lane] = (col0 + lane < p.Co) ? __ldg(p.ws + col0 + lane) : 0.0f;
      sc[lane + 32] = (col0 + 32 + lane < p.Co) ? __ldg(p.ws + col0 + 32 + lane) : 0.0f;
      uint32_t r0[32], r1[32];
      tmem_ld_32x32b_x32(tbase + c0, r0);
      tmem_ld_32x32b_x32(tbase + c0 + 32, r1);
      tmem_wait_ld();
      __syncwarp();
      #pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float4 wv = *reinterpret_cast<const float4 *>(sc + 4 * j);
        const uint32_t *rr = (j < 8) ? r0 : r1;
        const int b = (j & 7) * 4;
        const float v0 = __fmul_rn(__fmul_rn(__uint_as_float(rr[b + 0]), xsr), wv.x);
        const float v1 = __fmul_rn(__fmul_rn(__uint_as_float(rr[b + 1]), xsr), wv.y);
        const float v2 = __fmul_rn(__fmul_rn(__uint_as_float(rr[b + 2]), xsr), wv.z);
        const float v3 = __fmul_rn(__fmul_rn(__uint_as_float(rr[b + 3]), xsr), wv.w);
        packed[2 * j] = pack_bf16x2(v0, v1);
        packed[2 * j + 1] = pack_bf16x2(v2, v3);
      }
    }
    if (c0 + EPI_COLS >= BN_T) {
      // the whole accumulator has been read: hand it back to the MMA issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(release_bar);
    }
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
      tma_store_2d(tmC, cbuf, col_base + c0, store_row0);
      bulk_commit();
    }
  }
}

template <int BN, int STAGES, bool F32OUT>
__global__ void __launch_bounds__(kThreads, 1)
    ptpc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  using C = Cfg<BN, STAGES, F32OUT>;
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
  int *last_flag = reinterpret_cast<int *>(tmem_holder + 1);
  int *vote = last_flag + 1;  // [kEpiWarps]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

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
      mbar_init(&tempty[b], kEpiWarps);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      const uint64_t polA = policy_evict_last();
      const uint64_t polB = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      griddep_wait();  // Xq may come from the kernel launched just before
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x) {
        int m, n, kb0, kb1, tile, split;
        unit_coords(p, u, m, n, kb0, kb1, tile, split);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * BK, m * BM, polA);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * BK, n * BN, polB);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        atomicOr(p.status, kStatusTimeoutProducer);
        // let the loads already issued land before the CTA can exit
        for (int s = 0; s < STAGES; ++s) mbar_wait(&full[s], s < stage ? phase : phase ^ 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_e4m3_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.num_units && ok; u += gridDim.x, ++local) {
        int m, n, kb0, kb1, tile, split;
        unit_coords(p, u, m, n, kb0, kb1, tile, split);
        const int buf = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[buf], aphase ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * C::B_BYTES));
          #pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_e4m3(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
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
      // every MMA issued above completes before the tensor memory is freed
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // tensor-memory lane quarter = token rows q*32 .. q*32+31
    const int ew = warp - 2;             // staging buffer index
    const int et = threadIdx.x - 64;     // 0..127 within the epilogue warps
    uint8_t *cbuf = sC + ew * C::EPI_BUF;
    float *sc = sScale + ew * 64;
    int local = 0;
    bool ok = true;
    griddep_wait();  // x_scale may come from the kernel launched just before
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x, ++local) {
      int m, n, kb0, kb1, tile, split;
      unit_coords(p, u, m, n, kb0, kb1, tile, split);
      const int buf = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      const int row = m * BM + q * 32 + lane;
      float xsr = 0.0f;
      if (!F32OUT && row < p.T) xsr = __ldg(p.xs + row);
      // The decision to stop must be the same for every lane (tcgen05.ld is
      // warp-collective) and, in split-K mode, for all four epilogue warps
      // (they meet at named barriers below).
      bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], aphase));
      if (p.nsplit > 1) {
        if (lane == 0) vote[ew] = got ? 1 : 0;
        epi_bar();
        got = vote[0] && vote[1] && vote[2] && vote[3];
      }
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);

      if (p.nsplit == 1) {
        // ---- direct: scale, round, stage, TMA store
        epilogue_store_tile<BN, F32OUT>(&tmC, tbase, cbuf, sc, p, n * BN, m * BM + q * 32, xsr, lane,
                                        smem_u32(&tempty[buf]));
      } else {
        // ---- split-K: fp32 partial of this K range, last CTA reduces
        const int prow = p.T;  // split-K runs with a single 128-row block: rows 0..T-1
        float *part = p.partials + ((size_t)tile * p.nsplit + split) * (size_t)prow * BN;
        const bool warp_has_rows = q * 32 < prow;
        if (warp_has_rows) {
          #pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tbase + c0, r);
            tmem_wait_ld();
            if (row < prow) {
              float4 *dst = reinterpret_cast<float4 *>(part + (size_t)row * BN + c0);
              #pragma unroll
              for (int j = 0; j < 8; ++j)
                __stcg(dst + j, make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                                            __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3])));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[buf]);
        __threadfence();
        epi_bar();
        if (et == 0) {
          const uint32_t prev = atomicAdd(p.counters + tile, 1u);
          *last_flag = (prev == (uint32_t)(p.nsplit - 1)) ? 1 : 0;
        }
        epi_bar();
        if (*last_flag) {
          __threadfence();
          const float *base = p.partials + (size_t)tile * p.nsplit * (size_t)prow * BN;
          const int nv = prow * (BN / 4);
          for (int i = et; i < nv; i += 32 * kEpiWarps) {
            const int r = i / (BN / 4);
            const int c = (i - r * (BN / 4)) * 4;
            float4 acc = __ldcg(reinterpret_cast<const float4 *>(base + (size_t)r * BN + c));
            for (int s = 1; s < p.nsplit; ++s) {
              const float4 v = __ldcg(reinterpret_cast<const float4 *>(base + ((size_t)s * prow + r) * BN + c));
              acc.x = __fadd_rn(acc.x, v.x);
              acc.y = __fadd_rn(acc.y, v.y);
              acc.z = __fadd_rn(acc.z, v.z);
              acc.w = __fadd_rn(acc.w, v.w);
            }
            const int col = n * BN + c;
            if (col < p.Co) {  // Co % 16 == 0: the 4 columns are all in range
              if constexpr (F32OUT) {
                *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (size_t)r * p.Co + col) = acc;
              } else {
                const float a = __ldg(p.xs + r);
                const float4 wv = __ldg(reinterpret_cast<const float4 *>(p.ws + col));
                uint2 o;
                o.x = pack_bf16x2(__fmul_rn(__fmul_rn(acc.x, a), wv.x), __fmul_rn(__fmul_rn(acc.y, a), wv.y));
                o.y = pack_bf16x2(__fmul_rn(__fmul_rn(acc.z, a), wv.z), __fmul_rn(__fmul_rn(acc.w, a), wv.w));
                *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) + (size_t)r * p.Co + col) = o;
              }
            }
          }
          if (et == 0) p.counters[tile] = 0u;  // ready for the next call
        }
        epi_bar();
      }
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeoutEpilogue);
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
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
// 32 KB of operands per 128-deep K-block instead of 48 KB for the one-CTA
// 128 x 256 tile, for the same tensor work.
// ----------------------------------------------------------------------------
constexpr int kPairBN = 256;
constexpr int kPairHalfN = 128;

template <int STAGES, bool F32OUT>
struct PairCfg {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = kPairHalfN * BK;
  static constexpr int EPI_BUF = 32 * 128;
  static constexpr int TMEM_COLS = 512;
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + kEpiWarps * EPI_BUF +
                                 kEpiWarps * 64 * sizeof(float) + 256;
  static_assert(SMEM <= 232448, "shared memory");
};

template <int STAGES, bool F32OUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ptpc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  using C = PairCfg<STAGES, F32OUT>;
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
      const uint64_t polA = policy_evict_last();
      const uint64_t polB = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      griddep_wait();
      for (int u = cid; u < p.num_units && ok; u += ncl) {
        int m, n, kb0, kb1, tile, split;
        unit_coords(p, u, m, n, kb0, kb1, tile, split);
        const int a_row = m * (2 * BM) + (int)rank * BM;
        const int b_row = n * kPairBN + (int)rank * kPairHalfN;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            ok = false;
            break;
          }
          const uint32_t lead_full = mapa_shared(&full[stage], 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (C::A_BYTES + C::B_BYTES));
          tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, lead_full, kb * BK, a_row, polA);
          tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, lead_full, kb * BK, b_row, polB);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
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
      constexpr uint32_t idesc = idesc_e4m3_f32(2 * BM, kPairBN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int u = cid; u < p.num_units && ok; u += ncl, ++local) {
        int m, n, kb0, kb1, tile, split;
        unit_coords(p, u, m, n, kb0, kb1, tile, split);
        const int buf = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[buf], aphase ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(buf * kPairBN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_kmajor_desc(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bd = sw128_kmajor_desc(smem_u32(sB + stage * C::B_BYTES));
          #pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            mma_e4m3_pair(d, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                          (kb > kb0 || kk > 0) ? 1u : 0u);
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
    uint8_t *cbuf = sC + ew * C::EPI_BUF;
    float *sc = sScale + ew * 64;
    int local = 0;
    bool ok = true;
    griddep_wait();
    for (int u = cid; u < p.num_units; u += ncl, ++local) {
      int m, n, kb0, kb1, tile, split;
      unit_coords(p, u, m, n, kb0, kb1, tile, split);
      const int buf = local & 1;
      const uint32_t aphase = (local >> 1) & 1;
      const int row0 = m * (2 * BM) + (int)rank * BM + q * 32;
      const int row = row0 + lane;
      float xsr = 0.0f;
      if (!F32OUT && row < p.T) xsr = __ldg(p.xs + row);
      const bool got = __all_sync(0xffffffffu, mbar_wait(&tfull[buf], aphase));
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * kPairBN);
      epilogue_store_tile<kPairBN, F32OUT>(&tmC, tbase, cbuf, sc, p, n * kPairBN, row0, xsr, lane,
                                           mapa_shared(&tempty[buf], 0));
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeoutEpilogue);
    if (lane == 0) bulk_wait<0>();
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

bool make_map_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool F32OUT>
cudaError_t launch_cfg(const GemmProblem &pr, const GemmParams &gp, int grid, cudaStream_t st) {
  using C = Cfg<BN, STAGES, F32OUT>;
  auto kernel = ptpc_gemm_kernel<BN, STAGES, F32OUT>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_done[dev] = true;
  }
  CUtensorMap tmA, tmB, tmC;
  if (!make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Xq, pr.Ci, pr.T, pr.Ci, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Wq_t, pr.Ci, pr.Co, pr.Ci, BK, BN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool okC;
  if (F32OUT)
    okC = make_map_2d(&tmC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 4, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  else
    okC = make_map_2d(&tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 2, 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (!okC) return cudaErrorInvalidValue;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pr.pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmC, gp);
}

template <int STAGES, bool F32OUT>
cudaError_t launch_pair(const GemmProblem &pr, GemmParams gp, cudaStream_t st) {
  using C = PairCfg<STAGES, F32OUT>;
  auto kernel = ptpc_gemm_pair_kernel<STAGES, F32OUT>;
  static bool attr_done[64] = {};
  static int max_clusters[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const bool cache = dev >= 0 && dev < 64;
  if (!cache || !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * 74);
    q.blockDim = dim3(kThreads);
    q.dynamicSmemBytes = C::SMEM;
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, kernel, &q) != cudaSuccess || ncl <= 0) {
      cudaGetLastError();
      ncl = num_sms() / 2;
    }
    if (cache) {
      max_clusters[dev] = ncl;
      attr_done[dev] = true;
    } else {
      max_clusters[0] = ncl;
    }
  }
  const int ncl = std::max(1, std::min(gp.num_units, cache ? max_clusters[dev] : max_clusters[0]));
  CUtensorMap tmA, tmB, tmC;
  if (!make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Xq, pr.Ci, pr.T, pr.Ci, BK, BM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, pr.Wq_t, pr.Ci, pr.Co, pr.Ci, BK, kPairHalfN,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  bool okC;
  if (F32OUT)
    okC = make_map_2d(&tmC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 4, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  else
    okC = make_map_2d(&tmC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pr.out, pr.Co, pr.T, (uint64_t)pr.Co * 2, 64, 32,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (!okC) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * ncl);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pr.pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmC, gp);
}

struct Plan {
  int bn;
  int nsplit;
};

// Split-K only for a single 128-row block (decode-sized T): enough work units
// to keep the SMs streaming weights, bounded partial-sum traffic.
Plan choose_plan(int T, int Ci, int Co) {
  Plan pl{256, 1};
  const int sms = num_sms();
  const int num_kb = (Ci + BK - 1) / BK;
  if (T <= BM) {
    pl.bn = 128;
    const int tiles = (Co + pl.bn - 1) / pl.bn;
    int best = 1;
    for (int s = 1; s <= 16 && s <= num_kb / 2; ++s) {
      // partial traffic (write + read) relative to the weight bytes of a tile
      const double extra = (s > 1) ? (2.0 * s * T * 4.0) / (double)Ci : 0.0;
      if (extra > 0.15) break;
      best = s;
      if (tiles * s >= sms) break;
    }
    pl.nsplit = best;
  }
  return pl;
}

}  // namespace

int num_sms() {
  static int n = []() {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

void gemm_workspace_needs(int T, int Ci, int Co, size_t *counter_words, size_t *partial_floats) {
  const Plan pl = choose_plan(T, Ci, Co);
  const size_t tiles = (size_t)((T + BM - 1) / BM) * (size_t)((Co + pl.bn - 1) / pl.bn);
  *counter_words = tiles;
  *partial_floats = pl.nsplit > 1 ? tiles * pl.nsplit * (size_t)T * pl.bn : 0;
}

cudaError_t launch_scaled_gemm(const GemmProblem &pr, cudaStream_t st) {
  const Plan pl = choose_plan(pr.T, pr.Ci, pr.Co);
  GemmParams gp = {};
  gp.T = pr.T;
  gp.Co = pr.Co;
  gp.num_m = (pr.T + BM - 1) / BM;
  gp.num_n = (pr.Co + pl.bn - 1) / pl.bn;
  gp.num_kb = (pr.Ci + BK - 1) / BK;
  gp.group_m = 16;
  gp.nsplit = pl.nsplit;
  gp.num_units = gp.num_m * gp.num_n * gp.nsplit;
  gp.xs = pr.xs;
  gp.ws = pr.ws;
  gp.out = pr.out;
  gp.status = pr.status;
  gp.counters = pr.counters;
  gp.partials = pr.partials;
  if (pl.nsplit > 1 && pr.partial_floats < (size_t)gp.num_n * pl.nsplit * (size_t)pr.T * pl.bn)
    return cudaErrorInvalidValue;
  if (pr.T > BM && pl.nsplit == 1) {
    // CTA-pair 256 x 256 tiles
    gp.num_m = (pr.T + 2 * BM - 1) / (2 * BM);
    gp.num_n = (pr.Co + kPairBN - 1) / kPairBN;
    gp.group_m = 8;
    gp.num_units = gp.num_m * gp.num_n;
    return pr.f32_out ? launch_pair<6, true>(pr, gp, st) : launch_pair<6, false>(pr, gp, st);
  }
  const int grid = std::min(gp.num_units, num_sms());
  if (pl.bn == 256) {
    return pr.f32_out ? launch_cfg<256, 4, true>(pr, gp, grid, st) : launch_cfg<256, 4, false>(pr, gp, grid, st);
  }
  return pr.f32_out ? launch_cfg<128, 6, true>(pr, gp, grid, st) : launch_cfg<128, 6, false>(pr, gp, grid, st);
}

}  // namespace ptpc
