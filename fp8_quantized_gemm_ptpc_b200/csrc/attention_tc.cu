// Decode attention over the FP8 (E4M3) paged KV cache on the fifth-generation
// tensor cores (tcgen05), for head size 128, GQA groups of up to 16 query
// heads and cache blocks of a multiple of 8 positions.  Same arguments and
// results as the warp-level kernel in attention.cu (which takes every other
// shape); same cache layout:
//   codes  cache[(slot * Hkv + g) * D + d],  scale  scales[slot * Hkv + g].
//
// A CTA takes one (sequence, KV head, group of at most 8 of the KV head's
// query heads — a group of 9 to 16 takes two CTAs, which read the same
// tiles, the second mostly from L2) and a chunk of context positions, in
// tiles of 128 positions.  Warp 0 loads a tile's K and V codes with TMA (a
// 3-D tensor map over [slot][head][d], boxes of 16 positions, or 8 where the
// cache blocks hold an odd multiple of 8, into 128-byte swizzled tiles, one
// box a lane) into two rings of stages, one for K (a stage is free again once
// the tile's QK MMAs are done) and one for V (free once its PV MMAs are
// done), so neither ring waits for the other half's work.  It issues nothing
// else and runs as far ahead as the rings allow (a TMA instruction takes tens
// of cycles to issue whatever its box, hence the largest box a block allows).
// Warp 1 issues the MMAs from one thread:
//   S^T = K Q^T    (M = 128 positions, N = 16, K = d; A = the K tile, B = q)
//   O^T += V^T P^T (M = 128 values of d, N = 2 x 16, K = positions; A = the
//                   V tile read as an MN-major operand, B = P, MN-major)
// all kind::f8f6f4 E4M3 x E4M3 with fp32 accumulators in tensor memory.  q
// enters as two E4M3 terms (q = t1 + t2 / 16 after a power-of-two scale: 8
// significant bits, exact for a bf16 value of at least E4M3's smallest normal,
// 2^-6, after the scale; within 2^-14 below it) and
// P as three (P = t1 + t2 / 16 + t3 / 256: about 12 significant bits, like
// f16); the N columns hold term 1 of the group's 8 heads, then term 2 (and,
// for P, term 3 in a second MMA), so the terms share the MMAs.  The cache
// codes go in as they are, with no conversion.
// Warps 2-5 (thread i = tensor-memory lane i = position i of the tile, and
// value d = i of O; each loads its position's two scales two tiles ahead)
// run the online softmax in base 2: key scales, masking, exponentials, P
// written to shared memory.  The running maximum and the value-scale unit are
// lazy: a reference maximum per head moves (and O, in tensor memory, is
// rescaled) only when a score exceeds it by more than 8 (base-2 units), and
// then to 4 below the tile's maximum; the unit (a power of two) moves only
// when a value scale exceeds it.  So P stays below 2^8 (E4M3 holds 448), its
// largest values sit far above the smallest step its three E4M3 terms can
// express even when the value scales spread widely, and the common tile needs
// one barrier and no reduction.  S has two tensor-memory buffers, so the MMAs
// of tile i+1 run while the softmax works on tile i.  At the end the CTA
// writes (max, sum, accumulator) of its chunk for the combine kernel of
// attention.cu, or, when one chunk covers every context, the output itself.
// Every wait is bounded; a timeout sets a bit in the status word at the front
// of the workspace and the CTA stops (after letting its copies and MMAs
// finish).
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <mutex>

#include "attention_tc.h"
#include "sm100.cuh"

namespace ptpc {

namespace {

constexpr int kTcThreads = 192;  // warp 0 producer, warp 1 MMA issuer, warps 2-5 softmax
constexpr int kTcStages = 3;     // stages of each ring
constexpr int kTcTile = 128;     // positions a tile
constexpr int kTcD = 128;
constexpr int kTcKV = kTcTile * kTcD;  // bytes of one K or V tile
constexpr uint32_t kTcTmemCols = 64;   // S: 2 buffers x 16 columns at 0; O: 2 x 16 columns at 32
constexpr uint32_t kTcColO = 32;
constexpr uint32_t kStatusTimeoutAttn = 1u << 3;
constexpr float kRefLazy = 8.0f;    // a head's reference maximum moves when a score exceeds it by this
constexpr float kRefBelow = 4.0f;   // ... and then to this below the tile's maximum
constexpr int kTcMaxChunk = 4096;   // positions a CTA at most

struct TcParams {
  const __nv_bfloat16 *q;       // [B, Hq, D]
  const float *ks, *vs;         // [num_slots, Hkv]
  const int32_t *block_tables;  // [B, max_blocks]
  const int32_t *context_lens;  // [B]
  int Hq, Hkv, G, block_size, max_blocks, splits, chunk;
  int hgroups;                  // CTAs a KV head (query heads 8 a CTA)
  int box_rows;                 // positions a TMA box: 16, or 8 (a divisor of block_size)
  uint64_t bs_magic;            // ceil(2^64 / block_size)
  int64_t num_slots;
  float scale_log2;
  float *part_ml, *part_acc;
  __nv_bfloat16 *out;           // [B, Hq, D] when splits == 1 (no combine), else null
  uint32_t *status;
};

// Shared memory (from a 1024-byte aligned base).
struct TcSmem {
  static constexpr int K = 0;                                    // [stage] 16 KB
  static constexpr int V = K + kTcStages * kTcKV;                // [stage] 16 KB
  static constexpr int Q = V + kTcStages * kTcKV;                // 16 rows x 128 B: hi terms, then lo terms
  static constexpr int P = Q + 16 * 128;                         // [plane] 128 positions x 16 B
  static constexpr int P_PLANE = kTcTile * 16;                   // plane 0: terms 1, 2; plane 1: term 3, zeros
  static constexpr int RED = P + 2 * P_PLANE;                    // [warp][16]: per-warp maxima, sums
  static constexpr int SIG = RED + 4 * 16 * 4;                   // [head]: 1 / sigma of q
  static constexpr int BLK = SIG + 16 * 4;
  // then the chunk's block-table entries (size depends on the chunk), then
  // the barriers and the tensor-memory address
  static constexpr int kBarriers = 4 * kTcStages + 3 * 2 + 2;
};

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *m, uint64_t *bar, int32_t x, int32_t y,
                                            int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Non-blocking test of a phase (no suspension, unlike try_wait).
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Descriptor of an MN-major operand tile with the 128-byte swizzle: 128-byte
// rows along M (one swizzle atom wide: M = 128 bytes), 8-row atoms along K
// 1024 bytes apart.  Both byte offsets are 1024: the one between atoms along
// M is not used for a single atom.
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)(1024u >> 4) << 16;         // leading-dimension byte offset
  d |= (uint64_t)(1024u >> 4) << 32;         // stride-dimension byte offset: next 8 rows of K
  d |= (uint64_t)1 << 46;                    // descriptor version (tcgen05)
  d |= (uint64_t)2 << 61;                    // layout: 128-byte swizzle
  return d;
}

// Descriptor of an MN-major operand tile without swizzle whose N extent is
// 16 bytes: rows of 16 bytes, one per K index, 8-row core matrices 128 bytes
// apart.  Both byte offsets are 128: the one between 16-byte groups along N
// is not used for a single group.
__device__ __forceinline__ uint64_t plain_mnmajor16_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(128u >> 4) << 16;
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;  // layout 0: no swizzle
}

// Byte (row, col) of a 128-byte-swizzled tile with 128-byte rows.
__device__ __forceinline__ int sw128_off(int row, int col) {
  return row * 128 + ((((col >> 4) ^ (row & 7)) & 7) << 4) + (col & 15);
}

__device__ __forceinline__ uint32_t f32x2_e4m3x2(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float2 e4m3x2_f32x2(uint32_t two) {
  const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2 *>(&r));
}

// Barriers of the 128 softmax threads (warps 2-5).
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ int softmax_bar_count(bool v) {
  int n;
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.popc.u32 %0, 1, 128, q;\n\t}"
      : "=r"(n)
      : "r"((uint32_t)v)
      : "memory");
  return n;
}
__device__ __forceinline__ bool softmax_bar_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.and.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__global__ void __launch_bounds__(kTcThreads, 2)
    decode_attn_tc_kernel(const TcParams p, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const int nblk_max = p.chunk / 8 + 2;
  int *s_blk = reinterpret_cast<int *>(sm + TcSmem::BLK);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + ((TcSmem::BLK + nblk_max * 4 + 7) & ~7));
  uint64_t *k_full = bars;                    // [stage]: the tile's K bytes have landed
  uint64_t *k_empty = k_full + kTcStages;     // [stage]: the tile's QK MMAs are done
  uint64_t *v_full = k_empty + kTcStages;     // [stage]: the tile's V bytes have landed
  uint64_t *v_empty = v_full + kTcStages;     // [stage]: the tile's PV MMAs are done
  uint64_t *s_full = v_empty + kTcStages;     // [buffer]: S of a tile is in tensor memory
  uint64_t *s_empty = s_full + 2;             // [buffer]: the softmax has read it (128)
  uint64_t *p_full = s_empty + 2;             // [tile parity]: P written, O corrected (128)
  uint64_t *o_done = p_full + 2;              // one phase per PV
  uint64_t *drain = o_done + 1;               // the MMA issuer's last commit
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);

  const int split = blockIdx.x, kvh = blockIdx.y / p.hgroups, b = blockIdx.z;
  // this CTA's query heads: kvh * G + h0 + h, h < GC
  const int h0 = (blockIdx.y - kvh * p.hgroups) * 8;
  const int GC = min(8, p.G - h0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Independent loads, issued together: this thread's part of its head's
  // query (softmax warps), the context length and the block-table entries a
  // whole chunk spans (-1 past the table; entries past the context are never
  // read, positions there being rejected first).
  const int tq = threadIdx.x - 64;  // softmax thread 0..127: head tq / 16, values 8 (tq % 16) ..
  uint4 qw = make_uint4(0u, 0u, 0u, 0u);
  if (warp >= 2 && (tq >> 4) < GC)
    qw = *reinterpret_cast<const uint4 *>(p.q + ((int64_t)b * p.Hq + (int64_t)kvh * p.G + h0 + (tq >> 4)) * kTcD +
                                          (tq & 15) * 8);
  const int L = __ldg(p.context_lens + b);
  const int c0 = split * p.chunk;
  const int bi0 = (int)__umul64hi((uint64_t)c0, p.bs_magic);
  const int nbi = (int)__umul64hi((uint64_t)(c0 + p.chunk - 1), p.bs_magic) - bi0 + 1;  // <= chunk / 8 + 2
  for (int i = threadIdx.x; i < nbi; i += kTcThreads) {
    const int bi = bi0 + i;
    s_blk[i] = bi < p.max_blocks ? __ldg(p.block_tables + (int64_t)b * p.max_blocks + bi) : -1;
  }
  const int c1 = min(c0 + p.chunk, L);
  const int ntiles = c1 > c0 ? (c1 - c0 + kTcTile - 1) / kTcTile : 0;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 128);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTcTmemCols);
    tmem_relinquish();
  }
  // slot of position pos (-1: not read).  A block holds a multiple of
  // box_rows positions and tiles start at multiples of 128, so the positions
  // of a TMA box share one block: the box is read whole or not at all.
  auto slot_of = [&](int pos) -> int64_t {
    if (pos >= c1) return -1;
    const int bi = (int)__umul64hi((uint64_t)pos, p.bs_magic);
    const int blk = s_blk[bi - bi0];
    const int64_t sl = (int64_t)blk * p.block_size + (pos - bi * p.block_size);
    return (blk < 0 || sl >= p.num_slots) ? -1 : sl;
  };

  // softmax warps: q as two E4M3 terms (rows 0..7 = first terms of the heads,
  // rows 8..15 = second terms), 1 / sigma of each head into shared memory
  if (warp >= 2) {
    const int t = tq;  // 0..127
    const int h = t >> 4, d0 = (t & 15) * 8;
    float x[8];
    float amax = 0.0f;
    if (h < GC) {
      const uint32_t ww[4] = {qw.x, qw.y, qw.z, qw.w};
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ww[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
        amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    } else {
      #pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = 0.0f;
    }
    #pragma unroll
    for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    // sigma: a power of two that brings the largest |q| of the head to
    // [224, 448], at most 2^126 so that 1 / sigma stays a normal number
    const float sig = amax > 0.0f ? fminf(__uint_as_float(__float_as_uint(448.0f / amax) & 0x7F800000u),
                                          __uint_as_float(253u << 23))
                                  : 1.0f;
    if ((t & 15) == 0) reinterpret_cast<float *>(sm + TcSmem::SIG)[h] = 1.0f / sig;
    uint8_t *qs = sm + TcSmem::Q;
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = x[2 * i] * sig, c = x[2 * i + 1] * sig;
      const uint32_t hi = f32x2_e4m3x2(a, c);
      const float2 dh = e4m3x2_f32x2(hi);
      const uint32_t lo = f32x2_e4m3x2((a - dh.x) * 16.0f, (c - dh.y) * 16.0f);
      const int col = d0 + 2 * i;
      qs[sw128_off(h, col)] = (uint8_t)(hi & 0xFF);
      qs[sw128_off(h, col + 1)] = (uint8_t)(hi >> 8);
      qs[sw128_off(h + 8, col)] = (uint8_t)(lo & 0xFF);
      qs[sw128_off(h + 8, col + 1)] = (uint8_t)(lo >> 8);
    }
    // the V ring starts zeroed: rows of boxes that are never loaded then hold
    // zeros or an earlier tile's codes (finite), which P = 0 cancels
    uint4 *vz = reinterpret_cast<uint4 *>(sm + TcSmem::V);
    for (int j = t; j < kTcStages * kTcKV / 16; j += 128) vz[j] = make_uint4(0, 0, 0, 0);
    fence_async_shared();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Decisions are warp-uniform: a stage is refilled by all 32 lanes or none.
    // Order: K of tile j + 1, then V of tile j, the order in which the MMAs
    // free their stages (QK(j - 2) before PV(j - 3)).
    const int nbox = kTcTile / p.box_rows;
    const uint32_t box_bytes = (uint32_t)(p.box_rows * kTcD);
    bool ok = true;
    int k_issued = 0, v_issued = 0;
    // issue one half (K or V) of tile i into its ring
    auto issue = [&](int i, bool is_k) -> bool {
      const int s = i % kTcStages;
      uint64_t *full = is_k ? &k_full[s] : &v_full[s];
      if (i >= kTcStages) {
        uint64_t *empty = is_k ? &k_empty[s] : &v_empty[s];
        const bool w = mbar_wait(empty, (uint32_t)((i / kTcStages) - 1) & 1u);
        if (!__all_sync(0xffffffffu, w)) return false;
      }
      // box j loaded by lane j; a box that is not read leaves its rows as they
      // were.  The barrier's byte count is set before any copy is issued.
      const int64_t s0 = lane < nbox ? slot_of(c0 + i * kTcTile + p.box_rows * lane) : -1;
      const uint32_t boxes = __ballot_sync(0xffffffffu, s0 >= 0);
      if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)__popc(boxes) * box_bytes);
      __syncwarp();
      if (s0 >= 0)
        tma_load_3d(sm + (is_k ? TcSmem::K : TcSmem::V) + s * kTcKV + lane * (int)box_bytes, is_k ? &tmK : &tmV, full,
                    0, kvh, (int)s0);
      return true;
    };
    if (ntiles > 0) {
      ok = issue(0, true);
      k_issued = ok ? 1 : 0;
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      if (j + 1 < ntiles) {
        ok = issue(j + 1, true);
        if (!ok) break;
        k_issued = j + 2;
      }
      ok = issue(j, false);
      if (ok) v_issued = j + 1;
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeoutAttn);
    // every copy this warp issued completes before the CTA ends (bounded)
    if (lane == 0) {
      for (int i = std::max(0, k_issued - kTcStages); i < k_issued; ++i)
        mbar_wait(&k_full[i % kTcStages], (uint32_t)(i / kTcStages) & 1u);
      for (int i = std::max(0, v_issued - kTcStages); i < v_issued; ++i)
        mbar_wait(&v_full[i % kTcStages], (uint32_t)(i / kTcStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_f8f6f4_f32(128, 16, kMmaE4M3, kMmaE4M3);
      constexpr uint32_t idesc_pv = idesc_f8f6f4_f32(128, 16, kMmaE4M3, kMmaE4M3) | (1u << 15) | (1u << 16);
      const uint64_t qd = sw128_kmajor_desc(smem_u32(sm + TcSmem::Q));
      bool ok = true;
      auto qk = [&](int i) {
        const int s = i % kTcStages, bufi = i & 1;
        if (!mbar_wait(&k_full[s], (uint32_t)(i / kTcStages) & 1u)) return false;
        if (i >= 2 && !mbar_wait(&s_empty[bufi], (uint32_t)((i >> 1) - 1) & 1u)) return false;
        tc_fence_after();
        const uint64_t ad = sw128_kmajor_desc(smem_u32(sm + TcSmem::K + s * kTcKV));
        const uint32_t d = tmem_base + (uint32_t)(bufi * 16);
        #pragma unroll
        for (int kk = 0; kk < kTcD / 32; ++kk) mma_f8f6f4(d, ad + 2 * kk, qd + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
        mma_commit(&s_full[bufi]);
        mma_commit(&k_empty[s]);
        return true;
      };
      auto pv = [&](int i) {
        const int s = i % kTcStages, bufi = i & 1;
        if (!mbar_wait(&v_full[s], (uint32_t)(i / kTcStages) & 1u)) return false;
        if (!mbar_wait(&p_full[bufi], (uint32_t)(i >> 1) & 1u)) return false;
        tc_fence_after();
        const uint32_t pb = smem_u32(sm + TcSmem::P);
        const uint32_t vb = smem_u32(sm + TcSmem::V + s * kTcKV);
        #pragma unroll
        for (int kk = 0; kk < kTcTile / 32; ++kk) {
          const uint64_t ad = sw128_mnmajor_desc(vb + kk * 32 * 128);
          const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
          mma_f8f6f4(tmem_base + kTcColO, ad, plain_mnmajor16_desc(pb + kk * 32 * 16), idesc_pv, acc);
          mma_f8f6f4(tmem_base + kTcColO + 16, ad, plain_mnmajor16_desc(pb + TcSmem::P_PLANE + kk * 32 * 16), idesc_pv,
                     acc);
        }
        mma_commit(&v_empty[s]);
        mma_commit(o_done);
        return true;
      };
      // S of tile i + 1 is computed while the softmax works on tile i, but
      // PV of tile i does not wait for tile i + 1's K codes: QK(i + 1) goes
      // first only if they have landed.
      if (ntiles > 0) ok = qk(0);
      for (int i = 0; i < ntiles && ok; ++i) {
        const bool next = i + 1 < ntiles;
        if (next && mbar_test(&k_full[(i + 1) % kTcStages], (uint32_t)((i + 1) / kTcStages) & 1u)) {
          ok = qk(i + 1) && pv(i);
        } else {
          ok = pv(i);
          if (ok && next) ok = qk(i + 1);
        }
      }
      if (!ok) atomicOr(p.status, kStatusTimeoutAttn);
      // every MMA issued has completed before the CTA ends
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int pidx = q4 * 32 + lane;  // position in the tile; also the value d of O this lane holds
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    float *red = reinterpret_cast<float *>(sm + TcSmem::RED);
    float inv_sig[8];
    #pragma unroll
    for (int h = 0; h < 8; ++h) inv_sig[h] = reinterpret_cast<const float *>(sm + TcSmem::SIG)[h];

    float m[8], l[8];
    #pragma unroll
    for (int h = 0; h < 8; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.0f;
    }
    float unit = 0.0f;  // power of two >= every value scale seen (0: none yet)
    bool ok = true;     // this thread's waits; the loop leaves only on a decision all 128 take
    // this position's key and value scales, loaded two tiles ahead (0 where
    // the position is not read)
    auto load_scales = [&](int i, float &k, float &v) {
      const int64_t sl = i < ntiles ? slot_of(c0 + i * kTcTile + pidx) : -1;
      k = sl >= 0 ? __ldg(p.ks + sl * p.Hkv + kvh) : 0.0f;
      v = sl >= 0 ? __ldg(p.vs + sl * p.Hkv + kvh) : 0.0f;
    };
    // one tile; false when the 128 threads stop together.  The tile's scales
    // kr, vr were loaded two tiles earlier: two tiles a loop turn, each with
    // its own registers, reloaded only after use, so no register copy waits
    // for a load in flight.
    auto tile_step = [&](int i, const float kr, const float vr) __attribute__((always_inline)) -> bool {
      const int s = i % kTcStages, bufi = i & 1;
      const int pos = c0 + i * kTcTile + pidx;
      bool w = mbar_wait(&s_full[bufi], (uint32_t)(i >> 1) & 1u);
      tc_fence_after();
      uint32_t r[16];
      tmem_ld_32x32b_x16(tmem_base + lane_addr + (uint32_t)(bufi * 16), r);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_empty[bufi]);
      ok = ok && w;
      const bool valid = slot_of(pos) >= 0;
      const float ksc = kr * p.scale_log2;
      const float vsc = valid ? vr : 0.0f;
      float sv[8];
      bool need = vsc > unit;
      #pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float sc = fmaf(__uint_as_float(r[8 + h]), 0.0625f, __uint_as_float(r[h]));
        sv[h] = (valid && h < GC) ? sc * (ksc * inv_sig[h]) : -INFINITY;
        need = need || sv[h] > m[h] + kRefLazy;
      }
      // one barrier a tile: does any thread need the maxima, or has any wait
      // run out?
      float fac_o[8];
      bool corr = false;
      if (softmax_bar_count(need || !ok) != 0) {
        if (!softmax_bar_all(ok)) return false;
        // the tile's maximum per head and its largest value scale
        float tm[9];
        #pragma unroll
        for (int h = 0; h < 8; ++h) tm[h] = warp_max(sv[h]);
        tm[8] = warp_max(vsc);
        if (lane == 0) {
          #pragma unroll
          for (int h = 0; h < 9; ++h) red[q4 * 16 + h] = tm[h];
        }
        softmax_bar();
        #pragma unroll
        for (int h = 0; h < 9; ++h) tm[h] = fmaxf(fmaxf(red[h], red[16 + h]), fmaxf(red[32 + h], red[48 + h]));
        softmax_bar();  // red is reused
        // a head's reference maximum moves only when the tile's exceeds it
        // by kRefLazy (then to kRefBelow under the tile's maximum); the unit
        // only when a value scale exceeds it (then to the next power of two)
        float ufac = 1.0f;
        if (tm[8] > unit) {
          const float nu = __uint_as_float((__float_as_uint(tm[8]) + 0x007FFFFFu) & 0x7F800000u);
          if (unit > 0.0f) ufac = unit / nu;
          unit = nu;
        }
        corr = ufac != 1.0f;
        #pragma unroll
        for (int h = 0; h < 8; ++h) {
          float f = 1.0f;
          if (tm[h] > m[h] + kRefLazy) {
            const float mn = tm[h] - kRefBelow;
            if (m[h] != -INFINITY) f = exp2f(m[h] - mn);
            m[h] = mn;
          }
          corr = corr || f != 1.0f;
          fac_o[h] = f * ufac;
          l[h] *= f;
        }
      }
      const float inv_unit = unit > 0.0f ? 1.0f / unit : 0.0f;
      // P of this lane's position as three E4M3 terms: plane 0 holds terms 1
      // and 2 of heads 0..7, plane 1 term 3 (then zeros)
      float pv[8];
      #pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float e = m[h] == -INFINITY ? 0.0f : exp2f(sv[h] - m[h]);
        l[h] += e;
        pv[h] = e * vsc * inv_unit;
      }
      uint32_t w1[4], w2[4], w3[4];
      #pragma unroll
      for (int h = 0; h < 8; h += 2) {
        w1[h / 2] = f32x2_e4m3x2(pv[h], pv[h + 1]);
        const float2 d1 = e4m3x2_f32x2(w1[h / 2]);
        const float r0 = (pv[h] - d1.x) * 16.0f, r1 = (pv[h + 1] - d1.y) * 16.0f;
        w2[h / 2] = f32x2_e4m3x2(r0, r1);
        const float2 d2 = e4m3x2_f32x2(w2[h / 2]);
        w3[h / 2] = f32x2_e4m3x2((r0 - d2.x) * 16.0f, (r1 - d2.y) * 16.0f);
      }
      // PV of tile i - 1 has completed: O holds tiles 0 .. i-1 (it may be
      // corrected) and the P buffer (one, in shared memory) is free again.
      // (PV of tile i cannot start before this tile's P, so o_done is never
      // two phases ahead of this wait.)
      if (i >= 1) {
        ok = ok && mbar_wait(o_done, (uint32_t)(i - 1) & 1u);
        tc_fence_after();
      }
      if (corr && i > 0 && ok) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tmem_base + lane_addr + kTcColO, o);
        tmem_wait_ld();
        #pragma unroll
        for (int h = 0; h < 8; ++h) {
          o[h] = __float_as_uint(__uint_as_float(o[h]) * fac_o[h]);
          o[8 + h] = __float_as_uint(__uint_as_float(o[8 + h]) * fac_o[h]);
          o[16 + h] = __float_as_uint(__uint_as_float(o[16 + h]) * fac_o[h]);
        }
        tmem_st_32x32b_x32(tmem_base + lane_addr + kTcColO, o);
        tmem_wait_st();
      }
      tc_fence_before();
      uint8_t *prow = sm + TcSmem::P + pidx * 16;
      *reinterpret_cast<uint4 *>(prow) =
          make_uint4(w1[0] | (w1[1] << 16), w1[2] | (w1[3] << 16), w2[0] | (w2[1] << 16), w2[2] | (w2[3] << 16));
      *reinterpret_cast<uint4 *>(prow + TcSmem::P_PLANE) = make_uint4(w3[0] | (w3[1] << 16), w3[2] | (w3[3] << 16), 0u, 0u);
      // the last box of a context that ends inside it is loaded whole: its
      // rows past the context hold whatever the cache holds there (maybe
      // NaN codes), so they are zeroed once the box has landed (P = 0 times
      // them must be 0).  Every other row that is not read holds zeros or an
      // earlier tile's codes.
      if (i == ntiles - 1 && c1 % p.box_rows != 0) {
        ok = ok && mbar_wait(&v_full[s], (uint32_t)(i / kTcStages) & 1u);
        if (pos >= c1 && pos < (c1 / p.box_rows + 1) * p.box_rows) {
          uint4 *vrow = reinterpret_cast<uint4 *>(sm + TcSmem::V + s * kTcKV + pidx * 128);
          #pragma unroll
          for (int c = 0; c < 8; ++c) vrow[c] = make_uint4(0, 0, 0, 0);
        }
      }
      fence_async_shared();
      mbar_arrive(&p_full[bufi]);
      return true;
    };
    float k0, v0, k1, v1;
    load_scales(0, k0, v0);
    load_scales(1, k1, v1);
    #pragma unroll 1
    for (int i = 0; i < ntiles; i += 2) {
      const float ka = k0, va = v0;
      load_scales(i + 2, k0, v0);
      if (!tile_step(i, ka, va)) break;
      const float kb = k1, vb = v1;
      load_scales(i + 3, k1, v1);
      if (i + 1 < ntiles && !tile_step(i + 1, kb, vb)) break;
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeoutAttn);
    // the last PV, then O, the sums and the maxima of the chunk
    float o_out[8];
    #pragma unroll
    for (int h = 0; h < 8; ++h) o_out[h] = 0.0f;
    if (ok && ntiles > 0) {
      if (mbar_wait(o_done, (uint32_t)(ntiles - 1) & 1u)) {
        tc_fence_after();
        uint32_t o[32];
        tmem_ld_32x32b_x32(tmem_base + lane_addr + kTcColO, o);
        tmem_wait_ld();
        #pragma unroll
        for (int h = 0; h < 8; ++h)
          o_out[h] = fmaf(fmaf(__uint_as_float(o[16 + h]), 0.0625f, __uint_as_float(o[8 + h])), 0.0625f,
                          __uint_as_float(o[h])) * unit;
      } else if (lane == 0) {
        atomicOr(p.status, kStatusTimeoutAttn);
      }
    }
    // l: sum over the 128 positions' partial sums
    #pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      #pragma unroll
      for (int h = 0; h < 8; ++h) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
    }
    softmax_bar();  // red may still be read by a thread of the last tile
    if (lane == 0) {
      #pragma unroll
      for (int h = 0; h < 8; ++h) red[q4 * 16 + h] = l[h];
    }
    softmax_bar();
    #pragma unroll
    for (int h = 0; h < 8; ++h) {
      if (h >= GC) break;
      const int64_t idx = (((int64_t)b * p.Hq + (int64_t)kvh * p.G + h0 + h) * p.splits + split);
      const float lsum = red[h] + red[16 + h] + red[32 + h] + red[48 + h];
      if (p.out != nullptr) {
        // one chunk covers the context: the combine kernel's arithmetic for
        // a single chunk (o / l, rounded once), written here
        const int64_t oh = (int64_t)b * p.Hq + (int64_t)kvh * p.G + h0 + h;
        p.out[oh * kTcD + pidx] = __float2bfloat16_rn(lsum > 0.0f ? o_out[h] / lsum : 0.0f);
        continue;
      }
      p.part_acc[idx * kTcD + pidx] = o_out[h];
      if (pidx == 0) {
        p.part_ml[idx * 2] = ntiles > 0 ? m[h] : -INFINITY;
        p.part_ml[idx * 2 + 1] = lsum;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
}

// Dynamic shared memory of a CTA for a chunk of `chunk` positions.
size_t tc_smem_bytes(int chunk) {
  return 1024 + (size_t)TcSmem::BLK + (size_t)(chunk / 8 + 2) * 4 + 8 + TcSmem::kBarriers * 8 + 16;
}

typedef CUresult (*TcEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                               const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

TcEncodeFn tc_encode_fn() {
  static TcEncodeFn fn = []() -> TcEncodeFn {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<TcEncodeFn>(ptr);
  }();
  return fn;
}

// 3-D map of a cache [slots][Hkv][128] of bytes: boxes of 128 bytes x 1 head x
// 8 slots, 128-byte swizzle.  Cached for the last few caches (a decode step
// calls the kernel once a layer on the same caches).
bool tc_cache_map(CUtensorMap *m, const void *base, int Hkv, int64_t slots, int box_rows) {
  struct Entry {
    const void *base;
    int Hkv;
    int64_t slots;
    int box_rows;
    CUtensorMap map;
  };
  static std::mutex mu;
  static Entry cache[16];
  static int next = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry &e : cache)
    if (e.base == base && e.Hkv == Hkv && e.slots == slots && e.box_rows == box_rows) {
      *m = e.map;
      return true;
    }
  TcEncodeFn fn = tc_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kTcD, (cuuint64_t)Hkv, (cuuint64_t)slots};
  cuuint64_t strides[2] = {(cuuint64_t)kTcD, (cuuint64_t)kTcD * (cuuint64_t)Hkv};
  cuuint32_t box[3] = {(cuuint32_t)kTcD, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  cache[next] = Entry{base, Hkv, slots, box_rows, *m};
  next = (next + 1) % 16;
  return true;
}

}  // namespace

bool attn_tc_supported(int D, int G, int block_size) { return D == kTcD && G >= 1 && G <= 16 && block_size % 8 == 0; }

size_t attn_tc_smem_bytes(int chunk) { return tc_smem_bytes(chunk); }

int attn_tc_resident() {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 148, per_sm = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaFuncSetAttribute(decode_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc_smem_bytes(kTcMaxChunk));
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_attn_tc_kernel, kTcThreads, tc_smem_bytes(kTcMaxChunk)) !=
          cudaSuccess ||
      per_sm <= 0)
    per_sm = 1;
  cudaGetLastError();
  const int n = std::max(1, sms * per_sm);
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t launch_attn_tc(const void *q, const uint8_t *kc, const uint8_t *vc, const float *ks, const float *vs,
                           const int32_t *block_tables, const int32_t *context_lens, int B, int Hq, int Hkv,
                           int block_size, int max_blocks, int64_t num_slots, uint64_t bs_magic, int chunk,
                           int splits, float scale_log2, float *part_ml, float *part_acc, void *out,
                           uint32_t *status, cudaStream_t st) {
  if ((out != nullptr && splits != 1) || chunk % kTcTile != 0 || chunk > kTcMaxChunk || Hq % Hkv != 0 || !attn_tc_supported(kTcD, Hq / Hkv, block_size))
    return cudaErrorInvalidValue;
  const int box_rows = block_size % 16 == 0 ? 16 : 8;
  CUtensorMap tmK, tmV;
  if (!tc_cache_map(&tmK, kc, Hkv, num_slots, box_rows) || !tc_cache_map(&tmV, vc, Hkv, num_slots, box_rows))
    return cudaErrorInvalidValue;
  TcParams p = {};
  p.q = static_cast<const __nv_bfloat16 *>(q);
  p.ks = ks;
  p.vs = vs;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.hgroups = (p.G + 7) / 8;
  p.block_size = block_size;
  p.box_rows = box_rows;
  p.max_blocks = max_blocks;
  p.splits = splits;
  p.chunk = chunk;
  p.bs_magic = bs_magic;
  p.num_slots = num_slots;
  p.scale_log2 = scale_log2;
  p.part_ml = part_ml;
  p.part_acc = part_acc;
  p.out = static_cast<__nv_bfloat16 *>(out);
  p.status = status;
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t a = cudaFuncSetAttribute(decode_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)tc_smem_bytes(kTcMaxChunk));
    if (a != cudaSuccess) return a;
    attr_set[dev].store(true, std::memory_order_release);
  }
  if ((int64_t)Hkv * p.hgroups > 65535) return cudaErrorInvalidValue;
  decode_attn_tc_kernel<<<dim3(splits, Hkv * p.hgroups, B), kTcThreads, tc_smem_bytes(chunk), st>>>(p, tmK, tmV);
  return cudaGetLastError();
}

}  // namespace ptpc
