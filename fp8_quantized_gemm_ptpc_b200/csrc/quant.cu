// PTPC-FP8 quantisers for sm_100a.
//
// Per-token activation quantisation and per-output-channel weight
// quantisation ("PTPC-FP8: boosting vLLM performance on AMD ROCm", section
// "Per-Token Activation + Per-Channel Weight Quantization": Delta_X[T x 1],
// Delta_W[1 x Co]); the per-tensor variants of the page's "standard FP8"
// comparison (Delta_X[1], Delta_W[1]); and step 2 of the page's naive
// two-step path (section "The challenge: two-step vs fused").
//
// Every code is E4M3_satRNE(fp32_RN(x / s)) with s = fp32_RN(amax / 448).  The
// division is done without a per-element divide: with r = RN(1/s),
//   q0 = RN(x * r),  e = q0 * s - x (one FMA, exact),  q = RN(q0 - e * r),
// the one-step correction of Markstein ("Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. R&D 34(1), 1990).  The
// residual is formed as q0*s - x rather than x - q0*s so that x = -0 gives
// q = -0 (the other form returns +0 there).  For s >= 2^-100 this yields the
// IEEE quotient itself whenever |x/s| >= 2^-11 and the same E4M3 code for
// every pair of bf16 inputs (checked exhaustively against the CPU
// definition); groups with a smaller scale take the IEEE division __fdiv_rn.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp6.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "kernels.h"

namespace ptpc {

namespace {

constexpr float kFastPathMinScale = 0x1p-100f;

// Division mode shared by every element of a row / column.
enum : int { kZeroGroup = 0, kFast = 1, kSlow = 2 };

struct GroupScale {
  float s;     // dequantisation scale
  float r;     // RN(1/s) (fast mode only)
  int mode;
};

// Scale of a group from its largest magnitude (bf16 bits): amax / fmax, the
// format's largest finite value (448 for E4M3).
__device__ __forceinline__ GroupScale group_scale_from_amax_bits(uint32_t amax_bits16, float fmax = 448.0f) {
  GroupScale g;
  const float amax = __uint_as_float(amax_bits16 << 16);
  if (amax == 0.0f) {
    g.s = 1.0f;
    g.r = 1.0f;
    g.mode = kZeroGroup;
  } else {
    g.s = __fdiv_rn(amax, fmax);
    g.r = __frcp_rn(g.s);
    g.mode = g.s >= kFastPathMinScale ? kFast : kSlow;
  }
  return g;
}

__device__ __forceinline__ float quotient(float x, const GroupScale &g) {
  if (g.mode == kFast) {
    const float q0 = __fmul_rn(x, g.r);
    const float e = __fmaf_rn(q0, g.s, -x);
    return __fmaf_rn(-e, g.r, q0);
  }
  return __fdiv_rn(x, g.s);
}

// Two bf16 (low half = first element) -> two E4M3 codes (low byte = first).
__device__ __forceinline__ uint32_t quant_pair(uint32_t w, const GroupScale &g) {
  const float lo = __uint_as_float(w << 16);
  const float hi = __uint_as_float(w & 0xFFFF0000u);
  float2 q;
  q.x = quotient(lo, g);
  q.y = quotient(hi, g);
  return (uint32_t)__nv_cvt_float2_to_fp8x2(q, __NV_SATFINITE, __NV_E4M3);
}

// Fast path for two bf16 of one 32-bit word, with Blackwell's packed fp32x2
// arithmetic: the same three IEEE operations as quotient(), two lanes per
// instruction.  nx = -x is built during unpacking, so that
//   q0 = RN((-x) * (-r)) = RN(x * r),  e = RN(q0 * s + (-x)),  q = RN(e * (-r) + q0)
// (the residual form that keeps -0 as -0).  Returns the two E4M3 codes,
// first element in the low byte.
__device__ __forceinline__ uint32_t quant_nx2_fast(uint32_t nlo, uint32_t nhi, uint64_t s2, uint64_t nr2);

__device__ __forceinline__ uint32_t quant_pair_fast(uint32_t w, uint64_t s2, uint64_t nr2) {
  const uint32_t nlo = (w << 16) ^ 0x80000000u;       // -x of the first element
  const uint32_t nhi = (w & 0xFFFF0000u) ^ 0x80000000u;  // -x of the second element
  return quant_nx2_fast(nlo, nhi, s2, nr2);
}

// The fast-path arithmetic of quant_pair_fast on two elements given as the
// fp32 bits of their negations (first element -> low byte of the result).
__device__ __forceinline__ uint32_t quant_nx2_fast(uint32_t nlo, uint32_t nhi, uint64_t s2, uint64_t nr2) {
  uint64_t nx2, q0, e, q;
  asm("mov.b64 %0, {%1, %2};" : "=l"(nx2) : "r"(nlo), "r"(nhi));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q0) : "l"(nx2), "l"(nr2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e) : "l"(q0), "l"(s2), "l"(nx2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(q) : "l"(e), "l"(nr2), "l"(q0));
  uint32_t qlo, qhi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(qlo), "=r"(qhi) : "l"(q));
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "r"(qhi), "r"(qlo));
  return (uint32_t)c;
}

// Eight bf16 (16 bytes) -> eight codes (8 bytes), fast path.
__device__ __forceinline__ uint2 quant_vec_fast(const uint4 v, uint64_t s2, uint64_t nr2) {
  uint2 o;
  o.x = quant_pair_fast(v.x, s2, nr2) | (quant_pair_fast(v.y, s2, nr2) << 16);
  o.y = quant_pair_fast(v.z, s2, nr2) | (quant_pair_fast(v.w, s2, nr2) << 16);
  return o;
}

// The fast path on x as it is: with -r in place of r the three steps give
// -q exactly (signed zeros included: checked against the form above for every
// (bf16 amax, bf16 x) pair with s >= 2^-100), so the codes come out with
// their sign bits flipped, which one XOR per four codes undoes.  This saves
// building -x for every element.
__device__ __forceinline__ uint32_t quant_x2_negated(uint32_t w, uint64_t s2, uint64_t nr2) {
  const uint32_t lo = w << 16, hi = w & 0xFFFF0000u;
  uint64_t x2, nq0, e, nq;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x2) : "r"(lo), "r"(hi));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(nq0) : "l"(x2), "l"(nr2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e) : "l"(nq0), "l"(s2), "l"(x2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(nq) : "l"(e), "l"(nr2), "l"(nq0));
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(nq));
  uint16_t c;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "r"(b), "r"(a));
  return (uint32_t)c;
}

__device__ __forceinline__ uint2 quant_vec_fast_flip(const uint4 v, uint64_t s2, uint64_t nr2) {
  uint2 o;
  o.x = (quant_x2_negated(v.x, s2, nr2) | (quant_x2_negated(v.y, s2, nr2) << 16)) ^ 0x80808080u;
  o.y = (quant_x2_negated(v.z, s2, nr2) | (quant_x2_negated(v.w, s2, nr2) << 16)) ^ 0x80808080u;
  return o;
}

// Eight bf16 (16 bytes) -> eight codes (8 bytes), any mode.
__device__ __forceinline__ uint2 quant_vec(const uint4 v, const GroupScale &g) {
  if (g.mode == kZeroGroup) return make_uint2(0u, 0u);
  uint2 o;
  o.x = quant_pair(v.x, g) | (quant_pair(v.y, g) << 16);
  o.y = quant_pair(v.z, g) | (quant_pair(v.w, g) << 16);
  return o;
}

__device__ __forceinline__ uint64_t pack2(float a) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "r"(__float_as_uint(a)));
  return r;
}

// Quantises n vectors src[j0], src[j0 + step], ... of one group into
// dst[j] (8 codes each), choosing the arithmetic once for the whole run.
template <typename Src>
__device__ __forceinline__ void quant_run(Src src, uint2 *dst, int j0, int n, int step, const GroupScale &g) {
  if (g.mode == kFast) {
    const uint64_t s2 = pack2(g.s), nr2 = pack2(-g.r);
    for (int j = j0; j < n; j += step) dst[j] = quant_vec_fast(src(j), s2, nr2);
  } else if (g.mode == kSlow) {
    for (int j = j0; j < n; j += step) dst[j] = quant_vec(src(j), g);
  } else {
    for (int j = j0; j < n; j += step) dst[j] = make_uint2(0u, 0u);
  }
}

// max(|bf16|) of a 16-byte vector folded into acc (bf16x2 magnitudes; the
// sign bits of acc are meaningless).  One max.xorsign.abs per two elements.
__device__ __forceinline__ uint32_t absmax_bits(uint32_t acc, uint4 v) {
  asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(acc) : "r"(v.x));
  asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(acc) : "r"(v.y));
  asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(acc) : "r"(v.z));
  asm("max.xorsign.abs.bf16x2 %0, %0, %1;" : "+r"(acc) : "r"(v.w));
  return acc;
}

// Larger of the two 16-bit magnitudes of a folded accumulator.
__device__ __forceinline__ uint32_t fold_halves(uint32_t m) {
  m &= 0x7FFF7FFFu;
  return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }

// ----------------------------------------------------------------------------
// Per-token activation quantisation.
//
// A group of P threads (a multiple of 32) owns one row; each thread holds V
// 16-byte vectors of the row in registers, so the row is read from HBM once:
// load, |x| max, group reduction (warp shuffle, then shared memory across
// the group's warps), then quantise from registers and store 8 codes per
// vector.  R = blockDim / P rows per CTA.
// SRC: where the group scale's maximum comes from: kAmaxRow the row itself;
// kAmaxTensor a tensor-wide maximum computed by amax_kernel (the per-tensor
// comparison path, bf16 magnitude bits); kAmaxGiven an fp32 maximum per row
// supplied by the caller (the row split over tensor-parallel ranks).
// ----------------------------------------------------------------------------
enum : int { kAmaxRow = 0, kAmaxTensor = 1, kAmaxGiven = 2 };

template <int V, int SRC>
__global__ void __launch_bounds__(V >= 16 ? 512 : 1024) quant_act_kernel(const uint4 *__restrict__ X, int T, int nvec,
                                                         int64_t ldv, uint8_t *__restrict__ Xq,
                                                         float *__restrict__ xs, int P,
                                                         const uint32_t *__restrict__ tensor_amax,
                                                         const float *__restrict__ given_amax) {
  __shared__ uint32_t red[32];
  griddep_launch_dependents();
  // Launched as a programmatic dependent: X (and the buffers written below)
  // may belong to the kernel launched just before, which must finish first.
  griddep_wait();

  const int tid = threadIdx.x;
  const int rl = tid / P;
  const int lt = tid - rl * P;
  const int rows_per_cta = blockDim.x / P;
  const int64_t row = (int64_t)blockIdx.x * rows_per_cta + rl;
  const bool active = row < T;
  const uint4 *xr = X + row * ldv;

  uint4 v[V];
  uint32_t m = 0;
  #pragma unroll
  for (int i = 0; i < V; ++i) {
    const int j = lt + i * P;
    if (active && j < nvec) {
      v[i] = ld_stream(xr + j);
    } else {
      v[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  uint32_t amax_bits;
  if constexpr (SRC == kAmaxTensor) {
    amax_bits = *tensor_amax;
  } else if constexpr (SRC == kAmaxGiven) {
    amax_bits = active ? __float_as_uint(given_amax[row]) >> 16 : 0u;
  } else {
    #pragma unroll
    for (int i = 0; i < V; ++i) m = absmax_bits(m, v[i]);
    m = __reduce_max_sync(0xffffffffu, fold_halves(m));
    const int warps_per_row = P >> 5;
    if (warps_per_row > 1) {
      if ((tid & 31) == 0) red[tid >> 5] = m;
      __syncthreads();
      m = 0;
      const int w0 = rl * warps_per_row;
      for (int w = 0; w < warps_per_row; ++w) m = max(m, red[w0 + w]);
    }
    amax_bits = m;
  }
  const GroupScale g = group_scale_from_amax_bits(amax_bits);
  if (!active) return;
  if (lt == 0) xs[row] = g.s;

  uint2 *qr = reinterpret_cast<uint2 *>(Xq + row * (int64_t)nvec * 8);
  if (g.mode == kFast) {
    const uint64_t s2 = pack2(g.s), nr2 = pack2(-g.r);
    #pragma unroll
    for (int i = 0; i < V; ++i) {
      const int j = lt + i * P;
      if (j < nvec) qr[j] = quant_vec_fast(v[i], s2, nr2);
    }
  } else {
    #pragma unroll
    for (int i = 0; i < V; ++i) {
      const int j = lt + i * P;
      if (j < nvec) qr[j] = quant_vec(v[i], g);
    }
  }
}

// Rows that split exactly into V vectors per thread x P threads (P a
// multiple of 32): the same algorithm as quant_act_kernel without any
// per-vector bounds check, with P known at compile time for the common model
// widths (PC; 0 = P at run time) so every load and store takes an immediate
// offset, and the row's scale computed once by its first thread and
// broadcast through shared memory.  Measured with the same counters: 5.4
// instead of 9.7 instructions per element at 8192 columns, which is what
// decides the throughput when the power cap holds the SM clock near 1 GHz.
template <int V, int SRC, int PC>
__global__ void __launch_bounds__(V >= 16 ? 512 : 1024) quant_act_exact_kernel(
    const uint4 *__restrict__ X, int T, int64_t ldv, uint8_t *__restrict__ Xq, float *__restrict__ xs, int p_rt,
    const uint32_t *__restrict__ tensor_amax, const float *__restrict__ given_amax) {
  __shared__ uint32_t red[32];
  __shared__ float sb_s[32], sb_r[32];
  __shared__ int sb_mode[32];
  griddep_launch_dependents();
  griddep_wait();
  const int P = PC ? PC : p_rt;
  const int tid = threadIdx.x;
  const int rl = tid / P;
  const int lt = tid - rl * P;
  const int R = blockDim.x / P;
  const int64_t row = (int64_t)blockIdx.x * R + rl;
  const bool active = row < T;
  const uint4 *xr = X + row * ldv + lt;
  uint4 v[V];
  if (active) {
    #pragma unroll
    for (int i = 0; i < V; ++i) v[i] = ld_stream(xr + i * P);
  } else {
    #pragma unroll
    for (int i = 0; i < V; ++i) v[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if constexpr (SRC == kAmaxRow) {
    uint32_t m = 0;
    #pragma unroll
    for (int i = 0; i < V; ++i) m = absmax_bits(m, v[i]);
    m = __reduce_max_sync(0xffffffffu, fold_halves(m));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
  }
  if (lt == 0) {
    uint32_t amax_bits = 0;
    if constexpr (SRC == kAmaxTensor) {
      amax_bits = *tensor_amax;
    } else if constexpr (SRC == kAmaxGiven) {
      amax_bits = active ? __float_as_uint(given_amax[row]) >> 16 : 0u;
    } else {
      const int w0 = rl * (P >> 5);
      for (int w = 0; w < (P >> 5); ++w) amax_bits = max(amax_bits, red[w0 + w]);
    }
    const GroupScale g = group_scale_from_amax_bits(amax_bits);
    sb_s[rl] = g.s;
    sb_r[rl] = g.r;
    sb_mode[rl] = g.mode;
    if (active) xs[row] = g.s;
  }
  __syncthreads();
  if (!active) return;
  GroupScale g;
  g.s = sb_s[rl];
  g.r = sb_r[rl];
  g.mode = sb_mode[rl];
  uint2 *qr = reinterpret_cast<uint2 *>(Xq + row * (int64_t)V * P * 8) + lt;
  if (g.mode == kFast) {
    const uint64_t s2 = pack2(g.s), nr2 = pack2(-g.r);
    #pragma unroll
    for (int i = 0; i < V; ++i) qr[i * P] = quant_vec_fast_flip(v[i], s2, nr2);
  } else {
    #pragma unroll
    for (int i = 0; i < V; ++i) qr[i * P] = quant_vec(v[i], g);
  }
}

// Rows too long for registers: two passes over the row (the second read is
// normally served from L2).  One CTA per row.
template <int SRC>
__global__ void __launch_bounds__(1024) quant_act_long_kernel(const uint4 *__restrict__ X, int T, int nvec,
                                                              int64_t ldv, uint8_t *__restrict__ Xq,
                                                              float *__restrict__ xs,
                                                              const uint32_t *__restrict__ tensor_amax,
                                                              const float *__restrict__ given_amax) {
  __shared__ uint32_t red[32];
  __shared__ uint32_t row_amax;
  griddep_launch_dependents();
  griddep_wait();
  const int64_t row = blockIdx.x;
  const uint4 *xr = X + row * ldv;
  uint32_t amax_bits;
  if constexpr (SRC == kAmaxTensor) {
    amax_bits = *tensor_amax;
  } else if constexpr (SRC == kAmaxGiven) {
    amax_bits = __float_as_uint(given_amax[row]) >> 16;
  } else {
    uint32_t m = 0;
    for (int j = threadIdx.x; j < nvec; j += blockDim.x) m = absmax_bits(m, xr[j]);
    m = __reduce_max_sync(0xffffffffu, fold_halves(m));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t mm = 0;
      for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mm = max(mm, red[w]);
      row_amax = mm;
    }
    __syncthreads();
    amax_bits = row_amax;
  }
  const GroupScale g = group_scale_from_amax_bits(amax_bits);
  if (threadIdx.x == 0) xs[row] = g.s;
  uint2 *qr = reinterpret_cast<uint2 *>(Xq + row * (int64_t)nvec * 8);
  quant_run([&](int j) { return ld_stream(xr + j); }, qr, threadIdx.x, nvec, blockDim.x, g);
}

// Tensor-wide max |x| of rows x nvec 16-byte vectors (row pitch ldv
// vectors), as bf16 magnitude bits, into *amax (atomicMax; *amax must be 0
// beforehand).
__global__ void __launch_bounds__(512) amax_kernel(const uint4 *__restrict__ X, int64_t rows, int nvec,
                                                   int64_t ldv, uint32_t *__restrict__ amax) {
  uint32_t m = 0;
  const int64_t n8 = rows * nvec;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n8; j += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = j / nvec;
    m = absmax_bits(m, ld_stream(X + r * ldv + (j - r * nvec)));
  }
  m = __reduce_max_sync(0xffffffffu, fold_halves(m));
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax, m);
}

// ----------------------------------------------------------------------------
// Per-output-channel weight quantisation, pass 1: column maxima.
// W is Ci x Co row-major.  Each thread owns 8 adjacent columns (one 16-byte
// vector per row) and walks a slab of rows; the CTA's warps split the slab;
// the result is merged with atomicMax into col_amax[Co] (zeroed beforehand).
// ----------------------------------------------------------------------------
constexpr int kColThreads = 32;   // vectors (8 columns each) per CTA row
constexpr int kColWarps = 8;

__global__ void __launch_bounds__(kColThreads * kColWarps) col_amax_kernel(const uint4 *__restrict__ W, int Ci,
                                                                            int Co, int rows_per_cta,
                                                                            uint32_t *__restrict__ col_amax) {
  __shared__ uint32_t red[kColWarps][kColThreads][4];
  const int ncv = Co / 8;
  const int cv = blockIdx.x * kColThreads + (threadIdx.x & 31);
  const int warp = threadIdx.x >> 5;
  const int k0 = blockIdx.y * rows_per_cta;
  const int k1 = min(Ci, k0 + rows_per_cta);
  uint32_t m0 = 0, m1 = 0, m2 = 0, m3 = 0;
  if (cv < ncv) {
    for (int k = k0 + warp; k < k1; k += kColWarps) {
      const uint4 v = ld_stream(W + (int64_t)k * ncv + cv);
      m0 = __vmaxu2(m0, v.x & 0x7FFF7FFFu);
      m1 = __vmaxu2(m1, v.y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
      m3 = __vmaxu2(m3, v.w & 0x7FFF7FFFu);
    }
  }
  red[warp][threadIdx.x & 31][0] = m0;
  red[warp][threadIdx.x & 31][1] = m1;
  red[warp][threadIdx.x & 31][2] = m2;
  red[warp][threadIdx.x & 31][3] = m3;
  __syncthreads();
  if (warp == 0 && cv < ncv) {
    const int l = threadIdx.x & 31;
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t mm = 0;
      for (int w = 0; w < kColWarps; ++w) mm = __vmaxu2(mm, red[w][l][q]);
      const int col = cv * 8 + q * 2;
      if ((mm & 0xFFFFu) != 0) atomicMax(col_amax + col, mm & 0xFFFFu);
      if ((mm >> 16) != 0) atomicMax(col_amax + col + 1, mm >> 16);
    }
  }
}

// Tensor-wide amax broadcast into every column's slot (per-tensor weights).
__global__ void broadcast_amax_kernel(const uint32_t *__restrict__ src, uint32_t *__restrict__ dst, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) dst[i] = *src;
}

// ----------------------------------------------------------------------------
// Weight quantisation, between the passes: each column's scale from its
// maximum, once per column.  w_scale[o] = s; the column-maximum word is
// replaced by the bits of RN(1/s) (never 0 for a nonzero column), or 0 for an
// all-zero column, so pass 2 needs no division.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) weight_scales_kernel(uint32_t *__restrict__ col_amax,
                                                            float *__restrict__ w_scale, int Co, float fmax) {
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= Co) return;
  const GroupScale g = group_scale_from_amax_bits(col_amax[o], fmax);
  w_scale[o] = g.s;
  col_amax[o] = g.mode == kZeroGroup ? 0u : __float_as_uint(g.r);
}

// ----------------------------------------------------------------------------
// Weight quantisation, pass 2: quantise a 128 (k) x 64 (o) tile of W with its
// columns' scales and write it transposed into Wq_t (Co x Ci).  Thread
// (cv, kq) converts rows 4*kq .. 4*kq+3 of the 8 columns of vector cv, so for
// each column it holds 4 consecutive K codes: one 32-bit word into the
// shared tile [o][k], which is then written out as 16-byte row chunks.  Both
// the bf16 reads (along Co) and the code writes (along Ci) are coalesced.
// ----------------------------------------------------------------------------
constexpr int kTK = 128;   // K rows per tile
constexpr int kTO = 64;    // output channels per tile
constexpr int kTPitch = kTK + 4;

__global__ void __launch_bounds__(256) quant_weight_t_kernel(const uint4 *__restrict__ W, int Ci, int Co,
                                                             const uint32_t *__restrict__ col_rcp,
                                                             uint8_t *__restrict__ Wq_t,
                                                             const float *__restrict__ w_scale) {
  __shared__ __align__(16) uint8_t tile[kTO][kTPitch];
  const int o0 = blockIdx.x * kTO;
  const int k0 = blockIdx.y * kTK;
  const int ncv = Co / 8;
  const int cv = threadIdx.x & 7;      // 8-column vector within the tile
  const int kq = threadIdx.x >> 3;     // rows 4*kq .. 4*kq+3
  const int ocol = o0 + cv * 8;
  uint4 v[4];
  #pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int k = k0 + 4 * kq + r;
    v[r] = (k < Ci && ocol < Co) ? ld_stream(W + (int64_t)k * ncv + (ocol >> 3)) : make_uint4(0u, 0u, 0u, 0u);
  }
  // this vector's 8 column scales and reciprocals (Co % 16 == 0: all valid or none)
  float sc[8], rc[8];
  if (ocol < Co) {
    const float4 s0 = __ldg(reinterpret_cast<const float4 *>(w_scale + ocol));
    const float4 s1 = __ldg(reinterpret_cast<const float4 *>(w_scale + ocol + 4));
    const uint4 r0 = __ldg(reinterpret_cast<const uint4 *>(col_rcp + ocol));
    const uint4 r1 = __ldg(reinterpret_cast<const uint4 *>(col_rcp + ocol + 4));
    sc[0] = s0.x; sc[1] = s0.y; sc[2] = s0.z; sc[3] = s0.w;
    sc[4] = s1.x; sc[5] = s1.y; sc[6] = s1.z; sc[7] = s1.w;
    rc[0] = __uint_as_float(r0.x); rc[1] = __uint_as_float(r0.y);
    rc[2] = __uint_as_float(r0.z); rc[3] = __uint_as_float(r0.w);
    rc[4] = __uint_as_float(r1.x); rc[5] = __uint_as_float(r1.y);
    rc[6] = __uint_as_float(r1.z); rc[7] = __uint_as_float(r1.w);
  } else {
    #pragma unroll
    for (int c = 0; c < 8; ++c) {
      sc[c] = 1.0f;
      rc[c] = 0.0f;
    }
  }
  #pragma unroll
  for (int c = 0; c < 8; ++c) {
    GroupScale g;
    g.s = sc[c];
    g.r = rc[c];
    g.mode = __float_as_uint(rc[c]) == 0u ? kZeroGroup : (sc[c] >= kFastPathMinScale ? kFast : kSlow);
    uint32_t word = 0;
    if (g.mode == kFast) {
      // rows (0, 1) and (2, 3) of the column as packed pairs, the same IEEE
      // steps as the activation quantiser's fast path
      const uint64_t s2 = pack2(g.s), nr2 = pack2(-g.r);
      uint32_t nx[4];
      #pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t w2 = (c < 2) ? v[r].x : (c < 4) ? v[r].y : (c < 6) ? v[r].z : v[r].w;
        nx[r] = ((c & 1) ? (w2 & 0xFFFF0000u) : (w2 << 16)) ^ 0x80000000u;
      }
      word = quant_nx2_fast(nx[0], nx[1], s2, nr2) | (quant_nx2_fast(nx[2], nx[3], s2, nr2) << 16);
    } else if (g.mode == kSlow) {
      float q[4];
      #pragma unroll
      for (int r = 0; r < 4; ++r) {
        const uint32_t w2 = (c < 2) ? v[r].x : (c < 4) ? v[r].y : (c < 6) ? v[r].z : v[r].w;
        const float x = (c & 1) ? __uint_as_float(w2 & 0xFFFF0000u) : __uint_as_float(w2 << 16);
        q[r] = quotient(x, g);
      }
      const uint32_t lo = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(q[0], q[1]), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(q[2], q[3]), __NV_SATFINITE, __NV_E4M3);
      word = lo | (hi << 16);
    }
    *reinterpret_cast<uint32_t *>(&tile[cv * 8 + c][4 * kq]) = word;
  }
  __syncthreads();
  // write: 64 rows (o) x 128 bytes (k), 16 bytes per thread, two passes
  #pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int idx = threadIdx.x + pass * 256;
    const int orow = idx >> 3;           // 0..63
    const int kc = (idx & 7) * 16;       // 0..112
    const int o = o0 + orow;
    const int k = k0 + kc;
    if (o < Co && k < Ci) {
      const uint32_t *src = reinterpret_cast<const uint32_t *>(&tile[orow][kc]);
      *reinterpret_cast<uint4 *>(Wq_t + (int64_t)o * Ci + k) = make_uint4(src[0], src[1], src[2], src[3]);
    }
  }
}

// ----------------------------------------------------------------------------
// Sub-byte weight formats: FP4 E2M1 and FP6 E2M3 / E3M2 (the OCP MX element
// types that tcgen05.mma.kind::f8f6f4 reads), one scale per output channel
// s = amax / max_format, codes packed along K the way TMA's packed 4- and
// 6-bit tensor types read them: FP4 two codes a byte (the even K position in
// the low nibble), FP6 code j of every 16 at bits [6j, 6j + 6) of 12 bytes
// read as a little-endian integer.  The quotient is the activation
// quantiser's divide-free one (exhaustively equal in code to the IEEE
// quotient for these divisors too), computed on x as is with -r, which gives
// -q, so the sign bits of the finished codes are flipped once per word.
//
// A CTA quantises a 128 (K) x 64 (channel) tile: thread (cv, kq) converts K
// rows 8 kq .. 8 kq + 7 of the 8 channels of vector cv into 8 codes per
// channel (4 bytes of FP4 or 6 of FP6), placed in a shared tile [channel][K
// bytes], which is written out as 16-byte row chunks (the bf16 reads run
// along Co, the packed writes along Ci; both coalesced).  Ci % 128 == 0.
// ----------------------------------------------------------------------------
constexpr int kSbThreads = 128;

template <int WF>
struct SubFmt;
template <>
struct SubFmt<1> {  // E2M1
  static constexpr int bits = 4;
  static constexpr float fmax = 6.0f;
};
template <>
struct SubFmt<2> {  // E2M3
  static constexpr int bits = 6;
  static constexpr float fmax = 7.5f;
};
template <>
struct SubFmt<3> {  // E3M2
  static constexpr int bits = 6;
  static constexpr float fmax = 28.0f;
};

// Codes of two fp32 values (a: even K position, b: odd) in the format, a in
// the low nibble (FP4) or the low byte (FP6).
template <int WF>
__device__ __forceinline__ uint32_t cvt_sub_pair(float a, float b) {
  if constexpr (WF == 1)
    return (uint32_t)__nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest) & 0xFFu;
  else if constexpr (WF == 2)
    return (uint32_t)__nv_cvt_float2_to_fp6x2(make_float2(a, b), __NV_E2M3, cudaRoundNearest);
  else
    return (uint32_t)__nv_cvt_float2_to_fp6x2(make_float2(a, b), __NV_E3M2, cudaRoundNearest);
}

// Eight consecutive-K values of one channel (fp32 bits) -> packed codes:
// FP4 in the low 32 bits, FP6 in the low 48.  `flip`: the values are -q.
template <int WF>
__device__ __forceinline__ uint64_t pack8_sub(const float (&q)[8], bool flip) {
  uint64_t acc = 0;
  #pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t c = cvt_sub_pair<WF>(q[2 * p], q[2 * p + 1]);
    if constexpr (WF == 1) {
      acc |= (uint64_t)c << (8 * p);
    } else {
      acc |= (uint64_t)(c & 0x3Fu) << (12 * p);
      acc |= (uint64_t)((c >> 8) & 0x3Fu) << (12 * p + 6);
    }
  }
  if (flip) acc ^= (WF == 1) ? 0x88888888ull : 0x820820820820ull;
  return acc;
}

template <int WF>
__global__ void __launch_bounds__(kSbThreads) quant_weight_sub_kernel(const uint4 *__restrict__ W, int Ci, int Co,
                                                                     const uint32_t *__restrict__ col_rcp,
                                                                     uint8_t *__restrict__ Wp,
                                                                     const float *__restrict__ w_scale) {
  constexpr int B = SubFmt<WF>::bits;
  constexpr int RB = kTK * B / 8;      // packed bytes of 128 K codes: 64 (FP4) or 96 (FP6)
  constexpr int PITCH = RB + 16;
  constexpr int CB = 8 * B / 8;        // packed bytes of 8 codes: 4 or 6
  __shared__ __align__(16) uint8_t tile[kTO][PITCH];
  const int o0 = blockIdx.x * kTO;
  const int k0 = blockIdx.y * kTK;
  const int ncv = Co / 8;
  const int cv = threadIdx.x & 7;
  const int kq = threadIdx.x >> 3;     // K rows 8 kq .. 8 kq + 7
  const int ocol = o0 + cv * 8;
  const bool col_ok = ocol < Co;       // Co % 16 == 0: the 8 columns are valid together
  uint4 v[8];
  #pragma unroll
  for (int r = 0; r < 8; ++r)
    v[r] = col_ok ? ld_stream(W + (int64_t)(k0 + 8 * kq + r) * ncv + (ocol >> 3)) : make_uint4(0u, 0u, 0u, 0u);
  #pragma unroll
  for (int c = 0; c < 8; ++c) {
    float s = 1.0f, rc = 0.0f;
    if (col_ok) {
      s = __ldg(w_scale + ocol + c);
      rc = __uint_as_float(__ldg(col_rcp + ocol + c));
    }
    float x[8];
    #pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t w2 = (c < 2) ? v[r].x : (c < 4) ? v[r].y : (c < 6) ? v[r].z : v[r].w;
      x[r] = (c & 1) ? __uint_as_float(w2 & 0xFFFF0000u) : __uint_as_float(w2 << 16);
    }
    uint64_t packed = 0;
    if (__float_as_uint(rc) == 0u) {
      packed = 0;  // all-zero column (or a column past Co)
    } else if (s >= kFastPathMinScale) {
      float q[8];
      #pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float nq0 = __fmul_rn(x[r], -rc);
        const float e = __fmaf_rn(nq0, s, x[r]);
        q[r] = __fmaf_rn(e, -rc, nq0);
      }
      packed = pack8_sub<WF>(q, true);
    } else {
      float q[8];
      #pragma unroll
      for (int r = 0; r < 8; ++r) q[r] = __fdiv_rn(x[r], s);
      packed = pack8_sub<WF>(q, false);
    }
    uint8_t *dst = &tile[cv * 8 + c][kq * CB];
    if constexpr (CB == 4) {
      *reinterpret_cast<uint32_t *>(dst) = (uint32_t)packed;
    } else {
      reinterpret_cast<uint16_t *>(dst)[0] = (uint16_t)packed;
      reinterpret_cast<uint16_t *>(dst)[1] = (uint16_t)(packed >> 16);
      reinterpret_cast<uint16_t *>(dst)[2] = (uint16_t)(packed >> 32);
    }
  }
  __syncthreads();
  constexpr int CHUNKS = RB / 16;      // 16-byte chunks per channel row
  const int64_t row_bytes = (int64_t)Ci * B / 8;
  for (int i = threadIdx.x; i < kTO * CHUNKS; i += kSbThreads) {
    const int orow = i / CHUNKS;
    const int ch = i - orow * CHUNKS;
    const int o = o0 + orow;
    if (o < Co)
      *reinterpret_cast<uint4 *>(Wp + (int64_t)o * row_bytes + (int64_t)k0 * B / 8 + ch * 16) =
          *reinterpret_cast<const uint4 *>(&tile[orow][ch * 16]);
  }
}

// ----------------------------------------------------------------------------
// FP8 KV cache, append: every (token, head) vector of D values of K and V is
// quantised with the per-token rule (s = amax / 448, the activation
// quantiser's exact quotient) and written to its paged-cache slot:
//   codes  cache[(slot * H + h) * D + d],  scale  scales[slot * H + h],
// slot = slots[t] (block * block_size + offset; a negative slot skips the
// token, a slot past the cache is skipped too).  D / 8 lanes own a vector
// (one 16-byte load, 8 codes each); a warp holds 32 * 8 / D vectors.
// ----------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) kv_append_kernel(const uint4 *__restrict__ K, const uint4 *__restrict__ V,
                                                        const int64_t *__restrict__ slots, int T, int H,
                                                        int64_t num_slots, uint8_t *__restrict__ kc,
                                                        uint8_t *__restrict__ vc, float *__restrict__ ks,
                                                        float *__restrict__ vs) {
  constexpr int L = D / 8;              // lanes per vector
  griddep_launch_dependents();
  griddep_wait();
  const int64_t vec = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / L;   // (t, h) row of K and V
  const int lane = threadIdx.x % L;
  const bool active = vec < (int64_t)T * H;
  const int64_t t = active ? vec / H : 0;
  const int h = active ? (int)(vec - t * H) : 0;
  const int64_t slot = active ? slots[t] : -1;
  const bool write = active && slot >= 0 && slot < num_slots;
  #pragma unroll
  for (int which = 0; which < 2; ++which) {
    const uint4 *src = which == 0 ? K : V;
    const uint4 v = active ? ld_stream(src + vec * L + lane) : make_uint4(0u, 0u, 0u, 0u);
    uint32_t m = fold_halves(absmax_bits(0u, v));
    #pragma unroll
    for (int o = L / 2; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    const GroupScale g = group_scale_from_amax_bits(m);
    uint2 q;
    if (g.mode == kFast)
      q = quant_vec_fast(v, pack2(g.s), pack2(-g.r));
    else
      q = quant_vec(v, g);
    if (write) {
      uint8_t *dst = (which == 0 ? kc : vc) + (slot * H + h) * D;
      reinterpret_cast<uint2 *>(dst)[lane] = q;
      if (lane == 0) (which == 0 ? ks : vs)[slot * H + h] = g.s;
    }
  }
}

// ----------------------------------------------------------------------------
// Naive two-step path, step 2: out = bf16((y * x_scale[t]) * w_scale[o]).
// Each thread handles 8 consecutive outputs (two 16-byte fp32 loads, one
// 16-byte bf16 store).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) apply_scales_kernel(const float4 *__restrict__ y, int T, int Co,
                                                           const float *__restrict__ xs,
                                                           const float *__restrict__ ws,
                                                           uint4 *__restrict__ out) {
  const int nv = Co / 8;
  const int64_t total = (int64_t)T * nv;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / nv;
    const int c = (int)(i - t * nv) * 8;
    const float a = xs[t];
    const float4 y0 = __ldcs(y + 2 * i);
    const float4 y1 = __ldcs(y + 2 * i + 1);
    const float4 w0 = __ldg(reinterpret_cast<const float4 *>(ws + c));
    const float4 w1 = __ldg(reinterpret_cast<const float4 *>(ws + c + 4));
    const float v[8] = {__fmul_rn(__fmul_rn(y0.x, a), w0.x), __fmul_rn(__fmul_rn(y0.y, a), w0.y),
                        __fmul_rn(__fmul_rn(y0.z, a), w0.z), __fmul_rn(__fmul_rn(y0.w, a), w0.w),
                        __fmul_rn(__fmul_rn(y1.x, a), w1.x), __fmul_rn(__fmul_rn(y1.y, a), w1.y),
                        __fmul_rn(__fmul_rn(y1.z, a), w1.z), __fmul_rn(__fmul_rn(y1.w, a), w1.w)};
    uint32_t p[4];
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
      p[q] = *reinterpret_cast<uint32_t *>(&b);
    }
    out[i] = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

// Launch shape of the register-resident activation quantiser.
struct ActPlan {
  int V;    // vectors per thread (0: use the two-pass kernel)
  int P;    // threads per row
  int R;    // rows per CTA
};

ActPlan plan_act(int nvec) {
  ActPlan p{0, 0, 0};
  auto roundup32 = [](int x) { return (x + 31) / 32 * 32; };
  if (nvec <= 32 * 8) {
    int v = (nvec + 31) / 32;
    p.V = v <= 1 ? 1 : v <= 2 ? 2 : v <= 4 ? 4 : 8;
    p.P = 32;
  } else if (roundup32((nvec + 7) / 8) <= 1024) {
    p.V = 8;
    p.P = roundup32((nvec + 7) / 8);
  } else if (roundup32((nvec + 15) / 16) <= 512) {  // 64 data registers a thread: at most 512 threads
    p.V = 16;
    p.P = roundup32((nvec + 15) / 16);
  } else {
    return p;
  }
  p.R = p.P >= 256 ? 1 : 256 / p.P;
  return p;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel in the stream finishes, and waits for it with
// griddepcontrol.wait before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Exact split of a row of nvec vectors: V vectors per thread x P threads, P
// a multiple of 32 (at most 1024 threads, 512 with 16 vectors); V = 0 if no
// such split exists.
ActPlan plan_act_exact(int nvec) {
  for (int V : {8, 4, 16}) {
    if (nvec % (32 * V) != 0) continue;
    const int P = nvec / V;
    if (P > (V >= 16 ? 512 : 1024)) continue;
    return ActPlan{V, P, P >= 256 ? 1 : 256 / P};
  }
  return ActPlan{0, 0, 0};
}

template <int V, int SRC, int PC>
cudaError_t launch_exact(const ActPlan &p, const uint4 *Xv, int T, int64_t ldv, uint8_t *Xq, float *xs,
                         const uint32_t *tensor_amax, const float *given_amax, cudaStream_t st) {
  const int grid = (T + p.R - 1) / p.R;
  return launch_pdl(quant_act_exact_kernel<V, SRC, PC>, grid, p.P * p.R, st, Xv, T, ldv, Xq, xs, p.P, tensor_amax,
                    given_amax);
}

template <int SRC>
cudaError_t launch_act(const void *X, int T, int Ci, int64_t ldx, uint8_t *Xq, float *xs,
                       const uint32_t *tensor_amax, const float *given_amax, cudaStream_t st) {
  const int nvec = Ci / 8;
  const int64_t ldv = ldx / 8;
  const uint4 *Xv = static_cast<const uint4 *>(X);
  const ActPlan e = plan_act_exact(nvec);
  if (e.V == 8) {
    // the model widths of the workloads: 4096, 8192, 14336, 28672 columns
    switch (e.P) {
      case 64: return launch_exact<8, SRC, 64>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
      case 128: return launch_exact<8, SRC, 128>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
      case 224: return launch_exact<8, SRC, 224>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
      case 448: return launch_exact<8, SRC, 448>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
      default: return launch_exact<8, SRC, 0>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
    }
  }
  if (e.V == 4) return launch_exact<4, SRC, 0>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
  if (e.V == 16) return launch_exact<16, SRC, 0>(e, Xv, T, ldv, Xq, xs, tensor_amax, given_amax, st);
  const ActPlan p = plan_act(nvec);
  if (p.V == 0)
    return launch_pdl(quant_act_long_kernel<SRC>, T, 1024, st, Xv, T, nvec, ldv, Xq, xs, tensor_amax, given_amax);
  const int grid = (T + p.R - 1) / p.R;
  const int block = p.P * p.R;
  switch (p.V) {
    case 1: return launch_pdl(quant_act_kernel<1, SRC>, grid, block, st, Xv, T, nvec, ldv, Xq, xs, p.P, tensor_amax, given_amax);
    case 2: return launch_pdl(quant_act_kernel<2, SRC>, grid, block, st, Xv, T, nvec, ldv, Xq, xs, p.P, tensor_amax, given_amax);
    case 4: return launch_pdl(quant_act_kernel<4, SRC>, grid, block, st, Xv, T, nvec, ldv, Xq, xs, p.P, tensor_amax, given_amax);
    case 8: return launch_pdl(quant_act_kernel<8, SRC>, grid, block, st, Xv, T, nvec, ldv, Xq, xs, p.P, tensor_amax, given_amax);
    default: return launch_pdl(quant_act_kernel<16, SRC>, grid, block, st, Xv, T, nvec, ldv, Xq, xs, p.P, tensor_amax, given_amax);
  }
}

// ----------------------------------------------------------------------------
// Row maxima of a T x Ci bf16 slice (fp32, exact): one warp per row, 8 rows
// per CTA, 16-byte streaming loads, warp reduction.  The first half of the
// row-split quantisation (the second is quant_act_kernel<., kAmaxGiven>).
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) row_amax_kernel(const uint4 *__restrict__ X, int T, int nvec, int64_t ldv,
                                                       float *__restrict__ amax) {
  griddep_launch_dependents();
  griddep_wait();
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const uint4 *xr = X + (int64_t)row * ldv;
  uint32_t m = 0;
  for (int j = lane; j < nvec; j += 32) m = absmax_bits(m, ld_stream(xr + j));
  m = __reduce_max_sync(0xffffffffu, fold_halves(m));
  if (lane == 0) amax[row] = __uint_as_float(m << 16);
}

}  // namespace

cudaError_t launch_quant_act(const void *X, int T, int Ci, int64_t ldx, uint8_t *Xq, float *xs, cudaStream_t st) {
  return launch_act<kAmaxRow>(X, T, Ci, ldx, Xq, xs, nullptr, nullptr, st);
}

cudaError_t launch_quant_act_amax(const void *X, int T, int Ci, int64_t ldx, const float *amax, uint8_t *Xq,
                                  float *xs, cudaStream_t st) {
  return launch_act<kAmaxGiven>(X, T, Ci, ldx, Xq, xs, nullptr, amax, st);
}

cudaError_t launch_row_amax(const void *X, int T, int Ci, int64_t ldx, float *amax, cudaStream_t st) {
  return launch_pdl(row_amax_kernel, (T + 7) / 8, 256, st, static_cast<const uint4 *>(X), T, Ci / 8, ldx / 8, amax);
}

cudaError_t launch_quant_act_per_tensor(const void *X, int T, int Ci, int64_t ldx, uint8_t *Xq, float *xs,
                                        uint32_t *amax_slot, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax_slot, 0, sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const int64_t n8 = (int64_t)T * Ci / 8;
  int grid = (int)std::min<int64_t>((n8 + 511) / 512, (int64_t)num_sms() * 4);
  if (grid < 1) grid = 1;
  amax_kernel<<<grid, 512, 0, st>>>(static_cast<const uint4 *>(X), T, Ci / 8, ldx / 8, amax_slot);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_act<kAmaxTensor>(X, T, Ci, ldx, Xq, xs, amax_slot, nullptr, st)) != cudaSuccess) return e;
  // the workspace's scratch word is left zero for the next user
  return cudaMemsetAsync(amax_slot, 0, sizeof(uint32_t), st);
}

cudaError_t launch_quant_weight(const void *W, int Ci, int Co, uint8_t *Wq_t, float *w_scale, uint32_t *col_amax,
                                bool per_tensor, cudaStream_t st) {
  cudaError_t e;
  const uint4 *Wv = static_cast<const uint4 *>(W);
  if (per_tensor) {
    uint32_t *slot = col_amax + Co;
    if ((e = cudaMemsetAsync(slot, 0, sizeof(uint32_t), st)) != cudaSuccess) return e;
    const int64_t n8 = (int64_t)Ci * Co / 8;
    int grid = (int)std::min<int64_t>((n8 + 511) / 512, (int64_t)num_sms() * 4);
    amax_kernel<<<grid, 512, 0, st>>>(Wv, Ci, Co / 8, Co / 8, slot);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    broadcast_amax_kernel<<<(Co + 255) / 256, 256, 0, st>>>(slot, col_amax, Co);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
    if ((e = cudaMemsetAsync(col_amax, 0, sizeof(uint32_t) * (size_t)Co, st)) != cudaSuccess) return e;
    const int ncv = Co / 8;
    const int gx = (ncv + kColThreads - 1) / kColThreads;
    // enough row slabs to fill the GPU a few times over
    int slabs = std::max(1, (num_sms() * 4 + gx - 1) / gx);
    int rows_per_cta = (Ci + slabs - 1) / slabs;
    rows_per_cta = std::max(rows_per_cta, 64);
    slabs = (Ci + rows_per_cta - 1) / rows_per_cta;
    col_amax_kernel<<<dim3(gx, slabs), kColThreads * kColWarps, 0, st>>>(Wv, Ci, Co, rows_per_cta, col_amax);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  weight_scales_kernel<<<(Co + 255) / 256, 256, 0, st>>>(col_amax, w_scale, Co, 448.0f);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 grid((Co + kTO - 1) / kTO, (Ci + kTK - 1) / kTK);
  quant_weight_t_kernel<<<grid, 256, 0, st>>>(Wv, Ci, Co, col_amax, Wq_t, w_scale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the workspace's scratch words are left zero for the next user
  return cudaMemsetAsync(col_amax, 0, sizeof(uint32_t) * ((size_t)Co + 1), st);
}

cudaError_t launch_quant_weight_sub(const void *W, int Ci, int Co, int fmt, uint8_t *Wp, float *w_scale,
                                    uint32_t *col_amax, cudaStream_t st) {
  if (fmt < 1 || fmt > 3 || Ci % kTK != 0) return cudaErrorInvalidValue;
  cudaError_t e;
  const uint4 *Wv = static_cast<const uint4 *>(W);
  if ((e = cudaMemsetAsync(col_amax, 0, sizeof(uint32_t) * (size_t)Co, st)) != cudaSuccess) return e;
  const int ncv = Co / 8;
  const int gx = (ncv + kColThreads - 1) / kColThreads;
  int slabs = std::max(1, (num_sms() * 4 + gx - 1) / gx);
  int rows_per_cta = (Ci + slabs - 1) / slabs;
  rows_per_cta = std::max(rows_per_cta, 64);
  slabs = (Ci + rows_per_cta - 1) / rows_per_cta;
  col_amax_kernel<<<dim3(gx, slabs), kColThreads * kColWarps, 0, st>>>(Wv, Ci, Co, rows_per_cta, col_amax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const float fmax = fmt == 1 ? SubFmt<1>::fmax : fmt == 2 ? SubFmt<2>::fmax : SubFmt<3>::fmax;
  weight_scales_kernel<<<(Co + 255) / 256, 256, 0, st>>>(col_amax, w_scale, Co, fmax);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const dim3 grid((Co + kTO - 1) / kTO, Ci / kTK);
  if (fmt == 1)
    quant_weight_sub_kernel<1><<<grid, kSbThreads, 0, st>>>(Wv, Ci, Co, col_amax, Wp, w_scale);
  else if (fmt == 2)
    quant_weight_sub_kernel<2><<<grid, kSbThreads, 0, st>>>(Wv, Ci, Co, col_amax, Wp, w_scale);
  else
    quant_weight_sub_kernel<3><<<grid, kSbThreads, 0, st>>>(Wv, Ci, Co, col_amax, Wp, w_scale);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // the workspace's scratch words are left zero for the next user
  return cudaMemsetAsync(col_amax, 0, sizeof(uint32_t) * ((size_t)Co + 1), st);
}

cudaError_t launch_kv_append(const void *K, const void *V, const int64_t *slots, int T, int H, int D,
                             int64_t num_slots, uint8_t *kc, uint8_t *vc, float *ks, float *vs, cudaStream_t st) {
  const int64_t threads = (int64_t)T * H * (D / 8);
  const int grid = (int)((threads + 255) / 256);
  const uint4 *Kv = static_cast<const uint4 *>(K);
  const uint4 *Vv = static_cast<const uint4 *>(V);
  switch (D) {
    case 64: return launch_pdl(kv_append_kernel<64>, grid, 256, st, Kv, Vv, slots, T, H, num_slots, kc, vc, ks, vs);
    case 128: return launch_pdl(kv_append_kernel<128>, grid, 256, st, Kv, Vv, slots, T, H, num_slots, kc, vc, ks, vs);
    case 256: return launch_pdl(kv_append_kernel<256>, grid, 256, st, Kv, Vv, slots, T, H, num_slots, kc, vc, ks, vs);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_apply_scales(const float *y, const float *xs, const float *ws, int T, int Co, void *out,
                                cudaStream_t st) {
  const int64_t total = (int64_t)T * (Co / 8);
  int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)num_sms() * 8);
  if (grid < 1) grid = 1;
  apply_scales_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const float4 *>(y), T, Co, xs, ws,
                                            static_cast<uint4 *>(out));
  return cudaGetLastError();
}

}  // namespace ptpc
