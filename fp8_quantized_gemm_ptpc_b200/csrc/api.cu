// C ABI of the PTPC-FP8 library: argument checks, workspace layout and
// dispatch to the sm_100a kernels.  Declared in include/ptpc.h.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/ptpc.h"
#include "bench_probe.h"
#include "attention_tc.h"
#include "kernels.h"

namespace {

constexpr size_t kAlign = 256;
constexpr int64_t kMaxDim = 0x7FFFFFFF;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace layout of the GEMM entry points:
//   [0, 256)                 device status word (uint32 at offset 0)
//   [256, gemm bytes)        prefill shapes only: the split tail's counters and
//                            fp32 partial accumulators (ptpc::gemm_workspace_bytes)
// ptpc_linear appends Xq [T, Ci] and x_scale [T] after the GEMM's part.
constexpr size_t kGemmWorkspace = kAlign;  // the part every GEMM call needs

size_t gemm_ws(int64_t T, int64_t Ci, int64_t Co) { return ptpc::gemm_workspace_bytes((int)T, (int)Ci, (int)Co); }

// Once per device: the kernels are built for compute capability 10.0 only.
int check_device() {
  static std::mutex mu;
  static int state[64] = {};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PTPC_ERR_CUDA;
  if (dev < 0 || dev >= 64) return PTPC_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (state[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return PTPC_ERR_CUDA;
    state[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return state[dev] == 1 ? PTPC_OK : PTPC_ERR_UNSUPPORTED_DEVICE;
}

int check_shape_tci(int64_t T, int64_t Ci) {
  if (T < 0 || Ci <= 0) return Ci < 0 || T < 0 ? PTPC_ERR_INVALID_ARG : PTPC_ERR_UNSUPPORTED_SHAPE;
  if (Ci % 16 != 0 || Ci > kMaxDim || T > kMaxDim) return PTPC_ERR_UNSUPPORTED_SHAPE;
  return PTPC_OK;
}

// Row pitch of an activation: at least Ci elements, 16-byte rows.
int check_ldx(int64_t ldx, int64_t Ci) {
  if (ldx < Ci) return PTPC_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || ldx > kMaxDim) return PTPC_ERR_MISALIGNED;
  return PTPC_OK;
}

int check_co(int64_t Co) {
  if (Co < 0) return PTPC_ERR_INVALID_ARG;
  if (Co == 0 || Co % 16 != 0 || Co > kMaxDim) return PTPC_ERR_UNSUPPORTED_SHAPE;
  return PTPC_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? PTPC_OK : PTPC_ERR_CUDA; }

// Weight formats (ptpc_weight_format): bits per code.
int wfmt_bits(int fmt) { return fmt == PTPC_WFMT_E4M3 ? 8 : fmt == PTPC_WFMT_E2M1 ? 4 : 6; }

bool valid_wfmt(int fmt) { return fmt >= PTPC_WFMT_E4M3 && fmt <= PTPC_WFMT_E3M2; }

// Packed sub-byte weights: TMA's 4- and 6-bit tensor types read rows of whole
// 128-code boxes from 32-byte aligned addresses.
int check_subbyte(int fmt, int64_t Ci, const void *Wq) {
  if (fmt == PTPC_WFMT_E4M3) return PTPC_OK;
  if (Ci % 128 != 0) return PTPC_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(Wq) & 31u) != 0) return PTPC_ERR_MISALIGNED;
  return PTPC_OK;
}

int run_gemm(const uint8_t *Xq, const float *xs, const uint8_t *Wq_t, const float *ws, int64_t T, int64_t Ci,
             int64_t Co, void *out, bool f32_out, uint8_t *wsp, size_t ws_bytes, bool pdl, cudaStream_t st,
             int wfmt = 0) {
  ptpc::GemmProblem p{};
  p.wfmt = wfmt;
  p.ws_bytes = ws_bytes;
  p.Xq = Xq;
  p.xs = xs;
  p.Wq_t = Wq_t;
  p.ws = ws;
  p.T = (int)T;
  p.Ci = (int)Ci;
  p.Co = (int)Co;
  p.out = out;
  p.f32_out = f32_out;
  p.status = reinterpret_cast<uint32_t *>(wsp);
  p.pdl = pdl;
  return cuda_status(ptpc::launch_scaled_gemm(p, st));
}

}  // namespace

extern "C" {

const char *ptpc_status_string(int status) {
  switch (status) {
    case PTPC_OK: return "PTPC_OK";
    case PTPC_ERR_INVALID_ARG: return "PTPC_ERR_INVALID_ARG";
    case PTPC_ERR_MISALIGNED: return "PTPC_ERR_MISALIGNED";
    case PTPC_ERR_UNSUPPORTED_SHAPE: return "PTPC_ERR_UNSUPPORTED_SHAPE";
    case PTPC_ERR_WORKSPACE_TOO_SMALL: return "PTPC_ERR_WORKSPACE_TOO_SMALL";
    case PTPC_ERR_UNSUPPORTED_DEVICE: return "PTPC_ERR_UNSUPPORTED_DEVICE";
    case PTPC_ERR_CUDA: return "PTPC_ERR_CUDA";
    case PTPC_ERR_DEVICE_TIMEOUT: return "PTPC_ERR_DEVICE_TIMEOUT";
    case PTPC_ERR_NOT_IMPLEMENTED: return "PTPC_ERR_NOT_IMPLEMENTED";
    default: return "PTPC_ERR_UNKNOWN";
  }
}

size_t ptpc_workspace_size(int op, int64_t T, int64_t Ci, int64_t Co) {
  switch (op) {
    case PTPC_OP_QUANTIZE_WEIGHTS:
      if (check_shape_tci(0, Ci) != PTPC_OK || check_co(Co) != PTPC_OK) return 0;
      return kAlign + round_up((size_t)(Co + 1) * 4);
    case PTPC_OP_SCALED_MM:
      if (check_shape_tci(T, Ci) != PTPC_OK || check_co(Co) != PTPC_OK) return 0;
      return gemm_ws(T, Ci, Co);
    case PTPC_OP_BENCH_UNSCALED_MM:
      if (check_shape_tci(T, Ci) != PTPC_OK || check_co(Co) != PTPC_OK) return 0;
      return kGemmWorkspace;
    case PTPC_OP_LINEAR:
      if (check_shape_tci(T, Ci) != PTPC_OK || check_co(Co) != PTPC_OK) return 0;
      return gemm_ws(T, Ci, Co) + round_up((size_t)T * (size_t)Ci) + round_up((size_t)T * 4);
    case PTPC_OP_BENCH_PER_TENSOR:
      if (check_shape_tci(T, Ci) != PTPC_OK) return 0;
      return kAlign + kAlign;
    default:
      return 0;
  }
}

int ptpc_quantize_activations(const void *X, int64_t T, int64_t Ci, int64_t ldx, uint8_t *Xq, float *x_scale,
                              void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if ((s = check_ldx(ldx, Ci)) != PTPC_OK) return s;
  if (!X || !Xq || !x_scale) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(x_scale)) return PTPC_ERR_MISALIGNED;
  if ((s = check_device()) != PTPC_OK) return s;
  return cuda_status(ptpc::launch_quant_act(X, (int)T, (int)Ci, ldx, Xq, x_scale, (cudaStream_t)stream));
}

int ptpc_act_row_amax(const void *X, int64_t T, int64_t Ci, int64_t ldx, float *amax, void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if ((s = check_ldx(ldx, Ci)) != PTPC_OK) return s;
  if (!X || !amax) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(amax)) return PTPC_ERR_MISALIGNED;
  if ((s = check_device()) != PTPC_OK) return s;
  return cuda_status(ptpc::launch_row_amax(X, (int)T, (int)Ci, ldx, amax, (cudaStream_t)stream));
}

int ptpc_quantize_activations_amax(const void *X, int64_t T, int64_t Ci, int64_t ldx, const float *amax,
                                   uint8_t *Xq, float *x_scale, void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if ((s = check_ldx(ldx, Ci)) != PTPC_OK) return s;
  if (!X || !amax || !Xq || !x_scale) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(amax) || !aligned16(Xq) || !aligned16(x_scale)) return PTPC_ERR_MISALIGNED;
  if ((s = check_device()) != PTPC_OK) return s;
  return cuda_status(
      ptpc::launch_quant_act_amax(X, (int)T, (int)Ci, ldx, amax, Xq, x_scale, (cudaStream_t)stream));
}

int ptpc_quantize_weights(const void *W, int64_t Ci, int64_t Co, uint8_t *Wq_t, float *w_scale, void *ws,
                          size_t ws_bytes, void *stream) {
  int s = check_shape_tci(0, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (!W || !Wq_t || !w_scale || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wq_t) || !aligned16(w_scale) || !aligned16(ws)) return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_QUANTIZE_WEIGHTS, 0, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  uint32_t *col_amax = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + kAlign);
  return cuda_status(
      ptpc::launch_quant_weight(W, (int)Ci, (int)Co, Wq_t, w_scale, col_amax, false, (cudaStream_t)stream));
}

int ptpc_scaled_mm(const uint8_t *Xq, const float *x_scale, const uint8_t *Wq_t, const float *w_scale, int64_t T,
                   int64_t Ci, int64_t Co, void *out, void *ws, size_t ws_bytes, void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if (!Xq || !x_scale || !Wq_t || !w_scale || !out || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(x_scale) || !aligned16(Wq_t) || !aligned16(w_scale) || !aligned16(out) ||
      !aligned16(ws))
    return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_SCALED_MM, T, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  return run_gemm(Xq, x_scale, Wq_t, w_scale, T, Ci, Co, out, false, static_cast<uint8_t *>(ws), gemm_ws(T, Ci, Co),
                  false, (cudaStream_t)stream);
}

int ptpc_linear(const void *X, int64_t ldx, const uint8_t *Wq_t, const float *w_scale, int64_t T, int64_t Ci,
                int64_t Co, void *out, void *ws, size_t ws_bytes, void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if ((s = check_ldx(ldx, Ci)) != PTPC_OK) return s;
  if (!X || !Wq_t || !w_scale || !out || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wq_t) || !aligned16(w_scale) || !aligned16(out) || !aligned16(ws))
    return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_LINEAR, T, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  uint8_t *wsp = static_cast<uint8_t *>(ws);
  const size_t gws = gemm_ws(T, Ci, Co);
  uint8_t *Xq = wsp + gws;
  float *xs = reinterpret_cast<float *>(wsp + gws + round_up((size_t)T * (size_t)Ci));
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = cuda_status(ptpc::launch_quant_act(X, (int)T, (int)Ci, ldx, Xq, xs, st))) != PTPC_OK) return s;
  return run_gemm(Xq, xs, Wq_t, w_scale, T, Ci, Co, out, false, wsp, gws, true, st);
}

size_t ptpc_weight_bytes(int fmt, int64_t Ci, int64_t Co) {
  if (!valid_wfmt(fmt) || check_shape_tci(0, Ci) != PTPC_OK || check_co(Co) != PTPC_OK) return 0;
  if (fmt != PTPC_WFMT_E4M3 && Ci % 128 != 0) return 0;
  return (size_t)Co * (size_t)Ci * (size_t)wfmt_bits(fmt) / 8;
}

int ptpc_quantize_weights_fmt(const void *W, int64_t Ci, int64_t Co, int fmt, uint8_t *Wq, float *w_scale, void *ws,
                              size_t ws_bytes, void *stream) {
  if (!valid_wfmt(fmt)) return PTPC_ERR_INVALID_ARG;
  if (fmt == PTPC_WFMT_E4M3) return ptpc_quantize_weights(W, Ci, Co, Wq, w_scale, ws, ws_bytes, stream);
  int s = check_shape_tci(0, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (!W || !Wq || !w_scale || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(w_scale) || !aligned16(ws)) return PTPC_ERR_MISALIGNED;
  if ((s = check_subbyte(fmt, Ci, Wq)) != PTPC_OK) return s;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_QUANTIZE_WEIGHTS, 0, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  uint32_t *col_amax = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + kAlign);
  return cuda_status(
      ptpc::launch_quant_weight_sub(W, (int)Ci, (int)Co, fmt, Wq, w_scale, col_amax, (cudaStream_t)stream));
}

int ptpc_scaled_mm_fmt(const uint8_t *Xq, const float *x_scale, const uint8_t *Wq, const float *w_scale, int fmt,
                       int64_t T, int64_t Ci, int64_t Co, void *out, void *ws, size_t ws_bytes, void *stream) {
  if (!valid_wfmt(fmt)) return PTPC_ERR_INVALID_ARG;
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if (!Xq || !x_scale || !Wq || !w_scale || !out || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(x_scale) || !aligned16(Wq) || !aligned16(w_scale) || !aligned16(out) ||
      !aligned16(ws))
    return PTPC_ERR_MISALIGNED;
  if ((s = check_subbyte(fmt, Ci, Wq)) != PTPC_OK) return s;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_SCALED_MM, T, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  return run_gemm(Xq, x_scale, Wq, w_scale, T, Ci, Co, out, false, static_cast<uint8_t *>(ws), gemm_ws(T, Ci, Co),
                  false, (cudaStream_t)stream, fmt);
}

int ptpc_linear_fmt(const void *X, int64_t ldx, const uint8_t *Wq, const float *w_scale, int fmt, int64_t T,
                    int64_t Ci, int64_t Co, void *out, void *ws, size_t ws_bytes, void *stream) {
  if (!valid_wfmt(fmt)) return PTPC_ERR_INVALID_ARG;
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if ((s = check_ldx(ldx, Ci)) != PTPC_OK) return s;
  if (!X || !Wq || !w_scale || !out || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wq) || !aligned16(w_scale) || !aligned16(out) || !aligned16(ws))
    return PTPC_ERR_MISALIGNED;
  if ((s = check_subbyte(fmt, Ci, Wq)) != PTPC_OK) return s;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_LINEAR, T, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  uint8_t *wsp = static_cast<uint8_t *>(ws);
  const size_t gws = gemm_ws(T, Ci, Co);
  uint8_t *Xq = wsp + gws;
  float *xs = reinterpret_cast<float *>(wsp + gws + round_up((size_t)T * (size_t)Ci));
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = cuda_status(ptpc::launch_quant_act(X, (int)T, (int)Ci, ldx, Xq, xs, st))) != PTPC_OK) return s;
  return run_gemm(Xq, xs, Wq, w_scale, T, Ci, Co, out, false, wsp, gws, true, st, fmt);
}

int ptpc_gemm_tail_split(int64_t T, int64_t Ci, int64_t Co, size_t ws_bytes) {
  if (check_shape_tci(T, Ci) != PTPC_OK || check_co(Co) != PTPC_OK || T == 0) return 0;
  if (check_device() != PTPC_OK) return 0;
  return ptpc::gemm_tail_split((int)T, (int)Ci, (int)Co, ws_bytes);
}

int ptpc_gemm_swap_tokens(int64_t T, int64_t Ci, int64_t Co, size_t ws_bytes) {
  if (check_shape_tci(T, Ci) != PTPC_OK || check_co(Co) != PTPC_OK || T == 0) return 0;
  if (check_device() != PTPC_OK) return 0;
  return ptpc::gemm_swap_tokens((int)T, (int)Ci, (int)Co, ws_bytes);
}

// ------------------------------------------------------------------ FP8 KV cache

namespace {
int check_kv_dims(int64_t H, int64_t D, int64_t block_size, int64_t num_blocks) {
  if (H <= 0 || D <= 0 || block_size <= 0 || num_blocks <= 0) return PTPC_ERR_INVALID_ARG;
  if ((D != 64 && D != 128) || H > 1024 || block_size < 8 || block_size > 65536 || num_blocks > kMaxDim)
    return PTPC_ERR_UNSUPPORTED_SHAPE;
  return PTPC_OK;
}
}  // namespace

int ptpc_kv_cache_append(const void *K, const void *V, const int64_t *slots, int64_t T, int64_t H, int64_t D,
                         int64_t block_size, int64_t num_blocks, uint8_t *k_cache, uint8_t *v_cache, float *k_scale,
                         float *v_scale, void *stream) {
  int s = check_kv_dims(H, D, block_size, num_blocks);
  if (s != PTPC_OK) return s;
  if (T < 0) return PTPC_ERR_INVALID_ARG;
  if (T > kMaxDim || T * H > kMaxDim) return PTPC_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return PTPC_OK;
  if (!K || !V || !slots || !k_cache || !v_cache || !k_scale || !v_scale) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(K) || !aligned16(V) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slots) & 7u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    return PTPC_ERR_MISALIGNED;
  if ((s = check_device()) != PTPC_OK) return s;
  return cuda_status(ptpc::launch_kv_append(K, V, slots, (int)T, (int)H, (int)D, num_blocks * block_size, k_cache,
                                            v_cache, k_scale, v_scale, (cudaStream_t)stream));
}

size_t ptpc_decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t D, int64_t max_context) {
  if (B <= 0 || Hq <= 0 || (D != 64 && D != 128) || max_context < 0 || max_context > kMaxDim) return 0;
  return round_up(ptpc::attn_workspace_bytes((int)B, (int)Hq, (int)D, (int)max_context));
}

int ptpc_decode_attention(const void *q, const uint8_t *k_cache, const uint8_t *v_cache, const float *k_scale,
                          const float *v_scale, const int32_t *block_tables, const int32_t *context_lens, int64_t B,
                          int64_t Hq, int64_t Hkv, int64_t D, int64_t block_size, int64_t num_blocks,
                          int64_t max_blocks, int64_t max_context, float softmax_scale, void *out, void *ws,
                          size_t ws_bytes, void *stream) {
  int s = check_kv_dims(Hkv, D, block_size, num_blocks);
  if (s != PTPC_OK) return s;
  if (B < 0 || Hq <= 0 || max_blocks <= 0 || max_context < 0) return PTPC_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || Hq / Hkv > 16 || B > 65535 || Hkv > 65535 || max_context > kMaxDim ||
      max_blocks > kMaxDim / block_size || num_blocks > kMaxDim / block_size)
    return PTPC_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return PTPC_OK;
  if (!q || !k_cache || !v_cache || !k_scale || !v_scale || !block_tables || !context_lens || !out || !ws)
    return PTPC_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) || (reinterpret_cast<uintptr_t>(context_lens) & 3u))
    return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_decode_attention_workspace_size(B, Hq, D, max_context)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  return cuda_status(ptpc::launch_decode_attention(q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens,
                                                   (int)B, (int)Hq, (int)Hkv, (int)D, (int)block_size,
                                                   (int)max_blocks, num_blocks * block_size, (int)max_context,
                                                   softmax_scale, out, ws, (cudaStream_t)stream));
}

int ptpc_decode_attention_kernel(int64_t Hq, int64_t Hkv, int64_t D, int64_t block_size) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || Hq / Hkv > 16 || (D != 64 && D != 128) || block_size <= 0 ||
      block_size > kMaxDim)
    return 0;
  return ptpc::attn_kernel_choice((int)D, (int)(Hq / Hkv), (int)block_size);
}

int ptpc_gemm_ksplit(int64_t T, int64_t Ci, int64_t Co) {
  if (check_shape_tci(T, Ci) != PTPC_OK || check_co(Co) != PTPC_OK || T == 0) return 0;
  if (check_device() != PTPC_OK) return 0;
  return ptpc::gemm_ksplit((int)T, (int)Ci, (int)Co);
}

int ptpc_reload_tuning_overrides(void) {
  ptpc::reload_tuning();
  ptpc::attn_reload_tuning();
  return PTPC_OK;
}

int ptpc_bench_map_cache_selftest(void) { return ptpc::map_cache_selftest() == 0 ? PTPC_OK : PTPC_ERR_INVALID_ARG; }

int ptpc_bench_map_cache_stats(uint64_t *hits, uint64_t *misses) {
  if (!hits || !misses) return PTPC_ERR_INVALID_ARG;
  ptpc::map_cache_stats(hits, misses);
  return PTPC_OK;
}

int ptpc_selftest_wait_timeout(void *ws, void *stream) {
  if (!ws) return PTPC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PTPC_ERR_MISALIGNED;
  int s = check_device();
  if (s != PTPC_OK) return s;
  return cuda_status(ptpc::launch_wait_timeout_selftest(static_cast<uint32_t *>(ws), (cudaStream_t)stream));
}

int ptpc_get_device_status(void *ws, void *stream) {
  if (!ws) return PTPC_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PTPC_ERR_CUDA;
  if (cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return PTPC_ERR_CUDA;
  if (v == 0) return PTPC_OK;
  if (cudaMemset(ws, 0, sizeof v) != cudaSuccess) return PTPC_ERR_CUDA;
  return PTPC_ERR_DEVICE_TIMEOUT;
}

int ptpc_bench_unscaled_mm_f32(const uint8_t *Xq, const uint8_t *Wq_t, int64_t T, int64_t Ci, int64_t Co, float *y,
                               void *ws, size_t ws_bytes, void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if (!Xq || !Wq_t || !y || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(Wq_t) || !aligned16(y) || !aligned16(ws)) return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_BENCH_UNSCALED_MM, T, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  return run_gemm(Xq, nullptr, Wq_t, nullptr, T, Ci, Co, y, true, static_cast<uint8_t *>(ws), kGemmWorkspace,
                  false, (cudaStream_t)stream);
}

int ptpc_bench_clock_probe(uint64_t *records_dev, int max_records, uint64_t period_ns, uint64_t duration_ns,
                           int *count_dev, void *stream) {
  if (!records_dev || !count_dev || max_records < 2) return PTPC_ERR_INVALID_ARG;
  if (period_ns < 1000 || duration_ns > 120ull * 1000000000ull) return PTPC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(records_dev) & 7u) != 0 || (reinterpret_cast<uintptr_t>(count_dev) & 3u) != 0)
    return PTPC_ERR_MISALIGNED;
  int s = check_device();
  if (s != PTPC_OK) return s;
  return cuda_status(ptpc::launch_clock_probe(reinterpret_cast<unsigned long long *>(records_dev), max_records,
                                              period_ns, duration_ns, count_dev, (cudaStream_t)stream));
}

int ptpc_bench_apply_scales(const float *y, const float *x_scale, const float *w_scale, int64_t T, int64_t Co,
                            void *out, void *stream) {
  int s = check_co(Co);
  if (s != PTPC_OK) return s;
  if (T < 0) return PTPC_ERR_INVALID_ARG;
  if (T > kMaxDim) return PTPC_ERR_UNSUPPORTED_SHAPE;
  if (T == 0) return PTPC_OK;
  if (!y || !x_scale || !w_scale || !out) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(y) || !aligned16(x_scale) || !aligned16(w_scale) || !aligned16(out)) return PTPC_ERR_MISALIGNED;
  if ((s = check_device()) != PTPC_OK) return s;
  return cuda_status(ptpc::launch_apply_scales(y, x_scale, w_scale, (int)T, (int)Co, out, (cudaStream_t)stream));
}

int ptpc_bench_quantize_activations_per_tensor(const void *X, int64_t T, int64_t Ci, int64_t ldx, uint8_t *Xq,
                                               float *x_scale, void *ws, size_t ws_bytes, void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if ((s = check_ldx(ldx, Ci)) != PTPC_OK) return s;
  if (!X || !Xq || !x_scale || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xq) || !aligned16(x_scale) || !aligned16(ws)) return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_BENCH_PER_TENSOR, T, Ci, 0)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  uint32_t *slot = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + kAlign);
  return cuda_status(
      ptpc::launch_quant_act_per_tensor(X, (int)T, (int)Ci, ldx, Xq, x_scale, slot, (cudaStream_t)stream));
}

int ptpc_bench_quantize_weights_per_tensor(const void *W, int64_t Ci, int64_t Co, uint8_t *Wq_t, float *w_scale,
                                           void *ws, size_t ws_bytes, void *stream) {
  int s = check_shape_tci(0, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (!W || !Wq_t || !w_scale || !ws) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wq_t) || !aligned16(w_scale) || !aligned16(ws)) return PTPC_ERR_MISALIGNED;
  if (ws_bytes < ptpc_workspace_size(PTPC_OP_QUANTIZE_WEIGHTS, 0, Ci, Co)) return PTPC_ERR_WORKSPACE_TOO_SMALL;
  if ((s = check_device()) != PTPC_OK) return s;
  uint32_t *col_amax = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + kAlign);
  return cuda_status(
      ptpc::launch_quant_weight(W, (int)Ci, (int)Co, Wq_t, w_scale, col_amax, true, (cudaStream_t)stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Scaled GEMM with library-owned scratch (no allocation by the caller).
//
// Some callers cannot allocate device memory when they call the GEMM: an
// inference engine that partitions all of its device memory once at start-up
// and forbids allocation on the serving path, or a host integration that only
// hands over input and output buffers.  This entry point needs no workspace
// from them: its scratch (the GEMM's device status word) lives in the
// file-scope array below, which every GPU that loads this library holds until
// the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = 4096;  // per device

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// Device address of g_static_scratch for the current device.  In host code
// the name g_static_scratch is only a host-side stand-in; the real address is
// obtained once per device with that device current.
int static_scratch_address(uint8_t **out) {
  static std::mutex mu;
  static uint8_t *addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PTPC_ERR_CUDA;
  if (dev < 0 || dev >= 64) return PTPC_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return PTPC_ERR_CUDA;
    addr[dev] = static_cast<uint8_t *>(p);
  }
  *out = addr[dev];
  return PTPC_OK;
}

}  // namespace

static_assert(kGemmWorkspace <= kStaticScratchBytes, "the GEMM's scratch must fit in the static array");

extern "C" int ptpc_scaled_mm_static_scratch(const uint8_t *Xq, const float *x_scale, const uint8_t *Wq_t,
                                             const float *w_scale, int64_t T, int64_t Ci, int64_t Co, void *out,
                                             void *stream) {
  int s = check_shape_tci(T, Ci);
  if (s != PTPC_OK) return s;
  if ((s = check_co(Co)) != PTPC_OK) return s;
  if (T == 0) return PTPC_OK;
  if (!Xq || !x_scale || !Wq_t || !w_scale || !out) return PTPC_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(x_scale) || !aligned16(Wq_t) || !aligned16(w_scale) || !aligned16(out))
    return PTPC_ERR_MISALIGNED;
  if ((s = check_device()) != PTPC_OK) return s;
  uint8_t *scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != PTPC_OK) return s;
  // The GEMM only ORs timeout bits into the status word at the start of the
  // array and needs nothing else to start at zero.  The word is not cleared
  // here, so a timeout stays recorded until ptpc_static_scratch_status reads
  // it (the array is zero when the library is loaded).
  return run_gemm(Xq, x_scale, Wq_t, w_scale, T, Ci, Co, out, false, scratch, kStaticScratchBytes, false,
                  (cudaStream_t)stream);
}

extern "C" int ptpc_static_scratch_status(void *stream) {
  int s = check_device();
  if (s != PTPC_OK) return s;
  uint8_t *scratch = nullptr;
  if ((s = static_scratch_address(&scratch)) != PTPC_OK) return s;
  return ptpc_get_device_status(scratch, stream);
}
