// Host-side internals shared by the libvv translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <utility>

#include "../../include/vv.h"

namespace vv {

// Record an error for vv_last_error() and return its code.
vv_status set_error(vv_status code, const char* fmt, ...);
// Record a CUDA failure (if any) and return VV_ERR_CUDA, else VV_OK.
vv_status cuda_check(cudaError_t e, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define VV_CUDA(call)                                         \
  do {                                                        \
    vv_status _s = ::vv::cuda_check((call), #call);           \
    if (_s != VV_OK) return _s;                               \
  } while (0)

#define VV_CHECK_ARG(cond, ...)                                          \
  do {                                                                   \
    if (!(cond)) return ::vv::set_error(VV_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define VV_CHECK_SHAPE(cond, ...)                                  \
  do {                                                             \
    if (!(cond)) return ::vv::set_error(VV_ERR_SHAPE, __VA_ARGS__); \
  } while (0)

// Number of SMs of the current device (cached per device).
int sm_count();

// Launch with the programmatic-stream-serialization attribute when `pdl` is set.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   cudaStream_t stream, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------------ kernel launchers
// GEMV family (gemv.cu).  Each returns a CUDA error code of the launch.

struct GemvWeights {
  const uint8_t* q;
  const uint16_t* scales;
};

// y[n] = W[n, :] . xn + bias, W = [Wq; Wk; Wv] as three matrices (rows nq, nk, nv), K = H,
// xn = RMSNorm(x) with gamma. x source: x_f32 (residual) or, when embed != nullptr, the fp16
// embedding row (input_embeds, or embed_table[*token]); in that case the kernel also writes
// the residual x_resid = row.
struct QkvArgs {
  GemvWeights w[3];
  int rows[3];
  const uint16_t* bias[3];
  int K;
  const float* x_resid_in;      // fp32 [K] or nullptr when reading the embedding
  const uint16_t* embeds;       // fp16 [K] input_embeds, or nullptr
  const uint16_t* embed_table;  // fp16 [V, K] with token, or nullptr
  const int32_t* token;
  int vocab;
  float* x_resid_out;  // written when the embedding is the source
  const uint16_t* gamma;
  float eps;
  float* out;  // fp32 [rows0 + rows1 + rows2]
};
cudaError_t launch_qkv(const QkvArgs& a, cudaStream_t s, bool pdl);

// x_resid[n] += W[n, :] . x  (x fp32 [K], no norm).  Optional trace copy of the updated rows.
struct ResidArgs {
  GemvWeights w;
  int N, K;
  const float* x;
  float* x_resid;
  float* trace;  // fp32 [N] or nullptr: receives the updated residual rows
};
cudaError_t launch_resid(const ResidArgs& a, cudaStream_t s, bool pdl);

// h[n] = silu(Wg[n,:] . xn) * (Wu[n,:] . xn),  xn = RMSNorm(x_resid) with gamma.
struct GateUpArgs {
  GemvWeights wg, wu;
  int N, K;
  const float* x_resid;
  const uint16_t* gamma;
  float eps;
  float* h;  // fp32 [N]
};
cudaError_t launch_gateup(const GateUpArgs& a, cudaStream_t s, bool pdl);

// Standalone MatMulNBits GEMV: y[m, n] = x[m, :] . W[n, :] (+bias) in fp16, M <= 8.
cudaError_t launch_matmul_nbits_gemv(const uint16_t* x, GemvWeights w, const uint16_t* bias,
                                     int M, int N, int K, uint16_t* y, cudaStream_t s);

// Attention (attn.cu) ------------------------------------------------------------------------
struct AttnArgs {
  // standalone: q fp16 [Hq, D] rotated, all `len` positions in the cache.
  const uint16_t* q_f16;
  // fused decoder mode: q/k/v fp32 pre-RoPE from the QKV GEMV ([Hq*D | Hkv*D | Hkv*D]);
  // rotates q and k at *position, appends k/v at slot *length, attends over *length + 1.
  const float* qkv;
  const int32_t* position;
  const int32_t* length;
  const float* rope_cos;  // [max_position, D/2]
  const float* rope_sin;
  int max_position;
  uint16_t* k_cache;  // [Hkv, cap, D] of this layer
  uint16_t* v_cache;
  int len;  // standalone: valid positions
  int cap, Hq, Hkv;
  float scale;
  uint16_t* out_f16;  // standalone output [Hq, D]
  float* out_f32;     // fused output [Hq*D]
  float* ws_part;     // partials
  int* ws_count;      // per kv-head arrival counters
  int nchunks;
};
size_t attn_workspace_bytes(int Hq, int Hkv, int nchunks);
int attn_default_chunks(int Hkv, int cap);
cudaError_t launch_attn(const AttnArgs& a, bool fused, cudaStream_t s, bool pdl);

// lm_head (lmhead.cu) ---------------------------------------------------------------------
struct LmHeadArgs {
  const float* x;
  const uint16_t* gamma;
  const uint16_t* w;
  int V, H;
  float eps;
  float* logits;     // may be nullptr
  int32_t* idx;      // [1]
  float* ws_val;     // [grid] partial maxima
  int* ws_idx;       // [grid]
  int* ws_count;     // [1]
  int32_t* length;   // when non-null, the last CTA increments *length (decoder step)
};
int lm_head_grid(int V);
size_t lm_head_workspace_bytes(int V);
cudaError_t launch_lm_head(const LmHeadArgs& a, cudaStream_t s, bool pdl);

}  // namespace vv
