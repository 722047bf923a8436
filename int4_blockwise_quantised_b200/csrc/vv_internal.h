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

// Standalone MatMulNBits GEMV: y[m, n] = x[m, :] . W[n, :] (+bias) in fp16, M <= 8.
cudaError_t launch_matmul_nbits_gemv(const uint16_t* x, GemvWeights w, const uint16_t* bias,
                                     int M, int N, int K, uint16_t* y, cudaStream_t s);

// Attention (attn.cu) ------------------------------------------------------------------------
struct AttnArgs {
  const uint16_t* q_f16;  // fp16 [Hq, D], already rotated
  uint16_t* k_cache;      // [Hkv, cap, D]
  uint16_t* v_cache;
  int len;                // valid positions
  int cap, Hq, Hkv;
  float scale;
  uint16_t* out_f16;  // [Hq, D]
  float* ws_part;     // partials
  int* ws_count;      // per kv-head arrival counters
  int nchunks;
};
size_t attn_workspace_bytes(int Hq, int Hkv, int nchunks);
int attn_default_chunks(int Hkv, int cap);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t s);

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
