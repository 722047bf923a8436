// Causal GQA attention of the prefill (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace vv {

struct AttnPrefillArgs {
  const uint16_t* q;        // fp16 [S, Hq, D] rotated queries
  const uint16_t* k_cache;  // fp16 [Hkv, cap, D] of this layer (positions 0..S-1 written)
  const uint16_t* v_cache;
  uint16_t* out;            // fp16 [S, Hq * D]
  int S, cap, Hq, Hkv;
  float scale;
};

cudaError_t launch_attn_prefill(const AttnPrefillArgs& a, cudaStream_t s);

}  // namespace vv
