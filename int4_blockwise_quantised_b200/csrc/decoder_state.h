// Decoder state shared by decoder.cu and prefill.cu (not part of the public ABI).
#pragma once

#include <cuda_runtime.h>

#include <vector>

#include "../../include/vv.h"
#include "step.h"

struct vv_decoder {
  vv_config cfg;
  std::vector<vv_layer_weights> layers;
  const uint16_t* embed = nullptr;
  const uint16_t* lm_head = nullptr;
  const uint16_t* final_norm = nullptr;
  uint16_t* k_cache = nullptr;
  uint16_t* v_cache = nullptr;
  int device = 0;

  unsigned char* ws = nullptr;
  size_t ws_bytes = 0;
  float* rope_cos = nullptr;
  float* rope_sin = nullptr;
  int32_t* d_length = nullptr;
  int32_t* d_argmax = nullptr;
  int32_t* d_gen = nullptr;  // [done, count, position] of vv_decoder_generate
  // prefill's final norm + lm_head: fp32 residual of the last position and argmax partials
  float* x_last = nullptr;
  float* lm_val = nullptr;
  int* lm_idx = nullptr;
  int* lm_count = nullptr;
  // prefill workspace (allocated lazily by the prefill path)
  unsigned char* pws = nullptr;
  size_t pws_bytes = 0;
  // scales the prefill GEMMs read, [layer * 7 + matrix] (wq wk wv wo wgate wup wdown), with row
  // pitch pf_pitch[matrix] in elements (0: K/32).  A matrix whose K/32 is not a multiple of 8
  // reads a copy with the pitch padded to 8 blocks (pf_pad, owned).
  std::vector<const uint16_t*> pf_scales;
  int pf_pitch[7] = {0, 0, 0, 0, 0, 0, 0};
  uint16_t* pf_pad = nullptr;

  int nb = 1;                       // sequences stepped together (batch)
  int32_t len_host[2] = {0, 0};     // host copy of each sequence's length
  int32_t max_len() const { return nb > 1 && len_host[1] > len_host[0] ? len_host[1] : len_host[0]; }
  void advance_lengths(int32_t n) {
    for (int b = 0; b < nb; ++b) len_host[b] += n;
  }
  float* trace = nullptr;
  bool use_graph = true;
  vv::StepParams step = {};        // persistent-kernel parameters (per-call pointers patched)
  vv::StepLayer* d_layers = nullptr;
  cudaGraphExec_t gexec = nullptr;
  cudaStream_t capture_stream = nullptr;  // graphs are captured here, launched on the caller's
  const void* gkey[6] = {nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
};


namespace vv {
// Optional event trail of one prefill: an event after every launch, tagged with the launch's
// kind (kPfMisc: splice / norm / RoPE / copies, kPfDequant, kPfGemm, kPfAttn, kPfHead).
enum { kPfMisc = 0, kPfDequant = 1, kPfGemm = 2, kPfAttn = 3, kPfHead = 4, kPfKinds = 5 };
struct PrefillTimer {
  std::vector<cudaEvent_t> ev;
  std::vector<int> kind;
};
__global__ void set_int_kernel(int32_t* p, int32_t v);
__global__ void add_int_kernel(int32_t* p, int32_t v);
// Enqueue one decode step: one launch of the persistent step kernel.
cudaError_t enqueue_step(vv_decoder* d, const uint16_t* embeds, const int32_t* token,
                         const int32_t* position, float* logits, int32_t* argmax, cudaStream_t s);
// Prefill preparation at create: the pf_scales table (and padded scale copies where needed).
cudaError_t prefill_prepare(vv_decoder* d);
cudaError_t prefill_run(vv_decoder* dec, int seq, const int32_t* ids, const int32_t* pos, int S,
                        const uint16_t* audio, int N, int off, float* logits, int32_t* argmax,
                        cudaStream_t s, PrefillTimer* timer = nullptr);
}  // namespace vv
