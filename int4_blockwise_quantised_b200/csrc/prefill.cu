// decoder_init (prefill) ("vibevoice-asr-bitnet-onnx": decoder_init owns the embedding table and
// writes audio_features over the <|speech_pad|> rows starting at audio_offset; present K/V of all
// S positions; logits of the last position).
//
// This translation unit holds the embedding gather + audio splice and the prefill driver.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "decoder_state.h"

namespace vv {
namespace {

// out[i] = audio[i - off] for off <= i < off + N, else embed[ids[i]] (fp16 rows of H).
__global__ void __launch_bounds__(256) splice_kernel(const int32_t* __restrict__ ids, int S,
                                                     const uint16_t* __restrict__ embed, int V,
                                                     int H, const uint16_t* __restrict__ audio,
                                                     int N, int off, uint16_t* __restrict__ out) {
  const int row = blockIdx.x;
  if (row >= S) return;
  const uint4* src;
  if (row >= off && row < off + N) {
    src = reinterpret_cast<const uint4*>(audio + (size_t)(row - off) * H);
  } else {
    int id = ids[row];
    if (id < 0 || id >= V) {
      if (threadIdx.x == 0) set_device_error(VV_ERR_RANGE);
      id = min(max(id, 0), V - 1);
    }
    src = reinterpret_cast<const uint4*>(embed + (size_t)id * H);
  }
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * H);
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) dst[i] = src[i];
}

}  // namespace

cudaError_t prefill_run(vv_decoder* d, const int32_t* ids, const int32_t* pos, int S,
                        const uint16_t* audio, int N, int off, float* logits, int32_t* argmax,
                        cudaStream_t s) {
  const vv_config& c = d->cfg;
  const size_t need = (size_t)c.max_prefill * c.hidden * 2;
  if (d->pws_bytes < need) {
    if (d->pws) cudaFree(d->pws);
    d->pws = nullptr;
    d->pws_bytes = 0;
    cudaError_t e = cudaMalloc(&d->pws, need);
    if (e != cudaSuccess) return e;
    d->pws_bytes = need;
  }
  uint16_t* embeds = reinterpret_cast<uint16_t*>(d->pws);
  splice_kernel<<<S, 256, 0, s>>>(ids, S, d->embed, c.vocab, c.hidden, audio, N, off, embeds);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  set_int_kernel<<<1, 1, 0, s>>>(d->d_length, 0);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int i = 0; i < S; ++i) {
    const bool last = i == S - 1;
    e = enqueue_step(d, embeds + (size_t)i * c.hidden, nullptr, pos + i, last ? logits : nullptr,
                     last ? argmax : nullptr, s, last, nullptr);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace vv
