// Parameters of the persistent decode-step kernel (internal).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vv {

// Rows of the o-projection handled by one o-item (head h, row block): the item multiplies the
// 128 columns of head h (four 32-blocks) by rows [kORows * rb, kORows * rb + kORows).
constexpr int kORows = 128;
// Gate/up rows per slice: a CTA computes h for a slice of kSlice intermediate channels and then
// the matching kSlice columns (two 32-blocks) of the down projection for every output row.
constexpr int kSlice = 64;

struct StepLayer {
  const __half* in_norm;
  const __half* post_norm;
  const uint8_t* q[7];   // wq, wk, wv, wo, wgate, wup, wdown codes (caller's MatMulNBits layout)
  const __half* s[7];    // their scales
  const __half* bias[3]; // bq, bk, bv
  // Column images made at decoder creation (see step_wo_image / step_wd_image):
  const unsigned char* wo_img;  // items (head h, row block rb), kORows x 4 blocks each
  const unsigned char* wd_img;  // per CTA: H rows x (2 x its slices) blocks
};

// Batch: nb sequences are stepped together (nb <= step_max_batch()); every weight byte is read
// once for all of them.  Per-sequence buffers are laid out sequence-major: input_embeds [nb][H],
// token / position / argmax / length [nb], logits [nb][V], x_acc [nb][H], qkv [nb][nqkv],
// attn_part [nb][Hkv][max_tiles][8][132], head_val / head_idx [nb][grid], caches
// [L][nb][Hkv][cap][D].
struct StepParams {
  int H, L, Hq, Hkv, I, V;
  int nb;
  float eps, scale;
  const StepLayer* layers;  // device array [L]
  const __half* embed;
  const __half* lm_head;
  const __half* final_norm;
  void* k_cache;  // [L][nb][Hkv][cap][D] of the storage type kv_type
  void* v_cache;
  int kv_type;    // 0 fp16, 1 bf16, 2 fp32 (VV_KV_*)
  int cap;
  const float* rope_cos;
  const float* rope_sin;
  int max_position;
  // per-step inputs / outputs
  const __half* input_embeds;  // or nullptr -> embed[*token]
  const int32_t* token;
  const int32_t* position;
  float* logits;     // may be nullptr
  int32_t* argmax;
  float* trace;      // [L, H] or nullptr
  // workspace
  unsigned long long* x_acc;  // [H] residual stream, fixed point (2^-32 units)
  float* qkv;
  float* attn_part;
  int max_tiles;
  float* head_val;
  int* head_idx;
  int* head_count;
  int32_t* length;
  unsigned* bar_count;
  // greedy generation (vv_decoder_generate), all null otherwise: a launch finding *gen_done set
  // returns at once; else its last CTA counts the token (*gen_count), advances *position (which
  // then points at the generation's own position word) and sets *gen_done on a stop id.
  int32_t* gen_done;
  int32_t* gen_count;
  int32_t* gen_pos;
  int32_t stop_ids[8];
  int n_stop;
  uint64_t wait_ns;   // bound of every device-side wait (ns)
  uint64_t* stamps;   // timeline tap [grid][max_stamps] (globaltimer ns) or nullptr
  int max_stamps;
  // launch shape
  int grid;
  int stage_bytes;
  int nstages;
};

size_t step_smem_bytes(const StepParams& p);
int step_threads();
size_t step_attn_part_floats(int Hkv, int max_tiles);
int step_max_tiles(int cap);
cudaError_t step_configure(StepParams& p, int* blocks_per_sm);
void step_func_info(int nb, int* regs, int* max_threads, int* static_smem, int* local_bytes);
// Largest batch (sequences per step) of the step kernel.
int step_max_batch();
cudaError_t launch_step(const StepParams& p, cudaStream_t s);
// Column images: bytes per layer, and the kernels that build them from the caller's matrices.
size_t step_wo_image_bytes(int H, int Hq);
size_t step_wd_image_bytes(int H, int I, int grid);
cudaError_t step_build_images(const StepParams& p, const StepLayer* host_layers,
                              unsigned char* wo_img, unsigned char* wd_img, cudaStream_t s);
constexpr int kMaxStopIds = 8;
// Entries per CTA the timeline tap needs for a model of L layers: 15 L + 3 stamps and 8 trailing
// counters.
inline int step_timeline_stamps(int L) { return 15 * L + 3 + 8; }

}  // namespace vv
