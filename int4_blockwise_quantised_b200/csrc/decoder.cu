// The decoder object: decoder_step / decoder_init of the Qwen2 backbone
// ("vibevoice-asr-bitnet-onnx": decoder_init / decoder_step I/O listing; "VibeVoice-1.5B —
// Current Status", section "Architecture": pre-norm Qwen2 with q/k/v bias, GQA).
//
// Step = 5 kernels per layer + 1:
//   qkv   : RMSNorm(x) -> [Wq;Wk;Wv] int4 GEMV + bias (layer 0 reads the embedding row)
//   attn  : RoPE(q,k) at position, append k/v at slot `length`, split-K GQA attention
//   o     : x += Wo . attn
//   gateup: RMSNorm(x) -> gate/up int4 GEMV -> silu(g) * u
//   down  : x += Wd . h
//   head  : RMSNorm(x) -> fp16 lm_head GEMV -> logits, argmax; length += 1
// The residual x stays fp32 in the workspace.  Position and length live in device memory, so the
// whole step is captured once as a CUDA graph and replayed ("VibeVoice-ASR — ONNX export for
// Vernacula", section "Highlights": ~1950 launches per step of framework overhead under ONNX
// Runtime).  Every kernel after the first is launched with programmatic dependent launch so its
// weight prefetch overlaps the previous kernel.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <algorithm>
#include <cstring>
#include <new>
#include <vector>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "decoder_state.h"

namespace vv {

__global__ void set_int_kernel(int32_t* p, int32_t v) { *p = v; }
__global__ void add_int_kernel(int32_t* p, int32_t v) { *p += v; }

namespace {
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
}  // namespace

cudaError_t enqueue_step(vv_decoder* d, const uint16_t* embeds, const int32_t* token,
                         const int32_t* position, float* logits, int32_t* argmax,
                         cudaStream_t s) {
  StepParams p = d->step;
  p.input_embeds = reinterpret_cast<const __half*>(embeds);
  p.token = token;
  p.position = position;
  p.logits = logits;
  p.argmax = argmax ? argmax : d->d_argmax;
  p.trace = d->trace;
  return launch_step(p, s);
}

}  // namespace vv

using vv::set_error;

extern "C" {

vv_status vv_decoder_create(const vv_config* cfg, const vv_model_weights* w, uint16_t* k_cache,
                            uint16_t* v_cache, vv_decoder** out) {
  VV_CHECK_ARG(cfg && w && k_cache && v_cache && out && w->layers, "vv_decoder_create: null");
  *out = nullptr;
  const vv_config& c = *cfg;
  VV_CHECK_SHAPE(c.head_dim == 128, "head_dim %d (only 128)", c.head_dim);
  VV_CHECK_SHAPE(c.kv_dtype == VV_KV_F16 || c.kv_dtype == VV_KV_BF16 || c.kv_dtype == VV_KV_F32,
                 "kv_dtype %d", c.kv_dtype);
  VV_CHECK_SHAPE(c.batch >= 0 && c.batch <= vv::step_max_batch(), "batch %d (1 .. %d)", c.batch,
                 vv::step_max_batch());

  VV_CHECK_SHAPE(c.kv_dtype == VV_KV_F16 || c.max_prefill == 0,
                 "kv_dtype %d: the prefill (max_prefill > 0) writes an fp16 cache only", c.kv_dtype);
  VV_CHECK_SHAPE(c.n_kv >= 1 && c.n_kv <= 64 && c.n_q % c.n_kv == 0 && c.n_q / c.n_kv <= 8,
                 "n_q %d / n_kv %d", c.n_q, c.n_kv);
  VV_CHECK_SHAPE(c.hidden >= 128 && c.hidden % 128 == 0 && c.hidden <= 7680, "hidden %d",
                 c.hidden);
  VV_CHECK_SHAPE(c.inter >= 64 && c.inter % 256 == 0 && c.inter <= 65536, "inter %d", c.inter);
  VV_CHECK_SHAPE(c.n_q * c.head_dim <= 7680, "n_q*D %d", c.n_q * c.head_dim);
  VV_CHECK_SHAPE(c.layers >= 1 && c.vocab >= 1 && c.kv_capacity >= 1 && c.max_position >= 1 &&
                     c.max_prefill >= 0,
                 "layers/vocab/capacity/max_position");
  VV_CHECK_ARG(w->embed && w->lm_head && w->final_norm, "embed/lm_head/final_norm null");
  VV_CHECK_ARG(vv::aligned16(k_cache) && vv::aligned16(v_cache) && vv::aligned16(w->lm_head) &&
                   vv::aligned16(w->embed) && vv::aligned16(w->final_norm),
               "cache / table pointers must be 16-byte aligned");
  for (int l = 0; l < c.layers; ++l) {
    const vv_layer_weights& L = w->layers[l];
    const vv_packed_matrix* m[7] = {&L.wq, &L.wk, &L.wv, &L.wo, &L.wgate, &L.wup, &L.wdown};
    for (auto* p : m)
      VV_CHECK_ARG(p->q && p->scales && vv::aligned16(p->q) && vv::aligned16(p->scales),
                   "layer %d: packed weight null or not 16-byte aligned", l);
    VV_CHECK_ARG(L.input_norm && L.post_norm, "layer %d: norm gain null", l);
    // the kernels read gains and biases as vectors
    VV_CHECK_ARG(vv::aligned16(L.input_norm) && vv::aligned16(L.post_norm) &&
                     (!L.bq || vv::aligned16(L.bq)) && (!L.bk || vv::aligned16(L.bk)) &&
                     (!L.bv || vv::aligned16(L.bv)),
                 "layer %d: norm gain or bias not 16-byte aligned", l);
  }

  vv_decoder* d = new (std::nothrow) vv_decoder();
  if (!d) return set_error(VV_ERR_CUDA, "out of host memory");
  d->cfg = c;
  d->layers.assign(w->layers, w->layers + c.layers);
  d->embed = w->embed;
  d->lm_head = w->lm_head;
  d->final_norm = w->final_norm;
  d->k_cache = k_cache;
  d->v_cache = v_cache;
  cudaGetDevice(&d->device);

  const int H = c.hidden, D = c.head_dim;
  const int NB = c.batch > 1 ? c.batch : 1;
  d->nb = NB;
  const int grid = vv::sm_count();
  const int max_tiles = vv::step_max_tiles(c.kv_capacity);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = vv::align_up(off + bytes, 256);
    return o;
  };
  const size_t o_x = take((size_t)NB * H * 8);
  const size_t o_qkv = take((size_t)NB * (c.n_q + 2 * c.n_kv) * D * 4);
  const size_t o_cos = take((size_t)c.max_position * (D / 2) * 4);
  const size_t o_sin = take((size_t)c.max_position * (D / 2) * 4);
  const size_t o_len = take(16);
  const size_t o_arg = take(16);
  const size_t o_gen = take(16);  // generation: done flag, token count, position
  const size_t o_part = take((size_t)NB * vv::step_attn_part_floats(c.n_kv, max_tiles) * 4);
  const size_t o_hval = take((size_t)NB * grid * 4);
  const size_t o_hidx = take((size_t)NB * grid * 4);
  const size_t o_hcnt = take(16);
  const size_t o_bar = take(16);
  const size_t o_layers = take(sizeof(vv::StepLayer) * c.layers);
  const int lm_grid = vv::lm_head_grid(c.vocab);
  const size_t o_xl = take((size_t)H * 4);
  const size_t o_lmv = take((size_t)lm_grid * 4);
  const size_t o_lmi = take((size_t)lm_grid * 4);
  const size_t o_lmc = take(16);
  // column images of Wo and Wd (the o-proj and down phases read column blocks)
  const size_t wo_b = vv::step_wo_image_bytes(H, c.n_q);
  const size_t wd_b = vv::step_wd_image_bytes(H, c.inter, grid);
  const size_t o_wo = take(wo_b * c.layers);
  const size_t o_wd = take(wd_b * c.layers);
  d->ws_bytes = off;
  vv_status st = vv::cuda_check(cudaMalloc(&d->ws, d->ws_bytes), "cudaMalloc(decoder workspace)");
  if (st) {
    delete d;
    return st;
  }
  st = vv::cuda_check(cudaMemset(d->ws, 0, d->ws_bytes), "cudaMemset");
  unsigned char* b = d->ws;
  d->rope_cos = reinterpret_cast<float*>(b + o_cos);
  d->rope_sin = reinterpret_cast<float*>(b + o_sin);
  d->d_length = reinterpret_cast<int32_t*>(b + o_len);
  d->d_argmax = reinterpret_cast<int32_t*>(b + o_arg);
  d->d_gen = reinterpret_cast<int32_t*>(b + o_gen);
  d->x_last = reinterpret_cast<float*>(b + o_xl);
  d->lm_val = reinterpret_cast<float*>(b + o_lmv);
  d->lm_idx = reinterpret_cast<int*>(b + o_lmi);
  d->lm_count = reinterpret_cast<int*>(b + o_lmc);

  {
    vv::StepParams& p = d->step;
    p.H = H;
    p.nb = NB;
    p.L = c.layers;
    p.Hq = c.n_q;
    p.Hkv = c.n_kv;
    p.I = c.inter;
    p.V = c.vocab;
    p.eps = c.eps;
    p.scale = 1.0f / sqrtf((float)D);
    d->d_layers = reinterpret_cast<vv::StepLayer*>(b + o_layers);
    p.layers = d->d_layers;
    p.embed = reinterpret_cast<const __half*>(w->embed);
    p.lm_head = reinterpret_cast<const __half*>(w->lm_head);
    p.final_norm = reinterpret_cast<const __half*>(w->final_norm);
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.kv_type = c.kv_dtype;
    p.cap = c.kv_capacity;
    p.rope_cos = d->rope_cos;
    p.rope_sin = d->rope_sin;
    p.max_position = c.max_position;
    p.x_acc = reinterpret_cast<unsigned long long*>(b + o_x);
    p.qkv = reinterpret_cast<float*>(b + o_qkv);
    p.attn_part = reinterpret_cast<float*>(b + o_part);
    p.max_tiles = max_tiles;
    p.head_val = reinterpret_cast<float*>(b + o_hval);
    p.head_idx = reinterpret_cast<int*>(b + o_hidx);
    p.head_count = reinterpret_cast<int*>(b + o_hcnt);
    p.length = d->d_length;
    p.bar_count = reinterpret_cast<unsigned*>(b + o_bar);
    p.grid = grid;
    p.wait_ns = vv::kWaitLimitNs;
    p.nstages = 4;
    p.stage_bytes = 0;
    const size_t fixed = vv::step_smem_bytes(p);
    int smem_max = 0;
    cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, d->device);
    if (smem_max <= 0) smem_max = 232448;
    const long avail = (long)smem_max - (long)fixed;
    p.stage_bytes = (int)((avail / p.nstages) / 1024 * 1024);
    std::vector<vv::StepLayer> hl(c.layers);
    for (int l = 0; l < c.layers; ++l) {
      const vv_layer_weights& L = w->layers[l];
      const vv_packed_matrix* m[7] = {&L.wq, &L.wk, &L.wv, &L.wo, &L.wgate, &L.wup, &L.wdown};
      hl[l].in_norm = reinterpret_cast<const __half*>(L.input_norm);
      hl[l].post_norm = reinterpret_cast<const __half*>(L.post_norm);
      for (int k = 0; k < 7; ++k) {
        hl[l].q[k] = m[k]->q;
        hl[l].s[k] = reinterpret_cast<const __half*>(m[k]->scales);
      }
      hl[l].bias[0] = reinterpret_cast<const __half*>(L.bq);
      hl[l].bias[1] = reinterpret_cast<const __half*>(L.bk);
      hl[l].bias[2] = reinterpret_cast<const __half*>(L.bv);
      hl[l].wo_img = b + o_wo + (size_t)l * wo_b;
      hl[l].wd_img = b + o_wd + (size_t)l * wd_b;
    }
    if (!st)
      st = vv::cuda_check(cudaMemcpy(d->d_layers, hl.data(), sizeof(vv::StepLayer) * c.layers,
                                     cudaMemcpyHostToDevice),
                          "copy layer table");
    if (!st)
      st = vv::cuda_check(vv::step_build_images(p, hl.data(), b + o_wo, b + o_wd, nullptr),
                          "build column images");
    if (!st) st = vv::cuda_check(cudaDeviceSynchronize(), "build column images");
    int nb = 0;
    if (!st) st = vv::cuda_check(vv::step_configure(p, &nb), "step kernel configuration");
    if (!st && nb < 1) {
      int regs = 0, mt = 0, ss = 0, lb = 0;
      vv::step_func_info(NB, &regs, &mt, &ss, &lb);
      st = set_error(VV_ERR_SHAPE,
                     "persistent step: no stage size that holds an attention tile fits one CTA "
                     "per SM (regs %d, max threads %d, static smem %d, local %d, threads %d, "
                     "smem optin %d)",
                     regs, mt, ss, lb, vv::step_threads(), smem_max);
    }
  }

  // RoPE tables: angle = pos * theta^(-2i/D) in float64, cos/sin rounded once to fp32.
  if (!st) {
    std::vector<float> cs((size_t)c.max_position * (D / 2)), sn(cs.size());
    for (int i = 0; i < D / 2; ++i) {
      const double inv = std::pow((double)c.rope_theta, -2.0 * i / (double)D);
      for (int p = 0; p < c.max_position; ++p) {
        const double ang = (double)p * inv;
        cs[(size_t)p * (D / 2) + i] = (float)std::cos(ang);
        sn[(size_t)p * (D / 2) + i] = (float)std::sin(ang);
      }
    }
    st = vv::cuda_check(cudaMemcpy(d->rope_cos, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice),
                        "copy rope cos");
    if (!st)
      st = vv::cuda_check(
          cudaMemcpy(d->rope_sin, sn.data(), sn.size() * 4, cudaMemcpyHostToDevice),
          "copy rope sin");
  }
  if (!st && c.max_prefill > 0) st = vv::cuda_check(vv::prefill_prepare(d), "prefill scales");
  if (st) {
    cudaFree(d->ws);
    if (d->pf_pad) cudaFree(d->pf_pad);
    delete d;
    return st;
  }
  *out = d;
  return VV_OK;
}

vv_status vv_decoder_destroy(vv_decoder* d) {
  if (!d) return VV_OK;
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(d->device);
  if (d->gexec) cudaGraphExecDestroy(d->gexec);
  if (d->capture_stream) cudaStreamDestroy(d->capture_stream);
  if (d->ws) cudaFree(d->ws);
  if (d->pws) cudaFree(d->pws);
  if (d->pf_pad) cudaFree(d->pf_pad);
  cudaSetDevice(cur);
  delete d;
  return VV_OK;
}

vv_status vv_decoder_set_length(vv_decoder* d, int32_t len, vv_stream stream) {
  VV_CHECK_ARG(d, "null decoder");
  if (len < 0) return set_error(VV_ERR_RANGE, "length %d < 0", len);
  if (len > d->cfg.kv_capacity)
    return set_error(VV_ERR_CAPACITY, "length %d > capacity %d", len, d->cfg.kv_capacity);
  for (int b = 0; b < d->nb; ++b) {
    vv::set_int_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(d->d_length + b, len);
    VV_CUDA(cudaGetLastError());
    d->len_host[b] = len;
  }
  return VV_OK;
}

vv_status vv_decoder_set_lengths(vv_decoder* d, const int32_t* lens, vv_stream stream) {
  VV_CHECK_ARG(d && lens, "vv_decoder_set_lengths: null pointer");
  for (int b = 0; b < d->nb; ++b) {
    if (lens[b] < 0) return set_error(VV_ERR_RANGE, "sequence %d: length %d < 0", b, lens[b]);
    if (lens[b] > d->cfg.kv_capacity)
      return set_error(VV_ERR_CAPACITY, "sequence %d: length %d > capacity %d", b, lens[b],
                       d->cfg.kv_capacity);
  }
  for (int b = 0; b < d->nb; ++b) {
    vv::set_int_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(d->d_length + b, lens[b]);
    VV_CUDA(cudaGetLastError());
    d->len_host[b] = lens[b];
  }
  return VV_OK;
}

int32_t vv_decoder_length(const vv_decoder* d) { return d ? d->len_host[0] : -1; }

int32_t vv_decoder_sequence_length(const vv_decoder* d, int32_t seq) {
  return d && seq >= 0 && seq < d->nb ? d->len_host[seq] : -1;
}

int32_t vv_decoder_batch(const vv_decoder* d) { return d ? d->nb : 0; }

vv_status vv_decoder_set_trace(vv_decoder* d, float* layer_out) {
  VV_CHECK_ARG(d, "null decoder");
  d->trace = layer_out;
  return VV_OK;
}

vv_status vv_decoder_set_wait_limit(vv_decoder* d, int64_t limit_ns) {
  VV_CHECK_ARG(d, "null decoder");
  VV_CHECK_ARG(limit_ns >= 100000 && limit_ns <= 10000000000ll,
               "vv_decoder_set_wait_limit: %lld ns (1e5 .. 1e10)", (long long)limit_ns);
  d->step.wait_ns = (uint64_t)limit_ns;
  if (d->gexec) {  // the captured graph holds the old parameters
    cudaGraphExecDestroy(d->gexec);
    d->gexec = nullptr;
  }
  return VV_OK;
}

vv_status vv_decoder_set_graph(vv_decoder* d, int32_t enable) {
  VV_CHECK_ARG(d, "null decoder");
  d->use_graph = enable != 0;
  return VV_OK;
}

int32_t vv_decoder_step_launches(const vv_decoder* d) { return d ? 1 : 0; }

vv_status vv_decoder_step(vv_decoder* d, const uint16_t* input_embeds, const int32_t* token_id,
                          const int32_t* position_id, float* logits, int32_t* argmax_out,
                          vv_stream stream) {
  VV_CHECK_ARG(d && position_id, "vv_decoder_step: null decoder or position");
  VV_CHECK_ARG(input_embeds || token_id, "vv_decoder_step: need input_embeds or token_id");
  VV_CHECK_ARG(!input_embeds || vv::aligned16(input_embeds), "input_embeds not 16-byte aligned");
  if (d->max_len() + 1 > d->cfg.kv_capacity)
    return set_error(VV_ERR_CAPACITY, "KV cache full (%d of %d)", d->max_len(),
                     d->cfg.kv_capacity);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!d->use_graph) {
    VV_CUDA(vv::enqueue_step(d, input_embeds, token_id, position_id, logits, argmax_out, s));
    d->advance_lengths(1);
    return VV_OK;
  }
  const void* key[6] = {input_embeds, token_id, position_id, logits, argmax_out, d->trace};
  bool same = d->gexec != nullptr;
  for (int i = 0; i < 6 && same; ++i) same = key[i] == d->gkey[i];
  if (!same) {
    if (d->gexec) {
      cudaGraphExecDestroy(d->gexec);
      d->gexec = nullptr;
    }
    // Capture on the decoder's own stream (capture executes nothing, and the caller's stream
    // may be the legacy default stream, which cannot be captured); replay on the caller's.
    if (!d->capture_stream)
      VV_CUDA(cudaStreamCreateWithFlags(&d->capture_stream, cudaStreamNonBlocking));
    cudaStream_t cs = d->capture_stream;
    cudaGraph_t g = nullptr;
    VV_CUDA(cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal));
    cudaError_t le =
        vv::enqueue_step(d, input_embeds, token_id, position_id, logits, argmax_out, cs);
    cudaError_t ee = cudaStreamEndCapture(cs, &g);
    if (le != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      return vv::cuda_check(le, "step capture (launch)");
    }
    VV_CUDA(ee);
    cudaError_t ie = cudaGraphInstantiate(&d->gexec, g, 0);
    cudaGraphDestroy(g);
    VV_CUDA(ie);
    for (int i = 0; i < 6; ++i) d->gkey[i] = key[i];
  }
  VV_CUDA(cudaGraphLaunch(d->gexec, s));
  d->advance_lengths(1);
  return VV_OK;
}

vv_status vv_decoder_step_timeline(vv_decoder* d, const uint16_t* input_embeds,
                                   const int32_t* token_id, const int32_t* position_id,
                                   uint64_t* stamps, int32_t max_per_cta, int32_t* grid_out,
                                   int32_t* per_cta_out, vv_stream stream) {
  VV_CHECK_ARG(d && position_id && stamps && grid_out && per_cta_out, "null pointer");
  VV_CHECK_ARG(input_embeds || token_id, "need input_embeds or token_id");
  const int need = vv::step_timeline_stamps(d->cfg.layers);
  if (max_per_cta < need)
    return set_error(VV_ERR_CAPACITY, "max_per_cta %d < %d", max_per_cta, need);
  if (d->max_len() + 1 > d->cfg.kv_capacity)
    return set_error(VV_ERR_CAPACITY, "KV cache full");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int grid = d->step.grid;
  uint64_t* dst = nullptr;
  VV_CUDA(cudaMalloc(&dst, sizeof(uint64_t) * grid * max_per_cta));
  vv_status st = vv::cuda_check(cudaMemsetAsync(dst, 0, sizeof(uint64_t) * grid * max_per_cta, s),
                                "memset");
  vv::StepParams p = d->step;
  p.input_embeds = reinterpret_cast<const __half*>(input_embeds);
  p.token = token_id;
  p.position = position_id;
  p.logits = nullptr;
  p.argmax = d->d_argmax;
  p.trace = d->trace;
  p.stamps = dst;
  p.max_stamps = max_per_cta;
  if (!st) st = vv::cuda_check(vv::launch_step(p, s), "timeline step");
  if (!st)
    st = vv::cuda_check(cudaMemcpyAsync(stamps, dst, sizeof(uint64_t) * grid * max_per_cta,
                                        cudaMemcpyDeviceToHost, s),
                        "copy stamps");
  if (!st) st = vv::cuda_check(cudaStreamSynchronize(s), "sync");
  cudaFree(dst);
  if (st) return st;
  int n = 0;
  while (n < max_per_cta - 8 && stamps[n] != 0) ++n;
  *grid_out = grid;
  *per_cta_out = n;
  d->advance_lengths(1);
  return VV_OK;
}

vv_status vv_decoder_init(vv_decoder* d, const int32_t* input_ids, const int32_t* position_ids,
                          int64_t S, const uint16_t* audio_features, int64_t N,
                          int64_t audio_offset, float* logits, int32_t* argmax_out,
                          vv_stream stream) {
  return vv_decoder_init_seq(d, 0, input_ids, position_ids, S, audio_features, N, audio_offset,
                             logits, argmax_out, stream);
}

vv_status vv_decoder_init_seq(vv_decoder* d, int32_t seq, const int32_t* input_ids,
                              const int32_t* position_ids, int64_t S,
                              const uint16_t* audio_features, int64_t N, int64_t audio_offset,
                              float* logits, int32_t* argmax_out, vv_stream stream) {
  VV_CHECK_ARG(d && input_ids && position_ids, "vv_decoder_init: null pointer");
  VV_CHECK_ARG(seq >= 0 && seq < d->nb, "vv_decoder_init: sequence %d of a batch of %d", seq, d->nb);
  VV_CHECK_ARG(N == 0 || audio_features, "vv_decoder_init: audio_features null with N > 0");
  VV_CHECK_ARG(!audio_features || vv::aligned16(audio_features), "audio_features misaligned");
  if (S < 1) return set_error(VV_ERR_SHAPE, "S=%lld", (long long)S);
  if (N < 0 || audio_offset < 0 || audio_offset + N > S)
    return set_error(VV_ERR_RANGE, "audio_offset %lld + N %lld > S %lld", (long long)audio_offset,
                     (long long)N, (long long)S);
  if (S > d->cfg.kv_capacity || S > d->cfg.max_prefill)
    return set_error(VV_ERR_CAPACITY, "S=%lld > capacity %d or max_prefill %d", (long long)S,
                     d->cfg.kv_capacity, d->cfg.max_prefill);
  VV_CUDA(vv::prefill_run(d, seq, input_ids, position_ids, (int)S, audio_features, (int)N,
                          (int)audio_offset, logits, argmax_out,
                          static_cast<cudaStream_t>(stream)));
  d->len_host[seq] = (int32_t)S;
  return VV_OK;
}

vv_status vv_decoder_profile_init(vv_decoder* d, const int32_t* input_ids,
                                  const int32_t* position_ids, int64_t S,
                                  const uint16_t* audio_features, int64_t N, int64_t audio_offset,
                                  float* logits, int32_t* argmax_out, float* phase_ms,
                                  int32_t* launches, vv_stream stream) {
  VV_CHECK_ARG(d && input_ids && position_ids && phase_ms && launches,
               "vv_decoder_profile_init: null pointer");
  VV_CHECK_ARG(N == 0 || audio_features, "vv_decoder_profile_init: audio_features null");
  VV_CHECK_ARG(!audio_features || vv::aligned16(audio_features), "audio_features misaligned");
  if (S < 1) return set_error(VV_ERR_SHAPE, "S=%lld", (long long)S);
  if (N < 0 || audio_offset < 0 || audio_offset + N > S)
    return set_error(VV_ERR_RANGE, "audio_offset %lld + N %lld > S %lld", (long long)audio_offset,
                     (long long)N, (long long)S);
  if (S > d->cfg.kv_capacity || S > d->cfg.max_prefill)
    return set_error(VV_ERR_CAPACITY, "S=%lld > capacity %d or max_prefill %d", (long long)S,
                     d->cfg.kv_capacity, d->cfg.max_prefill);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  vv::PrefillTimer t;
  vv_status st = vv::cuda_check(vv::prefill_run(d, 0, input_ids, position_ids, (int)S, audio_features,
                                                (int)N, (int)audio_offset, logits, argmax_out, s,
                                                &t),
                                "profile prefill");
  if (!st) st = vv::cuda_check(cudaStreamSynchronize(s), "sync");
  if (!st) {
    for (int k = 0; k < vv::kPfKinds; ++k) {
      phase_ms[k] = 0.f;
      launches[k] = 0;
    }
    for (size_t i = 1; i < t.ev.size(); ++i) {
      float ms = 0.f;
      cudaEventElapsedTime(&ms, t.ev[i - 1], t.ev[i]);
      phase_ms[t.kind[i]] += ms;
      launches[t.kind[i]] += 1;
    }
    d->len_host[0] = (int32_t)S;
  }
  for (auto e : t.ev) cudaEventDestroy(e);
  return st;
}

vv_status vv_decoder_generate(vv_decoder* d, const int32_t* first_token, const int32_t* position,
                              int32_t n_steps, const int32_t* stop_ids, int32_t n_stop,
                              int32_t* tokens_out, int32_t* n_out, vv_stream stream) {
  VV_CHECK_ARG(d && first_token && position && tokens_out && n_out,
               "vv_decoder_generate: null pointer");
  VV_CHECK_ARG(n_stop >= 0 && n_stop <= vv::kMaxStopIds && (n_stop == 0 || stop_ids),
               "vv_decoder_generate: n_stop %d (0..%d)", n_stop, vv::kMaxStopIds);
  if (n_steps < 1) return set_error(VV_ERR_SHAPE, "n_steps=%d", n_steps);
  if (d->nb != 1) return set_error(VV_ERR_SHAPE, "vv_decoder_generate: batch %d (only 1)", d->nb);
  if (d->len_host[0] + n_steps > d->cfg.kv_capacity)
    return set_error(VV_ERR_CAPACITY, "%d + %d steps exceed the KV capacity %d", d->len_host[0],
                     n_steps, d->cfg.kv_capacity);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* done = d->d_gen;
  int32_t* count = d->d_gen + 1;
  int32_t* gpos = d->d_gen + 2;
  VV_CUDA(cudaMemsetAsync(d->d_gen, 0, 2 * sizeof(int32_t), s));
  VV_CUDA(cudaMemcpyAsync(gpos, position, sizeof(int32_t), cudaMemcpyDeviceToDevice, s));
  vv::StepParams p = d->step;
  p.input_embeds = nullptr;
  p.position = gpos;
  p.logits = nullptr;
  p.trace = d->trace;
  p.gen_done = done;
  p.gen_count = count;
  p.gen_pos = gpos;
  p.n_stop = n_stop;
  for (int j = 0; j < n_stop; ++j) p.stop_ids[j] = stop_ids[j];
  for (int i = 0; i < n_steps; ++i) {
    p.token = i == 0 ? first_token : tokens_out + (i - 1);
    p.argmax = tokens_out + i;
    VV_CUDA(vv::launch_step(p, s));
  }
  int32_t n = 0;
  VV_CUDA(cudaMemcpyAsync(&n, count, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
  VV_CUDA(cudaStreamSynchronize(s));
  d->len_host[0] += n;
  *n_out = n;
  // a device-side error during the generation (a bounded wait that ran out, a token or position
  // out of range) is this call's result
  return vv_sync_status(stream);
}

vv_status vv_decoder_sync_status(vv_decoder* d, vv_stream stream) {
  VV_CHECK_ARG(d, "null decoder");
  return vv_sync_status(stream);
}

}  // extern "C"
