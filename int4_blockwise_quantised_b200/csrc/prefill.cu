// decoder_init (prefill) ("vibevoice-asr-bitnet-onnx": decoder_init owns the embedding table and
// writes audio_features over the <|speech_pad|> rows starting at audio_offset; present K/V of all
// S positions; logits of the last position).
//
// Tensor-core path, per layer (S prompt positions, fp32 residual X [S, H]):
//   Xn  = RMSNorm(X)                                  (fp16, the GEMM operand)
//   Q, K, V = RoPE(Xn . [Wq;Wk;Wv]^T + b)             tcgen05 GEMM; its epilogue rotates q and k
//                                                     and writes fp16 Q and cache slots 0..S-1
//   O   = causal GQA attention                        tcgen05 flash attention (S, P, O in TMEM)
//   X  += O . Wo^T                                    tcgen05 GEMM, residual epilogue
//   Hm  = silu(Xn Wg^T) * (Xn Wu^T), Xn = RMSNorm(X)  tcgen05 GEMM over interleaved gate/up rows
//   X  += Hm . Wd^T                                   tcgen05 GEMM, residual epilogue
// Weights: for prompts of at most kFusedMaxM positions the GEMMs read the packed int4 matrices
// as they are (converter warps expand each 64-column block of codes to fp16, (code - 8) * scale
// rounded once, in shared memory right before the tensor cores read it); longer prompts
// dequantise the layer's four weight stacks to fp16 once at the start of the layer (one launch)
// and run the fp16 GEMM on them.  The last row then goes through the final RMSNorm + lm_head.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "decoder_state.h"
#include "gemm_tc.h"
#include "attn_prefill.h"

namespace vv {
namespace {

constexpr int D = 128;

// X[s] = audio[s - off] for off <= s < off + N, else embed[ids[s]]  (fp32 rows of H).
__global__ void __launch_bounds__(256) splice_x_kernel(const int32_t* __restrict__ ids, int S,
                                                       const __half* __restrict__ embed, int V,
                                                       int H, const __half* __restrict__ audio,
                                                       int N, int off, float* __restrict__ x) {
  const int row = blockIdx.x;
  if (row >= S) return;
  const __half* src;
  if (row >= off && row < off + N) {
    src = audio + (size_t)(row - off) * H;
  } else {
    int id = ids[row];
    if (id < 0 || id >= V) {
      if (threadIdx.x == 0) set_device_error(VV_ERR_RANGE);
      id = min(max(id, 0), V - 1);
    }
    src = embed + (size_t)id * H;
  }
  for (int i = threadIdx.x; i < H; i += blockDim.x) x[(size_t)row * H + i] = __half2float(src[i]);
}

// Xn[s] = X[s] / sqrt(mean(X[s]^2) + eps) * gamma  -> fp16.  One CTA of 128 threads per row; the
// row is read once and held in registers (H <= 128 * 4 * kNormVec), gamma read as 8-byte vectors.
constexpr int kNormVec = 15;  // hidden <= 7680
__global__ void __launch_bounds__(128) rmsnorm_rows_kernel(const float* __restrict__ x, int H,
                                                           const __half* __restrict__ gamma,
                                                           float eps, __half* __restrict__ out) {
  const int row = blockIdx.x;
  const float* xr = x + (size_t)row * H;
  float4 v[kNormVec];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kNormVec; ++i) {
    const int k = (threadIdx.x + i * 128) * 4;
    v[i] = k < H ? *reinterpret_cast<const float4*>(xr + k) : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
  }
  __shared__ float red[4];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  const float inv = rsqrtf((red[0] + red[1] + red[2] + red[3]) / (float)H + eps);
#pragma unroll
  for (int i = 0; i < kNormVec; ++i) {
    const int k = (threadIdx.x + i * 128) * 4;
    if (k < H) {
      const uint2 g = *reinterpret_cast<const uint2*>(gamma + k);
      const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&g.x));
      const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&g.y));
      const __half2 a = __floats2half2_rn(v[i].x * inv * g01.x, v[i].y * inv * g01.y);
      const __half2 b = __floats2half2_rn(v[i].z * inv * g23.x, v[i].w * inv * g23.y);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&a);
      pk.y = *reinterpret_cast<const uint32_t*>(&b);
      *reinterpret_cast<uint2*>(out + (size_t)row * H + k) = pk;
    }
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

namespace {
// Rows of `kb` fp16 scales copied to a row pitch of `pitch` >= kb elements, zero-padded.
__global__ void pad_scales_kernel(const uint16_t* __restrict__ src, int rows, int kb, int pitch,
                                  uint16_t* __restrict__ dst) {
  const int64_t n = (int64_t)rows * pitch;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / pitch), c = (int)(i % pitch);
    dst[i] = c < kb ? src[(size_t)r * kb + c] : (uint16_t)0;
  }
}
}  // namespace

// Prompts longer than this run each projection as a dequantisation pass + fp16 GEMM; shorter
// ones on the GEMM with the dequantisation fused in (it expands every weight once per 128-row
// block of the prompt, so it wins while there are few blocks).
constexpr int kFusedMaxM = 256;

cudaError_t prefill_prepare(vv_decoder* d) {
  const vv_config& c = d->cfg;
  const int H = c.hidden, HQD = c.n_q * D, I = c.inter;
  const int Km[7] = {H, H, H, HQD, H, H, I};
  const int Nm[7] = {c.n_q * D, c.n_kv * D, c.n_kv * D, H, I, I, H};
  size_t pad_elems = 0;
  for (int m = 0; m < 7; ++m) {
    const int kb = Km[m] / 32;
    d->pf_pitch[m] = kb % 8 == 0 ? 0 : (kb + 7) & ~7;
    if (d->pf_pitch[m]) pad_elems += (size_t)c.layers * Nm[m] * d->pf_pitch[m];
  }
  d->pf_scales.assign((size_t)c.layers * 7, nullptr);
  if (pad_elems) {
    cudaError_t e = cudaMalloc(&d->pf_pad, pad_elems * 2);
    if (e != cudaSuccess) return e;
  }
  size_t off = 0;
  for (int l = 0; l < c.layers; ++l) {
    const vv_layer_weights& L = d->layers[l];
    const vv_packed_matrix* mats[7] = {&L.wq, &L.wk, &L.wv, &L.wo, &L.wgate, &L.wup, &L.wdown};
    for (int m = 0; m < 7; ++m) {
      if (!d->pf_pitch[m]) {
        d->pf_scales[(size_t)l * 7 + m] = mats[m]->scales;
        continue;
      }
      uint16_t* dst = d->pf_pad + off;
      off += (size_t)Nm[m] * d->pf_pitch[m];
      pad_scales_kernel<<<256, 256>>>(mats[m]->scales, Nm[m], Km[m] / 32, d->pf_pitch[m], dst);
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      d->pf_scales[(size_t)l * 7 + m] = dst;
    }
  }
  return cudaDeviceSynchronize();
}

cudaError_t prefill_run(vv_decoder* d, int seq, const int32_t* ids, const int32_t* pos, int S,
                        const uint16_t* audio, int N, int off, float* logits, int32_t* argmax,
                        cudaStream_t s, PrefillTimer* timer) {
  // mark(k): the work enqueued since the previous mark is of kind k
  auto mark = [&](int k) -> cudaError_t {
    if (!timer) return cudaSuccess;
    cudaEvent_t ev;
    cudaError_t err = cudaEventCreate(&ev);
    if (err != cudaSuccess) return err;
    timer->ev.push_back(ev);
    timer->kind.push_back(k);
    return cudaEventRecord(ev, s);
  };
#define VV_MARK(k)                                   \
  do {                                               \
    if ((e = mark(k)) != cudaSuccess) return e;      \
  } while (0)
  const vv_config& c = d->cfg;
  const int H = c.hidden, Hq = c.n_q, Hkv = c.n_kv, I = c.inter, HQD = Hq * D;
  const int NQKV = (Hq + 2 * Hkv) * D;
  const int SM = c.max_prefill;
  // workspace layout (allocated once, sized for max_prefill)
  size_t off_b = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off_b;
    off_b = align256(off_b + bytes);
    return o;
  };
  const size_t o_x = take((size_t)SM * H * 4);
  const size_t o_xn = take((size_t)SM * (H > HQD ? H : HQD) * 2);
  const size_t o_q = take((size_t)SM * HQD * 2);
  const size_t o_h = take((size_t)SM * I * 2);
  // the two-pass path (S > kFusedMaxM): the current layer's weights in fp16, [q/k/v | o |
  // gate/up interleaved | down]
  const size_t w_qkv = (size_t)NQKV * H, w_o = (size_t)H * HQD, w_gu = (size_t)2 * I * H;
  const size_t w_layer = w_qkv + w_o + w_gu + (size_t)H * I;
  const size_t o_w16 = take(SM > kFusedMaxM ? w_layer * 2 : 0);
  const size_t need = off_b;
  if (d->pws_bytes < need) {
    if (d->pws) cudaFree(d->pws);
    d->pws = nullptr;
    d->pws_bytes = 0;
    cudaError_t e = cudaMalloc(&d->pws, need);
    if (e != cudaSuccess) return e;
    d->pws_bytes = need;
  }
  unsigned char* b = d->pws;
  float* X = reinterpret_cast<float*>(b + o_x);
  __half* Xn = reinterpret_cast<__half*>(b + o_xn);  // also the attention output O
  __half* Q = reinterpret_cast<__half*>(b + o_q);
  __half* Hm = reinterpret_cast<__half*>(b + o_h);
  __half* W16 = reinterpret_cast<__half*>(b + o_w16);
  const bool two_pass = S > kFusedMaxM;
  // layer l's fp16 weights (two-pass path): matrix m = 0 q/k/v, 1 o, 2 gate/up, 3 down
  auto w16_of = [&](int, int m) {
    const size_t offs[4] = {0, w_qkv, w_qkv + w_o, w_qkv + w_o + w_gu};
    return W16 + offs[m];
  };
  // one launch for the layer's four matrix stacks
  auto dequant_layer = [&](int l, cudaStream_t st) -> cudaError_t {
    const vv_layer_weights& w = d->layers[l];
    const DequantSrc ds[4] = {
        {{w.wq.q, w.wk.q, w.wv.q}, {w.wq.scales, w.wk.scales, w.wv.scales}, {HQD, Hkv * D, Hkv * D}, 3, 0},
        {{w.wo.q, nullptr, nullptr}, {w.wo.scales, nullptr, nullptr}, {H, 0, 0}, 1, 0},
        {{w.wgate.q, w.wup.q, nullptr}, {w.wgate.scales, w.wup.scales, nullptr}, {I, I, 0}, 2, 1},
        {{w.wdown.q, nullptr, nullptr}, {w.wdown.scales, nullptr, nullptr}, {H, 0, 0}, 1, 0}};
    const int rows[4] = {NQKV, H, 2 * I, H}, ks[4] = {H, HQD, H, I};
    __half* outs[4] = {w16_of(l, 0), w16_of(l, 1), w16_of(l, 2), w16_of(l, 3)};
    return launch_dequant_many(ds, rows, ks, outs, 4, st);
  };
  // One projection of layer l (matrix m): fused dequantisation in the GEMM for short prompts
  // (each weight is expanded once per 128-row block of the prompt), else the fp16 GEMM on the
  // weights dequantised at the start of the layer (each weight expanded once).
  auto project = [&](int l, int m, const uint16_t* A, const PackedB& pb, int N, int K, int epi,
                     const GemmEpilogue& ep) -> cudaError_t {
    cudaError_t err;
    if (!two_pass)
      err = launch_gemm_q4(A, pb, S, N, K, epi, ep, s);
    else
      err = launch_gemm_tc(A, reinterpret_cast<const uint16_t*>(w16_of(l, m)), S, N, K, epi, ep, s);
    if (err != cudaSuccess) return err;
    return mark(kPfGemm);
  };
  const size_t layer_kv = (size_t)Hkv * c.kv_capacity * D;
  cudaError_t e;

  VV_MARK(kPfMisc);
  splice_x_kernel<<<S, 256, 0, s>>>(ids, S, reinterpret_cast<const __half*>(d->embed), c.vocab, H,
                                    reinterpret_cast<const __half*>(audio), N, off, X);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  VV_MARK(kPfMisc);
  for (int l = 0; l < c.layers; ++l) {
    const vv_layer_weights& w = d->layers[l];
    // sequence seq's slice of layer l: caches are [L][batch][Hkv][cap][D]
    __half* kc = reinterpret_cast<__half*>(d->k_cache) + ((size_t)l * d->nb + seq) * layer_kv;
    __half* vc = reinterpret_cast<__half*>(d->v_cache) + ((size_t)l * d->nb + seq) * layer_kv;
    // ---- QKV
    rmsnorm_rows_kernel<<<S, 128, 0, s>>>(X, H, reinterpret_cast<const __half*>(w.input_norm), c.eps, Xn);
    VV_MARK(kPfMisc);
    PackedB pb = {};
    const uint16_t* const* ps = &d->pf_scales[(size_t)l * 7];
    pb.q[0] = w.wq.q; pb.s[0] = ps[0]; pb.rows[0] = HQD;
    pb.q[1] = w.wk.q; pb.s[1] = ps[1]; pb.rows[1] = Hkv * D;
    pb.q[2] = w.wv.q; pb.s[2] = ps[2]; pb.rows[2] = Hkv * D;
    pb.nseg = 3;
    pb.s_pitch = d->pf_pitch[0];
    // q/k/v + bias, rotary embedding at position_ids, fp16 Q and the K/V cache rows written by
    // the GEMM's epilogue
    GemmEpilogue ep = {};
    ep.out_f16 = Q;
    ep.bias = reinterpret_cast<const __half*>(w.bq);
    ep.bias_k = reinterpret_cast<const __half*>(w.bk);
    ep.bias_v = reinterpret_cast<const __half*>(w.bv);
    ep.ldo = HQD;
    ep.pos = pos;
    ep.rope_cos = d->rope_cos;
    ep.rope_sin = d->rope_sin;
    ep.max_pos = c.max_position;
    ep.hq = Hq;
    ep.hkv = Hkv;
    ep.cap = c.kv_capacity;
    ep.kc = kc;
    ep.vc = vc;
    if (two_pass) {
      if ((e = dequant_layer(l, s)) != cudaSuccess) return e;
      VV_MARK(kPfDequant);
    }
    if ((e = project(l, 0, reinterpret_cast<const uint16_t*>(Xn), pb, NQKV, H, kEpiRope, ep)) !=
        cudaSuccess)
      return e;
    // ---- attention -> O (in the Xn buffer)
    AttnPrefillArgs aa = {};
    aa.q = reinterpret_cast<const uint16_t*>(Q);
    aa.k_cache = reinterpret_cast<const uint16_t*>(kc);
    aa.v_cache = reinterpret_cast<const uint16_t*>(vc);
    aa.out = reinterpret_cast<uint16_t*>(Xn);
    aa.S = S;
    aa.cap = c.kv_capacity;
    aa.Hq = Hq;
    aa.Hkv = Hkv;
    aa.scale = 1.0f / sqrtf((float)D);
    if ((e = launch_attn_prefill(aa, s)) != cudaSuccess) return e;
    VV_MARK(kPfAttn);
    // ---- O projection + residual
    pb = {};
    pb.q[0] = w.wo.q; pb.s[0] = ps[3]; pb.rows[0] = H;
    pb.nseg = 1;
    pb.s_pitch = d->pf_pitch[3];
    ep = {};
    ep.out_f32 = X;
    ep.ldo = H;
    if ((e = project(l, 1, reinterpret_cast<const uint16_t*>(Xn), pb, H, HQD, kEpiResid, ep)) !=
        cudaSuccess)
      return e;
    // ---- gate/up + SwiGLU
    rmsnorm_rows_kernel<<<S, 128, 0, s>>>(X, H, reinterpret_cast<const __half*>(w.post_norm), c.eps, Xn);
    VV_MARK(kPfMisc);
    pb = {};
    pb.q[0] = w.wgate.q; pb.s[0] = ps[4]; pb.rows[0] = I;
    pb.q[1] = w.wup.q; pb.s[1] = ps[5]; pb.rows[1] = I;
    pb.nseg = 2;
    pb.interleave = 1;
    pb.s_pitch = d->pf_pitch[4];
    ep = {};
    ep.out_f16 = Hm;
    ep.ldo = I;
    if ((e = project(l, 2, reinterpret_cast<const uint16_t*>(Xn), pb, 2 * I, H, kEpiSwiglu, ep)) !=
        cudaSuccess)
      return e;
    // ---- down + residual
    pb = {};
    pb.q[0] = w.wdown.q; pb.s[0] = ps[6]; pb.rows[0] = H;
    pb.nseg = 1;
    pb.s_pitch = d->pf_pitch[6];
    ep = {};
    ep.out_f32 = X;
    ep.ldo = H;
    if ((e = project(l, 3, reinterpret_cast<const uint16_t*>(Hm), pb, H, I, kEpiResid, ep)) !=
        cudaSuccess)
      return e;

    if (d->trace) {
      e = cudaMemcpyAsync(d->trace + (size_t)l * H, X + (size_t)(S - 1) * H, (size_t)H * 4,
                          cudaMemcpyDeviceToDevice, s);
      if (e != cudaSuccess) return e;
      VV_MARK(kPfMisc);
    }
  }
  // ---- last position: final norm + lm_head + argmax; the residual row feeds later steps
  if ((e = cudaMemcpyAsync(d->x_last, X + (size_t)(S - 1) * H, (size_t)H * 4,
                           cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
    return e;
  LmHeadArgs la = {};
  la.x = d->x_last;
  la.gamma = d->final_norm;
  la.w = d->lm_head;
  la.V = c.vocab;
  la.H = H;
  la.eps = c.eps;
  la.logits = logits;
  la.idx = argmax ? argmax : d->d_argmax;
  la.ws_val = d->lm_val;
  la.ws_idx = d->lm_idx;
  la.ws_count = d->lm_count;
  la.length = nullptr;
  if ((e = launch_lm_head(la, s, false)) != cudaSuccess) return e;
  VV_MARK(kPfHead);
  set_int_kernel<<<1, 1, 0, s>>>(d->d_length + seq, S);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  VV_MARK(kPfMisc);
  return cudaSuccess;
#undef VV_MARK
}

}  // namespace vv
