// Final RMSNorm + fp16 lm_head GEMV + greedy argmax ("vibevoice-asr-bitnet-onnx": lm_head and
// embeddings stay fp16, greedy decode; "VibeVoice-1.5B — Current Status", section "Inference
// (ONNX)": logits = hidden . embed^T for the tied 1.5B head).
//
//   xn = x / sqrt(mean(x^2) + eps) * gamma;  logits[v] = sum_h W[v, h] xn[h];  idx = argmax
//
// HBM-bound stream of V x H fp16 (467 MB for the 1.5B head): one producer warp moves whole rows
// into a shared-memory ring with cp.async.bulk (evict-first), eight compute warps take R rows
// each per stage, fp32 products (packed f32x2 FMA) and warp-shuffle sums.  Each warp keeps its
// running (max, index) with the lowest index winning ties; CTAs publish partials and the last
// CTA to arrive reduces them (arrival counter, reset afterwards).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "vv_device.cuh"
#include "vv_internal.h"

namespace vv {
namespace {

constexpr int kWarps = 8;

template <int R, int STAGES>
struct LmCfg {
  static constexpr int kSR = kWarps * R;
  static size_t smem(int H) {
    return (size_t)STAGES * kSR * H * 2 + (size_t)H * 4 + 64 * 4 + 2 * STAGES * 8 + 64;
  }
};

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <int R, int STAGES>
__global__ void __launch_bounds__((kWarps + 1) * 32) lm_head_kernel(const LmHeadArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int SR = LmCfg<R, STAGES>::kSR;
  const int H = a.H;
  const size_t row_b = (size_t)H * 2;
  const size_t stage_b = SR * row_b;
  unsigned char* ring = smem;
  float* xs = reinterpret_cast<float*>(smem + STAGES * stage_b);
  float* red = xs + H;  // [64]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 64);
  uint64_t* empty = full + STAGES;
  __shared__ float s_val[kWarps];
  __shared__ int s_idx[kWarps];
  __shared__ int s_last;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = (int)((int64_t)a.V * blockIdx.x / gridDim.x);
  const int r1 = (int)((int64_t)a.V * (blockIdx.x + 1) / gridDim.x);
  const int nst = (r1 - r0 + SR - 1) / SR;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == kWarps) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int s = 0; s < nst; ++s) {
        const int slot = s % STAGES;
        if (s >= STAGES) mbar_wait(&empty[slot], ((s / STAGES) - 1) & 1);
        const int base = r0 + s * SR;
        const int nv = min(SR, r1 - base);
        const uint32_t bytes = (uint32_t)(nv * row_b);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_g2s_stream(ring + slot * stage_b,
                        reinterpret_cast<const unsigned char*>(a.w) + (size_t)base * row_b, bytes,
                        &full[slot], pol);
      }
    }
    return;
  }

  // ---- RMSNorm prologue: x (fp32, written by the previous kernel) -> xs, layout [2][H/8][4]
  const int tid = threadIdx.x, nthreads = kWarps * 32;
  pdl_wait();
  const int nch = H >> 3;
  float ss = 0.f;
  for (int k = tid * 4; k < H; k += nthreads * 4) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(a.x + k));
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) tot += red[i];
  const float inv = rsqrtf(tot / (float)H + a.eps);
  const __half* gm = reinterpret_cast<const __half*>(a.gamma);
  for (int k = tid * 4; k < H; k += nthreads * 4) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(a.x + k));
    const int c = k >> 3, part = (k >> 2) & 1;
    float4 y;
    y.x = v.x * inv * __half2float(gm[k + 0]);
    y.y = v.y * inv * __half2float(gm[k + 1]);
    y.z = v.z * inv * __half2float(gm[k + 2]);
    y.w = v.w * inv * __half2float(gm[k + 3]);
    reinterpret_cast<float4*>(xs)[part * nch + c] = y;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");

  const float4* xs4 = reinterpret_cast<const float4*>(xs);
  float best = -INFINITY;
  int best_i = 0x7fffffff;
  for (int s = 0; s < nst; ++s) {
    const int slot = s % STAGES;
    mbar_wait(&full[slot], (s / STAGES) & 1);
    const unsigned char* st = ring + slot * stage_b;
    const int base = r0 + s * SR;
    const int nv = min(SR, r1 - base);
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    if (warp * R < nv) {
#pragma unroll 2
      for (int c = lane; c < nch; c += 32) {
        const float4 xa = xs4[c], xb = xs4[nch + c];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 w = *reinterpret_cast<const uint4*>(st + (size_t)(warp * R + r) * row_b + c * 16);
          const float2 w0 = __half22float2(*reinterpret_cast<const __half2*>(&w.x));
          const float2 w1 = __half22float2(*reinterpret_cast<const __half2*>(&w.y));
          const float2 w2 = __half22float2(*reinterpret_cast<const __half2*>(&w.z));
          const float2 w3 = __half22float2(*reinterpret_cast<const __half2*>(&w.w));
          float2 p = make_float2(0.f, 0.f);
          p = __ffma2_rn(w0, make_float2(xa.x, xa.y), p);
          p = __ffma2_rn(w1, make_float2(xa.z, xa.w), p);
          p = __ffma2_rn(w2, make_float2(xb.x, xb.y), p);
          p = __ffma2_rn(w3, make_float2(xb.z, xb.w), p);
          acc[r] += p.x + p.y;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = warp_sum(acc[r]);
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&empty[slot]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int row = base + warp * R + r;
        if (warp * R + r < nv) {
          if (a.logits) a.logits[row] = acc[r];
          if (better(acc[r], row, best, best_i)) {
            best = acc[r];
            best_i = row;
          }
        }
      }
    }
  }
  // ---- CTA argmax, then the last CTA reduces over CTAs
  if (lane == 0) {
    s_val[warp] = best;
    s_idx[warp] = best_i;
  }
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
  if (tid == 0) {
    float bv = s_val[0];
    int bi = s_idx[0];
    for (int w = 1; w < kWarps; ++w)
      if (better(s_val[w], s_idx[w], bv, bi)) {
        bv = s_val[w];
        bi = s_idx[w];
      }
    a.ws_val[blockIdx.x] = bv;
    a.ws_idx[blockIdx.x] = bi;
    __threadfence();
    const int prev = atomicAdd(a.ws_count, 1);
    s_last = (prev == (int)gridDim.x - 1);
  }
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
  if (!s_last) return;
  __threadfence();
  if (warp == 0) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lane; i < (int)gridDim.x; i += 32) {
      const float v = __ldcg(a.ws_val + i);
      const int ix = __ldcg(a.ws_idx + i);
      if (better(v, ix, bv, bi)) {
        bv = v;
        bi = ix;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      *a.idx = bi == 0x7fffffff ? 0 : bi;
      *a.ws_count = 0;
      if (a.length) *a.length += 1;
    }
  }
}

template <int R, int STAGES>
cudaError_t launch_lm(const LmHeadArgs& a, int grid, cudaStream_t s, bool pdl) {
  const size_t smem = LmCfg<R, STAGES>::smem(a.H);
  auto k = lm_head_kernel<R, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch(k, dim3(grid), dim3((kWarps + 1) * 32), smem, s, pdl, a);
}

}  // namespace

int lm_head_grid(int V) {
  const int g = sm_count();
  return V < g * 8 ? (V + 7) / 8 : g;
}

size_t lm_head_workspace_bytes(int V) {
  const int g = lm_head_grid(V);
  return (size_t)g * 8 + 64;
}

cudaError_t launch_lm_head(const LmHeadArgs& a, cudaStream_t s, bool pdl) {
  const int grid = lm_head_grid(a.V);
  if (a.H <= 2048) return launch_lm<2, 2>(a, grid, s, pdl);
  return launch_lm<1, 2>(a, grid, s, pdl);
}

}  // namespace vv

extern "C" size_t vv_lm_head_argmax_workspace_size(int64_t V) {
  if (V < 1 || V > (int64_t(1) << 30)) return 0;
  return vv::lm_head_workspace_bytes((int)V);
}

extern "C" vv_status vv_lm_head_argmax(const float* x, const uint16_t* gamma, const uint16_t* w_lm,
                                       int64_t V, int64_t H, float eps, float* logits,
                                       int32_t* idx, void* ws, size_t ws_bytes,
                                       vv_stream stream) {
  VV_CHECK_ARG(x && gamma && w_lm && idx && ws, "vv_lm_head_argmax: null pointer");
  VV_CHECK_ARG(vv::aligned16(x) && vv::aligned16(w_lm) && vv::aligned16(ws),
               "vv_lm_head_argmax: pointers must be 16-byte aligned");
  VV_CHECK_SHAPE(H >= 64 && H % 64 == 0 && H <= 16384, "vv_lm_head_argmax: H=%lld",
                 (long long)H);
  VV_CHECK_SHAPE(V >= 1 && V < (int64_t(1) << 30), "vv_lm_head_argmax: V=%lld", (long long)V);
  const size_t need = vv::lm_head_workspace_bytes((int)V);
  if (ws_bytes < need)
    return vv::set_error(VV_ERR_CAPACITY, "vv_lm_head_argmax: workspace %zu < %zu", ws_bytes,
                         need);
  const int grid = vv::lm_head_grid((int)V);
  vv::LmHeadArgs a = {};
  a.x = x;
  a.gamma = gamma;
  a.w = w_lm;
  a.V = (int)V;
  a.H = (int)H;
  a.eps = eps;
  a.logits = logits;
  a.idx = idx;
  a.ws_val = static_cast<float*>(ws);
  a.ws_idx = reinterpret_cast<int*>(static_cast<char*>(ws) + (size_t)grid * 4);
  a.ws_count = reinterpret_cast<int*>(static_cast<char*>(ws) + (size_t)grid * 8);
  a.length = nullptr;
  return vv::cuda_check(vv::launch_lm_head(a, static_cast<cudaStream_t>(stream), false),
                        "lm_head launch");
}
