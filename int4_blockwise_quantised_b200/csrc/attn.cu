// Grouped-query decode attention over a GPU-resident fp16 KV cache
// ("VibeVoice-1.5B — Current Status", section "Done": one GroupQueryAttention per layer;
// "vibevoice-asr-bitnet-onnx": decoder_step past keys/values [L, 1, Hkv, P, D];
// "VibeVoice-ASR — ONNX export for Vernacula", section "Highlights": the cache stays on the GPU).
//
//   out[h] = softmax(scale * q[h] . K[g, t]  for all t) . V[g],  g = h / (Hq / Hkv)
//
// Split-K ("flash decoding"): grid = (chunks, Hkv).  A CTA owns one KV head and a run of 64-
// position tiles; one K/V tile load serves all G = Hq/Hkv query heads of the group.  Tiles move
// global -> shared with cp.async.bulk (positions of one head are contiguous) into a double
// buffer; softmax is online in fp32 in the log2 domain.  Each CTA writes (m, l, o) partials; the
// last CTA of a head (arrival counter, no spinning) merges them and resets the counter.
//
// Fused decoder mode: the QKV GEMV left q/k/v pre-RoPE in fp32.  Every CTA rotates its group's
// q (RoPE, table built on the host in float64); the CTA holding the last tile also rotates k,
// rounds k and v to fp16, stores them at slot `length` of the cache and into its own tile.
// Past tiles are prefetched before griddepcontrol.wait: they were written by kernels at least
// one whole step (and a non-overlapped kernel boundary) earlier.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "vv_device.cuh"
#include "vv_internal.h"

namespace vv {
namespace {

constexpr int D = 128;
constexpr int TT = 64;  // positions per tile
constexpr int kThreads = 256;
constexpr int kMaxG = 8;
constexpr int kPartStride = 132;  // floats per (chunk, head) partial: m, l, pad, pad, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxChunks = 256;  // upper bound of grid.x (chunks per KV head)

struct AttnSmem {
  __half k[2][TT * D];
  __half v[2][TT * D];
  float q[kMaxG][D];
  float s[kMaxG][TT];
  float m[kMaxG], l[kMaxG], corr[kMaxG];
  float mw[kMaxChunks][kMaxG];  // merge weights 2^(m_c - M) / L per (chunk, head)
  uint64_t bar[2];
  int is_last;
};

__global__ void __launch_bounds__(kThreads) attn_decode_kernel(const AttnArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(smem_raw);
  const int c = blockIdx.x, g = blockIdx.y, nchunks = gridDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv;

  const int past = a.len;
  const int npos = past;
  const int ntiles = (npos + TT - 1) / TT;
  const int tpc = (ntiles + nchunks - 1) / nchunks;
  const int t_begin = c * tpc;
  const int t_end = min(t_begin + tpc, ntiles);
  const int active = (ntiles + tpc - 1) / tpc;  // chunks that own at least one tile

  pdl_launch_dependents();
  if (t_begin >= t_end) {  // no work; not counted in `active`
    pdl_wait();
    return;
  }

  const __half* kc = reinterpret_cast<const __half*>(a.k_cache) + (size_t)g * a.cap * D;
  const __half* vc = reinterpret_cast<const __half*>(a.v_cache) + (size_t)g * a.cap * D;

  if (tid == 0) {
    mbar_init(&sm.bar[0], 1);
    mbar_init(&sm.bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // Issue the bulk load of tile t into buffer b: rows [t*TT, min(t*TT+TT, past)) from the cache.
  auto issue = [&](int t, int b) {
    const int p0 = t * TT;
    const int p1 = min(p0 + TT, past);
    const uint32_t bytes = p1 > p0 ? (uint32_t)(p1 - p0) * D * 2 : 0u;
    mbar_arrive_expect_tx(&sm.bar[b], 2 * bytes);
    if (bytes) {
      bulk_g2s(sm.k[b], kc + (size_t)p0 * D, bytes, &sm.bar[b]);
      bulk_g2s(sm.v[b], vc + (size_t)p0 * D, bytes, &sm.bar[b]);
    }
  };
  if (tid == 0) {
    issue(t_begin, 0);
    if (t_begin + 1 < t_end) issue(t_begin + 1, 1);
  }

  pdl_wait();

  // ---- q of the group, scaled into the log2 domain
  const float qscale = a.scale * kLog2e;
  for (int i = tid; i < G * D; i += kThreads) {
    const int h = i / D, d = i % D;
    const float qv = __half2float(reinterpret_cast<const __half*>(a.q_f16)[(size_t)(g * G + h) * D + d]);
    sm.q[h][d] = qv * qscale;
  }
  if (tid < kMaxG) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  __syncthreads();

  // Output ownership: thread -> dim d = tid % 128, heads hh, hh+2, hh+4, hh+6 (hh = tid / 128).
  const int od = tid & (D - 1), hh = tid >> 7;
  float o[kMaxG / 2];
#pragma unroll
  for (int j = 0; j < kMaxG / 2; ++j) o[j] = 0.f;

  // q fragment per lane for the score phase: dims 4*lane .. 4*lane+3 of every head.
  float4 qf[kMaxG];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h)
    qf[h] = h < G ? *reinterpret_cast<const float4*>(&sm.q[h][4 * lane]) : make_float4(0, 0, 0, 0);

  for (int t = t_begin; t < t_end; ++t) {
    const int b = (t - t_begin) & 1;
    mbar_wait(&sm.bar[b], ((t - t_begin) >> 1) & 1);
    const int p0 = t * TT;
    const int n = min(TT, npos - p0);

    // scores: warp w -> positions w, w+8, ...
    for (int p = warp; p < n; p += 2 * (kThreads / 32)) {
      const int p2 = p + kThreads / 32;
      const bool has2 = p2 < n;
      const uint2 kr = *reinterpret_cast<const uint2*>(&sm.k[b][p * D + 4 * lane]);
      const uint2 kr2 = has2 ? *reinterpret_cast<const uint2*>(&sm.k[b][p2 * D + 4 * lane])
                             : make_uint2(0u, 0u);
      const float2 k01 = __half22float2(*reinterpret_cast<const __half2*>(&kr.x));
      const float2 k23 = __half22float2(*reinterpret_cast<const __half2*>(&kr.y));
      const float2 j01 = __half22float2(*reinterpret_cast<const __half2*>(&kr2.x));
      const float2 j23 = __half22float2(*reinterpret_cast<const __half2*>(&kr2.y));
      float sd[2 * kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        sd[h] = qf[h].x * k01.x + qf[h].y * k01.y + qf[h].z * k23.x + qf[h].w * k23.y;
        sd[kMaxG + h] = qf[h].x * j01.x + qf[h].y * j01.y + qf[h].z * j23.x + qf[h].w * j23.y;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < 2 * kMaxG; ++i) sd[i] += __shfl_xor_sync(0xffffffffu, sd[i], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
          if (h < G) {
            sm.s[h][p] = sd[h];
            if (has2) sm.s[h][p2] = sd[kMaxG + h];
          }
        }
      }
    }
    __syncthreads();
    // online softmax per head: warp h
    if (warp < G) {
      const int h = warp;
      const float s0 = lane < n ? sm.s[h][lane] : -INFINITY;
      const float s1 = lane + 32 < n ? sm.s[h][lane + 32] : -INFINITY;
      const float mt = warp_max(fmaxf(s0, s1));
      const float mo = sm.m[h];
      const float mn = fmaxf(mo, mt);
      const float e0 = lane < n ? exp2f(s0 - mn) : 0.f;
      const float e1 = lane + 32 < n ? exp2f(s1 - mn) : 0.f;
      sm.s[h][lane] = e0;
      sm.s[h][lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      if (lane == 0) {
        const float cr = exp2f(mo - mn);  // mo = -inf on the first tile -> 0
        sm.corr[h] = cr;
        sm.l[h] = sm.l[h] * cr + sum;
        sm.m[h] = mn;
      }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kMaxG / 2; ++j) {
      const int h = hh + 2 * j;
      if (h < G) o[j] *= sm.corr[h];
    }
    for (int p = 0; p < n; ++p) {
      const float vv = __half2float(sm.v[b][p * D + od]);
#pragma unroll
      for (int j = 0; j < kMaxG / 2; ++j) {
        const int h = hh + 2 * j;
        if (h < G) o[j] = fmaf(sm.s[h][p], vv, o[j]);
      }
    }
    __syncthreads();  // buffer b and the score rows are free again
    if (tid == 0 && t + 2 < t_end) issue(t + 2, b);
  }

  if (active == 1) {
#pragma unroll
    for (int j = 0; j < kMaxG / 2; ++j) {
      const int h = hh + 2 * j;
      if (h < G) {
        const float r = o[j] / sm.l[h];
        const size_t idx = (size_t)(g * G + h) * D + od;
        reinterpret_cast<__half*>(a.out_f16)[idx] = __float2half_rn(r);
      }
    }
    return;
  }

  // ---- partials, then the last CTA of this head merges.
  float* part = a.ws_part + ((size_t)g * nchunks + c) * kMaxG * kPartStride;
#pragma unroll
  for (int j = 0; j < kMaxG / 2; ++j) {
    const int h = hh + 2 * j;
    if (h < G) part[h * kPartStride + 4 + od] = o[j];
  }
  if (tid < G) {
    part[tid * kPartStride + 0] = sm.m[tid];
    part[tid * kPartStride + 1] = sm.l[tid];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(&a.ws_count[g], 1);
    sm.is_last = (prev == active - 1);
  }
  __syncthreads();
  if (!sm.is_last) return;
  __threadfence();

  const float* base = a.ws_part + (size_t)g * nchunks * kMaxG * kPartStride;
  // per head: M = max m_c, L = sum l_c 2^(m_c - M); weights w_c = 2^(m_c - M) / L to smem
  if (warp < G) {
    const int h = warp;
    float mx = -INFINITY;
    for (int cc = lane; cc < active; cc += 32)
      mx = fmaxf(mx, __ldcg(base + ((size_t)cc * kMaxG + h) * kPartStride));
    mx = warp_max(mx);
    float L = 0.f;
    for (int cc = lane; cc < active; cc += 32) {
      const float* pp = base + ((size_t)cc * kMaxG + h) * kPartStride;
      const float e = exp2f(__ldcg(pp) - mx);
      sm.mw[cc][h] = e;
      L += __ldcg(pp + 1) * e;
    }
    L = warp_sum(L);
    const float invL = 1.f / L;
    for (int cc = lane; cc < active; cc += 32) sm.mw[cc][h] *= invL;
  }
  __syncthreads();
  // out[h][d] = sum_c w_c o_c[h][d]: independent loads, 8 chunks in flight per thread
#pragma unroll
  for (int j = 0; j < kMaxG / 2; ++j) {
    const int h = hh + 2 * j;
    if (h < G) {
      float acc = 0.f;
      int cc = 0;
      for (; cc + 8 <= active; cc += 8) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = __ldcg(base + ((size_t)(cc + u) * kMaxG + h) * kPartStride + 4 + od);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = fmaf(sm.mw[cc + u][h], v[u], acc);
      }
      for (; cc < active; ++cc)
        acc = fmaf(sm.mw[cc][h], __ldcg(base + ((size_t)cc * kMaxG + h) * kPartStride + 4 + od),
                   acc);
      const size_t idx = (size_t)(g * G + h) * D + od;
      reinterpret_cast<__half*>(a.out_f16)[idx] = __float2half_rn(acc);
    }
  }
  if (tid == 0) a.ws_count[g] = 0;
}

}  // namespace

int attn_default_chunks(int Hkv, int cap) {
  const int tiles = (cap + TT - 1) / TT;
  int per_head = sm_count() / (Hkv > 0 ? Hkv : 1);
  if (per_head < 1) per_head = 1;
  int n = tiles < per_head ? (tiles > 0 ? tiles : 1) : per_head;
  return n > kMaxChunks ? kMaxChunks : n;
}

size_t attn_workspace_bytes(int Hq, int Hkv, int nchunks) {
  (void)Hq;
  return (size_t)Hkv * nchunks * kMaxG * kPartStride * sizeof(float) + 256;
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(AttnSmem);
  dim3 grid(a.nchunks, a.Hkv);
  auto k = attn_decode_kernel;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch(k, grid, dim3(kThreads), smem, s, false, a);
}

}  // namespace vv

extern "C" size_t vv_gqa_decode_attn_workspace_size(int32_t Hq, int32_t Hkv, int32_t D_,
                                                    int32_t cap) {
  if (Hkv <= 0 || cap <= 0 || D_ != 128) return 0;
  const int nch = vv::attn_default_chunks(Hkv, cap);
  return vv::attn_workspace_bytes(Hq, Hkv, nch);
}

extern "C" vv_status vv_gqa_decode_attn(const uint16_t* q, const uint16_t* k_cache,
                                        const uint16_t* v_cache, int32_t len, int32_t cap,
                                        int32_t Hq, int32_t Hkv, int32_t D_, float scale,
                                        uint16_t* out, void* ws, size_t ws_bytes,
                                        vv_stream stream) {
  VV_CHECK_ARG(q && k_cache && v_cache && out && ws, "vv_gqa_decode_attn: null pointer");
  VV_CHECK_ARG(vv::aligned16(q) && vv::aligned16(k_cache) && vv::aligned16(v_cache) &&
                   vv::aligned16(out) && vv::aligned16(ws),
               "vv_gqa_decode_attn: pointers must be 16-byte aligned");
  VV_CHECK_SHAPE(D_ == 128, "vv_gqa_decode_attn: D=%d (only 128)", D_);
  VV_CHECK_SHAPE(Hkv >= 1 && Hkv <= 64 && Hq >= Hkv && Hq % Hkv == 0 && Hq / Hkv <= 8,
                 "vv_gqa_decode_attn: Hq=%d Hkv=%d", Hq, Hkv);
  VV_CHECK_SHAPE(cap >= 1 && len >= 1 && len <= cap, "vv_gqa_decode_attn: len=%d cap=%d", len,
                 cap);
  const int nch = vv::attn_default_chunks(Hkv, cap);
  const size_t need = vv::attn_workspace_bytes(Hq, Hkv, nch);
  if (ws_bytes < need)
    return vv::set_error(VV_ERR_CAPACITY, "vv_gqa_decode_attn: workspace %zu < %zu", ws_bytes,
                         need);
  vv::AttnArgs a = {};
  a.q_f16 = q;
  a.k_cache = const_cast<uint16_t*>(k_cache);
  a.v_cache = const_cast<uint16_t*>(v_cache);
  a.len = len;
  a.cap = cap;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.scale = scale;
  a.out_f16 = out;
  a.ws_part = static_cast<float*>(ws);
  a.ws_count = reinterpret_cast<int*>(static_cast<char*>(ws) + need - 256);
  a.nchunks = nch;
  return vv::cuda_check(vv::launch_attn(a, static_cast<cudaStream_t>(stream)),
                        "attention launch");
}

// ------------------------------------------------------------------------------------------------
// Scratch-free variant of vv_gqa_decode_attn.
//
// Some callers cannot allocate device memory at the point where they run attention: a host
// application that has handed the whole GPU memory budget to its own pool (a serving engine that
// pre-reserves the KV cache, a real-time audio pipeline that forbids allocation on its processing
// thread because cudaMalloc can block and synchronise the device), or a plugin that is not
// allowed to create allocations of its own.  For them the split-K partials and arrival counters
// live in one file-scope device array instead of a caller workspace.  Every GPU that loads this
// library holds the array (kNoAllocScratchBytes) until the process exits.
namespace vv {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(256) << 10;  // 256 KiB
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};  // device address of the array, per device ordinal
}  // namespace
}  // namespace vv

static __device__ __align__(256) unsigned char g_attn_scratch[vv::kNoAllocScratchBytes];

extern "C" vv_status vv_gqa_decode_attn_noalloc(const uint16_t* q, const uint16_t* k_cache,
                                                const uint16_t* v_cache, int32_t len, int32_t cap,
                                                int32_t Hq, int32_t Hkv, int32_t D_, float scale,
                                                uint16_t* out, vv_stream stream) {
  VV_CHECK_ARG(q && k_cache && v_cache && out, "vv_gqa_decode_attn_noalloc: null pointer");
  VV_CHECK_ARG(vv::aligned16(q) && vv::aligned16(k_cache) && vv::aligned16(v_cache) &&
                   vv::aligned16(out),
               "vv_gqa_decode_attn_noalloc: pointers must be 16-byte aligned");
  VV_CHECK_SHAPE(D_ == 128, "vv_gqa_decode_attn_noalloc: D=%d (only 128)", D_);
  VV_CHECK_SHAPE(Hkv >= 1 && Hkv <= 64 && Hq >= Hkv && Hq % Hkv == 0 && Hq / Hkv <= 8,
                 "vv_gqa_decode_attn_noalloc: Hq=%d Hkv=%d", Hq, Hkv);
  VV_CHECK_SHAPE(cap >= 1 && len >= 1 && len <= cap, "vv_gqa_decode_attn_noalloc: len=%d cap=%d",
                 len, cap);
  const int nch = vv::attn_default_chunks(Hkv, cap);
  const size_t need = vv::attn_workspace_bytes(Hq, Hkv, nch);
  if (need > vv::kNoAllocScratchBytes)
    return vv::set_error(VV_ERR_CAPACITY,
                         "vv_gqa_decode_attn_noalloc: needs %zu bytes of scratch, the static array "
                         "holds %zu (use vv_gqa_decode_attn with a caller workspace)",
                         need, vv::kNoAllocScratchBytes);
  int dev = 0;
  VV_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return vv::set_error(VV_ERR_INVALID_ARG, "device ordinal %d", dev);
  // The array's address is per device: the stream must belong to the current device.
  int sdev = dev;
  VV_CUDA(cudaStreamGetDevice(static_cast<cudaStream_t>(stream), &sdev));
  if (sdev != dev)
    return vv::set_error(VV_ERR_INVALID_ARG,
                         "vv_gqa_decode_attn_noalloc: stream of device %d, current device %d",
                         sdev, dev);
  void* base = nullptr;
  {
    // First call on a device: look up the array's device address with that device current.
    std::lock_guard<std::mutex> lock(vv::g_noalloc_mu);
    if (!vv::g_noalloc_ptr[dev]) {
      void* p = nullptr;
      VV_CUDA(cudaGetSymbolAddress(&p, g_attn_scratch));
      vv::g_noalloc_ptr[dev] = p;
    }
    base = vv::g_noalloc_ptr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(base);
  // The arrival counters must start at zero (the partials are fully rewritten by every call).
  VV_CUDA(cudaMemsetAsync(ws + need - 256, 0, 256, s));
  vv::AttnArgs a = {};
  a.q_f16 = q;
  a.k_cache = const_cast<uint16_t*>(k_cache);
  a.v_cache = const_cast<uint16_t*>(v_cache);
  a.len = len;
  a.cap = cap;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.scale = scale;
  a.out_f16 = out;
  a.ws_part = reinterpret_cast<float*>(ws);
  a.ws_count = reinterpret_cast<int*>(ws + need - 256);
  a.nchunks = nch;
  return vv::cuda_check(vv::launch_attn(a, s), "attention (no-alloc) launch");
}
