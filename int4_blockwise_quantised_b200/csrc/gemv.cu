// Dequant-fused int4 GEMV for batch-1 decode (MatMulNBits: "VibeVoice-1.5B — Current Status",
// section "Done"; block 32, symmetric, q = w/s + 8: "vibevoice-asr-bitnet-onnx", MatMulNBits
// paragraph).
//
//   y[n] = sum_b scale[n, b] * sum_{i<32} (code[n, 32b+i] - 8) * x[32b+i]
//
// Design (HBM-bound; every weight byte is read exactly once):
//  * One producer warp streams whole weight rows (codes + scales, both contiguous per row) into
//    a ring of shared-memory stages with cp.async.bulk (TMA, non-tensor form, this CTA only) and
//    mbarrier completion.  Weights do not depend on the previous kernel, so the producer fills
//    the ring BEFORE griddepcontrol.wait: under programmatic dependent launch the next GEMV's
//    weights are already in flight while the previous kernel finishes.
//  * Compute warps form a WR x WK grid: WK warps split the K axis of a row group (partials
//    reduced through shared memory), WR warps take different row groups.  A lane handles
//    half-blocks (16 columns = 8 bytes of codes) hb = slot, slot + 32*WK, ...
//  * x (after the fused RMSNorm prologue where there is one) lives in shared memory as fp32 in
//    a lane-interleaved order so every 16-byte x load of a warp is bank-conflict free.
//  * Dequant: exact (code - 8) in fp32 via the 2^23 magic-number trick, fp32 products and sums
//    with packed f32x2 FMAs, one fp32 scale multiply per half-block.
//
// Requirements of this path: K % 256 == 0 (so per-row scale runs are 16-byte multiples),
// K <= 16384 (x fits in shared memory), 16-byte aligned pointers.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "gemm_tc.h"

namespace vv {
namespace {

constexpr int kMaxK = 16384;

// --------------------------------------------------------------------------------- x staging
// Element k of x goes to float index ((2*w + (j & 1)) * NHB + hb) * 4 + (j >> 1) where
// hb = k / 16, e = k % 16, w = e / 8, j = e % 8, NHB = K / 16.
__device__ __forceinline__ int x_slot(int k, int nhb) {
  const int hb = k >> 4, e = k & 15, w = e >> 3, j = e & 7;
  return (((w << 1) | (j & 1)) * nhb + hb) * 4 + (j >> 1);
}

// Compute warps stage x into shared memory.  Source fp32 or fp16; optional RMSNorm with fp16
// gamma (y = x * rsqrt(mean(x^2) + eps) * gamma).  `nthreads` compute threads, tid < nthreads.
// Uses red_tmp[32] for the block reduction.  Named barrier 1 over the compute threads.
__device__ __forceinline__ void compute_bar(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

template <bool NORM>
__device__ void stage_x(float* xs, const float* __restrict__ src32, const __half* __restrict__ src16,
                        const __half* __restrict__ gamma, float eps, int K, int tid, int nthreads,
                        float* red_tmp) {
  const int nhb = K >> 4;
  constexpr int kReg = 4;  // float4 chunks held in registers per thread (K <= 16 * nthreads)
  auto load4 = [&](int k) -> float4 {
    if (src32) return __ldcg(reinterpret_cast<const float4*>(src32 + k));
    const uint2 h = __ldcg(reinterpret_cast<const uint2*>(src16 + k));
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
    return make_float4(a.x, a.y, b.x, b.y);
  };
  const bool in_regs = K <= kReg * 4 * nthreads;
  float4 v[kReg];
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kReg; ++i) {
      const int k = (tid + i * nthreads) * 4;
      v[i] = k < K ? load4(k) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  float inv = 1.f;
  if (NORM) {
    float ss = 0.f;
    if (in_regs) {
#pragma unroll
      for (int i = 0; i < kReg; ++i)
        ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    } else {
      for (int k = tid * 4; k < K; k += nthreads * 4) {
        const float4 t = load4(k);
        ss += t.x * t.x + t.y * t.y + t.z * t.z + t.w * t.w;
      }
    }
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red_tmp[tid >> 5] = ss;
    compute_bar(nthreads);
    float tot = 0.f;
    for (int i = 0; i < nthreads / 32; ++i) tot += red_tmp[i];
    inv = rsqrtf(tot / (float)K + eps);
  }
  auto put = [&](int k, float4 t) {
    float y[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float yy = y[i];
      if (NORM) yy = yy * inv * __half2float(gamma[k + i]);
      xs[x_slot(k + i, nhb)] = yy;
    }
  };
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kReg; ++i) {
      const int k = (tid + i * nthreads) * 4;
      if (k < K) put(k, v[i]);
    }
  } else {
    for (int k = tid * 4; k < K; k += nthreads * 4) put(k, load4(k));
  }
  compute_bar(nthreads);
}

// ------------------------------------------------------------------------------- ops (epilogue)
// Each op describes: number of segments (matrices read per stage), the CTA -> rows mapping, the
// x source, and what happens to a finished row group.

struct MatmulArgs {
  const uint16_t* x;
  GemvWeights w;
  const uint16_t* bias;
  int N, K;
  uint16_t* y;
};

struct OpMatmul {  // standalone MatMulNBits, M = 1: y fp16 = W . x + bias
  static constexpr int NSEG = 1;
  static constexpr bool NORM = false;
  MatmulArgs a;
  __device__ void rows(int cta, const uint8_t** q, const __half** s, int& r0, int& r1,
                       int& mat) const {
    r0 = (int)((int64_t)a.N * cta / gridDim.x);
    r1 = (int)((int64_t)a.N * (cta + 1) / gridDim.x);
    q[0] = a.w.q;
    s[0] = reinterpret_cast<const __half*>(a.w.scales);
    mat = 0;
  }
  __device__ void load_x(float* xs, int tid, int nthreads, float* red) const {
    stage_x<false>(xs, nullptr, reinterpret_cast<const __half*>(a.x), nullptr, 0.f, a.K, tid,
                   nthreads, red);
  }
  __device__ void finish(int, int row, float y) const {
    const __half* b = reinterpret_cast<const __half*>(a.bias);
    reinterpret_cast<__half*>(a.y)[row] = __float2half_rn(y + (b ? __half2float(b[row]) : 0.f));
  }
};

// ----------------------------------------------------------------------------------- kernel
template <int R, int WK, int WR, int STAGES, int NSEG>
struct GemvCfg {
  static constexpr int kR = R, kWK = WK, kWR = WR, kStages = STAGES, kNseg = NSEG;
  static constexpr int kRps = R / NSEG;        // rows per segment in a group
  static constexpr int kSR = WR * kRps;        // rows per segment per stage
  static constexpr int kComputeWarps = WR * WK;
  static constexpr int kThreads = (kComputeWarps + 1) * 32;
  static_assert(R % NSEG == 0, "group rows must split evenly over segments");
  static size_t stage_bytes(int K) { return (size_t)NSEG * kSR * (K / 32) * 18; }
  static size_t smem_bytes(int K) {
    return STAGES * stage_bytes(K) + (size_t)K * 4 + 2 * WR * R * WK * 4 + 32 * 4 +
           2 * STAGES * 8 + 16;
  }
};

template <class Op, class C>
__global__ void __launch_bounds__(C::kThreads) gemv_kernel(const Op op, const int K) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int R = C::kR, WK = C::kWK, WR = C::kWR, STAGES = C::kStages, NSEG = C::kNseg;
  constexpr int RPS = C::kRps, SR = C::kSR, NCW = C::kComputeWarps;
  const int KB = K >> 5;
  const int NHB = K >> 4;
  const size_t row_q = (size_t)KB * 16, row_s = (size_t)KB * 2;
  const size_t seg_q = SR * row_q, seg_s = SR * row_s;
  const size_t stage_b = NSEG * (seg_q + seg_s);

  unsigned char* ring = smem;
  float* xs = reinterpret_cast<float*>(smem + STAGES * stage_b);
  float* red = xs + K;                  // [2][WR][R][WK]
  float* red_tmp = red + 2 * WR * R * WK;  // [32]
  uint64_t* full = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(red_tmp + 32) + 7) & ~uintptr_t(7));
  uint64_t* empty = full + STAGES;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t* gq[NSEG];
  const __half* gs[NSEG];
  int r0, r1, mat;
  op.rows(blockIdx.x, gq, gs, r0, r1, mat);
  const int nrows = r1 - r0;
  const int nst = (nrows + SR - 1) / SR;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NCW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  if (warp == NCW) {
    // ---------------------------------------------------------------- producer (weights only)
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      for (int s = 0; s < nst; ++s) {
        const int slot = s % STAGES;
        if (s >= STAGES) mbar_wait(&empty[slot], ((s / STAGES) - 1) & 1);
        const int base = r0 + s * SR;
        const int nv = min(SR, r1 - base);
        const uint32_t bq = (uint32_t)(nv * row_q), bs = (uint32_t)(nv * row_s);
        mbar_arrive_expect_tx(&full[slot], NSEG * (bq + bs));
        unsigned char* st = ring + slot * stage_b;
#pragma unroll
        for (int g = 0; g < NSEG; ++g) {
          bulk_g2s_stream(st + g * seg_q, gq[g] + (size_t)base * row_q, bq, &full[slot], pol);
          bulk_g2s_stream(st + NSEG * seg_q + g * seg_s,
                          reinterpret_cast<const unsigned char*>(gs[g]) + (size_t)base * row_s,
                          bs, &full[slot], pol);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------------------ compute
  const int tid = threadIdx.x;
  const int nthreads = NCW * 32;
  pdl_wait();
  op.load_x(xs, tid, nthreads, red_tmp);

  const int wr = warp / WK, wk = warp % WK;
  const int slot0 = wk * 32 + lane;
  const float4* xs4 = reinterpret_cast<const float4*>(xs);

  for (int s = 0; s < nst; ++s) {
    const int slot = s % STAGES;
    mbar_wait(&full[slot], (s / STAGES) & 1);
    const unsigned char* st = ring + slot * stage_b;
    const int base = r0 + s * SR;
    const int nv = min(SR, r1 - base);

    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const int lr0 = wr * RPS;  // first local row (per segment) of this warp's group
    if (lr0 < nv) {
#pragma unroll 2
      for (int hb = slot0; hb < NHB; hb += WK * 32) {
        const float4 xe0 = xs4[hb], xo0 = xs4[NHB + hb];
        const float4 xe1 = xs4[2 * NHB + hb], xo1 = xs4[3 * NHB + hb];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int g = r / RPS, lr = lr0 + (r % RPS);
          const unsigned char* rq = st + g * seg_q + (size_t)lr * row_q;
          const __half* rs =
              reinterpret_cast<const __half*>(st + NSEG * seg_q + g * seg_s + (size_t)lr * row_s);
          const uint2 wv = *reinterpret_cast<const uint2*>(rq + hb * 8);
          const float sc = __half2float(rs[hb >> 1]);
          float2 p = make_float2(0.f, 0.f);
          p = dot8_nbits(wv.x, xe0, xo0, p);
          p = dot8_nbits(wv.y, xe1, xo1, p);
          acc[r] = fmaf(sc, p.x + p.y, acc[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = warp_sum(acc[r]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);

    if (WK == 1) {
      if (lane == 0 && lr0 < nv) {
        if constexpr (NSEG == 1) {
#pragma unroll
          for (int r = 0; r < R; ++r)
            if (lr0 + r < nv) op.finish(mat, base + lr0 + r, acc[r]);
        } else {
#pragma unroll
          for (int r = 0; r < RPS; ++r)
            if (lr0 + r < nv) op.finish2(base + lr0 + r, acc[r], acc[RPS + r]);
        }
      }
    } else {
      float* rb = red + (s & 1) * WR * R * WK;
      if (lane == 0) {
#pragma unroll
        for (int r = 0; r < R; ++r) rb[(wr * R + r) * WK + wk] = acc[r];
      }
      compute_bar(nthreads);
      if (wk == 0 && lane < R && lr0 + (lane % RPS) < nv) {
        float tot[NSEG];
#pragma unroll
        for (int g = 0; g < NSEG; ++g) {
          tot[g] = 0.f;
          const int r = g * RPS + (lane % RPS);
#pragma unroll
          for (int k = 0; k < WK; ++k) tot[g] += rb[(wr * R + r) * WK + k];
        }
        if constexpr (NSEG == 1) {
          op.finish(mat, base + lr0 + lane, tot[0]);
        } else {
          if (lane < RPS) op.finish2(base + lr0 + lane, tot[0], tot[1]);
        }
      }
    }
  }
}

template <class Op, class C>
cudaError_t launch_gemv(const Op& op, int K, int grid, cudaStream_t s, bool pdl) {
  const size_t smem = C::smem_bytes(K);
  auto k = gemv_kernel<Op, C>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch(k, dim3(grid), dim3(C::kThreads), smem, s, pdl, op, K);
}

int grid_for_rows(int N, int rows_per_cta_min) {
  int g = sm_count();
  const int maxg = (N + rows_per_cta_min - 1) / rows_per_cta_min;
  return g < maxg ? g : (maxg > 0 ? maxg : 1);
}

}  // namespace

// Generic fallback GEMV for any K % 32 == 0 and M <= 8: one warp per output row, x read from
// global (L2-resident), plain loads.  Used by vv_matmul_nbits when the TMA path does not apply.
namespace {
template <int M>
__global__ void __launch_bounds__(256) gemv_generic_kernel(const __half* __restrict__ x,
                                                           const uint8_t* __restrict__ q,
                                                           const __half* __restrict__ sc,
                                                           const __half* __restrict__ bias, int N,
                                                           int K, __half* __restrict__ y) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int KB = K >> 5;
  for (int n = warp; n < N; n += nwarps) {
    float acc[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc[m] = 0.f;
    for (int hb = lane; hb < 2 * KB; hb += 32) {
      const uint2 wv = *reinterpret_cast<const uint2*>(q + (size_t)n * KB * 16 + hb * 8);
      const float s = __half2float(sc[(size_t)n * KB + (hb >> 1)]);
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const __half* xr = x + (size_t)m * K + hb * 16;
        float xv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) xv[i] = __half2float(xr[i]);
        float2 p = make_float2(0.f, 0.f);
        p = dot8_nbits(wv.x, make_float4(xv[0], xv[2], xv[4], xv[6]),
                       make_float4(xv[1], xv[3], xv[5], xv[7]), p);
        p = dot8_nbits(wv.y, make_float4(xv[8], xv[10], xv[12], xv[14]),
                       make_float4(xv[9], xv[11], xv[13], xv[15]), p);
        acc[m] = fmaf(s, p.x + p.y, acc[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float v = warp_sum(acc[m]);
      if (lane == 0)
        y[(size_t)m * N + n] = __float2half_rn(v + (bias ? __half2float(bias[n]) : 0.f));
    }
  }
}

template <int M>
cudaError_t launch_generic(const uint16_t* x, GemvWeights w, const uint16_t* bias, int N, int K,
                           uint16_t* y, cudaStream_t s) {
  int grid = (N + 7) / 8;
  const int cap = sm_count() * 8;
  if (grid > cap) grid = cap;
  gemv_generic_kernel<M><<<grid, 256, 0, s>>>(
      reinterpret_cast<const __half*>(x), w.q, reinterpret_cast<const __half*>(w.scales),
      reinterpret_cast<const __half*>(bias), N, K, reinterpret_cast<__half*>(y));
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_matmul_nbits_gemv(const uint16_t* x, GemvWeights w, const uint16_t* bias,
                                     int M, int N, int K, uint16_t* y, cudaStream_t s) {
  if (M == 1 && K % 256 == 0 && K <= kMaxK) {
    OpMatmul op;
    op.a = MatmulArgs{x, w, bias, N, K, y};
    const int grid = grid_for_rows(N, 4);
    if (K <= 2048) return launch_gemv<OpMatmul, GemvCfg<4, 1, 8, 3, 1>>(op, K, grid, s, false);
    if (K <= 4096) return launch_gemv<OpMatmul, GemvCfg<4, 2, 4, 3, 1>>(op, K, grid, s, false);
    return launch_gemv<OpMatmul, GemvCfg<4, 6, 1, 3, 1>>(op, K, grid, s, false);
  }
  switch (M) {
    case 1: return launch_generic<1>(x, w, bias, N, K, y, s);
    case 2: return launch_generic<2>(x, w, bias, N, K, y, s);
    case 3: return launch_generic<3>(x, w, bias, N, K, y, s);
    case 4: return launch_generic<4>(x, w, bias, N, K, y, s);
    case 5: return launch_generic<5>(x, w, bias, N, K, y, s);
    case 6: return launch_generic<6>(x, w, bias, N, K, y, s);
    case 7: return launch_generic<7>(x, w, bias, N, K, y, s);
    default: return launch_generic<8>(x, w, bias, N, K, y, s);
  }
}

}  // namespace vv

extern "C" vv_status vv_matmul_nbits(const uint16_t* x, const uint8_t* q, const uint16_t* scales,
                                     const uint16_t* bias, int64_t M, int64_t N, int64_t K,
                                     int32_t block, uint16_t* y, vv_stream stream) {
  VV_CHECK_ARG(x && q && scales && y, "vv_matmul_nbits: null pointer");
  VV_CHECK_ARG(vv::aligned16(x) && vv::aligned16(q) && vv::aligned16(scales) && vv::aligned16(y) &&
                   (!bias || vv::aligned16(bias)),
               "vv_matmul_nbits: pointers must be 16-byte aligned");
  VV_CHECK_SHAPE(block == 32, "vv_matmul_nbits: block %d (only 32)", block);
  VV_CHECK_SHAPE(K >= 32 && K % 32 == 0 && K < (1 << 30), "vv_matmul_nbits: K=%lld", (long long)K);
  VV_CHECK_SHAPE(N >= 1 && N < (1 << 30), "vv_matmul_nbits: N=%lld", (long long)N);
  VV_CHECK_SHAPE(M >= 1 && M < (1 << 24), "vv_matmul_nbits: M=%lld", (long long)M);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M <= 8)
    return vv::cuda_check(vv::launch_matmul_nbits_gemv(x, vv::GemvWeights{q, scales}, bias, (int)M,
                                                       (int)N, (int)K, y, s),
                          "matmul_nbits GEMV launch");
  // many rows: tcgen05 GEMM with the int4 operand dequantised in shared memory
  vv::PackedB pb = {};
  pb.q[0] = q;
  pb.s[0] = scales;
  pb.rows[0] = (int)N;
  pb.nseg = 1;
  VV_CHECK_SHAPE(vv::gemm_q4_supported(pb, (int)N, (int)K),
                 "vv_matmul_nbits: M=%lld > 8 needs N %% 128 == 0 and K %% 256 == 0 (N=%lld K=%lld)",
                 (long long)M, (long long)N, (long long)K);
  vv::GemmEpilogue e = {};
  e.out_f16 = reinterpret_cast<__half*>(y);
  e.bias = reinterpret_cast<const __half*>(bias);
  e.ldo = (int)N;
  return vv::cuda_check(vv::launch_gemm_q4(x, pb, (int)M, (int)N, (int)K, vv::kEpiF16, e, s),
                        "matmul_nbits tensor-core launch");
}
