// tcgen05 tensor-core GEMM for the prefill: C[M, N] = A[M, K] . B[N, K]^T, fp16 in, fp32 out.
// (Prefill of decoder_init, "vibevoice-asr-bitnet-onnx": decoder_init contract; all projections
// of the S prompt positions are real dense contractions.)
//
// Persistent: one CTA per SM walks the 128 x BN output tiles (BN = 256, 192 or 128: the widest
// that fills the last wave of SMs about as well as any), K in blocks of 64.
//   warp 0      : TMA producer (cp.async.bulk.tensor 2D, 128-byte swizzle, this CTA only) into a
//                 ring of (A 128x64, B BNx64) fp16 stages, mbarrier complete_tx; the ring runs on
//                 across tile boundaries;
//   warp 1      : allocates 2 x BN TMEM columns (two accumulators), one thread issues
//                 tcgen05.mma kind::f16 (M = 128, N = BN, K = 16, fp32 accumulate in TMEM);
//                 tcgen05.commit releases stages and hands a finished accumulator over;
//   warps 2..5  : epilogue -- tcgen05.ld 32 lanes x 32 columns per step, fused operation, store;
//                 the accumulator is released back to the MMA warp, so the epilogue of tile i
//                 overlaps the main loop of tile i + 1.
// Epilogues: BIAS (fp32 out + fp16 bias), RESID (fp32 x += acc), SWIGLU (columns interleaved
// gate/up -> fp16 silu(g) * u), F16 (fp16 out + fp16 bias), ROPE (q/k/v + bias, rotary embedding
// of the query and key heads, fp16 queries and K/V cache rows out).  Rows >= M are masked (TMA
// zero-fills the A tail).  Every mbarrier wait is bounded; TMEM is released before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "gemm_tc.h"

namespace vv {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kStageA = BM * BK * 2;  // 16 KB
constexpr uint32_t kRingBytes = 192 * 1024;
template <int BN>
struct Cfg {
  static constexpr uint32_t kStageB = BN * BK * 2;
  static constexpr int kStages = kRingBytes / (kStageA + kStageB);  // 4 (BN 256, 192), 6 (BN 128)
  // two accumulators of BN columns; the allocation is a power of two
  static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256 : 512;
  // instruction descriptor: D f32, A/B f16, both K-major, N = BN, M = 128
  static constexpr uint32_t kIdesc =
      (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
};

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  // start address >> 4 | LBO 16 B (unused for swizzled K-major) | SBO 1024 B (8 rows x 128 B)
  // | version 1 (bit 46) | layout SWIZZLE_128B (2 << 61)
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// kEpiRope: columns [c0 + p, +32) (v1) and [c0 + 64 + p, +32) (v2) of head c0 / 128 for one row.
__device__ __forceinline__ void epilogue_rope(const GemmEpilogue& e, float (&v1)[32],
                                              float (&v2)[32], int row, int c0, int p) {
  constexpr int D = 128;
  const int head = c0 / D;
  const __half* bh;  // this head's bias (uniform over the tile)
  if (head < e.hq)
    bh = e.bias ? e.bias + (size_t)head * D : nullptr;
  else if (head < e.hq + e.hkv)
    bh = e.bias_k ? e.bias_k + (size_t)(head - e.hq) * D : nullptr;
  else
    bh = e.bias_v ? e.bias_v + (size_t)(head - e.hq - e.hkv) * D : nullptr;
  if (bh) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      const uint4 b1 = *reinterpret_cast<const uint4*>(bh + p + j);
      const uint4 b2 = *reinterpret_cast<const uint4*>(bh + D / 2 + p + j);
      const __half* h1 = reinterpret_cast<const __half*>(&b1);
      const __half* h2 = reinterpret_cast<const __half*>(&b2);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        v1[j + t] += __half2float(h1[t]);
        v2[j + t] += __half2float(h2[t]);
      }
    }
  }
  if (head < e.hq + e.hkv) {  // query or key head: rotate the pairs (d, d + 64), d = p + j
    int pos = e.pos[row];
    if (pos < 0 || pos >= e.max_pos) {
      set_device_error(VV_ERR_RANGE);
      pos = min(max(pos, 0), e.max_pos - 1);
    }
    const float* ct = e.rope_cos + (size_t)pos * (D / 2) + p;
    const float* st = e.rope_sin + (size_t)pos * (D / 2) + p;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 cs = *reinterpret_cast<const float4*>(ct + j);
      const float4 sn = *reinterpret_cast<const float4*>(st + j);
      const float c4[4] = {cs.x, cs.y, cs.z, cs.w}, s4[4] = {sn.x, sn.y, sn.z, sn.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float x1 = v1[j + t], x2 = v2[j + t];
        v1[j + t] = x1 * c4[t] - x2 * s4[t];
        v2[j + t] = x2 * c4[t] + x1 * s4[t];
      }
    }
  }
  __half* dst;
  if (head < e.hq)
    dst = e.out_f16 + (size_t)row * e.ldo + (size_t)head * D;
  else if (head < e.hq + e.hkv)
    dst = e.kc + ((size_t)(head - e.hq) * e.cap + row) * D;
  else
    dst = e.vc + ((size_t)(head - e.hq - e.hkv) * e.cap + row) * D;
#pragma unroll
  for (int j = 0; j < 32; j += 8) {
    __align__(16) __half a[8], b[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      a[t] = __float2half_rn(v1[j + t]);
      b[t] = __float2half_rn(v2[j + t]);
    }
    *reinterpret_cast<uint4*>(dst + p + j) = *reinterpret_cast<const uint4*>(a);
    *reinterpret_cast<uint4*>(dst + D / 2 + p + j) = *reinterpret_cast<const uint4*>(b);
  }
}

template <int EPI, int BN>
__device__ __forceinline__ void epilogue_chunk(const GemmEpilogue& e, const float (&v)[32], int row,
                                               int col) {
  if (EPI == kEpiBias) {
    float* out = e.out_f32 + (size_t)row * e.ldo + col;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      float4 o;
      o.x = v[j + 0] + (e.bias ? __half2float(e.bias[col + j + 0]) : 0.f);
      o.y = v[j + 1] + (e.bias ? __half2float(e.bias[col + j + 1]) : 0.f);
      o.z = v[j + 2] + (e.bias ? __half2float(e.bias[col + j + 2]) : 0.f);
      o.w = v[j + 3] + (e.bias ? __half2float(e.bias[col + j + 3]) : 0.f);
      *reinterpret_cast<float4*>(out + j) = o;
    }
  } else if (EPI == kEpiResid) {
    float* out = e.out_f32 + (size_t)row * e.ldo + col;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      float4 o = *reinterpret_cast<float4*>(out + j);
      o.x += v[j + 0];
      o.y += v[j + 1];
      o.z += v[j + 2];
      o.w += v[j + 3];
      *reinterpret_cast<float4*>(out + j) = o;
    }
  } else if (EPI == kEpiF16) {
    __half* out = e.out_f16 + (size_t)row * e.ldo + col;
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      __half h8[8];
#pragma unroll
      for (int t = 0; t < 8; ++t)
        h8[t] = __float2half_rn(v[j + t] + (e.bias ? __half2float(e.bias[col + j + t]) : 0.f));
      *reinterpret_cast<uint4*>(out + j) = *reinterpret_cast<uint4*>(h8);
    }
  } else {  // SwiGLU over interleaved (gate, up) columns -> fp16
    __half* out = e.out_f16 + (size_t)row * e.ldo + col / 2;
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
      __half h4[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float g = v[2 * (j + t)], u = v[2 * (j + t) + 1];
        h4[t] = __float2half_rn(g / (1.f + __expf(-g)) * u);
      }
      *reinterpret_cast<uint2*>(out + j) = *reinterpret_cast<uint2*>(h4);
    }
  }
}

// One accumulator row of a tile through the epilogue (kEpiRope: the two halves of each head
// together).
template <int EPI, int BN>
__device__ __forceinline__ void epilogue_row(const GemmEpilogue& e, uint32_t base, int row, int M,
                                             int col0) {
  if constexpr (EPI == kEpiRope) {
    static_assert(BN % 128 == 0, "rope tiles hold whole heads");
#pragma unroll 1
    for (int hb = 0; hb < BN; hb += 128)
#pragma unroll 1
      for (int p = 0; p < 64; p += 32) {
        float v1[32], v2[32];
        tmem_ld32(base + (uint32_t)(hb + p), v1);
        tmem_ld32(base + (uint32_t)(hb + 64 + p), v2);
        if (row < M) epilogue_rope(e, v1, v2, row, col0 + hb, p);
      }
  } else {
    for (int c = 0; c < BN; c += 32) {
      float v[32];
      tmem_ld32(base + (uint32_t)c, v);
      if (row < M) epilogue_chunk<EPI, BN>(e, v, row, col0 + c);
    }
  }
}


template <int EPI, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmEpilogue e, const int M, const int N, const int K) {
  using C = Cfg<BN>;
  constexpr int STAGES = C::kStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;
  unsigned char* sB = smem + STAGES * kStageA;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * C::kStageB);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;    // [2] epilogue -> MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = N / BN;
  const int tiles = ((M + BM - 1) / BM) * n_tiles;
  const int kblocks = K / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);  // one arrival per epilogue warp
    }
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;  // running k-block counter across tiles
      for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int m_blk = t / n_tiles, n_blk = t % n_tiles;
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const int s = g % STAGES;
          if (g >= STAGES) mbar_wait(&empty[s], ((g / STAGES) - 1) & 1);
          mbar_arrive_expect_tx(&full[s], kStageA + C::kStageB);
          tma_load_2d(sA + s * kStageA, &tmA, kb * BK, m_blk * BM, &full[s]);
          tma_load_2d(sB + s * C::kStageB, &tmB, kb * BK, n_blk * BN, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int g = 0, i = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int buf = i & 1;
        if (i >= 2) mbar_wait(&acc_empty[buf], ((i >> 1) - 1) & 1);  // epilogue done with it
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const int s = g % STAGES;
          mbar_wait(&full[s], (g / STAGES) & 1);
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kStageA), b0 = smem_u32(sB + s * C::kStageB);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)  // 32 bytes per K=16 slice inside the swizzled row
            umma_f16(d, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), C::kIdesc,
                     (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[s]);  // stage free once these MMAs have read it
        }
        umma_commit(&acc_full[buf]);  // accumulator complete
      }
    }
    __syncwarp();
  } else {
    // epilogue warps 2..5: TMEM lanes 32 * (warp % 4) .. + 31
    const int q = warp & 3;
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int m_blk = t / n_tiles, n_blk = t % n_tiles;
      const int buf = i & 1;
      const int row = m_blk * BM + q * 32 + lane;
      mbar_wait(&acc_full[buf], (i >> 1) & 1);
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
      epilogue_row<EPI, BN>(e, base, row, M, n_blk * BN);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------- packed int4 B operand
// The same GEMM with B given as MatMulNBits codes + fp16 scales (up to three row segments of one
// matrix stack, or two segments interleaved row by row): the int4 weights are dequantised into
// the fp16 B tile in shared memory, never written to global memory.
//   warp 0      : TMA producer: per 64-wide k block, the A tile (fp16 128 x 64), the codes
//                 (BN rows x 32 bytes) and the scales (BN rows x 8 blocks, the 256-wide group
//                 holding this k block) into a ring of raw stages;
//   warp 1      : TMEM allocation, one thread issues tcgen05.mma kind::f16 from the A stage and
//                 the converted B stage; commits release both;
//   warps 2..5  : epilogue (as above);
//   warps 6..9  : converters: codes + scale -> fp16((code - 8) * scale) (one rounding, as the
//                 fp32 product rounded to fp16) written in the 128-byte-swizzled K-major layout
//                 of a B stage (a second, smaller ring).
constexpr int kQThreads = 320;
template <int BN>
struct QCfg {
  static constexpr uint32_t kCodes = BN * 32;     // codes of one k block (64 columns)
  static constexpr uint32_t kScales = BN * 16;    // scales of 8 blocks (256 columns)
  static constexpr uint32_t kRaw = kStageA + kCodes + kScales;
  static constexpr int kRawStages = 4;
  static constexpr uint32_t kStageB = BN * BK * 2;
  static constexpr int kBStages = 2;
  static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256 : 512;
  static constexpr uint32_t kIdesc = Cfg<BN>::kIdesc;
};

struct PackedMaps {
  CUtensorMap q[3];  // uint8 [rows_m, K/2], box {32, BN (or BN/2 interleaved)}
  CUtensorMap s[3];  // fp16 [rows_m, K/32], box {8, BN (or BN/2)}
  int row0[4];       // first output row of each segment (non-interleaved), row0[nseg] = N
  int nseg;
  int interleave;
};

__device__ __forceinline__ void tma_load_2d_u(void* dst, const CUtensorMap* tm, int c0, int c1,
                                              uint64_t* bar) {
  tma_load_2d(dst, tm, c0, c1, bar);
}

// (code - 8) * scale for the 8 elements of one code word, natural order, as 4 fp16 pairs.
__device__ __forceinline__ uint4 dequant8_f16(uint32_t w, uint32_t s2) {
  uint32_t o[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    uint32_t y, h, d;
    // byte t of w into bytes 0 and 2; low nibble -> low half, high nibble -> high half mantissa
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(y) : "r"(w), "r"((uint32_t)(t | 0x40 | (t << 8) | 0x4000)));
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(y), "r"(0x00F0000Fu), "r"(0x64006400u));
    // (1024 + c) - 1032 = c - 8; (1024 + 16 c) / 16 - 72 = c - 8  (exact in fp16)
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(h), "r"(0x2C003C00u), "r"(0xD480E408u));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[t]) : "r"(d), "r"(s2));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int EPI, int BN>
__global__ void __launch_bounds__(kQThreads, 1)
    gemm_q4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ PackedMaps pm,
                   const GemmEpilogue e, const int M, const int N, const int K) {
  using C = QCfg<BN>;
  constexpr int RS = C::kRawStages, BS = C::kBStages;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sB = smem;                       // BS x kStageB (1024-aligned)
  unsigned char* sRaw = smem + BS * C::kStageB;    // RS x kRaw (A first: 1024-aligned)
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(sRaw + RS * C::kRaw);
  uint64_t* raw_empty = raw_full + RS;
  uint64_t* b_full = raw_empty + RS;
  uint64_t* b_empty = b_full + BS;
  uint64_t* acc_full = b_empty + BS;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = N / BN;
  const int tiles = ((M + BM - 1) / BM) * n_tiles;
  const int kblocks = K / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < RS; ++i) {
      mbar_init(&raw_full[i], 1);
      mbar_init(&raw_empty[i], 1 + 4);  // the MMA commit (A read) + 4 converter warps (codes)
    }
    for (int i = 0; i < BS; ++i) {
      mbar_init(&b_full[i], 4);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
        const int m_blk = t / n_tiles, n_blk = t % n_tiles;
        const int n0 = n_blk * BN;
        // segment and its first row of this tile (tiles never straddle segments)
        int sg = 0, r0 = 0;
        if (!pm.interleave) {
          while (sg + 1 < pm.nseg && n0 >= pm.row0[sg + 1]) ++sg;
          r0 = n0 - pm.row0[sg];
        } else {
          r0 = n0 / 2;
        }
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const int s = g % RS;
          if (g >= RS) mbar_wait(&raw_empty[s], ((g / RS) - 1) & 1);
          mbar_arrive_expect_tx(&raw_full[s], C::kRaw);
          unsigned char* st = sRaw + s * C::kRaw;
          tma_load_2d(st, &tmA, kb * BK, m_blk * BM, &raw_full[s]);
          const int sx = (kb * 2) & ~7;  // first of the 8 scale blocks holding this k block
          if (!pm.interleave) {
            tma_load_2d(st + kStageA, &pm.q[sg], kb * 32, r0, &raw_full[s]);
            tma_load_2d(st + kStageA + C::kCodes, &pm.s[sg], sx, r0, &raw_full[s]);
          } else {
            tma_load_2d(st + kStageA, &pm.q[0], kb * 32, r0, &raw_full[s]);
            tma_load_2d(st + kStageA + C::kCodes / 2, &pm.q[1], kb * 32, r0, &raw_full[s]);
            tma_load_2d(st + kStageA + C::kCodes, &pm.s[0], sx, r0, &raw_full[s]);
            tma_load_2d(st + kStageA + C::kCodes + C::kScales / 2, &pm.s[1], sx, r0, &raw_full[s]);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int g = 0, i = 0;
      for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
        const int buf = i & 1;
        if (i >= 2) mbar_wait(&acc_empty[buf], ((i >> 1) - 1) & 1);
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const int s = g % RS, sb = g % BS;
          mbar_wait(&raw_full[s], (g / RS) & 1);
          mbar_wait(&b_full[sb], (g / BS) & 1);
          tc_fence_after();
          const uint32_t a0 = smem_u32(sRaw + s * C::kRaw), b0 = smem_u32(sB + sb * C::kStageB);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_f16(d, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), C::kIdesc,
                     (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(&raw_empty[s]);
          umma_commit(&b_empty[sb]);
        }
        umma_commit(&acc_full[buf]);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    const int q = warp & 3;
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int m_blk = t / n_tiles, n_blk = t % n_tiles;
      const int buf = i & 1;
      const int row = m_blk * BM + q * 32 + lane;
      mbar_wait(&acc_full[buf], (i >> 1) & 1);
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN);
      epilogue_row<EPI, BN>(e, base, row, M, n_blk * BN);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  } else {
    // converters: thread ct owns B rows ct, ct + 128 (< BN)
    const int ct = threadIdx.x - 6 * 32;
    int g = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb, ++g) {
        const int s = g % RS, sb = g % BS;
        mbar_wait(&raw_full[s], (g / RS) & 1);
        if (g >= BS) mbar_wait(&b_empty[sb], ((g / BS) - 1) & 1);
        const unsigned char* codes = sRaw + s * C::kRaw + kStageA;
        const __half* scl = reinterpret_cast<const __half*>(codes + C::kCodes);
        unsigned char* bt = sB + sb * C::kStageB;
        const int sj = (kb * 2) & 7;  // this k block's first scale within the 8 loaded
#pragma unroll
        for (int rr = 0; rr < (BN + 127) / 128; ++rr) {
          const int n = ct + rr * 128;
          if (n < BN) {
            // source row of output row n in the codes / scales tiles
            const int src = pm.interleave ? (n & 1) * (BN / 2) + (n >> 1) : n;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const uint4 cw = *reinterpret_cast<const uint4*>(codes + src * 32 + j * 16);
              const uint16_t sh = reinterpret_cast<const uint16_t*>(scl)[src * 8 + sj + j];
              const uint32_t s2 = (uint32_t)sh | ((uint32_t)sh << 16);
              const uint32_t w4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int chunk = 4 * j + c;  // 16-byte chunk of the 128-byte row
                *reinterpret_cast<uint4*>(bt + n * 128 + ((chunk ^ (n & 7)) << 4)) =
                    dequant8_f16(w4[c], s2);
              }
            }
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&b_full[sb]);
          mbar_arrive(&raw_empty[s]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// fp16 row-major [rows, cols] (cols contiguous), box {64 cols, box_rows}, 128-byte swizzle.
bool make_map(CUtensorMap* tm, const void* base, int rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Wave efficiency of a tile count on the SMs: tiles / (waves * SMs).
static double wave_eff(long tiles, int sms) {
  const long waves = (tiles + sms - 1) / sms;
  return (double)tiles / (double)(waves * sms);
}

namespace {

// Generic 2D tensor map: [rows, cols] of `dtype` elements of `esize` bytes, box {bc, br}.
bool make_map2(CUtensorMap* tm, CUtensorMapDataType dtype, int esize, const void* base, int rows,
               int cols, int bc, int br) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
  cuuint32_t box[2] = {(cuuint32_t)bc, (cuuint32_t)br};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int scale_pitch(const PackedB& B, int K) { return B.s_pitch > 0 ? B.s_pitch : K / 32; }

template <int BN>
size_t q4_smem_bytes() {
  using C = QCfg<BN>;
  return C::kBStages * C::kStageB + C::kRawStages * C::kRaw + (2 * C::kRawStages + 2 * C::kBStages + 4) * 8 +
         16 + 1024;
}

template <int EPI, int BN>
cudaError_t run_q4(const CUtensorMap& ta, const PackedMaps& pm, const GemmEpilogue& e, int M,
                   int N, int K, int grid, cudaStream_t s) {
  const size_t smem = q4_smem_bytes<BN>();
  cudaError_t err = cudaFuncSetAttribute(gemm_q4_kernel<EPI, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  gemm_q4_kernel<EPI, BN><<<grid, kQThreads, smem, s>>>(ta, pm, e, M, N, K);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_q4_bn(const uint16_t* A, const PackedB& B, int M, int N, int K, int epi,
                         const GemmEpilogue& e, cudaStream_t s) {
  CUtensorMap ta;
  if (!make_map(&ta, A, M, K, BM)) return cudaErrorInvalidValue;
  PackedMaps pm = {};
  pm.nseg = B.nseg;
  pm.interleave = B.interleave;
  const int br = B.interleave ? BN / 2 : BN;
  int r = 0;
  for (int g = 0; g < B.nseg; ++g) {
    if (!make_map2(&pm.q[g], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B.q[g], B.rows[g], K / 2, 32, br) ||
        !make_map2(&pm.s[g], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, B.s[g], B.rows[g], scale_pitch(B, K), 8, br))
      return cudaErrorInvalidValue;
    pm.row0[g] = r;
    r += B.rows[g];
  }
  pm.row0[B.nseg] = r;
  const int tiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  switch (epi) {
    case kEpiBias: return run_q4<kEpiBias, BN>(ta, pm, e, M, N, K, grid, s);
    case kEpiResid: return run_q4<kEpiResid, BN>(ta, pm, e, M, N, K, grid, s);
    case kEpiSwiglu: return run_q4<kEpiSwiglu, BN>(ta, pm, e, M, N, K, grid, s);
    case kEpiF16: return run_q4<kEpiF16, BN>(ta, pm, e, M, N, K, grid, s);
    case kEpiRope:
      if constexpr (BN % 128 == 0) return run_q4<kEpiRope, BN>(ta, pm, e, M, N, K, grid, s);
      return cudaErrorInvalidValue;  // tiles of 192 columns split heads
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

namespace {
// The whole matrix stack dequantised to fp16 [total_rows, K] (the B operand of gemm_tc_kernel):
// one thread per 32-weight block, (code - 8) * scale rounded once to fp16 (dequant8_f16), rows
// of up to three segments, or two segments interleaved row by row.
__global__ void __launch_bounds__(256) dequant_f16_kernel(const DequantSrc src, int total_rows,
                                                          int K, __half* __restrict__ out) {
  const int KB = K >> 5;
  const int64_t nblk = (int64_t)total_rows * KB;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk;
       b += (int64_t)gridDim.x * blockDim.x) {
    const int orow = (int)(b / KB), kb = (int)(b % KB);
    int m, r;
    if (src.interleave) {
      m = orow & 1;
      r = orow >> 1;
    } else {
      m = 0;
      r = orow;
      while (m < src.nseg - 1 && r >= src.rows[m]) r -= src.rows[m++];
    }
    const uint4 codes = __ldg(reinterpret_cast<const uint4*>(src.q[m] + ((size_t)r * KB + kb) * 16));
    const uint32_t sh = src.s[m][(size_t)r * KB + kb];
    const uint32_t s2 = sh | (sh << 16);
    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)orow * K + (size_t)kb * 32);
    dst[0] = dequant8_f16(codes.x, s2);
    dst[1] = dequant8_f16(codes.y, s2);
    dst[2] = dequant8_f16(codes.z, s2);
    dst[3] = dequant8_f16(codes.w, s2);
  }
}

}  // namespace

namespace {
// Several matrix stacks in one launch.  Work unit = (output row, piece of 1024 columns): one warp,
// lane l expanding code words 128 * piece + l + 32 t (t < 4; 8 weights each), all loads issued
// before the first store, so each store instruction of a warp writes 512 contiguous bytes.  Job j
// covers units [first[j], first[j + 1]).
constexpr int kDqWords = 4;                   // code words per lane per unit
constexpr int kDqCols = 32 * kDqWords * 8;    // columns per unit
struct DequantJobs {
  DequantSrc src[4];
  __half* out[4];
  int K[4];
  int first[5];
  int n;
};

__global__ void __launch_bounds__(256) dequant_jobs_kernel(const DequantJobs jb) {
  const int lane = threadIdx.x & 31;
  const int total = jb.first[jb.n];
  const int nw = (int)gridDim.x * (int)(blockDim.x >> 5);
  for (int u = (int)blockIdx.x * (int)(blockDim.x >> 5) + (int)(threadIdx.x >> 5); u < total;
       u += nw) {
    int j = 0;
    while (j + 1 < jb.n && u >= jb.first[j + 1]) ++j;
    const DequantSrc& src = jb.src[j];
    const int K = jb.K[j], KB = K >> 5, PK = (K + kDqCols - 1) / kDqCols, nwords = K >> 3;
    const int v = u - jb.first[j];
    const int orow = v / PK;
    const int c0 = (v - orow * PK) * (32 * kDqWords) + lane;  // first code word of this lane
    int m, r;
    if (src.interleave) {
      m = orow & 1;
      r = orow >> 1;
    } else {
      m = 0;
      r = orow;
      while (m < src.nseg - 1 && r >= src.rows[m]) r -= src.rows[m++];
    }
    // word c of a row = word c % 4 of block c / 4: 8 consecutive weights
    const uint32_t* qr = reinterpret_cast<const uint32_t*>(src.q[m]) + (size_t)r * KB * 4;
    const uint16_t* sr = src.s[m] + (size_t)r * KB;
    uint32_t w[kDqWords], sh[kDqWords];
#pragma unroll
    for (int t = 0; t < kDqWords; ++t) {
      const int c = c0 + 32 * t;
      w[t] = c < nwords ? __ldg(qr + c) : 0u;
      sh[t] = c < nwords ? (uint32_t)__ldg(sr + (c >> 2)) : 0u;
    }
    uint4* dst = reinterpret_cast<uint4*>(jb.out[j] + (size_t)orow * K);
#pragma unroll
    for (int t = 0; t < kDqWords; ++t) {
      const int c = c0 + 32 * t;
      if (c < nwords) dst[c] = dequant8_f16(w[t], sh[t] | (sh[t] << 16));
    }
  }
}
}  // namespace

cudaError_t launch_dequant_many(const DequantSrc* src, const int* rows, const int* K,
                                __half* const* out, int n, cudaStream_t s) {
  if (n < 1 || n > 4) return cudaErrorInvalidValue;
  DequantJobs jb = {};
  jb.n = n;
  jb.first[0] = 0;
  for (int j = 0; j < n; ++j) {
    if (K[j] % 32 != 0 || rows[j] < 0) return cudaErrorInvalidValue;
    jb.src[j] = src[j];
    jb.out[j] = out[j];
    jb.K[j] = K[j];
    const int64_t next = (int64_t)jb.first[j] + (int64_t)rows[j] * ((K[j] + kDqCols - 1) / kDqCols);
    if (next > 0x7fffffff) return cudaErrorInvalidValue;
    jb.first[j + 1] = (int)next;
  }
  int64_t grid = ((int64_t)jb.first[n] + 7) / 8;  // 8 warps per CTA
  const int64_t cap = (int64_t)sm_count() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  dequant_jobs_kernel<<<(int)grid, 256, 0, s>>>(jb);
  return cudaGetLastError();
}

cudaError_t launch_dequant_f16(const DequantSrc& src, int total_rows, int K, __half* out,
                               cudaStream_t s) {
  const int64_t nblk = (int64_t)total_rows * (K >> 5);
  int64_t grid = (nblk + 255) / 256;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  dequant_f16_kernel<<<(int)grid, 256, 0, s>>>(src, total_rows, K, out);
  return cudaGetLastError();
}

namespace {

template <int BN>
size_t smem_bytes() {
  return Cfg<BN>::kStages * (kStageA + Cfg<BN>::kStageB) + 2 * Cfg<BN>::kStages * 8 + 4 * 8 + 16 +
         1024;
}

template <int EPI, int BN>
cudaError_t run_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmEpilogue& e, int M,
                     int N, int K, int grid, cudaStream_t s) {
  const size_t smem = smem_bytes<BN>();
  cudaError_t err = cudaFuncSetAttribute(gemm_tc_kernel<EPI, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  gemm_tc_kernel<EPI, BN><<<grid, kThreads, smem, s>>>(ta, tb, e, M, N, K);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const uint16_t* A, const uint16_t* B, int M, int N, int K, int epi,
                      const GemmEpilogue& e, cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!make_map(&ta, A, M, K, BM) || !make_map(&tb, B, N, K, BN)) return cudaErrorInvalidValue;
  const int tiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = tiles < sm_count() ? tiles : sm_count();
  switch (epi) {
    case kEpiBias: return run_gemm<kEpiBias, BN>(ta, tb, e, M, N, K, grid, s);
    case kEpiResid: return run_gemm<kEpiResid, BN>(ta, tb, e, M, N, K, grid, s);
    case kEpiSwiglu: return run_gemm<kEpiSwiglu, BN>(ta, tb, e, M, N, K, grid, s);
    case kEpiF16: return run_gemm<kEpiF16, BN>(ta, tb, e, M, N, K, grid, s);
    case kEpiRope:
      if constexpr (BN % 128 == 0) return run_gemm<kEpiRope, BN>(ta, tb, e, M, N, K, grid, s);
      return cudaErrorInvalidValue;  // tiles of 192 columns split heads
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool gemm_q4_supported(const PackedB& B, int N, int K) {
  if (K < BK || K % BK != 0 || B.nseg < 1 || B.nseg > 3) return false;
  const int sp = scale_pitch(B, K);
  if (sp % 8 != 0 || sp < ((K / 32 + 7) & ~7)) return false;
  if (B.interleave) return B.nseg == 2 && B.rows[0] == B.rows[1] && N == 2 * B.rows[0] && N % 128 == 0;
  int tot = 0;
  for (int g = 0; g < B.nseg; ++g) {
    if (B.rows[g] % 128 != 0) return false;
    tot += B.rows[g];
  }
  return tot == N;
}

cudaError_t launch_gemm_q4(const uint16_t* A, const PackedB& B, int M, int N, int K, int epi,
                           const GemmEpilogue& e, cudaStream_t s) {
  if (M < 1 || !gemm_q4_supported(B, N, K) || !aligned16(A)) return cudaErrorInvalidValue;
  if (epi == kEpiRope && (N % 128 != 0 || !e.pos || !e.kc || !e.vc)) return cudaErrorInvalidValue;
  for (int g = 0; g < B.nseg; ++g)
    if (!aligned16(B.q[g]) || !aligned16(B.s[g])) return cudaErrorInvalidValue;
  const int sms = sm_count();
  const long mt = (M + BM - 1) / BM;
  // tile width: segments (or interleaved pairs) must hold whole tiles; among the widths that
  // fit, the widest whose wave efficiency is within 0.1 of the best
  auto fits = [&](int w) {
    if (N % w != 0 || (epi == kEpiRope && w % 128 != 0)) return false;
    if (B.interleave) return (w / 2) % 8 == 0;
    for (int g = 0; g < B.nseg; ++g)
      if (B.rows[g] % w != 0) return false;
    return true;
  };
  const int widths[3] = {256, 192, 128};
  double best = 0.0;
  for (int w : widths)
    if (fits(w)) best = std::max(best, wave_eff(mt * (N / w), sms));
  for (int w : widths) {
    if (!fits(w) || wave_eff(mt * (N / w), sms) < best - 0.1) continue;
    if (w == 256) return launch_q4_bn<256>(A, B, M, N, K, epi, e, s);
    if (w == 192) return launch_q4_bn<192>(A, B, M, N, K, epi, e, s);
    return launch_q4_bn<128>(A, B, M, N, K, epi, e, s);
  }
  return cudaErrorInvalidValue;
}

size_t gemm_tc_smem() { return smem_bytes<256>(); }


cudaError_t launch_gemm_tc(const uint16_t* A, const uint16_t* B, int M, int N, int K, int epi,
                           const GemmEpilogue& e, cudaStream_t s) {
  if (M < 1 || N % 64 != 0 || K % BK != 0 || K < BK) return cudaErrorInvalidValue;
  if (epi == kEpiRope && (N % 128 != 0 || !e.pos || !e.kc || !e.vc)) return cudaErrorInvalidValue;
  if (!aligned16(A) || !aligned16(B)) return cudaErrorInvalidValue;
  const int sms = sm_count();
  const long mt = (M + BM - 1) / BM;
  // the widest tile whose wave efficiency is within 0.1 of the best available width
  const int widths[3] = {256, 192, 128};
  auto fits = [&](int w) { return N % w == 0 && (epi != kEpiRope || w % 128 == 0); };
  double best = 0.0;
  for (int w : widths)
    if (fits(w)) best = std::max(best, wave_eff(mt * (N / w), sms));
  for (int w : widths) {
    if (!fits(w) || wave_eff(mt * (N / w), sms) < best - 0.1) continue;
    if (w == 256) return launch_bn<256>(A, B, M, N, K, epi, e, s);
    if (w == 192) return launch_bn<192>(A, B, M, N, K, epi, e, s);
    return launch_bn<128>(A, B, M, N, K, epi, e, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vv
