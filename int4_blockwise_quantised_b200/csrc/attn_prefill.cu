// Causal grouped-query attention for the prefill ("vibevoice-asr-bitnet-onnx": decoder_init over
// S positions; attention is causal and query head h reads key/value head h / (Hq/Hkv)).
//
//   O[i, h] = sum_{j <= i} softmax_j(scale * Q[i, h] . K[j, g]) V[j, g]
//
// One CTA = 64 queries x one query head, 4 warps of 16 queries.  Key/value blocks of 64
// positions stream global -> shared with cp.async (16-byte chunks XOR-swizzled by row so the
// ldmatrix reads are bank-conflict free), double-buffered.  S = Q K^T and O += P V run on
// mma.sync m16n8k16 (fp16 in, fp32 accumulate); the online softmax lives in registers (exp2 of
// scores pre-scaled by log2 e); P is re-packed from the S accumulators into A fragments.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "attn_prefill.h"

namespace vv {
namespace {

constexpr int D = 128;
constexpr int QB = 64;  // queries per CTA
constexpr int KB = 64;  // keys per block
constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {  // byte offset inside a tile
  return (uint32_t)(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // zero-fill past the end of the sequence
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

constexpr int kTile = KB * D * 2;  // 16 KB
constexpr int kSmem = 4 * kTile;     // K and V, double-buffered

__global__ void __launch_bounds__(kThreads) attn_prefill_kernel(const AttnPrefillArgs a) {
  extern __shared__ __align__(128) unsigned char smem_dyn[];
  unsigned char* sK[2] = {smem_dyn, smem_dyn + kTile};
  unsigned char* sV[2] = {smem_dyn + 2 * kTile, smem_dyn + 3 * kTile};
  const int qb = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv, g = h / G;
  const int S = a.S;
  const int q0 = qb * QB;
  const __half* kc = reinterpret_cast<const __half*>(a.k_cache) + (size_t)g * a.cap * D;
  const __half* vc = reinterpret_cast<const __half*>(a.v_cache) + (size_t)g * a.cap * D;
  const float sl2 = a.scale * kLog2e;

  // ---- Q fragments of this warp's 16 rows (A operand, row-major), straight from global
  const int gq = lane >> 2, tq = lane & 3;
  const int r_lo = q0 + warp * 16 + gq, r_hi = r_lo + 8;
  uint32_t qf[8][4];
  {
    const __half* q = reinterpret_cast<const __half*>(a.q);
    const size_t ld = (size_t)a.Hq * D;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c0 = ks * 16 + 2 * tq;
      auto ld2 = [&](int r, int c) -> uint32_t {
        if (r >= S) return 0u;
        return *reinterpret_cast<const uint32_t*>(q + (size_t)r * ld + (size_t)h * D + c);
      };
      qf[ks][0] = ld2(r_lo, c0);
      qf[ks][1] = ld2(r_hi, c0);
      qf[ks][2] = ld2(r_lo, c0 + 8);
      qf[ks][3] = ld2(r_hi, c0 + 8);
    }
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

  const int nkb = min((q0 + QB - 1) / KB, (S - 1) / KB) + 1;  // causal: blocks up to the diagonal
  auto load_kv = [&](int kb, int buf) {
    const int k0 = kb * KB;
    for (int i = threadIdx.x; i < KB * (D / 8); i += kThreads) {
      const int r = i >> 4, c = i & 15;
      const bool ok = k0 + r < S;
      const size_t off = (size_t)(ok ? k0 + r : 0) * D + c * 8;
      cp_async16(smem_u32(sK[buf]) + swz(r, c), kc + off, ok);
      cp_async16(smem_u32(sV[buf]) + swz(r, c), vc + off, ok);
    }
    cp_async_commit();
  };
  load_kv(0, 0);

  for (int kb = 0; kb < nkb; ++kb) {
    const int buf = kb & 1;
    if (kb + 1 < nkb) {
      load_kv(kb + 1, buf ^ 1);
      cp_async_wait1();
    } else {
      cp_async_wait0();
    }
    __syncthreads();
    const uint32_t kbase = smem_u32(sK[buf]), vbase = smem_u32(sV[buf]);
    // ---- S = Q K^T : 16 rows x 64 keys per warp (8 n-tiles of 8 keys)
    float sc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {  // pairs of n-tiles: keys 16jp .. 16jp+15
        // matrices: (keys 16jp+0..7, d 16ks+0..7), (same keys, d +8..15),
        //           (keys 16jp+8..15, d 16ks+0..7), (keys +8..15, d +8..15)
        const int mi = lane >> 3, rr = lane & 7;
        const int key = jp * 16 + ((mi >> 1) << 3) + rr;
        const int chunk = ks * 2 + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + swz(key, chunk), b0, b1, b2, b3);
        mma16816(sc[2 * jp], qf[ks], b0, b1);
        mma16816(sc[2 * jp + 1], qf[ks], b2, b3);
      }
    }
    // ---- scale, causal mask, online softmax (rows lo = gq, hi = gq + 8 of this warp)
    const int k0 = kb * KB;
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + j * 8 + 2 * tq + (e & 1);
        const int row = (e < 2) ? r_lo : r_hi;
        float v = sc[j][e] * sl2;
        if (key > row || key >= S) v = -INFINITY;
        sc[j][e] = v;
      }
      mx_lo = fmaxf(mx_lo, fmaxf(sc[j][0], sc[j][1]));
      mx_hi = fmaxf(mx_hi, fmaxf(sc[j][2], sc[j][3]));
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, off));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, off));
    }
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    // rows with no valid key yet keep -inf; use 0 as the reference to avoid inf - inf
    const float ref_lo = mn_lo == -INFINITY ? 0.f : mn_lo;
    const float ref_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float cr_lo = exp2f(m_lo - ref_lo), cr_hi = exp2f(m_hi - ref_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    float sum_lo = 0.f, sum_hi = 0.f;
    uint32_t pf[4][4];  // P as A fragments, 4 k-steps of 16 keys
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = exp2f(sc[j][0] - ref_lo), p1 = exp2f(sc[j][1] - ref_lo);
      const float p2 = exp2f(sc[j][2] - ref_hi), p3 = exp2f(sc[j][3] - ref_hi);
      sum_lo += p0 + p1;
      sum_hi += p2 + p3;
      const int s = j >> 1, half = j & 1;
      pf[s][half * 2 + 0] = pack_h2(p0, p1);  // a0 / a2: row lo
      pf[s][half * 2 + 1] = pack_h2(p2, p3);  // a1 / a3: row hi
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, off);
      sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, off);
    }
    l_lo = l_lo * cr_lo + sum_lo;
    l_hi = l_hi * cr_hi + sum_hi;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= cr_lo;
      o[i][1] *= cr_lo;
      o[i][2] *= cr_hi;
      o[i][3] *= cr_hi;
    }
    // ---- O += P V : 16 d n-tiles of 8, 4 key k-steps of 16
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {  // pairs of d n-tiles: d 16dp .. 16dp+15
        // .trans matrices: (keys 16s+0..7, d 16dp+0..7), (keys 16s+8..15, d 16dp+0..7),
        //                  (keys 16s+0..7, d 16dp+8..15), (keys +8..15, d +8..15)
        const int mi = lane >> 3, rr = lane & 7;
        const int key = s * 16 + ((mi & 1) << 3) + rr;
        const int chunk = dp * 2 + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + swz(key, chunk), b0, b1, b2, b3);
        mma16816(o[2 * dp], pf[s], b0, b1);
        mma16816(o[2 * dp + 1], pf[s], b2, b3);
      }
    }
    __syncthreads();  // buffer `buf` is reloaded two iterations later
  }
  // ---- normalise and store O [S, Hq * D] fp16
  const float il_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, il_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
  __half* out = reinterpret_cast<__half*>(a.out);
  const size_t ld = (size_t)a.Hq * D;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int d = i * 8 + 2 * tq;
    if (r_lo < S)
      *reinterpret_cast<uint32_t*>(out + (size_t)r_lo * ld + (size_t)h * D + d) =
          pack_h2(o[i][0] * il_lo, o[i][1] * il_lo);
    if (r_hi < S)
      *reinterpret_cast<uint32_t*>(out + (size_t)r_hi * ld + (size_t)h * D + d) =
          pack_h2(o[i][2] * il_hi, o[i][3] * il_hi);
  }
}

}  // namespace

cudaError_t launch_attn_prefill(const AttnPrefillArgs& a, cudaStream_t s) {
  cudaError_t e =
      cudaFuncSetAttribute(attn_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.S + QB - 1) / QB, a.Hq);
  attn_prefill_kernel<<<grid, kThreads, kSmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace vv
