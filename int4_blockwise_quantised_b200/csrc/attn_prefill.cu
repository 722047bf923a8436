// Causal grouped-query attention for the prefill ("vibevoice-asr-bitnet-onnx": decoder_init over
// S positions; attention is causal and query head h reads key/value head h / (Hq/Hkv)).
//
//   O[i, h] = sum_{j <= i} softmax_j(scale * Q[i, h] . K[j, g]) V[j, g]
//
// Flash attention on the 5th-generation tensor cores.  One CTA = 128 queries x one query head;
// key/value blocks of 128 positions up to the diagonal.
//   warp 0      : TMA producer of the Q tile (once) and the K tiles (128 x 128 fp16, 128-byte
//                 swizzle, two 64-column boxes each) into a three-stage ring; a K stage is free
//                 again as soon as the S MMAs that read it are done;
//   warp 10     : TMA producer of the V tiles into a two-stage ring (free after P.V);
//   warp 1      : allocates TMEM (three S / P buffers + O: 512 columns), one thread issues the
//                 MMAs: S_j = Q K_j^T (kind::f16, A = Q and B = K_j from shared memory,
//                 K-major) into buffer j % 3, and O += P_j V_j (A = P_j from tensor memory, B =
//                 V_j from shared memory read MN-major, i.e. straight from the row-major cache
//                 tile); S_{j+2} is queued right behind P_j V_j, so the tensor pipe has the next
//                 scores to compute while the softmax of block j + 1 runs;
//   warps 2..9  : softmax, two threads per query row (TMEM lane), 64 keys each: reads S_j,
//                 applies the scale (log2 domain) and the causal mask, exponentiates against the
//                 row's running maximum and writes P_j (fp16) over S_j in tensor memory (the two
//                 halves of a row exchange the block maximum first); O is rescaled only when
//                 a block's maximum exceeds the running one by more than 2^8 (the exponentials
//                 stay below 2^8, and the final division uses the same maxima); at the end O / l
//                 is rounded to fp16 and stored.
// Every mbarrier wait is bounded; TMEM is released before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "attn_prefill.h"

namespace vv {
namespace {

constexpr int D = 128;
constexpr int BQ = 128;   // queries per CTA (TMEM lanes)
constexpr int BKV = 128;  // keys per block
constexpr int kThreads = 352;  // K producer, MMA issuer, 8 softmax warps, V producer
constexpr int kVWarp = 10;
constexpr int kKStages = 3;   // K tiles in flight (a stage is free once its S MMAs are done)
constexpr int kVStages = 2;   // V tiles in flight (free once the P.V MMAs are done)
constexpr int kSBufs = 3;     // S / P buffers in tensor memory (+ O: 512 columns)
constexpr int kTiles = 1 + kKStages + kVStages;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;  // log2 headroom before O is rescaled
constexpr uint32_t kTile = 128 * 128 * 2;  // one 128 x 128 fp16 tile: two 64-column atoms
constexpr uint32_t kAtom = 128 * 128;      // 128 rows x 128 bytes
constexpr uint32_t kBarBytes = 256;         // mbarriers + the TMEM address slot

// instruction descriptors (kind::f16, D f32, M = 128, N = 128): S (both K-major); PV (B MN-major)
constexpr uint32_t kIdescS = (1u << 4) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kIdescPV = kIdescS | (1u << 16);

// K-major, 128-byte swizzle: SBO = 1024 (8 rows x 128 B)
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major, 128-byte swizzle: LBO = next 64 N-elements (the second 64-column atom), SBO = next 8
// K-rows (1024 B)
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(kAtom >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
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
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x by the special-function unit (flushes results below 2^-126 to zero; -inf -> 0).  P is
// rounded to fp16 afterwards, far coarser than the instruction's error.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named barrier of the two softmax warps that share TMEM lane quarter q (ids 1..4, 64 threads).
__device__ __forceinline__ void pair_sync(int q) {
  asm volatile("bar.sync %0, 64;" ::"r"(q + 1) : "memory");
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

struct Maps {
  CUtensorMap q;   // fp16 [S, Hq * D], box {64, 128}
  CUtensorMap kv[2];  // fp16 [Hkv][S][D] (K, V): dims {D, S, Hkv}, box {64, 128, 1}
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_tc_kernel(const __grid_constant__ Maps mp, const AttnPrefillArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem;
  unsigned char* sK = smem + kTile;      // kKStages stages
  unsigned char* sV = smem + (1 + kKStages) * kTile;  // kVStages stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTiles * kTile);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                 // [kKStages]
  uint64_t* k_empty = k_full + kKStages;       // [kKStages]
  uint64_t* v_full = k_empty + kKStages;       // [kVStages]
  uint64_t* v_empty = v_full + kVStages;       // [kVStages]
  uint64_t* s_full = v_empty + kVStages;       // [kSBufs]
  uint64_t* p_full = s_full + kSBufs;          // [kSBufs]
  uint64_t* pv_done = p_full + kSBufs;         // [kSBufs]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + kSBufs);
  // softmax exchange: block maxima [block parity][half][row], final sums [half][row]
  float (*xm)[2][BQ] = reinterpret_cast<float (*)[2][BQ]>(smem + kTiles * kTile + kBarBytes);
  float (*xl)[BQ] =
      reinterpret_cast<float (*)[BQ]>(smem + kTiles * kTile + kBarBytes + 4 * BQ * 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.S;
  const int nqb = (S + BQ - 1) / BQ;
  // heaviest work first: block index -> (query block from the end, head)
  const int qb = nqb - 1 - (int)blockIdx.x / a.Hq;
  const int h = (int)blockIdx.x % a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const int q0 = qb * BQ;
  const int nkb = qb + 1;  // key blocks up to the diagonal

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
      mbar_init(&pv_done[i], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = *tmem_slot;
  auto tS = [tmem](int b) { return tmem + (uint32_t)(b * 128); };  // S_j / P_j: buffer j % 3
  const uint32_t tO = tmem + 384;

  if (warp == 0) {
    // Q once, then K_j into stage j % kKStages once S_{j - kKStages} has read that stage
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kTile);
      tma_load_2d(sQ, &mp.q, h * D, q0, q_full);
      tma_load_2d(sQ + kAtom, &mp.q, h * D + 64, q0, q_full);
      for (int j = 0; j < nkb; ++j) {
        const int st = j % kKStages;
        if (j >= kKStages) mbar_wait(&k_empty[st], (j / kKStages - 1) & 1);
        unsigned char* kt = sK + st * kTile;
        mbar_arrive_expect_tx(&k_full[st], kTile);
        tma_load_3d(kt, &mp.kv[0], 0, j * BKV, g, &k_full[st]);
        tma_load_3d(kt + kAtom, &mp.kv[0], 64, j * BKV, g, &k_full[st]);
      }
    }
  } else if (warp == kVWarp) {
    // V_j into stage j % kVStages once PV_{j - kVStages} has read that stage
    if (lane == 0) {
      for (int j = 0; j < nkb; ++j) {
        const int st = j % kVStages;
        if (j >= kVStages) mbar_wait(&v_empty[st], (j / kVStages - 1) & 1);
        unsigned char* vt = sV + st * kTile;
        mbar_arrive_expect_tx(&v_full[st], kTile);
        tma_load_3d(vt, &mp.kv[1], 0, j * BKV, g, &v_full[st]);
        tma_load_3d(vt + kAtom, &mp.kv[1], 64, j * BKV, g, &v_full[st]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      mbar_wait(q_full, 0);
      const uint32_t qa = smem_u32(sQ);
      // S_j into buffer j % 3: 8 K-steps of 16 (32 bytes inside a 128-byte row, atom per 64);
      // the K stage is released when these MMAs complete
      auto issue_s = [&](int j) {
        const int st = j % kKStages;
        mbar_wait(&k_full[st], (j / kKStages) & 1);
        tc_after();
        const uint32_t kb = smem_u32(sK + st * kTile);
        const uint32_t d = tS(j % kSBufs);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (uint32_t)(k >> 2) * kAtom + (uint32_t)(k & 3) * 32;
          mma_ss(d, desc_k_sw128(qa + off), desc_k_sw128(kb + off), kIdescS, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j % kSBufs]);
        mma_commit(&k_empty[st]);
      };
      issue_s(0);
      if (nkb > 1) issue_s(1);
      for (int j = 0; j < nkb; ++j) {
        const int bj = j % kSBufs, vs = j % kVStages;
        mbar_wait(&p_full[bj], (j / kSBufs) & 1);
        mbar_wait(&v_full[vs], (j / kVStages) & 1);
        tc_after();
        const uint32_t vb = smem_u32(sV + vs * kTile);
        // O += P_j V_j: K = keys, 16 per step (8 TMEM columns of fp16 pairs; 2 x 8 rows of V)
#pragma unroll
        for (int k = 0; k < BKV / 16; ++k)
          mma_ts(tO, tS(bj) + (uint32_t)(k * 8), desc_mn_sw128(vb + (uint32_t)k * 2048), kIdescPV,
                 (j > 0 || k > 0) ? 1u : 0u);
        mma_commit(&v_empty[vs]);
        mma_commit(&pv_done[bj]);
        if (j + 2 < nkb) {
          // S_{j+2} goes into the buffer of P_{j-1}: queued right behind PV_j once PV_{j-1}
          // has read it
          if (j >= 1) {
            mbar_wait(&pv_done[(j - 1) % kSBufs], ((j - 1) / kSBufs) & 1);
            tc_after();
          }
          issue_s(j + 2);
        }
      }
    }
    __syncwarp();
  } else {
    // softmax / epilogue: two threads per query row.  TMEM lane quarter = warp % 4 (row = query
    // q0 + quarter * 32 + lane); half = which 64 keys of a block (and which 64 columns of O) the
    // thread takes.  The halves of a row exchange block maxima (and at the end their sums)
    // through shared memory behind a named barrier of the quarter's two warps.
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t col = (uint32_t)(half * 64);
    const float c = a.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    for (int j = 0; j < nkb; ++j) {
      const int bj = j % kSBufs, xs = j & 1;
      mbar_wait(&s_full[bj], (j / kSBufs) & 1);
      tc_after();
      uint32_t sr[2][32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) tmem_ld32(tS(bj) + lane_off + col + (uint32_t)(cc * 32), sr[cc]);
      tmem_wait_ld();
      const int k0 = j * BKV + half * 64;
      float mb = -INFINITY;  // maximum of the raw scores (the scale c is positive)
      if (j == nkb - 1) {    // diagonal block: keys after the query are masked
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            if (k0 + cc * 32 + t > qi) sr[cc][t] = __float_as_uint(-INFINITY);
            mb = fmaxf(mb, __uint_as_float(sr[cc][t]));
          }
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
          for (int t = 0; t < 32; ++t) mb = fmaxf(mb, __uint_as_float(sr[cc][t]));
        }
      }
      mb *= c;  // into the log2 domain
      // row maximum of the block: both halves' S loads are complete before either writes P
      // over the S buffer (half 1's P columns hold half 0's S keys 32..63)
      xm[xs][half][r] = mb;
      tc_before();
      pair_sync(quarter);
      tc_after();
      mb = fmaxf(mb, xm[xs][half ^ 1][r]);
      // lazy rescale: move the reference maximum only when this block's exceeds it by > 2^8
      const bool move = mb > m_used + kRescale;
      const float m_new = move ? mb : m_used;
      const float corr = move ? exp2f(m_used - m_new) : 1.f;  // 0 on the first block
      if (j > 0 && __any_sync(0xffffffffu, move)) {
        // O holds sum over blocks < j: wait until PV_{j-1} has written it, then rescale this
        // thread's 64 columns
        mbar_wait(&pv_done[(j - 1) % kSBufs], ((j - 1) / kSBufs) & 1);
        tc_after();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + col + (uint32_t)(cc * 32), o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * corr);
          tmem_st32(tO + lane_off + col + (uint32_t)(cc * 32), o);
        }
      }
      l *= corr;
      m_used = m_new;
      // P_j = 2^(s - m_used) as fp16 pairs: keys 64 half .. 64 half + 63 into columns
      // 32 half .. 32 half + 31 of the S buffer
      uint32_t pp[32];
      float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
        for (int t = 0; t < 32; t += 2) {
          const float e0 = ex2_approx(fmaf(__uint_as_float(sr[cc][t]), c, -m_used));
          const float e1 = ex2_approx(fmaf(__uint_as_float(sr[cc][t + 1]), c, -m_used));
          ls0 += e0;
          ls1 += e1;
          pp[cc * 16 + (t >> 1)] = pack_h2(e0, e1);
        }
      }
      const float ls = ls0 + ls1;
      l += ls;
      tmem_st32(tS(bj) + lane_off + (uint32_t)(half * 32), pp);
      tmem_wait_st();
      tc_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[bj]);
    }
    // epilogue: O / (l of both halves) -> fp16, this thread's 64 columns
    xl[half][r] = l;
    pair_sync(quarter);
    l += xl[half ^ 1][r];
    mbar_wait(&pv_done[(nkb - 1) % kSBufs], ((nkb - 1) / kSBufs) & 1);
    tc_after();
    const float il = l > 0.f ? 1.f / l : 0.f;
    __half* out = reinterpret_cast<__half*>(a.out) + (size_t)qi * a.Hq * D + (size_t)h * D + col;
#pragma unroll
    for (int cc = 0; cc < 2; ++cc) {
      uint32_t o[32];
      tmem_ld32(tO + lane_off + col + (uint32_t)(cc * 32), o);
      tmem_wait_ld();
      if (qi < S) {
#pragma unroll
        for (int t = 0; t < 32; t += 8) {
          uint4 v;
          v.x = pack_h2(__uint_as_float(o[t + 0]) * il, __uint_as_float(o[t + 1]) * il);
          v.y = pack_h2(__uint_as_float(o[t + 2]) * il, __uint_as_float(o[t + 3]) * il);
          v.z = pack_h2(__uint_as_float(o[t + 4]) * il, __uint_as_float(o[t + 5]) * il);
          v.w = pack_h2(__uint_as_float(o[t + 6]) * il, __uint_as_float(o[t + 7]) * il);
          *reinterpret_cast<uint4*>(out + cc * 32 + t) = v;
        }
      }
    }
  }
  tc_before();
  __syncthreads();
  if (warp == 1) {
    tc_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

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

constexpr size_t kSmem = kTiles * kTile + kBarBytes + 6 * BQ * 4 + 1024;

}  // namespace

cudaError_t launch_attn_prefill(const AttnPrefillArgs& a, cudaStream_t s) {
  auto fn = encode_fn();
  if (!fn || a.S < 1 || a.Hq % a.Hkv != 0) return cudaErrorInvalidValue;
  Maps mp;
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.Hq * D, (cuuint64_t)a.S};
    cuuint64_t strides[1] = {(cuuint64_t)a.Hq * D * 2};
    cuuint32_t box[2] = {64, BQ};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&mp.q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(a.q), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  for (int t = 0; t < 2; ++t) {
    // rows past S read as zeros (the cache may hold anything there)
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.S, (cuuint64_t)a.Hkv};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)a.cap * D * 2};
    cuuint32_t box[3] = {64, BKV, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const uint16_t* base = t == 0 ? a.k_cache : a.v_cache;
    if (fn(&mp.kv[t], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(base), dims,
           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  if (e != cudaSuccess) return e;
  const int nqb = (a.S + BQ - 1) / BQ;
  attn_prefill_tc_kernel<<<nqb * a.Hq, kThreads, kSmem, s>>>(mp, a);
  return cudaGetLastError();
}

}  // namespace vv
