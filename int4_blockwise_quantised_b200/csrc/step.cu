// Persistent decode-step kernel: the whole decoder_step (all layers + lm_head) in one
// cooperative launch ("vibevoice-asr-bitnet-onnx": decoder_step contract; "VibeVoice-ASR — ONNX
// export for Vernacula", section "Highlights": the step's ~1950 launches are the overhead to
// remove).
//
// One CTA per SM.  Warp 0..NW-1 compute, warp NW is the producer.
//
// The producer walks a static per-CTA schedule of everything the step streams from HBM -- for each
// layer: its rows of [Wq;Wk;Wv], its K/V tiles, its rows of Wo, of Wgate+Wup, of Wdown; then its
// rows of the lm_head -- and moves it with cp.async.bulk into a ring of shared-memory stages.
// Weights and past K/V do not depend on the step's activations, so the producer never waits for
// them: HBM keeps streaming across phase boundaries, limited only by the ring's depth.
//
// Compute warps walk the same schedule.  Before each phase they pass a grid-wide barrier (the
// phase's input is an activation vector produced by every CTA), stage that vector in shared
// memory / registers (with the fused RMSNorm where the layer has one), then consume the phase's
// stages.  Phases per layer:
//   QKV  : y = [Wq;Wk;Wv] . RMSNorm(x) + b              -> qkv (fp32); the CTA's q/k/v rows
//          form one stream of stages even where they straddle two matrices
//   ATTN : per (kv head, 64-position tile): RoPE(q), RoPE(k_new) + append at slot `length`,
//          online-softmax partial (m, l, o); up to 32 tiles per head the O staging of every CTA
//          merges the partials, beyond that the last CTA of a head merges them -> attn (fp32)
//   O    : x += Wo . attn
//   GU   : h = silu(Wg . RMSNorm(x)) * (Wu . RMSNorm(x))
//   DOWN : x += Wd . h
// then HEAD: logits = W_lm . RMSNorm(x), argmax (last CTA reduces), length += 1.
// GEMV stages run in one of three modes: x in registers (K <= 1536), whole rows per warp with x
// in shared memory (larger K, many rows), or each row split over three warps (larger K, few
// rows).  In greedy generation (StepParams::gen_done set) a launch after a stop token returns
// at once, and the last CTA advances the generation's position and token count.
//
// The grid barrier is a monotonic arrival counter in global memory (barrier k completes at
// (k + 1) x grid arrivals; the last CTA of the launch resets it); every wait is bounded
// (VV_ERR_TIMEOUT in the device error word after 2 s, then the kernel carries on).  The
// cooperative launch guarantees that all CTAs are resident.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "step.h"

namespace vv {
namespace {

constexpr int NW = 15;                 // compute warps (+1 producer: 512 threads, 4-warp register granules)
constexpr int kThreads = (NW + 1) * 32;
constexpr int D = 128;
constexpr int TT = 64;                 // attention tile (positions)
constexpr int kRowH = D + 8;           // halves per K/V row in a stage: 272 bytes, so consecutive
                                       // rows start 4 banks apart (conflict-free 16-byte reads)
constexpr int kMaxG = 8;
constexpr int kPart = 132;             // floats per (tile, head) partial: m, l, -, -, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kRegHB = 3;              // half-blocks per lane held in registers (K <= 1536)
constexpr int kMergeInO = 32;          // up to this many tiles per head, every CTA merges the
                                       // attention partials while staging the o-projection input

enum Phase { PH_QKV = 0, PH_ATTN, PH_O, PH_GU, PH_DOWN, PH_HEAD };

__device__ __forceinline__ void cbar() {  // compute warps only
  asm volatile("bar.sync 1, %0;" ::"n"(NW * 32) : "memory");
}

__device__ __forceinline__ void cta_range(int n, int cta, int ncta, int& r0, int& r1) {
  r0 = (int)((int64_t)n * cta / ncta);
  r1 = (int)((int64_t)n * (cta + 1) / ncta);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_u32(unsigned* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Timeline tap: thread 0 of each CTA records %globaltimer at fixed points of the schedule
// (barrier arrival, barrier exit, x staged, end) when p.stamps is set.
__device__ __forceinline__ void stamp(const StepParams& p, int& k) {
  if (p.stamps && threadIdx.x == 0) {
    if (k < p.max_stamps) p.stamps[(size_t)blockIdx.x * p.max_stamps + k] = globaltimer_ns();
    ++k;
  }
}

// Grid-wide barrier among the compute warps of all CTAs.  The arrival counter only grows during
// a launch (barrier k completes when it reaches (k + 1) * gridDim.x) and the last CTA of the
// lm_head phase resets it, so an arrival is one fire-and-forget release-add and the wait one
// acquire poll.  Bounded wait.
__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ void grid_barrier(const StepParams& p, unsigned& nbar, int& sk) {
  cbar();
  stamp(p, sk);
  if (threadIdx.x == 0) {
    const unsigned target = (nbar + 1) * gridDim.x;
    red_release_add(p.bar_count, 1u);
    if (ld_acquire_u32(p.bar_count) < target) {
      const uint64_t t0 = globaltimer_ns();
      while (ld_acquire_u32(p.bar_count) < target) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          set_device_error(VV_ERR_TIMEOUT);
          break;
        }
      }
    }
  }
  ++nbar;
  stamp(p, sk);
  cbar();
}

// --------------------------------------------------------------------------------- schedule
// Rows per stage of a packed matrix with K columns (codes + scales per row), nseg matrices per
// stage (gate/up share a stage).
__device__ __forceinline__ int packed_row_bytes(int K) { return (K >> 5) * 18; }
__device__ __forceinline__ int rows_per_stage(int row_bytes, int nseg, int stage_bytes) {
  int r = stage_bytes / (row_bytes * nseg);
  return r > 64 ? 64 : r;
}

// Rows per stage of a phase: bounded by the stage size, and for the split-K (large K, few rows)
// path by kSplitRows so that kSplitRows x kSplitW = NW warps share a stage.  `rows` is the
// CTA's row count for the phase: with x in shared memory and at least 2 NW units, warps take
// whole rows instead (row mode) and stages are filled.  Producer and consumers compute the same.
constexpr int kSplitW = 3;                // warps per row when K is large
constexpr int kSplitRows = NW / kSplitW;  // 5 rows per stage
__device__ __forceinline__ bool row_mode(int K, int nseg, int rows) {
  return K > 32 * kRegHB * 16 && rows * nseg >= 2 * NW;
}
__device__ __forceinline__ int phase_rps(int K, int nseg, int stage_bytes, int rows) {
  const int r = rows_per_stage((K >> 5) * 18, nseg, stage_bytes);
  return (K > 32 * kRegHB * 16 && !row_mode(K, nseg, rows)) ? min(r, kSplitRows) : r;
}

struct Ring {
  uint64_t wait_ns;  // time this thread spent blocked in ring waits (timeline tap)
  unsigned char* base;
  uint64_t* full;
  uint64_t* empty;
  int stage_bytes;
  int nstages;
  int idx;  // running stage counter
  int ph;          // phase kind of the stages being consumed (timeline tap)
  uint64_t* tapw;  // timeline tap: per-phase-kind ring wait of compute thread 0 (else null)
  __device__ unsigned char* slot_ptr(int i) const { return base + (size_t)(i % nstages) * stage_bytes; }
};

// Producer side of one stage: wait for the slot, post the byte count, issue the copies.
struct Copy {
  const void* src;
  uint32_t bytes;
  uint32_t dst_off;
};

// Ring wait with wait-time accounting.
__device__ __forceinline__ void ring_wait(Ring& r, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  mbar_wait(bar, parity);
  const uint64_t dt = globaltimer_ns() - t0;
  r.wait_ns += dt;
  if (r.tapw) r.tapw[r.ph] += dt;
}

// The producer's wait for a free slot: it runs stages ahead of the consumers, so it sleeps
// between polls instead of spinning through the issue slots its SM sub-partition shares with
// compute warps.  Bounded like every wait (kWaitLimitNs).
__device__ __forceinline__ void producer_wait(Ring& r, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  for (unsigned it = 1;; ++it) {
    __nanosleep(256);
    if (mbar_try_wait(bar, parity)) break;
    if ((it & 63) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
      set_device_error(VV_ERR_TIMEOUT);
      break;
    }
  }
  r.wait_ns += globaltimer_ns() - t0;
}

__device__ __forceinline__ void produce(Ring& r, const Copy* c, int n, uint64_t pol) {
  const int s = r.idx++;
  const int slot = s % r.nstages;
  if (s >= r.nstages) producer_wait(r, &r.empty[slot], ((s / r.nstages) - 1) & 1);
  uint32_t tot = 0;
  for (int i = 0; i < n; ++i) tot += c[i].bytes;
  mbar_arrive_expect_tx(&r.full[slot], tot);
  unsigned char* dst = r.base + (size_t)slot * r.stage_bytes;
  for (int i = 0; i < n; ++i)
    if (c[i].bytes) bulk_g2s_stream(dst + c[i].dst_off, c[i].src, c[i].bytes, &r.full[slot], pol);
}

// One attention tile: `rows` past K rows and V rows (256 bytes each) into the padded row layout
// (kRowH halves per row; V after TT K rows).
__device__ void produce_kv_rows(Ring& r, const __half* k, const __half* v, int rows, uint64_t pol) {
  const int s = r.idx++;
  const int slot = s % r.nstages;
  if (s >= r.nstages) producer_wait(r, &r.empty[slot], ((s / r.nstages) - 1) & 1);
  mbar_arrive_expect_tx(&r.full[slot], (uint32_t)rows * D * 2 * 2);
  unsigned char* dst = r.base + (size_t)slot * r.stage_bytes;
  for (int i = 0; i < rows; ++i) {
    bulk_g2s_stream(dst + (size_t)i * kRowH * 2, k + (size_t)i * D, D * 2, &r.full[slot], pol);
    bulk_g2s_stream(dst + (size_t)(TT + i) * kRowH * 2, v + (size_t)i * D, D * 2, &r.full[slot], pol);
  }
}

// Stream rows [r0, r1) of a packed matrix (and optionally the same rows of a second one).
__device__ void produce_packed(Ring& r, const uint8_t* q0, const __half* s0, const uint8_t* q1,
                               const __half* s1, int K, int r0, int r1, uint64_t pol) {
  const int nseg = q1 ? 2 : 1;
  const int rq = (K >> 5) * 16, rs = (K >> 5) * 2;
  const int rps = phase_rps(K, nseg, r.stage_bytes, r1 - r0);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    Copy c[4];
    int k = 0;
    // layout: [seg0 codes (rps rows)][seg1 codes][seg0 scales][seg1 scales]
    c[k++] = Copy{q0 + (size_t)a * rq, (uint32_t)(n * rq), 0u};
    if (q1) c[k++] = Copy{q1 + (size_t)a * rq, (uint32_t)(n * rq), (uint32_t)(rps * rq)};
    c[k++] = Copy{reinterpret_cast<const unsigned char*>(s0) + (size_t)a * rs, (uint32_t)(n * rs),
                  (uint32_t)(nseg * rps * rq)};
    if (q1)
      c[k++] = Copy{reinterpret_cast<const unsigned char*>(s1) + (size_t)a * rs,
                    (uint32_t)(n * rs), (uint32_t)(nseg * rps * rq + rps * rs)};
    produce(r, c, k, pol);
  }
}

// Stream logical rows [r0, r1) of [Wq; Wk; Wv] (bounds: first row of each matrix); a stage may
// hold rows of two matrices, laid out as one matrix of consecutive rows.
__device__ void produce_qkv(Ring& r, const StepLayer& w, int K, int r0, int r1,
                            const int (&bounds)[4], uint64_t pol) {
  const int rq = (K >> 5) * 16, rs = (K >> 5) * 2;
  const int rps = phase_rps(K, 1, r.stage_bytes, r1 - r0);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    Copy c[6];
    int k = 0;
    for (int m = 0; m < 3; ++m) {
      const int lo = max(a, bounds[m]), hi = min(a + n, bounds[m + 1]);
      if (lo >= hi) continue;
      c[k++] = Copy{w.q[m] + (size_t)(lo - bounds[m]) * rq, (uint32_t)((hi - lo) * rq),
                    (uint32_t)((lo - a) * rq)};
      c[k++] = Copy{reinterpret_cast<const unsigned char*>(w.s[m]) + (size_t)(lo - bounds[m]) * rs,
                    (uint32_t)((hi - lo) * rs), (uint32_t)(rps * rq + (lo - a) * rs)};
    }
    produce(r, c, k, pol);
  }
}

// Tiles (kv head g, tile t) owned by this CTA: items i = cta + k * ncta < Hkv * ntiles.
__device__ __forceinline__ int ntiles_for(int past) { return (past + 1 + TT - 1) / TT; }

__device__ void producer(const StepParams& p, Ring& r, int past) {
  const uint64_t pol = policy_evict_first();
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int H = p.H, Hq = p.Hq, Hkv = p.Hkv, I = p.I;
  const int nqkv = (Hq + 2 * Hkv) * D;
  const int nt = ntiles_for(past);
  for (int l = 0; l < p.L; ++l) {
    const StepLayer& w = p.layers[l];
    // QKV: logical rows [0, nqkv) over the three matrices
    int r0, r1;
    cta_range(nqkv, cta, ncta, r0, r1);
    const int bounds[4] = {0, Hq * D, (Hq + Hkv) * D, nqkv};
    produce_qkv(r, w, H, r0, r1, bounds, pol);
    // ATTN: past K/V rows of the tiles
    for (int it = cta; it < Hkv * nt; it += ncta) {
      const int g = it / nt, t = it % nt;
      const int p0 = t * TT, p1 = min(p0 + TT, past);
      const size_t off = ((size_t)(l * Hkv + g) * p.cap + p0) * D;
      produce_kv_rows(r, p.k_cache + off, p.v_cache + off, max(p1 - p0, 0), pol);
    }
    cta_range(H, cta, ncta, r0, r1);
    produce_packed(r, w.q[3], w.s[3], nullptr, nullptr, Hq * D, r0, r1, pol);
    cta_range(I, cta, ncta, r0, r1);
    produce_packed(r, w.q[4], w.s[4], w.q[5], w.s[5], H, r0, r1, pol);
    cta_range(H, cta, ncta, r0, r1);
    produce_packed(r, w.q[6], w.s[6], nullptr, nullptr, I, r0, r1, pol);
  }
  // HEAD: fp16 rows of the lm_head
  int r0, r1;
  cta_range(p.V, cta, ncta, r0, r1);
  const int rb = H * 2;
  const int rps = min(64, r.stage_bytes / rb);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    Copy c[1] = {Copy{p.lm_head + (size_t)a * H, (uint32_t)(n * rb), 0u}};
    produce(r, c, 1, pol);
  }
}

// ------------------------------------------------------------------------ compute helpers
// x staging.  Source fp32 (or fp16 embedding row), optional RMSNorm with fp16 gamma; the result
// is rounded once to fp16 (the GEMV's activation type) and stored in the half2-pair layout of the
// dequant-dot: element k (hb = k/16, word = (k/8)%2, j = k%8) goes to uint4 (word * NHB + hb),
// component j%4, half j/4, i.e. the pairs (x0,x4) (x1,x5) (x2,x6) (x3,x7) of each word.  A warp
// reading half-blocks hb = lane + 32i touches consecutive 16-byte chunks (no bank conflicts).
// All compute threads; ends with a compute barrier.
__device__ __forceinline__ int xh_slot(int k, int nhb) {
  const int hb = k >> 4, word = (k >> 3) & 1, j = k & 7;
  return ((word * nhb + hb) * 4 + (j & 3)) * 2 + (j >> 2);
}

__device__ void stage_x(__half* xs, float* red, const float* src32, const __half* src16,
                        const __half* gamma, float eps, int K, float* copy_out) {
  const int tid = threadIdx.x;
  constexpr int NT = NW * 32;
  constexpr int kReg = 5;  // float4 chunks per thread kept in registers (K <= 4 * 5 * NT = 9600)
  const int nhb = K >> 4;
  auto load4 = [&](int k) -> float4 {
    if (src32) return __ldcg(reinterpret_cast<const float4*>(src32 + k));
    const uint2 hv = __ldcg(reinterpret_cast<const uint2*>(src16 + k));
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
    return make_float4(a.x, a.y, b.x, b.y);
  };
  auto put = [&](int k, float4 t, float inv) {
    float y[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float u = y[e];
      if (gamma) u = u * inv * __half2float(gamma[k + e]);
      xs[xh_slot(k + e, nhb)] = __float2half_rn(u);
    }
  };
  auto norm_inv = [&](float ss) {
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    cbar();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < NW; ++i) tot += red[i];
    return rsqrtf(tot / (float)K + eps);
  };
  if (K > kReg * 4 * NT) {  // large K (7B down projection): two passes over the source
    float ss = 0.f;
    for (int k = tid * 4; k < K; k += NT * 4) {
      const float4 t = load4(k);
      if (copy_out) *reinterpret_cast<float4*>(copy_out + k) = t;
      ss += t.x * t.x + t.y * t.y + t.z * t.z + t.w * t.w;
    }
    const float inv = gamma ? norm_inv(ss) : 1.f;
    for (int k = tid * 4; k < K; k += NT * 4) put(k, load4(k), inv);
    cbar();
    return;
  }
  float4 v[kReg];
  uint2 gv[kReg];  // gamma halves, loaded with x so their latency overlaps
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kReg; ++i) {
    const int k = (tid + i * NT) * 4;
    if (k < K) {
      if (gamma) gv[i] = *reinterpret_cast<const uint2*>(gamma + k);
      v[i] = load4(k);
      if (copy_out) *reinterpret_cast<float4*>(copy_out + k) = v[i];
      ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    } else {
      v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const float inv = gamma ? norm_inv(ss) : 1.f;
#pragma unroll
  for (int i = 0; i < kReg; ++i) {
    const int k = (tid + i * NT) * 4;
    if (k < K) {
      float y[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      if (gamma) {
        const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&gv[i].x));
        const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&gv[i].y));
        y[0] *= inv * g01.x;
        y[1] *= inv * g01.y;
        y[2] *= inv * g23.x;
        y[3] *= inv * g23.y;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) xs[xh_slot(k + e, nhb)] = __float2half_rn(y[e]);
    }
  }
  cbar();
}

// Dot of one half-block (8 bytes of codes = 16 columns) with its two x words (half2 pairs).
__device__ __forceinline__ float hb_doth(uint2 wv, uint4 xa, uint4 xb) {
  return dot8_h(wv.x, xa) + dot8_h(wv.y, xb);
}

// One stage with x in shared memory and whole rows per warp (large K, rows plentiful): warp w
// takes units [w R, w R + R), lanes stride the half-blocks, one shuffle reduction per unit; no
// cross-warp reduction, so no barrier inside the stage.
template <int R, class RowQ, class RowS, class Fin>
__device__ __forceinline__ void smemx_pass(RowQ rowq, RowS rows, const uint4* xs4, int K, int units,
                                           int nseg, int a, Fin fin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NHB = K >> 4;
  for (int u0 = warp * R; u0 < units; u0 += NW * R) {
    const unsigned char* wq[R];
    const __half* ws[R];
    int lr[R];
    bool ok[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int u = u0 + k;
      ok[k] = u < units;
      const int uu = ok[k] ? u : u0;
      const int sg = nseg == 2 ? (uu & 1) : 0;
      lr[k] = nseg == 2 ? (uu >> 1) : uu;
      wq[k] = rowq(sg, lr[k]);
      ws[k] = rows(sg, lr[k]);
    }
    float acc[R];
#pragma unroll
    for (int k = 0; k < R; ++k) acc[k] = 0.f;
#pragma unroll 2
    for (int hb = lane; hb < NHB; hb += 32) {
      const uint4 xa = xs4[hb], xb = xs4[NHB + hb];
#pragma unroll
      for (int k = 0; k < R; ++k) {
        const uint2 wv = *reinterpret_cast<const uint2*>(wq[k] + hb * 8);
        acc[k] = fmaf(__half2float(ws[k][hb >> 1]), hb_doth(wv, xa, xb), acc[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) acc[k] = warp_sum(acc[k]);
    if (lane == 0) {
      if (nseg == 2) {
#pragma unroll
        for (int k = 0; k + 1 < R; k += 2)
          if (ok[k]) fin(a + lr[k], acc[k], acc[k + 1]);
      } else {
#pragma unroll
        for (int k = 0; k < R; ++k)
          if (ok[k]) fin(a + lr[k], acc[k], 0.f);
      }
    }
  }
}

// One stage of the register-x path: warp w takes units [w R, w R + R), then [w R + NW R, ...);
// unit u is (segment, row) = (u & 1, u >> 1) for gate/up pairs, else (0, u).  Lanes stride the
// half-blocks; one shuffle reduction per unit; lane 0 finishes the rows.
template <int R, class RowQ, class RowS, class Fin>
__device__ __forceinline__ void regx_pass(RowQ rowq, RowS rows, const uint4 (&xr)[kRegHB][2], int K,
                                          int units, int nseg, int a, Fin fin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NHB = K >> 4;
  for (int u0 = warp * R; u0 < units; u0 += NW * R) {
    int sg[R], lr[R];
    bool ok[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int u = u0 + k;
      ok[k] = u < units;
      const int uu = ok[k] ? u : u0;
      sg[k] = nseg == 2 ? (uu & 1) : 0;
      lr[k] = nseg == 2 ? (uu >> 1) : uu;
    }
    float acc[R];
#pragma unroll
    for (int k = 0; k < R; ++k) acc[k] = 0.f;
#pragma unroll
    for (int j = 0; j < kRegHB; ++j) {
      const int hb = lane + 32 * j;
      if (hb < NHB) {
#pragma unroll
        for (int k = 0; k < R; ++k) {
          const uint2 wv = *reinterpret_cast<const uint2*>(rowq(sg[k], lr[k]) + hb * 8);
          const float sc = __half2float(rows(sg[k], lr[k])[hb >> 1]);
          acc[k] = fmaf(sc, hb_doth(wv, xr[j][0], xr[j][1]), acc[k]);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k) acc[k] = warp_sum(acc[k]);
    if (lane == 0) {
      if (nseg == 2) {
#pragma unroll
        for (int k = 0; k + 1 < R; k += 2)
          if (ok[k]) fin(a + lr[k], acc[k], acc[k + 1]);
      } else {
#pragma unroll
        for (int k = 0; k < R; ++k)
          if (ok[k]) fin(a + lr[k], acc[k], 0.f);
      }
    }
  }
}

// Consume the stages of a packed-matrix phase.  fin(row, y0, y1) is called once per output row
// (y1: the up value of a gate/up pair, nseg = 2).
//  * K <= 1536 (x in registers xr): each warp takes 4 rows per pass (or 2 gate/up pairs) for
//    instruction-level parallelism; lanes stride the half-blocks; shuffle reduction.
//  * larger K (x in shared memory, interleaved): each row is split over kSplitW warps, partial
//    sums meet in shared memory (red2) and the first warp of the row finishes it.
template <class Fin>
__device__ __forceinline__ void consume_packed(Ring& r, const __half* xs, const uint4 (&xr)[kRegHB][2],
                                               bool regx, int K, int r0, int r1, int nseg,
                                               float* red2, Fin fin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = K >> 5, NHB = K >> 4;
  const int rq = KB * 16, rs = KB * 2;
  const int rps = phase_rps(K, nseg, r.stage_bytes, r1 - r0);
  const bool rowmode = row_mode(K, nseg, r1 - r0);
  const uint4* xs4 = reinterpret_cast<const uint4*>(xs);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    const int s = r.idx++;
    const int slot = s % r.nstages;
    ring_wait(r, &r.full[slot], (s / r.nstages) & 1);
    const unsigned char* st = r.base + (size_t)slot * r.stage_bytes;
    const unsigned char* scb = st + (size_t)nseg * rps * rq;
    auto rowq = [&](int sg, int lr) { return st + (size_t)(sg * rps + lr) * rq; };
    auto rows = [&](int sg, int lr) {
      return reinterpret_cast<const __half*>(scb + (size_t)(sg * rps + lr) * rs);
    };
    if (regx) {
      // R row slots per warp pass: as many as keep every warp busy (R = 1 for the small
      // phases, up to 4 for instruction-level parallelism when rows are plentiful); gate/up
      // pairs stay inside one warp (R >= 2).
      const int units = n * nseg;
      if (nseg == 1 && units <= NW)
        regx_pass<1>(rowq, rows, xr, K, units, nseg, a, fin);
      else if (units <= 2 * NW)
        regx_pass<2>(rowq, rows, xr, K, units, nseg, a, fin);
      else
        regx_pass<4>(rowq, rows, xr, K, units, nseg, a, fin);
    } else if (rowmode) {
      smemx_pass<2>(rowq, rows, xs4, K, n * nseg, nseg, a, fin);
    } else {
      // split-K: warp w -> row w / kSplitW, slice w % kSplitW
      const int lrow = warp / kSplitW, slice = warp % kSplitW;
      float acc0 = 0.f, acc1 = 0.f;
      if (lrow < n) {
        const unsigned char* q0 = rowq(0, lrow);
        const __half* sc0 = rows(0, lrow);
        const unsigned char* q1 = rowq(nseg - 1, lrow);
        const __half* sc1 = rows(nseg - 1, lrow);
        for (int hb = lane + 32 * slice; hb < NHB; hb += 32 * kSplitW) {
          const uint4 xa = xs4[hb], xb = xs4[NHB + hb];
          const uint2 w0 = *reinterpret_cast<const uint2*>(q0 + hb * 8);
          acc0 = fmaf(__half2float(sc0[hb >> 1]), hb_doth(w0, xa, xb), acc0);
          if (nseg == 2) {
            const uint2 w1 = *reinterpret_cast<const uint2*>(q1 + hb * 8);
            acc1 = fmaf(__half2float(sc1[hb >> 1]), hb_doth(w1, xa, xb), acc1);
          }
        }
      }
      acc0 = warp_sum(acc0);
      acc1 = warp_sum(acc1);
      if (lane == 0) {
        red2[warp * 2 + 0] = acc0;
        red2[warp * 2 + 1] = acc1;
      }
      cbar();
      if (lane == 0 && slice == 0 && lrow < n) {
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int k = 0; k < kSplitW; ++k) {
          y0 += red2[(warp + k) * 2 + 0];
          y1 += red2[(warp + k) * 2 + 1];
        }
        fin(a + lrow, y0, y1);
      }
      cbar();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[slot]);
  }
}

// Preload the lane's half-blocks of x (fp16 pair layout in xs) into registers.
__device__ __forceinline__ void load_xr(const __half* xs, uint4 (&xr)[kRegHB][2], int K) {
  const int lane = threadIdx.x & 31;
  const int NHB = K >> 4;
  const uint4* xs4 = reinterpret_cast<const uint4*>(xs);
#pragma unroll
  for (int j = 0; j < kRegHB; ++j) {
    const int hb = lane + 32 * j;
    xr[j][0] = hb < NHB ? xs4[hb] : make_uint4(0u, 0u, 0u, 0u);
    xr[j][1] = hb < NHB ? xs4[NHB + hb] : make_uint4(0u, 0u, 0u, 0u);
  }
}

struct AttnScratch {
  float cs[D / 2], sn[D / 2];  // RoPE cos/sin at this step's position
  float q[kMaxG][D];
  float s[kMaxG][TT];
  float m[kMaxG], l[kMaxG];
  float mw[256][kMaxG];
  float pv[4][kMaxG][D];  // P.V partial sums per position quarter
  int is_last;
};

__device__ __forceinline__ bool merge_in_o(const StepParams& p, int nt) {
  return nt <= kMergeInO && p.Hkv * nt * (p.Hq / p.Hkv) <= 256 * kMaxG;
}

// Stage the o-projection input straight from the attention partials (merge_in_o case): per head
// M = max_t m_t, L = sum_t l_t 2^(m_t - M), o[h][d] = sum_t 2^(m_t - M) o_t[h][d] / L; rounded to
// fp16 into the GEMV layout.  Each thread merges its 4 dims online over batches of 6 tiles, the
// batch's m, l and o loads all in flight together.  Ends with a compute barrier.
__device__ void stage_attn_merged(const StepParams& p, __half* xs, int nt) {
  const int tid = threadIdx.x;
  const int G = p.Hq / p.Hkv, K = p.Hq * D, nhb = K >> 4;
  constexpr int kB = 6;
  for (int k4 = tid; k4 < K / 4; k4 += NW * 32) {
    const int k = k4 * 4;
    const int hh = k >> 7, d = k & (D - 1);
    const int g = hh / G, h = hh % G;
    const float* base = p.attn_part + ((size_t)g * p.max_tiles * kMaxG + h) * kPart;
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int t0 = 0; t0 < nt; t0 += kB) {
      float4 v[kB];
      float mt[kB], lt[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        if (t0 + u < nt) {
          const float* pt = base + (size_t)(t0 + u) * kMaxG * kPart;
          mt[u] = __ldcg(pt);
          lt[u] = __ldcg(pt + 1);
          v[u] = __ldcg(reinterpret_cast<const float4*>(pt + 4 + d));
        } else {
          mt[u] = -INFINITY;
          lt[u] = 0.f;
          v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float bm = M;
#pragma unroll
      for (int u = 0; u < kB; ++u) bm = fmaxf(bm, mt[u]);
      const float c = exp2f(M - bm);  // 0 on the first batch (M = -inf)
      L *= c;
      acc.x *= c;
      acc.y *= c;
      acc.z *= c;
      acc.w *= c;
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const float e = exp2f(mt[u] - bm);
        L = fmaf(lt[u], e, L);
        acc.x = fmaf(e, v[u].x, acc.x);
        acc.y = fmaf(e, v[u].y, acc.y);
        acc.z = fmaf(e, v[u].z, acc.z);
        acc.w = fmaf(e, v[u].w, acc.w);
      }
      M = bm;
    }
    const float inv = 1.f / L;
    xs[xh_slot(k + 0, nhb)] = __float2half_rn(acc.x * inv);
    xs[xh_slot(k + 1, nhb)] = __float2half_rn(acc.y * inv);
    xs[xh_slot(k + 2, nhb)] = __float2half_rn(acc.z * inv);
    xs[xh_slot(k + 3, nhb)] = __float2half_rn(acc.w * inv);
  }
  cbar();
}

__device__ void attn_item(const StepParams& p, Ring& r, AttnScratch& as, int l, int g, int t,
                          int past, int pos) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.Hq / p.Hkv;
  const int nt = ntiles_for(past);
  const int npos = past + 1;
  const int p0 = t * TT;
  const int n = min(TT, npos - p0);
  const float* qkv = p.qkv;
  // q of the group (rotated, scaled into the log2 domain) and, on the tile holding the new
  // position, the new k/v: every global load is issued before any is used (one L2 round trip).
  const float qscale = p.scale * kLog2e;
  const bool newpos = t == nt - 1;
  constexpr int kQPer = (kMaxG * D + NW * 32 - 1) / (NW * 32);  // q element pairs per thread
  float qa[kQPer], qb[kQPer];
#pragma unroll
  for (int j = 0; j < kQPer; ++j) {
    const int i = tid + j * NW * 32;
    qa[j] = qb[j] = 0.f;
    if (i < G * D) {
      const int h = i / D, d = i % D;
      const float* qh = qkv + (size_t)(g * G + h) * D;
      const int fi = d & (D / 2 - 1);
      qa[j] = __ldcg(qh + fi);
      qb[j] = __ldcg(qh + fi + D / 2);
    }
  }
  float ka = 0.f, kb = 0.f, vv = 0.f;
  if (newpos && tid < D) {
    const int d = tid, fi = d & (D / 2 - 1);
    const float* kh = qkv + (size_t)(p.Hq + g) * D;
    ka = __ldcg(kh + fi);
    kb = __ldcg(kh + fi + D / 2);
    vv = __ldcg(qkv + (size_t)(p.Hq + p.Hkv + g) * D + d);
  }
#pragma unroll
  for (int j = 0; j < kQPer; ++j) {
    const int i = tid + j * NW * 32;
    if (i < G * D) {
      const int h = i / D, d = i % D;
      const int fi = d & (D / 2 - 1);
      const float cs = as.cs[fi], sn = as.sn[fi];
      as.q[h][d] = (d < D / 2 ? qa[j] * cs - qb[j] * sn : qb[j] * cs + qa[j] * sn) * qscale;
    }
  }
  const int s = r.idx++;
  const int slot = s % r.nstages;
  ring_wait(r, &r.full[slot], (s / r.nstages) & 1);
  __half* kt = reinterpret_cast<__half*>(r.base + (size_t)slot * r.stage_bytes);
  __half* vt = kt + TT * kRowH;
  if (newpos && tid < D) {  // this tile holds the new position: rotate k, append k/v
    const int d = tid, fi = d & (D / 2 - 1);
    const float cs = as.cs[fi], sn = as.sn[fi];
    const __half kn = __float2half_rn(d < D / 2 ? ka * cs - kb * sn : kb * cs + ka * sn);
    const __half vn = __float2half_rn(vv);
    const size_t off = ((size_t)(l * p.Hkv + g) * p.cap + past) * D + d;
    p.k_cache[off] = kn;
    p.v_cache[off] = vn;
    kt[(past - p0) * kRowH + d] = kn;
    vt[(past - p0) * kRowH + d] = vn;
  }
  cbar();
  // scores: warp w -> head w/2, positions (w%2)*32 + lane.  All lanes walk the chunks in the same
  // order, so the q reads are broadcasts; the padded K rows keep the k reads conflict-free.
  for (int item = warp; item < 2 * G; item += NW) {
    const int h = item >> 1, pp = (item & 1) * 32 + lane;
    {
      float sc = -INFINITY;
      if (pp < n) {
        const __half* kr = kt + pp * kRowH;
        float2 acc = make_float2(0.f, 0.f), acc2 = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
          const int cc = c;
          const uint4 kv = *reinterpret_cast<const uint4*>(kr + cc * 8);
          const float4 qa = *reinterpret_cast<const float4*>(&as.q[h][cc * 8]);
          const float4 qb = *reinterpret_cast<const float4*>(&as.q[h][cc * 8 + 4]);
          acc = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&kv.x)), make_float2(qa.x, qa.y), acc);
          acc2 = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&kv.y)), make_float2(qa.z, qa.w), acc2);
          acc = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&kv.z)), make_float2(qb.x, qb.y), acc);
          acc2 = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&kv.w)), make_float2(qb.z, qb.w), acc2);
        }
        sc = (acc.x + acc.y) + (acc2.x + acc2.y);
      }
      as.s[h][pp] = sc;
    }
  }
  cbar();
  if (warp < G) {  // softmax statistics of this tile, per head
    const int h = warp;
    const float s0 = as.s[h][lane], s1 = as.s[h][lane + 32];
    const float mt = warp_max(fmaxf(s0, s1));
    const float e0 = lane < n ? exp2f(s0 - mt) : 0.f;
    const float e1 = lane + 32 < n ? exp2f(s1 - mt) : 0.f;
    as.s[h][lane] = e0;
    as.s[h][lane + 32] = e1;
    const float sum = warp_sum(e0 + e1);
    if (lane == 0) {
      as.m[h] = mt;
      as.l[h] = sum;
    }
  }
  cbar();
  // P.V: unit = (head h, 8-dim octet o, position quarter q); V rows read as 16-byte vectors (the
  // 16 octets of a row on consecutive lanes: conflict-free), quarters combined through shared
  // memory (as.pv), then written as the tile's partial.
  {
    const int units = G * 16 * 4;
    for (int u = tid; u < units; u += NW * 32) {
      const int o = u & 15, q = (u >> 4) & 3, h = u >> 6;
      float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
      const float* ph = as.s[h];
      const int p_end = min(n, q * 16 + 16);
      for (int pp = q * 16; pp < p_end; ++pp) {
        const uint4 v8 = *reinterpret_cast<const uint4*>(vt + pp * kRowH + o * 8);
        const float w = ph[pp];
        const float2 ww = make_float2(w, w);
        a0 = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&v8.x)), ww, a0);
        a1 = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&v8.y)), ww, a1);
        a2 = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&v8.z)), ww, a2);
        a3 = __ffma2_rn(__half22float2(*reinterpret_cast<const __half2*>(&v8.w)), ww, a3);
      }
      float4* dst = reinterpret_cast<float4*>(&as.pv[q][h][o * 8]);
      dst[0] = make_float4(a0.x, a0.y, a1.x, a1.y);
      dst[1] = make_float4(a2.x, a2.y, a3.x, a3.y);
    }
    cbar();
    float* part = p.attn_part + ((size_t)(g * p.max_tiles + t) * kMaxG) * kPart;
    for (int idx = tid; idx < G * D; idx += NW * 32) {
      const int h = idx >> 7, d = idx & (D - 1);
      part[h * kPart + 4 + d] = (as.pv[0][h][d] + as.pv[1][h][d]) + (as.pv[2][h][d] + as.pv[3][h][d]);
    }
    if (tid < G) {
      part[tid * kPart + 0] = as.m[tid];
      part[tid * kPart + 1] = as.l[tid];
    }
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(&r.empty[slot]);
  // Short caches: the partials are merged by every CTA when it stages the o-projection input
  // (after the grid barrier, which orders these stores).  Long caches: the last tile of head g to
  // finish merges g's partials here.
  if (merge_in_o(p, nt)) return;
  __threadfence();
  cbar();
  if (tid == 0) {
    const int prev = atomicAdd(&p.attn_count[g], 1);
    as.is_last = prev == nt - 1;
  }
  cbar();
  if (!as.is_last) return;
  __threadfence();
  const float* base = p.attn_part + (size_t)g * p.max_tiles * kMaxG * kPart;
  if (warp < G) {  // merge weights of head h: every m, l load in flight at once
    const int h = warp;
    constexpr int kPer = 256 / 32;  // nt <= max_tiles <= 256
    float mv[kPer], lv[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int c = lane + 32 * j;
      mv[j] = -INFINITY;
      lv[j] = 0.f;
      if (c < nt) {
        const float* pp = base + ((size_t)c * kMaxG + h) * kPart;
        mv[j] = __ldcg(pp);
        lv[j] = __ldcg(pp + 1);
      }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < kPer; ++j) mx = fmaxf(mx, mv[j]);
    mx = warp_max(mx);
    float L = 0.f;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      mv[j] = exp2f(mv[j] - mx);  // 0 for absent tiles
      L = fmaf(lv[j], mv[j], L);
    }
    L = warp_sum(L);
    const float inv = 1.f / L;
#pragma unroll
    for (int j = 0; j < kPer; ++j)
      if (lane + 32 * j < nt) as.mw[lane + 32 * j][h] = mv[j] * inv;
  }
  cbar();
  // o merge: (head, 4-dim column) x tile half -> partial sums in as.pv, then the halves add up
  const int cols = G * (D / 4);
  const int halves = (NW * 32) / cols >= 2 ? 2 : 1;
  const int tsplit = (nt + halves - 1) / halves;
  for (int idx = tid; idx < cols * halves; idx += NW * 32) {
    const int col = idx % cols, part = idx / cols;
    const int h = col / (D / 4), d4 = col % (D / 4);
    const int t0 = part * tsplit, t1 = min(nt, t0 + tsplit);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = t0; c0 < t1; c0 += 8) {
      const int m = min(8, t1 - c0);
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = u < m ? __ldcg(reinterpret_cast<const float4*>(base + ((size_t)(c0 + u) * kMaxG + h) * kPart + 4) + d4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (u < m) {
          const float w = as.mw[c0 + u][h];
          acc.x = fmaf(w, v[u].x, acc.x);
          acc.y = fmaf(w, v[u].y, acc.y);
          acc.z = fmaf(w, v[u].z, acc.z);
          acc.w = fmaf(w, v[u].w, acc.w);
        }
      }
    }
    *reinterpret_cast<float4*>(&as.pv[part][h][4 * d4]) = acc;
  }
  cbar();
  for (int idx = tid; idx < cols; idx += NW * 32) {
    const int h = idx / (D / 4), d4 = idx % (D / 4);
    float4 acc = *reinterpret_cast<const float4*>(&as.pv[0][h][4 * d4]);
    if (halves == 2) {
      const float4 b2 = *reinterpret_cast<const float4*>(&as.pv[1][h][4 * d4]);
      acc.x += b2.x;
      acc.y += b2.y;
      acc.z += b2.z;
      acc.w += b2.w;
    }
    *reinterpret_cast<float4*>(p.attn_out + (size_t)(g * G + h) * D + 4 * d4) = acc;
  }
  if (tid == 0) p.attn_count[g] = 0;
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__global__ void __launch_bounds__(kThreads, 1) step_kernel(const StepParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  Ring r;
  r.wait_ns = 0;
  r.ph = 0;
  // timeline tap: the last 8 stamps of a CTA's row hold thread 0's ring wait per phase kind
  // (QKV, ATTN, O, GU, DOWN, HEAD at max-8 .. max-3), then the producer's done time and its
  // blocked time.
  r.tapw = (p.stamps && threadIdx.x == 0) ? p.stamps + (size_t)blockIdx.x * p.max_stamps + p.max_stamps - 8
                                          : nullptr;
  r.base = smem;
  r.stage_bytes = p.stage_bytes;
  r.nstages = p.nstages;
  r.idx = 0;
  __half* xs = reinterpret_cast<__half*>(smem + (size_t)p.nstages * p.stage_bytes);
  AttnScratch& as = *reinterpret_cast<AttnScratch*>(smem + (size_t)p.nstages * p.stage_bytes +
                                                     (size_t)p.x_floats * 2);
  float* red = reinterpret_cast<float*>(&as + 1);  // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(red + 64) + 15) &
                                               ~uintptr_t(15));
  r.full = bars;
  r.empty = bars + p.nstages;
  __shared__ float s_val[NW];
  __shared__ int s_idx[NW];
  __shared__ int s_last;

  // generation stopped by an earlier step of the same vv_decoder_generate call: every CTA sees
  // the same word (written by the previous launch) and leaves before touching anything
  if (p.gen_done && __ldcg(p.gen_done) != 0) return;
  const int past = *p.length;
  if (tid == 0) {
    for (int i = 0; i < p.nstages; ++i) {
      mbar_init(&r.full[i], 1);
      mbar_init(&r.empty[i], NW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    if (lane == 0) {
      producer(p, r, past);
      if (p.stamps) {
        uint64_t* row = p.stamps + (size_t)blockIdx.x * p.max_stamps;
        row[p.max_stamps - 1] = r.wait_ns;          // producer blocked on free slots
        row[p.max_stamps - 2] = globaltimer_ns();   // producer done issuing
      }
    }
    return;
  }

  // ----------------------------------------------------------------------------- compute
  unsigned gen = 0;  // barriers passed in this launch
  int sk = 0;        // timeline stamp index
  stamp(p, sk);
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int H = p.H, Hq = p.Hq, Hkv = p.Hkv, I = p.I;
  const int nqkv = (Hq + 2 * Hkv) * D;
  const int nt = ntiles_for(past);
  int pos = *p.position;
  if (pos < 0 || pos >= p.max_position) {
    if (tid == 0 && cta == 0) set_device_error(VV_ERR_RANGE);
    pos = min(max(pos, 0), p.max_position - 1);
  }
  uint4 xr[kRegHB][2];
  for (int i = tid; i < D / 2; i += NW * 32) {
    as.cs[i] = p.rope_cos[(size_t)pos * (D / 2) + i];
    as.sn[i] = p.rope_sin[(size_t)pos * (D / 2) + i];
  }
  // This CTA's rows of the residual (the o-proj and down phases update exactly these rows).
  int hr0, hr1;
  cta_range(H, cta, ncta, hr0, hr1);
  float* xown = red + 32;  // up to 32 rows (H <= 32 * gridDim.x)

  for (int l = 0; l < p.L; ++l) {
    const StepLayer& w = p.layers[l];
    // ---------------------------------------------------------------- QKV
    r.ph = 0;
    if (l == 0) {
      const __half* e16 = p.input_embeds;
      if (!e16) {
        int tok = __ldcg(p.token);
        if (tok < 0 || tok >= p.V) {
          if (tid == 0 && cta == 0) set_device_error(VV_ERR_RANGE);
          tok = min(max(tok, 0), p.V - 1);
        }
        e16 = p.embed + (size_t)tok * H;
      }
      for (int i = tid; i < hr1 - hr0; i += NW * 32) xown[i] = __half2float(e16[hr0 + i]);
      stage_x(xs, red, nullptr, e16, w.in_norm, p.eps, H, cta == 0 ? p.x_resid : nullptr);
      stamp(p, sk);
    } else {
      grid_barrier(p, gen, sk);
      stage_x(xs, red, p.x_resid, nullptr, w.in_norm, p.eps, H, nullptr);
      stamp(p, sk);
    }
    const bool regH = H <= 32 * kRegHB * 16;
    {
      int r0, r1;
      cta_range(nqkv, cta, ncta, r0, r1);
      const int bounds[4] = {0, Hq * D, (Hq + Hkv) * D, nqkv};
      // this CTA's q/k/v biases -> shared memory (as.q is free until the attention phase)
      float* bias_s = &as.q[0][0];
      for (int i = tid; i < r1 - r0; i += NW * 32) {
        const int row = r0 + i;
        const int m = row < bounds[1] ? 0 : (row < bounds[2] ? 1 : 2);
        const __half* b = w.bias[m];
        bias_s[i] = b ? __half2float(b[row - bounds[m]]) : 0.f;
      }
      if (regH) load_xr(xs, xr, H);
      cbar();
      // [Wq; Wk; Wv] as one matrix of nqkv rows (the producer joins the segments)
      const float* bs = bias_s - r0;
      consume_packed(r, xs, xr, regH, H, r0, r1, 1, &as.s[0][0],
                     [&](int row, float y, float) { p.qkv[row] = y + bs[row]; });
    }
    // ---------------------------------------------------------------- ATTN
    r.ph = 1;
    grid_barrier(p, gen, sk);
    for (int it = cta; it < Hkv * nt; it += ncta) attn_item(p, r, as, l, it / nt, it % nt, past, pos);
    // ---------------------------------------------------------------- O
    r.ph = 2;
    grid_barrier(p, gen, sk);
    if (merge_in_o(p, nt)) {
      stage_attn_merged(p, xs, nt);
    } else {
      stage_x(xs, red, p.attn_out, nullptr, nullptr, 0.f, Hq * D, nullptr);
    }
    stamp(p, sk);
    const bool regO = Hq * D <= 32 * kRegHB * 16;
    if (regO) load_xr(xs, xr, Hq * D);
    {
      int r0, r1;
      cta_range(H, cta, ncta, r0, r1);
      consume_packed(r, xs, xr, regO, Hq * D, r0, r1, 1, &as.s[0][0], [&](int row, float y, float) {
        const float v = xown[row - hr0] + y;
        xown[row - hr0] = v;
        p.x_resid[row] = v;
      });
    }
    // ---------------------------------------------------------------- GU
    r.ph = 3;
    grid_barrier(p, gen, sk);
    stage_x(xs, red, p.x_resid, nullptr, w.post_norm, p.eps, H, nullptr);
    stamp(p, sk);
    if (regH) load_xr(xs, xr, H);
    {
      int r0, r1;
      cta_range(I, cta, ncta, r0, r1);
      consume_packed(r, xs, xr, regH, H, r0, r1, 2, &as.s[0][0], [&](int row, float g, float u) {
        p.h[row] = g / (1.f + __expf(-g)) * u;
      });
    }
    // ---------------------------------------------------------------- DOWN
    r.ph = 4;
    grid_barrier(p, gen, sk);
    stage_x(xs, red, p.h, nullptr, nullptr, 0.f, I, nullptr);
    stamp(p, sk);
    {
      int r0, r1;
      cta_range(H, cta, ncta, r0, r1);
      float* tr = p.trace ? p.trace + (size_t)l * H : nullptr;
      consume_packed(r, xs, xr, false, I, r0, r1, 1, &as.s[0][0], [&](int row, float y, float) {
        const float v = xown[row - hr0] + y;
        xown[row - hr0] = v;
        p.x_resid[row] = v;
        if (tr) tr[row] = v;
      });
    }
  }
  // ------------------------------------------------------------------------------ HEAD
  r.ph = 5;
  grid_barrier(p, gen, sk);
  stage_x(xs, red, p.x_resid, nullptr, p.final_norm, p.eps, H, nullptr);
  stamp(p, sk);
  float best = -INFINITY;
  int best_i = 0x7fffffff;
  {
    int r0, r1;
    cta_range(p.V, cta, ncta, r0, r1);
    const int rb = H * 2;
    const int rps = min(64, r.stage_bytes / rb);
    const int nch = H >> 3;  // 16-byte chunks per row
    // x of 16-byte weight chunk c (8 columns: half-block c/2, word c%2) = pair word (c%2, c/2);
    // held in registers for c = lane + 32 j when the row fits (H <= 1536)
    const int nhb = H >> 4;
    const uint4* xs4 = reinterpret_cast<const uint4*>(xs);
    const bool regHead = nch <= 32 * 2 * kRegHB;
    if (regHead) {
#pragma unroll
      for (int j = 0; j < 2 * kRegHB; ++j) {
        const int c = lane + 32 * j;
        xr[j >> 1][j & 1] = c < nch ? xs4[(c & 1) * nhb + (c >> 1)] : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    for (int a = r0; a < r1; a += rps) {
      const int n = min(rps, r1 - a);
      const int s = r.idx++;
      const int slot = s % r.nstages;
      ring_wait(r, &r.full[slot], (s / r.nstages) & 1);
      const unsigned char* st = r.base + (size_t)slot * r.stage_bytes;
      for (int i = warp; i < n; i += NW) {
        const unsigned char* row = st + (size_t)i * rb;
        float acc = 0.f;
        // weights (w0,w1)(w2,w3)(w4,w5)(w6,w7) against x pairs (x0,x4)(x1,x5)(x2,x6)(x3,x7)
        auto chunk = [&](const uint4 wv, const uint4 xv) {
          uint32_t p04, p15, p26, p37;
          asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(p04) : "r"(wv.x), "r"(wv.z));
          asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(p15) : "r"(wv.x), "r"(wv.z));
          asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(p26) : "r"(wv.y), "r"(wv.w));
          asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(p37) : "r"(wv.y), "r"(wv.w));
          acc = fma2_f16_f32(p04, xv.x, acc);
          acc = fma2_f16_f32(p15, xv.y, acc);
          acc = fma2_f16_f32(p26, xv.z, acc);
          acc = fma2_f16_f32(p37, xv.w, acc);
        };
        if (regHead) {
#pragma unroll
          for (int j = 0; j < 2 * kRegHB; ++j) {
            const int c = lane + 32 * j;
            if (c < nch) chunk(*reinterpret_cast<const uint4*>(row + c * 16), xr[j >> 1][j & 1]);
          }
        } else {
          for (int c = lane; c < nch; c += 32)
            chunk(*reinterpret_cast<const uint4*>(row + c * 16), xs4[(c & 1) * nhb + (c >> 1)]);
        }
        const float v = warp_sum(acc);
        if (lane == 0) {
          const int vr = a + i;
          if (p.logits) p.logits[vr] = v;
          if (better(v, vr, best, best_i)) {
            best = v;
            best_i = vr;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&r.empty[slot]);
    }
  }
  if (lane == 0) {
    s_val[warp] = best;
    s_idx[warp] = best_i;
  }
  cbar();
  stamp(p, sk);
  if (tid == 0) {
    float bv = s_val[0];
    int bi = s_idx[0];
    for (int w2 = 1; w2 < NW; ++w2)
      if (better(s_val[w2], s_idx[w2], bv, bi)) {
        bv = s_val[w2];
        bi = s_idx[w2];
      }
    p.head_val[cta] = bv;
    p.head_idx[cta] = bi;
    __threadfence();
    s_last = atomicAdd(p.head_count, 1) == ncta - 1;
  }
  cbar();
  if (!s_last) return;
  __threadfence();
  if (warp == 0) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lane; i < ncta; i += 32) {
      const float v = __ldcg(p.head_val + i);
      const int ix = __ldcg(p.head_idx + i);
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
      const int tok = bi == 0x7fffffff ? 0 : bi;
      *p.argmax = tok;
      *p.head_count = 0;
      *p.bar_count = 0u;  // every CTA has passed every barrier of this launch
      *p.length = past + 1;
      if (p.gen_done) {  // every CTA read the position at its start, long before this point
        *p.gen_count += 1;
        *p.gen_pos += 1;
        for (int j = 0; j < p.n_stop; ++j)
          if (tok == p.stop_ids[j]) *p.gen_done = 1;
      }
    }
  }
}

}  // namespace

size_t step_smem_bytes(int stage_bytes, int nstages, int x_floats) {
  // x is staged in fp16: x_floats halves
  return (size_t)nstages * stage_bytes + (size_t)x_floats * 2 + sizeof(AttnScratch) + 64 * 4 +
         2 * nstages * 8 + 64;
}

int step_threads() { return kThreads; }

size_t step_attn_part_floats(int Hkv, int max_tiles) {
  return (size_t)Hkv * max_tiles * kMaxG * kPart;
}

int step_max_tiles(int cap) { return (cap + TT - 1) / TT; }

// Pick the largest stage size (>= 32 KB, 1 KB steps) for which one CTA per SM is resident.
cudaError_t step_configure(StepParams& p, int* blocks_per_sm) {
  cudaError_t e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  *blocks_per_sm = 0;
  // a stage must hold one attention tile: 2 x TT padded rows of kRowH halves (34 KB)
  for (; p.stage_bytes >= 2 * TT * kRowH * 2; p.stage_bytes -= 1024) {
    const size_t smem = step_smem_bytes(p.stage_bytes, p.nstages, p.x_floats);
    e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, step_kernel, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (nb >= 1) {
      *blocks_per_sm = nb;
      return cudaSuccess;
    }
  }
  return cudaSuccess;
}

void step_func_info(int* regs, int* max_threads, int* static_smem, int* local_bytes) {
  cudaFuncAttributes fa = {};
  cudaFuncGetAttributes(&fa, step_kernel);
  *regs = fa.numRegs;
  *max_threads = fa.maxThreadsPerBlock;
  *static_smem = (int)fa.sharedSizeBytes;
  *local_bytes = (int)fa.localSizeBytes;
}

cudaError_t launch_step(const StepParams& p, cudaStream_t s) {
  const size_t smem = step_smem_bytes(p.stage_bytes, p.nstages, p.x_floats);
  cudaError_t e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, step_kernel, p);
}

}  // namespace vv
