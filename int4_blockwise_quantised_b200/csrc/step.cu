// Persistent decode-step kernel: the whole decoder_step (all layers + lm_head) in one
// cooperative launch ("vibevoice-asr-bitnet-onnx": decoder_step contract; "VibeVoice-ASR — ONNX
// export for Vernacula", section "Highlights": the step's ~1950 launches are the overhead to
// remove).
//
// One CTA per SM.  Warps 0..NW-1 compute, warp NW is the producer.
//
// Producer: walks a static per-CTA schedule of everything the step streams from HBM and moves it
// with cp.async.bulk into a ring of shared-memory stages.  Weights and past K/V do not depend on
// the step's activations, so HBM keeps streaming across phase boundaries, limited only by the
// ring's depth.
//
// Compute warps, per layer (four dependent phases, a grid barrier before each but the first):
//   QKV  : xn = RMSNorm(x); this CTA's rows of [Wq;Wk;Wv] . xn + b  -> qkv (fp32)
//   ATTN : items (kv head g, 64-position tile): RoPE(q), RoPE(k_new) + append at slot `length`,
//          online-softmax partial (m, l, o) per head
//   O    : items (head h, 128-row block): merge head h's partials -> o_h, then the 128 columns
//          of Wo that multiply o_h, for the block's rows; the products are added into x
//   GU+D : xn = RMSNorm(x); for each of this CTA's 64-channel slices: gate/up rows -> h =
//          silu(g) u; then the slice's 64 columns of Wd for all H rows, added into x
// then HEAD: logits = W_lm . RMSNorm(x), argmax (last CTA reduces), length += 1.
//
// The residual x lives in global memory as 64-bit fixed point (units of 2^-32): the o-proj and
// down partial products of many CTAs are added with integer atomics, so the sum does not depend
// on their order (bit-reproducible), and each phase that needs x reads it back after a barrier.
//
// int4 GEMV arithmetic (every packed matrix): the activation vector is written once per phase in
// 16-bit block fixed point, X_k = round(x_k 2^(15 - E_b)) with 2^E_b > max|x| over the 32-block b
// (|X| <= 32767); dp2a multiplies int16 pairs of X with the unsigned 4-bit codes c (unpacked to
// bytes), so sum_k (c_k - 8) X_k over a half-block is exact in int32 (the -8 X term is folded
// into the accumulator's start value); each half-block sum becomes one fp32 value, multiplied by
// the block's fp16 scale and 2^(E_b - 15), and accumulated in fp32.  The lm_head (fp16 weights)
// uses exact fp16 x fp16 products with fp32 accumulation (fma.rn.f32.f16).
//
// The grid barrier is a monotonic arrival counter in global memory (barrier k completes at
// (k + 1) x grid arrivals; the last CTA of the launch resets it); every wait is bounded
// (VV_ERR_TIMEOUT in the device error word after 2 s, then the kernel carries on).  The
// cooperative launch guarantees that all CTAs are resident.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "vv_device.cuh"
#include "vv_internal.h"
#include "step.h"

namespace vv {
namespace {

constexpr int NW = 15;                 // compute warps (+1 producer: 512 threads, 4-warp register granules)
constexpr int kThreads = (NW + 1) * 32;
constexpr int NT = NW * 32;            // compute threads
constexpr int D = 128;
constexpr int TT = 64;                 // attention tile (positions)
constexpr int kTileVOff = TT * D * 2;  // V rows of a tile start here: 64 rows of 2 bytes or 32 of 4
constexpr int kMaxG = 8;
constexpr int kMaxB = 2;               // sequences stepped together (batch)
constexpr int kPart = 132;             // floats per (tile, head) partial: m, l, -, -, o[128]
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxK = 16384;           // largest GEMV input length (hidden, n_q * D)
constexpr int kHeadRegHB = 3;          // lm_head: x chunks per lane held in registers (H <= 1536)
constexpr float kFix = 4294967296.f;   // residual fixed point: 2^32 units per 1.0
constexpr float kUnfix = 2.3283064365386963e-10f;  // 2^-32

__device__ __forceinline__ void cbar() {  // compute warps only
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

__device__ __forceinline__ void cta_range(int n, int cta, int ncta, int& r0, int& r1) {
  r0 = (int)((int64_t)n * cta / ncta);
  r1 = (int)((int64_t)n * (cta + 1) / ncta);
}

// This CTA's rows of the stacked [Wq; Wk; Wv] (n rows, n even): split in pairs of rows, so
// that every run of scale rows a stage copies starts and ends on a 16-byte boundary (a row of
// scales is K/16 bytes, a multiple of 8 for K % 128 == 0).
__device__ __forceinline__ void qkv_range(int n, int cta, int ncta, int& r0, int& r1) {
  cta_range(n / 2, cta, ncta, r0, r1);
  r0 *= 2;
  r1 *= 2;
}

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_add_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Residual fixed point: value -> 2^-32 units (two's complement in the 64-bit word) and back.
__device__ __forceinline__ unsigned long long to_fix(float v) {
  return (unsigned long long)__float2ll_rn(v * kFix);
}
__device__ __forceinline__ float from_fix(unsigned long long v) {
  return __ll2float_rn((long long)v) * kUnfix;
}

__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Timeline tap: thread 0 of each CTA records %globaltimer at fixed points of the schedule when
// p.stamps is set.
__device__ __forceinline__ void stamp(const StepParams& p, int& k) {
  if (p.stamps && threadIdx.x == 0) {
    if (k < p.max_stamps - 8) p.stamps[(size_t)blockIdx.x * p.max_stamps + k] = globaltimer_ns();
    ++k;
  }
}

// Grid-wide barrier among the compute warps of all CTAs.  The arrival counter only grows during
// a launch (barrier k completes when it reaches (k + 1) * gridDim.x) and the last CTA of the
// lm_head phase resets it, so an arrival is one fire-and-forget release-add and the wait one
// acquire poll.  Bounded wait.  Stamps: arrival, exit.
__device__ void grid_barrier(const StepParams& p, unsigned& nbar, int& sk) {
  cbar();
  stamp(p, sk);
  if (threadIdx.x == 0) {
    red_release_add(p.bar_count, 1u);
    wait_counter_geq(p.bar_count, (nbar + 1) * gridDim.x, p.wait_ns);
  }
  ++nbar;
  stamp(p, sk);
  cbar();
}

// ------------------------------------------------------------------------------ stage ring
struct Ring {
  uint64_t wait_ns;  // time this thread spent blocked in ring waits (timeline tap)
  uint64_t wait_limit;  // bound of every wait (StepParams::wait_ns)
  unsigned char* base;
  uint32_t base_a;   // shared-space address of base
  uint64_t* full;
  uint64_t* empty;
  int stage_bytes;
  int nstages;
  int slot;          // slot of the next stage (running counter modulo nstages)
  uint32_t par;      // parity of the next stage's round (stage index / nstages, low bit)
  bool wrapped;      // at least one full round of the ring done (producer: slots need freeing)
  int ph;            // phase kind of the stages being consumed (timeline tap)
  uint64_t* tapw;    // timeline tap: per-phase-kind ring wait of compute thread 0 (else null)
};

// Advance the ring position by one stage; returns the slot taken.
__device__ __forceinline__ int ring_next(Ring& r, uint32_t& par, bool& wrapped) {
  const int slot = r.slot;
  par = r.par;
  wrapped = r.wrapped;
  if (++r.slot == r.nstages) {
    r.slot = 0;
    r.par ^= 1u;
    r.wrapped = true;
  }
  return slot;
}

struct Copy {
  const void* src;
  uint32_t bytes;
  uint32_t dst_off;
};

__device__ __forceinline__ void ring_wait(Ring& r, uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  mbar_wait(bar, parity, r.wait_limit);
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
    if ((it & 63) == 0 && wait_expired(t0, r.wait_limit)) {
      set_device_error(VV_ERR_TIMEOUT);
      break;
    }
  }
  r.wait_ns += globaltimer_ns() - t0;
}

// Producer side: take the next slot (waiting until the consumers have freed it, from the second
// round on) and arm its full barrier for `tx_bytes`; returns the slot.
__device__ __forceinline__ int produce_begin(Ring& r, uint32_t tx_bytes) {
  uint32_t par;
  bool wrapped;
  const int slot = ring_next(r, par, wrapped);
  if (wrapped) producer_wait(r, &r.empty[slot], par ^ 1u);
  mbar_arrive_expect_tx(&r.full[slot], tx_bytes);
  return slot;
}

__device__ __forceinline__ void produce(Ring& r, const Copy* c, int n, uint64_t pol) {
  uint32_t tot = 0;
  for (int i = 0; i < n; ++i) tot += c[i].bytes;
  const int slot = produce_begin(r, tot);
  unsigned char* dst = r.base + (size_t)slot * r.stage_bytes;
  for (int i = 0; i < n; ++i)
    if (c[i].bytes) bulk_g2s_stream(dst + c[i].dst_off, c[i].src, c[i].bytes, &r.full[slot], pol);
}

// Consumer side: wait for the next stage; returns its shared-space address (and the slot).
__device__ __forceinline__ uint32_t consume_begin(Ring& r, int& slot) {
  uint32_t par;
  bool wrapped;
  slot = ring_next(r, par, wrapped);
  ring_wait(r, &r.full[slot], par);
  return r.base_a + (uint32_t)(slot * r.stage_bytes);
}
__device__ __forceinline__ void consume_end(Ring& r, int slot) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&r.empty[slot]);
}

// --------------------------------------------------------------------------- stage geometry
// Row phases (QKV, gate/up): stage = [seg0 codes rps rows][seg1 codes][seg0 scales][seg1 scales],
// rows of K/32 x 16 code bytes and K/32 x 2 scale bytes (K % 128 == 0: a scale row is a multiple
// of 8 bytes, so runs of an even number of rows from an even row are 16-byte aligned).  Column phases (o-proj, down): stage =
// [codes rps rows x nb x 16][scales rps rows x nb x 2] of a column image.
__device__ __forceinline__ int rows_per_stage(int row_bytes, int stage_bytes) {
  int r = stage_bytes / row_bytes;
  return r & ~7;  // a multiple of 8 rows keeps every scale run 16-byte aligned
}

// One attention tile: past K rows and V rows (D elements of elem_bytes each, consecutive in the
// cache; `row_units` = rows x elem_bytes) with one copy each: K rows at the stage base, V rows
// kTileVOff bytes after them.
__device__ void produce_kv_rows(Ring& r, const unsigned char* k, const unsigned char* v,
                                int row_units, uint64_t pol) {
  const uint32_t bytes = (uint32_t)row_units * D;
  const int slot = produce_begin(r, 2 * bytes);
  unsigned char* dst = r.base + (size_t)slot * r.stage_bytes;
  if (bytes) {
    bulk_g2s_stream(dst, k, bytes, &r.full[slot], pol);
    bulk_g2s_stream(dst + kTileVOff, v, bytes, &r.full[slot], pol);
  }
}

// Rows [r0, r1) of a packed matrix, and the same rows of a second one (gate/up).
__device__ void produce_rows(Ring& r, const uint8_t* q0, const __half* s0, const uint8_t* q1,
                             const __half* s1, int K, int r0, int r1, uint64_t pol) {
  const int nseg = q1 ? 2 : 1;
  const int rq = (K >> 5) * 16, rs = (K >> 5) * 2;
  const int rps = rows_per_stage((rq + rs) * nseg, r.stage_bytes);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    Copy c[4];
    int k = 0;
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

// Logical rows [r0, r1) of [Wq; Wk; Wv] (bounds: first row of each matrix); a stage may hold
// rows of two matrices, laid out as one matrix of consecutive rows.
__device__ void produce_qkv(Ring& r, const StepLayer& w, int K, int r0, int r1,
                            const int (&bounds)[4], uint64_t pol) {
  const int rq = (K >> 5) * 16, rs = (K >> 5) * 2;
  const int rps = rows_per_stage(rq + rs, r.stage_bytes);
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

// A column image of `rows` rows x nb blocks: [codes rows x nb x 16][scales rows x nb x 2].
__device__ void produce_cols(Ring& r, const unsigned char* img, int rows, int nb, uint64_t pol) {
  const int rps = rows_per_stage(nb * 18, r.stage_bytes);
  const unsigned char* sc = img + (size_t)rows * nb * 16;
  for (int a = 0; a < rows; a += rps) {
    const int n = min(rps, rows - a);
    Copy c[2] = {Copy{img + (size_t)a * nb * 16, (uint32_t)(n * nb * 16), 0u},
                 Copy{sc + (size_t)a * nb * 2, (uint32_t)(n * nb * 2), (uint32_t)(rps * nb * 16)}};
    produce(r, c, 2, pol);
  }
}

// The attention items of a launch: sequence b has nt[b] tiles of tt positions per KV head;
// items are numbered sequence-major, (b, g, t) for b < nb, g < Hkv, t < nt[b].  Tiles of 32
// positions when doubling the tiles of 64 still gives every item its own CTA (always for 4-byte
// K/V, whose 32 rows fill kTileVOff), else 64.  Producer and consumers compute the same plan.
struct AttnPlan {
  int tt;
  int nt[kMaxB];
  int total;
};
__device__ __forceinline__ int kv_bytes(const StepParams& p) { return p.kv_type == 2 ? 4 : 2; }
// lm_head rows per stage: as many as fit (at most 64), rounded down to a multiple of the compute
// warps when there are more than NW (each warp takes whole rows: 16 rows on 15 warps would give
// one warp two rows and make every stage take two rows' time).  Producer and consumers agree.
__device__ __forceinline__ int head_rows_per_stage(int stage_bytes, int row_bytes) {
  const int n = min(64, stage_bytes / row_bytes);
  return n > NW ? n / NW * NW : n;
}
__device__ __forceinline__ int ntiles_for(int past, int tt) { return (past + 1 + tt - 1) / tt; }
__device__ __forceinline__ AttnPlan attn_plan(const StepParams& p, const int* past) {
  AttnPlan a;
  int n64 = 0;
  for (int b = 0; b < p.nb; ++b) n64 += ntiles_for(past[b], TT);
  a.tt = (kv_bytes(p) == 4 || 2 * p.Hkv * n64 <= (int)gridDim.x) ? TT / 2 : TT;
  a.total = 0;
  for (int b = 0; b < kMaxB; ++b) {
    a.nt[b] = b < p.nb ? ntiles_for(past[b], a.tt) : 0;
    a.total += p.Hkv * a.nt[b];
  }
  return a;
}
__device__ __forceinline__ void attn_item_of(const AttnPlan& a, int Hkv, int it, int& b, int& g,
                                             int& t) {
  b = 0;
  while (b + 1 < kMaxB && it >= Hkv * a.nt[b]) it -= Hkv * a.nt[b++];
  g = it / a.nt[b];
  t = it % a.nt[b];
}
__device__ __forceinline__ int n_slices(const StepParams& p) { return p.I / kSlice; }
__device__ __forceinline__ int slices_of(const StepParams& p, int cta) {
  const int ns = n_slices(p);
  return ns > cta ? (ns - 1 - cta) / (int)gridDim.x + 1 : 0;
}
__device__ __forceinline__ size_t wd_cta_stride(const StepParams& p) {
  const int nsl_max = (n_slices(p) + gridDim.x - 1) / gridDim.x;
  return (size_t)p.H * nsl_max * 2 * 18;
}

// CTA c's down-column image stores row (i + wd_rot) mod H at position i: the CTAs walk x from
// different rows, so their residual additions reach different L2 lines at the same time.
__host__ __device__ __forceinline__ int wd_rot(int H, int c, int grid) {
  return (int)((((long long)c * H) / grid) & ~31LL) % H;
}

__device__ void producer(const StepParams& p, Ring& r, const int* past) {
  const uint64_t pol = policy_evict_first();
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int H = p.H, Hq = p.Hq, Hkv = p.Hkv;
  const int nqkv = (Hq + 2 * Hkv) * D;
  const AttnPlan plan = attn_plan(p, past);
  const int nrb = H / kORows;
  const int nsl = slices_of(p, cta);
  const int ns = n_slices(p);
  int o0, o1;
  cta_range(Hq * nrb, cta, ncta, o0, o1);
  int r0, r1;  // this CTA's lm_head rows
  cta_range(p.V, cta, ncta, r0, r1);
  for (int l = 0; l < p.L; ++l) {
    const StepLayer& w = p.layers[l];
    int q0, q1;
    qkv_range(nqkv, cta, ncta, q0, q1);
    const int bounds[4] = {0, Hq * D, (Hq + Hkv) * D, nqkv};
    produce_qkv(r, w, H, q0, q1, bounds, pol);
    for (int it = cta; it < plan.total; it += ncta) {
      int b, g, t;
      attn_item_of(plan, Hkv, it, b, g, t);
      const int p0 = t * plan.tt, p1 = min(p0 + plan.tt, past[b]);
      const size_t off = ((size_t)((l * p.nb + b) * Hkv + g) * p.cap + p0) * D;
      const int eb = kv_bytes(p);
      produce_kv_rows(r, static_cast<const unsigned char*>(p.k_cache) + off * eb,
                      static_cast<const unsigned char*>(p.v_cache) + off * eb, max(p1 - p0, 0) * eb,
                      pol);
    }
    for (int i = o0; i < o1; ++i)
      produce_cols(r, w.wo_img + (size_t)i * kORows * 4 * 18, kORows, 4, pol);
    for (int s = cta; s < ns; s += ncta)
      produce_rows(r, w.q[4], w.s[4], w.q[5], w.s[5], H, s * kSlice, (s + 1) * kSlice, pol);
    if (nsl > 0) produce_cols(r, w.wd_img + (size_t)cta * wd_cta_stride(p), H, 2 * nsl, pol);
  }
  // HEAD: fp16 rows of the lm_head
  const int rb = H * 2;
  const int rps = head_rows_per_stage(r.stage_bytes, rb);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    Copy c[1] = {Copy{p.lm_head + (size_t)a * H, (uint32_t)(n * rb), 0u}};
    produce(r, c, 1, pol);
  }
}

// ------------------------------------------------------------------ GEMV operand (X) staging
// The activation operand of the int4 GEMVs, in shared memory:
//   xq   uint4 [2][NHB]: half-block hb, code word w (elements 8w..8w+7 of the half-block) ->
//        int16 pairs (X0,X2) (X4,X6) (X1,X3) (X5,X7) in the dp2a order of the unpacked codes
//        (low nibbles = even elements, high nibbles = odd elements);
//   corr int [NHB]: -8 * sum of X over the half-block;
//   fb   float [NHB/2]: 2^(E_b - 15) per 32-block.
struct XOp {
  uint4* xq;
  int* corr;
  float* fb;
  uint32_t xq_a, corr_a, fb_a;  // the same, as shared-space addresses
};

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((e + 127) << 23); }

// Write X of the 4 consecutive elements k..k+3 (k % 4 == 0) held by this thread.  Every thread
// of the compute group calls this for chunk slots in lockstep (the 32-block of k is spread over
// 8 consecutive threads, the half-block over 4); `valid` false for padding slots.
__device__ __forceinline__ void put_x4(const XOp& xo, int NHB, int k, float4 y, bool valid) {
  float m = valid ? fmaxf(fmaxf(fabsf(y.x), fabsf(y.y)), fmaxf(fabsf(y.z), fabsf(y.w))) : 0.f;
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
  // 2^E > m: E = unbiased exponent of m + 1 (denormals and zero -> the smallest normal)
  int E = max((__float_as_int(m) >> 23) & 0xFF, 1) - 126;
  E = max(E, -100);
  const float sc = pow2f(15 - E);
  auto q = [&](float v) { return min(max(__float2int_rn(v * sc), -32767), 32767); };
  const int X0 = q(y.x), X1 = q(y.y), X2 = q(y.z), X3 = q(y.w);
  int sx = valid ? X0 + X1 + X2 + X3 : 0;
  sx += __shfl_xor_sync(0xffffffffu, sx, 1);
  sx += __shfl_xor_sync(0xffffffffu, sx, 2);
  if (!valid) return;
  const int hb = k >> 4, w = (k >> 3) & 1, j0 = k & 7;  // j0 in {0, 4}
  uint32_t* dst = reinterpret_cast<uint32_t*>(xo.xq) + (size_t)(w * NHB + hb) * 4;
  auto pk = [](int a, int b) { return (uint32_t)(uint16_t)(int16_t)a | ((uint32_t)(uint16_t)(int16_t)b << 16); };
  dst[j0 >> 2] = pk(X0, X2);
  dst[2 + (j0 >> 2)] = pk(X1, X3);
  if ((k & 15) == 0) xo.corr[hb] = -8 * sx;
  if ((k & 31) == 0) xo.fb[k >> 5] = pow2f(E - 15);
}

// Stage a K-vector (K % 32 == 0, K <= 4 * 4 * NT) as the GEMV operand: y = src (* rsqrt(mean
// src^2 + eps) * gamma when gamma is set).  load(k) returns elements k..k+3 as fp32.  Optional
// fp32 copy of src (trace).  All compute threads; ends with a compute barrier.
template <class Load>
__device__ void stage_idp(const XOp& xo, Load load, const __half* gamma, float eps, int K,
                          float* red, float* copy_out) {
  const int tid = threadIdx.x;
  constexpr int kC = 4;  // chunks of 4 per thread
  const int NHB = K >> 4;
  float4 v[kC];
  uint2 gv[kC];  // gamma halves, loaded with x so that both arrive in one round trip
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kC; ++i) {
    const int k = (tid + i * NT) * 4;
    if (gamma && k < K) gv[i] = *reinterpret_cast<const uint2*>(gamma + k);
    v[i] = k < K ? load(k) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int i = 0; i < kC; ++i) {
    const int k = (tid + i * NT) * 4;
    if (k < K && copy_out) *reinterpret_cast<float4*>(copy_out + k) = v[i];
    ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
  }
  if (gamma) {
    ss = warp_sum(ss);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    cbar();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < NW; ++i) tot += red[i];
    const float inv = rsqrtf(tot / (float)K + eps);
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      const int k = (tid + i * NT) * 4;
      if (k < K) {
        const float2 g01 = __half22float2(*reinterpret_cast<const __half2*>(&gv[i].x));
        const float2 g23 = __half22float2(*reinterpret_cast<const __half2*>(&gv[i].y));
        v[i].x *= inv * g01.x;
        v[i].y *= inv * g01.y;
        v[i].z *= inv * g23.x;
        v[i].w *= inv * g23.y;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kC; ++i) {
    const int k = (tid + i * NT) * 4;
    if (i * NT * 4 < K) put_x4(xo, NHB, k, v[i], k < K);  // warp-uniform slot condition
  }
  cbar();
}

// ----------------------------------------------------------------------------- int4 GEMV
// Shared-memory loads by 32-bit shared-space address.
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ float lds_half(uint32_t a) {
  unsigned short h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(a));
  return __half2float(__ushort_as_half(h));
}

// One half-block (16 weights: two code words) against its X pairs: exact int32 sum of
// (c - 8) X, starting from corr = -8 sum X (two independent dp2a chains).
__device__ __forceinline__ int hb_dot(uint2 wv, uint4 xa, uint4 xb, int corr) {
  const uint32_t l0 = wv.x & 0x0F0F0F0Fu, h0 = (wv.x >> 4) & 0x0F0F0F0Fu;
  const uint32_t l1 = wv.y & 0x0F0F0F0Fu, h1 = (wv.y >> 4) & 0x0F0F0F0Fu;
  int s = corr, t = 0;
  s = dp2a_lo(xa.x, l0, s);
  t = dp2a_lo(xb.x, l1, t);
  s = dp2a_hi(xa.y, l0, s);
  t = dp2a_hi(xb.y, l1, t);
  s = dp2a_lo(xa.z, h0, s);
  t = dp2a_lo(xb.z, h1, t);
  s = dp2a_hi(xa.w, h0, s);
  t = dp2a_hi(xb.w, h1, t);
  return s + t;
}

// The units of one stage: unit u = (row u / NSEG, matrix u % NSEG); the code bytes of (row, m)
// start at q0 + (m rps + row) rq, its scales at s0 + (m rps + row) rs (shared-space addresses).
struct UnitMap {
  uint32_t q0, s0;
  int rps, rq, rs;
};

// Rows per pass (R) for `units` units with 2^lg_gpw lane groups per warp: the R in {1, 2, 4}
// ({2, 4} for pairs) that minimises the busiest warp's share (R x its passes), the larger R on
// ties.  Shifts and a division by the constant NW only (this runs for every stage).
__device__ __forceinline__ int pick_r(int units, int lg_gpw, bool pair) {
  int best = pair ? 2 : 1, cost_best = 1 << 30;
#pragma unroll
  for (int lr = 0; lr <= 2; ++lr) {
    const int R = 1 << lr;
    if (R < best) continue;
    const int sh = lg_gpw + lr;
    const int passes = (units + (1 << sh) - 1) >> sh;
    const int cost = R * ((passes + NW - 1) / NW);
    if (cost <= cost_best) {
      best = R;
      cost_best = cost;
    }
  }
  return best;
}

// The units of one stage against the staged X of NB sequences (the weights are read once for
// all of them): LPR lanes per unit (lane % LPR strides the half-blocks), R units per lane group
// and pass.  fin(u, y0, y1) is called by the group's first lane once per unit with y0[b] the
// result of sequence b (y1 unused), or with NSEG == 2 once per row with both matrices' results.
template <int LPR, int R, int NSEG, int NB, class Fin>
__device__ __forceinline__ void gemv_pass(const XOp* xo, int NHB, int units, const UnitMap& m,
                                          Fin fin) {
  static_assert(NSEG == 1 || R % NSEG == 0, "pairs need an even R");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int GPW = 32 / LPR;
  const int sub = lane % LPR, grp = lane / LPR;
  // the loop bound is warp-uniform (every lane runs the same iterations, as the full-mask
  // shuffles below require); lane groups past the last unit work on a clamped unit, skip fin
  for (int ub = warp * GPW * R; ub < units; ub += NW * GPW * R) {
    const int u0 = ub + grp * R;
    uint32_t qa[R], sa[R];
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int u = min(u0 + k, units - 1);
      const int idx = NSEG == 1 ? u : (u % NSEG) * m.rps + u / NSEG;
      qa[k] = m.q0 + (uint32_t)(idx * m.rq);
      sa[k] = m.s0 + (uint32_t)(idx * m.rs);
    }
    float acc[R][NB];
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[k][b] = 0.f;
#pragma unroll 2
    for (int hb = sub; hb < NHB; hb += LPR) {
      uint4 xa[NB], xb[NB];
      int cr[NB];
      float f[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        xa[b] = lds128(xo[b].xq_a + hb * 16);
        xb[b] = lds128(xo[b].xq_a + (NHB + hb) * 16);
        cr[b] = (int)lds32(xo[b].corr_a + hb * 4);
        f[b] = __uint_as_float(lds32(xo[b].fb_a + (hb >> 1) * 4));
      }
#pragma unroll
      for (int k = 0; k < R; ++k) {
        const uint2 wv = lds64(qa[k] + hb * 8);
        const float sc = lds_half(sa[k] + (hb >> 1) * 2);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          acc[k][b] = fmaf(sc * f[b], (float)hb_dot(wv, xa[b], xb[b], cr[b]), acc[k][b]);
      }
    }
#pragma unroll
    for (int k = 0; k < R; ++k)
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) acc[k][b] += __shfl_xor_sync(0xffffffffu, acc[k][b], o);
    if (sub == 0) {
#pragma unroll
      for (int k = 0; k < R; k += NSEG)
        if (u0 + k < units) fin(u0 + k, acc[k], acc[k + NSEG - 1]);
    }
  }
}

// One stage: lanes per unit from the row length (a lane takes about 4 half-blocks of short rows;
// rows longer than 16 half-blocks take a whole warp), rows per pass from the unit count.
template <int NSEG, int NB, class Fin>
__device__ __forceinline__ void gemv_stage(const XOp* xo, int NHB, int units, const UnitMap& m,
                                           Fin fin) {
  auto go = [&](auto lpr_c) {
    constexpr int LPR = decltype(lpr_c)::value;
    constexpr int kLgGpw = LPR == 32 ? 0 : LPR == 4 ? 3 : LPR == 2 ? 4 : 5;
    const int R = pick_r(units, kLgGpw, NSEG == 2);
    if constexpr (NSEG == 1) {
      if (R == 1) {
        gemv_pass<LPR, 1, NSEG, NB>(xo, NHB, units, m, fin);
        return;
      }
    }
    if (R == 2)
      gemv_pass<LPR, 2, NSEG, NB>(xo, NHB, units, m, fin);
    else
      gemv_pass<LPR, 4, NSEG, NB>(xo, NHB, units, m, fin);
  };
  if (NHB > 16) {
    go(std::integral_constant<int, 32>());
  } else if (NHB > 8) {
    go(std::integral_constant<int, 4>());
  } else if constexpr (NSEG == 1) {
    if (NHB > 4)
      go(std::integral_constant<int, 2>());
    else
      go(std::integral_constant<int, 1>());
  } else {
    go(std::integral_constant<int, 4>());
  }
}

// Row phase: the stages of rows [r0, r1) of NSEG matrices.  fin(row, y0, y1) with y0[b], y1[b].
template <int NSEG, int NB, class Fin>
__device__ void consume_rows(Ring& r, const XOp* xo, int K, int r0, int r1, Fin fin) {
  const int KB = K >> 5, NHB = K >> 4;
  const int rq = KB * 16, rs = KB * 2;
  const int rps = rows_per_stage((rq + rs) * NSEG, r.stage_bytes);
  for (int a = r0; a < r1; a += rps) {
    const int n = min(rps, r1 - a);
    int slot;
    const uint32_t st = consume_begin(r, slot);
    const UnitMap m{st, st + (uint32_t)(NSEG * rps * rq), rps, rq, rs};
    gemv_stage<NSEG, NB>(xo, NHB, n * NSEG, m,
                         [&](int u, const float* y0, const float* y1) { fin(a + u / NSEG, y0, y1); });
    consume_end(r, slot);
  }
}

// Column phase: the stages of a column image of `rows_total` rows x nb blocks (K = 32 nb).
// fin(row, y) with y[b].
template <int NB, class Fin>
__device__ void consume_cols(Ring& r, const XOp* xo, int rows_total, int nb, Fin fin) {
  const int NHB = nb * 2;
  const int rps = rows_per_stage(nb * 18, r.stage_bytes);
  for (int a = 0; a < rows_total; a += rps) {
    const int n = min(rps, rows_total - a);
    int slot;
    const uint32_t st = consume_begin(r, slot);
    const UnitMap m{st, st + (uint32_t)(rps * nb * 16), rps, nb * 16, nb * 2};
    gemv_stage<1, NB>(xo, NHB, n, m, [&](int u, const float* y, const float*) { fin(a + u, y); });
    consume_end(r, slot);
  }
}

// ------------------------------------------------------------------------------- attention
// K/V storage types of the cache (and of the attention tiles in shared memory): fp16 (the
// contract), bf16 and fp32 (the variants).  load8 widens 8 consecutive elements to fp32 pairs.
struct KvF16 {
  using T = __half;
  static constexpr int kBytes = 2;
  __device__ static T from(float v) { return __float2half_rn(v); }
  __device__ static void load8(const T* p, float2 (&f)[4]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    f[0] = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
    f[1] = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
    f[2] = __half22float2(*reinterpret_cast<const __half2*>(&u.z));
    f[3] = __half22float2(*reinterpret_cast<const __half2*>(&u.w));
  }
};
struct KvBF16 {
  using T = __nv_bfloat16;
  static constexpr int kBytes = 2;
  __device__ static T from(float v) { return __float2bfloat16_rn(v); }
  __device__ static void load8(const T* p, float2 (&f)[4]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  }
};
struct KvF32 {
  using T = float;
  static constexpr int kBytes = 4;
  __device__ static T from(float v) { return v; }
  __device__ static void load8(const T* p, float2 (&f)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    f[0] = make_float2(a.x, a.y);
    f[1] = make_float2(a.z, a.w);
    f[2] = make_float2(b.x, b.y);
    f[3] = make_float2(b.z, b.w);
  }
};
struct AttnScratch {
  float cs[kMaxB][D / 2], sn[kMaxB][D / 2];  // RoPE cos/sin at each sequence's position
  float q[kMaxG][D];
  float s[kMaxG][TT];
  float m[kMaxG], l[kMaxG];
  float pv[4][kMaxG][D];  // P.V partial sums per position quarter
};

template <class KV>
__device__ void attn_item(const StepParams& p, Ring& r, AttnScratch& as, int l, int b, int g,
                          int t, int past, int tt) {
  using T = typename KV::T;
  const float* cs_b = as.cs[b];
  const float* sn_b = as.sn[b];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.Hq / p.Hkv;
  const int nt = ntiles_for(past, tt);
  const int npos = past + 1;
  const int p0 = t * tt;
  const int n = min(tt, npos - p0);
  const float* qkv = p.qkv + (size_t)b * (p.Hq + 2 * p.Hkv) * D;
  // q of the group (rotated, scaled into the log2 domain) and, on the tile holding the new
  // position, the new k/v: every global load is issued before any is used (one L2 round trip).
  const float qscale = p.scale * kLog2e;
  const bool newpos = t == nt - 1;
  constexpr int kQPer = (kMaxG * D + NT - 1) / NT;  // q element pairs per thread
  float qa[kQPer], qb[kQPer];
#pragma unroll
  for (int j = 0; j < kQPer; ++j) {
    const int i = tid + j * NT;
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
    const int i = tid + j * NT;
    if (i < G * D) {
      const int h = i / D, d = i % D;
      const int fi = d & (D / 2 - 1);
      const float cs = cs_b[fi], sn = sn_b[fi];
      as.q[h][d] = (d < D / 2 ? qa[j] * cs - qb[j] * sn : qb[j] * cs + qa[j] * sn) * qscale;
    }
  }
  int slot;
  consume_begin(r, slot);
  T* kt = reinterpret_cast<T*>(r.base + (size_t)slot * r.stage_bytes);
  T* vt = reinterpret_cast<T*>(r.base + (size_t)slot * r.stage_bytes + kTileVOff);
  if (newpos && tid < D) {  // this tile holds the new position: rotate k, append k/v
    const int d = tid, fi = d & (D / 2 - 1);
    const float cs = cs_b[fi], sn = sn_b[fi];
    const T kn = KV::from(d < D / 2 ? ka * cs - kb * sn : kb * cs + ka * sn);
    const T vn = KV::from(vv);
    const size_t off = ((size_t)((l * p.nb + b) * p.Hkv + g) * p.cap + past) * D + d;
    static_cast<T*>(p.k_cache)[off] = kn;
    static_cast<T*>(p.v_cache)[off] = vn;
    kt[(past - p0) * D + d] = kn;
    vt[(past - p0) * D + d] = vn;
  }
  cbar();
  // scores: item = (head, half of the tile); a warp takes one item, lpd lanes per position (1 for
  // tiles of 64, 2 for tiles of 32, each lane then summing 64 of the 128 dims), so every lane has
  // work.  K rows are 256 bytes apart: a lane walks its chunks starting at one that depends on the
  // position, so the 8 lanes of a 16-byte load phase read 8 different chunks (distinct banks; the
  // q reads are 2-way).
  {
    const int lpd = tt == TT ? 1 : 2;
    const int nch = 16 / lpd;  // 16-byte chunks of the row per lane
    const int half = lane % lpd;
    for (int item = warp; item < 2 * G; item += NW) {
      const int h = item >> 1, pp = (item & 1) * (32 / lpd) + lane / lpd;
      float sc = -INFINITY;
      if (pp < n) {
        const T* kr = kt + pp * D;
        float2 acc = make_float2(0.f, 0.f), acc2 = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int c = 0; c < nch; ++c) {
          const int cc = ((c + pp) & (nch - 1)) + half * nch;
          float2 k8[4];
          KV::load8(kr + cc * 8, k8);
          const float4 qa4 = *reinterpret_cast<const float4*>(&as.q[h][cc * 8]);
          const float4 qb4 = *reinterpret_cast<const float4*>(&as.q[h][cc * 8 + 4]);
          acc = __ffma2_rn(k8[0], make_float2(qa4.x, qa4.y), acc);
          acc2 = __ffma2_rn(k8[1], make_float2(qa4.z, qa4.w), acc2);
          acc = __ffma2_rn(k8[2], make_float2(qb4.x, qb4.y), acc);
          acc2 = __ffma2_rn(k8[3], make_float2(qb4.z, qb4.w), acc2);
        }
        sc = (acc.x + acc.y) + (acc2.x + acc2.y);
      }
      if (lpd == 2) sc += __shfl_xor_sync(0xffffffffu, sc, 1);  // the pair's two halves
      if (half == 0) as.s[h][pp] = sc;
    }
  }
  cbar();
  if (warp < G) {  // softmax statistics of this tile, per head
    const int h = warp;
    // positions past the tile's n (all of 32..63 for tiles of 32) hold no score of this item
    const float s0 = lane < n ? as.s[h][lane] : -INFINITY;
    const float s1 = lane + 32 < n ? as.s[h][lane + 32] : -INFINITY;
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
  // P.V: unit = (head h, 8-dim octet o, position quarter q of tt/4 positions); V rows read as
  // 16-byte vectors (the 16 octets of a row on consecutive lanes: conflict-free), quarters
  // combined through shared memory (as.pv), then written as the tile's partial.
  {
    const int units = G * 16 * 4;
    const int ppu = tt / 4;
    for (int u = tid; u < units; u += NT) {
      const int o = u & 15, q = (u >> 4) & 3, h = u >> 6;
      float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
      const float* ph = as.s[h];
      const int p_end = min(n, q * ppu + ppu);
#pragma unroll 4
      for (int pp = q * ppu; pp < p_end; ++pp) {
        float2 v8[4];
        KV::load8(vt + pp * D + o * 8, v8);
        const float w = ph[pp];
        const float2 ww = make_float2(w, w);
        a0 = __ffma2_rn(v8[0], ww, a0);
        a1 = __ffma2_rn(v8[1], ww, a1);
        a2 = __ffma2_rn(v8[2], ww, a2);
        a3 = __ffma2_rn(v8[3], ww, a3);
      }
      float4* dst = reinterpret_cast<float4*>(&as.pv[q][h][o * 8]);
      dst[0] = make_float4(a0.x, a0.y, a1.x, a1.y);
      dst[1] = make_float4(a2.x, a2.y, a3.x, a3.y);
    }
    cbar();
    float* part = p.attn_part + (((size_t)b * p.Hkv + g) * p.max_tiles + t) * kMaxG * kPart;
    for (int idx = tid; idx < G * D; idx += NT) {
      const int h = idx >> 7, d = idx & (D - 1);
      part[h * kPart + 4 + d] = (as.pv[0][h][d] + as.pv[1][h][d]) + (as.pv[2][h][d] + as.pv[3][h][d]);
    }
    if (tid < G) {
      part[tid * kPart + 0] = as.m[tid];
      part[tid * kPart + 1] = as.l[tid];
    }
  }
  consume_end(r, slot);
  cbar();  // as.s / as.pv are reused by the next item
}

// Merge head h's partials over the nt tiles: M = max_t m_t, L = sum_t l_t 2^(m_t - M),
// o[d] = sum_t 2^(m_t - M) o_t[d] / L.  Threads (d4, tile slice): 32 float4 columns x up to
// 15 tile slices, combined through shared memory.  Result in out[128] (fp32, shared).
__device__ void merge_head(const StepParams& p, int b, int h, int nt, float* scratch, float* out) {
  const int tid = threadIdx.x;
  const int G = p.Hq / p.Hkv, g = h / G, hh = h % G;
  const float* base =
      p.attn_part + (((size_t)b * p.Hkv + g) * p.max_tiles * kMaxG + hh) * kPart;
  const int d4 = tid & 31, ts = tid >> 5;  // ts in [0, NW)
  float M = -INFINITY, L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // up to 4 tiles per thread per round: all their loads are issued before the first is used
  for (int t0 = ts; t0 < nt; t0 += 4 * NW) {
    float mt[4], lt[4];
    float4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + j * NW;
      if (t < nt) {
        const float* pt = base + (size_t)t * kMaxG * kPart;
        mt[j] = __ldcg(pt);
        lt[j] = __ldcg(pt + 1);
        v[j] = __ldcg(reinterpret_cast<const float4*>(pt + 4) + d4);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (t0 + j * NW >= nt) break;
      const float bm = fmaxf(M, mt[j]);
      const float c = exp2f(M - bm), e = exp2f(mt[j] - bm);
      L = L * c + lt[j] * e;
      acc.x = acc.x * c + e * v[j].x;
      acc.y = acc.y * c + e * v[j].y;
      acc.z = acc.z * c + e * v[j].z;
      acc.w = acc.w * c + e * v[j].w;
      M = bm;
    }
  }
  // scratch: [NW][32][6]
  float* sp = scratch + (ts * 32 + d4) * 6;
  sp[0] = M;
  sp[1] = L;
  sp[2] = acc.x;
  sp[3] = acc.y;
  sp[4] = acc.z;
  sp[5] = acc.w;
  cbar();
  if (tid < 32) {
    float Mx = -INFINITY;
    for (int s = 0; s < NW; ++s) Mx = fmaxf(Mx, scratch[(s * 32 + tid) * 6]);
    float Lt = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < NW; ++s) {
      const float* q = scratch + (s * 32 + tid) * 6;
      const float e = q[0] == -INFINITY ? 0.f : exp2f(q[0] - Mx);
      Lt = fmaf(q[1], e, Lt);
      a.x = fmaf(q[2], e, a.x);
      a.y = fmaf(q[3], e, a.y);
      a.z = fmaf(q[4], e, a.z);
      a.w = fmaf(q[5], e, a.w);
    }
    const float inv = 1.f / Lt;
    reinterpret_cast<float4*>(out)[tid] = make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv);
  }
  cbar();
}

// --------------------------------------------------------------------------- lm_head x
// fp16 x in the half2-pair layout of the fp16 head dot: element k (hb = k/16, word = (k/8)%2,
// j = k%8) at uint4 (word * NHB + hb), component j%4, half j/4.
__device__ __forceinline__ int xh_slot(int k, int nhb) {
  const int hb = k >> 4, word = (k >> 3) & 1, j = k & 7;
  return ((word * nhb + hb) * 4 + (j & 3)) * 2 + (j >> 2);
}

__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1) step_kernel(const StepParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int H = p.H, Hq = p.Hq, Hkv = p.Hkv;
  Ring r;
  r.wait_ns = 0;
  r.wait_limit = p.wait_ns;
  r.ph = 0;
  // timeline tap: the last 8 stamps of a CTA's row hold thread 0's ring wait per phase kind
  // (QKV, ATTN, O, GU, DOWN, HEAD at max-8 .. max-3), then the producer's done time and its
  // blocked time.
  r.tapw = (p.stamps && threadIdx.x == 0) ? p.stamps + (size_t)blockIdx.x * p.max_stamps + p.max_stamps - 8
                                          : nullptr;
  r.base = smem;
  r.stage_bytes = p.stage_bytes;
  r.nstages = p.nstages;
  r.base_a = smem_u32(smem);
  r.slot = 0;
  r.par = 0;
  r.wrapped = false;
  // shared layout after the ring, per sequence b: xq [2][kMaxK/16] uint4 | corr [kMaxK/16] |
  // fb [kMaxK/32] | hbuf; then AttnScratch | red[64] | mbarriers
  unsigned char* sp = smem + (size_t)p.nstages * p.stage_bytes;
  const int maxK = max(H, Hq * D);
  const int nhb_max = maxK / 16;
  const int nsl = slices_of(p, blockIdx.x);
  XOp xo[NB];
  float* hbuf[NB];  // h of this CTA's slices, then o_h of an o-item
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    xo[b].xq = reinterpret_cast<uint4*>(sp);
    sp += (size_t)nhb_max * 2 * 16;
    xo[b].corr = reinterpret_cast<int*>(sp);
    sp += (size_t)nhb_max * 4;
    xo[b].fb = reinterpret_cast<float*>(sp);
    sp += (size_t)nhb_max * 2;
    xo[b].xq_a = smem_u32(xo[b].xq);
    xo[b].corr_a = smem_u32(xo[b].corr);
    xo[b].fb_a = smem_u32(xo[b].fb);
    hbuf[b] = reinterpret_cast<float*>(sp);
    sp += (size_t)max(nsl * kSlice, D) * 4;
    sp = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sp) + 15) & ~uintptr_t(15));
  }
  AttnScratch& as = *reinterpret_cast<AttnScratch*>(sp);
  float* red = reinterpret_cast<float*>(&as + 1);  // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(red + 64) + 15) &
                                               ~uintptr_t(15));
  r.full = bars;
  r.empty = bars + p.nstages;
  __shared__ float s_val[NB][NW];
  __shared__ int s_idx[NB][NW];
  __shared__ int s_last;

  // generation stopped by an earlier step of the same vv_decoder_generate call: every CTA sees
  // the same word (written by the previous launch) and leaves before touching anything
  if (p.gen_done && __ldcg(p.gen_done) != 0) return;
  int past[kMaxB];
#pragma unroll
  for (int b = 0; b < kMaxB; ++b) past[b] = b < NB ? p.length[b] : 0;
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
  const int nqkv = (Hq + 2 * Hkv) * D;
  const AttnPlan plan = attn_plan(p, past);
  const int nrb = H / kORows;
  const int ns = n_slices(p);
  const __half* e16[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    int pos = p.position[b];
    if (pos < 0 || pos >= p.max_position) {
      if (tid == 0 && cta == 0) set_device_error(VV_ERR_RANGE);
      pos = min(max(pos, 0), p.max_position - 1);
    }
    for (int i = tid; i < D / 2; i += NT) {
      as.cs[b][i] = p.rope_cos[(size_t)pos * (D / 2) + i];
      as.sn[b][i] = p.rope_sin[(size_t)pos * (D / 2) + i];
    }
    e16[b] = p.input_embeds ? p.input_embeds + (size_t)b * H : nullptr;
    if (!e16[b]) {
      int tok = __ldcg(p.token + b);
      if (tok < 0 || tok >= p.V) {
        if (tid == 0 && cta == 0) set_device_error(VV_ERR_RANGE);
        tok = min(max(tok, 0), p.V - 1);
      }
      e16[b] = p.embed + (size_t)tok * H;
    }
  }
  auto load_emb = [&](int b, int k) -> float4 {
    const uint2 hv = __ldcg(reinterpret_cast<const uint2*>(e16[b] + k));
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&hv.x));
    const float2 c = __half22float2(*reinterpret_cast<const __half2*>(&hv.y));
    return make_float4(a.x, a.y, c.x, c.y);
  };
  auto load_x = [&](int b, int k) -> float4 {
    const unsigned long long* xb = p.x_acc + (size_t)b * H;
    const ulonglong2 a = __ldcg(reinterpret_cast<const ulonglong2*>(xb + k));
    const ulonglong2 c = __ldcg(reinterpret_cast<const ulonglong2*>(xb + k + 2));
    return make_float4(from_fix(a.x), from_fix(a.y), from_fix(c.x), from_fix(c.y));
  };
  // residual = embedding: this CTA's share of rows, before the first barrier (the o-phase adds
  // come after two more barriers)
  {
    int hr0, hr1;
    cta_range(H / 4, cta, ncta, hr0, hr1);
#pragma unroll
    for (int b = 0; b < NB; ++b)
      for (int i = hr0 + tid; i < hr1; i += NT) {
        const float4 v = load_emb(b, 4 * i);
        unsigned long long* xb = p.x_acc + (size_t)b * H + 4 * i;
        reinterpret_cast<ulonglong2*>(xb)[0] = make_ulonglong2(to_fix(v.x), to_fix(v.y));
        reinterpret_cast<ulonglong2*>(xb)[1] = make_ulonglong2(to_fix(v.z), to_fix(v.w));
      }
  }
  int o0, o1;
  cta_range(Hq * nrb, cta, ncta, o0, o1);

  for (int l = 0; l < p.L; ++l) {
    const StepLayer& w = p.layers[l];
    // ---------------------------------------------------------------- QKV
    r.ph = 0;
    int r0, r1;
    qkv_range(nqkv, cta, ncta, r0, r1);
    // this CTA's q/k/v biases (at most NT rows): the load is issued before the barrier (the
    // biases do not depend on x), the store to shared memory after it (as.q is free until the
    // attention phase; stage_idp's barriers order the stores before the GEMV reads them)
    float bias_v = 0.f;
    if (tid < r1 - r0) {
      const int bounds[4] = {0, Hq * D, (Hq + Hkv) * D, nqkv};
      const int row = r0 + tid;
      const int m = row < bounds[1] ? 0 : (row < bounds[2] ? 1 : 2);
      const __half* bp = w.bias[m];
      if (bp) bias_v = __half2float(__ldg(bp + (row - bounds[m])));
    }
    if (l > 0) grid_barrier(p, gen, sk);
    if (tid < r1 - r0) (&as.q[0][0])[tid] = bias_v;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (l == 0) {
        stage_idp(xo[b], [&](int k) { return load_emb(b, k); }, w.in_norm, p.eps, H, red, nullptr);
      } else {
        float* tr = (p.trace && cta == 0 && b == 0) ? p.trace + (size_t)(l - 1) * H : nullptr;
        stage_idp(xo[b], [&](int k) { return load_x(b, k); }, w.in_norm, p.eps, H, red, tr);
      }
    }
    stamp(p, sk);
    {
      const float* bs = &as.q[0][0] - r0;
      consume_rows<1, NB>(r, xo, H, r0, r1, [&](int row, const float* y, const float*) {
#pragma unroll
        for (int b = 0; b < NB; ++b) p.qkv[(size_t)b * nqkv + row] = y[b] + bs[row];
      });
    }
    // ---------------------------------------------------------------- ATTN
    r.ph = 1;
    grid_barrier(p, gen, sk);
    for (int it = cta; it < plan.total; it += ncta) {
      int b, g, t;
      attn_item_of(plan, Hkv, it, b, g, t);
      if (p.kv_type == 0)
        attn_item<KvF16>(p, r, as, l, b, g, t, past[b], plan.tt);
      else if (p.kv_type == 1)
        attn_item<KvBF16>(p, r, as, l, b, g, t, past[b], plan.tt);
      else
        attn_item<KvF32>(p, r, as, l, b, g, t, past[b], plan.tt);
    }
    stamp(p, sk);
    // ---------------------------------------------------------------- O
    r.ph = 2;
    grid_barrier(p, gen, sk);
    {
      int cur_h = -1;
      for (int i = o0; i < o1; ++i) {
        const int h = i / nrb, rb = i % nrb;
        if (h != cur_h) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            merge_head(p, b, h, plan.nt[b], &as.pv[0][0][0], hbuf[b]);
            const float* hb = hbuf[b];
            stage_idp(xo[b], [&](int k) { return *reinterpret_cast<const float4*>(hb + k); },
                      nullptr, 0.f, D, red, nullptr);
          }
          cur_h = h;
        }
        unsigned long long* xr = p.x_acc + (size_t)rb * kORows;
        consume_cols<NB>(r, xo, kORows, 4, [&](int row, const float* y) {
#pragma unroll
          for (int b = 0; b < NB; ++b) red_add_u64(xr + (size_t)b * H + row, to_fix(y[b]));
        });
      }
    }
    stamp(p, sk);
    // ---------------------------------------------------------------- GU + DOWN
    r.ph = 3;
    grid_barrier(p, gen, sk);
    if (nsl > 0) {
#pragma unroll
      for (int b = 0; b < NB; ++b)
        stage_idp(xo[b], [&](int k) { return load_x(b, k); }, w.post_norm, p.eps, H, red, nullptr);
      stamp(p, sk);
      int j = 0;
      for (int s = cta; s < ns; s += ncta, ++j) {
        const int off = j * kSlice - s * kSlice;
        consume_rows<2, NB>(r, xo, H, s * kSlice, (s + 1) * kSlice,
                            [&](int row, const float* g, const float* u) {
#pragma unroll
          for (int b = 0; b < NB; ++b) hbuf[b][off + row] = __fdividef(g[b], 1.f + __expf(-g[b])) * u[b];
        });
      }
      cbar();
      stamp(p, sk);
      r.ph = 4;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float* hb = hbuf[b];
        stage_idp(xo[b], [&](int k) { return *reinterpret_cast<const float4*>(hb + k); }, nullptr,
                  0.f, nsl * kSlice, red, nullptr);
      }
      stamp(p, sk);
      const int rot = wd_rot(H, cta, ncta);
      consume_cols<NB>(r, xo, H, 2 * nsl, [&](int i, const float* y) {
        const int row = i + rot < H ? i + rot : i + rot - H;
#pragma unroll
        for (int b = 0; b < NB; ++b) red_add_u64(p.x_acc + (size_t)b * H + row, to_fix(y[b]));
      });
    } else {
      stamp(p, sk);
      stamp(p, sk);
      stamp(p, sk);
    }
    stamp(p, sk);
  }
  // ------------------------------------------------------------------------------ HEAD
  r.ph = 5;
  grid_barrier(p, gen, sk);
  const int nhb = H >> 4;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    // final RMSNorm, x rounded once to fp16 in the pair layout of the fp16 head dot
    __half* xs = reinterpret_cast<__half*>(xo[b].xq);
    float* tr = (p.trace && cta == 0 && b == 0) ? p.trace + (size_t)(p.L - 1) * H : nullptr;
    float ss = 0.f;
    for (int k = tid * 4; k < H; k += NT * 4) {
      const float4 v = load_x(b, k);
      if (tr) *reinterpret_cast<float4*>(tr + k) = v;
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    cbar();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < NW; ++i) tot += red[i];
    const float inv = rsqrtf(tot / (float)H + p.eps);
    for (int k = tid * 4; k < H; k += NT * 4) {
      const float4 v = load_x(b, k);
      const float y[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        xs[xh_slot(k + e, nhb)] = __float2half_rn(y[e] * inv * __half2float(p.final_norm[k + e]));
    }
    cbar();
  }
  stamp(p, sk);
  float best[NB];
  int best_i[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    best[b] = -INFINITY;
    best_i[b] = 0x7fffffff;
  }
  {
    int r0, r1;
    cta_range(p.V, cta, ncta, r0, r1);
    const int rb = H * 2;
    const int rps = head_rows_per_stage(r.stage_bytes, rb);
    const int nch = H >> 3;  // 16-byte chunks per row
    // x of 16-byte weight chunk c (8 columns: half-block c/2, word c%2) = pair word (c%2, c/2);
    // held in registers for c = lane + 32 j when the row fits (H <= 1536) and one sequence runs
    const uint4* xs4[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) xs4[b] = reinterpret_cast<const uint4*>(xo[b].xq);
    const bool regHead = NB == 1 && nch <= 32 * 2 * kHeadRegHB;
    uint4 xr[2 * kHeadRegHB];
    if (regHead) {
#pragma unroll
      for (int j = 0; j < 2 * kHeadRegHB; ++j) {
        const int c = lane + 32 * j;
        xr[j] = c < nch ? xs4[0][(c & 1) * nhb + (c >> 1)] : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    for (int a = r0; a < r1; a += rps) {
      const int n = min(rps, r1 - a);
      int slot;
      consume_begin(r, slot);
      const unsigned char* st = r.base + (size_t)slot * r.stage_bytes;
      for (int i = warp; i < n; i += NW) {
        const unsigned char* row = st + (size_t)i * rb;
        float acc[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
        // weights (w0,w1)(w2,w3)(w4,w5)(w6,w7) against x pairs (x0,x4)(x1,x5)(x2,x6)(x3,x7)
        auto chunk = [&](const uint4 wv, auto xv_of) {
          uint32_t p04, p15, p26, p37;
          asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(p04) : "r"(wv.x), "r"(wv.z));
          asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(p15) : "r"(wv.x), "r"(wv.z));
          asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(p26) : "r"(wv.y), "r"(wv.w));
          asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(p37) : "r"(wv.y), "r"(wv.w));
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const uint4 xv = xv_of(b);
            acc[b] = fma2_f16_f32(p04, xv.x, acc[b]);
            acc[b] = fma2_f16_f32(p15, xv.y, acc[b]);
            acc[b] = fma2_f16_f32(p26, xv.z, acc[b]);
            acc[b] = fma2_f16_f32(p37, xv.w, acc[b]);
          }
        };
        if (regHead) {
#pragma unroll
          for (int j = 0; j < 2 * kHeadRegHB; ++j) {
            const int c = lane + 32 * j;
            if (c < nch) chunk(*reinterpret_cast<const uint4*>(row + c * 16), [&](int) { return xr[j]; });
          }
        } else {
          for (int c = lane; c < nch; c += 32)
            chunk(*reinterpret_cast<const uint4*>(row + c * 16),
                  [&](int b) { return xs4[b][(c & 1) * nhb + (c >> 1)]; });
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float v = warp_sum(acc[b]);
          if (lane == 0) {
            const int vr = a + i;
            if (p.logits) p.logits[(size_t)b * p.V + vr] = v;
            if (better(v, vr, best[b], best_i[b])) {
              best[b] = v;
              best_i[b] = vr;
            }
          }
        }
      }
      consume_end(r, slot);
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      s_val[b][warp] = best[b];
      s_idx[b][warp] = best_i[b];
    }
  }
  cbar();
  stamp(p, sk);
  if (tid == 0) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float bv = s_val[b][0];
      int bi = s_idx[b][0];
      for (int w2 = 1; w2 < NW; ++w2)
        if (better(s_val[b][w2], s_idx[b][w2], bv, bi)) {
          bv = s_val[b][w2];
          bi = s_idx[b][w2];
        }
      p.head_val[(size_t)b * ncta + cta] = bv;
      p.head_idx[(size_t)b * ncta + cta] = bi;
    }
    __threadfence();
    s_last = atomicAdd(p.head_count, 1) == ncta - 1;
  }
  cbar();
  if (!s_last) return;
  __threadfence();
  if (warp < NB) {  // warp b reduces sequence b
    const int b = warp;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int i = lane; i < ncta; i += 32) {
      const float v = __ldcg(p.head_val + (size_t)b * ncta + i);
      const int ix = __ldcg(p.head_idx + (size_t)b * ncta + i);
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
      p.argmax[b] = tok;
      p.length[b] = past[b] + 1;
      if (p.gen_done) {  // batch 1 only; every CTA read the position at its start
        *p.gen_count += 1;
        *p.gen_pos += 1;
        for (int j = 0; j < p.n_stop; ++j)
          if (tok == p.stop_ids[j]) *p.gen_done = 1;
      }
    }
  }
  cbar();  // warps 0..NB-1 have read the partials and the counter use is over
  if (tid == 0) {
    *p.head_count = 0;
    *p.bar_count = 0u;  // every CTA has passed every barrier of this launch
  }
}

// ------------------------------------------------------------------------ column images
// Wo (rows H, columns Hq * D): item i = (h, rb) -> rows [kORows rb, +kORows) x blocks
// [4h, 4h + 4): codes [kORows][4][16] then scales [kORows][4].
__global__ void wo_image_kernel(const uint8_t* __restrict__ q, const __half* __restrict__ s, int H,
                                int Hq, unsigned char* __restrict__ img) {
  const int KB = Hq * D / 32;
  const int nrb = H / kORows;
  const int64_t total = (int64_t)Hq * nrb * kORows * 4;  // (item, row, block) triples
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int b = (int)(t & 3);
    const int rr = (int)((t >> 2) % kORows);
    const int i = (int)((t >> 2) / kORows);
    const int h = i / nrb, rb = i % nrb;
    const int row = rb * kORows + rr, blk = 4 * h + b;
    unsigned char* it = img + (size_t)i * kORows * 4 * 18;
    reinterpret_cast<uint4*>(it)[rr * 4 + b] =
        *reinterpret_cast<const uint4*>(q + ((size_t)row * KB + blk) * 16);
    reinterpret_cast<__half*>(it + kORows * 4 * 16)[rr * 4 + b] = s[(size_t)row * KB + blk];
  }
}

// Wd (rows H, columns I): CTA c's image holds its slices c, c + grid, ... (64 columns = 2 blocks
// each): codes [H][2 nsl][16] then scales [H][2 nsl], rows rotated by wd_rot; CTA images
// `stride` bytes apart.
__global__ void wd_image_kernel(const uint8_t* __restrict__ q, const __half* __restrict__ s, int H,
                                int I, int grid, size_t stride, unsigned char* __restrict__ img) {
  const int KB = I / 32;
  const int ns = I / kSlice;
  const int64_t total = (int64_t)H * KB;  // (row, block)
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int row = (int)(t / KB), blk = (int)(t % KB);
    const int sl = blk / 2, c = sl % grid, j = sl / grid;
    const int nsl = (ns - 1 - c) / grid + 1;
    const int nb = 2 * nsl;
    const int col = 2 * j + (blk & 1);
    unsigned char* ci = img + (size_t)c * stride;
    const int rot = wd_rot(H, c, grid);
    const int pos = row >= rot ? row - rot : row - rot + H;
    reinterpret_cast<uint4*>(ci)[(size_t)pos * nb + col] =
        *reinterpret_cast<const uint4*>(q + ((size_t)row * KB + blk) * 16);
    reinterpret_cast<__half*>(ci + (size_t)H * nb * 16)[(size_t)pos * nb + col] =
        s[(size_t)row * KB + blk];
  }
}

}  // namespace

size_t step_wo_image_bytes(int H, int Hq) { return (size_t)Hq * (H / kORows) * kORows * 4 * 18; }

size_t step_wd_image_bytes(int H, int I, int grid) {
  const int ns = I / kSlice;
  const int nsl_max = (ns + grid - 1) / grid;
  return (size_t)grid * H * nsl_max * 2 * 18;
}

cudaError_t step_build_images(const StepParams& p, const StepLayer* hl, unsigned char* wo_img,
                              unsigned char* wd_img, cudaStream_t s) {
  const size_t wo_b = step_wo_image_bytes(p.H, p.Hq);
  const size_t wd_b = step_wd_image_bytes(p.H, p.I, p.grid);
  const int ns = p.I / kSlice;
  const size_t stride = (size_t)p.H * ((ns + p.grid - 1) / p.grid) * 2 * 18;
  for (int l = 0; l < p.L; ++l) {
    wo_image_kernel<<<p.grid * 4, 256, 0, s>>>(hl[l].q[3], hl[l].s[3], p.H, p.Hq,
                                               wo_img + (size_t)l * wo_b);
    wd_image_kernel<<<p.grid * 4, 256, 0, s>>>(hl[l].q[6], hl[l].s[6], p.H, p.I, p.grid, stride,
                                               wd_img + (size_t)l * wd_b);
  }
  return cudaGetLastError();
}

size_t step_smem_bytes(const StepParams& p) {
  const int maxK = std::max(p.H, p.Hq * D);
  const int nhb_max = maxK / 16;
  const int ns = p.I / kSlice;
  const int nsl_max = (ns + p.grid - 1) / p.grid;
  size_t b = (size_t)p.nstages * p.stage_bytes;
  for (int s = 0; s < std::max(p.nb, 1); ++s) {
    b += (size_t)nhb_max * 2 * 16 + (size_t)nhb_max * 4 + (size_t)nhb_max * 2;
    b += (size_t)std::max(nsl_max * kSlice, D) * 4;
    b = (b + 15) & ~size_t(15);
  }
  b += sizeof(AttnScratch) + 64 * 4 + 16 + 2 * p.nstages * 8 + 64;
  return b;
}

int step_threads() { return kThreads; }

int step_max_batch() { return kMaxB; }

size_t step_attn_part_floats(int Hkv, int max_tiles) {
  return (size_t)Hkv * max_tiles * kMaxG * kPart;
}

int step_max_tiles(int cap) { return (cap + 1 + TT / 2 - 1) / (TT / 2); }

namespace {
// The kernel instance of a batch size.
const void* step_fn(int nb) {
  return nb == 2 ? reinterpret_cast<const void*>(step_kernel<2>)
                 : reinterpret_cast<const void*>(step_kernel<1>);
}
}  // namespace

// Pick the largest stage size (>= one attention tile, 1 KB steps) for which one CTA per SM is
// resident.
cudaError_t step_configure(StepParams& p, int* blocks_per_sm) {
  const void* fn = step_fn(p.nb);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  *blocks_per_sm = 0;
  for (; p.stage_bytes >= 2 * TT * D * 2; p.stage_bytes -= 1024) {
    const size_t smem = step_smem_bytes(p);
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
      cudaGetLastError();
      continue;
    }
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (nb >= 1) {
      *blocks_per_sm = nb;
      return cudaSuccess;
    }
  }
  return cudaSuccess;
}

void step_func_info(int nb, int* regs, int* max_threads, int* static_smem, int* local_bytes) {
  cudaFuncAttributes fa = {};
  cudaFuncGetAttributes(&fa, step_fn(nb));
  *regs = fa.numRegs;
  *max_threads = fa.maxThreadsPerBlock;
  *static_smem = (int)fa.sharedSizeBytes;
  *local_bytes = (int)fa.localSizeBytes;
}

cudaError_t launch_step(const StepParams& p, cudaStream_t s) {
  const void* fn = step_fn(p.nb);
  const size_t smem = step_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  void* args[] = {const_cast<StepParams*>(&p)};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace vv
