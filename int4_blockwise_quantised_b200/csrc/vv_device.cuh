// Device-side helpers shared by the libvv kernels (sm_100a only).
//
// Bounded waits: every spin on an mbarrier or a flag gives up after a time limit, records
// VV_ERR_TIMEOUT in the library's device error word and lets the thread carry on, so a kernel
// never hangs the GPU; the host reads the word through vv_sync_status().
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/vv.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libvv targets sm_100a only"
#endif

namespace vv {

// Library-wide device error word (first error wins); defined in abi.cu.
extern __device__ int g_device_error;

__device__ __forceinline__ void set_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Default limit for any single wait: far above any legitimate wait inside one kernel.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// A wait gives up once its own limit has passed, or as soon as another wait anywhere on the
// device has already timed out (so a kernel whose schedule went wrong finishes quickly instead
// of letting every later wait run out its own limit).
__device__ __forceinline__ bool wait_expired(uint64_t t0, uint64_t limit_ns) {
  if (globaltimer_ns() - t0 > limit_ns) return true;
  return *reinterpret_cast<volatile int*>(&g_device_error) == VV_ERR_TIMEOUT;
}

// ----------------------------------------------------------------------------------------------
// Programmatic dependent launch (PDL).  griddepcontrol.wait blocks until the preceding kernel in
// the stream has completed and its memory is visible; it is a no-op when the kernel was not
// launched with the programmatic-serialization attribute.  launch_dependents lets the next
// kernel start its independent prologue (weight prefetch) early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ----------------------------------------------------------------------------------------------
// mbarrier + bulk async copy (TMA, non-tensor form, into this CTA's shared memory).
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the phase completes or
// about `hint_ns` pass, instead of spinning through issue slots.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; gives up after limit_ns (default
// kWaitLimitNs), records VV_ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_hint(bar, parity, 20000u)) {
    if (wait_expired(t0, limit_ns)) {
      set_device_error(VV_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait until the global counter *p reaches `target` (acquire); gives up after limit_ns, records
// VV_ERR_TIMEOUT and returns false.  The grid barriers of the step kernel wait through this.
__device__ __forceinline__ bool wait_counter_geq(const unsigned* p, unsigned target,
                                                 uint64_t limit_ns = kWaitLimitNs) {
  if (ld_acquire_u32(p) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_u32(p) < target) {
    if (wait_expired(t0, limit_ns)) {
      set_device_error(VV_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Bulk copy global -> shared::cta, completion signalled on `bar` (complete_tx bytes).
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 eviction-first hint for data streamed exactly once (weights).
__device__ __forceinline__ void bulk_g2s_stream(void* dst_smem, const void* src_gmem,
                                                uint32_t bytes, uint64_t* bar,
                                                uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], "
      "%2, [%3], %4;" ::"r"(smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ----------------------------------------------------------------------------------------------
// Reductions.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ----------------------------------------------------------------------------------------------
// int4 dequant-dot of one 32-bit word of MatMulNBits codes.
//
// Word bytes j = 0..3 hold elements 2j (low nibble) and 2j+1 (high nibble).  Each byte is moved
// into the low mantissa bits of the float 2^23 (byte_perm with 0x4B000000), which gives
// 2^23 + c exactly; the low nibbles are masked to c, the high ones to 16c.  One packed
// add/fma then yields (c - 8) exactly, and the products with x accumulate in fp32.
// x8e = (x0, x2, x4, x6), x8o = (x1, x3, x5, x7) of the word's 8 columns.
__device__ __forceinline__ float2 dot8_nbits(uint32_t w, float4 x8e, float4 x8o, float2 acc) {
  const uint32_t lo = w & 0x0F0F0F0Fu;
  const uint32_t hi = w & 0xF0F0F0F0u;
  const uint32_t M = 0x4B000000u;
  float2 l01 = make_float2(__uint_as_float(__byte_perm(lo, M, 0x7440)),
                           __uint_as_float(__byte_perm(lo, M, 0x7441)));
  float2 l23 = make_float2(__uint_as_float(__byte_perm(lo, M, 0x7442)),
                           __uint_as_float(__byte_perm(lo, M, 0x7443)));
  float2 h01 = make_float2(__uint_as_float(__byte_perm(hi, M, 0x7440)),
                           __uint_as_float(__byte_perm(hi, M, 0x7441)));
  float2 h23 = make_float2(__uint_as_float(__byte_perm(hi, M, 0x7442)),
                           __uint_as_float(__byte_perm(hi, M, 0x7443)));
  const float2 bias_lo = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
  const float2 sixteenth = make_float2(0.0625f, 0.0625f);
  const float2 bias_hi = make_float2(-524296.0f, -524296.0f);    // -(2^19 + 8)
  l01 = __fadd2_rn(l01, bias_lo);
  l23 = __fadd2_rn(l23, bias_lo);
  h01 = __ffma2_rn(h01, sixteenth, bias_hi);
  h23 = __ffma2_rn(h23, sixteenth, bias_hi);
  acc = __ffma2_rn(l01, make_float2(x8e.x, x8e.y), acc);
  acc = __ffma2_rn(l23, make_float2(x8e.z, x8e.w), acc);
  acc = __ffma2_rn(h01, make_float2(x8o.x, x8o.y), acc);
  acc = __ffma2_rn(h23, make_float2(x8o.z, x8o.w), acc);
  return acc;
}

// ----------------------------------------------------------------------------------------------
// int4 dequant-dot, half2 form.  One 32-bit word of codes (elements 0..7) is unpacked with the
// 0x6400 (= 1024.0 in fp16) magic: lop3 places nibble pairs (0,4), (1,5), (2,6), (3,7) into the
// mantissas of two fp16 lanes, then one packed add/fma removes the bias, which yields the exact
// values (code - 8) in fp16.  Products with fp16 activations are formed by the mixed-precision
// fma.rn.f32.f16 (both factors fp16, exact product, fp32 accumulate), so nothing is rounded but
// the fp32 sums.  x8 holds the activations as half2 pairs (x0,x4), (x1,x5), (x2,x6), (x3,x7).
__device__ __forceinline__ void unpack8_h2(uint32_t w, uint32_t (&d)[4]) {
  const uint32_t w8 = w >> 8;
  uint32_t h0, h1, h2, h3;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h0) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h1) : "r"(w), "r"(0x00F000F0u), "r"(0x64006400u));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h2) : "r"(w8), "r"(0x000F000Fu), "r"(0x64006400u));
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h3) : "r"(w8), "r"(0x00F000F0u), "r"(0x64006400u));
  // (1024 + c) - 1032 = c - 8;  (1024 + 16c) / 16 - 72 = c - 8   (all exact in fp16)
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d[0]) : "r"(h0), "r"(0x64086408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d[1]) : "r"(h1), "r"(0x2C002C00u), "r"(0xD480D480u));
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d[2]) : "r"(h2), "r"(0x64086408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d[3]) : "r"(h3), "r"(0x2C002C00u), "r"(0xD480D480u));
}

// acc += a.lo * b.lo + a.hi * b.hi with fp16 factors and an fp32 accumulator.
__device__ __forceinline__ float fma2_f16_f32(uint32_t a, uint32_t b, float acc) {
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(b));
  return acc;
}

// Exact sum over one word: sum_i (code_i - 8) * x_i in fp32.
__device__ __forceinline__ float dot8_h(uint32_t w, uint4 x8) {
  uint32_t d[4];
  unpack8_h2(w, d);
  float acc = 0.f;
  acc = fma2_f16_f32(d[0], x8.x, acc);
  acc = fma2_f16_f32(d[1], x8.y, acc);
  acc = fma2_f16_f32(d[2], x8.z, acc);
  acc = fma2_f16_f32(d[3], x8.w, acc);
  return acc;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

}  // namespace vv
