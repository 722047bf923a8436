// MatMulNBits packing ("vibevoice-asr-bitnet-onnx": ternarisation formula and MatMulNBits
// paragraph; "VibeVoice-1.5B — Current Status", section "Done": ModelBuilder int4 build).
//
// vv_ternary_scale: s = 1 / mean|W| with an exactly computed sum.  The GPU bins |w| by fp32
// exponent and adds the 24-bit integer significands of each bin in uint64 (exact for fewer than
// 2^40 elements); the host then adds the bins as one wide integer and rounds it once to float64.
// The result is therefore the correctly rounded sum, independent of reduction order.
//
// vv_pack_nbits: one warp per 32-column block; lane i owns column 32b+i.  IEEE float32 with
// explicit round-to-nearest intrinsics (no contraction), C roundf (half away from zero).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "vv_device.cuh"
#include "vv_internal.h"

namespace vv {
namespace {

constexpr int kBins = 256;

__global__ void __launch_bounds__(256) abs_exponent_bins_kernel(const float* __restrict__ w,
                                                                int64_t count,
                                                                unsigned long long* bins,
                                                                int* nonfinite) {
  __shared__ unsigned long long sbins[kBins];
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) sbins[i] = 0ull;
  __syncthreads();
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    const uint32_t bits = __float_as_uint(w[i]) & 0x7FFFFFFFu;
    const uint32_t e = bits >> 23;
    const uint32_t m = bits & 0x7FFFFFu;
    if (e == 0xFFu) {
      atomicExch(nonfinite, 1);
      continue;
    }
    if (bits == 0) continue;
    // value = sig * 2^(max(e,1) - 150), sig < 2^24
    const uint32_t sig = (e == 0) ? m : (m | 0x800000u);
    const uint32_t bin = (e == 0) ? 1u : e;
    atomicAdd(&sbins[bin], (unsigned long long)sig);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += blockDim.x)
    if (sbins[i]) atomicAdd(&bins[i], sbins[i]);
}

// Sum_b bins[b] * 2^(b - 150) rounded once (to nearest, ties to even) to double.
double exact_bins_to_double(const unsigned long long* bins) {
  // Integer I = sum_b bins[b] << (b - 1); value = I * 2^-149.  b <= 254 -> < 2^(253 + 64).
  constexpr int kLimbs = 12;  // 384 bits
  uint32_t acc[kLimbs];
  memset(acc, 0, sizeof(acc));
  for (int b = 1; b < 255; ++b) {
    const unsigned long long v = bins[b];
    if (!v) continue;
    const int sh = b - 1;
    const int limb = sh / 32, bit = sh % 32;
    // v << bit spans up to 96 bits -> three limbs
    unsigned long long lo = (v & 0xFFFFFFFFull) << bit;
    unsigned long long hi = (v >> 32) << bit;
    uint32_t part[4] = {(uint32_t)lo, (uint32_t)(lo >> 32), 0, 0};
    unsigned long long t = (unsigned long long)part[1] + (uint32_t)hi;
    part[1] = (uint32_t)t;
    t = (t >> 32) + (hi >> 32);
    part[2] = (uint32_t)t;
    part[3] = (uint32_t)(t >> 32);
    unsigned long long carry = 0;
    for (int k = 0; k < 4 || carry; ++k) {
      if (limb + k >= kLimbs) break;
      unsigned long long s = (unsigned long long)acc[limb + k] + (k < 4 ? part[k] : 0) + carry;
      acc[limb + k] = (uint32_t)s;
      carry = s >> 32;
    }
  }
  int top = -1;
  for (int k = kLimbs - 1; k >= 0 && top < 0; --k)
    if (acc[k]) top = k * 32 + (31 - __builtin_clz(acc[k]));
  if (top < 0) return 0.0;
  auto bit_at = [&](int p) -> uint32_t { return p < 0 ? 0u : (acc[p / 32] >> (p % 32)) & 1u; };
  // mantissa = bits [top-52, top]; round bit = top-53; sticky = anything below.
  unsigned long long mant = 0;
  for (int p = top; p >= top - 52; --p) mant = (mant << 1) | bit_at(p);
  const uint32_t round_bit = bit_at(top - 53);
  bool sticky = false;
  for (int p = top - 54; p >= 0 && !sticky; --p) sticky = bit_at(p) != 0;
  int exp2 = top - 52 - 149;
  if (round_bit && (sticky || (mant & 1ull))) {
    ++mant;
    if (mant == (1ull << 53)) {
      mant >>= 1;
      ++exp2;
    }
  }
  return std::ldexp((double)mant, exp2);
}

__global__ void __launch_bounds__(256) pack_nbits_kernel(const float* __restrict__ w, int64_t N,
                                                         int64_t K, int64_t KB, int mode,
                                                         float ternary_s, uint8_t* __restrict__ q,
                                                         __half* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t nblocks = N * KB;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const bool tern_zero = !(isfinite(ternary_s) && ternary_s > 0.f);
  __half tern_scale16 = __float2half_rn(0.f);
  if (mode == VV_TERNARY && !tern_zero) tern_scale16 = __float2half_rn(__fdiv_rn(1.0f, ternary_s));

  for (int64_t blk = warp_global; blk < nblocks; blk += nwarps) {
    const int64_t n = blk / KB;
    const int64_t b = blk - n * KB;
    const int64_t col = b * 32 + lane;
    const float x = (col < K) ? w[n * K + col] : 0.f;
    int code = 8;
    __half scale16;
    if (mode == VV_TERNARY) {
      scale16 = tern_scale16;
      if (!tern_zero) {
        const float t = __fmul_rn(x, ternary_s);
        const float c = fminf(fmaxf(t, -1.0f), 1.0f);
        code = (int)roundf(c) + 8;
      }
    } else {
      const float amax = warp_max(fabsf(x));
      scale16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
      const float s = __half2float(scale16);
      if (s != 0.f) {
        float r = roundf(__fdiv_rn(x, s));
        r = fminf(fmaxf(r, -8.0f), 7.0f);
        code = (int)r + 8;
      }
    }
    if (col >= K) code = 8;
    const int partner = __shfl_down_sync(0xffffffffu, code, 1);
    if ((lane & 1) == 0) q[blk * 16 + (lane >> 1)] = (uint8_t)(code | (partner << 4));
    if (lane == 0) scales[blk] = scale16;
  }
}

}  // namespace
}  // namespace vv

extern "C" {

vv_status vv_ternary_scale(const float* w, int64_t count, float* s_out, vv_stream stream) {
  VV_CHECK_ARG(w && s_out, "vv_ternary_scale: null pointer");
  VV_CHECK_SHAPE(count >= 1 && count < (int64_t(1) << 40), "vv_ternary_scale: count %lld",
                 (long long)count);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned long long* d_bins = nullptr;
  int* d_flag = nullptr;
  VV_CUDA(cudaMallocAsync(&d_bins, vv::kBins * sizeof(unsigned long long) + 16, s));
  d_flag = reinterpret_cast<int*>(d_bins + vv::kBins);
  vv_status st = VV_OK;
  unsigned long long h_bins[vv::kBins];
  int h_flag = 0;
  do {
    st = vv::cuda_check(
        cudaMemsetAsync(d_bins, 0, vv::kBins * sizeof(unsigned long long) + 16, s), "memset");
    if (st) break;
    int grid = vv::sm_count() * 4;
    const int64_t need = (count + 255) / 256;
    if (need < grid) grid = (int)need;
    vv::abs_exponent_bins_kernel<<<grid, 256, 0, s>>>(w, count, d_bins, d_flag);
    st = vv::cuda_check(cudaGetLastError(), "abs_exponent_bins_kernel");
    if (st) break;
    st = vv::cuda_check(cudaMemcpyAsync(h_bins, d_bins, sizeof(h_bins), cudaMemcpyDeviceToHost, s),
                        "copy bins");
    if (st) break;
    st = vv::cuda_check(cudaMemcpyAsync(&h_flag, d_flag, sizeof(int), cudaMemcpyDeviceToHost, s),
                        "copy flag");
    if (st) break;
    st = vv::cuda_check(cudaStreamSynchronize(s), "sync");
  } while (0);
  cudaFreeAsync(d_bins, s);
  if (st) return st;
  if (h_flag) return vv::set_error(VV_ERR_INVALID_ARG, "vv_ternary_scale: non-finite input");
  const double total = vv::exact_bins_to_double(h_bins);
  if (total == 0.0) {
    *s_out = INFINITY;
    return VV_OK;
  }
  const double mean = total / (double)count;
  *s_out = (float)(1.0 / mean);
  return VV_OK;
}

vv_status vv_pack_nbits(const float* w, int64_t N, int64_t K, int32_t block, int32_t mode,
                        float ternary_s, uint8_t* q_out, uint16_t* scales_out, vv_stream stream) {
  VV_CHECK_ARG(w && q_out && scales_out, "vv_pack_nbits: null pointer");
  VV_CHECK_ARG(mode == VV_TERNARY || mode == VV_SYM_INT4, "vv_pack_nbits: mode %d", mode);
  VV_CHECK_SHAPE(block == 32, "vv_pack_nbits: block %d (only 32)", block);
  VV_CHECK_SHAPE(N >= 1 && K >= 1, "vv_pack_nbits: N=%lld K=%lld", (long long)N, (long long)K);
  const int64_t KB = (K + 31) / 32;
  const int64_t nblocks = N * KB;
  int64_t grid = (nblocks + 7) / 8;
  const int64_t cap = (int64_t)vv::sm_count() * 16;
  if (grid > cap) grid = cap;
  vv::pack_nbits_kernel<<<(unsigned)grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      w, N, K, KB, mode, ternary_s, q_out, reinterpret_cast<__half*>(scales_out));
  return vv::cuda_check(cudaGetLastError(), "pack_nbits_kernel");
}

}  // extern "C"
