// tcgen05 GEMM for the prefill (internal).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vv {

constexpr int kEpiBias = 0;    // out_f32[m, n] = acc + bias[n]
constexpr int kEpiResid = 1;   // out_f32[m, n] += acc
constexpr int kEpiSwiglu = 2;  // out_f16[m, n/2] = silu(acc[m, n]) * acc[m, n+1], n even
constexpr int kEpiF16 = 3;     // out_f16[m, n] = fp16(acc + bias[n])
// q/k/v with rotary embedding: y = acc + the head's bias (bias / bias_k / bias_v); the columns of
// query and key heads are rotated
// at position pos[m] (pairs d, d + D/2 of a head of D = 128); queries -> out_f16[m, n] (fp16,
// row stride ldo = hq * D), keys / values -> kc / vc [head][cap][D] at slot m (fp16)
constexpr int kEpiRope = 4;

struct GemmEpilogue {
  float* out_f32;
  __half* out_f16;
  const __half* bias;
  int ldo;  // row stride of the output in elements
  // kEpiRope only (bias = the query bias; any of the three may be null: no bias)
  const __half* bias_k;   // [hkv * D]
  const __half* bias_v;   // [hkv * D]
  const int32_t* pos;     // [M] position ids
  const float* rope_cos;  // [max_pos][D/2]
  const float* rope_sin;
  int max_pos, hq, hkv, cap;
  __half* kc;
  __half* vc;
};

size_t gemm_tc_smem();
// A: fp16 [M, K] row-major; B: fp16 [N, K] row-major; N % 128 == 0 or N % 192 == 0 (kEpiRope:
// N % 128 == 0), K % 64 == 0.
cudaError_t launch_gemm_tc(const uint16_t* A, const uint16_t* B, int M, int N, int K, int epi,
                           const GemmEpilogue& e, cudaStream_t s);

// Up to three packed MatMulNBits matrices (row segments, same K) dequantised into one fp16
// [rows, K] matrix, element (code - 8) * scale rounded once to fp16.  interleave = 1 (two
// segments of equal rows): output row 2n is row n of segment 0, row 2n + 1 row n of segment 1.
// Scales with a row pitch of K/32.
struct DequantSrc {
  const uint8_t* q[3];
  const uint16_t* s[3];
  int rows[3];
  int nseg;
  int interleave;
};
cudaError_t launch_dequant_f16(const DequantSrc& src, int total_rows, int K, __half* out,
                               cudaStream_t s);
// Up to four such matrix stacks (rows[j] x K[j] each, into out[j]) in one launch.
cudaError_t launch_dequant_many(const DequantSrc* src, const int* rows, const int* K,
                                __half* const* out, int n, cudaStream_t s);

// B operand as packed MatMulNBits matrices, dequantised inside the GEMM (no fp16 copy in global
// memory): up to three row segments (N = sum of rows, each a multiple of 128), or two segments
// of equal rows interleaved row by row (interleave = 1, N = 2 * rows).  K % 64 == 0.  Codes
// [rows, K/32, 16]; scales fp16 with a row pitch of s_pitch elements (0: K/32), a multiple of 8
// (the tensor-map row pitch must be a multiple of 16 bytes) and >= the 8-aligned block count.
struct PackedB {
  const uint8_t* q[3];
  const uint16_t* s[3];
  int rows[3];
  int nseg;
  int interleave;
  int s_pitch;
};
bool gemm_q4_supported(const PackedB& B, int N, int K);
cudaError_t launch_gemm_q4(const uint16_t* A, const PackedB& B, int M, int N, int K, int epi,
                           const GemmEpilogue& e, cudaStream_t s);

}  // namespace vv
