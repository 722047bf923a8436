/*
 * libvv — int4 blockwise-quantised Qwen2 decoder step on NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes only.  "device" pointers are CUDA global-memory addresses on
 * the current device; "host" pointers are ordinary CPU memory.  Half-precision values are passed
 * as uint16_t bit patterns (IEEE binary16).  A stream argument is a cudaStream_t passed as
 * void* (NULL = the legacy default stream).  Calls are asynchronous on that stream unless
 * stated otherwise.
 *
 * Ownership: the caller allocates and owns every input, output, weight and KV-cache buffer;
 * libvv borrows them for the duration of a call (or, for vv_decoder_create, for the decoder's
 * lifetime) and never frees them.  libvv owns only the workspace a decoder allocates in
 * vv_decoder_create and frees in vv_decoder_destroy.
 *
 * Errors: every call returns vv_status (VV_OK = 0).  No exception crosses the ABI.
 * vv_last_error() returns the text of the calling thread's most recent error.  Errors found on
 * the device (a wait that timed out, a token id out of range) are recorded in a device error
 * word and reported by vv_sync_status() / vv_decoder_sync_status().
 *
 * Sources of the operations (web pages on the VibeVoice ONNX exports):
 *   [BITNET]  "vibevoice-asr-bitnet-onnx" model page (Masterx): ternarisation formula,
 *             MatMulNBits packing paragraph, tier table, decoder_init / decoder_step I/O listing.
 *   [STATUS]  "VibeVoice-1.5B — Current Status" (Prince-1/VibeVoice-1.5B-Onnx): sections
 *             "Architecture", "Done" (140 MatMulNBits + 28 GroupQueryAttention, int4 ModelBuilder
 *             build) and "Inference (ONNX)" (KV-incremental decode loop, tied lm_head).
 *   [ASR]     "VibeVoice-ASR — ONNX export for Vernacula": section "Highlights" (GPU-resident KV
 *             cache, 1950 launches per step of framework overhead).
 */
#ifndef VV_H_
#define VV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t vv_status;

#define VV_OK 0
#define VV_ERR_INVALID_ARG 1 /* null / misaligned pointer, bad enum value */
#define VV_ERR_SHAPE 2       /* inconsistent or unsupported sizes */
#define VV_ERR_CAPACITY 3    /* KV cache or workspace too small */
#define VV_ERR_RANGE 4       /* index out of range (audio splice, position, token id) */
#define VV_ERR_CUDA 5        /* a CUDA runtime call failed; text in vv_last_error */
#define VV_ERR_TIMEOUT 6     /* a bounded device-side wait expired */

/* Quantisation modes of vv_pack_nbits. */
#define VV_SYM_INT4 0 /* scale = max|w_block| / 7 */
#define VV_TERNARY 1  /* BitNet ternary with a per-tensor scale s */

typedef void* vv_stream; /* cudaStream_t */

/* Library version string (static storage). */
const char* vv_version(void);

/* Copy the calling thread's last error text into buf (NUL-terminated, truncated to n).
 * Returns the last error code. */
vv_status vv_last_error(char* buf, size_t n);

/* Synchronise `stream` and return (and clear) the device error word of the current device.
 * While the word holds VV_ERR_TIMEOUT, every bounded wait of later kernels gives up at once (a
 * kernel whose schedule went wrong ends quickly); clear it with this call. */
vv_status vv_sync_status(vv_stream stream);

/* Self-test of the bounded device waits (no counterpart in the pages: a property of this
 * library).  Launches one CTA on `stream` that waits, through the same helpers the kernels use,
 * for a signal that never comes -- which = 0: an mbarrier phase nobody completes (the stage-ring
 * wait); which = 1: a global counter nobody increments (the grid-barrier wait; scratch: device,
 * 16 bytes, 16-byte aligned, zeroed by the call) -- and gives up after limit_ns, recording
 * VV_ERR_TIMEOUT in the device error word, which the next vv_sync_status returns.  The kernel
 * then exits normally; the context stays usable.  limit_ns in [1e3, 1e8].
 * Errors: VV_ERR_INVALID_ARG. */
vv_status vv_wait_selftest(int32_t which, int64_t limit_ns, void* scratch, vv_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Packing ([BITNET] ternarisation and MatMulNBits paragraphs; [STATUS] "Done": int4 build).
 *
 * Layout produced (the public ONNX Runtime MatMulNBits layout, bits = 4, block = 32):
 *   q_out      device uint8  [N, KB, 16], KB = ceil(K / 32).  Block b of row n holds columns
 *              32b .. 32b+31; byte j holds column 32b+2j in its low nibble and 32b+2j+1 in its
 *              high nibble.  Stored code = round(w / scale) + 8 (implicit zero point 8).
 *   scales_out device fp16   [N, KB].
 * Dequantised weight = (code - 8) * scale.  Columns past K are padded with code 8.
 */

/* Per-tensor ternary scale s = 1 / mean(|W|) ([BITNET] ternarisation formula).
 * w: device fp32 [count].  s_out: HOST float.  mean is the correctly rounded float64 sum of
 * |w| divided by count (float64), s = float32(1.0 / mean); a zero tensor gives s = +inf.
 * Synchronous: returns after the value is on the host.  count in [1, 2^40). */
vv_status vv_ternary_scale(const float* w, int64_t count, float* s_out, vv_stream stream);

/* Quantise and pack W [N, K] (device fp32, row-major).
 *   mode VV_TERNARY:  code = round(clamp(float32(w * s), -1, 1)) + 8 in {7, 8, 9};
 *                     every block's scale = fp16(float32(1 / s)); s = ternary_s (from
 *                     vv_ternary_scale); s not finite or <= 0 -> all codes 8, scale 0.
 *   mode VV_SYM_INT4: scale = fp16(float32(max|w_block|) / 7);
 *                     code = clamp(round(float32(w / scale)), -8, 7) + 8; zero scale -> codes 8.
 * round() is half away from zero; all arithmetic is IEEE float32 without contraction, so the
 * result is bit-reproducible.  block must be 32.  Inputs must be finite.
 * Errors: VV_ERR_INVALID_ARG (null, mode), VV_ERR_SHAPE (N, K < 1, block != 32). */
vv_status vv_pack_nbits(const float* w, int64_t N, int64_t K, int32_t block, int32_t mode,
                        float ternary_s, uint8_t* q_out, uint16_t* scales_out,
                        vv_stream stream);

/* ---------------------------------------------------------------------------------------------
 * MatMulNBits ([STATUS] "Done": com.microsoft::MatMulNBits, 5 per layer).
 *   y[m, n] = sum_k x[m, k] * (code[n, k] - 8) * scale[n, k / 32]  (+ bias[n])
 * x device fp16 [M, K]; q/scales as produced by vv_pack_nbits for [N, K]; bias device fp16 [N]
 * or NULL; y device fp16 [M, N].  One launch, no scratch:
 *   1 <= M <= 8: dequant-fused GEMV (each weight byte read once for all M rows); products and
 *                sums in fp32, one rounding to fp16 at the end.  K % 32 == 0.
 *   M > 8:       tcgen05 tensor-core GEMM; the int4 codes are expanded inside the kernel, in
 *                shared memory, to the fp16 operand fp16((code - 8) * scale) (rounded once:
 *                exact for ternary weights, within 2^-12 relative for int4) and multiplied with
 *                fp32 accumulation in tensor memory (the prefill's projections, [BITNET]
 *                decoder_init contract).  N % 128 == 0, K % 256 == 0, M < 2^24.
 * Requirements: block == 32, all pointers 16-byte aligned.
 * Errors: VV_ERR_INVALID_ARG, VV_ERR_SHAPE (K % 32, N < 1, the M > 8 shape rules). */
vv_status vv_matmul_nbits(const uint16_t* x, const uint8_t* q, const uint16_t* scales,
                          const uint16_t* bias, int64_t M, int64_t N, int64_t K, int32_t block,
                          uint16_t* y, vv_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Grouped-query decode attention ([STATUS] "Done": com.microsoft::GroupQueryAttention, one per
 * layer; [BITNET] decoder_step: past keys/values [L, 1, Hkv, P, D]).
 *   out[h, :] = softmax(scale * q[h, :] . K[g, t, :] for t < len) . V[g, :, :],  g = h / (Hq/Hkv)
 * q device fp16 [Hq, D] (already rotated); k_cache / v_cache device fp16 [Hkv, cap, D]
 * (positions 0..len-1 valid, stride cap); out device fp16 [Hq, D].  All positions < len are
 * visible (decoder_step has no mask input).  Softmax and accumulation in fp32.
 * ws: device workspace of at least vv_gqa_decode_attn_workspace_size(Hq, Hkv, D, cap) bytes,
 * zero-filled once before its first use; every call leaves its counters at zero again.  Calls
 * sharing one ws must not overlap on the GPU.
 * Requirements: D == 128, 1 <= Hkv <= 64, Hq % Hkv == 0, Hq / Hkv <= 8, 1 <= len <= cap.
 * Errors: VV_ERR_INVALID_ARG, VV_ERR_SHAPE, VV_ERR_CAPACITY (ws too small). */
size_t vv_gqa_decode_attn_workspace_size(int32_t Hq, int32_t Hkv, int32_t D, int32_t cap);
vv_status vv_gqa_decode_attn(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                             int32_t len, int32_t cap, int32_t Hq, int32_t Hkv, int32_t D,
                             float scale, uint16_t* out, void* ws, size_t ws_bytes,
                             vv_stream stream);

/* Same operation, arguments and requirements as vv_gqa_decode_attn, for callers that cannot
 * allocate device memory when they run attention (an application that has given its whole GPU
 * memory budget to its own pool, a real-time audio thread that may not call cudaMalloc because it
 * can block and synchronise the device, a plugin that may not own allocations).  No workspace
 * argument: the scratch (split-K partials and arrival counters) is a file-scope device array of
 * 256 KiB that every GPU loading this library holds until the process exits.  No counterpart in
 * the pages: this is a property of this library, not of the method.
 *  - The first call on a device looks up the array's device address with that device current;
 *    make that first call before any stream capture.  `stream` must belong to the current device
 *    (VV_ERR_INVALID_ARG otherwise: the array's address differs per device).
 *  - The call allocates nothing (no cudaMalloc/cudaFree); it clears the arrival counters with
 *    cudaMemsetAsync on `stream` and then launches the kernel.
 *  - All calls share the one array, which keeps the previous call's partials: calls that overlap
 *    on the GPU (different streams without ordering) race and corrupt each other's results.
 *  - Errors: as vv_gqa_decode_attn, plus VV_ERR_CAPACITY when the shape needs more scratch than
 *    the array holds: Hkv x chunks x 8 x 132 floats + 256 bytes must fit in 256 KiB, i.e.
 *    Hkv x chunks <= 62 (chunks = min(ceil(cap/64), SMs/Hkv)); with 2 KV heads that is a cache of
 *    up to 1984 positions, with 4 KV heads up to 960. */
vv_status vv_gqa_decode_attn_noalloc(const uint16_t* q, const uint16_t* k_cache,
                                     const uint16_t* v_cache, int32_t len, int32_t cap, int32_t Hq,
                                     int32_t Hkv, int32_t D, float scale, uint16_t* out,
                                     vv_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Final RMSNorm + fp16 lm_head + greedy argmax ([BITNET]: lm_head stays fp16, greedy decode;
 * [STATUS] "Inference (ONNX)": logits = hidden . embed^T with the tied table).
 *   xn = x / sqrt(mean(x^2) + eps) * gamma;  logits[v] = sum_h w_lm[v, h] * xn[h]  (fp32)
 *   idx = argmax_v logits[v], lowest index on ties.
 * x device fp32 [H] (the residual before the final norm); gamma device fp16 [H]; w_lm device
 * fp16 [V, H]; logits device fp32 [V] or NULL; idx device int32 [1].
 * ws: device workspace of vv_lm_head_argmax_workspace_size(V) bytes, zero-filled once before
 * its first use (left zeroed by every call).  Requirements: H % 64 == 0, 64 <= H <= 16384.
 * Errors: VV_ERR_INVALID_ARG, VV_ERR_SHAPE, VV_ERR_CAPACITY. */
size_t vv_lm_head_argmax_workspace_size(int64_t V);
vv_status vv_lm_head_argmax(const float* x, const uint16_t* gamma, const uint16_t* w_lm,
                            int64_t V, int64_t H, float eps, float* logits, int32_t* idx,
                            void* ws, size_t ws_bytes, vv_stream stream);

/* ---------------------------------------------------------------------------------------------
 * Decoder ([BITNET] decoder_init / decoder_step contracts; [ASR] "Highlights": KV cache kept
 * resident on the GPU, step replayed as one CUDA graph instead of ~1950 launches).
 *
 * The KV cache is the caller's: k_cache and v_cache are device [L, 1, Hkv, cap, D] each, of the
 * storage type cfg.kv_dtype: fp16 (VV_KV_F16, the contract's type), or the variants bf16
 * (VV_KV_BF16) and fp32 (VV_KV_F32) ("VibeVoice-ASR — ONNX export for Vernacula", Highlights:
 * an fp32 cache against fp16 drift).  The pointers are passed as uint16_t* whatever the type.
 * "past K/V in, present K/V out" happens in place: after a call, positions 0..length-1 of the
 * cache are the present keys/values (viewed [L, 1, Hkv, length, D] with stride cap).
 * Keys are stored after RoPE.
 */
typedef struct vv_config {
  int32_t hidden;      /* H  (1536 for the 1.5B backbone, 3584 for 7B) */
  int32_t layers;      /* L  (28) */
  int32_t n_q;         /* query heads  (12 / 28) */
  int32_t n_kv;        /* key-value heads (2 / 4) */
  int32_t head_dim;    /* D  (128; the only supported value) */
  int32_t inter;       /* SwiGLU intermediate (8960 / 18944) */
  int32_t vocab;       /* V  (151936 / 152064) */
  float eps;           /* RMSNorm epsilon (1e-6) */
  float rope_theta;    /* RoPE base (1e6) */
  int32_t kv_capacity; /* cap: slots per layer and head in the caller's cache */
  int32_t max_position;/* RoPE table length: position ids must lie in [0, max_position) */
  int32_t max_prefill; /* largest S accepted by vv_decoder_init (0 = no prefill workspace) */
  int32_t kv_dtype;    /* VV_KV_F16 (0), VV_KV_BF16 (1) or VV_KV_F32 (2); the prefill needs F16 */
  int32_t batch;       /* sequences stepped together, 1 or 2 (0 means 1); batch 2 is the
                          CFG pair / two streams ("VibeVoice-1.5B — Current Status": the
                          negative context stepped alongside the positive one); each sequence
                          is prefilled by vv_decoder_init_seq */
} vv_config;

#define VV_KV_F16 0
#define VV_KV_BF16 1
#define VV_KV_F32 2

typedef struct vv_packed_matrix {
  const uint8_t* q;       /* device uint8 [N, K/32, 16] */
  const uint16_t* scales; /* device fp16 [N, K/32] */
} vv_packed_matrix;

typedef struct vv_layer_weights {
  const uint16_t* input_norm; /* fp16 [H]   RMSNorm before attention */
  const uint16_t* post_norm;  /* fp16 [H]   RMSNorm before the MLP */
  vv_packed_matrix wq;        /* [Hq*D, H] */
  vv_packed_matrix wk;        /* [Hkv*D, H] */
  vv_packed_matrix wv;        /* [Hkv*D, H] */
  vv_packed_matrix wo;        /* [H, Hq*D] */
  vv_packed_matrix wgate;     /* [I, H] */
  vv_packed_matrix wup;       /* [I, H] */
  vv_packed_matrix wdown;     /* [H, I] */
  const uint16_t* bq;         /* fp16 [Hq*D]  (q/k/v carry biases in Qwen2) */
  const uint16_t* bk;         /* fp16 [Hkv*D] */
  const uint16_t* bv;         /* fp16 [Hkv*D] */
} vv_layer_weights;

typedef struct vv_model_weights {
  const uint16_t* embed;          /* device fp16 [V, H] token embedding table */
  const uint16_t* lm_head;        /* device fp16 [V, H]; equal to embed when tied */
  const uint16_t* final_norm;     /* device fp16 [H] */
  const vv_layer_weights* layers; /* HOST array of L entries, copied by vv_decoder_create */
} vv_model_weights;

typedef struct vv_decoder vv_decoder;

/* Create a decoder on the current device.  All weight pointers are borrowed for the decoder's
 * lifetime; k_cache/v_cache likewise.  Allocates the decoder's workspace.  Length starts at 0.
 * Requirements: head_dim == 128, n_kv <= 64, n_q % n_kv == 0, n_q/n_kv <= 8, hidden a multiple
 * of 128 (<= 7680; 896 for the Realtime-0.5B backbone), inter a multiple of 256 (<= 65536),
 * n_q * head_dim <= 7680, 1 <= kv_capacity, 1 <= max_position; every device pointer (caches,
 * tables, packed matrices, norm gains, biases) 16-byte aligned.  With max_prefill > 0, the
 * scales of matrices whose K / 32 is not a multiple of 8 are copied once with a padded row
 * pitch for the prefill GEMMs (the decoder owns the copy).
 * Errors: VV_ERR_INVALID_ARG, VV_ERR_SHAPE, VV_ERR_CUDA (allocation). */
vv_status vv_decoder_create(const vv_config* cfg, const vv_model_weights* weights,
                            uint16_t* k_cache, uint16_t* v_cache, vv_decoder** out);
vv_status vv_decoder_destroy(vv_decoder* dec);

/* Set the number of valid cache positions (rewind / reset / adopt a cache filled elsewhere) of
 * every sequence.  Enqueued on `stream`.  Errors: VV_ERR_CAPACITY if len > kv_capacity,
 * VV_ERR_RANGE if < 0. */
vv_status vv_decoder_set_length(vv_decoder* dec, int32_t len, vv_stream stream);
/* The same per sequence: lens is a HOST int32 array of `batch` lengths. */
vv_status vv_decoder_set_lengths(vv_decoder* dec, const int32_t* lens, vv_stream stream);
/* Length of sequence 0 / of sequence `seq` (-1 for a bad handle or index); the batch size. */
int32_t vv_decoder_length(const vv_decoder* dec);
int32_t vv_decoder_sequence_length(const vv_decoder* dec, int32_t seq);
int32_t vv_decoder_batch(const vv_decoder* dec);

/* One decode step (decoder_step) of the decoder's B = batch sequences; every weight byte is
 * read once for all of them.  Arrays are sequence-major:
 *   input_embeds: device fp16 [B, H], or NULL to gather rows token_id[b] of the embedding table
 *   token_id:     device int32 [B] (used only when input_embeds is NULL)
 *   position_id:  device int32 [B]; RoPE angle = position * theta^(-2i/D)
 *   logits:       device fp32 [B, V] or NULL
 *   argmax_out:   device int32 [B] or NULL (greedy token, lowest index on ties)
 * Sequence b reads and appends cache [L, b, Hkv, ·, D] (the caches are [L, B, Hkv, cap, D]):
 * its K/V go to slot length_b of every layer, then length_b += 1.  The first
 * call with a given set of pointers captures the step as a CUDA graph; later calls replay it.
 * Errors: VV_ERR_INVALID_ARG, VV_ERR_CAPACITY (length == kv_capacity).  A position outside
 * [0, max_position) or a token outside [0, V) is reported by vv_decoder_sync_status. */
vv_status vv_decoder_step(vv_decoder* dec, const uint16_t* input_embeds, const int32_t* token_id,
                          const int32_t* position_id, float* logits, int32_t* argmax_out,
                          vv_stream stream);

/* Prefill (decoder_init): embeds = embed[input_ids]; rows [audio_offset, audio_offset + N) are
 * replaced by audio_features; causal attention over the S positions; writes present K/V at
 * slots 0..S-1, sets length = S, and emits the last position's logits / argmax.
 *   input_ids, position_ids: device int32 [S]; audio_features: device fp16 [N, H] or NULL (N=0)
 * All S positions go through tensor-core GEMMs at once (each packed matrix is dequantised to an
 * fp16 operand, rounded once: exact for ternary weights, within 2^-12 relative for int4; for
 * S <= 256 inside the GEMM, for longer prompts one launch per layer into a one-layer fp16 buffer
 * of the prefill workspace), with
 * fp32 accumulation and an fp32 residual.  The first call allocates a prefill workspace sized
 * for max_prefill (kept until vv_decoder_destroy).  Asynchronous on `stream`.
 * Errors: VV_ERR_RANGE (audio_offset + N > S, negative offset), VV_ERR_CAPACITY (S > cap or
 * S > max_prefill), VV_ERR_INVALID_ARG. */
vv_status vv_decoder_init(vv_decoder* dec, const int32_t* input_ids, const int32_t* position_ids,
                          int64_t S, const uint16_t* audio_features, int64_t N,
                          int64_t audio_offset, float* logits, int32_t* argmax_out,
                          vv_stream stream);

/* vv_decoder_init for sequence `seq` of a batch decoder (vv_decoder_init is seq = 0): the
 * prompt's K/V go to cache slice [L, seq, Hkv, ·, D] and only that sequence's length is set.
 * Errors as vv_decoder_init, and VV_ERR_INVALID_ARG for seq outside [0, batch). */
vv_status vv_decoder_init_seq(vv_decoder* dec, int32_t seq, const int32_t* input_ids,
                              const int32_t* position_ids, int64_t S,
                              const uint16_t* audio_features, int64_t N, int64_t audio_offset,
                              float* logits, int32_t* argmax_out, vv_stream stream);

/* Debug tap: when layer_out (device fp32 [L, H]) is non-NULL, each later step writes the
 * residual stream after every layer into it (init writes the last position's).  NULL turns it
 * off.  Changing it re-captures the step graph. */
vv_status vv_decoder_set_trace(vv_decoder* dec, float* layer_out);

/* Bound of every device-side wait of the step kernel (grid barriers, the stage ring), in ns;
 * default 2e9.  A wait that runs out records VV_ERR_TIMEOUT (reported by
 * vv_decoder_sync_status) and lets the kernel finish; once one wait has timed out, all others
 * give up at once.  limit_ns in [1e5, 1e10].  Errors: VV_ERR_INVALID_ARG. */
vv_status vv_decoder_set_wait_limit(vv_decoder* dec, int64_t limit_ns);

/* Turn CUDA-graph replay of the step on (default) or off (plain launches every call). */
vv_status vv_decoder_set_graph(vv_decoder* dec, int32_t enable);

/* Synchronise `stream` and return (and clear) the device error word. */
vv_status vv_decoder_sync_status(vv_decoder* dec, vv_stream stream);

/* Greedy generation on the device ("vibevoice-asr-bitnet-onnx": the driver's greedy decode
 * with stop tokens): up to n_steps decode steps, the token of step i being the argmax of step
 * i - 1 (step 0: *first_token), positions *position, *position + 1, ...; each step appends to
 * the KV cache like vv_decoder_step.  A step whose argmax is one of stop_ids (HOST array of
 * n_stop <= 8 ids, e.g. 151645 and 151643) ends the generation: the remaining launches return
 * at once.  first_token, position: device int32 [1]; tokens_out: device int32 [n_steps], entry i
 * = argmax of step i (entries past the stop are untouched); n_out: HOST int32, the number of
 * steps run (the stop token included).  Needs the persistent step kernel.  Synchronous: one host
 * synchronisation for the whole generation.  Batch 1 only.
 * Errors: VV_ERR_INVALID_ARG, VV_ERR_SHAPE (n_steps < 1, batch > 1), VV_ERR_CAPACITY (length + n_steps >
 * capacity); a device-side error recorded during the generation (VV_ERR_RANGE for a token or
 * position out of range, VV_ERR_TIMEOUT) is returned by this call itself (and cleared), with
 * *n_out still set. */
vv_status vv_decoder_generate(vv_decoder* dec, const int32_t* first_token, const int32_t* position,
                              int32_t n_steps, const int32_t* stop_ids, int32_t n_stop,
                              int32_t* tokens_out, int32_t* n_out, vv_stream stream);

/* Profiling variant of vv_decoder_init: the same prefill (same arguments, same results and
 * cache contents), with a CUDA event recorded after every launch.  Synchronous.  phase_ms: HOST
 * float [5] and launches: HOST int32 [5] receive the device time and the number of launches (or
 * copies) of each kind: [0] embedding splice, RMSNorm, RoPE/KV write, bias and trace copies;
 * [1] weight dequantisation to fp16; [2] tensor-core GEMMs; [3] causal attention; [4] final
 * norm + lm_head + argmax.  Prompts of S <= 256 positions run the GEMMs with the int4 → fp16
 * expansion fused in (kind [1] stays 0); longer prompts dequantise each layer's four weight
 * stacks in one launch into an fp16 buffer (kind [1]) and run fp16 GEMMs on it.  Errors as
 * vv_decoder_init. */
vv_status vv_decoder_profile_init(vv_decoder* dec, const int32_t* input_ids,
                                  const int32_t* position_ids, int64_t S,
                                  const uint16_t* audio_features, int64_t N, int64_t audio_offset,
                                  float* logits, int32_t* argmax_out, float* phase_ms,
                                  int32_t* launches, vv_stream stream);

/* Timeline tap of the persistent step kernel: runs one step (appending a position like
 * vv_decoder_step, without graph capture) with every CTA recording the device clock
 * (%globaltimer, ns) at fixed points of its schedule: kernel start; for each layer (layers > 0
 * first: barrier arrive / exit before q/k/v) x staged for q/k/v, arrive / exit / done of the
 * attention phase, arrive / exit / done of the o-projection, arrive / exit of the gate/up +
 * down phase, x staged, gate/up done, h staged, layer end (15 stamps per layer, 13 for layer
 * 0); then arrive / exit / x staged of the lm_head and the end.  stamps: HOST uint64
 * [grid * max_per_cta]; *grid_out and *per_cta_out receive the CTA count and the number of
 * stamps each CTA wrote.  The last 8 entries of each CTA's row are not stamps: compute thread
 * 0's time blocked on the stage ring per phase kind (QKV, attention, o-proj, gate/up, down,
 * lm_head; ns), then the producer's finishing time and its time blocked on free slots.
 * Synchronous.  VV_ERR_CAPACITY when max_per_cta < 15 L + 11. */
vv_status vv_decoder_step_timeline(vv_decoder* dec, const uint16_t* input_embeds,
                                   const int32_t* token_id, const int32_t* position_id,
                                   uint64_t* stamps, int32_t max_per_cta, int32_t* grid_out,
                                   int32_t* per_cta_out, vv_stream stream);

/* Number of kernel launches one vv_decoder_step enqueues (for launch accounting): 1 (the
 * persistent step kernel). */
int32_t vv_decoder_step_launches(const vv_decoder* dec);

#ifdef __cplusplus
}
#endif

#endif /* VV_H_ */
