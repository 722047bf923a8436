"""Oracle: the per-step operators of the Qwen2 decoder, in float64 (test infrastructure only).

Each function is the plain definition of the operation; numpy ``matmul``/``einsum``/``exp`` are
the only library steps.  Sources: the Qwen2 backbone ("VibeVoice-1.5B — Current Status",
section "Architecture": q/k/v with bias, 12 query / 2 key-value heads, tied embeddings), the
Liger fusions that name RoPE, RMSNorm and SwiGLU for Qwen2 ("VibeVoice Administrator &
Developer Guide", section 9.7) and the MatMulNBits / GroupQueryAttention graph ops
("VibeVoice-1.5B — Current Status", section "Done").
"""

import numpy as np

from . import pack as _pack


def rmsnorm(x, gamma, eps):
    """y = x / sqrt(mean(x^2) + eps) * gamma over the last axis (float64)."""
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(gamma).astype(np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * g


def rope_inv_freq(head_dim, theta):
    """inv_freq_i = theta^(-2i/D), i = 0 .. D/2-1 (HF rotate-half convention, use_mrope false)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / head_dim)


def rope(x, pos, theta):
    """Rotate-half RoPE.  x [..., D]; pos broadcastable to x.shape[:-1]; angle in float64.

    out[i]       = x[i] cos(a_i) - x[i + D/2] sin(a_i)
    out[i + D/2] = x[i + D/2] cos(a_i) + x[i] sin(a_i),   a_i = pos * inv_freq_i
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(D, theta)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def round_bf16(x):
    """Round to bfloat16 (8 significant bits, fp32 exponent range), nearest with ties to even;
    returned as float64 values.  The storage rounding of the bf16 KV-cache variant (the fp16 /
    fp32 cache trade-off of "VibeVoice-ASR — ONNX export for Vernacula", Highlights, with a
    third storage type).  x = m 2^e with 0.5 <= |m| < 1 (frexp); m is rounded to a multiple of
    2^-8.  Zero stays zero; the cache values here are far from bf16's subnormal and overflow
    ranges, which are not modelled."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def kv_round(x, kv_dtype):
    """A K/V value as stored in a cache of kv_dtype (np.float16, np.float32, "bf16", or
    np.float64 for no storage rounding): an array of kv_dtype, float64 for "bf16"."""
    if isinstance(kv_dtype, str):
        assert kv_dtype == "bf16", kv_dtype
        return round_bf16(x)
    return np.asarray(x, dtype=np.float64).astype(kv_dtype)


def repeat_kv(kv, group):
    """[Hkv, ...] -> [Hkv*group, ...]: query head h reads key/value head h // group."""
    return np.repeat(np.asarray(kv), group, axis=0)


def softmax(s, axis=-1):
    s = np.asarray(s, dtype=np.float64)
    e = np.exp(s - np.max(s, axis=axis, keepdims=True))
    return e / np.sum(e, axis=axis, keepdims=True)


def gqa_decode_attention(q, K, V, scale):
    """One query position over T cached positions, all visible (decoder_step has no mask input).

    q [Hq, D]; K, V [Hkv, T, D] -> out [Hq, D] = softmax(q . K^T * scale) . V per head,
    with K/V heads repeated Hq/Hkv times (grouped-query attention).
    """
    q = np.asarray(q, dtype=np.float64)
    Hq = q.shape[0]
    Hkv = K.shape[0]
    assert Hq % Hkv == 0
    Kr = repeat_kv(np.asarray(K, dtype=np.float64), Hq // Hkv)
    Vr = repeat_kv(np.asarray(V, dtype=np.float64), Hq // Hkv)
    p = softmax(np.einsum("hd,htd->ht", q, Kr) * scale)
    return np.einsum("ht,htd->hd", p, Vr)


def gqa_causal_attention(Q, K, V, scale):
    """Causal prefill attention.  Q [S, Hq, D]; K, V [S, Hkv, D] -> [S, Hq, D].
    Position i sees positions 0..i."""
    Q = np.asarray(Q, dtype=np.float64)
    S, Hq, D = Q.shape
    Hkv = K.shape[1]
    Kr = repeat_kv(np.asarray(K, dtype=np.float64).transpose(1, 0, 2), Hq // Hkv)  # [Hq, S, D]
    Vr = repeat_kv(np.asarray(V, dtype=np.float64).transpose(1, 0, 2), Hq // Hkv)
    s = np.einsum("ihd,hjd->hij", Q, Kr) * scale
    mask = np.triu(np.ones((S, S), dtype=bool), k=1)
    s[:, mask] = -np.inf
    p = softmax(s, axis=-1)
    return np.einsum("hij,hjd->ihd", p, Vr)


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu(gate, up):
    """h = silu(gate) * up."""
    return silu(gate) * np.asarray(up, dtype=np.float64)


def linear(x, weight, bias=None):
    """y = x @ W^T (+ bias) with W either a packed (q, scales) pair (MatMulNBits) or a dense
    array [N, K].  Packed weights are dequantised exactly to float64 first."""
    x = np.asarray(x, dtype=np.float64)
    K = x.shape[-1]
    if isinstance(weight, tuple):
        W = _pack.dequant(weight[0], weight[1], K)
    else:
        W = np.asarray(weight).astype(np.float64)
    y = x @ W.T
    if bias is not None:
        y = y + np.asarray(bias).astype(np.float64)
    return y


def matmul_nbits(x, q, scales, K, bias=None):
    """MatMulNBits: x [M, K] (or [K]) times the dequantised W[N, K]^T, plus optional bias."""
    return linear(np.asarray(x, dtype=np.float64)[..., :K], (q, scales), bias)


def lm_head_logits(x, w_lm, row_chunk=16384):
    """logits = W_lm . x for an fp16 [V, H] head (not quantised), in float64, chunked over rows."""
    x = np.asarray(x, dtype=np.float64)
    V = w_lm.shape[0]
    out = np.empty(V, dtype=np.float64)
    for r0 in range(0, V, row_chunk):
        out[r0:r0 + row_chunk] = np.asarray(w_lm[r0:r0 + row_chunk]).astype(np.float64) @ x
    return out


def greedy_argmax(logits):
    """Greedy token: index of the maximum logit, lowest index on ties."""
    return int(np.argmax(np.asarray(logits)))
