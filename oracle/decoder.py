"""Oracle: the decoder_init / decoder_step contracts of the Qwen2 backbone (test infrastructure
only; see ``oracle/__init__``).

Contracts ("vibevoice-asr-bitnet-onnx" model page, graph I/O listing):

    decoder_init(input_ids[1,S], position_ids[1,S], audio_features[1,N,H], audio_offset[1])
        -> logits[1,1,V], present_keys/values [L,1,Hkv,S,D]
    decoder_step(input_embeds[1,1,H], position_ids[1,1], past_keys/values [L,1,Hkv,P,D])
        -> logits[1,1,V], present_keys/values [L,1,Hkv,P+1,D]

decoder_init owns the embedding table and writes audio_features over the rows
[audio_offset, audio_offset + N) (the <|speech_pad|> positions).

Layer (pre-norm Qwen2, "VibeVoice-1.5B — Current Status", section "Architecture"):
    xn = RMSNorm(x); q,k,v = Wq xn + bq, Wk xn + bk, Wv xn + bv; RoPE(q, k) at position_ids;
    append k, v to the cache; o = GQA(q, K, V); x += Wo o;
    xn = RMSNorm(x); x += Wd (silu(Wg xn) * (Wu xn)).
Final: logits = W_lm . RMSNorm(x) (W_lm = the fp16 embedding table when tied).

Readings: K is cached after RoPE; keys/values are stored as float16 (the contract's storage type)
and attention always reads the stored float16 values, the current position included; every
other quantity is float64.  The attention scale is 1/sqrt(D).  decoder_step sees all cached
positions (no mask input); decoder_init is causal.
"""

import math
from dataclasses import dataclass

import numpy as np

from . import ops


@dataclass(frozen=True)
class Config:
    hidden: int
    layers: int
    n_q: int
    n_kv: int
    head_dim: int
    inter: int
    vocab: int
    eps: float = 1e-6
    theta: float = 1e6


def splice_embeddings(embed, input_ids, audio_features=None, audio_offset=0):
    """Gather fp16 rows of the embedding table for input_ids [S] and overwrite rows
    [audio_offset, audio_offset + N) with audio_features [N, H].  Returns float16 [S, H]."""
    e = np.asarray(embed)[np.asarray(input_ids, dtype=np.int64)].astype(np.float16)
    if audio_features is not None and len(audio_features) > 0:
        n = audio_features.shape[0]
        assert 0 <= audio_offset and audio_offset + n <= e.shape[0]
        e[audio_offset:audio_offset + n] = np.asarray(audio_features, dtype=np.float16)
    return e


def _attn_in(cfg, lw, x, pos):
    """RMSNorm + q/k/v projections + bias + RoPE.  x [T, H] -> q [T, Hq, D], k/v [T, Hkv, D]."""
    D = cfg.head_dim
    xn = ops.rmsnorm(x, lw["input_norm"], cfg.eps)
    q = ops.linear(xn, lw["wq"], lw["bq"]).reshape(-1, cfg.n_q, D)
    k = ops.linear(xn, lw["wk"], lw["bk"]).reshape(-1, cfg.n_kv, D)
    v = ops.linear(xn, lw["wv"], lw["bv"]).reshape(-1, cfg.n_kv, D)
    p = np.asarray(pos, dtype=np.float64)
    q = ops.rope(q, p[:, None], cfg.theta)
    k = ops.rope(k, p[:, None], cfg.theta)
    return q, k, v


def _mlp_out(cfg, lw, x, o):
    """x += Wo o; x += Wd swiglu(Wg RMSNorm(x), Wu RMSNorm(x)).  x [T, H], o [T, Hq*D]."""
    x = x + ops.linear(o, lw["wo"])
    xn = ops.rmsnorm(x, lw["post_norm"], cfg.eps)
    h = ops.swiglu(ops.linear(xn, lw["wgate"]), ops.linear(xn, lw["wup"]))
    return x + ops.linear(h, lw["wdown"])


def final_logits(cfg, weights, x):
    xn = ops.rmsnorm(x, weights["final_norm"], cfg.eps)
    return ops.lm_head_logits(xn, weights["lm_head"])


def decoder_step(cfg, weights, input_embeds, position, k_cache, v_cache, kv_dtype=np.float16):
    """One decode step at batch 1.

    input_embeds float16 [H]; position int; k_cache/v_cache: per layer [Hkv, P, D] (the P past
    positions) of the cache's storage type kv_dtype (np.float16, np.float32, "bf16", or np.float64
    for a cache without storage rounding).  Returns dict with logits float64 [V], argmax,
    layer_out float64 [L, H] (the residual after each layer), k_new/v_new [L, Hkv, D] rounded
    to kv_dtype (arrays of kv_dtype; float64 holding bf16 values for "bf16").  The contract stores K/V in float16 ("vibevoice-asr-bitnet-onnx",
    decoder_step I/O); kv_dtype=np.float32 is the fp32-cache variant of "VibeVoice-ASR — ONNX
    export for Vernacula" (Highlights), where only the storage rounding differs.
    """
    x = np.asarray(input_embeds, dtype=np.float16).astype(np.float64)[None, :]
    scale = 1.0 / math.sqrt(cfg.head_dim)
    outs, k_new, v_new = [], [], []
    for li, lw in enumerate(weights["layers"]):
        q, k, v = _attn_in(cfg, lw, x, [position])
        k16 = ops.kv_round(k[0], kv_dtype)
        v16 = ops.kv_round(v[0], kv_dtype)
        K = np.concatenate([ops.kv_round(k_cache[li], kv_dtype), k16[:, None, :]], axis=1)
        V = np.concatenate([ops.kv_round(v_cache[li], kv_dtype), v16[:, None, :]], axis=1)
        o = ops.gqa_decode_attention(q[0], K.astype(np.float64), V.astype(np.float64), scale)
        x = _mlp_out(cfg, lw, x, o.reshape(1, -1))
        outs.append(x[0].copy())
        k_new.append(k16)
        v_new.append(v16)
    logits = final_logits(cfg, weights, x[0])
    return {
        "logits": logits,
        "argmax": ops.greedy_argmax(logits),
        "layer_out": np.stack(outs),
        "k_new": np.stack(k_new),
        "v_new": np.stack(v_new),
    }


def decoder_init(cfg, weights, input_ids, position_ids, audio_features=None, audio_offset=0,
                 embeds=None):
    """Prefill of S positions (causal).  Either input_ids (+ optional audio splice) or a ready
    float16 embeds [S, H] array.  Returns dict with logits float64 [V] of the last position,
    argmax, k/v float16 [L, Hkv, S, D], layer_out float64 [L, H] (last position's residual after
    each layer)."""
    if embeds is None:
        embeds = splice_embeddings(weights["embed"], input_ids, audio_features, audio_offset)
    x = np.asarray(embeds, dtype=np.float16).astype(np.float64)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    ks, vs, outs = [], [], []
    for lw in weights["layers"]:
        q, k, v = _attn_in(cfg, lw, x, position_ids)
        k16 = k.astype(np.float16)
        v16 = v.astype(np.float16)
        o = ops.gqa_causal_attention(q, k16.astype(np.float64), v16.astype(np.float64), scale)
        x = _mlp_out(cfg, lw, x, o.reshape(o.shape[0], -1))
        ks.append(k16.transpose(1, 0, 2))
        vs.append(v16.transpose(1, 0, 2))
        outs.append(x[-1].copy())
    logits = final_logits(cfg, weights, x[-1])
    return {
        "logits": logits,
        "argmax": ops.greedy_argmax(logits),
        "k": np.stack(ks),
        "v": np.stack(vs),
        "layer_out": np.stack(outs),
    }
