"""Seeded synthetic inputs shared by the tests, the benchmark, the oracle checks and the CUDA path.

This module holds only random-number draws and workload shapes: none of the method's
arithmetic (no packing, no norms, no attention).  Every draw uses numpy's PCG64 with an explicit
seed, so the oracle and the GPU path see the same bytes.

Seeding recipe: matrix m (0..6 = q, k, v, o, gate, up, down) of layer l uses seed
``base + 1000*l + m``; per-layer vectors use ``base + 1000*l + 10 + j``; model-wide tensors use
``base + 900000 + j``; per-run tensors (KV, embeds, audio, ids) use ``base + 800000 + j``.
"""

from dataclasses import dataclass

import numpy as np

MATRICES = ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown")


@dataclass(frozen=True)
class Shape:
    """Qwen2 backbone dimensions of a workload."""

    name: str
    hidden: int
    layers: int
    n_q: int
    n_kv: int
    head_dim: int
    inter: int
    vocab: int
    tied: bool
    eps: float = 1e-6
    theta: float = 1e6

    def matrix_shape(self, m):
        """(N, K) of matrix m in MATRICES order."""
        H, D, I = self.hidden, self.head_dim, self.inter
        return {
            "wq": (self.n_q * D, H),
            "wk": (self.n_kv * D, H),
            "wv": (self.n_kv * D, H),
            "wo": (H, self.n_q * D),
            "wgate": (I, H),
            "wup": (I, H),
            "wdown": (H, I),
        }[m]


# Qwen2.5-1.5B backbone of VibeVoice-1.5B / ASR-BitNet and Qwen2.5-7B of VibeVoice-ASR(-HF).
SHAPE_1P5B = Shape("qwen2-1.5b", 1536, 28, 12, 2, 128, 8960, 151936, tied=True)
SHAPE_7B = Shape("qwen2-7b", 3584, 28, 28, 4, 128, 18944, 152064, tied=False)
# Realtime-0.5B backbone: 20 layers, hidden 896 (the pages' figures).  The pages give no head
# counts or MLP width: 7 query heads and 1 KV head of dimension 128 (7 x 128 = 896, the head
# dimension of the other backbones) and the Qwen2.5-0.5B MLP width 4864 are this build's reading.
SHAPE_0P5B = Shape("realtime-0.5b", 896, 20, 7, 1, 128, 4864, 151936, tied=True)
# Small shapes for fast parity runs; several tiles and a ragged tail on every axis that has one.
SHAPE_TINY = Shape("tiny", 256, 2, 4, 2, 128, 768, 1000, tied=True)
SHAPE_SMALL = Shape("small", 1536, 2, 12, 2, 128, 8960, 4099, tied=True)


def rng(seed):
    return np.random.Generator(np.random.PCG64(int(seed)))


def normal_f32(shape, std, seed):
    """float32 N(0, std^2)."""
    a = rng(seed).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def normal_f16(shape, std, seed):
    """float16 N(0, std^2) (drawn in float32, rounded to float16)."""
    return normal_f32(shape, std, seed).astype(np.float16)


def uniform_f16(shape, lo, hi, seed):
    return rng(seed).uniform(lo, hi, size=shape).astype(np.float16)


def master(shape, m, layer, std, base=0):
    """fp32 master of matrix m (name in MATRICES) of a layer, N(0, std^2)."""
    N, K = shape.matrix_shape(m)
    return normal_f32((N, K), std, base + 1000 * layer + MATRICES.index(m))


def layer_vectors(shape, layer, base=0):
    """fp16 norm gains U(0.5, 1.5) and q/k/v biases N(0, 0.02^2) of a layer."""
    H, D = shape.hidden, shape.head_dim
    s = base + 1000 * layer + 10
    return {
        "input_norm": uniform_f16((H,), 0.5, 1.5, s + 0),
        "post_norm": uniform_f16((H,), 0.5, 1.5, s + 1),
        "bq": normal_f16((shape.n_q * D,), 0.02, s + 2),
        "bk": normal_f16((shape.n_kv * D,), 0.02, s + 3),
        "bv": normal_f16((shape.n_kv * D,), 0.02, s + 4),
    }


def model_tables(shape, base=0):
    """fp16 embedding table [V, H] N(0, 0.02^2), lm_head (the same array when tied) and the final
    norm gain U(0.5, 1.5)."""
    V, H = shape.vocab, shape.hidden
    embed = normal_f16((V, H), 0.02, base + 900000)
    lm = embed if shape.tied else normal_f16((V, H), 0.02, base + 900001)
    return {"embed": embed, "lm_head": lm,
            "final_norm": uniform_f16((H,), 0.5, 1.5, base + 900002)}


def past_kv(shape, P, base=0):
    """Synthetic past K/V: fp16 N(0,1), [L, Hkv, P, D] each (K taken as already rotated)."""
    L, G, D = shape.layers, shape.n_kv, shape.head_dim
    k = normal_f16((L, G, P, D), 1.0, base + 800000)
    v = normal_f16((L, G, P, D), 1.0, base + 800001)
    return k, v


def input_embeds(shape, steps=1, base=0):
    """fp16 N(0,1) input_embeds, [steps, H]."""
    return normal_f16((steps, shape.hidden), 1.0, base + 800002)


def asr_prompt(shape, n_audio, prefix=20, suffix=10, speech_pad=151648, base=0):
    """ASR-shaped prompt: `prefix` text ids, n_audio speech_pad ids, `suffix` text ids (text ids
    uniform in [0, 151643) clipped to the vocabulary), and fp16 N(0,1) audio_features
    [n_audio, H].  Returns (ids int32 [S], positions int32 [S], audio_features, audio_offset)."""
    r = rng(base + 800003)
    hi = min(151643, shape.vocab)
    pre = r.integers(0, hi, size=prefix)
    suf = r.integers(0, hi, size=suffix)
    pad = min(speech_pad, shape.vocab - 1)
    ids = np.concatenate([pre, np.full(n_audio, pad), suf]).astype(np.int32)
    pos = np.arange(ids.size, dtype=np.int32)
    feats = normal_f16((n_audio, shape.hidden), 1.0, base + 800004)
    return ids, pos, feats, prefix


def frames_for_audio(seconds, rate=24000, hop=3200):
    """N = ceil(T / 3200) audio frames for T samples at 24 kHz."""
    T = int(round(seconds * rate))
    return -(-T // hop)
