"""Pins of the oracle's operators (CPU only): closed forms, special cases, an independent
complex-number RoPE, pure-Python brute force on tiny inputs, and invariants (GQA == MHA with
repeated KV, uniform keys -> mean of V, causal prefill rows == decode attention)."""

import cmath
import math

import numpy as np
import pytest

from conftest import read_golden
from oracle import ops, pack
import synth


# ---------------------------------------------------------------- MatMulNBits GEMV
def test_gemv_one_hot_reads_golden_block():
    keyed, _ = read_golden("matmulnbits_block_layout.txt")
    q = np.array([int(x, 16) for x in keyed["bytes"]], np.uint8).reshape(1, 1, 16)
    scales = np.array([[float(keyed["scale"][0])]], np.float16)
    values = [float(v) for v in keyed["values"]]
    for k in range(32):
        x = np.zeros(32)
        x[k] = 1.0
        assert ops.matmul_nbits(x, q, scales, 32)[0] == values[k]


def test_gemv_bruteforce_nibble_loop():
    """Tiny GEMV against a scalar loop that reads nibbles straight from the bytes."""
    N, K = 5, 96
    W = synth.normal_f32((N, K), 0.02, 1)
    q, sc = pack.pack_sym_int4(W)
    x = synth.normal_f32((K,), 1.0, 2).astype(np.float64)
    bias = synth.normal_f16((N,), 0.02, 3)
    y = ops.matmul_nbits(x, q, sc, K, bias)
    for n in range(N):
        acc = 0.0
        for k in range(K):
            byte = int(q[n, k // 32, (k % 32) // 2])
            code = byte & 0xF if k % 2 == 0 else byte >> 4
            acc += (code - 8) * float(sc[n, k // 32]) * float(x[k])
        acc += float(bias[n])
        assert abs(acc - y[n]) <= 1e-12 * max(1.0, abs(acc))


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_vector_closed_form():
    H, eps = 48, 1e-6
    g = synth.uniform_f16((H,), 0.5, 1.5, 4)
    for c in (-3.0, 0.001, 2.5):
        y = ops.rmsnorm(np.full(H, c), g, eps)
        expect = g.astype(np.float64) * c / math.sqrt(c * c + eps)
        assert np.allclose(y, expect, rtol=1e-14, atol=0)


def test_rmsnorm_bruteforce():
    x = synth.normal_f32((7,), 1.0, 9).astype(np.float64)
    g = synth.uniform_f16((7,), 0.5, 1.5, 10)
    ms = sum(v * v for v in x) / 7
    expect = [float(x[i]) / math.sqrt(ms + 1e-6) * float(g[i]) for i in range(7)]
    assert np.allclose(ops.rmsnorm(x, g, 1e-6), expect, rtol=1e-14, atol=0)


# ---------------------------------------------------------------- RoPE
def test_rope_identity_at_position_zero():
    x = synth.normal_f32((3, 128), 1.0, 1).astype(np.float64)
    assert np.array_equal(ops.rope(x, np.zeros(3), 1e6), x)


def test_rope_matches_complex_rotation():
    """Pair (x_i, x_{i+D/2}) as the complex number x_i + j x_{i+D/2}, rotated by
    exp(j * pos * theta^(-2i/D))."""
    D, theta = 128, 1e6
    x = synth.normal_f32((D,), 1.0, 2).astype(np.float64)
    for pos in (1, 128, 4529):
        y = ops.rope(x[None, :], np.array([pos]), theta)[0]
        for i in range(D // 2):
            z = complex(x[i], x[i + D // 2]) * cmath.exp(1j * pos * theta ** (-2.0 * i / D))
            assert abs(y[i] - z.real) < 1e-9 and abs(y[i + D // 2] - z.imag) < 1e-9


def test_rope_relative_position_and_norm():
    D = 128
    q = synth.normal_f32((D,), 1.0, 3).astype(np.float64)
    k = synth.normal_f32((D,), 1.0, 4).astype(np.float64)
    a = ops.rope(q[None], np.array([100]), 1e6)[0] @ ops.rope(k[None], np.array([37]), 1e6)[0]
    b = ops.rope(q[None], np.array([1063]), 1e6)[0] @ ops.rope(k[None], np.array([1000]), 1e6)[0]
    assert abs(a - b) < 1e-9
    assert abs(np.linalg.norm(ops.rope(q[None], np.array([77]), 1e6)) - np.linalg.norm(q)) < 1e-12


# ---------------------------------------------------------------- attention
def test_attention_uniform_keys_gives_mean_of_values():
    Hq, Hkv, T, D = 6, 2, 9, 16
    q = synth.normal_f32((Hq, D), 1.0, 5).astype(np.float64)
    K = np.broadcast_to(synth.normal_f32((Hkv, 1, D), 1.0, 6), (Hkv, T, D)).astype(np.float64)
    V = synth.normal_f32((Hkv, T, D), 1.0, 7).astype(np.float64)
    o = ops.gqa_decode_attention(q, K, V, 1 / math.sqrt(D))
    for h in range(Hq):
        assert np.allclose(o[h], V[h // 3].mean(axis=0), rtol=1e-12, atol=1e-12)


def test_attention_dominant_key_selects_its_value():
    Hq, Hkv, T, D = 2, 1, 6, 8
    q = synth.normal_f32((Hq, D), 1.0, 8).astype(np.float64)
    q[1] = q[0]
    K = synth.normal_f32((Hkv, T, D), 0.01, 9).astype(np.float64)
    K[0, 4] = 50.0 * q[0]
    V = synth.normal_f32((Hkv, T, D), 1.0, 10).astype(np.float64)
    o = ops.gqa_decode_attention(q, K, V, 1 / math.sqrt(D))
    assert np.allclose(o[0], V[0, 4], atol=1e-9)


def test_gqa_equals_mha_with_repeated_heads():
    Hq, Hkv, T, D = 12, 2, 11, 32
    q = synth.normal_f32((Hq, D), 1.0, 11).astype(np.float64)
    K = synth.normal_f32((Hkv, T, D), 1.0, 12).astype(np.float64)
    V = synth.normal_f32((Hkv, T, D), 1.0, 13).astype(np.float64)
    Kmha = np.stack([K[h // 6] for h in range(Hq)])
    Vmha = np.stack([V[h // 6] for h in range(Hq)])
    a = ops.gqa_decode_attention(q, K, V, 0.17)
    b = ops.gqa_decode_attention(q, Kmha, Vmha, 0.17)
    assert np.array_equal(a, b)


def test_attention_bruteforce_tiny():
    Hq, Hkv, D = 4, 2, 8
    for T in range(1, 6):
        q = synth.normal_f32((Hq, D), 1.0, 20 + T).astype(np.float64)
        K = synth.normal_f32((Hkv, T, D), 1.0, 30 + T).astype(np.float64)
        V = synth.normal_f32((Hkv, T, D), 1.0, 40 + T).astype(np.float64)
        o = ops.gqa_decode_attention(q, K, V, 1 / math.sqrt(D))
        for h in range(Hq):
            g = h // (Hq // Hkv)
            s = [sum(q[h, d] * K[g, t, d] for d in range(D)) / math.sqrt(D) for t in range(T)]
            m = max(s)
            e = [math.exp(v - m) for v in s]
            z = sum(e)
            for d in range(D):
                ref = sum(e[t] / z * V[g, t, d] for t in range(T))
                assert abs(o[h, d] - ref) < 1e-12


def test_causal_prefill_rows_equal_decode():
    S, Hq, Hkv, D = 7, 4, 2, 16
    Q = synth.normal_f32((S, Hq, D), 1.0, 50).astype(np.float64)
    K = synth.normal_f32((S, Hkv, D), 1.0, 51).astype(np.float64)
    V = synth.normal_f32((S, Hkv, D), 1.0, 52).astype(np.float64)
    full = ops.gqa_causal_attention(Q, K, V, 0.25)
    for i in range(S):
        dec = ops.gqa_decode_attention(Q[i], K[: i + 1].transpose(1, 0, 2),
                                       V[: i + 1].transpose(1, 0, 2), 0.25)
        assert np.allclose(full[i], dec, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- SwiGLU / argmax
def test_silu_closed_forms():
    assert ops.silu(np.array([0.0]))[0] == 0.0
    assert abs(ops.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    assert abs(ops.silu(np.array([-40.0]))[0]) < 1e-15
    assert abs(ops.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    g = np.array([0.5, -2.0])
    u = np.array([3.0, 0.25])
    assert np.allclose(ops.swiglu(g, u), [0.5 / (1 + math.exp(-0.5)) * 3.0,
                                          -2.0 / (1 + math.exp(2.0)) * 0.25], rtol=1e-15)


def test_argmax_lowest_index_on_ties():
    assert ops.greedy_argmax(np.array([1.0, 3.0, 2.0, 3.0])) == 1
    assert ops.greedy_argmax(np.array([-1.0, -1.0])) == 0


@pytest.mark.parametrize("seconds", [1, 600, 0.1, 13.3333])
def test_frame_count_golden(seconds):
    _, rows = read_golden("asr_frame_count.txt")
    table = {r[0]: int(r[1]) for r in rows}
    assert synth.frames_for_audio(seconds) == table[float(seconds)]


# ---------------------------------------------------------------- bf16 storage rounding
def test_round_bf16_ties_to_even_at_eight_bits():
    """bf16 keeps 8 significant bits: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 and goes to
    the even neighbour 1; 1 + 3 2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)."""
    cases = {1.0: 1.0, 1.0 + 2.0**-8: 1.0, 1.0 + 3 * 2.0**-8: 1.0 + 2.0**-6,
             1.0 + 2.0**-7: 1.0 + 2.0**-7, -3.0: -3.0, 0.0: 0.0,
             1.0 + 2.0**-8 + 2.0**-20: 1.0 + 2.0**-7, 255.5: 256.0, 254.5: 254.0}
    for x, want in cases.items():
        assert ops.round_bf16(np.array([x]))[0] == want, x


def test_round_bf16_matches_torch_on_fp32_values():
    """For values exactly representable in fp32, rounding straight from them is torch's
    fp32 -> bfloat16 conversion (round to nearest even), an independent implementation."""
    import torch

    g = np.random.default_rng(5)
    x = (g.standard_normal(20000) * np.exp(g.uniform(-20, 20, 20000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ops.round_bf16(x.astype(np.float64)), want)


def test_round_bf16_error_bound_and_idempotence():
    g = np.random.default_rng(6)
    x = g.standard_normal(10000) * 37.0
    r = ops.round_bf16(x)
    assert np.all(np.abs(r - x) <= np.abs(x) * 2.0**-8)
    assert np.array_equal(ops.round_bf16(r), r)


def test_kv_round_storage_types():
    x = np.array([1.0 + 2.0**-12, -2.5 + 2.0**-30])
    assert ops.kv_round(x, np.float16).dtype == np.float16
    assert ops.kv_round(x, np.float16)[0] == 1.0  # 2^-12 is below fp16's half ulp at 1
    assert ops.kv_round(x, np.float32)[1] == np.float32(-2.5 + 2.0**-30)
    assert np.array_equal(ops.kv_round(x, np.float64), x)
    assert np.array_equal(ops.kv_round(x, "bf16"), ops.round_bf16(x))
