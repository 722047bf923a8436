"""Pins of the oracle's packing against what the pages and arithmetic fix (CPU only).

* ternary codes are only {7, 8, 9} and every block carries the one ternary scale
  ("vibevoice-asr-bitnet-onnx": q = w/s + 8 in {7,8,9}, per-block scale = the ternary scale);
* the packed int4 tier decodes to exactly the fp16 tier's weights (same page: ternary x scale
  values are exact in fp16 and in block int4, so every tier decodes the same model);
* symmetric int4: the block max maps to code 1 or 15, |dequant - w| <= scale/2, packing is
  idempotent through dequantisation, crafted ties round away from zero;
* the byte layout matches a block written out by hand (tests/golden/matmulnbits_block_layout.txt).
"""

from fractions import Fraction

import numpy as np
import pytest

from conftest import read_golden
from oracle import pack
import synth


def _golden_block():
    keyed, _ = read_golden("matmulnbits_block_layout.txt")
    b = np.array([int(x, 16) for x in keyed["bytes"]], dtype=np.uint8)
    codes = np.array([int(x) for x in keyed["codes"]], dtype=np.uint8)
    scale = np.float16(float(keyed["scale"][0]))
    values = np.array([float(x) for x in keyed["values"]])
    return b, codes, scale, values


def test_layout_matches_handwritten_block():
    b, codes, scale, values = _golden_block()
    q = b.reshape(1, 1, 16)
    assert np.array_equal(pack.nibble_unpack(q)[0], codes)
    assert np.array_equal(pack.nibble_pack(codes.reshape(1, 32)), q)
    deq = pack.dequant(q, np.array([[scale]], np.float16), 32)
    assert np.array_equal(deq[0], values)


def test_layout_pack_of_handwritten_values():
    """Packing the written-out values with a scale that makes them exact reproduces the bytes."""
    b, codes, scale, values = _golden_block()
    W = (values.astype(np.float32)).reshape(1, 32)
    # Block max |w| = 4 -> scale = 4/7 is not 0.5, so build the codes through the ternary-free
    # path: a block whose max is 3.5 = 7 * 0.5 gives scale exactly 0.5.  Values -4 clamp to -8.
    q, sc = pack.pack_sym_int4(np.where(W < -3.5, np.float32(-3.5), W))
    assert sc[0, 0] == np.float16(0.5)
    expect = codes.copy()
    expect[expect == 0] = 1  # -4 was replaced by -3.5 -> code 1
    assert np.array_equal(pack.nibble_unpack(q)[0], expect)


@pytest.mark.parametrize("shape", [(64, 96), (37, 70), (8, 1536)])
def test_ternary_codes_and_single_scale(shape):
    W = synth.normal_f32(shape, 0.02, 11)
    s = pack.ternary_scale(W)
    q, sc = pack.pack_ternary(W, s)
    codes = pack.nibble_unpack(q)[:, : shape[1]]
    assert set(np.unique(codes).tolist()) == {7, 8, 9}
    pad = pack.nibble_unpack(q)[:, shape[1]:]
    assert np.all(pad == 8)
    assert np.all(sc == sc[0, 0])
    assert sc[0, 0] == np.float16(np.float32(1.0) / s)


def test_ternary_scale_exact_rational():
    """mean|W| from an exact rational sum, rounded once to float64, then s = float32(1/mean)."""
    W = synth.normal_f32((13, 29), 0.02, 5)
    exact = sum(Fraction(float(abs(v))) for v in W.ravel())
    mean = float(exact) / W.size
    assert pack.ternary_scale(W) == np.float32(1.0 / mean)


def test_ternary_tiers_decode_identically():
    """fp16 tier weight fp16(fl32(round(clamp(W s))/s)) == int4 tier dequant, bitwise."""
    W = synth.normal_f32((48, 320), 0.02, 7)
    s = pack.ternary_scale(W)
    r = pack.round_half_away(np.clip(W * s, np.float32(-1), np.float32(1))).astype(np.float32)
    w_fp32_tier = r / s  # float32 division, as the fp32 tier stores W'
    w_fp16_tier = w_fp32_tier.astype(np.float16)
    q, sc = pack.pack_ternary(W, s)
    deq = pack.dequant(q, sc, W.shape[1])
    assert np.array_equal(deq, w_fp16_tier.astype(np.float64))


def test_ternary_zero_tensor():
    W = np.zeros((4, 64), np.float32)
    s = pack.ternary_scale(W)
    assert np.isinf(s)
    q, sc = pack.pack_ternary(W, s)
    assert np.all(pack.nibble_unpack(q) == 8) and np.all(sc == 0)


def test_ternary_crafted_ties():
    # s = 2 (exact): W*s = +-0.5 exactly -> round away from zero -> +-1; 1.5 clamps to 1.
    W = np.array([[0.25, -0.25, 0.75, -0.75, 0.2, -0.2, 0.0, 3.0] + [0.0] * 24], np.float32)
    q, sc = pack.pack_ternary(W, np.float32(2.0))
    codes = pack.nibble_unpack(q)[0, :8]
    assert codes.tolist() == [9, 7, 9, 7, 8, 8, 8, 9]
    assert sc[0, 0] == np.float16(0.5)


def test_round_half_away_float32_edge():
    # Largest float32 below 0.5: a float32 floor(|t| + 0.5) would wrongly give 1.
    t = np.array([np.nextafter(np.float32(0.5), np.float32(0)), 0.5, -0.5, 1.5, -2.5, 2.4999998],
                 dtype=np.float32)
    assert pack.round_half_away(t).tolist() == [0.0, 1.0, -1.0, 2.0, -3.0, 2.0]


def test_sym_int4_crafted_ties():
    # amax = 0.4375 = 7/16 -> scale exactly 1/16; w = k/16 + 1/32 lands exactly on a tie.
    vals = [0.4375, 0.03125, -0.03125, 0.09375, -0.09375, 0.15625, -0.4375, 0.0]
    W = np.array([vals + [0.0] * 24], np.float32)
    q, sc = pack.pack_sym_int4(W)
    assert sc[0, 0] == np.float16(0.0625)
    assert pack.nibble_unpack(q)[0, :8].tolist() == [15, 9, 7, 10, 6, 11, 1, 8]


def test_sym_int4_block_max_error_bound_and_idempotence():
    W = synth.normal_f32((96, 1000), 0.02, 3)  # 1000 = 31 blocks + a ragged tail of 8
    q, sc = pack.pack_sym_int4(W)
    K = W.shape[1]
    codes = pack.nibble_unpack(q)
    deq = pack.dequant(q, sc, K)
    s64 = np.repeat(sc.astype(np.float64), 32, axis=1)[:, :K]
    # error bound (no clamping happens for normal-range scales)
    assert np.all(np.abs(deq - W.astype(np.float64)) <= 0.5 * s64 * (1 + 1e-6))
    # the element of largest magnitude in every full block maps to code 1 or 15
    Wb = W[:, : 31 * 32].reshape(96, 31, 32)
    arg = np.argmax(np.abs(Wb), axis=2)
    top = np.take_along_axis(codes[:, : 31 * 32].reshape(96, 31, 32), arg[..., None], 2)[..., 0]
    assert np.all((top == 1) | (top == 15))
    # padding codes are 8
    assert np.all(codes[:, K:] == 8)
    # idempotence: pack(dequant(pack(W))) == pack(W)
    q2, sc2 = pack.pack_sym_int4(deq.astype(np.float32))
    assert np.array_equal(q2, q) and np.array_equal(sc2, sc)


def test_sym_int4_zero_and_tiny_blocks():
    W = np.zeros((2, 64), np.float32)
    W[1, 32:] = 1e-9  # amax/7 underflows fp16 -> scale 0 -> all codes 8
    q, sc = pack.pack_sym_int4(W)
    assert np.all(pack.nibble_unpack(q) == 8)
    assert np.all(sc == 0)


def test_sym_int4_all_sixteen_codes_roundtrip():
    """Every code 1..15 at every position of a block survives dequant -> pack (code 0 is never
    produced by max|w|/7 scaling; -8 would need |w| > max)."""
    for shift in range(32):
        codes = (np.arange(32) + shift) % 15 + 1
        codes[0] = 15  # make sure the block max is 7*scale
        vals = (codes.astype(np.float32) - 8) * np.float32(0.125)
        q, sc = pack.pack_sym_int4(vals.reshape(1, 32))
        assert sc[0, 0] == np.float16(0.125)
        assert np.array_equal(pack.nibble_unpack(q)[0], codes.astype(np.uint8))
