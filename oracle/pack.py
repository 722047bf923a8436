"""Oracle: MatMulNBits-style int4 packing (test infrastructure only; see ``oracle/__init__``).

Layout (not printed on the pages; the public ONNX Runtime ``com.microsoft::MatMulNBits``
definition is taken): a weight W[N, K] becomes

* ``q``      uint8 [N, KB, 16], KB = ceil(K/32): block b of row n holds the 32 codes of
             columns 32b .. 32b+31; byte j holds column 32b+2j in its LOW nibble and column
             32b+2j+1 in its HIGH nibble;
* ``scales`` float16 [N, KB]: one scale per block; no zero-point tensor (implicit zero point 8).

Dequantised value: (code - 8) * scale.  Columns past K (when K is not a multiple of 32) are
padded with code 8.

Readings of points the pages leave open:

* rounding is "half away from zero" (C ``roundf``), done in float64 so that |t| + 0.5 is exact;
* packing arithmetic is IEEE float32, one rounding per operation, no fused multiply-add;
* the ternary per-tensor mean|W| is the correctly rounded float64 sum (``math.fsum``) divided by
  the element count, and s = float32(1 / mean);
* ternary block scale = float16(float32(1/s)), the same for every block of the tensor;
* int4 block scale = float16(float32(max|w_block| / 7)), code = clamp(round(w/scale), -8, 7) + 8;
* a zero block (or a ternary tensor whose mean|W| is zero) gets scale 0 and all codes 8.
"""

import math

import numpy as np

BLOCK = 32


def n_blocks(K):
    """Number of 32-column blocks per row."""
    return -(-int(K) // BLOCK)


def round_half_away(t):
    """Round to the nearest integer, ties away from zero, for float32/float64 arrays.

    Computed in float64: for a float32 input |t| + 0.5 is then exact, so floor() decides the
    tie correctly (in float32, 0.49999997 + 0.5 would round up to 1.0).
    """
    t64 = np.asarray(t, dtype=np.float64)
    return np.copysign(np.floor(np.abs(t64) + 0.5), t64)


def nibble_pack(codes):
    """codes uint8 [N, KB*32] with values 0..15 -> packed uint8 [N, KB, 16] (low nibble first)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, C = codes.shape
    assert C % BLOCK == 0
    pairs = codes.reshape(N, C // BLOCK, 16, 2)
    return (pairs[..., 0] | (pairs[..., 1] << 4)).astype(np.uint8)


def nibble_unpack(q):
    """packed uint8 [N, KB, 16] -> codes uint8 [N, KB*32] (inverse of ``nibble_pack``)."""
    q = np.asarray(q, dtype=np.uint8)
    N, KB, _ = q.shape
    lo = q & 0x0F
    hi = q >> 4
    return np.stack([lo, hi], axis=-1).reshape(N, KB * BLOCK)


def ternary_scale(W):
    """Per-tensor BitNet scale s = 1 / mean(|W|) ("vibevoice-asr-bitnet-onnx", ternarisation
    paragraph).  mean = fsum(|W|) / count in float64; s = float32(1.0 / mean).  A tensor with
    mean 0 gives s = +inf (treated as a zero tensor by ``pack_ternary``)."""
    a = np.abs(np.asarray(W, dtype=np.float32)).astype(np.float64).ravel()
    total = math.fsum(a)
    if total == 0.0:
        return np.float32(np.inf)
    mean = total / a.size
    return np.float32(1.0 / mean)


def pack_ternary(W, s):
    """Ternarise and pack W[N, K] with the per-tensor scale s.

    t = float32(W * s); c = clamp(t, -1, 1); r = round(c) in {-1, 0, 1}; code = r + 8 in {7, 8, 9};
    every block's scale is float16(float32(1 / s)) ("vibevoice-asr-bitnet-onnx": stored
    q = w/s + 8 in {7, 8, 9}, block 32, per-block scale = the ternary scale).
    Returns (q uint8 [N, KB, 16], scales float16 [N, KB]).
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    KB = n_blocks(K)
    s = np.float32(s)
    codes = np.full((N, KB * BLOCK), 8, dtype=np.uint8)
    if not (np.isfinite(s) and s > 0):
        scale16 = np.float16(0.0)
    else:
        t = W * s  # one float32 rounding
        c = np.clip(t, np.float32(-1.0), np.float32(1.0))
        r = round_half_away(c)
        codes[:, :K] = (r + 8.0).astype(np.uint8)
        scale16 = np.float16(np.float32(1.0) / s)
    scales = np.full((N, KB), scale16, dtype=np.float16)
    return nibble_pack(codes), scales


def pack_sym_int4(W):
    """General symmetric int4 per block of 32 (scale = max|w|/7).

    scale16 = float16(float32(max|w_block|) / 7); t = float32(w / float32(scale16));
    code = clamp(round(t), -8, 7) + 8; a block whose scale16 is 0 gets all codes 8.
    Returns (q uint8 [N, KB, 16], scales float16 [N, KB]).
    """
    W = np.asarray(W, dtype=np.float32)
    N, K = W.shape
    KB = n_blocks(K)
    Wp = np.zeros((N, KB * BLOCK), dtype=np.float32)
    Wp[:, :K] = W
    Wb = Wp.reshape(N, KB, BLOCK)
    amax = np.max(np.abs(Wb), axis=2)
    scale16 = (amax / np.float32(7.0)).astype(np.float16)
    s32 = scale16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = Wb / s32[..., None]
    r = np.clip(round_half_away(np.where(s32[..., None] == 0, 0.0, t)), -8.0, 7.0)
    codes = (r + 8.0).astype(np.uint8)
    codes[s32 == 0] = 8
    return nibble_pack(codes.reshape(N, KB * BLOCK)), scale16


def dequant(q, scales, K):
    """(code - 8) * scale in float64, shape [N, K] (padding columns dropped)."""
    q = np.asarray(q, dtype=np.uint8)
    N, KB, _ = q.shape
    codes = nibble_unpack(q).astype(np.float64) - 8.0
    sc = np.repeat(np.asarray(scales, dtype=np.float16).astype(np.float64), BLOCK, axis=1)
    return (codes * sc)[:, :K]
