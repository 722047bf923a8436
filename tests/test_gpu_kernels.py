"""GPU parity of the single-op entry points against the oracle (through the C ABI).

Bars: packing and ternary scale bit-exact; GEMV one-hot exact after the single fp16 rounding,
random x within 1e-3 normwise (fp32 accumulation + one fp16 output rounding, bound 2^-11);
attention and lm_head within the 2e-3 contract tolerance; argmax equal where the oracle's top-2
margin exceeds 1e-2.
"""

import math

import numpy as np
import pytest
import torch

import synth
from helpers import TOL, normwise
from oracle import ops as oops
from oracle import pack as opack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vv():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from int4_blockwise_quantised_b200 import _vv

    return _vv


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# ------------------------------------------------------------------------------------ packing
PACK_SHAPES = [(1536, 1536), (256, 1536), (1536, 8960), (96, 1000), (3, 33), (5, 3584)]


@pytest.mark.parametrize("shape", PACK_SHAPES)
@pytest.mark.parametrize("mode", ["sym", "ternary"])
def test_pack_bit_exact(vv, shape, mode):
    W = synth.normal_f32(shape, 0.02, 100 + shape[0])
    W[0, :32] = 0.0  # a zero block
    if shape[1] >= 64:
        W[1, 32:64] = np.float32(0.4375) * np.array([1, 1 / 14, -1 / 14, 3 / 14] * 8, np.float32)
    if mode == "ternary":
        s_ora = opack.ternary_scale(W)
        s_gpu = vv.vv_ternary_scale(dev(W))
        assert np.float32(s_gpu) == s_ora
        q_o, sc_o = opack.pack_ternary(W, s_ora)
        q_g, sc_g = vv.vv_pack_nbits(dev(W), vv.VV_TERNARY, s_gpu)
    else:
        q_o, sc_o = opack.pack_sym_int4(W)
        q_g, sc_g = vv.vv_pack_nbits(dev(W), vv.VV_SYM_INT4)
    assert np.array_equal(q_g.cpu().numpy(), q_o)
    assert np.array_equal(sc_g.cpu().numpy().view(np.uint16), sc_o.view(np.uint16))


def test_ternary_scale_exact_on_adversarial_mix(vv):
    r = synth.rng(7)
    parts = [synth.normal_f32((100000,), 1e-3, 1), np.float32(1e30) * r.random(7).astype(np.float32),
             np.array([1e-45, 3e-42, 1.17e-38, 0.0], np.float32),
             synth.normal_f32((12345,), 1e5, 2)]
    W = np.concatenate(parts).astype(np.float32)
    assert np.float32(vv.vv_ternary_scale(dev(W))) == opack.ternary_scale(W)
    Z = np.zeros(1000, np.float32)
    assert math.isinf(vv.vv_ternary_scale(dev(Z)))


def test_pack_crafted_ties(vv):
    W = np.array([[0.4375, 0.03125, -0.03125, 0.09375, -0.09375, 0.15625, -0.4375, 0.0] + [0.0] * 24],
                 np.float32)
    q, sc = vv.vv_pack_nbits(dev(W), vv.VV_SYM_INT4)
    assert opack.nibble_unpack(q.cpu().numpy())[0, :8].tolist() == [15, 9, 7, 10, 6, 11, 1, 8]
    T = np.array([[0.25, -0.25, 0.75, -0.75, 0.2, -0.2, 0.0, 3.0] + [0.0] * 24], np.float32)
    q, sc = vv.vv_pack_nbits(dev(T), vv.VV_TERNARY, 2.0)
    assert opack.nibble_unpack(q.cpu().numpy())[0, :8].tolist() == [9, 7, 9, 7, 8, 8, 8, 9]


# --------------------------------------------------------------------------------------- GEMV
GEMV_SHAPES = [(1536, 1536), (256, 1536), (8960, 1536), (1536, 8960), (3584, 3584), (512, 3584),
               (18944, 3584), (3584, 18944), (100, 2048), (37, 992)]


@pytest.mark.parametrize("N,K", GEMV_SHAPES)
def test_gemv_random(vv, N, K):
    W = synth.normal_f32((N, K), 0.02, N + K)
    q, sc = opack.pack_sym_int4(W)
    x = synth.normal_f16((K,), 1.0, 5)
    b = synth.normal_f16((N,), 0.02, 6)
    ref = oops.matmul_nbits(x.astype(np.float64), q, sc, K, b)
    y = vv.vv_matmul_nbits(dev(x).reshape(1, K), dev(q), dev(sc), dev(b))
    assert normwise(y.cpu().numpy()[0].astype(np.float64), ref) <= 1e-3


def test_gemv_one_hot_layout_exact(vv):
    N, K = 64, 1536
    W = synth.normal_f32((N, K), 0.02, 9)
    q, sc = opack.pack_sym_int4(W)
    deq = opack.dequant(q, sc, K)
    X = np.zeros((8, K), np.float16)
    cols = [0, 1, 2, 15, 16, 17, 31, 1535]
    for i, k in enumerate(cols):
        X[i, k] = 1.0
    for i, k in enumerate(cols):
        y = vv.vv_matmul_nbits(dev(X[i:i + 1]), dev(q), dev(sc))
        assert np.array_equal(y.cpu().numpy()[0], deq[:, k].astype(np.float16))
    Y = vv.vv_matmul_nbits(dev(X), dev(q), dev(sc))  # M = 8 path
    for i, k in enumerate(cols):
        assert np.array_equal(Y.cpu().numpy()[i], deq[:, k].astype(np.float16))


@pytest.mark.parametrize("M", [2, 3, 8])
def test_gemv_multirow(vv, M):
    N, K = 300, 1536
    W = synth.normal_f32((N, K), 0.02, 10)
    q, sc = opack.pack_sym_int4(W)
    X = synth.normal_f16((M, K), 1.0, 11)
    ref = oops.matmul_nbits(X.astype(np.float64), q, sc, K)
    Y = vv.vv_matmul_nbits(dev(X), dev(q), dev(sc))
    assert normwise(Y.cpu().numpy().astype(np.float64), ref) <= 1e-3


# ------------------------------------------------------------- tensor-core MatMulNBits (many rows)
def test_gemm_tc_one_hot_layout_exact(vv):
    """Row m of x is one-hot at column k_m (M = 14 > 8: the tensor-core path, int4 expanded in
    shared memory): y[m] must be the fp16 dequantised column k_m exactly (single product, fp32
    accumulate, one rounding).  Columns span swizzle chunks, 64-column k blocks and the 256-column
    scale groups."""
    N, K = 512, 1536
    W = synth.normal_f32((N, K), 0.02, 19)
    q, sc = opack.pack_sym_int4(W)
    deq = opack.dequant(q, sc, K)
    cols = [0, 1, 7, 8, 15, 16, 31, 32, 63, 64, 100, 777, 1000, 1535]
    X = np.zeros((len(cols), K), np.float16)
    for i, k in enumerate(cols):
        X[i, k] = 1.0
    Y = vv.vv_matmul_nbits(dev(X), dev(q), dev(sc)).cpu().numpy()
    for i, k in enumerate(cols):
        assert np.array_equal(Y[i], deq[:, k].astype(np.float16)), (i, k)


# 256-, 192- and 128-wide tiles, a single tile, ragged M tails, and enough tiles (4530 rows) that
# every CTA of the persistent grid cycles through both accumulators (M > 8: tensor-core path)
GEMM_TC_SHAPES = [(9, 256, 256), (37, 1024, 1536), (128, 2048, 1536), (129, 512, 8960),
                  (300, 1536, 8960), (513, 256, 3584), (600, 128, 256), (1000, 1536, 512),
                  (4530, 2048, 1536), (4530, 1536, 1536)]


@pytest.mark.parametrize("M,N,K", GEMM_TC_SHAPES)
def test_gemm_tc_random(vv, M, N, K):
    """Random x, bias: within 1e-3 normwise (fp16 weight rounding 2^-12 relative, fp32
    accumulation, fp16 output rounding)."""
    W = synth.normal_f32((N, K), 0.02, M + N + K)
    q, sc = opack.pack_sym_int4(W)
    X = synth.normal_f16((M, K), 1.0, 21)
    b = synth.normal_f16((N,), 0.02, 22)
    ref = oops.matmul_nbits(X.astype(np.float64), q, sc, K, b)
    Y = vv.vv_matmul_nbits(dev(X), dev(q), dev(sc), dev(b))
    assert normwise(Y.cpu().numpy().astype(np.float64), ref) <= 1e-3


def test_gemm_tc_ternary_matches_gemv(vv):
    """Ternary weights: the tensor-core path (M = 16) and the GEMV path (two calls of M = 8)
    agree row by row."""
    N, K = 1536, 1536
    W = synth.normal_f32((N, K), 0.02, 23)
    s = opack.ternary_scale(W)
    q, sc = opack.pack_ternary(W, s)
    X = synth.normal_f16((16, K), 1.0, 24)
    a = vv.vv_matmul_nbits(dev(X), dev(q), dev(sc)).cpu().numpy().astype(np.float64)
    g = np.concatenate([vv.vv_matmul_nbits(dev(X[i:i + 8]), dev(q), dev(sc)).cpu().numpy()
                        for i in (0, 8)]).astype(np.float64)
    assert normwise(a, g) <= 1e-3


def test_gemm_tc_rejects_bad_shapes(vv):
    """M > 8 needs N % 128 == 0 and K % 256 == 0 (the GEMV path, M <= 8, does not)."""
    q = torch.zeros((100, 2, 16), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((100, 2), dtype=torch.float16, device="cuda")
    x = torch.zeros((12, 64), dtype=torch.float16, device="cuda")
    with pytest.raises(vv.VVError) as e:
        vv.vv_matmul_nbits(x, q, sc)
    assert e.value.code == vv.VV_ERR_SHAPE
    q2 = torch.zeros((128, 2, 16), dtype=torch.uint8, device="cuda")
    sc2 = torch.zeros((128, 2), dtype=torch.float16, device="cuda")
    with pytest.raises(vv.VVError) as e:
        vv.vv_matmul_nbits(x, q2, sc2)  # K = 64
    assert e.value.code == vv.VV_ERR_SHAPE
    vv.vv_matmul_nbits(x[:8], q, sc)  # M <= 8: any N, K % 32
    vv.vv_sync_status()


# ---------------------------------------------------------------------------------- attention
def _attn_case(vv, Hq, Hkv, length, cap, seed, kscale=1.0):
    D = 128
    q = synth.normal_f16((Hq, D), 1.0, seed)
    # the valid positions are drawn independently of `cap`; slots past `length` stay zero
    K = np.zeros((Hkv, cap, D), np.float16)
    V = np.zeros((Hkv, cap, D), np.float16)
    K[:, :length] = synth.normal_f16((Hkv, length, D), kscale, seed + 1)
    V[:, :length] = synth.normal_f16((Hkv, length, D), 1.0, seed + 2)
    ref = oops.gqa_decode_attention(q.astype(np.float64), K[:, :length].astype(np.float64),
                                    V[:, :length].astype(np.float64), 1 / math.sqrt(D))
    ws = torch.zeros(vv.vv_gqa_decode_attn_workspace_size(Hq, Hkv, D, cap), dtype=torch.uint8,
                     device="cuda")
    out = vv.vv_gqa_decode_attn(dev(q), dev(K), dev(V), length, 1 / math.sqrt(D), ws)
    return out.cpu().numpy().astype(np.float64), ref


@pytest.mark.parametrize("Hq,Hkv", [(12, 2), (28, 4), (8, 8), (16, 2)])
@pytest.mark.parametrize("length", [1, 63, 64, 65, 1025, 4785])
def test_attention_matches_oracle(vv, Hq, Hkv, length):
    out, ref = _attn_case(vv, Hq, Hkv, length, max(length, 4800), 20 + length)
    assert normwise(out, ref) <= TOL


def test_attention_split_count_invariance(vv):
    # The same data attended with different capacities (-> different chunk counts).
    a, ref = _attn_case(vv, 12, 2, 1000, 1000, 3)
    b, _ = _attn_case(vv, 12, 2, 1000, 9000, 3)
    assert normwise(a, ref) <= TOL and normwise(b, ref) <= TOL
    assert normwise(a, b) <= 1e-3


def test_attention_uniform_keys_mean_of_values(vv):
    D, Hq, Hkv, L = 128, 12, 2, 700
    q = synth.normal_f16((Hq, D), 1.0, 1)
    K = np.broadcast_to(synth.normal_f16((Hkv, 1, D), 1.0, 2), (Hkv, L, D)).copy()
    V = synth.normal_f16((Hkv, L, D), 1.0, 3)
    ws = torch.zeros(vv.vv_gqa_decode_attn_workspace_size(Hq, Hkv, D, L), dtype=torch.uint8,
                     device="cuda")
    out = vv.vv_gqa_decode_attn(dev(q), dev(K), dev(V), L, 1 / math.sqrt(D), ws).cpu().numpy()
    mean = V.astype(np.float64).mean(axis=1)
    for h in range(Hq):
        assert normwise(out[h], mean[h // 6]) <= TOL


# ------------------------------------------------------------------------------------ lm_head
@pytest.mark.parametrize("V,H", [(151936, 1536), (152064, 3584), (1000, 256), (4099, 1536)])
def test_lm_head_argmax(vv, V, H):
    x = synth.normal_f32((H,), 1.0, 31)
    g = synth.uniform_f16((H,), 0.5, 1.5, 32)
    W = synth.normal_f16((V, H), 0.02, 33)
    ref = oops.lm_head_logits(oops.rmsnorm(x.astype(np.float64), g, 1e-6), W)
    ws = torch.zeros(vv.vv_lm_head_argmax_workspace_size(V), dtype=torch.uint8, device="cuda")
    lg, idx = vv.vv_lm_head_argmax(dev(x), dev(g), dev(W), 1e-6, ws)
    assert normwise(lg.cpu().numpy(), ref) <= TOL
    top2 = np.sort(ref)[-2:]
    if top2[1] - top2[0] > 1e-2:
        assert int(idx.item()) == int(np.argmax(ref))
    # second call reuses the workspace (counter reset by the kernel)
    _, idx2 = vv.vv_lm_head_argmax(dev(x), dev(g), dev(W), 1e-6, ws, logits=False)
    assert int(idx2.item()) == int(idx.item())


def test_lm_head_ties_lowest_index(vv):
    V, H = 5000, 256
    W = synth.normal_f16((V, H), 0.02, 40)
    W[4321] = W[77] = np.full(H, 0.5, np.float16)  # two identical best rows
    x = np.ones(H, np.float32)
    g = np.ones(H, np.float16)
    ws = torch.zeros(vv.vv_lm_head_argmax_workspace_size(V), dtype=torch.uint8, device="cuda")
    _, idx = vv.vv_lm_head_argmax(dev(x), dev(g), dev(W), 1e-6, ws)
    assert int(idx.item()) == 77
