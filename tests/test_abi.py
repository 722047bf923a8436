"""The C-ABI library loads without a GPU, exports every function include/vv.h declares, and its
host-side argument checks reject bad calls before touching CUDA (CPU only)."""

import ctypes

import pytest

vv = pytest.importorskip("int4_blockwise_quantised_b200._vv")


def test_exports_every_declared_function():
    names = vv.header_functions()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(vv.lib, n)]
    assert missing == []


def test_version_string():
    assert "sm_100a" in vv.vv_version()


def test_host_side_argument_checks():
    lib = vv.lib
    fake = 1 << 20  # aligned, never dereferenced: every check below fails before any CUDA call
    assert lib.vv_pack_nbits(None, 4, 64, 32, vv.VV_SYM_INT4, 0.0, fake, fake, None) == vv.VV_ERR_INVALID_ARG
    assert lib.vv_pack_nbits(fake, 4, 64, 16, vv.VV_SYM_INT4, 0.0, fake, fake, None) == vv.VV_ERR_SHAPE
    assert lib.vv_pack_nbits(fake, 4, 64, 32, 7, 0.0, fake, fake, None) == vv.VV_ERR_INVALID_ARG
    assert lib.vv_matmul_nbits(fake, fake, fake, None, 1, 8, 48, 32, fake, None) == vv.VV_ERR_SHAPE
    assert lib.vv_matmul_nbits(fake, fake, fake, None, 9, 8, 64, 32, fake, None) == vv.VV_ERR_SHAPE
    assert lib.vv_matmul_nbits(fake + 2, fake, fake, None, 1, 8, 64, 32, fake, None) == vv.VV_ERR_INVALID_ARG
    assert lib.vv_gqa_decode_attn(fake, fake, fake, 5, 4, 12, 2, 128, 0.1, fake, fake, 1 << 20,
                                  None) == vv.VV_ERR_SHAPE  # len > cap
    assert lib.vv_gqa_decode_attn(fake, fake, fake, 3, 4, 12, 5, 128, 0.1, fake, fake, 1 << 20,
                                  None) == vv.VV_ERR_SHAPE  # Hq % Hkv
    assert lib.vv_gqa_decode_attn(fake, fake, fake, 3, 4, 12, 2, 64, 0.1, fake, fake, 1 << 20,
                                  None) == vv.VV_ERR_SHAPE  # D != 128
    assert lib.vv_lm_head_argmax(fake, fake, fake, 100, 200, 1e-6, None, fake, fake, 1 << 20,
                                 None) == vv.VV_ERR_SHAPE  # H % 256
    assert lib.vv_decoder_set_length(None, 3, None) == vv.VV_ERR_INVALID_ARG
    code, text = vv.last_error()
    assert code == vv.VV_ERR_INVALID_ARG and "null" in text

    n = ctypes.c_int32()
    ids = (ctypes.c_int32 * 9)()
    assert lib.vv_decoder_generate(None, fake, fake, 4, ids, 0, fake, ctypes.byref(n),
                                   None) == vv.VV_ERR_INVALID_ARG
    assert lib.vv_decoder_generate(fake, fake, fake, 4, ids, 9, fake, ctypes.byref(n),
                                   None) == vv.VV_ERR_INVALID_ARG  # more than 8 stop ids


def test_decoder_create_rejects_bad_config():
    cfg = vv.vv_config(1536, 1, 12, 5, 128, 8960, 1000, 1e-6, 1e6, 16, 16, 0)  # 12 % 5 != 0
    layers = (vv.vv_layer_weights * 1)()
    mw = vv.vv_model_weights(1 << 20, 1 << 20, 1 << 20, layers)
    h = ctypes.c_void_p()
    st = vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), 1 << 20, 1 << 20,
                                  ctypes.byref(h))
    assert st == vv.VV_ERR_SHAPE and not h.value
    cfg.n_kv = 2
    cfg.head_dim = 64
    st = vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), 1 << 20, 1 << 20,
                                  ctypes.byref(h))
    assert st == vv.VV_ERR_SHAPE
    cfg.head_dim = 128  # null packed weights in the layer array
    st = vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), 1 << 20, 1 << 20,
                                  ctypes.byref(h))
    assert st == vv.VV_ERR_INVALID_ARG


def test_decoder_create_rejects_misaligned_gain_or_bias():
    """Norm gains and q/k/v biases are read as vectors by the kernels: a pointer off a 16-byte
    boundary is an argument error at create time (checked before any device work)."""
    base = 1 << 20
    cfg = vv.vv_config(1536, 1, 12, 2, 128, 8960, 1000, 1e-6, 1e6, 16, 16, 0)
    layers = (vv.vv_layer_weights * 1)()
    L = layers[0]
    L.input_norm = L.post_norm = base
    for name in ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown"):
        m = getattr(L, name)
        m.q = m.scales = base
    L.bq = L.bk = base
    L.bv = base + 2  # fp16-aligned but not 16-byte aligned
    mw = vv.vv_model_weights(base, base, base, layers)
    h = ctypes.c_void_p()
    st = vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), base, base,
                                  ctypes.byref(h))
    code, text = vv.last_error()
    assert st == vv.VV_ERR_INVALID_ARG and not h.value and "bias" in text
    L.bv = base
    L.post_norm = base + 8
    st = vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), base, base,
                                  ctypes.byref(h))
    assert st == vv.VV_ERR_INVALID_ARG and not h.value
