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


def _valid_create_args(base=1 << 20):
    """A 1.5B-shaped config with fake, 16-byte aligned device pointers (never dereferenced: the
    checks below fail before any device work)."""
    cfg = vv.vv_config(1536, 1, 12, 2, 128, 8960, 1000, 1e-6, 1e6, 16, 16, 0, 0, 1)
    layers = (vv.vv_layer_weights * 1)()
    L = layers[0]
    L.input_norm = L.post_norm = L.bq = L.bk = L.bv = base
    for name in ("wq", "wk", "wv", "wo", "wgate", "wup", "wdown"):
        m = getattr(L, name)
        m.q = m.scales = base
    mw = vv.vv_model_weights(base, base, base, layers)
    return cfg, layers, mw


@pytest.mark.parametrize("field,value", [
    ("head_dim", 64), ("kv_dtype", 3), ("batch", 3), ("batch", -1), ("n_kv", 0), ("n_kv", 5),
    ("n_kv", 65), ("hidden", 1600), ("hidden", 7808), ("inter", 9088), ("layers", 0),
    ("kv_capacity", 0), ("max_position", 0), ("max_prefill", -1)])
def test_decoder_create_config_limits(field, value):
    """Each documented create-time limit (head_dim 128, kv_dtype and batch ranges, n_q % n_kv,
    hidden and inter multiples and caps, positive sizes) is a VV_ERR_SHAPE before device work."""
    cfg, layers, mw = _valid_create_args()
    setattr(cfg, field, value)
    h = ctypes.c_void_p()
    st = vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), 1 << 20, 1 << 20,
                                  ctypes.byref(h))
    assert st == vv.VV_ERR_SHAPE and not h.value, (field, value, vv.last_error())


def test_decoder_create_group_and_prefill_limits():
    """Query heads per KV head <= 8, n_q * head_dim <= 7680, and a prefill workspace only with the
    fp16 cache the prefill writes."""
    h = ctypes.c_void_p()
    for n_q, n_kv in ((18, 2), (64, 8)):  # 9 query heads per group; 8192 query columns
        cfg, layers, mw = _valid_create_args()
        cfg.n_q, cfg.n_kv = n_q, n_kv
        assert vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), 1 << 20, 1 << 20,
                                        ctypes.byref(h)) == vv.VV_ERR_SHAPE
    cfg, layers, mw = _valid_create_args()
    cfg.kv_dtype, cfg.max_prefill = vv.VV_KV_BF16, 16
    assert vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), 1 << 20, 1 << 20,
                                    ctypes.byref(h)) == vv.VV_ERR_SHAPE
    assert "prefill" in vv.last_error()[1]


def test_decoder_create_pointer_checks():
    """Null tables, misaligned caches and misaligned packed matrices are VV_ERR_INVALID_ARG."""
    h = ctypes.c_void_p()
    base = 1 << 20
    cfg, layers, mw = _valid_create_args()
    mw.embed = None
    assert vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), base, base,
                                    ctypes.byref(h)) == vv.VV_ERR_INVALID_ARG
    cfg, layers, mw = _valid_create_args()
    assert vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), base + 8, base,
                                    ctypes.byref(h)) == vv.VV_ERR_INVALID_ARG
    cfg, layers, mw = _valid_create_args()
    layers[0].wdown.scales = base + 4
    assert vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), base, base,
                                    ctypes.byref(h)) == vv.VV_ERR_INVALID_ARG
    assert "packed weight" in vv.last_error()[1]
    cfg, layers, mw = _valid_create_args()
    layers[0].input_norm = None
    assert vv.lib.vv_decoder_create(ctypes.byref(cfg), ctypes.byref(mw), base, base,
                                    ctypes.byref(h)) == vv.VV_ERR_INVALID_ARG
