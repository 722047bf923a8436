"""Pins of the oracle's decoder (CPU only).

* a tiny model (H=64, 2 layers, 4 query / 2 key-value heads, D=16, V=97) against an independent
  scalar implementation written with Python loops, complex-number RoPE and math.exp;
* KV-incremental decode equals full causal prefill ("VibeVoice-1.5B — Current Status", section
  "Inference (ONNX)": KV-incremental == full, cos 1.0);
* the ternary int4 tier decodes token-exactly like the fp16 tier ("vibevoice-asr-bitnet-onnx",
  tier table: fp16 and int4 tiers token-EXACT);
* the audio splice overwrites exactly rows [audio_offset, audio_offset + N).
"""

import cmath
import math

import numpy as np

from oracle import decoder, pack
import synth

TINY = decoder.Config(hidden=64, layers=2, n_q=4, n_kv=2, head_dim=16, inter=96, vocab=97)
TINY_SHAPE = synth.Shape("t", 64, 2, 4, 2, 16, 96, 97, tied=True)


def build_model(shape, cfg, mode="int4", std=0.2):
    layers = []
    for li in range(shape.layers):
        lw = dict(synth.layer_vectors(shape, li))
        masters = {m: synth.master(shape, m, li, std) for m in synth.MATRICES}
        for m, W in masters.items():
            if mode == "int4":
                lw[m] = pack.pack_sym_int4(W)
            elif mode == "ternary":
                lw[m] = pack.pack_ternary(W, pack.ternary_scale(W))
            elif mode == "ternary_fp16_tier":
                s = pack.ternary_scale(W)
                r = pack.round_half_away(np.clip(W * s, np.float32(-1), np.float32(1)))
                lw[m] = (r.astype(np.float32) / s).astype(np.float16)
        layers.append(lw)
    tables = synth.model_tables(shape)
    tables["embed"] = (tables["embed"].astype(np.float32) * 20).astype(np.float16)
    tables["lm_head"] = tables["embed"]
    return dict(tables, layers=layers)


# ------------------------------------------------------------ independent scalar model
def _nib(wq, n, k):
    q, sc = wq
    byte = int(q[n, k // 32, (k % 32) // 2])
    code = byte & 0xF if k % 2 == 0 else byte >> 4
    return (code - 8) * float(sc[n, k // 32])


def _mv(wq, x, nrows):
    return [sum(_nib(wq, n, k) * x[k] for k in range(len(x))) for n in range(nrows)]


def _norm(x, g, eps):
    r = math.sqrt(sum(v * v for v in x) / len(x) + eps)
    return [x[i] / r * float(g[i]) for i in range(len(x))]


def _rot(vec, pos, theta):
    D = len(vec)
    out = [0.0] * D
    for i in range(D // 2):
        z = complex(vec[i], vec[i + D // 2]) * cmath.exp(1j * pos * theta ** (-2.0 * i / D))
        out[i], out[i + D // 2] = z.real, z.imag
    return out


def scalar_step(cfg, W, emb, pos, kc, vc):
    H, D, Hq, Hkv = cfg.hidden, cfg.head_dim, cfg.n_q, cfg.n_kv
    x = [float(v) for v in emb]
    kn, vn = [], []
    for li, lw in enumerate(W["layers"]):
        xn = _norm(x, lw["input_norm"], cfg.eps)
        q = [a + float(b) for a, b in zip(_mv(lw["wq"], xn, Hq * D), lw["bq"])]
        k = [a + float(b) for a, b in zip(_mv(lw["wk"], xn, Hkv * D), lw["bk"])]
        v = [a + float(b) for a, b in zip(_mv(lw["wv"], xn, Hkv * D), lw["bv"])]
        q = sum((_rot(q[h * D:(h + 1) * D], pos, cfg.theta) for h in range(Hq)), [])
        k = sum((_rot(k[h * D:(h + 1) * D], pos, cfg.theta) for h in range(Hkv)), [])
        k16 = [float(np.float16(a)) for a in k]
        v16 = [float(np.float16(a)) for a in v]
        kn.append(k16)
        vn.append(v16)
        P = kc[li].shape[1]
        o = []
        for h in range(Hq):
            g = h * Hkv // Hq
            keys = [[float(a) for a in kc[li][g, t]] for t in range(P)] + [k16[g * D:(g + 1) * D]]
            vals = [[float(a) for a in vc[li][g, t]] for t in range(P)] + [v16[g * D:(g + 1) * D]]
            s = [sum(q[h * D + d] * kk[d] for d in range(D)) / math.sqrt(D) for kk in keys]
            m = max(s)
            e = [math.exp(a - m) for a in s]
            z = sum(e)
            o += [sum(e[t] * vals[t][d] for t in range(len(e))) / z for d in range(D)]
        x = [a + b for a, b in zip(x, _mv(lw["wo"], o, H))]
        xn = _norm(x, lw["post_norm"], cfg.eps)
        gt = _mv(lw["wgate"], xn, cfg.inter)
        up = _mv(lw["wup"], xn, cfg.inter)
        hmid = [a / (1 + math.exp(-a)) * b for a, b in zip(gt, up)]
        x = [a + b for a, b in zip(x, _mv(lw["wdown"], hmid, H))]
    xn = _norm(x, W["final_norm"], cfg.eps)
    logits = [sum(float(W["lm_head"][r, c]) * xn[c] for c in range(H)) for r in range(cfg.vocab)]
    return logits, kn, vn


def test_tiny_model_matches_scalar_implementation():
    W = build_model(TINY_SHAPE, TINY)
    P = 5
    kc, vc = synth.past_kv(TINY_SHAPE, P)
    emb = synth.input_embeds(TINY_SHAPE)[0]
    pos = 130
    ora = decoder.decoder_step(TINY, W, emb, pos, list(kc), list(vc))
    logits, kn, vn = scalar_step(TINY, W, emb, pos, kc, vc)
    ref = np.array(logits)
    assert np.max(np.abs(ora["logits"] - ref)) <= 1e-10 * np.max(np.abs(ref))
    for li in range(TINY.layers):
        for name, a, b in (("k", ora["k_new"][li].ravel(), kn[li]), ("v", ora["v_new"][li].ravel(), vn[li])):
            diff = np.abs(a.astype(np.float64) - np.array(b))
            ulp = np.spacing(np.abs(a)).astype(np.float64)
            assert np.all(diff <= ulp), name


def test_kv_incremental_equals_full_prefill():
    W = build_model(TINY_SHAPE, TINY)
    S = 7
    ids = synth.rng(99).integers(0, TINY.vocab, size=S)
    pos = np.arange(S)
    full = decoder.decoder_init(TINY, W, ids, pos)
    head = decoder.decoder_init(TINY, W, ids[:-1], pos[:-1])
    step = decoder.decoder_step(TINY, W, W["embed"][ids[-1]], S - 1,
                                list(head["k"]), list(head["v"]))
    assert np.allclose(step["logits"], full["logits"], rtol=1e-10, atol=1e-10)
    assert np.allclose(step["layer_out"], full["layer_out"], rtol=1e-10, atol=1e-10)
    for li in range(TINY.layers):
        a = full["k"][li][:, -1].astype(np.float64)
        assert np.all(np.abs(a - step["k_new"][li]) <= np.spacing(np.abs(full["k"][li][:, -1])))
    assert step["argmax"] == full["argmax"]


def test_ternary_int4_tier_equals_fp16_tier():
    P = 4
    kc, vc = synth.past_kv(TINY_SHAPE, P)
    emb = synth.input_embeds(TINY_SHAPE)[0]
    a = decoder.decoder_step(TINY, build_model(TINY_SHAPE, TINY, "ternary"), emb, 9, list(kc), list(vc))
    b = decoder.decoder_step(TINY, build_model(TINY_SHAPE, TINY, "ternary_fp16_tier"), emb, 9,
                             list(kc), list(vc))
    assert np.array_equal(a["logits"], b["logits"])
    assert a["argmax"] == b["argmax"]


def test_audio_splice_rows():
    embed = synth.normal_f16((50, 8), 1.0, 3)
    ids = np.array([1, 2, 49, 49, 49, 3], np.int32)
    feats = synth.normal_f16((3, 8), 1.0, 4)
    e = decoder.splice_embeddings(embed, ids, feats, 2)
    assert np.array_equal(e[:2], embed[[1, 2]])
    assert np.array_equal(e[2:5], feats)
    assert np.array_equal(e[5], embed[3])


def test_fp32_kv_cache_variant_differs_only_by_storage_rounding():
    """kv_dtype=float32 keeps the new K/V at fp32; with the k/v projections zero and position 0
    (RoPE = identity) the new K/V are the fp16 biases themselves, so both storage types give
    identical results; in general the fp32 K/V rounds to the fp16 K/V within half an ulp."""
    W = build_model(TINY_SHAPE, TINY)
    kp, vp = synth.past_kv(TINY_SHAPE, 5)
    emb = W["embed"][11]
    a = decoder.decoder_step(TINY, W, emb, 5, list(kp), list(vp))
    b = decoder.decoder_step(TINY, W, emb, 5, [k.astype(np.float32) for k in kp],
                             [v.astype(np.float32) for v in vp], kv_dtype=np.float32)
    assert b["k_new"].dtype == np.float32 and a["k_new"].dtype == np.float16
    k16 = a["k_new"].astype(np.float64)
    assert np.all(np.abs(b["k_new"].astype(np.float16).astype(np.float64) - k16)
                  <= np.spacing(np.abs(a["k_new"])).astype(np.float64))
    assert not np.array_equal(a["logits"], b["logits"])  # the storage type does take effect
    assert np.max(np.abs(a["logits"] - b["logits"])) <= 1e-2 * np.max(np.abs(a["logits"]))
    # zero k/v projections at position 0: new k = bk, v = bv exactly -> identical results
    Z = dict(W, layers=[dict(lw) for lw in W["layers"]])
    zero = pack.pack_sym_int4(np.zeros((TINY.n_kv * TINY.head_dim, TINY.hidden), np.float32))
    for lw in Z["layers"]:
        lw["wk"] = zero
        lw["wv"] = zero
    e16 = [np.zeros((TINY.n_kv, 0, TINY.head_dim), np.float16)] * TINY.layers
    e32 = [np.zeros((TINY.n_kv, 0, TINY.head_dim), np.float32)] * TINY.layers
    c = decoder.decoder_step(TINY, Z, emb, 0, e16, e16)
    d = decoder.decoder_step(TINY, Z, emb, 0, e32, e32, kv_dtype=np.float32)
    assert np.array_equal(c["logits"], d["logits"])
    assert np.array_equal(c["k_new"].astype(np.float32), d["k_new"])
