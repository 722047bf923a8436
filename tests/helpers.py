"""Shared test fixtures: the same seeded synthetic inputs fed to the oracle and to libvv."""

import numpy as np

import synth
from oracle import decoder as odec
from oracle import pack as opack

TOL = 2e-3  # normwise max|gpu - oracle| / max|oracle| (contract tolerance)


def normwise(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def ocfg(shape):
    return odec.Config(hidden=shape.hidden, layers=shape.layers, n_q=shape.n_q, n_kv=shape.n_kv,
                       head_dim=shape.head_dim, inter=shape.inter, vocab=shape.vocab,
                       eps=shape.eps, theta=shape.theta)


def std_for(shape):
    return 0.015 if shape.hidden == 3584 else 0.02


def masters_fn(shape, base=0):
    std = std_for(shape)
    return lambda li, m: synth.master(shape, m, li, std, base)


def vectors_fn(shape, base=0):
    return lambda li: synth.layer_vectors(shape, li, base)


def oracle_model(shape, mode, base=0, layers=None):
    """Oracle weights dict: packed by oracle.pack from the synth masters."""
    mf, vf = masters_fn(shape, base), vectors_fn(shape, base)
    out = []
    for li in range(shape.layers if layers is None else layers):
        lw = dict(vf(li))
        for m in synth.MATRICES:
            W = mf(li, m)
            if mode == "ternary":
                lw[m] = opack.pack_ternary(W, opack.ternary_scale(W))
            else:
                lw[m] = opack.pack_sym_int4(W)
        out.append(lw)
    return dict(synth.model_tables(shape, base), layers=out)


def gpu_model(shape, mode, device="cuda", base=0):
    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import PackedModel

    m = _vv.VV_TERNARY if mode == "ternary" else _vv.VV_SYM_INT4
    return PackedModel(shape, m, masters_fn(shape, base), vectors_fn(shape, base),
                       synth.model_tables(shape, base), device)


# --------------------------------------------------------------------------- GPU-side helpers
def dev(a):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def fill_cache(dec, kp, vp):
    P = kp.shape[2]
    dec.k_cache[:, 0, :, :P] = dev(kp)
    dec.v_cache[:, 0, :, :P] = dev(vp)
    dec.set_length(P)


def run_steps(shape, mode, P, steps, cap=None, graph=True, check_kv=True):
    """Teacher-forced decode of `steps` positions from a synthetic past of P positions, every
    layer output, the logits, the argmax and the appended K/V checked against the oracle; returns
    the worst layer-output error."""
    import torch

    from int4_blockwise_quantised_b200.model import Decoder

    cfg = ocfg(shape)
    W = oracle_model(shape, mode)
    model = gpu_model(shape, mode)
    cap = cap or P + steps + 5
    dec = Decoder(model, cap)
    dec.set_graph(graph)
    kp, vp = synth.past_kv(shape, P)
    fill_cache(dec, kp, vp)
    kc = [kp[l].copy() for l in range(shape.layers)]
    vc = [vp[l].copy() for l in range(shape.layers)]
    trace = torch.zeros((shape.layers, shape.hidden), dtype=torch.float32, device="cuda")
    dec.set_trace(trace)
    emb = synth.input_embeds(shape, steps)
    pos_t = torch.zeros(1, dtype=torch.int32, device="cuda")
    emb_t = torch.zeros(shape.hidden, dtype=torch.float16, device="cuda")
    logits = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    amax = torch.zeros(1, dtype=torch.int32, device="cuda")
    worst = 0.0
    for s in range(steps):
        pos = P + s
        pos_t.fill_(pos)
        emb_t.copy_(dev(emb[s]))
        dec.step(pos_t, input_embeds=emb_t, logits=logits, argmax=amax)
        dec.sync_status()
        ora = odec.decoder_step(cfg, W, emb[s], pos, kc, vc)
        lo = trace.cpu().numpy()
        for l in range(shape.layers):
            e = normwise(lo[l], ora["layer_out"][l])
            worst = max(worst, e)
            assert e <= TOL, f"step {s} layer {l}: {e}"
        e = normwise(logits.cpu().numpy(), ora["logits"])
        assert e <= TOL, f"step {s} logits: {e}"
        ref = ora["logits"]
        top2 = np.sort(ref)[-2:]
        if top2[1] - top2[0] > 1e-2:
            assert int(amax.item()) == ora["argmax"]
        if check_kv:
            # appended K/V: floating point -> contract tolerance; the slot is checked exactly below
            slot = P + s
            kg = dec.k_cache[:, 0, :, slot].cpu().numpy()
            vg = dec.v_cache[:, 0, :, slot].cpu().numpy()
            assert normwise(kg, ora["k_new"]) <= TOL and normwise(vg, ora["v_new"]) <= TOL
        for l in range(shape.layers):
            kc[l] = np.concatenate([kc[l], ora["k_new"][l][:, None, :]], axis=1)
            vc[l] = np.concatenate([vc[l], ora["v_new"][l][:, None, :]], axis=1)
    # untouched slots: past positions bit-identical, beyond length still zero
    n = P + steps
    assert np.array_equal(dec.k_cache[:, 0, :, :P].cpu().numpy(), kp)
    assert torch.count_nonzero(dec.k_cache[:, 0, :, n:]).item() == 0
    assert dec.length == n
    return worst


