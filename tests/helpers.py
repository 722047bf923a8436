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
