"""GPU parity of the decoder (decoder_step / decoder_init through the C ABI) against the oracle.

Contract: every layer output (the residual after the MLP), the logits and the appended K/V within
2e-3 normwise; the append goes to slot P exactly and every other cache slot stays bit-identical;
greedy argmax equal wherever the oracle's top-2 margin exceeds 1e-2.  Multi-step runs
are teacher-forced with the oracle's tokens (trajectories never fork at near-ties).
"""

import numpy as np
import pytest
import torch

import synth
from helpers import TOL, dev, fill_cache, gpu_model, normwise, ocfg, oracle_model, run_steps
from oracle import decoder as odec

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def test_single_layer_ternary_config():
    """One decoder layer, ternary weights, P = 128 at position 128 (one-layer workload)."""
    shape = synth.Shape("layer1", 1536, 1, 12, 2, 128, 8960, 151936, tied=True)
    run_steps(shape, "ternary", 128, 1)


def test_tiny_int4_multistep_graph():
    run_steps(synth.SHAPE_TINY, "int4", 5, 6)


def test_tiny_int4_multistep_no_graph():
    run_steps(synth.SHAPE_TINY, "int4", 70, 3, graph=False)


def test_small_real_dims_multistep():
    run_steps(synth.SHAPE_SMALL, "int4", 1024, 4)


def test_small_ternary_long_context():
    run_steps(synth.SHAPE_SMALL, "ternary", 4530, 2)


def test_wide_hidden_uneven_slices():
    """hidden 2048, 16/2 heads, intermediate 5632: 88 gate/up slices over the SMs (most CTAs
    without one), 16 x 16 o-proj items, and a GEMV input longer than 1536."""
    shape = synth.Shape("wide", 2048, 2, 16, 2, 128, 5632, 4099, tied=True)
    run_steps(shape, "int4", 300, 2)


def test_single_layer_7b_shapes():
    """One decoder layer at 7B shapes (hidden 3584, 28/4 heads, intermediate 18944, untied
    152064-row head): ~31 q/k/v rows per CTA, two gate/up slices per CTA (so the down columns of
    a CTA span two slices), several o-proj items per CTA over two heads."""
    shape = synth.Shape("layer7b", 3584, 1, 28, 4, 128, 18944, 152064, tied=False)
    run_steps(shape, "int4", 128, 1)


def test_graph_and_plain_launches_bit_identical():
    from int4_blockwise_quantised_b200.model import Decoder

    shape = synth.SHAPE_TINY
    model = gpu_model(shape, "int4")
    outs = []
    for graph in (True, False):
        dec = Decoder(model, 64)
        dec.set_graph(graph)
        kp, vp = synth.past_kv(shape, 9)
        fill_cache(dec, kp, vp)
        lg = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
        pos = torch.tensor([9], dtype=torch.int32, device="cuda")
        tok = torch.tensor([17], dtype=torch.int32, device="cuda")
        for _ in range(3):
            dec.step(pos, token=tok, logits=lg)
            pos += 1
        torch.cuda.synchronize()
        outs.append((lg.cpu().numpy().copy(), dec.k_cache.cpu().numpy().copy()))
        dec.close()
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


def test_token_id_input_gathers_embedding():
    from int4_blockwise_quantised_b200.model import Decoder

    shape = synth.SHAPE_TINY
    model = gpu_model(shape, "int4")
    W = oracle_model(shape, "int4")
    dec = Decoder(model, 16)
    kp, vp = synth.past_kv(shape, 3)
    fill_cache(dec, kp, vp)
    lg = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    dec.step(torch.tensor([3], dtype=torch.int32, device="cuda"),
             token=torch.tensor([421], dtype=torch.int32, device="cuda"), logits=lg)
    dec.sync_status()
    ora = odec.decoder_step(ocfg(shape), W, W["embed"][421], 3, list(kp), list(vp))
    assert normwise(lg.cpu().numpy(), ora["logits"]) <= TOL


def test_capacity_and_range_errors():
    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import Decoder

    shape = synth.SHAPE_TINY
    model = gpu_model(shape, "int4")
    dec = Decoder(model, 4, max_position=8)
    pos = torch.tensor([0], dtype=torch.int32, device="cuda")
    tok = torch.tensor([1], dtype=torch.int32, device="cuda")
    for i in range(4):
        pos.fill_(i)
        dec.step(pos, token=tok)
    dec.sync_status()
    with pytest.raises(_vv.VVError) as e:
        dec.step(pos, token=tok)
    assert e.value.code == _vv.VV_ERR_CAPACITY
    with pytest.raises(_vv.VVError):
        dec.set_length(5)
    dec.set_length(0)
    pos.fill_(100)  # outside the RoPE table -> device-side range error, reported at sync
    dec.step(pos, token=tok)
    with pytest.raises(_vv.VVError) as e:
        dec.sync_status()
    assert e.value.code == _vv.VV_ERR_RANGE
    tok.fill_(shape.vocab + 5)
    pos.fill_(1)
    dec.step(pos, token=tok)
    with pytest.raises(_vv.VVError) as e:
        dec.sync_status()
    assert e.value.code == _vv.VV_ERR_RANGE
    dec.sync_status()  # cleared


# ------------------------------------------------------------------------------------ prefill
@pytest.mark.parametrize("shape,mode,S,N", [(synth.SHAPE_TINY, "int4", 37, 20),
                                            (synth.SHAPE_SMALL, "ternary", 70, 40),
                                            (synth.SHAPE_SMALL, "int4", 300, 200),
                                            (synth.Shape("0.5b-2l", 896, 2, 7, 1, 128, 4864,
                                                         2053, tied=True), "int4", 150, 100)])
def test_prefill_then_steps_match_oracle(shape, mode, S, N):
    from int4_blockwise_quantised_b200.model import Decoder

    cfg = ocfg(shape)
    W = oracle_model(shape, mode)
    model = gpu_model(shape, mode)
    ids, pos, feats, off = synth.asr_prompt(shape, N, prefix=7, suffix=S - N - 7)
    dec = Decoder(model, S + 8, max_prefill=S)
    trace = torch.zeros((shape.layers, shape.hidden), dtype=torch.float32, device="cuda")
    dec.set_trace(trace)
    lg = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    am = torch.zeros(1, dtype=torch.int32, device="cuda")
    dec.init(dev(ids), dev(pos), dev(feats), off, logits=lg, argmax=am)
    dec.sync_status()
    ora = odec.decoder_init(cfg, W, ids, pos, feats, off)
    assert dec.length == S
    assert normwise(lg.cpu().numpy(), ora["logits"]) <= TOL
    lo = trace.cpu().numpy()
    for l in range(shape.layers):
        assert normwise(lo[l], ora["layer_out"][l]) <= TOL
    kg = dec.k_cache[:, 0, :, :S].cpu().numpy()
    assert normwise(kg, ora["k"]) <= TOL
    assert normwise(dec.v_cache[:, 0, :, :S].cpu().numpy(), ora["v"]) <= TOL
    # continue decoding from the prefilled cache (teacher-forced with the oracle's argmax)
    kc = [ora["k"][l] for l in range(shape.layers)]
    vc = [ora["v"][l] for l in range(shape.layers)]
    tok = ora["argmax"]
    for s in range(2):
        p = S + s
        dec.step(torch.tensor([p], dtype=torch.int32, device="cuda"),
                 token=torch.tensor([tok], dtype=torch.int32, device="cuda"), logits=lg)
        st = odec.decoder_step(cfg, W, W["embed"][tok], p, kc, vc)
        assert normwise(lg.cpu().numpy(), st["logits"]) <= TOL
        kc = [np.concatenate([kc[l], st["k_new"][l][:, None]], 1) for l in range(shape.layers)]
        vc = [np.concatenate([vc[l], st["v_new"][l][:, None]], 1) for l in range(shape.layers)]
        tok = st["argmax"]


def test_prefill_rejects_bad_splice():
    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import Decoder

    shape = synth.SHAPE_TINY
    dec = Decoder(gpu_model(shape, "int4"), 32, max_prefill=16)
    ids = torch.zeros(10, dtype=torch.int32, device="cuda")
    feats = torch.zeros((5, shape.hidden), dtype=torch.float16, device="cuda")
    with pytest.raises(_vv.VVError) as e:
        dec.init(ids, ids, feats, audio_offset=6)
    assert e.value.code == _vv.VV_ERR_RANGE
    with pytest.raises(_vv.VVError) as e:
        dec.init(torch.zeros(20, dtype=torch.int32, device="cuda"),
                 torch.zeros(20, dtype=torch.int32, device="cuda"))
    assert e.value.code == _vv.VV_ERR_CAPACITY


def test_prefill_full_length_one_layer():
    """One 1.5B-sized layer over a full ASR prompt (S = 4530 positions: 36 row tiles with a
    ragged tail, 71 causal key blocks), int4 weights, checked against the oracle."""
    from int4_blockwise_quantised_b200.model import Decoder

    shape = synth.Shape("layer1", 1536, 1, 12, 2, 128, 8960, 151936, tied=True)
    cfg = ocfg(shape)
    W = oracle_model(shape, "int4")
    model = gpu_model(shape, "int4")
    S = 4530
    N = synth.frames_for_audio(600.0)  # 10 minutes of 24 kHz audio -> 4500 frames
    ids, pos, feats, off = synth.asr_prompt(shape, N, prefix=7, suffix=S - N - 7)
    dec = Decoder(model, S + 8, max_prefill=S)
    trace = torch.zeros((1, shape.hidden), dtype=torch.float32, device="cuda")
    dec.set_trace(trace)
    lg = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    dec.init(dev(ids), dev(pos), dev(feats), off, logits=lg)
    dec.sync_status()
    ora = odec.decoder_init(cfg, W, ids, pos, feats, off)
    assert normwise(lg.cpu().numpy(), ora["logits"]) <= TOL
    assert normwise(trace.cpu().numpy()[0], ora["layer_out"][0]) <= TOL
    assert normwise(dec.k_cache[:, 0, :, :S].cpu().numpy(), ora["k"]) <= TOL
    assert normwise(dec.v_cache[:, 0, :, :S].cpu().numpy(), ora["v"]) <= TOL
    assert torch.count_nonzero(dec.k_cache[:, 0, :, S:]).item() == 0


# --------------------------------------------------------------------------- greedy generate
def test_generate_greedy_loop_on_device():
    """vv_decoder_generate: each step's argmax feeds the next step on the device; the tokens are
    the oracle's greedy choices (teacher-forced with the GPU's own tokens: equal wherever the
    oracle's top-2 margin exceeds 1e-2, else one of its top two), equal to step-by-step decoding,
    and a stop id ends the generation early with the rest of the output untouched."""
    from int4_blockwise_quantised_b200.model import Decoder

    shape = synth.SHAPE_TINY
    cfg = ocfg(shape)
    W = oracle_model(shape, "int4")
    model = gpu_model(shape, "int4")
    P, N = 9, 6
    dec = Decoder(model, P + N + 4)
    kp, vp = synth.past_kv(shape, P)
    fill_cache(dec, kp, vp)
    first = torch.tensor([17], dtype=torch.int32, device="cuda")
    pos = torch.tensor([P], dtype=torch.int32, device="cuda")
    toks, n = dec.generate(first, pos, N)
    dec.sync_status()
    assert n == N and dec.length == P + N
    gen = toks.cpu().numpy().tolist()
    # oracle, teacher-forced with the generated tokens
    kc = [kp[l].copy() for l in range(shape.layers)]
    vc = [vp[l].copy() for l in range(shape.layers)]
    tok = 17
    for i in range(N):
        ora = odec.decoder_step(cfg, W, W["embed"][tok], P + i, kc, vc)
        order = np.argsort(ora["logits"])
        if ora["logits"][order[-1]] - ora["logits"][order[-2]] > 1e-2:
            assert gen[i] == ora["argmax"], (i, gen[i], ora["argmax"])
        else:
            assert gen[i] in (order[-1], order[-2])
        for l in range(shape.layers):
            kc[l] = np.concatenate([kc[l], ora["k_new"][l][:, None, :]], axis=1)
            vc[l] = np.concatenate([vc[l], ora["v_new"][l][:, None, :]], axis=1)
        tok = gen[i]
    # step-by-step decoding from the same state gives the same tokens
    dec.set_length(P)
    t = first.clone()
    p2 = pos.clone()
    seq = []
    for i in range(N):
        dec.step(p2, token=t, argmax=t)
        p2 += 1
        seq.append(int(t.item()))
    assert seq == gen
    # a stop id ends the generation; later entries stay as they were
    stop = gen[2]
    n_exp = gen.index(stop) + 1
    dec.set_length(P)
    out = torch.full((N,), -1, dtype=torch.int32, device="cuda")
    toks2, n2 = dec.generate(first, pos, N, stop_ids=(stop, 151645), tokens_out=out)
    dec.sync_status()
    assert n2 == n_exp and dec.length == P + n_exp
    got = toks2.cpu().numpy().tolist()
    assert got[:n_exp] == gen[:n_exp] and all(v == -1 for v in got[n_exp:])
