"""Batch-2 decode: two sequences stepped together by one persistent step kernel, the CFG pair of
"VibeVoice-1.5B — Current Status" (a negative context stepped alongside the positive one) or
two independent streams.  Each sequence has its own past length, position, input, KV cache
slice [L, b, Hkv, cap, D], logits and argmax; each is checked against the batch-1 oracle on its
own inputs (2e-3 normwise on the logits and the appended K/V; layer outputs of sequence 0)."""

import numpy as np
import pytest
import torch

import synth
from helpers import TOL, dev, gpu_model, normwise, ocfg, oracle_model
from oracle import decoder as odec
from oracle import ops as oops

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def run_pair(shape, mode, Ps, steps, kv=(torch.float16, np.float16), tokens=False):
    from int4_blockwise_quantised_b200.model import Decoder

    tdt, odt = kv
    cfg = ocfg(shape)
    W = oracle_model(shape, mode)
    model = gpu_model(shape, mode)
    L, B = shape.layers, 2
    dec = Decoder(model, max(Ps) + steps + 8, kv_dtype=tdt, batch=B)
    assert dec.batch == 2
    pasts = [synth.past_kv(shape, Ps[b], base=17 * b) for b in range(B)]
    kc, vc = [], []
    for b in range(B):
        kp, vp = pasts[b]
        dec.k_cache[:, b, :, :Ps[b]] = dev(kp).to(tdt)
        dec.v_cache[:, b, :, :Ps[b]] = dev(vp).to(tdt)
        kc.append([oops.kv_round(kp[l], odt) for l in range(L)])
        vc.append([oops.kv_round(vp[l], odt) for l in range(L)])
    dec.set_lengths(Ps)
    assert [dec.sequence_length(b) for b in range(B)] == list(Ps)
    trace = torch.zeros((L, shape.hidden), dtype=torch.float32, device="cuda")
    dec.set_trace(trace)
    embs = [synth.input_embeds(shape, steps, base=5 * b) for b in range(B)]
    toks = [[(101 + 37 * s + 911 * b) % shape.vocab for s in range(steps)] for b in range(B)]
    pos_t = torch.zeros(B, dtype=torch.int32, device="cuda")
    emb_t = torch.zeros((B, shape.hidden), dtype=torch.float16, device="cuda")
    tok_t = torch.zeros(B, dtype=torch.int32, device="cuda")
    logits = torch.zeros((B, shape.vocab), dtype=torch.float32, device="cuda")
    amax = torch.zeros(B, dtype=torch.int32, device="cuda")
    worst = 0.0
    for s in range(steps):
        for b in range(B):
            pos_t[b] = Ps[b] + s
            if tokens:
                tok_t[b] = toks[b][s]
            else:
                emb_t[b] = dev(embs[b][s])
        if tokens:
            dec.step(pos_t, token=tok_t, logits=logits, argmax=amax)
        else:
            dec.step(pos_t, input_embeds=emb_t, logits=logits, argmax=amax)
        dec.sync_status()
        lg = logits.cpu().numpy()
        for b in range(B):
            x = W["embed"][toks[b][s]] if tokens else embs[b][s]
            ora = odec.decoder_step(cfg, W, x, Ps[b] + s, kc[b], vc[b], kv_dtype=odt)
            e = normwise(lg[b], ora["logits"])
            worst = max(worst, e)
            assert e <= TOL, f"step {s} seq {b} logits: {e}"
            ref = ora["logits"]
            top2 = np.sort(ref)[-2:]
            if top2[1] - top2[0] > 1e-2:
                assert int(amax[b].item()) == ora["argmax"], (s, b)
            slot = Ps[b] + s
            kg = dec.k_cache[:, b, :, slot].float().cpu().numpy()
            vg = dec.v_cache[:, b, :, slot].float().cpu().numpy()
            assert normwise(kg, ora["k_new"]) <= TOL and normwise(vg, ora["v_new"]) <= TOL
            if b == 0:
                lo = trace.cpu().numpy()
                for l in range(L):
                    assert normwise(lo[l], ora["layer_out"][l]) <= TOL, (s, l)
            for l in range(L):
                kc[b][l] = np.concatenate([kc[b][l], ora["k_new"][l][:, None]], 1)
                vc[b][l] = np.concatenate([vc[b][l], ora["v_new"][l][:, None]], 1)
    for b in range(B):
        assert dec.sequence_length(b) == Ps[b] + steps
        # past slots untouched, slots beyond the length still zero
        kp, _ = pasts[b]
        assert torch.equal(dec.k_cache[:, b, :, :Ps[b]], dev(kp).to(tdt))
        assert torch.count_nonzero(dec.k_cache[:, b, :, Ps[b] + steps:]).item() == 0
    return worst


def test_batch2_small_different_lengths():
    """2 layers at 1.5B widths, pasts of 300 and 517 positions (different tile counts per
    sequence), seeded embeddings, 4 steps."""
    run_pair(synth.SHAPE_SMALL, "int4", (300, 517), 4)


def test_batch2_token_inputs_ternary():
    """Token-id inputs (embedding rows gathered on the device per sequence), ternary weights."""
    run_pair(synth.SHAPE_SMALL, "ternary", (64, 1), 3, tokens=True)


def test_batch2_fp32_cache():
    """The fp32-KV variant with two sequences (4-byte rows: 32-position tiles)."""
    run_pair(synth.SHAPE_TINY, "int4", (200, 90), 3, kv=(torch.float32, np.float32))


def test_batch2_full_1p5b():
    """The 28-layer 1.5B decoder at batch 2 (full vocabulary, tied head), pasts 1024 and 700."""
    run_pair(synth.SHAPE_1P5B, "int4", (1024, 700), 2)


def test_batch2_rejects_bad_batch_and_generate():
    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import Decoder

    model = gpu_model(synth.SHAPE_TINY, "int4")
    with pytest.raises(_vv.VVError) as e:
        Decoder(model, 64, batch=3)
    assert e.value.code == _vv.VV_ERR_SHAPE
    dec = Decoder(model, 64, batch=2)
    with pytest.raises(_vv.VVError) as e:
        dec.generate(torch.zeros(1, dtype=torch.int32, device="cuda"),
                     torch.zeros(1, dtype=torch.int32, device="cuda"), 4)
    assert e.value.code == _vv.VV_ERR_SHAPE
    ids = torch.zeros(8, dtype=torch.int32, device="cuda")
    with pytest.raises(_vv.VVError) as e:
        dec.init(ids, ids, seq=2)
    assert e.value.code == _vv.VV_ERR_INVALID_ARG


def test_batch2_prefill_each_sequence_then_step():
    """The CFG pair from two prompts: each sequence prefilled into its own cache slice
    (vv_decoder_init_seq), then batch-2 steps, every result against the oracle per sequence."""
    from int4_blockwise_quantised_b200.model import Decoder

    shape, mode = synth.SHAPE_SMALL, "int4"
    cfg = ocfg(shape)
    W = oracle_model(shape, mode)
    model = gpu_model(shape, mode)
    L, B = shape.layers, 2
    prompts = [synth.asr_prompt(shape, 40, prefix=7, suffix=23), synth.asr_prompt(shape, 20, prefix=5,
                                                                               suffix=12, base=3)]
    Ss = [p[0].size for p in prompts]
    dec = Decoder(model, max(Ss) + 8, max_prefill=max(Ss), batch=B)
    lg1 = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    kc, vc, toks = [], [], []
    for b in range(B):
        ids, pos, feats, off = prompts[b]
        dec.init(dev(ids), dev(pos), dev(feats), off, logits=lg1, seq=b)
        dec.sync_status()
        ora = odec.decoder_init(cfg, W, ids, pos, feats, off)
        assert normwise(lg1.cpu().numpy(), ora["logits"]) <= TOL
        assert dec.sequence_length(b) == Ss[b]
        assert normwise(dec.k_cache[:, b, :, :Ss[b]].cpu().numpy(), ora["k"]) <= TOL
        kc.append([ora["k"][l] for l in range(L)])
        vc.append([ora["v"][l] for l in range(L)])
        toks.append(ora["argmax"])
    # the other sequence's slice stays untouched by each prefill
    assert torch.count_nonzero(dec.k_cache[:, 1, :, Ss[1]:]).item() == 0
    logits = torch.zeros((B, shape.vocab), dtype=torch.float32, device="cuda")
    for s in range(2):
        pos_t = torch.tensor([Ss[b] + s for b in range(B)], dtype=torch.int32, device="cuda")
        tok_t = torch.tensor(toks, dtype=torch.int32, device="cuda")
        dec.step(pos_t, token=tok_t, logits=logits)
        dec.sync_status()
        lg = logits.cpu().numpy()
        for b in range(B):
            st = odec.decoder_step(cfg, W, W["embed"][toks[b]], Ss[b] + s, kc[b], vc[b])
            assert normwise(lg[b], st["logits"]) <= TOL, (s, b)
            kc[b] = [np.concatenate([kc[b][l], st["k_new"][l][:, None]], 1) for l in range(L)]
            vc[b] = [np.concatenate([vc[b][l], st["v_new"][l][:, None]], 1) for l in range(L)]
            toks[b] = st["argmax"]
