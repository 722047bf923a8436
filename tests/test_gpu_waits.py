"""Failure detection on the device without a GPU fault: every wait in the kernels is bounded.

vv_wait_selftest runs the two wait helpers the kernels use (the stage-ring mbarrier wait and the
grid-barrier counter poll) against a signal that never comes, with a 1 ms limit; the wait must
give up, record VV_ERR_TIMEOUT in the device error word (reported once by vv_sync_status) and
leave the context usable: a decoder step afterwards runs clean and matches the oracle."""

import time

import numpy as np
import pytest
import torch

import synth
from helpers import TOL, gpu_model, normwise, ocfg, oracle_model
from oracle import decoder as odec

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1])
def test_wait_times_out_and_reports(which):
    from int4_blockwise_quantised_b200 import _vv

    assert torch.cuda.is_available()
    scratch = torch.zeros(4, dtype=torch.int32, device="cuda")
    _vv.vv_sync_status()  # start clean
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    _vv.vv_wait_selftest(which, 1_000_000, scratch)
    with pytest.raises(_vv.VVError) as e:
        _vv.vv_sync_status()
    dt = time.perf_counter() - t0
    assert e.value.code == _vv.VV_ERR_TIMEOUT
    assert 1e-3 <= dt < 1.0, dt  # gave up after its own limit, not the 2 s default
    _vv.vv_sync_status()  # the word was cleared by the report


def test_argument_checks():
    from int4_blockwise_quantised_b200 import _vv

    assert _vv.lib.vv_wait_selftest(2, 1_000_000, None, None) == _vv.VV_ERR_INVALID_ARG
    assert _vv.lib.vv_wait_selftest(0, 10, None, None) == _vv.VV_ERR_INVALID_ARG
    assert _vv.lib.vv_wait_selftest(1, 1_000_000, None, None) == _vv.VV_ERR_INVALID_ARG


def test_decoder_runs_clean_after_a_timeout():
    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import Decoder

    _vv.vv_wait_selftest(0, 1_000_000)
    with pytest.raises(_vv.VVError):
        _vv.vv_sync_status()
    shape = synth.SHAPE_TINY
    W = oracle_model(shape, "int4")
    dec = Decoder(gpu_model(shape, "int4"), 16)
    kp, vp = synth.past_kv(shape, 5)
    dec.k_cache[:, 0, :, :5] = torch.from_numpy(kp).cuda()
    dec.v_cache[:, 0, :, :5] = torch.from_numpy(vp).cuda()
    dec.set_length(5)
    lg = torch.zeros(shape.vocab, dtype=torch.float32, device="cuda")
    emb = synth.input_embeds(shape)[0]
    dec.step(torch.tensor([5], dtype=torch.int32, device="cuda"),
             input_embeds=torch.from_numpy(emb).cuda(), logits=lg)
    dec.sync_status()
    ora = odec.decoder_step(ocfg(shape), W, emb, 5, list(kp), list(vp))
    assert normwise(lg.cpu().numpy(), ora["logits"]) <= TOL
