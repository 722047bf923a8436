"""The scratch-free attention entry point (vv_gqa_decode_attn_noalloc) against the workspace one.

vv_gqa_decode_attn_noalloc serves callers that cannot allocate device memory when they run
attention; it keeps its split-K scratch in a static device array instead of a caller workspace.
This file is collected last so that a failure here never hides the other tests; it must pass on
its own in a fresh process as well as after them.  Two calls in a row (different lengths, so the
second reuses the array the first one left behind) are compared with vv_gqa_decode_attn and
directly with the oracle's grouped-query attention.
"""

import math

import numpy as np
import pytest
import torch

import synth
from helpers import TOL, normwise
from oracle import ops

pytestmark = pytest.mark.gpu


def test_noalloc_attention_matches_workspace_entry_point():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from int4_blockwise_quantised_b200 import _vv

    Hq, Hkv, D, cap = 12, 2, 128, 1984  # the largest 2-KV-head cache the 256 KiB scratch serves
    K = torch.from_numpy(synth.normal_f16((Hkv, cap, D), 1.0, 71)).cuda()
    V = torch.from_numpy(synth.normal_f16((Hkv, cap, D), 1.0, 72)).cuda()
    ws = torch.zeros(_vv.vv_gqa_decode_attn_workspace_size(Hq, Hkv, D, cap), dtype=torch.uint8,
                     device="cuda")
    for call, (length, seed) in enumerate([(1984, 73), (1025, 74)]):
        q = torch.from_numpy(synth.normal_f16((Hq, D), 1.0, seed)).cuda()
        ref = _vv.vv_gqa_decode_attn(q, K, V, length, 1 / math.sqrt(D), ws)
        got = _vv.vv_gqa_decode_attn_noalloc(q, K, V, length, 1 / math.sqrt(D))
        _vv.vv_sync_status()
        e = normwise(got.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64))
        assert e <= TOL, f"call {call}: normwise difference {e}"
        ora = ops.gqa_decode_attention(q.cpu().numpy(), K[:, :length].cpu().numpy(),
                                       V[:, :length].cpu().numpy(), 1 / math.sqrt(D))
        e = normwise(got.cpu().numpy().astype(np.float64), ora)
        assert e <= TOL, f"call {call}: normwise error against the oracle {e}"


def test_noalloc_attention_rejects_oversized_scratch():
    from int4_blockwise_quantised_b200 import _vv

    # a 4800-position cache with 2 KV heads needs more split-K partials than the 256 KiB array
    # holds (the chunk count depends on the SM count; the workspace size says how many)
    assert _vv.vv_gqa_decode_attn_workspace_size(12, 2, 128, 4800) > 256 * 1024
    q = torch.zeros((12, 128), dtype=torch.float16, device="cuda")
    kv = torch.zeros((2, 4800, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(_vv.VVError) as e:
        _vv.vv_gqa_decode_attn_noalloc(q, kv, kv, 4785, 0.1)
    assert e.value.code == _vv.VV_ERR_CAPACITY
