"""Parity at full depth and at the stated decode configurations (the pages' evidence is
token-exactness and KV-incremental == full recompute at the real model depth: "vibevoice-asr-
bitnet-onnx", tier table; "VibeVoice-1.5B — Current Status", "Inference (ONNX)").

Every test is teacher-forced: each step's input is the oracle's previous argmax embedding (or a
seeded embedding), every layer output and the logits are compared at 2e-3 normwise."""

import pytest
import torch

import synth
from helpers import run_steps

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def need_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def test_decode_1p5b_28_layers_p1024():
    """The 28-layer 1.5B decoder_step as the benchmark runs it (int4 symmetric block-32 weights,
    tied 151936-row fp16 head, past P = 1024), 8 appended steps, all 28 layer outputs each step."""
    run_steps(synth.SHAPE_1P5B, "int4", 1024, 8)


def test_decode_7b_two_layers_p4096():
    """7B shapes with two layers at P = 4096: 4 KV heads x 65 attention tiles (two items on some
    CTAs), 784 o-proj items (several per CTA, crossing heads), two gate/up slices per CTA."""
    shape = synth.Shape("7b-2l", 3584, 2, 28, 4, 128, 18944, 152064, tied=False)
    run_steps(shape, "int4", 4096, 2)


def test_decode_asr_ternary_across_p4736():
    """ASR-shaped long context, ternary weights: steps from P = 4731 to 4738 cross the point
    (past + 1 = 4737) where the 2 KV heads need 150 attention tiles, more than one per CTA."""
    run_steps(synth.SHAPE_SMALL, "ternary", 4731, 8)


def test_decode_realtime_0p5b_20_layers():
    """The Realtime-0.5B backbone at full depth (20 layers, hidden 896 = 7 column blocks of the
    o-proj image, one KV head of 7 query heads, 76 gate/up slices on 148 CTAs), P = 512, 4 steps."""
    run_steps(synth.SHAPE_0P5B, "int4", 512, 4)
