"""The measurement arithmetic of bench.py against the figures the workload definition fixes
(CPU only): algorithmic bytes per decode step and FLOPs per prefill."""

import pytest

import bench
import synth

L15, L7 = synth.SHAPE_1P5B, synth.SHAPE_7B


def params_per_layer(s):
    H, D = s.hidden, s.head_dim
    return H * (s.n_q + 2 * s.n_kv) * D + s.n_q * D * H + 3 * H * s.inter


def test_parameter_counts():
    assert params_per_layer(L15) == 46_792_704
    assert params_per_layer(L7) == 233_046_016


def test_prefill_flops_are_two_per_parameter_per_position_plus_causal_attention():
    S = 4530
    f = bench.prefill_flops(L15, S)
    assert f["gemm"] == 2 * S * params_per_layer(L15) * L15.layers  # 1.187e13
    assert f["attention"] == 4 * L15.n_q * L15.head_dim * (S * (S + 1) // 2) * L15.layers
    assert f["gemm"] == pytest.approx(1.187e13, rel=1e-3)
    assert f["attention"] == pytest.approx(1.77e12, rel=3e-3)


@pytest.mark.parametrize("shape,per_pos", [(L15, 28_672), (L7, 57_344)])
def test_step_bytes_grow_by_one_position_of_kv(shape, per_pos):
    assert bench.step_bytes(shape, 1025) - bench.step_bytes(shape, 1024) == per_pos


@pytest.mark.parametrize("shape,P,total", [(L15, 1024, 1.234e9), (L7, 4096, 5.00e9)])
def test_step_bytes_match_the_workload_totals(shape, P, total):
    # packed weights (18 bytes per 32 weights) + fp16 lm_head + KV + small vectors
    b = bench.step_bytes(shape, P)
    assert b == pytest.approx(total, rel=4e-3)
    packed = params_per_layer(shape) * 18 // 32 * shape.layers
    head = shape.vocab * shape.hidden * 2
    kv = 2 * shape.layers * shape.n_kv * P * shape.head_dim * 2
    assert packed + head + kv <= b <= 1.002 * (packed + head + kv)
