"""Pins for the oracle's input activations (int8_linear(input_act=...),
comfy-kitchen 0.2.40 "HIP backend": the activation is folded into the fused
ConvRot quantiser's load). The pages do not list the activations; the ones
built are relu, silu and the tanh form of gelu, each in fp32 on the widened
bf16 input and rounded to bf16 before the rotation. The oracle's own e^x is
checked against float64 exp; the activations against float64 formulas and
torch's bf16 implementations; the wiring against torch's exact relu."""
import numpy as np
import pytest
import torch

import oracle
import workloads


def ulps32(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    a = np.where(a < 0, np.int64(-2 ** 31) - a, a)
    b = np.where(b < 0, np.int64(-2 ** 31) - b, b)
    return np.abs(a - b)


def test_exp_matches_float64_within_4_ulp():
    x = np.concatenate([np.linspace(-87.0, 88.5, 40001, dtype=np.float32),
                        np.float32([0.0, -0.0, 1e-30, -1e-30, 0.34657359, -0.34657359])])
    got = oracle.exp(x)
    ref = np.exp(x.astype(np.float64)).astype(np.float32)
    assert ulps32(got, ref).max() <= 4


def test_exp_special_values():
    x = np.float32([-200.0, -104.5, 89.0, 200.0, 0.0, 1.0])
    got = oracle.exp(x)
    assert got[0] == 0.0 and got[1] == 0.0
    assert np.isinf(got[2]) and np.isinf(got[3])
    assert got[4] == 1.0
    assert ulps32(got[5], np.float32(np.e)) <= 1


def test_exp_subnormal_range_absolute_error():
    x = np.linspace(-103.9, -87.4, 2001, dtype=np.float32)
    got = oracle.exp(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    assert np.all(np.abs(got - ref) <= 2.0 ** -149 * 2 + ref * 2.0 ** -22)


def _x():
    rng = np.random.default_rng(3)
    return np.concatenate([rng.standard_normal(20000).astype(np.float32) * 3,
                           np.float32([0.0, -0.0, 50.0, -50.0, 100.0, -100.0, 1e-20, -1e-20])])


def test_relu_exact():
    x = _x()
    assert np.array_equal(oracle.act("relu", x), np.maximum(x, np.float32(0)))


def test_silu_matches_float64():
    x = _x()
    ref = (x.astype(np.float64) / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)
    got = oracle.act("silu", x)
    big = np.abs(ref) > 1e-30
    assert ulps32(got[big], ref[big]).max() <= 8
    assert got[-1] == ref[-1] or abs(got[-1]) < 1e-19


def test_gelu_tanh_matches_float64():
    x = _x()
    xd = x.astype(np.float64)
    u = np.sqrt(2.0 / np.pi) * (xd + 0.044715 * xd ** 3)
    # 0.5 x (1 + tanh(u)) written without the cancellation near tanh(u) = -1
    with np.errstate(over="ignore"):  # e^(-2u) = inf for very negative x: ref -> -0
        ref = xd / (1.0 + np.exp(-2.0 * u))
    got = oracle.act("gelu_tanh", x).astype(np.float64)
    # fp32 rounding of the argument 2u is amplified by e^(-2u): relative error
    # grows with |2u| (conditioning, not the method)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * (2.0 ** -19 + np.abs(2 * u) * 2.0 ** -21) + 1e-37)
    # and it is the tanh form: 0.5 x (1 + tanh(u)) where that is well conditioned
    ok = xd > -3.0
    tanh_form = 0.5 * xd * (1.0 + np.tanh(u))
    assert np.all(np.abs(got[ok] - tanh_form[ok]) <= np.abs(tanh_form[ok]) * 2.0 ** -18 + 1e-30)


@pytest.mark.parametrize("name,fn", [
    ("silu", lambda t: torch.nn.functional.silu(t)),
    ("gelu_tanh", lambda t: torch.nn.functional.gelu(t, approximate="tanh")),
])
def test_bf16_activation_close_to_torch(name, fn):
    # torch's tanh-form gelu underflows to 0 below about x = -5 (1 + tanh(u)
    # cancels in fp32); compare where both are accurate
    xs = _x()
    x = torch.from_numpy(xs[xs > -4.0]).to(torch.bfloat16)
    mine = oracle.f32_to_bf16(oracle.act(name, x.float().numpy()))
    theirs = workloads.bf16_bits(fn(x.float()).to(torch.bfloat16))
    d = np.abs(mine.astype(np.int32) - theirs.astype(np.int32))
    assert (d <= 1).all()
    assert (d != 0).mean() < 0.01


def test_quantize_with_relu_equals_quantize_of_torch_relu():
    cfg = workloads.custom(6, 768, 8, seed=9)
    X, _, _ = workloads.make_inputs(cfg)
    a = oracle.quantize_rows_bf16(workloads.bf16_bits(X), act="relu")
    b = oracle.quantize_rows_bf16(workloads.bf16_bits(torch.relu(X)))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("name", ["silu", "gelu_tanh"])
def test_quantize_with_act_equals_quantize_of_rounded_act(name):
    cfg = workloads.custom(5, 512, 8, seed=10)
    X, _, _ = workloads.make_inputs(cfg)
    a_bits = oracle.f32_to_bf16(oracle.act(name, X.float().numpy()))
    a = oracle.quantize_rows_bf16(workloads.bf16_bits(X), act=name)
    b = oracle.quantize_rows_bf16(a_bits)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
