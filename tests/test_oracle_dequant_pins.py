"""Pins for the oracle's dequantize_int8_simple(_dtype) and
quantize_int8_tensorwise (comfy-kitchen 0.2.40, "Huawei Ascend backend";
ComfyUI-AppleSilicon-FP8 README row 17: tensorwise quantisation before ConvRot
is the ~16% error negative control)."""
import numpy as np
import torch

import oracle
import workloads


def test_dequantize_is_a_single_fp32_rounding():
    rng = np.random.default_rng(2)
    Q = rng.integers(-127, 128, size=(9, 256)).astype(np.int8)
    s = rng.uniform(1e-4, 1.0, 9).astype(np.float32)
    Yf, Yb = oracle.dequantize_int8(Q, s, per_row=True)
    ref = (Q.astype(np.float64) * s[:, None].astype(np.float64)).astype(np.float32)  # exact product rounded once
    assert np.array_equal(Yf, ref)
    assert np.array_equal(Yb, workloads.bf16_bits(torch.from_numpy(ref).to(torch.bfloat16)))
    Yf1, _ = oracle.dequantize_int8(Q, s[:1], per_row=False)
    assert np.array_equal(Yf1, (Q.astype(np.float64) * np.float64(s[0])).astype(np.float32))


def test_tensorwise_quant_bound_and_scale():
    cfg = workloads.custom(6, 512, 8, seed=12)
    X, _, _ = workloads.make_inputs(cfg)
    x = X.float().numpy().astype(np.float64)
    Q, s = oracle.quantize_int8_tensorwise(workloads.bf16_bits(X))
    assert s == np.float32(np.float32(np.abs(x).max()) / np.float32(127))
    assert np.abs(Q.astype(np.int32)).max() == 127
    err = np.abs(Q.astype(np.float64) * np.float64(s) - x)
    assert np.all(err <= np.float64(s) * (0.5 + 128 * 2.0 ** -23))


def test_tensorwise_round_trip_golden():
    """x = 127 at one place makes s = 1: codes are round-half-even(x)."""
    x = np.zeros((2, 256), np.float32)
    x[0, :6] = [127.0, 2.5, -2.5, 3.5, 0.5, -126.5]
    X = torch.from_numpy(x).to(torch.bfloat16)
    Q, s = oracle.quantize_int8_tensorwise(workloads.bf16_bits(X))
    assert s == 1.0 and list(Q[0, :6]) == [127, 2, -2, 4, 0, -126] and not Q[1].any()
