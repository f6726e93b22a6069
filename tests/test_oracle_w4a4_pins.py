"""Pins for the oracle's convrot_w4a4_linear (comfy-kitchen 0.2.40, "Huawei
Ascend backend": ConvRot then signed INT4 quantisation of both operands,
activation codes in INT8 storage, packed weights unpacked to INT8 for INT32
accumulation; ComfyUI-AppleSilicon-FP8 README row 22 reports about 22.5%
relative error for ConvRot W4A4 on a real model, far above INT8's)."""
import json
import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_int4_ties_golden():
    g = json.load(open(os.path.join(GOLDEN, "int4_ties_and_nibbles.json")))
    row = np.zeros(g["K"], np.float32)
    row[: len(g["row"])] = g["row"]
    q, s = oracle.quant_rows(row[None, :], qmax=7)
    assert s[0] == np.float32(1.0)
    codes = np.zeros(g["K"], np.int8)
    codes[: len(g["codes"])] = g["codes"]
    assert np.array_equal(q[0], codes)


def test_unpack_nibbles_golden():
    g = json.load(open(os.path.join(GOLDEN, "int4_ties_and_nibbles.json")))
    b = np.array(g["bytes"], np.uint8)[None, :]
    assert list(oracle.unpack_int4(b)[0]) == g["unpacked"]


def test_unpack_all_bytes_brute_force():
    b = np.arange(256, dtype=np.uint8)[None, :]
    u = oracle.unpack_int4(b)[0]
    for v in range(256):
        lo, hi = v & 15, v >> 4
        assert u[2 * v] == (lo - 16 if lo >= 8 else lo)
        assert u[2 * v + 1] == (hi - 16 if hi >= 8 else hi)


def test_int4_error_bound_and_range():
    rng = np.random.default_rng(1)
    y = rng.standard_normal((64, 512)).astype(np.float32)
    y[::3, 5] = 30.0
    q, s = oracle.quant_rows(y, qmax=7)
    assert q.min() >= -7 and q.max() <= 7
    assert np.all(np.abs(q.astype(np.int32)).max(axis=1) == 7)
    err = np.abs(q.astype(np.float64) * s[:, None] - y.astype(np.float64))
    assert np.all(err <= s[:, None].astype(np.float64) * (0.5 + 8 * 2.0 ** -23))


def test_int4_weights_are_rotated_codes_packed():
    cfg = workloads.custom(1, 768, 40, seed=4)
    _, W, _ = workloads.make_inputs(cfg)
    q4, s4 = oracle.rotate_quant_weight_int4(W.numpy())
    y = oracle.rot256(W.numpy().reshape(-1, 256)).reshape(W.shape)
    q, s = oracle.quant_rows(y, qmax=7)
    assert np.array_equal(oracle.unpack_int4(q4), q) and np.array_equal(s4, s)


def test_w4a4_linear_brute_force():
    cfg = workloads.custom(5, 512, 7 * 8, seed=6)
    X, W, bias = workloads.make_inputs(cfg)
    q4, s4 = oracle.rotate_quant_weight_int4(W.numpy())
    Y, Qx, s_x, acc = oracle.convrot_w4a4_linear(workloads.bf16_bits(X), q4, s4,
                                                 workloads.bf16_bits(bias))
    Qw = oracle.unpack_int4(q4)
    for m in range(Qx.shape[0]):
        for n in range(0, Qw.shape[0], 7):
            assert acc[m, n] == sum(int(a) * int(b) for a, b in zip(Qx[m], Qw[n]))
    assert np.abs(Qx).max() <= 7


def test_w4a4_error_band():
    """Much coarser than INT8 (about 22.5% on the page's model), still a
    useful approximation of X W^T."""
    cfg = workloads.CONFIGS[0]
    X, W, bias = workloads.make_inputs(cfg)
    xd, wd = X.double().numpy(), W.double().numpy()
    ref = xd @ wd.T + bias.double().numpy()[None, :]
    q4, s4 = oracle.rotate_quant_weight_int4(W.numpy())
    Y4 = oracle.bf16_to_f32(oracle.convrot_w4a4_linear(workloads.bf16_bits(X), q4, s4,
                                                       workloads.bf16_bits(bias))[0])
    Qw, s_w = oracle.rotate_quant_weight(W.numpy())
    Y8 = oracle.bf16_to_f32(oracle.int8_linear(workloads.bf16_bits(X), Qw, s_w,
                                               workloads.bf16_bits(bias))[0])
    e4 = np.linalg.norm(Y4 - ref) / np.linalg.norm(ref)
    e8 = np.linalg.norm(Y8 - ref) / np.linalg.norm(ref)
    assert 0.05 < e4 < 0.5, e4
    assert e4 > 4 * e8, (e4, e8)
