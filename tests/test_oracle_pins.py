"""Pins for the CPU oracle: checks against closed forms, invariants, brute
force and an independent library, so that a plausible mistake anywhere in the
oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
rounding) fails one of them. CPU only.

Sources (page title, section):
  - sglang PR "Tune Kitchen INT8 row splitting for SM120", Accuracy Test:
    BF16 activations and bias, INT8 weights, FP32 row scales, ConvRot256; the
    split and single-call outputs are bit-exact.
  - ComfyUI-AppleSilicon-FP8 README, "What it fixes" row 17: rotate online,
    per-row quantise, INT8 x INT8 -> INT32, per-row rescale + bias epilogue;
    tensorwise quantisation before ConvRot gives about 16% error; row 12: the
    INT32 sums stay inside the int32 range.
  - comfy-kitchen 0.2.40, "Huawei Ascend backend": quantize_int8_rowwise,
    quantize_and_rotate_rowwise, int8_linear.
"""
import json
import os

import numpy as np
import pytest
import torch

import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def popcount(x: int) -> int:
    return bin(x).count("1")


# ---------------------------------------------------------------- rotation


def test_rot256_basis_is_sylvester_hadamard_over_16(oracle_lib):
    """rot256(e_i)[j] == (-1)^popcount(i & j) / 16 exactly, for every i, j.
    Pins stage order/pairing (a wrong pairing gives another matrix) and the
    1/16 normalisation."""
    eye = np.eye(256, dtype=np.float32)
    H = oracle_lib.rot256(eye)  # row i = rot256(e_i)
    ref = np.array([[(-1.0) ** popcount(i & j) / 16.0 for j in range(256)] for i in range(256)])
    assert np.array_equal(H.astype(np.float64), ref)


def test_rot256_orthonormal_exact(oracle_lib):
    """H H^T = I exactly: entries are +-1/16, products and sums are exact."""
    H = oracle_lib.rot256(np.eye(256, dtype=np.float32)).astype(np.float64)
    assert np.array_equal(H @ H.T, np.eye(256))


def test_rot256_is_an_involution_on_small_integers(oracle_lib):
    rng = np.random.default_rng(7)
    x = rng.integers(-8, 9, size=(16, 256)).astype(np.float32)
    y = oracle_lib.rot256(x)
    assert np.array_equal(oracle_lib.rot256(y), x)


def test_rot256_parseval(oracle_lib):
    rng = np.random.default_rng(8)
    x = rng.standard_normal((32, 256)).astype(np.float32)
    y = oracle_lib.rot256(x).astype(np.float64)
    nx = np.linalg.norm(x.astype(np.float64), axis=1)
    ny = np.linalg.norm(y, axis=1)
    assert np.allclose(nx, ny, rtol=1e-6, atol=0)


def test_rot256_constant_goes_to_dc(oracle_lib):
    c = np.float32(1.5)
    y = oracle_lib.rot256(np.full(256, c, np.float32))
    ref = np.zeros(256, np.float32)
    ref[0] = 16 * c
    assert np.array_equal(y, ref)


def test_rot256_matches_fp64_matrix_product(oracle_lib):
    """fp32 butterfly within a few fp32 ulps of the exact fp64 product H x."""
    H = np.array([[(-1.0) ** popcount(i & j) / 16.0 for j in range(256)] for i in range(256)])
    rng = np.random.default_rng(9)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    y = oracle_lib.rot256(x).astype(np.float64)
    ref = x.astype(np.float64) @ H.T
    scale = np.abs(x).sum(axis=1, keepdims=True) / 16.0
    assert np.all(np.abs(y - ref) <= 8 * 2.0 ** -24 * scale * 8)


@pytest.mark.parametrize("cfg", [
    workloads.CONFIGS[0],
    workloads.custom(64, 5376, 96, seed=11),
    workloads.custom(32, 28672, 48, seed=12, x_dist="laplace", w_std=0.01),
])
def test_rotation_preserves_the_gemm(oracle_lib, cfg):
    """(X H)(W H)^T == X W^T within 1e-4 relative (Frobenius), both in fp64
    from the same inputs; H is applied block by block along K."""
    X, W, _ = workloads.make_inputs(cfg)
    x = X.float().numpy()
    w = W.numpy()
    xr = oracle_lib.rot256(x.reshape(-1, 256)).reshape(x.shape).astype(np.float64)
    wr = oracle_lib.rot256(w.reshape(-1, 256)).reshape(w.shape).astype(np.float64)
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    got = xr @ wr.T
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 1e-4, rel


# ---------------------------------------------------------------- quantiser


def test_quant_ties_to_even_golden(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "quant_ties_to_even.json")))
    row = np.zeros(g["K"], np.float32)
    row[: len(g["row"])] = g["row"]
    q, s = oracle_lib.quant_rows(row[None, :])
    assert s[0] == np.float32(g["scale"])
    codes = np.zeros(g["K"], np.int8)
    codes[: len(g["codes"])] = g["codes"]
    assert np.array_equal(q[0], codes)
    # the same row through the BF16 entry point without rotation
    xb = torch.from_numpy(row[None, :]).to(torch.bfloat16)
    q2, s2 = oracle_lib.quantize_rows_bf16(workloads.bf16_bits(xb), rotate=False)
    assert np.array_equal(q2[0], codes) and s2[0] == np.float32(1.0)


def _rand_rows(seed, R=64, K=512):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((R, K)).astype(np.float32)
    y[::7] *= np.float32(1e-3)
    y[1::5, 3] = np.float32(40.0)  # outliers
    return y


def test_quant_dequant_error_at_most_half_scale(oracle_lib):
    y = _rand_rows(1)
    q, s = oracle_lib.quant_rows(y)
    err = np.abs(q.astype(np.float64) * s[:, None].astype(np.float64) - y.astype(np.float64))
    # half a step, plus the fp32 rounding of the quotient y/s (|y/s| <= 127)
    bound = s[:, None].astype(np.float64) * (0.5 + 128 * 2.0 ** -23)
    assert np.all(err <= bound)


def test_quant_range_and_full_scale_hit(oracle_lib):
    y = _rand_rows(2)
    q, s = oracle_lib.quant_rows(y)
    assert q.min() >= -127 and q.max() <= 127
    assert np.all(np.abs(q.astype(np.int32)).max(axis=1) == 127)
    assert np.all(s > 0)


def test_quant_is_odd(oracle_lib):
    y = _rand_rows(3)
    q, s = oracle_lib.quant_rows(y)
    qn, sn = oracle_lib.quant_rows(-y)
    assert np.array_equal(qn.astype(np.int32), -q.astype(np.int32))
    assert np.array_equal(sn, s)


@pytest.mark.parametrize("k", [-20, -3, 1, 5, 30])
def test_quant_power_of_two_scale_invariance(oracle_lib, k):
    y = _rand_rows(4)
    q, s = oracle_lib.quant_rows(y)
    f = np.float32(2.0 ** k)
    q2, s2 = oracle_lib.quant_rows(y * f)
    assert np.array_equal(q2, q)
    assert np.array_equal(s2, s * f)


def test_quant_zero_row(oracle_lib):
    y = np.zeros((2, 256), np.float32)
    y[1, 5] = np.float32(-0.0)
    q, s = oracle_lib.quant_rows(y)
    assert np.all(q == 0) and np.all(s == 0)


def test_quantize_rotate_equals_rotation_then_quant(oracle_lib):
    cfg = workloads.custom(9, 768, 8, seed=5)
    X, _, _ = workloads.make_inputs(cfg)
    Qx, s_x = oracle_lib.quantize_rows_bf16(workloads.bf16_bits(X))
    y = oracle_lib.rot256(X.float().numpy().reshape(-1, 256)).reshape(X.shape)
    q, s = oracle_lib.quant_rows(y)
    assert np.array_equal(Qx, q) and np.array_equal(s_x, s)


def test_quantize_rows_respects_row_stride(oracle_lib):
    cfg = workloads.custom(5, 512, 8, seed=6)
    X, _, _ = workloads.make_inputs(cfg)
    xb = workloads.bf16_bits(X)
    wide = np.full((5, 512 + 64), 0x7F80, np.uint16)  # +inf padding must be ignored
    wide[:, :512] = xb
    a = oracle_lib.quantize_rows_bf16(xb)
    b = oracle_lib.quantize_rows_bf16(wide, K=512)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_weight_prep_matches_activation_path_on_bf16_exact_values(oracle_lib):
    """Weight and activation quantisers are the same method: on fp32 values
    that are exactly representable in BF16 they give identical codes/scales."""
    cfg = workloads.custom(7, 512, 8, seed=13)
    X, _, _ = workloads.make_inputs(cfg)
    qa, sa = oracle_lib.quantize_rows_bf16(workloads.bf16_bits(X))
    qw, sw = oracle_lib.rotate_quant_weight(X.float().numpy())
    assert np.array_equal(qa, qw) and np.array_equal(sa, sw)


# ---------------------------------------------------------------- GEMM


@pytest.mark.parametrize("M,N,K", [(1, 1, 256), (3, 17, 256), (17, 3, 512), (17, 17, 512)])
def test_gemm_brute_force(oracle_lib, M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    a = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    b = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    acc = oracle_lib.gemm_i32(a, b)
    for m in range(M):
        for n in range(N):
            ref = sum(int(a[m, k]) * int(b[n, k]) for k in range(K))
            assert acc[m, n] == ref


def test_gemm_extreme_codes_fit_int32(oracle_lib):
    """K = 28672 (the longest reduction on the pages) with every code +-127."""
    K = 28672
    a = np.full((2, K), 127, np.int8)
    a[1] = -127
    b = np.full((1, K), 127, np.int8)
    acc = oracle_lib.gemm_i32(a, b)
    assert acc[0, 0] == 462450688 and acc[1, 0] == -462450688
    assert 462450688 < 2 ** 31


def test_gemm_row_permutation(oracle_lib):
    rng = np.random.default_rng(3)
    a = rng.integers(-127, 128, size=(12, 256)).astype(np.int8)
    b = rng.integers(-127, 128, size=(5, 256)).astype(np.int8)
    p = rng.permutation(12)
    assert np.array_equal(oracle_lib.gemm_i32(a[p], b), oracle_lib.gemm_i32(a, b)[p])


# ---------------------------------------------------------------- epilogue


def test_bf16_rne_matches_torch(oracle_lib):
    rng = np.random.default_rng(4)
    base = rng.standard_normal(3000).astype(np.float32) * np.float32(100)
    u = base.view(np.uint32).copy()
    u[:1000] = (u[:1000] & 0xFFFF0000) | 0x8000  # exact ties
    u[1000:1100] = (u[1000:1100] & 0xFFFF0000) | 0x7FFF
    u[1100:1200] = (u[1100:1200] & 0xFFFF0000) | 0x8001
    f = u.view(np.float32)
    f = np.concatenate([f, np.array([0.0, -0.0, 3.3895314e38, -3.3895314e38, 1e-40, -1e-40],
                                    np.float32)])
    got = oracle_lib.f32_to_bf16(f)
    ref = workloads.bf16_bits(torch.from_numpy(f).to(torch.bfloat16))
    assert np.array_equal(got, ref)


def test_epilogue_zero_acc_gives_bias(oracle_lib):
    rng = np.random.default_rng(5)
    bias = torch.from_numpy(rng.standard_normal(64).astype(np.float32)).to(torch.bfloat16)
    acc = np.zeros((3, 64), np.int32)
    Y = oracle_lib.epilogue(acc, np.ones(3, np.float32) * 0.37, np.ones(64, np.float32) * 1.7,
                            workloads.bf16_bits(bias))
    assert np.array_equal(Y, np.broadcast_to(workloads.bf16_bits(bias), (3, 64)))


def test_epilogue_unit_scales_is_acc_plus_bias(oracle_lib):
    rng = np.random.default_rng(6)
    acc = rng.integers(-5000, 5000, size=(4, 32)).astype(np.int32)
    bias = torch.from_numpy(rng.standard_normal(32).astype(np.float32)).to(torch.bfloat16)
    Y = oracle_lib.epilogue(acc, np.ones(4, np.float32), np.ones(32, np.float32),
                            workloads.bf16_bits(bias))
    ref = (torch.from_numpy(acc).float() + bias.float()[None, :]).to(torch.bfloat16)
    assert np.array_equal(Y, workloads.bf16_bits(ref))


def test_epilogue_no_bias_and_power_of_two_scales(oracle_lib):
    acc = np.array([[3, -7, 100, 0]], np.int32)
    Y = oracle_lib.epilogue(acc, np.array([0.25], np.float32), np.array([2, 4, 8, 0.5], np.float32))
    ref = torch.tensor([[1.5, -7.0, 200.0, 0.0]]).to(torch.bfloat16)
    assert np.array_equal(Y, workloads.bf16_bits(ref))


def test_epilogue_row_and_column_scales_are_not_swapped(oracle_lib):
    rng = np.random.default_rng(7)
    acc = rng.integers(-10 ** 6, 10 ** 6, size=(5, 9)).astype(np.int32)
    sx = rng.uniform(0.5, 2, 5).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-3, 9).astype(np.float32)
    bias = torch.from_numpy(rng.standard_normal(9).astype(np.float32)).to(torch.bfloat16)
    Y = oracle_lib.bf16_to_f32(oracle_lib.epilogue(acc, sx, sw, workloads.bf16_bits(bias)))
    ref = acc.astype(np.float64) * sx[:, None] * sw[None, :] + bias.double().numpy()[None, :]
    assert np.all(np.abs(Y - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)


# ---------------------------------------------------------------- end to end


def _linear_errors(oracle_lib, cfg):
    X, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = oracle_lib.rotate_quant_weight(W.numpy())
    Y, Qx, s_x, acc = oracle_lib.int8_linear(workloads.bf16_bits(X), Qw, s_w, workloads.bf16_bits(bias))
    x = X.double().numpy()
    w = W.double().numpy()
    ref = x @ w.T + bias.double().numpy()[None, :]
    y = oracle_lib.bf16_to_f32(Y).astype(np.float64)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    # negative control: tensorwise INT8 on the unrotated activation and weight
    sxt = np.abs(x).max() / 127.0
    swt = np.abs(w).max() / 127.0
    xq = np.clip(np.rint(x / sxt), -127, 127) * sxt
    wq = np.clip(np.rint(w / swt), -127, 127) * swt
    neg = xq @ wq.T + bias.double().numpy()[None, :]
    rel_neg = np.linalg.norm(neg - ref) / np.linalg.norm(ref)
    return rel, rel_neg


def test_end_to_end_error_band_and_negative_control(oracle_lib):
    """Rotate-then-per-row INT8 lands near the ~1% error the pages report for
    clean W8A8; tensorwise quantisation without the rotation is far worse."""
    rel, rel_neg = _linear_errors(oracle_lib, workloads.CONFIGS[0])
    assert rel < 0.05, rel
    assert rel_neg > 4 * rel, (rel, rel_neg)


def test_rows_are_independent_split_equals_single(oracle_lib):
    """Output rows do not depend on how M is split (pages: split vs single
    call bit-exact)."""
    cfg = workloads.custom(37, 512, 40, seed=21)
    X, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = oracle_lib.rotate_quant_weight(W.numpy())
    xb = workloads.bf16_bits(X)
    bb = workloads.bf16_bits(bias)
    full = oracle_lib.int8_linear(xb, Qw, s_w, bb)[0]
    parts = [oracle_lib.int8_linear(xb[a:b], Qw, s_w, bb)[0] for a, b in [(0, 16), (16, 17), (17, 37)]]
    assert np.array_equal(full, np.concatenate(parts))


def test_linear_rows_matches_full(oracle_lib):
    cfg = workloads.custom(20, 512, 24, seed=22)
    X, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = oracle_lib.rotate_quant_weight(W.numpy())
    Y, Qx, s_x, _ = oracle_lib.int8_linear(workloads.bf16_bits(X), Qw, s_w, workloads.bf16_bits(bias))
    rows = np.array([19, 0, 7])
    Yr = oracle_lib.linear_rows(Qx, s_x, Qw, s_w, workloads.bf16_bits(bias), rows)
    assert np.array_equal(Yr, Y[rows])


def test_page_shapes_match_workloads():
    g = json.load(open(os.path.join(GOLDEN, "pages_workloads.json")))
    shapes = {(c.M, c.K, c.N) for c in workloads.CONFIGS}
    for mkn in g["timed_shapes_MKN"][:3] + g["policy_shapes_MKN"]:
        if tuple(mkn) in {(8193, 5376, 16128), (32700, 5376, 16128), (14850, 7168, 28672)}:
            assert tuple(mkn) in shapes
    assert any(c.K == g["policy_reduction_K"] for c in workloads.CONFIGS)


# ---------------------------------------------------------------- hand-derived rounding cases


def test_rot256_stage_order_ascending(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "rot256_stage_order.json")))
    hs = [1 << i for i in range(8)]
    for a in range(8):
        for b in range(a + 1, 8):
            ha, hb = hs[a], hs[b]
            x = np.zeros(256, np.float32)
            x[0] = 1.0
            x[ha] = np.float32(2.0 ** -24)
            x[ha + hb] = np.float32(2.0 ** -24)
            y = oracle_lib.rot256(x)
            assert y[0] == np.float32(g["expected_out0"]), (ha, hb, y[0])
            assert y[0] != np.float32(g["wrong_order_out0"])


def test_quant_uses_ieee_division(oracle_lib):
    g = json.load(open(os.path.join(GOLDEN, "quant_division_not_reciprocal.json")))
    row = np.zeros(256, np.float32)
    row[: len(g["row"])] = g["row"]
    q, s = oracle_lib.quant_rows(row[None, :])
    assert s[0] == np.float32(g["scale"])
    assert list(q[0, : len(g["codes"])]) == g["codes"]
