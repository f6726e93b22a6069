"""Pins for the oracle's ConvRot NVFP4 functions (CPU, independent of the oracle).

Sources: ComfyUI-HSWQ-Loader-and-Tools, "NVFP4 torch.compile Fix", section 5-1
(nvfp4_gemm.py): the E2M1 value table, 16-value blocks, block scales in the
128 x 4 blocked layout that from_blocked undoes, a per-tensor scale, and
dequantisation as value x (per-tensor scale x block scale). The quantiser's
two-level scaling is this build's reading (see the oracle's NVFP4 section).
What pins it here: the page's table (golden), brute force over the E2M1 grid,
PyTorch's float8_e4m3fn conversions (an independent implementation), the
tile geometry stated in words, exact algebra (power-of-two invariance), the
quantisation error bound, and fp64 matrix products of independently decoded
values.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_e2m1_values.json")))
LUT = np.array(GOLD["values"], dtype=np.float32)


def test_e2m1_table_matches_the_page():
    got = oracle.e2m1_to_f32(range(16))
    assert np.array_equal(got.view(np.uint32), LUT.view(np.uint32))  # -0 included


def _nearest_e2m1_brute(v: float) -> int:
    a = abs(v)
    mags = [abs(float(x)) for x in LUT[:8]]
    if a >= 6.0:
        c = 7
    else:
        best, bd = 0, a
        for c in range(1, 8):
            d = abs(a - mags[c])
            if d < bd or (d == bd and c % 2 == 0):
                best, bd = c, d
        c = best
    return c | (8 if np.signbit(v) else 0)


def test_e2m1_rounding_brute_force():
    rng = np.random.default_rng(0)
    vals = list(rng.uniform(-8, 8, 4000).astype(np.float32))
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    for m in mids:  # ties and their neighbours
        for s in (1.0, -1.0):
            for dv in (0.0, 1e-6, -1e-6):
                vals.append(np.float32(s * (m + dv)))
    vals += [np.float32(x) for x in (0.0, -0.0, 6.0, -6.0, 100.0, -1e30, 1e-30)]
    got = oracle.f32_to_e2m1(vals)
    want = np.array([_nearest_e2m1_brute(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)
    # ties to the even mantissa: 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    assert list(oracle.f32_to_e2m1(mids)) == [0, 2, 2, 4, 4, 6, 6]


def test_e4m3_decode_matches_torch():
    codes = [c for c in range(256) if c not in (0x7F, 0xFF)]
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    got = oracle.e4m3_to_f32(codes)
    assert np.array_equal(got, ref)


def test_e4m3_rounding_matches_torch_below_saturation():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(0, 448, 3000), np.exp(rng.uniform(np.log(1e-4), np.log(440), 3000)),
                        [0.0, 2.0 ** -9, 1.5 * 2.0 ** -9, 2.0 ** -10, 0.9 * 2.0 ** -10, 1.0625, 1.1875, 447.0,
                         448.0]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.f32_to_e4m3(v), ref)


def test_e4m3_saturates_at_448():
    assert list(oracle.f32_to_e4m3([448.0, 449.0, 470.0, 1e9])) == [0x7E] * 4


def test_blocked_scale_layout_geometry():
    """A 512-byte tile seen as 32 lines of 16 bytes: line i, byte j holds the
    scale of row 32 * (j // 4) + i (of the tile's 128 rows) and column j % 4 (of
    its 4 columns); tiles run over the column blocks first, then row blocks."""
    R, C = 300, 12  # 3 row blocks (padded), 3 column blocks
    tiles_c = (C + 3) // 4
    seen = set()
    for rb in range(3):
        for cb in range(tiles_c):
            base = (rb * tiles_c + cb) * 512
            for i in range(32):
                for j in range(16):
                    r = 128 * rb + 32 * (j // 4) + i
                    c = 4 * cb + j % 4
                    off = oracle.nvfp4_sf_offset(r, c, C)
                    assert off == base + 16 * i + j
                    seen.add(off)
    assert len(seen) == oracle.nvfp4_sf_bytes(R, 16 * C) == 3 * 128 * 12


def _decode_np(Q, S, s_t, K, hi_first=False):
    """Independent decode: page table + torch E4M3, layout from the geometry pin."""
    R = Q.shape[0]
    lo, hi = (Q & 15).astype(np.int64), (Q >> 4).astype(np.int64)
    first, second = (hi, lo) if hi_first else (lo, hi)
    codes = np.stack([first, second], axis=-1).reshape(R, K)
    C = K // 16
    r = np.arange(R)[:, None]
    c = np.arange(C)[None, :]
    off = (((r // 128) * ((C + 3) // 4) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4)
    sc = torch.from_numpy(S[off].astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    return LUT[codes].astype(np.float64) * np.repeat(sc, 16, axis=1) * float(s_t), codes, sc


def _rotated_fp64(X):
    H = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(256)] for i in range(256)]) / 16.0
    M, K = X.shape
    return (X.astype(np.float64).reshape(M, K // 256, 256) @ H.T).reshape(M, K)


@pytest.mark.parametrize("M,K,seed", [(5, 256, 0), (130, 512, 1), (3, 5376, 2)])
def test_quantiser_properties(M, K, seed):
    cfg = workloads.custom(M, K, 8, seed=seed)
    X, _, _ = workloads.make_inputs(cfg)
    Xb = workloads.bf16_bits(X)
    Q, S, s_t = oracle.quantize_rotate_nvfp4(Xb)
    Y = _rotated_fp64(workloads.from_bf16_bits(Xb).float().numpy())
    amax = np.abs(Y).max()
    assert abs(s_t - amax / 2688.0) <= 1e-6 * s_t
    dq, codes, sc = _decode_np(Q, S, s_t, K)
    # every block scale is the E4M3 rounding (torch) of (block amax / 6) / s_t
    bam = np.abs(Y).reshape(M, K // 16, 16).max(axis=2)
    t = ((bam / 6.0) / s_t).astype(np.float32)
    want = torch.from_numpy(np.minimum(t, 448.0)).to(torch.float8_e4m3fn).double().numpy()
    close = np.abs(t - (bam / 6.0 / s_t)) < 1e-4 * np.maximum(t, 1e-30)  # away from fp32 rounding doubts
    assert np.array_equal(sc[close], want[close])
    # error bound: half the E2M1 spacing at the value (1 above 4, else 0.5 or 0.25), times d
    d = np.repeat(sc, 16, axis=1) * s_t
    a = np.abs(Y) / np.where(d > 0, d, 1.0)
    half = np.where(a >= 4.0, 1.0, np.where(a >= 2.0, 0.5, np.where(a >= 1.0, 0.25, 0.25)))
    err = np.abs(dq - Y)
    sat = a > 6.0
    assert np.all(err[~sat] <= half[~sat] * d[~sat] * (1 + 1e-5) + 1e-30)
    assert np.all(np.abs(dq[sat]) == 6.0 * d[sat])
    # blocks with a normal E4M3 scale reach the largest code
    normal = sc >= 2.0 ** -6
    top = np.abs(LUT[codes]).reshape(M, K // 16, 16).max(axis=2)
    assert np.all(top[normal] == 6.0)


def test_power_of_two_invariance_and_zero_tensor():
    cfg = workloads.custom(4, 512, 8, seed=9)
    X, _, _ = workloads.make_inputs(cfg)
    Q1, S1, s1 = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    Q2, S2, s2 = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X * 8))
    assert np.array_equal(Q1, Q2) and np.array_equal(S1, S2) and s2 == 8 * s1
    Z = np.zeros((3, 256), dtype=np.uint16)
    Qz, Sz, sz = oracle.quantize_rotate_nvfp4(Z)
    assert sz == 0.0 and not Qz.any() and not Sz.any()


def test_weights_path_equals_bf16_path_on_bf16_values():
    cfg = workloads.custom(7, 768, 8, seed=4)
    X, _, _ = workloads.make_inputs(cfg)
    a = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    b = oracle.rotate_quant_weight_nvfp4(X.float().numpy())
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


@pytest.mark.parametrize("hi_first", [False, True])
def test_dequantize_matches_independent_decode(hi_first):
    cfg = workloads.custom(9, 512, 8, seed=6)
    X, _, _ = workloads.make_inputs(cfg)
    Q, S, s_t = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    got = oracle.dequantize_nvfp4(Q, S, s_t, hi_first=hi_first)
    want, _, _ = _decode_np(Q, S, s_t, 512, hi_first=hi_first)
    # fp32 product (s_t * scale) * value versus the fp64 product: one rounding each
    assert np.allclose(got, want, rtol=2 ** -22, atol=0)
    if hi_first:
        base = oracle.dequantize_nvfp4(Q, S, s_t, hi_first=False)
        sw = base.reshape(9, 256, 2)[:, :, ::-1].reshape(9, 512)
        assert np.array_equal(got, sw)


def test_linear_rows_match_fp64_products():
    M, K, N = 6, 512, 10
    cfg = workloads.custom(M, K, N, seed=12)
    X, W, bias = workloads.make_inputs(cfg)
    Qa, Sa, sa = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X))
    Qw, Sw, sw = oracle.rotate_quant_weight_nvfp4(W.numpy())
    A, _, _ = _decode_np(Qa, Sa, 1.0, K)
    B, _, _ = _decode_np(Qw, Sw, 1.0, K)
    acc = A @ B.T
    ref = acc * np.float64(np.float32(sa) * np.float32(sw)) + workloads.from_bf16_bits(
        workloads.bf16_bits(bias)).double().numpy()[None, :]
    Y, mag = oracle.nvfp4_linear_rows(Qa, Sa, sa, Qw, Sw, sw, workloads.bf16_bits(bias))
    got = workloads.from_bf16_bits(Y).double().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6)
    assert np.all(mag >= np.abs(acc * sa * sw) * (1 - 1e-6))


def test_rounding_ties_worked_by_hand():
    """Inputs whose rotated values land on rounding ties, with the results
    worked out by hand from the definition (ConvRot256 of a row with one or
    two non-zeros is known in closed form: H e_0 = all ones, H e_1 alternates
    signs, then x 1/16).

    Row 0 = 258048 e_0: every rotated value is 16128, so s_t = 16128 / 2688 = 6
    and the block scale quotient is 448 (E4M3 0x7E). Row a e_0: block absmax
    a / 16, quotient a / 576: a = 612 gives 1.0625, the tie between E4M3 1 and
    1.125 (even: 1.0, byte 0x38); a = 8 and a = 1 give 0.01389 and 0.001736,
    E4M3 subnormals 7 x 2^-9 and 1 x 2^-9. Row a e_0 + b e_1 with a + b = 576:
    scale 1.0, divisor 6; even places hold 36 / 6 = 6 (code 7), odd places
    (a - b) / 96, the E2M1 ties 0.25 -> 0, 0.75 -> 1.0 (code 2), 2.5 -> 2
    (code 4), 5 -> 4 (code 6). Element 2j sits in the low nibble of byte j."""
    rows = [[(0, 258048.0)], [(0, 612.0)], [(0, 8.0)], [(0, 1.0)],
            [(0, 300.0), (1, 276.0)], [(0, 324.0), (1, 252.0)], [(0, 408.0), (1, 168.0)],
            [(0, 528.0), (1, 48.0)]]
    X = torch.zeros((len(rows), 256), dtype=torch.float32)
    for r, entries in enumerate(rows):
        for c, v in entries:
            X[r, c] = v
    Q, S, s_t = oracle.quantize_rotate_nvfp4(workloads.bf16_bits(X.to(torch.bfloat16)))
    assert np.float32(s_t) == np.float32(6.0)
    want_scale = [0x7E, 0x38, 0x07, 0x01, 0x38, 0x38, 0x38, 0x38]
    for r, b in enumerate(want_scale):
        assert [int(S[oracle.nvfp4_sf_offset(r, c, 16)]) for c in range(16)] == [b] * 16
    for r, byte in zip(range(4, 8), [0x07, 0x27, 0x47, 0x67]):
        assert np.all(Q[r] == byte), (r, Q[r][:4])
    # row 0: every value is 16128 and the divisor 448 x 6 = 2688, so every code is +6 (7)
    assert np.all(Q[0] == 0x77)
