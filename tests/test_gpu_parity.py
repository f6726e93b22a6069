"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bar (ConvRot256 INT8 linear as defined in include/ck.h):
  * INT8 codes, FP32 row scales and INT32 accumulators: bit-exact.
  * BF16 outputs: within 1 bf16 ulp (the distance between the two bit
    patterns on the ordered bf16 line); the kernel computes the epilogue with
    the same fp32 operations in the same order, so 0 is expected.
Inputs come from the seeded generators in ``workloads`` (shared by both
sides); every expected value comes from ``oracle``.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity_helpers import assert_bf16_close, tile_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import int8_quantized_linear_convrot256_b200 as m

    m.clear_device_error()
    yield m
    assert m.device_error() == m.CK_OK


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    if t.dtype == torch.bfloat16:
        return workloads.bf16_bits(t)
    return t.numpy()


def dev(t):
    return t.cuda()


# ------------------------------------------------------------------ quantiser


QUANT_SHAPES = [(1, 256), (3, 512), (37, 768), (129, 5376), (7, 7168), (5, 28672),
                (2, 32768), (3, 33024), (2, 132864), (300, 256), (1000, 512)]


@pytest.mark.parametrize("M,K", QUANT_SHAPES)
def test_quantize_rotate_bit_exact(ck, M, K):
    cfg = workloads.custom(M, K, 8, seed=M * 7 + K)
    X, _, _ = workloads.make_inputs(cfg)
    Qx, s_x = ck.quantize_rotate_rowwise(dev(X))
    rq, rs = oracle.quantize_rows_bf16(workloads.bf16_bits(X), rotate=True)
    assert np.array_equal(to_np(s_x).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(to_np(Qx), rq)


@pytest.mark.parametrize("M,K", [(5, 256), (33, 1024), (4, 33024)])
def test_quantize_norotate_bit_exact(ck, M, K):
    cfg = workloads.custom(M, K, 8, seed=M + K)
    X, _, _ = workloads.make_inputs(cfg)
    for fn in (ck.quantize_int8_rowwise, ck.test_quantize_rowwise_norotate):
        Qx, s_x = fn(dev(X))
        rq, rs = oracle.quantize_rows_bf16(workloads.bf16_bits(X), rotate=False)
        assert np.array_equal(to_np(s_x).view(np.uint32), rs.view(np.uint32))
        assert np.array_equal(to_np(Qx), rq)


def test_quantize_row_stride(ck):
    cfg = workloads.custom(19, 768, 8, seed=3)
    X, _, _ = workloads.make_inputs(cfg)
    wide = torch.full((19, 768 + 136), float("nan"), dtype=torch.bfloat16)
    wide[:, :768] = X
    Xv = dev(wide)[:, :768]
    assert Xv.stride(0) == 904
    Qx, s_x = ck.quantize_rotate_rowwise(Xv)
    rq, rs = oracle.quantize_rows_bf16(workloads.bf16_bits(X))
    assert np.array_equal(to_np(Qx), rq) and np.array_equal(to_np(s_x), rs)


def test_quantize_special_rows(ck):
    """Zero rows, ties (no rotation, s = 1), tiny rows whose scale is below
    2^-120 (exact division path), huge and negative rows."""
    K = 512
    rows = np.zeros((8, K), np.float32)
    rows[1, :16] = [127.0, -127.0, 0.5, 1.5, 2.5, 3.5, -0.5, -2.5, -3.5, 0.4921875, 126.5, -126.5,
                    0.0, 7.25, -7.75, 100.5]
    rng = np.random.default_rng(0)
    rows[2] = rng.standard_normal(K) * 1e-38
    rows[3] = rng.standard_normal(K) * 3e38 / 300
    rows[4] = -np.abs(rng.standard_normal(K))
    rows[5, 7] = 1e-40
    rows[6] = rng.standard_normal(K) * 2.0 ** -110
    rows[7] = 1.0
    X = torch.from_numpy(rows).to(torch.bfloat16)
    xb = workloads.bf16_bits(X)
    for rot in (True, False):
        fn = ck.quantize_rotate_rowwise if rot else ck.quantize_int8_rowwise
        Qx, s_x = fn(dev(X))
        rq, rs = oracle.quantize_rows_bf16(xb, rotate=rot)
        assert np.array_equal(to_np(s_x).view(np.uint32), rs.view(np.uint32)), rot
        assert np.array_equal(to_np(Qx), rq), rot


def test_quantize_near_half_integers_take_exact_path(ck):
    """Rows whose scale is a power of two (absmax = 127 * 2^e) and whose
    values are (k + 0.5) * 2^e: every y / s is an exact tie, so the fast
    reciprocal path must hand them to the exact division (ties to even)."""
    K = 256
    rng = np.random.default_rng(5)
    M = 64
    rows = np.zeros((M, K), np.float32)
    for m in range(M):
        e = int(rng.integers(-10, 11))
        s = np.float32(2.0 ** e)
        k = rng.integers(-126, 126, K).astype(np.float32) + np.float32(0.5)
        rows[m] = k * s
        rows[m, 0] = np.float32(127) * s
    X = torch.from_numpy(rows).to(torch.bfloat16)
    assert np.array_equal(X.float().numpy(), rows)  # exactly representable
    Qx, s_x = ck.quantize_int8_rowwise(dev(X))
    rq, rs = oracle.quantize_rows_bf16(workloads.bf16_bits(X), rotate=False)
    assert np.array_equal(to_np(Qx), rq) and np.array_equal(to_np(s_x), rs)
    assert np.all(np.abs(rq[:, 1:].astype(np.int32)) % 2 == 0)  # ties went to even


@pytest.mark.parametrize("q", [127, 7])
def test_row_divisor_is_the_ieee_quotient(ck, q):
    """The quantiser's row divisor (one product and one fma in the kernel) is
    the IEEE quotient fl(amax / q) for every fp32 significand of the lowest
    binade the fast path takes (2^-103), of 1 and of the largest finite one;
    its reciprocal (one Newton step) is within 2^-24 + 2^-43 of 1 / div. The
    expected quotients are numpy's fp32 divisions on the host."""
    sig = np.arange(1 << 23, dtype=np.uint32)
    for e in (-103, 0, 127):
        a = ((np.uint32(127 + e) << np.uint32(23)) | sig).view(np.float32)
        div, rc = ck.test_row_quant_params(torch.from_numpy(a).cuda(), q)
        expect = a / np.float32(q)
        got = div.cpu().numpy()
        bad = np.flatnonzero(got.view(np.uint32) != expect.view(np.uint32))
        assert bad.size == 0, (e, a[bad[:5]])
        # rc * div is exact in float64 (two 24-bit significands)
        err = (rc.double() * div.double() - 1.0).abs().max().item()
        assert err <= 2.0 ** -24 + 2.0 ** -43, (e, err)
    # below 2^-103 the exact path is taken: no reciprocal
    div, rc = ck.test_row_quant_params(torch.tensor([2.0 ** -104, 0.0], device="cuda"), q)
    assert rc.cpu().tolist() == [0.0, 0.0]


@pytest.mark.parametrize("N,K", [(8, 256), (264, 768), (520, 5376), (16, 33024)])
def test_rotate_quant_weight_bit_exact(ck, N, K):
    cfg = workloads.custom(1, K, N, seed=N + K)
    _, W, _ = workloads.make_inputs(cfg)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    rq, rs = oracle.rotate_quant_weight(W.numpy())
    assert np.array_equal(to_np(s_w).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(to_np(Qw), rq)


# ------------------------------------------------------------------ GEMM


GEMM_SHAPES = [(1, 8, 256), (3, 17 * 8, 256), (127, 256, 512), (128, 256, 512), (129, 264, 768),
               (300, 520, 512), (257, 1032, 1024), (640, 512, 2048), (1, 256, 5376),
               # the 2-SM kernel's raster walks groups of 21 N-tiles: a full group,
               # a second group of 2 (the last one ragged), and ragged M
               (300, 21 * 256 + 264, 256),
               # three groups of 21, 21 and 1 N-tiles over three M-tiles
               (520, 43 * 256 - 8, 256)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_i32_bit_exact(ck, M, N, K):
    rng = np.random.default_rng(M * 31 + N * 7 + K)
    a = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    b = rng.integers(-127, 128, size=(N, K)).astype(np.int8)
    acc = ck.test_int8_gemm_i32(dev(torch.from_numpy(a)), dev(torch.from_numpy(b)))
    assert np.array_equal(to_np(acc), oracle.gemm_i32(a, b))


def test_gemm_i32_extreme_codes(ck):
    K = 28672
    a = np.full((130, K), 127, np.int8)
    a[1::2] = -127
    b = np.full((16, K), 127, np.int8)
    b[3] = -127
    acc = to_np(ck.test_int8_gemm_i32(dev(torch.from_numpy(a)), dev(torch.from_numpy(b))))
    assert np.array_equal(acc, oracle.gemm_i32(a, b))
    assert acc[0, 0] == 462450688 and acc[1, 0] == -462450688


# ------------------------------------------------------------------ whole linear


def _oracle_linear(X, W, bias):
    Qw, s_w = oracle.rotate_quant_weight(W.numpy())
    bb = None if bias is None else workloads.bf16_bits(bias)
    Y, Qx, s_x, acc = oracle.int8_linear(workloads.bf16_bits(X), Qw, s_w, bb)
    return Y, Qw, s_w


LINEAR_SHAPES = [(128, 512, 512), (1, 256, 8), (129, 768, 264), (255, 512, 520), (257, 1024, 256),
                 (300, 5376, 512), (64, 28672, 264),
                 # the epilogue across the 2-SM raster's N-tile groups (21, then 2)
                 (300, 256, 21 * 256 + 264)]


@pytest.mark.parametrize("M,K,N", LINEAR_SHAPES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_int8_linear_matches_oracle(ck, M, K, N, with_bias):
    cfg = workloads.custom(M, K, N, seed=M + K + N)
    X, W, bias = workloads.make_inputs(cfg)
    if not with_bias:
        bias = None
    Yr, Qw_r, s_w_r = _oracle_linear(X, W, bias)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    assert np.array_equal(to_np(Qw), Qw_r)
    Y = ck.int8_linear(dev(X), Qw, s_w, None if bias is None else dev(bias))
    assert_bf16_close(to_np(Y), Yr)


def test_int8_gemm_rowscale_matches_oracle(ck):
    cfg = workloads.custom(200, 1024, 264, seed=77)
    X, W, bias = workloads.make_inputs(cfg)
    Yr, Qw_r, s_w_r = _oracle_linear(X, W, bias)
    Qx, s_x = ck.quantize_rotate_rowwise(dev(X))
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    Y = ck.int8_gemm_rowscale(Qx, s_x, Qw, s_w, dev(bias))
    assert_bf16_close(to_np(Y), Yr)


def test_empty_m_is_a_noop(ck):
    Qw = torch.zeros((8, 256), dtype=torch.int8, device="cuda")
    s_w = torch.ones(8, device="cuda")
    X = torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda")
    Y = ck.int8_linear(X, Qw, s_w)
    assert Y.shape == (0, 8)


def test_row_split_invariance(ck):
    """Outputs for M = 8193 in one launch equal those of the same rows split
    into calls of 8192 + 1 and 4096 + 4096 + 1 (bit-exact)."""
    cfg = workloads.custom(8193, 512, 264, seed=8193)
    X, W, bias = workloads.make_inputs(cfg)
    Xd, bd = dev(X), dev(bias)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    full = to_np(ck.int8_linear(Xd, Qw, s_w, bd))
    for cuts in ([0, 8192, 8193], [0, 4096, 8192, 8193]):
        parts = [to_np(ck.int8_linear(Xd[a:b], Qw, s_w, bd)) for a, b in zip(cuts[:-1], cuts[1:])]
        assert np.array_equal(np.concatenate(parts), full)


def test_dirty_workspace_and_output_are_overwritten(ck):
    cfg = workloads.custom(130, 512, 264, seed=5)
    X, W, bias = workloads.make_inputs(cfg)
    Yr, _, _ = _oracle_linear(X, W, bias)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    ws = torch.full((ck.workspace_bytes(130, 512),), 0x5A, dtype=torch.uint8, device="cuda")
    out = torch.full((130, 264), float("nan"), dtype=torch.bfloat16, device="cuda")
    ck.int8_linear(dev(X), Qw, s_w, dev(bias), out=out, workspace=ws)
    assert_bf16_close(to_np(out), Yr)


# ------------------------------------------------------------------ full-size configs


def _sample_rows(M):
    rows = {0, 1, 126, 127, 128, 129, M // 2, M - 129, M - 128, M - 2, M - 1}
    rng = np.random.default_rng(M)
    rows |= set(rng.integers(0, M, 24).tolist())
    rows |= set(tile_rows(M).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < M), np.int64)


GUARD = 0x5A


@pytest.mark.slow
@pytest.mark.parametrize("cfg", workloads.CONFIGS, ids=[c.name for c in workloads.CONFIGS])
def test_full_size_config(ck, cfg):
    """At the full sizes, in the launch configuration the benchmark times:
    every code and row scale of activations and weights bit-exact; all N
    outputs of one row in every 256-row M-tile (its position in the tile
    varying), tile edges and the ragged last row against the oracle computed
    row by row; the 2-SM GEMM's INT32 accumulators of a 300-row slice at the
    full K and N; and guard bands after the codes, the row scales and Y
    left untouched."""
    X, W, bias = workloads.make_inputs(cfg)
    Xd, Wd, bd = dev(X), dev(W), dev(bias)
    Qw, s_w = ck.rotate_quant_weight(Wd)
    del Wd
    rqw, rsw = oracle.rotate_quant_weight(W.numpy())
    assert np.array_equal(to_np(s_w).view(np.uint32), rsw.view(np.uint32))
    assert np.array_equal(to_np(Qw), rqw)
    del W

    need = ck.workspace_bytes(cfg.M, cfg.K)
    ws = torch.full((need + 4096,), GUARD, dtype=torch.uint8, device="cuda")
    Ybuf = torch.full((cfg.M + 2, cfg.N), 0.0, dtype=torch.bfloat16, device="cuda")
    Ybuf.view(torch.uint8).fill_(GUARD)
    Y = ck.int8_linear(Xd, Qw, s_w, bd, out=Ybuf[: cfg.M], workspace=ws)
    torch.cuda.synchronize()
    assert Y.data_ptr() == Ybuf.data_ptr()
    off = (cfg.M * cfg.K + 255) // 256 * 256
    Qx = ws[: cfg.M * cfg.K].view(cfg.M, cfg.K).view(torch.int8)
    s_x = ws[off: off + 4 * cfg.M].view(torch.float32)
    # guard bands: the padding after the codes, everything after the scales,
    # the two rows after Y
    assert bool((ws[cfg.M * cfg.K: off] == GUARD).all())
    assert bool((ws[off + 4 * cfg.M:] == GUARD).all())
    assert bool((Ybuf[cfg.M:].view(torch.uint8) == GUARD).all())

    rqx, rsx = oracle.quantize_rows_bf16(workloads.bf16_bits(X))
    assert np.array_equal(to_np(s_x).view(np.uint32), rsx.view(np.uint32))
    assert np.array_equal(to_np(Qx), rqx)

    rows = _sample_rows(cfg.M)
    Yr = oracle.linear_rows(rqx, rsx, rqw, rsw, workloads.bf16_bits(bias), rows)
    Ys = to_np(Y[torch.from_numpy(rows).cuda()])
    assert_bf16_close(Ys, Yr)

    lo = cfg.M // 2 - 150
    acc = ck.test_int8_gemm_i32(Qx[lo: lo + 300].contiguous(), Qw)  # M > 128: 2-SM kernel
    assert np.array_equal(to_np(acc), oracle.gemm_i32(rqx[lo: lo + 300], rqw))


# ------------------------------------------------------------------ input activation


def _act_inputs(M, K, seed):
    cfg = workloads.custom(M, K, 8, seed=seed)
    X, _, _ = workloads.make_inputs(cfg)
    x = X.float()
    x[:, 3] = torch.linspace(-120.0, 120.0, M)  # exp over- and underflow ranges
    x[::5, 7] = -1.0e4
    x[1::7, 9] = 3.0e4
    x[::3] *= 3.0
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("act", ["none", "relu", "silu", "gelu_tanh"])
def test_input_act_every_bf16_input(ck, act):
    """The activation as the quantiser applies it, on every finite bf16
    input, equals the oracle's bf16 rounding of the exact act(x) bit for bit."""
    bits = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    X = workloads.from_bf16_bits(bits)
    got = to_np(ck.test_input_act(dev(X), act))
    finite = (bits & 0x7F80) != 0x7F80
    want = oracle.act_bf16(act, bits)
    bad = np.nonzero((got != want) & finite)[0]
    assert bad.size == 0, [(hex(int(bits[i])), hex(int(got[i])), hex(int(want[i]))) for i in bad[:8]]


@pytest.mark.parametrize("act", ["relu", "silu", "gelu_tanh"])
@pytest.mark.parametrize("M,K", [(37, 768), (130, 5376), (9, 28672), (2, 32768), (3, 33024)])
def test_quantize_rotate_act_bit_exact(ck, act, M, K):
    X = _act_inputs(M, K, seed=M + K)
    Qx, s_x = ck.quantize_rotate_rowwise_act(dev(X), act)
    rq, rs = oracle.quantize_rows_bf16(workloads.bf16_bits(X), rotate=True, act=act)
    assert np.array_equal(to_np(s_x).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(to_np(Qx), rq)


@pytest.mark.parametrize("act", ["none", "relu", "silu", "gelu_tanh"])
def test_int8_linear_act_matches_oracle(ck, act):
    M, K, N = 300, 1024, 264
    cfg = workloads.custom(M, K, N, seed=31)
    _, W, bias = workloads.make_inputs(cfg)
    X = _act_inputs(M, K, seed=32)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    rqw, rsw = oracle.rotate_quant_weight(W.numpy())
    Y = ck.int8_linear(dev(X), Qw, s_w, dev(bias), input_act=act)
    Yr = oracle.int8_linear(workloads.bf16_bits(X), rqw, rsw, workloads.bf16_bits(bias), act=act)[0]
    assert_bf16_close(to_np(Y), Yr)


@pytest.mark.slow
@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
def test_int8_linear_act_full_size(ck, act):
    """int8_linear(input_act) on the ragged M8193/K5376/N16128 workload:
    every code and row scale, and all outputs of one row per 256-row M-tile."""
    cfg = workloads.CONFIGS[1]
    X, W, bias = workloads.make_inputs(cfg)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    rqw, rsw = oracle.rotate_quant_weight(W.numpy())
    del W
    ws = torch.empty((ck.workspace_bytes(cfg.M, cfg.K),), dtype=torch.uint8, device="cuda")
    Y = ck.int8_linear(dev(X), Qw, s_w, dev(bias), workspace=ws, input_act=act)
    torch.cuda.synchronize()
    off = (cfg.M * cfg.K + 255) // 256 * 256
    Qx = to_np(ws[: cfg.M * cfg.K].view(cfg.M, cfg.K).view(torch.int8))
    s_x = to_np(ws[off: off + 4 * cfg.M].view(torch.float32))
    rqx, rsx = oracle.quantize_rows_bf16(workloads.bf16_bits(X), act=act)
    assert np.array_equal(s_x.view(np.uint32), rsx.view(np.uint32))
    assert np.array_equal(Qx, rqx)
    rows = tile_rows(cfg.M)
    Yr = oracle.linear_rows(rqx, rsx, rqw, rsw, workloads.bf16_bits(bias), rows)
    assert_bf16_close(to_np(Y[torch.from_numpy(rows).cuda()]), Yr)


# ------------------------------------------------------------------ convrot_w4a4_linear


@pytest.mark.parametrize("M,K", [(37, 768), (130, 5376), (9, 28672), (3, 33024)])
def test_quantize_rotate_int4_bit_exact(ck, M, K):
    cfg = workloads.custom(M, K, 8, seed=M + 3 * K)
    X, _, _ = workloads.make_inputs(cfg)
    Qx, s_x = ck.quantize_rotate_rowwise_int4(dev(X))
    rq, rs = oracle.quantize_rows_bf16(workloads.bf16_bits(X), rotate=True, qmax=7)
    assert np.array_equal(to_np(s_x).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(to_np(Qx), rq)


@pytest.mark.parametrize("N,K", [(8, 256), (264, 768), (520, 5376), (16, 33024)])
def test_rotate_quant_weight_int4_bit_exact(ck, N, K):
    cfg = workloads.custom(1, K, N, seed=N + 5 * K)
    _, W, _ = workloads.make_inputs(cfg)
    Qw4, s_w = ck.rotate_quant_weight_int4(dev(W))
    r4, rs = oracle.rotate_quant_weight_int4(W.numpy())
    assert np.array_equal(to_np(s_w).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(to_np(Qw4), r4)


def test_unpack_int4_bit_exact(ck):
    rng = np.random.default_rng(11)
    b = rng.integers(0, 256, size=(300, 2048), dtype=np.uint8)
    b[0, :256] = np.arange(256, dtype=np.uint8)
    got = to_np(ck.unpack_int4(dev(torch.from_numpy(b))))
    assert np.array_equal(got, oracle.unpack_int4(b))


@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (300, 1024, 264), (129, 5376, 520)])
def test_convrot_w4a4_linear_matches_oracle(ck, M, K, N):
    cfg = workloads.custom(M, K, N, seed=M + K + 7 * N)
    X, W, bias = workloads.make_inputs(cfg)
    Qw4, s_w = ck.rotate_quant_weight_int4(dev(W))
    r4, rs = oracle.rotate_quant_weight_int4(W.numpy())
    Y = ck.convrot_w4a4_linear(dev(X), Qw4, s_w, dev(bias))
    Yr = oracle.convrot_w4a4_linear(workloads.bf16_bits(X), r4, rs, workloads.bf16_bits(bias))[0]
    assert_bf16_close(to_np(Y), Yr)


@pytest.mark.parametrize("M,K,N", [(1, 256, 8), (300, 1024, 264), (129, 5376, 520)])
def test_convrot_w4a4_linear_unpacked_weights(ck, M, K, N):
    """The same linear on weights unpacked once: identical to the packed
    entry point and to the oracle."""
    cfg = workloads.custom(M, K, N, seed=M + 3 * K + N)
    X, W, bias = workloads.make_inputs(cfg)
    Qw4, s_w = ck.rotate_quant_weight_int4(dev(W))
    Qw = ck.unpack_int4(Qw4)
    r4, rs = oracle.rotate_quant_weight_int4(W.numpy())
    Y = to_np(ck.convrot_w4a4_linear_unpacked(dev(X), Qw, s_w, dev(bias)))
    assert np.array_equal(Y, to_np(ck.convrot_w4a4_linear(dev(X), Qw4, s_w, dev(bias))))
    Yr = oracle.convrot_w4a4_linear(workloads.bf16_bits(X), r4, rs, workloads.bf16_bits(bias))[0]
    assert_bf16_close(Y, Yr)


@pytest.mark.slow
def test_convrot_w4a4_linear_full_size_sampled_rows(ck):
    cfg = workloads.CONFIGS[1]  # ragged M8193/K5376/N16128
    X, W, bias = workloads.make_inputs(cfg)
    Qw4, s_w = ck.rotate_quant_weight_int4(dev(W))
    r4, rs = oracle.rotate_quant_weight_int4(W.numpy())
    assert np.array_equal(to_np(Qw4), r4)
    Y = ck.convrot_w4a4_linear(dev(X), Qw4, s_w, dev(bias))
    rows = _sample_rows(cfg.M)
    Qx, s_x = oracle.quantize_rows_bf16(workloads.bf16_bits(X), rotate=True, qmax=7)
    Yr = oracle.linear_rows(Qx, s_x, oracle.unpack_int4(r4), rs, workloads.bf16_bits(bias), rows)
    assert_bf16_close(to_np(Y[torch.from_numpy(rows).cuda()]), Yr)


# ------------------------------------------------------------------ dequantize / tensorwise


@pytest.mark.parametrize("per_row", [True, False])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dequantize_int8_bit_exact(ck, per_row, dtype):
    rng = np.random.default_rng(21)
    Q = rng.integers(-127, 128, size=(77, 768)).astype(np.int8)
    s = rng.uniform(1e-6, 3.0, 77).astype(np.float32)
    Yf, Yb = oracle.dequantize_int8(Q, s if per_row else s[:1], per_row=per_row)
    out = ck.dequantize_int8(dev(torch.from_numpy(Q)), dev(torch.from_numpy(s if per_row else s[:1])),
                             per_row=per_row, dtype=dtype)
    got = to_np(out)
    if dtype == torch.float32:
        assert np.array_equal(got.view(np.uint32), Yf.view(np.uint32))
    else:
        assert np.array_equal(got, Yb)


@pytest.mark.parametrize("M,K", [(1, 256), (300, 1000), (4097, 512)])
def test_quantize_int8_tensorwise_bit_exact(ck, M, K):
    cfg = workloads.custom(M, 1024, 8, seed=M + K)
    X, _, _ = workloads.make_inputs(cfg)
    Xv = dev(X)[:, :K]  # row stride 1024 >= K
    Q, s = ck.quantize_int8_tensorwise(Xv)
    rQ, rs = oracle.quantize_int8_tensorwise(workloads.bf16_bits(X[:, :K].contiguous()))
    assert to_np(s)[0].view(np.uint32) == np.float32(rs).view(np.uint32)
    assert np.array_equal(to_np(Q), rQ)


# ------------------------------------------------- host buffers, pipelined copies


def _host_tensor(X, pinned, strided):
    M, K = X.shape
    buf = torch.zeros((M, K + (256 if strided else 0)), dtype=torch.bfloat16, pin_memory=pinned)
    buf[:, :K] = X
    return buf[:, :K]


@pytest.mark.parametrize("M,chunk,pinned,strided", [(785, 256, True, False), (785, 256, False, True),
                                                    (100, 4096, True, True), (1, 256, True, False),
                                                    (512, 256, True, False)])
def test_int8_linear_host_matches_oracle(ck, M, chunk, pinned, strided):
    K, N = 768, 264
    cfg = workloads.custom(M, K, N, seed=M + chunk)
    X, W, bias = workloads.make_inputs(cfg)
    Yr, _, _ = _oracle_linear(X, W, bias)
    Qw, s_w = ck.rotate_quant_weight(dev(W))
    Xh = _host_tensor(X, pinned, strided)
    out = torch.full((M, N), 7.0, dtype=torch.bfloat16, pin_memory=pinned)
    Y = ck.int8_linear_host(Xh, Qw, s_w, dev(bias), out=out, chunk_rows=chunk)
    torch.cuda.current_stream().synchronize()
    assert Y.data_ptr() == out.data_ptr()
    assert_bf16_close(workloads.bf16_bits(Y), Yr)


def test_int8_linear_host_equals_device_call_with_act_and_reused_workspace(ck):
    """Two calls back to back on one workspace (different inputs, silu) give
    exactly the device-side int8_linear results, at a size that spans several
    GEMM tiles per chunk and a ragged last chunk."""
    K, N = 5376, 520
    Qw = None
    ws = None
    for seed, M in ((1, 1300), (2, 777)):
        cfg = workloads.custom(M, K, N, seed=seed)
        X, W, bias = workloads.make_inputs(cfg)
        if Qw is None:
            Qw, s_w = ck.rotate_quant_weight(dev(W))
            ws = torch.empty(ck.host_workspace_bytes(512, N, K), dtype=torch.uint8, device="cuda")
        ref = to_np(ck.int8_linear(dev(X), Qw, s_w, dev(bias), input_act="silu"))
        Xh = _host_tensor(X, True, False)
        Y = ck.int8_linear_host(Xh, Qw, s_w, dev(bias), chunk_rows=512, workspace=ws,
                                input_act="silu")
        torch.cuda.current_stream().synchronize()
        assert np.array_equal(workloads.bf16_bits(Y), ref)
