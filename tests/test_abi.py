"""CPU checks of the C ABI: the library loads without a GPU, exports every
function include/ck.h declares, and its host-side validation returns the
documented status before touching the device (fake, never-dereferenced
addresses are enough for that)."""
import ctypes
import os
import re

import pytest

import int8_quantized_linear_convrot256_b200 as ck

FAKE = 0x10000  # 64 KiB: 256-byte aligned, never dereferenced
MIS = FAKE + 4


def header_functions():
    text = open(ck.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ck_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_function_is_exported():
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(ck.lib, n), n
    assert set(names) == set(ck._SIGS), "binding and header disagree"


def test_checked_build_exports_the_same_functions():
    """libck_checked.so (the build with device-side index checks) has the
    same C ABI, and says which build it is."""
    path = os.path.join(os.path.dirname(ck.LIB_PATH), "libck_checked.so")
    if not os.path.exists(path):
        pytest.skip("libck_checked.so not built")
    checked = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(checked, n), n
    checked.ck_is_checked_build.restype = ctypes.c_int
    assert checked.ck_is_checked_build() == 1
    assert ck.lib.ck_is_checked_build() == (1 if ck.LIB_PATH.endswith("libck_checked.so") else 0)


def test_status_strings():
    for s in range(8):
        assert ck.status_string(s).startswith("CK_")
    assert "unknown" in ck.status_string(99)


def test_workspace_bytes():
    assert ck.workspace_bytes(0, 256) == 0
    assert ck.workspace_bytes(3, 256) == 768 + 256
    assert ck.workspace_bytes(32700, 5376) == 32700 * 5376 + ((4 * 32700 + 255) // 256) * 256


def lin(X=FAKE, ldx=512, Qw=FAKE, s_w=FAKE, bias=None, Y=FAKE, M=4, N=8, K=512, ws=FAKE,
        ws_bytes=1 << 30):
    return ck.lib.ck_int8_linear(X, ldx, Qw, s_w, bias, Y, M, N, K, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(X=None), ck.CK_ERR_INVALID_VALUE),
    (dict(Y=None), ck.CK_ERR_INVALID_VALUE),
    (dict(ws=None), ck.CK_ERR_INVALID_VALUE),
    (dict(M=-1), ck.CK_ERR_INVALID_VALUE),
    (dict(K=0), ck.CK_ERR_INVALID_VALUE),
    (dict(ldx=256), ck.CK_ERR_INVALID_VALUE),
    (dict(K=300, ldx=512), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(K=132864 + 256, ldx=132864 + 256), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(N=12), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(M=1 << 31), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(X=MIS), ck.CK_ERR_MISALIGNED),
    (dict(ldx=516), ck.CK_ERR_MISALIGNED),
    (dict(Y=MIS), ck.CK_ERR_MISALIGNED),
    (dict(bias=MIS), ck.CK_ERR_MISALIGNED),
    (dict(ws=FAKE + 16), ck.CK_ERR_MISALIGNED),
    (dict(ws_bytes=100), ck.CK_ERR_WORKSPACE),
    (dict(M=0), ck.CK_OK),
    (dict(N=0), ck.CK_OK),
])
def test_int8_linear_validation(kw, status):
    assert lin(**kw) == status


def test_valid_call_without_a_gpu_fails_cleanly():
    import torch

    if torch.cuda.is_available():
        pytest.skip("has a GPU")
    # passes validation, then the device query fails: CUDA error, no crash
    assert lin() in (ck.CK_ERR_CUDA, ck.CK_ERR_ARCH)


@pytest.mark.parametrize("args,status", [
    ((FAKE, 4, 512, 512, FAKE, FAKE), ck.CK_OK),
    ((None, 4, 512, 512, FAKE, FAKE), ck.CK_ERR_INVALID_VALUE),
    ((FAKE, 4, 500, 512, FAKE, FAKE), ck.CK_ERR_UNSUPPORTED_SHAPE),
    ((FAKE, 4, 512, 256, FAKE, FAKE), ck.CK_ERR_INVALID_VALUE),
    ((MIS, 4, 512, 512, FAKE, FAKE), ck.CK_ERR_MISALIGNED),
    ((FAKE, 4, 512, 512, FAKE, FAKE + 2), ck.CK_ERR_MISALIGNED),
    ((FAKE, 0, 512, 512, FAKE, FAKE), ck.CK_OK),
])
def test_quantize_validation(args, status):
    for fn in (ck.lib.ck_quantize_rotate_rowwise, ck.lib.ck_quantize_int8_rowwise,
               ck.lib.ck_test_quantize_rowwise_norotate):
        got = fn(*args, None)
        if status == ck.CK_OK and args[1] > 0:
            import torch

            if torch.cuda.is_available():
                continue
            assert got in (ck.CK_ERR_CUDA, ck.CK_ERR_ARCH)
        else:
            assert got == status


def test_weight_and_gemm_validation():
    L = ck.lib
    assert L.ck_rotate_quant_weight(None, 4, 256, FAKE, FAKE, None) == ck.CK_ERR_INVALID_VALUE
    assert L.ck_rotate_quant_weight(FAKE, 4, 200, FAKE, FAKE, None) == ck.CK_ERR_UNSUPPORTED_SHAPE
    assert L.ck_rotate_quant_weight(FAKE, 4, 256, FAKE, FAKE + 4, None) == ck.CK_ERR_MISALIGNED
    assert L.ck_rotate_quant_weight(FAKE, 0, 256, FAKE, FAKE, None) == ck.CK_OK
    g = L.ck_int8_gemm_rowscale
    assert g(FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 12, 256, None) == ck.CK_ERR_UNSUPPORTED_SHAPE
    assert g(FAKE, None, FAKE, FAKE, None, FAKE, 4, 8, 256, None) == ck.CK_ERR_INVALID_VALUE
    assert g(FAKE, FAKE + 2, FAKE, FAKE, None, FAKE, 4, 8, 256, None) == ck.CK_ERR_MISALIGNED
    t = L.ck_test_int8_gemm_i32
    assert t(FAKE, FAKE, None, 4, 8, 256, None) == ck.CK_ERR_INVALID_VALUE
    assert t(FAKE, FAKE, FAKE + 8, 4, 8, 256, None) == ck.CK_ERR_MISALIGNED
    assert L.ck_test_inject_producer_stall(2, 0) == ck.CK_ERR_INVALID_VALUE
    assert L.ck_test_inject_producer_stall(0, 0) == ck.CK_OK


def test_row_quant_params_validation():
    f = ck.lib.ck_test_row_quant_params
    assert f(FAKE, 4, 126, FAKE, FAKE, None) == ck.CK_ERR_INVALID_VALUE
    assert f(FAKE, -1, 127, FAKE, FAKE, None) == ck.CK_ERR_INVALID_VALUE
    assert f(None, 4, 7, FAKE, FAKE, None) == ck.CK_ERR_INVALID_VALUE
    assert f(None, 0, 127, None, None, None) == ck.CK_OK


def test_binding_rejects_cpu_tensors():
    import torch

    with pytest.raises(ValueError, match="CUDA"):
        ck.quantize_rotate_rowwise(torch.zeros((2, 256), dtype=torch.bfloat16))


def lin_host(X=FAKE, ldx=512, act=0, Qw=FAKE, s_w=FAKE, bias=None, Y=FAKE, M=4, N=8, K=512,
             chunk=2, ws=FAKE, ws_bytes=1 << 30):
    return ck.lib.ck_int8_linear_host(X, ldx, act, Qw, s_w, bias, Y, M, N, K, chunk, ws, ws_bytes,
                                      None)


def test_host_workspace_bytes():
    assert ck.host_workspace_bytes(0, 8, 256) == 0
    # two input chunks, two output chunks, the chunk's codes and row scales
    r, N, K = 4096, 16128, 5376
    want = 2 * r * K * 2 + 2 * r * N * 2 + r * K + 4 * r
    assert ck.host_workspace_bytes(r, N, K) == want
    assert ck.host_workspace_bytes(3, 8, 256) == 2 * 1536 + 2 * 256 + 768 + 256


@pytest.mark.parametrize("kw,status", [
    (dict(X=None), ck.CK_ERR_INVALID_VALUE),
    (dict(Y=None), ck.CK_ERR_INVALID_VALUE),
    (dict(ws=None), ck.CK_ERR_INVALID_VALUE),
    (dict(chunk=0), ck.CK_ERR_INVALID_VALUE),
    (dict(act=7), ck.CK_ERR_INVALID_VALUE),
    (dict(ldx=256), ck.CK_ERR_INVALID_VALUE),
    (dict(K=300, ldx=512), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(N=12), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(Qw=MIS), ck.CK_ERR_MISALIGNED),
    (dict(ws=FAKE + 16), ck.CK_ERR_MISALIGNED),
    (dict(ws_bytes=1024), ck.CK_ERR_WORKSPACE),
    (dict(M=0), ck.CK_OK),
])
def test_int8_linear_host_validation(kw, status):
    assert lin_host(**kw) == status


def test_nvfp4_scale_bytes():
    assert ck.nvfp4_scale_bytes(0, 256) == 0
    assert ck.nvfp4_scale_bytes(1, 256) == 128 * 16
    assert ck.nvfp4_scale_bytes(129, 5376) == 256 * 336
    assert ck.nvfp4_workspace_bytes(3, 256) == 512 + 2048 + 256


@pytest.mark.parametrize("call,status", [
    (lambda: ck.lib.ck_quantize_rotate_nvfp4(FAKE, 4, 512, 512, FAKE, FAKE, FAKE, None), None),
    (lambda: ck.lib.ck_quantize_rotate_nvfp4(FAKE, 4, 33024, 33024, FAKE, FAKE, FAKE, None),
     ck.CK_ERR_UNSUPPORTED_SHAPE),
    (lambda: ck.lib.ck_quantize_rotate_nvfp4(FAKE, 4, 300, 512, FAKE, FAKE, FAKE, None),
     ck.CK_ERR_UNSUPPORTED_SHAPE),
    (lambda: ck.lib.ck_quantize_rotate_nvfp4(None, 4, 512, 512, FAKE, FAKE, FAKE, None),
     ck.CK_ERR_INVALID_VALUE),
    (lambda: ck.lib.ck_quantize_rotate_nvfp4(FAKE, 4, 512, 512, MIS, FAKE, FAKE, None),
     ck.CK_ERR_MISALIGNED),
    (lambda: ck.lib.ck_rotate_quant_weight_nvfp4(FAKE, 4, 512, FAKE, MIS, FAKE, None),
     ck.CK_ERR_MISALIGNED),
    (lambda: ck.lib.ck_nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 12, 512, None),
     ck.CK_ERR_UNSUPPORTED_SHAPE),
    (lambda: ck.lib.ck_nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 4, 8, 512, None),
     ck.CK_ERR_INVALID_VALUE),
    (lambda: ck.lib.ck_nvfp4_gemm(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 0, 8, 512, None),
     ck.CK_OK),
    (lambda: ck.lib.ck_convrot_nvfp4_linear(FAKE, 512, FAKE, FAKE, FAKE, None, FAKE, 4, 8, 512, FAKE,
                                            16, None), ck.CK_ERR_WORKSPACE),
    (lambda: ck.lib.ck_dequantize_nvfp4(FAKE, FAKE, FAKE, 4, 512, 0, MIS, None), ck.CK_ERR_MISALIGNED),
])
def test_nvfp4_validation(call, status):
    got = call()
    if status is None:  # a valid call: without a GPU it can only fail in the CUDA runtime
        assert got in (ck.CK_ERR_CUDA, ck.CK_ERR_ARCH)
    else:
        assert got == status


def norm(X=FAKE, ldx=512, R=None, ldr=512, Ro=None, ldo=512, g=None, eps=1e-6, M=4, K=512, Y=FAKE):
    return ck.lib.ck_rmsnorm_residual(X, ldx, R, ldr, Ro, ldo, g, eps, M, K, Y, None)


@pytest.mark.parametrize("kw,status", [
    (dict(X=None), ck.CK_ERR_INVALID_VALUE),
    (dict(Y=None), ck.CK_ERR_INVALID_VALUE),
    (dict(M=-1), ck.CK_ERR_INVALID_VALUE),
    (dict(K=0), ck.CK_ERR_INVALID_VALUE),
    (dict(ldx=256), ck.CK_ERR_INVALID_VALUE),
    (dict(R=FAKE, ldr=256), ck.CK_ERR_INVALID_VALUE),
    (dict(Ro=FAKE, ldo=256), ck.CK_ERR_INVALID_VALUE),
    (dict(eps=0.0), ck.CK_ERR_INVALID_VALUE),
    (dict(eps=-1e-6), ck.CK_ERR_INVALID_VALUE),
    (dict(eps=float("nan")), ck.CK_ERR_INVALID_VALUE),
    (dict(eps=float("inf")), ck.CK_ERR_INVALID_VALUE),
    (dict(K=300, ldx=512), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(X=MIS), ck.CK_ERR_MISALIGNED),
    (dict(ldx=516), ck.CK_ERR_MISALIGNED),
    (dict(R=MIS), ck.CK_ERR_MISALIGNED),
    (dict(R=FAKE, ldr=516), ck.CK_ERR_MISALIGNED),
    (dict(Ro=MIS), ck.CK_ERR_MISALIGNED),
    (dict(g=MIS), ck.CK_ERR_MISALIGNED),
    (dict(Y=MIS), ck.CK_ERR_MISALIGNED),
    (dict(M=0), ck.CK_OK),
])
def test_rmsnorm_validation(kw, status):
    assert norm(**kw) == status


def lin_norm(X=FAKE, ldx=512, R=None, ldr=512, Ro=None, ldo=512, g=None, eps=1e-6, Qw=FAKE,
             s_w=FAKE, bias=None, Y=FAKE, M=4, N=8, K=512, ws=FAKE, ws_bytes=1 << 30):
    return ck.lib.ck_int8_linear_norm(X, ldx, R, ldr, Ro, ldo, g, eps, Qw, s_w, bias, Y, M, N, K,
                                      ws, ws_bytes, None)


def test_norm_workspace_bytes():
    # K <= CK_NORM_FUSED_MAX_K: the normalisation runs inside the quantiser,
    # so only the codes and row scales need room; above it the normalised
    # rows come first
    assert ck.NORM_FUSED_MAX_K == 14336
    assert ck.norm_workspace_bytes(0, 256) == 0
    assert ck.norm_workspace_bytes(3, 256) == ck.workspace_bytes(3, 256) == 768 + 256
    M, K = 32700, 5376
    assert ck.norm_workspace_bytes(M, K) == ck.workspace_bytes(M, K)
    assert ck.norm_workspace_bytes(5, 14336) == ck.workspace_bytes(5, 14336)
    assert ck.norm_workspace_bytes(5, 14592) == 5 * 14592 * 2 + ck.workspace_bytes(5, 14592)


@pytest.mark.parametrize("kw,status", [
    (dict(X=None), ck.CK_ERR_INVALID_VALUE),
    (dict(Y=None), ck.CK_ERR_INVALID_VALUE),
    (dict(ws=None), ck.CK_ERR_INVALID_VALUE),
    (dict(eps=0.0), ck.CK_ERR_INVALID_VALUE),
    (dict(ldx=256), ck.CK_ERR_INVALID_VALUE),
    (dict(K=300, ldx=512), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(N=12), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(g=MIS), ck.CK_ERR_MISALIGNED),
    (dict(Qw=MIS), ck.CK_ERR_MISALIGNED),
    (dict(ws=FAKE + 16), ck.CK_ERR_MISALIGNED),
    (dict(ws_bytes=1024), ck.CK_ERR_WORKSPACE),
    (dict(K=14592, ldx=14592, ldr=14592, ldo=14592, ws_bytes=4 * 14592 * 2), ck.CK_ERR_WORKSPACE),
    (dict(M=0), ck.CK_OK),
    (dict(N=0), ck.CK_OK),
])
def test_int8_linear_norm_validation(kw, status):
    assert lin_norm(**kw) == status


def quant_norm(X=FAKE, ldx=512, R=None, ldr=512, Ro=None, ldo=512, g=None, eps=1e-6, M=4, K=512,
               Qx=FAKE, s_x=FAKE):
    return ck.lib.ck_quantize_rotate_rowwise_norm(X, ldx, R, ldr, Ro, ldo, g, eps, M, K, Qx, s_x,
                                                  None)


@pytest.mark.parametrize("kw,status", [
    (dict(X=None), ck.CK_ERR_INVALID_VALUE),
    (dict(Qx=None), ck.CK_ERR_INVALID_VALUE),
    (dict(eps=0.0), ck.CK_ERR_INVALID_VALUE),
    (dict(M=-1), ck.CK_ERR_INVALID_VALUE),
    (dict(K=300), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(K=14592, ldx=14592), ck.CK_ERR_UNSUPPORTED_SHAPE),
    (dict(X=MIS), ck.CK_ERR_MISALIGNED),
    (dict(R=FAKE, ldr=516), ck.CK_ERR_MISALIGNED),
    (dict(Qx=MIS), ck.CK_ERR_MISALIGNED),
    (dict(M=0), ck.CK_OK),
])
def test_quantize_rotate_rowwise_norm_validation(kw, status):
    assert quant_norm(**kw) == status
