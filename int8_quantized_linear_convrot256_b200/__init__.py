"""ConvRot256 INT8 linear for NVIDIA B200 (sm_100a).

Thin Python binding of ``libck.so`` (the C ABI declared in ``include/ck.h``):
every function here only checks and marshals its arguments and calls the
entry point of the same name; all arithmetic runs in the library's CUDA
kernels. PyTorch supplies device memory and streams. There is no CPU path:
if ``libck.so`` is missing, importing this package raises ImportError, and a
call on a device that is not a B200 raises ``CKError`` (CK_ERR_ARCH). With
the environment variable CK_LIBRARY=libck_checked.so the package loads the
checked build instead (device-side bounds checks; ``checked_violations()``).

    import int8_quantized_linear_convrot256_b200 as ck
    Qw, s_w = ck.rotate_quant_weight(W_fp32_cuda)          # offline, once
    Y = ck.int8_linear(X_bf16_cuda, Qw, s_w, bias_bf16)    # per forward

Method (web pages, by title and section): comfy-kitchen 0.2.40 "Huawei
Ascend backend" (quantize_int8_rowwise, quantize_and_rotate_rowwise,
int8_linear); sglang PR "Tune Kitchen INT8 row splitting for SM120",
Accuracy Test (BF16 activations and bias, INT8 weights, FP32 row scales,
ConvRot256); ComfyUI-AppleSilicon-FP8 README row 17 (rotate online, per-row
quantise, INT8 x INT8 -> INT32, rescale + bias fused into the store).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, os.path.basename(os.environ.get("CK_LIBRARY", "libck.so")))
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "ck.h")

CK_OK = 0
CK_ERR_INVALID_VALUE = 1
CK_ERR_UNSUPPORTED_SHAPE = 2
CK_ERR_MISALIGNED = 3
CK_ERR_WORKSPACE = 4
CK_ERR_ARCH = 5
CK_ERR_CUDA = 6
CK_ERR_DEVICE_TIMEOUT = 7
MAX_K = 132864
ACTS = {"none": 0, "relu": 1, "silu": 2, "gelu_tanh": 3}
NOALLOC_SCRATCH_BYTES = 32 << 20

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python int8_quantized_linear_convrot256_b200/build.py`"
        " (add --checked for libck_checked.so)"
        " (there is no CPU fallback)")

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_st = ctypes.c_int

lib = ctypes.CDLL(LIB_PATH)
_SIGS = {
    "ck_rotate_quant_weight": (_st, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "ck_quantize_rotate_rowwise": (_st, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "ck_quantize_int8_rowwise": (_st, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "ck_int8_linear_workspace_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "ck_int8_linear": (_st, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                             ctypes.c_size_t, _vp]),
    "ck_int8_gemm_rowscale": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "ck_quantize_rotate_rowwise_act": (_st, [_vp, _i64, _i64, _i64, _st, _vp, _vp, _vp]),
    "ck_int8_linear_act": (_st, [_vp, _i64, _st, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                 ctypes.c_size_t, _vp]),
    "ck_rmsnorm_residual": (_st, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, ctypes.c_float, _i64,
                                  _i64, _vp, _vp]),
    "ck_int8_linear_norm_workspace_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "ck_quantize_rotate_rowwise_norm": (_st, [_vp, _i64, _vp, _i64, _vp, _i64, _vp,
                                              ctypes.c_float, _i64, _i64, _vp, _vp, _vp]),
    "ck_int8_linear_norm": (_st, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, ctypes.c_float, _vp, _vp,
                                  _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp]),
    "ck_rotate_quant_weight_int4": (_st, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "ck_unpack_int4": (_st, [_vp, _i64, _i64, _vp, _vp]),
    "ck_quantize_rotate_rowwise_int4": (_st, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "ck_convrot_w4a4_linear_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "ck_convrot_w4a4_linear": (_st, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                     ctypes.c_size_t, _vp]),
    "ck_convrot_w4a4_linear_unpacked": (_st, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                              _vp, ctypes.c_size_t, _vp]),
    "ck_dequantize_int8": (_st, [_vp, _vp, _i64, _i64, _st, _st, _vp, _vp]),
    "ck_quantize_int8_tensorwise": (_st, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "ck_int8_linear_noalloc": (_st, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "ck_int8_linear_host_workspace_bytes": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "ck_nvfp4_scale_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "ck_quantize_rotate_nvfp4": (_st, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "ck_rotate_quant_weight_nvfp4": (_st, [_vp, _i64, _i64, _vp, _vp, _vp, _vp]),
    "ck_dequantize_nvfp4": (_st, [_vp, _vp, _vp, _i64, _i64, _st, _vp, _vp]),
    "ck_nvfp4_gemm": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "ck_convrot_nvfp4_linear_workspace_bytes": (ctypes.c_size_t, [_i64, _i64]),
    "ck_convrot_nvfp4_linear": (_st, [_vp, _i64, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                      ctypes.c_size_t, _vp]),
    "ck_int8_linear_host": (_st, [_vp, _i64, _st, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                  _vp, ctypes.c_size_t, _vp]),
    "ck_status_string": (ctypes.c_char_p, [_st]),
    "ck_get_device_error": (_st, []),
    "ck_is_checked_build": (ctypes.c_int, []),
    "ck_checked_violations": (ctypes.c_uint, []),
    "ck_clear_device_error": (_st, []),
    "ck_test_int8_gemm_i32": (_st, [_vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "ck_test_quantize_rowwise_norotate": (_st, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "ck_test_inject_producer_stall": (_st, [ctypes.c_int, _i64]),
    "ck_test_input_act": (_st, [_vp, _i64, _st, _vp, _vp]),
    "ck_test_row_quant_params": (_st, [_vp, _i64, ctypes.c_int, _vp, _vp, _vp]),
    "ck_test_i8_mma_peak": (_st, [_i64, ctypes.POINTER(ctypes.c_int), _vp]),
    "ck_test_checked_fire": (_st, [_vp]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class CKError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(status: int) -> str:
    return lib.ck_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != CK_OK:
        raise CKError(status, where)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D, got shape {tuple(t.shape)}")
    if t.numel() and t.stride(-1) != 1:
        raise ValueError(f"{name} must have unit stride in its last dimension")


def _rows_contiguous(t: torch.Tensor, name: str) -> None:
    if t.numel() and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def workspace_bytes(M: int, K: int) -> int:
    return int(lib.ck_int8_linear_workspace_bytes(M, K))


def rotate_quant_weight(W: torch.Tensor, Qw: torch.Tensor | None = None,
                        s_w: torch.Tensor | None = None, stream=None):
    """Offline: ConvRot256 along K and per-output-row INT8 of fp32 W [N, K]."""
    _need(W, "W", torch.float32, 2)
    _rows_contiguous(W, "W")
    N, K = W.shape
    if Qw is None:
        Qw = torch.empty((N, K), dtype=torch.int8, device=W.device)
    if s_w is None:
        s_w = torch.empty((N,), dtype=torch.float32, device=W.device)
    _need(Qw, "Qw", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    _check(lib.ck_rotate_quant_weight(_ptr(W), N, K, _ptr(Qw), _ptr(s_w), _stream(stream)),
           "ck_rotate_quant_weight")
    return Qw, s_w


def _quant(fn, name, X, Qx, s_x, stream):
    _need(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    if Qx is None:
        Qx = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if s_x is None:
        s_x = torch.empty((M,), dtype=torch.float32, device=X.device)
    _need(Qx, "Qx", torch.int8, 2)
    _rows_contiguous(Qx, "Qx")
    _need(s_x, "s_x", torch.float32, 1)
    _check(fn(_ptr(X), M, K, ldx, _ptr(Qx), _ptr(s_x), _stream(stream)), name)
    return Qx, s_x


def quantize_rotate_rowwise(X: torch.Tensor, Qx=None, s_x=None, stream=None):
    """quantize_and_rotate_rowwise: ConvRot256 + per-row INT8 of bf16 X [M, K]
    (row stride X.stride(0)). Returns (Qx int8 [M, K], s_x fp32 [M])."""
    return _quant(lib.ck_quantize_rotate_rowwise, "ck_quantize_rotate_rowwise", X, Qx, s_x, stream)


def quantize_rotate_rowwise_act(X: torch.Tensor, act: str, Qx=None, s_x=None, stream=None):
    """quantize_and_rotate_rowwise after an input activation ("none", "relu",
    "silu", "gelu_tanh"), applied inside the quantiser's load."""
    a = ACTS[act]
    return _quant(lambda *args: lib.ck_quantize_rotate_rowwise_act(*args[:4], a, *args[4:]),
                  "ck_quantize_rotate_rowwise_act", X, Qx, s_x, stream)


def quantize_int8_rowwise(X: torch.Tensor, Qx=None, s_x=None, stream=None):
    """quantize_int8_rowwise: per-row INT8 of bf16 X [M, K] without rotation."""
    return _quant(lib.ck_quantize_int8_rowwise, "ck_quantize_int8_rowwise", X, Qx, s_x, stream)


def test_quantize_rowwise_norotate(X: torch.Tensor, Qx=None, s_x=None, stream=None):
    return _quant(lib.ck_test_quantize_rowwise_norotate, "ck_test_quantize_rowwise_norotate",
                  X, Qx, s_x, stream)


test_quantize_rowwise_norotate.__test__ = False


def int8_linear(X: torch.Tensor, Qw: torch.Tensor, s_w: torch.Tensor,
                bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, stream=None,
                input_act: str = "none") -> torch.Tensor:
    """Y[M, N] = bf16(((int8 GEMM of rotate+quantised act(X) with Qw) * s_x) * s_w + bias).
    ``input_act`` ("none", "relu", "silu", "gelu_tanh") is applied inside the
    quantiser's load (ck_int8_linear_act); "none" calls ck_int8_linear."""
    _need(X, "X", torch.bfloat16, 2)
    _need(Qw, "Qw", torch.int8, 2)
    _rows_contiguous(Qw, "Qw")
    _need(s_w, "s_w", torch.float32, 1)
    M, K = X.shape
    N = Qw.shape[0]
    if Qw.shape[1] != K or s_w.shape[0] != N:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, Qw {tuple(Qw.shape)}, s_w {tuple(s_w.shape)}")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
        if bias.shape[0] != N:
            raise ValueError("bias must have N elements")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    need = workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    ws_bytes = workspace.numel() * workspace.element_size()
    if input_act == "none":
        _check(lib.ck_int8_linear(_ptr(X), ldx, _ptr(Qw), _ptr(s_w), _ptr(bias), _ptr(out), M, N,
                                  K, _ptr(workspace), ws_bytes, _stream(stream)), "ck_int8_linear")
    else:
        _check(lib.ck_int8_linear_act(_ptr(X), ldx, ACTS[input_act], _ptr(Qw), _ptr(s_w),
                                      _ptr(bias), _ptr(out), M, N, K, _ptr(workspace), ws_bytes,
                                      _stream(stream)), "ck_int8_linear_act")
    return out


def _row_stride(t: torch.Tensor, K: int) -> int:
    return t.stride(0) if t.shape[0] > 1 else max(K, t.stride(0))


def _norm_args(X, residual, residual_out, g):
    _need(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if X.stride(1) != 1:
        raise ValueError("X must have a unit column stride")
    for name, t in (("residual", residual), ("residual_out", residual_out)):
        if t is not None:
            _need(t, name, torch.bfloat16, 2)
            if tuple(t.shape) != (M, K) or t.stride(1) != 1:
                raise ValueError(f"{name} must be [M, K] bf16 with unit column stride")
    if g is not None:
        _need(g, "g", torch.bfloat16, 1)
        if g.shape[0] != K or not g.is_contiguous():
            raise ValueError("g must be a contiguous [K] bf16 tensor")
    ldr = _row_stride(residual, K) if residual is not None else K
    ldo = _row_stride(residual_out, K) if residual_out is not None else K
    return M, K, ldr, ldo


def rmsnorm_residual(X: torch.Tensor, residual: torch.Tensor | None = None,
                     g: torch.Tensor | None = None, eps: float = 1e-6,
                     residual_out: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """The input RMSNorm of int8_linear (ck_rmsnorm_residual): h = bf16(X +
    residual) (h = X without one), written to ``residual_out`` when given (it
    may be ``residual`` itself); returns bf16((h / sqrt(mean(h^2) + eps)) * g)."""
    M, K, ldr, ldo = _norm_args(X, residual, residual_out, g)
    if out is None:
        out = torch.empty((M, K), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    _check(lib.ck_rmsnorm_residual(_ptr(X), _row_stride(X, K), _ptr(residual), ldr,
                                   _ptr(residual_out), ldo, _ptr(g), float(eps), M, K, _ptr(out),
                                   _stream(stream)), "ck_rmsnorm_residual")
    return out


NORM_FUSED_MAX_K = 14336


def quantize_rotate_rowwise_norm(X: torch.Tensor, residual: torch.Tensor | None = None,
                                 g: torch.Tensor | None = None, eps: float = 1e-6,
                                 residual_out: torch.Tensor | None = None, Qx=None, s_x=None,
                                 stream=None):
    """quantize_and_rotate_rowwise of the input RMSNorm of X in one kernel
    (ck_quantize_rotate_rowwise_norm): the normalised rows are never stored.
    Returns (Qx int8 [M, K], s_x fp32 [M]); K <= NORM_FUSED_MAX_K."""
    M, K, ldr, ldo = _norm_args(X, residual, residual_out, g)
    if Qx is None:
        Qx = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if s_x is None:
        s_x = torch.empty((M,), dtype=torch.float32, device=X.device)
    _need(Qx, "Qx", torch.int8, 2)
    _rows_contiguous(Qx, "Qx")
    _need(s_x, "s_x", torch.float32, 1)
    _check(lib.ck_quantize_rotate_rowwise_norm(_ptr(X), _row_stride(X, K), _ptr(residual), ldr,
                                               _ptr(residual_out), ldo, _ptr(g), float(eps), M, K,
                                               _ptr(Qx), _ptr(s_x), _stream(stream)),
           "ck_quantize_rotate_rowwise_norm")
    return Qx, s_x


def norm_workspace_bytes(M: int, K: int) -> int:
    return int(lib.ck_int8_linear_norm_workspace_bytes(M, K))


def int8_linear_norm(X: torch.Tensor, Qw: torch.Tensor, s_w: torch.Tensor,
                     bias: torch.Tensor | None = None, residual: torch.Tensor | None = None,
                     g: torch.Tensor | None = None, eps: float = 1e-6,
                     residual_out: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """int8_linear on the input RMSNorm (and residual) of X (ck_int8_linear_norm)."""
    M, K, ldr, ldo = _norm_args(X, residual, residual_out, g)
    _need(Qw, "Qw", torch.int8, 2)
    _rows_contiguous(Qw, "Qw")
    _need(s_w, "s_w", torch.float32, 1)
    N = Qw.shape[0]
    if Qw.shape[1] != K or s_w.shape[0] != N:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, Qw {tuple(Qw.shape)}, s_w {tuple(s_w.shape)}")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
        if bias.shape[0] != N:
            raise ValueError("bias must have N elements")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    need = norm_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.ck_int8_linear_norm(_ptr(X), _row_stride(X, K), _ptr(residual), ldr,
                                   _ptr(residual_out), ldo, _ptr(g), float(eps), _ptr(Qw),
                                   _ptr(s_w), _ptr(bias), _ptr(out), M, N, K, _ptr(workspace),
                                   ws_bytes, _stream(stream)), "ck_int8_linear_norm")
    return out


def host_workspace_bytes(chunk_rows: int, N: int, K: int) -> int:
    return int(lib.ck_int8_linear_host_workspace_bytes(chunk_rows, N, K))


def int8_linear_host(X: torch.Tensor, Qw: torch.Tensor, s_w: torch.Tensor,
                     bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     chunk_rows: int = 2048, workspace: torch.Tensor | None = None, stream=None,
                     input_act: str = "none") -> torch.Tensor:
    """int8_linear for X and Y in host memory (ck_int8_linear_host): the rows
    go through the GPU in chunks with the copies in and out overlapped with the
    kernels. X and ``out`` should be pinned CPU tensors for the overlap; the
    result is ready once ``stream`` (default: the current stream of Qw's
    device) has completed."""
    if X.device.type != "cpu":
        raise ValueError("X must be a CPU tensor (use int8_linear for device tensors)")
    if X.dtype != torch.bfloat16 or X.dim() != 2 or X.stride(1) != 1:
        raise ValueError("X must be a 2-D bf16 CPU tensor with unit column stride")
    _need(Qw, "Qw", torch.int8, 2)
    _rows_contiguous(Qw, "Qw")
    _need(s_w, "s_w", torch.float32, 1)
    M, K = X.shape
    N = Qw.shape[0]
    if Qw.shape[1] != K or s_w.shape[0] != N:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, Qw {tuple(Qw.shape)}, s_w {tuple(s_w.shape)}")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
    if (out.device.type != "cpu" or out.dtype != torch.bfloat16 or tuple(out.shape) != (M, N)
            or not out.is_contiguous()):
        raise ValueError("out must be a contiguous [M, N] bf16 CPU tensor")
    chunk_rows = max(1, min(int(chunk_rows), max(M, 1)))
    need = host_workspace_bytes(chunk_rows, N, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=Qw.device)
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    with torch.cuda.device(Qw.device):
        _check(lib.ck_int8_linear_host(_ptr(X), ldx, ACTS[input_act], _ptr(Qw), _ptr(s_w),
                                       _ptr(bias), _ptr(out), M, N, K, chunk_rows,
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)), "ck_int8_linear_host")
    return out


def int8_linear_noalloc(X: torch.Tensor, Qw: torch.Tensor, s_w: torch.Tensor,
                        bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """int8_linear for callers that cannot allocate device memory: the codes
    and row scales go to the library's fixed 32 MiB device array instead of a
    workspace (needs workspace_bytes(M, K) <= NOALLOC_SCRATCH_BYTES). Calls on
    one device share that array, so they must not overlap on the GPU. ``out``
    should be passed by such callers (otherwise this wrapper allocates it)."""
    _need(X, "X", torch.bfloat16, 2)
    _need(Qw, "Qw", torch.int8, 2)
    _rows_contiguous(Qw, "Qw")
    _need(s_w, "s_w", torch.float32, 1)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    M, K = X.shape
    N = Qw.shape[0]
    if Qw.shape[1] != K or s_w.shape[0] != N or (bias is not None and bias.shape[0] != N):
        raise ValueError("shape mismatch between X, Qw, s_w and bias")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    for t, name in ((Qw, "Qw"), (s_w, "s_w"), (bias, "bias"), (out, "out")):
        if t is not None and t.device != X.device:
            raise ValueError(f"{name} is on {t.device}, X on {X.device}")
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    with torch.cuda.device(X.device):
        _check(lib.ck_int8_linear_noalloc(_ptr(X), ldx, _ptr(Qw), _ptr(s_w), _ptr(bias),
                                          _ptr(out), M, N, K, _stream(stream)),
               "ck_int8_linear_noalloc")
    return out


def rotate_quant_weight_int4(W: torch.Tensor, Qw4: torch.Tensor | None = None,
                             s_w: torch.Tensor | None = None, stream=None):
    """Offline: ConvRot256 + per-row signed INT4 of fp32 W [N, K], packed two
    codes per byte. Returns (Qw4 uint8 [N, K/2], s_w fp32 [N])."""
    _need(W, "W", torch.float32, 2)
    _rows_contiguous(W, "W")
    N, K = W.shape
    if Qw4 is None:
        Qw4 = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    if s_w is None:
        s_w = torch.empty((N,), dtype=torch.float32, device=W.device)
    _need(Qw4, "Qw4", torch.uint8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    _check(lib.ck_rotate_quant_weight_int4(_ptr(W), N, K, _ptr(Qw4), _ptr(s_w), _stream(stream)),
           "ck_rotate_quant_weight_int4")
    return Qw4, s_w


def unpack_int4(Qw4: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Packed INT4 [N, K/2] -> int8 codes [N, K]."""
    _need(Qw4, "Qw4", torch.uint8, 2)
    _rows_contiguous(Qw4, "Qw4")
    N, K = Qw4.shape[0], 2 * Qw4.shape[1]
    if out is None:
        out = torch.empty((N, K), dtype=torch.int8, device=Qw4.device)
    _need(out, "out", torch.int8, 2)
    _check(lib.ck_unpack_int4(_ptr(Qw4), N, K, _ptr(out), _stream(stream)), "ck_unpack_int4")
    return out


def quantize_rotate_rowwise_int4(X: torch.Tensor, Qx=None, s_x=None, stream=None):
    """ConvRot256 + per-row signed INT4 codes (int8 storage, [-7, 7]) of bf16 X."""
    return _quant(lib.ck_quantize_rotate_rowwise_int4, "ck_quantize_rotate_rowwise_int4", X, Qx,
                  s_x, stream)


def w4a4_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib.ck_convrot_w4a4_linear_workspace_bytes(M, N, K))


def convrot_w4a4_linear(X: torch.Tensor, Qw4: torch.Tensor, s_w: torch.Tensor,
                        bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """convrot_w4a4_linear: INT4 codes of rotated X times the unpacked INT4
    weights, INT32 accumulation, int8_linear's epilogue."""
    _need(X, "X", torch.bfloat16, 2)
    _need(Qw4, "Qw4", torch.uint8, 2)
    _rows_contiguous(Qw4, "Qw4")
    _need(s_w, "s_w", torch.float32, 1)
    M, K = X.shape
    N = Qw4.shape[0]
    if 2 * Qw4.shape[1] != K or s_w.shape[0] != N:
        raise ValueError("shape mismatch between X, Qw4 and s_w")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    need = w4a4_workspace_bytes(M, N, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    _check(lib.ck_convrot_w4a4_linear(_ptr(X), ldx, _ptr(Qw4), _ptr(s_w), _ptr(bias), _ptr(out),
                                      M, N, K, _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)), "ck_convrot_w4a4_linear")
    return out


def convrot_w4a4_linear_unpacked(X: torch.Tensor, Qw: torch.Tensor, s_w: torch.Tensor,
                                 bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                                 workspace: torch.Tensor | None = None,
                                 stream=None) -> torch.Tensor:
    """convrot_w4a4_linear on weights unpacked once offline (``unpack_int4``:
    int8 codes in [-7, 7], [N, K]); no unpack per call."""
    _need(X, "X", torch.bfloat16, 2)
    _need(Qw, "Qw", torch.int8, 2)
    _rows_contiguous(Qw, "Qw")
    _need(s_w, "s_w", torch.float32, 1)
    M, K = X.shape
    N = Qw.shape[0]
    if Qw.shape[1] != K or s_w.shape[0] != N:
        raise ValueError("shape mismatch between X, Qw and s_w")
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    need = workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    _check(lib.ck_convrot_w4a4_linear_unpacked(_ptr(X), ldx, _ptr(Qw), _ptr(s_w), _ptr(bias),
                                               _ptr(out), M, N, K, _ptr(workspace),
                                               workspace.numel() * workspace.element_size(),
                                               _stream(stream)),
           "ck_convrot_w4a4_linear_unpacked")
    return out


def dequantize_int8(Q: torch.Tensor, s: torch.Tensor, per_row: bool = True,
                    dtype: torch.dtype = torch.float32, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """dequantize_int8_simple (fp32) / _dtype (bf16): float(Q) * s."""
    _need(Q, "Q", torch.int8, 2)
    _rows_contiguous(Q, "Q")
    _need(s, "s", torch.float32, 1)
    if dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("dtype must be float32 or bfloat16")
    rows, K = Q.shape
    if out is None:
        out = torch.empty((rows, K), dtype=dtype, device=Q.device)
    _need(out, "out", dtype, 2)
    _check(lib.ck_dequantize_int8(_ptr(Q), _ptr(s), rows, K, int(per_row),
                                  int(dtype == torch.bfloat16), _ptr(out), _stream(stream)),
           "ck_dequantize_int8")
    return out


def quantize_int8_tensorwise(X: torch.Tensor, Q: torch.Tensor | None = None,
                             s: torch.Tensor | None = None, stream=None):
    """quantize_int8_tensorwise: one scale for the whole bf16 tensor."""
    _need(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    if Q is None:
        Q = torch.empty((M, K), dtype=torch.int8, device=X.device)
    if s is None:
        s = torch.empty((1,), dtype=torch.float32, device=X.device)
    _check(lib.ck_quantize_int8_tensorwise(_ptr(X), M, K, ldx, _ptr(Q), _ptr(s), _stream(stream)),
           "ck_quantize_int8_tensorwise")
    return Q, s


def int8_gemm_rowscale(Qx: torch.Tensor, s_x: torch.Tensor, Qw: torch.Tensor, s_w: torch.Tensor,
                       bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """The GEMM + fused epilogue on already quantised activations."""
    _need(Qx, "Qx", torch.int8, 2)
    _rows_contiguous(Qx, "Qx")
    _need(Qw, "Qw", torch.int8, 2)
    _rows_contiguous(Qw, "Qw")
    _need(s_x, "s_x", torch.float32, 1)
    _need(s_w, "s_w", torch.float32, 1)
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
    M, K = Qx.shape
    N = Qw.shape[0]
    if Qw.shape[1] != K or s_x.shape[0] != M or s_w.shape[0] != N:
        raise ValueError("shape mismatch between Qx, s_x, Qw and s_w")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Qx.device)
    _need(out, "out", torch.bfloat16, 2)
    _rows_contiguous(out, "out")
    _check(lib.ck_int8_gemm_rowscale(_ptr(Qx), _ptr(s_x), _ptr(Qw), _ptr(s_w), _ptr(bias),
                                     _ptr(out), M, N, K, _stream(stream)), "ck_int8_gemm_rowscale")
    return out


def test_int8_gemm_i32(Qx: torch.Tensor, Qw: torch.Tensor, out: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """Raw INT32 accumulators of the GEMM (test hook)."""
    _need(Qx, "Qx", torch.int8, 2)
    _need(Qw, "Qw", torch.int8, 2)
    M, K = Qx.shape
    N = Qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.int32, device=Qx.device)
    _check(lib.ck_test_int8_gemm_i32(_ptr(Qx), _ptr(Qw), _ptr(out), M, N, K, _stream(stream)),
           "ck_test_int8_gemm_i32")
    return out


test_int8_gemm_i32.__test__ = False


def test_input_act(X: torch.Tensor, act: str, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """The input activation alone, as the quantiser applies it (test hook):
    X contiguous bf16 with numel % 256 == 0."""
    if X.dtype != torch.bfloat16 or not X.is_cuda or not X.is_contiguous():
        raise ValueError("X must be a contiguous CUDA bf16 tensor")
    if out is None:
        out = torch.empty_like(X)
    _check(lib.ck_test_input_act(_ptr(X), X.numel(), ACTS[act], _ptr(out), _stream(stream)),
           "ck_test_input_act")
    return out


test_input_act.__test__ = False


def test_row_quant_params(amax: torch.Tensor, q: int = 127, stream=None):
    """The rotated quantiser's per-row divisor and reciprocal for each row
    absmax in `amax` (contiguous CUDA fp32; test hook). Returns (div, rc)."""
    if amax.dtype != torch.float32 or not amax.is_cuda or not amax.is_contiguous():
        raise ValueError("amax must be a contiguous CUDA float32 tensor")
    div = torch.empty_like(amax)
    rc = torch.empty_like(amax)
    _check(lib.ck_test_row_quant_params(_ptr(amax), amax.numel(), q, _ptr(div), _ptr(rc),
                                        _stream(stream)), "ck_test_row_quant_params")
    return div, rc


test_row_quant_params.__test__ = False


def test_i8_mma_peak(mmas_per_pair: int, stream=None) -> int:
    """Launches the INT8 tensor-core peak probe; returns the operations it
    performs (4194304 per pair MMA) for the caller's event timing."""
    pairs = ctypes.c_int(0)
    _check(lib.ck_test_i8_mma_peak(mmas_per_pair, ctypes.byref(pairs), _stream(stream)),
           "ck_test_i8_mma_peak")
    return 2 * 256 * 256 * 32 * mmas_per_pair * pairs.value


test_i8_mma_peak.__test__ = False


def device_error() -> int:
    """Synchronises the device; returns CK_ERR_DEVICE_TIMEOUT if a kernel gave up on a wait."""
    return int(lib.ck_get_device_error())


def is_checked_build() -> bool:
    """True when the loaded library is the checked build (libck_checked.so)."""
    return bool(lib.ck_is_checked_build())


def checked_violations() -> int:
    """Class bits of the checked build's failed checks since the last call
    (1 global store, 2 global load, 4 shared memory, 8 bulk copy, 16 TMEM),
    then cleared; always 0 for libck.so. Synchronises the current device."""
    return int(lib.ck_checked_violations())


def test_checked_fire(stream=None) -> None:
    """Test hook: one failed index check with no access behind it (class bit
    4 in the checked build; a no-op in libck.so)."""
    _check(lib.ck_test_checked_fire(_stream(stream)), "ck_test_checked_fire")


def clear_device_error() -> None:
    _check(lib.ck_clear_device_error(), "ck_clear_device_error")


def inject_producer_stall(mode: int = 1, wait_limit_ns: int = 0) -> None:
    _check(lib.ck_test_inject_producer_stall(mode, wait_limit_ns), "ck_test_inject_producer_stall")


# ----------------------------------------------------------------- ConvRot NVFP4


def nvfp4_scale_bytes(rows: int, K: int) -> int:
    return int(lib.ck_nvfp4_scale_bytes(rows, K))


def _nvfp4_out(rows, K, device):
    Q = torch.empty((rows, K // 2), dtype=torch.uint8, device=device)
    S = torch.empty((max(nvfp4_scale_bytes(rows, K), 1),), dtype=torch.uint8, device=device)
    s_t = torch.empty((1,), dtype=torch.float32, device=device)
    return Q, S, s_t


def quantize_rotate_nvfp4(X: torch.Tensor, Q=None, S=None, s_t=None, stream=None):
    """ConvRot NVFP4 of bf16 X [M, K]: (codes [M, K/2] uint8, blocked E4M3
    scales (uint8), per-tensor scale [1] fp32), all on X's device; Q, S and
    s_t may be given (sizes as returned)."""
    _need(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    if Q is None or S is None or s_t is None:
        Q, S, s_t = _nvfp4_out(M, K, X.device)
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    _check(lib.ck_quantize_rotate_nvfp4(_ptr(X), M, K, ldx, _ptr(Q), _ptr(S), _ptr(s_t),
                                        _stream(stream)), "ck_quantize_rotate_nvfp4")
    return Q, S, s_t


def rotate_quant_weight_nvfp4(W: torch.Tensor, stream=None):
    _need(W, "W", torch.float32, 2)
    _rows_contiguous(W, "W")
    N, K = W.shape
    Q, S, s_t = _nvfp4_out(N, K, W.device)
    _check(lib.ck_rotate_quant_weight_nvfp4(_ptr(W), N, K, _ptr(Q), _ptr(S), _ptr(s_t),
                                            _stream(stream)), "ck_rotate_quant_weight_nvfp4")
    return Q, S, s_t


def dequantize_nvfp4(Q: torch.Tensor, S: torch.Tensor, s_t: torch.Tensor, hi_first: bool = False,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(Q, "Q", torch.uint8, 2)
    rows, K2 = Q.shape
    if out is None:
        out = torch.empty((rows, 2 * K2), dtype=torch.float32, device=Q.device)
    _check(lib.ck_dequantize_nvfp4(_ptr(Q), _ptr(S), _ptr(s_t), rows, 2 * K2, int(bool(hi_first)),
                                   _ptr(out), _stream(stream)), "ck_dequantize_nvfp4")
    return out


def nvfp4_gemm(Qa, Sa, s_ta, Qw, Sw, s_tw, bias: torch.Tensor | None = None,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(Qa, "Qa", torch.uint8, 2)
    _need(Qw, "Qw", torch.uint8, 2)
    M, K2 = Qa.shape
    N = Qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=Qa.device)
    _check(lib.ck_nvfp4_gemm(_ptr(Qa), _ptr(Sa), _ptr(s_ta), _ptr(Qw), _ptr(Sw), _ptr(s_tw),
                             _ptr(bias), _ptr(out), M, N, 2 * K2, _stream(stream)), "ck_nvfp4_gemm")
    return out


def nvfp4_workspace_bytes(M: int, K: int) -> int:
    return int(lib.ck_convrot_nvfp4_linear_workspace_bytes(M, K))


def convrot_nvfp4_linear(X: torch.Tensor, Qw, Sw, s_tw, bias: torch.Tensor | None = None,
                         out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """ConvRot NVFP4 linear: rotate + NVFP4-quantise X, block-scaled FP4 GEMM,
    Y = bf16(acc * s_ta * s_tw + bias)."""
    _need(X, "X", torch.bfloat16, 2)
    M, K = X.shape
    N = Qw.shape[0]
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    need = nvfp4_workspace_bytes(M, K)
    if workspace is None:
        workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=X.device)
    ldx = X.stride(0) if M > 1 else max(K, X.stride(0))
    _check(lib.ck_convrot_nvfp4_linear(_ptr(X), ldx, _ptr(Qw), _ptr(Sw), _ptr(s_tw), _ptr(bias),
                                       _ptr(out), M, N, K, _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)), "ck_convrot_nvfp4_linear")
    return out
