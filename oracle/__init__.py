"""CPU oracle for the ConvRot256 INT8 linear path (test infrastructure).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs are the only callers.
The CUDA product path never imports this package, and this package imports
nothing from the product.

The arithmetic lives in ``convrot_oracle.c`` (plain C, IEEE fp32, no
contraction; double precision where a step is defined as the bf16 rounding of
an exact value); this module compiles it with gcc on first use and wraps it with
numpy arrays. BF16 values travel as numpy ``uint16`` bit patterns.

What each function follows (page title, section):
  - ``rot256``: ConvRot256 as named in the sglang PR "Tune Kitchen INT8 row
    splitting for SM120" (Accuracy Test) and called a Hadamard rotation in the
    ComfyUI-AppleSilicon-FP8 README ("What it fixes", row 17); read as the
    normalised Sylvester Walsh-Hadamard transform, stages h = 1..128, then /16.
  - ``quantize_rows``: comfy-kitchen 0.2.40, "Huawei Ascend backend"
    (quantize_int8_rowwise, quantize_and_rotate_rowwise); s = absmax/127,
    q = round-half-even(y/s) clamped to [-127, 127].
  - ``gemm_i32`` / ``epilogue`` / ``int8_linear``: ComfyUI-AppleSilicon-FP8
    README row 17 (INT8 x INT8 -> INT32, per-row rescale + bias in the store
    epilogue) and comfy-kitchen "int8_linear".
  - ``act_bf16`` (input_act): comfy-kitchen 0.2.40, "HIP backend"
    (int8_linear(input_act=...) folded into the quantiser's load); each bf16
    input becomes the bf16 value nearest to the exact relu / silu / tanh-form
    gelu of it, evaluated in double precision.
  - ``rmsnorm_rows``: comfy-kitchen 0.2.40, "Huawei Ascend backend"
    (int8_linear's input RMSNorm and residual arguments): h = bf16(x + r),
    y = the bf16 value nearest to the exact h g / sqrt(mean(h^2) + eps).
  - ``e2m1_*``, ``e4m3_*``, ``nvfp4_*``: ComfyUI-HSWQ-Loader-and-Tools, "NVFP4
    torch.compile Fix", section 5-1 (nvfp4_gemm.py): the E2M1 value table,
    16-value blocks, the blocked scale layout that from_blocked undoes, a
    per-tensor scale, dequantisation and a_dq @ w_dq.T + bias; the quantiser
    (two-level scales: s_t = amax / 2688, E4M3 block scales) is this build's
    reading, stated in convrot_oracle.c.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "convrot_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
          "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle library with gcc (in-tree) and return its path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _P(t):
    return ctypes.POINTER(t)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            # A test may point this at a deliberately broken copy of the
            # oracle to show that the pins catch the mistake.
            override = os.environ.get("CONVROT_ORACLE_LIB")
            L = ctypes.CDLL(override if override else build())
            i64, f32p = ctypes.c_int64, _P(ctypes.c_float)
            u16p, i8p, i32p = _P(ctypes.c_uint16), _P(ctypes.c_int8), _P(ctypes.c_int32)
            L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.oracle_bf16_to_f32.restype = ctypes.c_float
            L.oracle_f32_to_bf16_rne.argtypes = [ctypes.c_float]
            L.oracle_f32_to_bf16_rne.restype = ctypes.c_uint16
            L.oracle_rot256.argtypes = [f32p]
            L.oracle_rot256.restype = None
            L.oracle_quant_row.argtypes = [f32p, i64, i8p, f32p]
            L.oracle_quant_row.restype = None
            L.oracle_quantize_rows_bf16.argtypes = [u16p, i64, i64, i64, ctypes.c_int, i8p, f32p]
            L.oracle_quantize_rows_bf16.restype = ctypes.c_int
            L.oracle_quantize_rows_bf16_act.argtypes = [u16p, i64, i64, i64, ctypes.c_int,
                                                        ctypes.c_int, i8p, f32p]
            L.oracle_quantize_rows_bf16_act.restype = ctypes.c_int
            L.oracle_quantize_rows_bf16_q.argtypes = [u16p, i64, i64, i64, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_float, i8p, f32p]
            L.oracle_quantize_rows_bf16_q.restype = ctypes.c_int
            L.oracle_quant_row_q.argtypes = [f32p, i64, ctypes.c_float, i8p, f32p]
            L.oracle_quant_row_q.restype = None
            u8p = _P(ctypes.c_uint8)
            L.oracle_rotate_quant_weight_int4.argtypes = [f32p, i64, i64, u8p, f32p]
            L.oracle_rotate_quant_weight_int4.restype = ctypes.c_int
            L.oracle_unpack_int4.argtypes = [u8p, i64, i64, i8p]
            L.oracle_unpack_int4.restype = None
            L.oracle_dequantize_int8.argtypes = [i8p, f32p, i64, i64, ctypes.c_int, f32p, u16p]
            L.oracle_dequantize_int8.restype = None
            L.oracle_quantize_int8_tensorwise.argtypes = [u16p, i64, i64, i64, i8p, f32p]
            L.oracle_quantize_int8_tensorwise.restype = None
            L.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
            L.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
            L.oracle_act_f64.argtypes = [ctypes.c_int, ctypes.c_double]
            L.oracle_act_f64.restype = ctypes.c_double
            L.oracle_act_bf16_array.argtypes = [ctypes.c_int, u16p, i64, u16p]
            L.oracle_act_bf16_array.restype = None
            L.oracle_rotate_quant_weight.argtypes = [f32p, i64, i64, i8p, f32p]
            L.oracle_rotate_quant_weight.restype = ctypes.c_int
            L.oracle_gemm_i32.argtypes = [i8p, i8p, i64, i64, i64, i32p]
            L.oracle_gemm_i32.restype = None
            L.oracle_epilogue.argtypes = [i32p, f32p, f32p, u16p, i64, i64, u16p]
            L.oracle_epilogue.restype = None
            L.oracle_linear_rows.argtypes = [i8p, f32p, i8p, f32p, u16p, i64, i64,
                                             _P(ctypes.c_int64), i64, u16p]
            L.oracle_linear_rows.restype = None
            L.oracle_e2m1_to_f32.argtypes = [ctypes.c_uint8]
            L.oracle_e2m1_to_f32.restype = ctypes.c_float
            L.oracle_f32_to_e2m1_rne.argtypes = [ctypes.c_float]
            L.oracle_f32_to_e2m1_rne.restype = ctypes.c_uint8
            L.oracle_e4m3_to_f32.argtypes = [ctypes.c_uint8]
            L.oracle_e4m3_to_f32.restype = ctypes.c_float
            L.oracle_f32_to_e4m3_rne.argtypes = [ctypes.c_float]
            L.oracle_f32_to_e4m3_rne.restype = ctypes.c_uint8
            L.oracle_nvfp4_sf_offset.argtypes = [i64, i64, i64]
            L.oracle_nvfp4_sf_offset.restype = i64
            L.oracle_nvfp4_sf_bytes.argtypes = [i64, i64]
            L.oracle_nvfp4_sf_bytes.restype = i64
            L.oracle_quantize_rotate_nvfp4_bf16.argtypes = [u16p, i64, i64, i64, u8p, u8p, f32p]
            L.oracle_quantize_rotate_nvfp4_bf16.restype = ctypes.c_int
            L.oracle_rotate_quant_weight_nvfp4.argtypes = [f32p, i64, i64, u8p, u8p, f32p]
            L.oracle_rotate_quant_weight_nvfp4.restype = ctypes.c_int
            L.oracle_dequantize_nvfp4.argtypes = [u8p, u8p, ctypes.c_float, i64, i64, ctypes.c_int,
                                                  f32p]
            L.oracle_dequantize_nvfp4.restype = None
            L.oracle_nvfp4_linear_rows.argtypes = [u8p, u8p, ctypes.c_float, i64, u8p, u8p,
                                                   ctypes.c_float, i64, u16p, i64,
                                                   _P(ctypes.c_int64), i64, u16p,
                                                   _P(ctypes.c_double)]
            L.oracle_nvfp4_linear_rows.restype = None
            L.oracle_rmsnorm_rows.argtypes = [u16p, i64, u16p, i64, u16p, ctypes.c_float, i64,
                                              i64, u16p, u16p, u16p]
            L.oracle_rmsnorm_rows.restype = ctypes.c_int
            L.oracle_num_threads.argtypes = []
            L.oracle_num_threads.restype = ctypes.c_int
            _lib = L
    return _lib


def _ptr(a: np.ndarray, ct):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(_P(ct))


def num_threads() -> int:
    """OpenMP threads the oracle's row loops use (OMP_NUM_THREADS, else all cores)."""
    return lib().oracle_num_threads()


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    """fp32 -> bf16 bits, round-to-nearest-even (the oracle's own C routine)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    L = lib()
    out = np.empty(x.shape, np.uint16)
    flat, fo = x.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        fo[i] = L.oracle_f32_to_bf16_rne(float(flat[i]))
    return out


def rot256(v) -> np.ndarray:
    """ConvRot256 of one block (or of each row of a [R, 256] array), fp32."""
    a = np.array(v, dtype=np.float32, copy=True)
    flat = a.reshape(-1, 256)
    L = lib()
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        L.oracle_rot256(_ptr(row, ctypes.c_float))
        flat[r] = row
    return flat.reshape(a.shape)


def quant_rows(y, qmax: float = 127.0) -> tuple[np.ndarray, np.ndarray]:
    """Per-row symmetric quantisation of fp32 rows [R, K] (no rotation) to
    codes in [-qmax, qmax] (127: INT8, 7: signed INT4 in int8 storage)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    y2 = y.reshape(-1, y.shape[-1])
    R, K = y2.shape
    q = np.empty((R, K), np.int8)
    s = np.empty(R, np.float32)
    L = lib()
    for r in range(R):
        row = np.ascontiguousarray(y2[r])
        qr = np.empty(K, np.int8)
        sr = np.empty(1, np.float32)
        L.oracle_quant_row_q(_ptr(row, ctypes.c_float), K, float(qmax), _ptr(qr, ctypes.c_int8),
                             _ptr(sr, ctypes.c_float))
        q[r], s[r] = qr, sr[0]
    return q, s


ACTS = {"none": 0, "relu": 1, "silu": 2, "gelu_tanh": 3}


def f64_to_bf16(v) -> np.ndarray:
    """float64 -> bf16 bits, round-to-nearest-even from the double value directly."""
    v = np.asarray(v, dtype=np.float64)
    L = lib()
    return np.array([L.oracle_f64_to_bf16_rne(float(t)) for t in v.reshape(-1)],
                    np.uint16).reshape(v.shape)


def act_f64(name: str, x) -> np.ndarray:
    """The activation evaluated in double precision (before any rounding)."""
    x = np.asarray(x, dtype=np.float64)
    L = lib()
    a = ACTS[name]
    return np.array([L.oracle_act_f64(a, float(t)) for t in x.reshape(-1)],
                    np.float64).reshape(x.shape)


def act_bf16(name: str, x_bits) -> np.ndarray:
    """input_act as the quantiser applies it: each bf16 input (uint16 bits)
    becomes the bf16 value nearest to the exact act(x), ties to even."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    y = np.empty_like(x)
    lib().oracle_act_bf16_array(ACTS[name], _ptr(x.reshape(-1), ctypes.c_uint16), x.size,
                                _ptr(y.reshape(-1), ctypes.c_uint16))
    return y


def quantize_rows_bf16(X_bits: np.ndarray, rotate: bool = True, K: int | None = None,
                       act: str = "none", qmax: float = 127.0):
    """quantize_and_rotate_rowwise (rotate=True) or quantize_int8_rowwise
    (rotate=False) on BF16 rows, optionally after an input activation
    (``act`` in ACTS). ``X_bits`` is uint16 [M, ldx]; the first K columns of
    each row are used (K defaults to ldx)."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, ld = X_bits.shape
    K = ld if K is None else K
    Qx = np.empty((M, K), np.int8)
    s_x = np.empty(M, np.float32)
    rc = lib().oracle_quantize_rows_bf16_q(_ptr(X_bits, ctypes.c_uint16), M, K, ld, int(rotate),
                                           ACTS[act], float(qmax), _ptr(Qx, ctypes.c_int8),
                                           _ptr(s_x, ctypes.c_float))
    if rc:
        raise ValueError(f"oracle_quantize_rows_bf16 failed ({rc}): K={K} must be a multiple of 256")
    return Qx, s_x


def rotate_quant_weight(W) -> tuple[np.ndarray, np.ndarray]:
    """Offline weight preparation: ConvRot256 along K, then per-output-row INT8."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Qw = np.empty((N, K), np.int8)
    s_w = np.empty(N, np.float32)
    rc = lib().oracle_rotate_quant_weight(_ptr(W, ctypes.c_float), N, K, _ptr(Qw, ctypes.c_int8),
                                          _ptr(s_w, ctypes.c_float))
    if rc:
        raise ValueError(f"oracle_rotate_quant_weight failed ({rc})")
    return Qw, s_w


def rotate_quant_weight_int4(W) -> tuple[np.ndarray, np.ndarray]:
    """convrot_w4a4_linear's weight preparation: ConvRot256, per-row signed INT4
    (s = absmax / 7), two codes per byte (element 2j in the low nibble).
    Returns (Qw4 uint8 [N, K/2], s_w fp32 [N])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Qw4 = np.empty((N, K // 2), np.uint8)
    s_w = np.empty(N, np.float32)
    rc = lib().oracle_rotate_quant_weight_int4(_ptr(W, ctypes.c_float), N, K,
                                               _ptr(Qw4, ctypes.c_uint8), _ptr(s_w, ctypes.c_float))
    if rc:
        raise ValueError(f"oracle_rotate_quant_weight_int4 failed ({rc})")
    return Qw4, s_w


def unpack_int4(Q4: np.ndarray) -> np.ndarray:
    """Packed INT4 [rows, K/2] -> int8 codes [rows, K]."""
    Q4 = np.ascontiguousarray(Q4, dtype=np.uint8)
    rows, half = Q4.shape
    Q8 = np.empty((rows, 2 * half), np.int8)
    lib().oracle_unpack_int4(_ptr(Q4, ctypes.c_uint8), rows, 2 * half, _ptr(Q8, ctypes.c_int8))
    return Q8


def convrot_w4a4_linear(X_bits, Qw4, s_w, bias_bits=None):
    """convrot_w4a4_linear: ConvRot256 + per-row signed INT4 codes of X (in int8
    storage), the packed INT4 weights unpacked to int8, INT32 GEMM, the same
    epilogue as int8_linear. Returns (Y bits, Qx, s_x, acc)."""
    Qx, s_x = quantize_rows_bf16(X_bits, rotate=True, qmax=7.0)
    acc = gemm_i32(Qx, unpack_int4(Qw4))
    return epilogue(acc, s_x, s_w, bias_bits), Qx, s_x, acc


def dequantize_int8(Q, s, per_row: bool = True):
    """dequantize_int8_simple(_dtype): returns (fp32 [rows, K], bf16 bits [rows, K])."""
    Q = np.ascontiguousarray(Q, dtype=np.int8)
    s = np.ascontiguousarray(np.atleast_1d(s), dtype=np.float32)
    rows, K = Q.shape
    Yf = np.empty((rows, K), np.float32)
    Yb = np.empty((rows, K), np.uint16)
    lib().oracle_dequantize_int8(_ptr(Q, ctypes.c_int8), _ptr(s, ctypes.c_float), rows, K,
                                 int(per_row), _ptr(Yf, ctypes.c_float), _ptr(Yb, ctypes.c_uint16))
    return Yf, Yb


def quantize_int8_tensorwise(X_bits):
    """quantize_int8_tensorwise on BF16 X: returns (Q int8 [M, K], s fp32 scalar)."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    Q = np.empty((M, K), np.int8)
    s = np.empty(1, np.float32)
    lib().oracle_quantize_int8_tensorwise(_ptr(X_bits, ctypes.c_uint16), M, K, K,
                                          _ptr(Q, ctypes.c_int8), _ptr(s, ctypes.c_float))
    return Q, s[0]


def gemm_i32(Qx: np.ndarray, Qw: np.ndarray) -> np.ndarray:
    Qx = np.ascontiguousarray(Qx, dtype=np.int8)
    Qw = np.ascontiguousarray(Qw, dtype=np.int8)
    M, K = Qx.shape
    N, K2 = Qw.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    lib().oracle_gemm_i32(_ptr(Qx, ctypes.c_int8), _ptr(Qw, ctypes.c_int8), M, N, K,
                          _ptr(acc, ctypes.c_int32))
    return acc


def epilogue(acc, s_x, s_w, bias_bits=None) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    M, N = acc.shape
    Y = np.empty((M, N), np.uint16)
    bp = None
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        bp = _ptr(bias_bits, ctypes.c_uint16)
    lib().oracle_epilogue(_ptr(acc, ctypes.c_int32), _ptr(s_x, ctypes.c_float),
                          _ptr(s_w, ctypes.c_float), bp, M, N, _ptr(Y, ctypes.c_uint16))
    return Y


def linear_rows(Qx, s_x, Qw, s_w, bias_bits, rows) -> np.ndarray:
    """Output rows ``rows`` of the linear, each computed on its own."""
    Qx = np.ascontiguousarray(Qx, dtype=np.int8)
    Qw = np.ascontiguousarray(Qw, dtype=np.int8)
    s_x = np.ascontiguousarray(s_x, dtype=np.float32)
    s_w = np.ascontiguousarray(s_w, dtype=np.float32)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    N, K = Qw.shape
    Y = np.empty((rows.size, N), np.uint16)
    bp = None
    if bias_bits is not None:
        bias_bits = np.ascontiguousarray(bias_bits, dtype=np.uint16)
        bp = _ptr(bias_bits, ctypes.c_uint16)
    lib().oracle_linear_rows(_ptr(Qx, ctypes.c_int8), _ptr(s_x, ctypes.c_float),
                             _ptr(Qw, ctypes.c_int8), _ptr(s_w, ctypes.c_float), bp, N, K,
                             _ptr(rows, ctypes.c_int64), rows.size, _ptr(Y, ctypes.c_uint16))
    return Y


def int8_linear(X_bits, Qw, s_w, bias_bits=None, act: str = "none"):
    """The whole forward: quantize_and_rotate_rowwise on X (after the input
    activation ``act``), INT32 GEMM, epilogue. Returns (Y bits [M,N], Qx, s_x, acc)."""
    Qx, s_x = quantize_rows_bf16(X_bits, rotate=True, act=act)
    acc = gemm_i32(Qx, Qw)
    return epilogue(acc, s_x, s_w, bias_bits), Qx, s_x, acc


# --------------------------------------------------------- input RMSNorm

def rmsnorm_rows(X_bits, residual_bits=None, g_bits=None, eps: float = 1e-6,
                 with_alt: bool = False):
    """The input RMSNorm with an optional residual (the C oracle's reading:
    h = bf16(x + r), y = the bf16 value nearest to h g / sqrt(mean(h^2) + eps)).
    Returns (Y bits [M, K], h bits), and with ``with_alt`` also Yalt: the
    other bf16 neighbour where the exact value lies within 2^-34 (relative)
    of a rounding midpoint, Y elsewhere (both then count as correct)."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    Y = np.empty((M, K), np.uint16)
    H = np.empty((M, K), np.uint16)
    Ya = np.empty((M, K), np.uint16)
    rp = gp = None
    ldr = K
    if residual_bits is not None:
        residual_bits = np.ascontiguousarray(residual_bits, dtype=np.uint16)
        assert residual_bits.shape == (M, K)
        rp = _ptr(residual_bits, ctypes.c_uint16)
    if g_bits is not None:
        g_bits = np.ascontiguousarray(g_bits, dtype=np.uint16)
        assert g_bits.shape == (K,)
        gp = _ptr(g_bits, ctypes.c_uint16)
    rc = lib().oracle_rmsnorm_rows(_ptr(X_bits, ctypes.c_uint16), K, rp, ldr, gp, float(eps), M,
                                   K, _ptr(Y, ctypes.c_uint16), _ptr(H, ctypes.c_uint16),
                                   _ptr(Ya, ctypes.c_uint16))
    if rc != 0:
        raise ValueError(f"oracle_rmsnorm_rows failed ({rc}); K must be a multiple of 256")
    return (Y, H, Ya) if with_alt else (Y, H)


def int8_linear_norm(X_bits, Qw, s_w, bias_bits=None, residual_bits=None, g_bits=None,
                     eps: float = 1e-6):
    """int8_linear after the input RMSNorm (and residual): the normalised bf16
    rows go through quantize_and_rotate_rowwise, the INT32 GEMM and the
    epilogue. Returns (Y bits [M, N], h bits, Qx, s_x)."""
    Yn, H = rmsnorm_rows(X_bits, residual_bits, g_bits, eps)
    Qx, s_x = quantize_rows_bf16(Yn, rotate=True)
    acc = gemm_i32(Qx, Qw)
    return epilogue(acc, s_x, s_w, bias_bits), H, Qx, s_x


# ----------------------------------------------------------------- NVFP4


def e2m1_to_f32(codes) -> np.ndarray:
    L = lib()
    c = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([L.oracle_e2m1_to_f32(int(x)) for x in c], dtype=np.float32)


def f32_to_e2m1(v) -> np.ndarray:
    L = lib()
    x = np.asarray(v, dtype=np.float32).ravel()
    return np.array([L.oracle_f32_to_e2m1_rne(float(t)) for t in x], dtype=np.uint8)


def e4m3_to_f32(codes) -> np.ndarray:
    L = lib()
    c = np.asarray(codes, dtype=np.uint8).ravel()
    return np.array([L.oracle_e4m3_to_f32(int(x)) for x in c], dtype=np.float32)


def f32_to_e4m3(v) -> np.ndarray:
    L = lib()
    x = np.asarray(v, dtype=np.float32).ravel()
    return np.array([L.oracle_f32_to_e4m3_rne(float(t)) for t in x], dtype=np.uint8)


def nvfp4_sf_offset(r: int, c: int, C: int) -> int:
    return int(lib().oracle_nvfp4_sf_offset(r, c, C))


def nvfp4_sf_bytes(R: int, K: int) -> int:
    return int(lib().oracle_nvfp4_sf_bytes(R, K))


def _nvfp4_out(R, K):
    return (np.zeros((R, K // 2), dtype=np.uint8), np.zeros(nvfp4_sf_bytes(R, K), dtype=np.uint8),
            np.zeros(1, dtype=np.float32))


def quantize_rotate_nvfp4(X_bits: np.ndarray):
    """ConvRot NVFP4 of bf16 rows: (codes [M, K/2], blocked scales, s_t)."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    Q, S, st = _nvfp4_out(M, K)
    rc = lib().oracle_quantize_rotate_nvfp4_bf16(_ptr(X_bits, ctypes.c_uint16), M, K, K,
                                                  _ptr(Q, ctypes.c_uint8), _ptr(S, ctypes.c_uint8),
                                                  _ptr(st, ctypes.c_float))
    assert rc == 0, rc
    return Q, S, float(st[0])


def rotate_quant_weight_nvfp4(W):
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    Q, S, st = _nvfp4_out(N, K)
    rc = lib().oracle_rotate_quant_weight_nvfp4(_ptr(W, ctypes.c_float), N, K,
                                                _ptr(Q, ctypes.c_uint8), _ptr(S, ctypes.c_uint8),
                                                _ptr(st, ctypes.c_float))
    assert rc == 0, rc
    return Q, S, float(st[0])


def dequantize_nvfp4(Q, S, s_t: float, hi_first: bool = False) -> np.ndarray:
    Q = np.ascontiguousarray(Q, dtype=np.uint8)
    S = np.ascontiguousarray(S, dtype=np.uint8)
    R, K2 = Q.shape
    out = np.zeros((R, 2 * K2), dtype=np.float32)
    lib().oracle_dequantize_nvfp4(_ptr(Q, ctypes.c_uint8), _ptr(S, ctypes.c_uint8), float(s_t),
                                  R, 2 * K2, int(bool(hi_first)), _ptr(out, ctypes.c_float))
    return out


def nvfp4_linear_rows(Qa, Sa, s_ta, Qw, Sw, s_tw, bias_bits=None, rows=None):
    """Rows of Y = bf16(float(sum) * s_ta * s_tw + bias); also sum |term| * alpha."""
    Qa = np.ascontiguousarray(Qa, dtype=np.uint8)
    Qw = np.ascontiguousarray(Qw, dtype=np.uint8)
    Sa = np.ascontiguousarray(Sa, dtype=np.uint8)
    Sw = np.ascontiguousarray(Sw, dtype=np.uint8)
    M, K2 = Qa.shape
    N = Qw.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    Y = np.zeros((len(rows), N), dtype=np.uint16)
    mag = np.zeros((len(rows), N), dtype=np.float64)
    bb = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    lib().oracle_nvfp4_linear_rows(_ptr(Qa, ctypes.c_uint8), _ptr(Sa, ctypes.c_uint8), float(s_ta), M,
                                   _ptr(Qw, ctypes.c_uint8), _ptr(Sw, ctypes.c_uint8), float(s_tw), N,
                                   None if bb is None else _ptr(bb, ctypes.c_uint16), 2 * K2,
                                   _ptr(rows, ctypes.c_int64), len(rows),
                                   _ptr(Y, ctypes.c_uint16), _ptr(mag, ctypes.c_double))
    return Y, mag
