"""CPU oracle for the BitNet b1.58 BitLinear forward pass (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (``bitlinear_b1_fwd_b200``) never imports it and shares no code with it.

The arithmetic lives in ``bitlinear_oracle.c`` (plain single-threaded C, no
fast-math); this module only builds it with gcc, loads it with ctypes and
marshals numpy arrays.  bf16 arrays travel as ``numpy.uint16`` bit patterns.

Every function is pinned by the CPU tests in ``tests/test_oracle_*.py`` (worked
examples of the pages, closed forms, exact sums, brute force); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitlinear_oracle.c")
LIB_PATH = os.path.join(HERE, "liboracle.so")
# A test of the pins themselves builds copies of the oracle with one planted
# mistake each and points this variable at such a copy (never set otherwise).
_PLANTED = os.environ.get("BL_ORACLE_PLANTED_LIB")
if _PLANTED:
    LIB_PATH = _PLANTED

F32, BF16, I8, I32 = 0, 1, 2, 3
PACK_I2, PACK_T5, PACK_B1 = 0, 1, 2

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE arithmetic: no fast-math, no FMA)."""
    if _PLANTED:
        return LIB_PATH  # a prebuilt copy with a planted mistake
    if (not force and os.path.exists(LIB_PATH)
            and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC)):
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math",
           "-ffp-contract=off", "-fno-strict-aliasing", "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib() -> C.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(LIB_PATH)
            p, i64, f, d, i = C.c_void_p, C.c_int64, C.c_float, C.c_double, C.c_int
            L.orc_absmean_sum.argtypes = [p, i, i64, i64]
            L.orc_absmean_sum.restype = d
            L.orc_signed_sum.argtypes = [p, i, i64, i64]
            L.orc_signed_sum.restype = d
            L.orc_binarize_weights.argtypes = [p, i, i64, i64, p, p, p]
            L.orc_binarize_weights.restype = None
            L.orc_backward_dx.argtypes = [p, i64, i64, p, i, i64, f, p]
            L.orc_backward_dx.restype = None
            L.orc_backward_dw.argtypes = [p, i, p, p, f, i64, i64, i64, p]
            L.orc_backward_dw.restype = None
            L.orc_gamma.argtypes = [p, i, i64, i64]
            L.orc_gamma.restype = f
            L.orc_ternarize.argtypes = [p, i, i64, i64, f, f, p]
            L.orc_ternarize.restype = None
            L.orc_packed_row_bytes.argtypes = [i64, i]
            L.orc_packed_row_bytes.restype = i64
            L.orc_pack.argtypes = [p, i64, i64, i, p]
            L.orc_pack.restype = i
            L.orc_unpack.argtypes = [p, i64, i64, i, p]
            L.orc_unpack.restype = i
            L.orc_act_quant.argtypes = [p, i, i64, i64, p, p]
            L.orc_act_quant.restype = None
            L.orc_matmul_i32.argtypes = [p, p, i64, i64, i64, p]
            L.orc_matmul_i32.restype = None
            L.orc_dequant.argtypes = [p, f, p, i64, i64, p, i]
            L.orc_dequant.restype = None
            L.orc_forward.argtypes = [p, i, f, i64, i64, p, i, p, i64, p, i]
            L.orc_forward.restype = i
            L.orc_onebit.argtypes = [p, i64, p, p, p]
            L.orc_onebit.restype = None
            L.orc_layernorm.argtypes = [p, i, p, p, f, i64, i64, p]
            L.orc_layernorm.restype = None
            L.orc_layernorm_quant.argtypes = [p, i, p, p, f, i64, i64, p, p, p]
            L.orc_layernorm_quant.restype = None
            L.orc_f32_to_bf16.argtypes = [f]
            L.orc_f32_to_bf16.restype = C.c_uint16
            L.orc_bf16_to_f32.argtypes = [C.c_uint16]
            L.orc_bf16_to_f32.restype = f
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"float input must be float32 or bf16 bits (uint16), got {a.dtype}")


def _threads() -> int:
    return max(1, os.cpu_count() or 1)


# --- step 1 -----------------------------------------------------------------

def absmean_sum(W: np.ndarray) -> float:
    """fp64 sum of |w| over W [N, K] in the fixed reduction order."""
    N, K = W.shape
    return lib().orc_absmean_sum(_ptr(W), _dt(W), N, K)


def gamma(W: np.ndarray) -> np.float32:
    """gamma = mean |W| (fp64 in the fixed order, rounded to fp32)."""
    N, K = W.shape
    return np.float32(lib().orc_gamma(_ptr(W), _dt(W), N, K))


# --- step 2 -----------------------------------------------------------------

def ternarize(W: np.ndarray, g: float, eps: float = 1e-5, parallel: bool = False) -> np.ndarray:
    N, K = W.shape
    codes = np.empty((N, K), np.int8)
    L = lib()
    if not parallel or N < 2:
        L.orc_ternarize(_ptr(W), _dt(W), N, K, float(g), float(eps), _ptr(codes))
        return codes
    rows = np.array_split(np.arange(N), _threads())

    def run(r):
        if len(r) == 0:
            return
        a, b = int(r[0]), int(r[-1]) + 1
        L.orc_ternarize(_ptr(W) + a * K * W.itemsize, _dt(W), b - a, K, float(g),
                        float(eps), _ptr(codes) + a * K)
    with ThreadPoolExecutor(len(rows)) as ex:
        list(ex.map(run, rows))
    return codes


# --- step 3 -----------------------------------------------------------------

def packed_row_bytes(K: int, fmt: int) -> int:
    return int(lib().orc_packed_row_bytes(K, fmt))


def pack(codes: np.ndarray, fmt: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    N, K = codes.shape
    out = np.empty((N, packed_row_bytes(K, fmt)), np.uint8)
    rc = lib().orc_pack(_ptr(codes), N, K, fmt, _ptr(out))
    if rc != 0:
        raise ValueError("code outside {-1, 0, 1} ({-1, 1} for the 1-bit format)")
    return out


def unpack(packed: np.ndarray, N: int, K: int, fmt: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    assert packed.shape == (N, packed_row_bytes(K, fmt))
    codes = np.empty((N, K), np.int8)
    rc = lib().orc_unpack(_ptr(packed), N, K, fmt, _ptr(codes))
    if rc == -1:
        raise ValueError("invalid packed code")
    if rc == -2:
        raise ValueError("padding digit is not weight 0")
    return codes


# --- step 4 -----------------------------------------------------------------

def act_quant(x: np.ndarray):
    """Per-token absmax INT8: returns (x_q int8 [M, K], scale fp32 [M])."""
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    s = np.empty((M,), np.float32)
    lib().orc_act_quant(_ptr(x), _dt(x), M, K, _ptr(xq), _ptr(s))
    return xq, s


# --- step 5 -----------------------------------------------------------------

def matmul_i32(codes: np.ndarray, xq: np.ndarray, parallel: bool = False) -> np.ndarray:
    """acc [M, N] = x_q [M, K] . codes [N, K]^T in int32."""
    N, K = codes.shape
    M, K2 = xq.shape
    assert K == K2
    L = lib()
    if not parallel:
        acc = np.empty((M, N), np.int32)
        L.orc_matmul_i32(_ptr(codes), _ptr(xq), M, N, K, _ptr(acc))
        return acc
    # split the output columns (rows of codes) across threads
    parts = [r for r in np.array_split(np.arange(N), _threads()) if len(r)]
    outs = [np.empty((M, len(r)), np.int32) for r in parts]

    def run(i):
        a = int(parts[i][0])
        L.orc_matmul_i32(_ptr(codes) + a * K, _ptr(xq), M, len(parts[i]), K, _ptr(outs[i]))
    with ThreadPoolExecutor(len(parts)) as ex:
        list(ex.map(run, range(len(parts))))
    return np.ascontiguousarray(np.concatenate(outs, axis=1))


# --- step 6 -----------------------------------------------------------------

def dequant(acc: np.ndarray, g: float, scale: np.ndarray, ydt: int = F32) -> np.ndarray:
    acc = np.ascontiguousarray(acc, dtype=np.int32)
    M, N = acc.shape
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    dt = {F32: np.float32, BF16: np.uint16, I32: np.int32}[ydt]
    y = np.empty((M, N), dt)
    lib().orc_dequant(_ptr(acc), float(g), _ptr(scale), M, N, _ptr(y), ydt)
    return y


def forward(packed: np.ndarray, fmt: int, g: float, N: int, K: int, x: np.ndarray,
            ydt: int = F32, scale: np.ndarray | None = None):
    """Whole forward.  x float32 / bf16-bits [M, K] is quantized inside; x int8
    is taken as x_q with the given per-token ``scale``.  Returns (y, scale)."""
    M = x.shape[0]
    xdt = I8 if x.dtype == np.int8 else _dt(x)
    if xdt == I8:
        assert scale is not None
        s = np.ascontiguousarray(scale, dtype=np.float32)
    else:
        s = np.empty((M,), np.float32)
    dt = {F32: np.float32, BF16: np.uint16, I32: np.int32}[ydt]
    y = np.empty((M, N), dt)
    rc = lib().orc_forward(_ptr(np.ascontiguousarray(packed)), fmt, float(g), N, K,
                           _ptr(x), xdt, _ptr(s), M, _ptr(y), ydt)
    if rc != 0:
        raise ValueError(f"oracle forward failed ({rc})")
    return y, s


# --- 1-bit helper (the pages' five-weight comparison) ---------------------------

def onebit(w: np.ndarray):
    """1-bit BitNet weights: returns (signs int8, alpha, beta)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    b = np.empty(w.shape, np.int8)
    a = C.c_float()
    be = C.c_float()
    lib().orc_onebit(_ptr(w), w.size, _ptr(b), C.byref(a), C.byref(be))
    return b, np.float32(a.value), np.float32(be.value)


# --- 1-bit variant: alpha, beta and the {-1, +1} codes of a whole matrix ----------

def signed_sum(W: np.ndarray) -> float:
    """fp64 sum of w over W [N, K] in the fixed reduction order of step 1."""
    N, K = W.shape
    return lib().orc_signed_sum(_ptr(W), _dt(W), N, K)


def binarize_weights(W: np.ndarray):
    """1-bit weights of W [N, K]: returns (alpha, beta, codes int8 in {-1, +1})."""
    N, K = W.shape
    codes = np.empty((N, K), np.int8)
    a = C.c_float()
    b = C.c_float()
    lib().orc_binarize_weights(_ptr(W), _dt(W), N, K, C.byref(a), C.byref(b), _ptr(codes))
    return np.float32(a.value), np.float32(b.value), codes


# --- STE backward -------------------------------------------------------------------

def backward_dx(codes: np.ndarray, dy: np.ndarray, g: float, parallel: bool = False) -> np.ndarray:
    """dx [M, K] = gamma * dy [M, N] . W_q [N, K] (fp64 in the fixed chunk order, fp32 out)."""
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    dy = np.ascontiguousarray(dy)
    N, K = codes.shape
    M = dy.shape[0]
    assert dy.shape == (M, N)
    dx = np.empty((M, K), np.float32)
    L = lib()
    if not parallel or M < 2:
        L.orc_backward_dx(_ptr(codes), N, K, _ptr(dy), _dt(dy), M, float(g), _ptr(dx))
        return dx
    toks = [r for r in np.array_split(np.arange(M), _threads()) if len(r)]

    def run(r):
        a, b = int(r[0]), int(r[-1]) + 1
        L.orc_backward_dx(_ptr(codes), N, K, _ptr(dy) + a * N * dy.itemsize, _dt(dy), b - a, float(g),
                          _ptr(dx) + a * K * 4)
    with ThreadPoolExecutor(len(toks)) as ex:
        list(ex.map(run, toks))
    return dx


def backward_dw(dy: np.ndarray, xq: np.ndarray, scale: np.ndarray, g: float) -> np.ndarray:
    """dW [N, K] = gamma * dy^T . x_deq, x_deq = x_q * s / 127 (fp64 in token order, fp32 out)."""
    dy = np.ascontiguousarray(dy)
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    M, N = dy.shape
    K = xq.shape[1]
    assert xq.shape == (M, K) and scale.shape == (M,)
    dw = np.empty((N, K), np.float32)
    lib().orc_backward_dw(_ptr(dy), _dt(dy), _ptr(xq), _ptr(scale), float(g), M, N, K, _ptr(dw))
    return dw


def f32_to_bf16(v: float) -> int:
    return int(lib().orc_f32_to_bf16(float(v)))


def bf16_to_f32(h: int) -> np.float32:
    return np.float32(lib().orc_bf16_to_f32(int(h)))


# --- pre-norm: LayerNorm + per-token INT8 quantization ---------------------------

def layernorm(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm of each token (fixed-order fp64 mean and variance), bf16 bits out."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    g = np.ascontiguousarray(g, dtype=np.float32)
    b = np.ascontiguousarray(b, dtype=np.float32)
    y = np.empty((M, K), np.uint16)
    lib().orc_layernorm(_ptr(x), _dt(x), _ptr(g), _ptr(b), float(eps), M, K, _ptr(y))
    return y


def layernorm_quant(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float = 1e-5):
    """LayerNorm then per-token absmax INT8: returns (y bf16 bits, x_q, scale)."""
    x = np.ascontiguousarray(x)
    M, K = x.shape
    g = np.ascontiguousarray(g, dtype=np.float32)
    b = np.ascontiguousarray(b, dtype=np.float32)
    y = np.empty((M, K), np.uint16)
    xq = np.empty((M, K), np.int8)
    s = np.empty((M,), np.float32)
    lib().orc_layernorm_quant(_ptr(x), _dt(x), _ptr(g), _ptr(b), float(eps), M, K, _ptr(y), _ptr(xq), _ptr(s))
    return y, xq, s
