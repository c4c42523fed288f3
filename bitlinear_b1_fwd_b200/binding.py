"""ctypes binding of ``libbitlinear.so`` (the C ABI in ``include/bitlinear.h``).

Argument marshalling only: every function here turns torch tensors into
pointers, sizes and a stream handle and calls the library entry point of the
same name.  All computation runs in the library's CUDA kernels; there is no
CPU path.  If the library has not been built the first call raises.
"""
from __future__ import annotations

import ctypes as C
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbitlinear.so")

BL_OK, BL_ERR_INVALID_VALUE, BL_ERR_UNSUPPORTED, BL_ERR_MISALIGNED = 0, 1, 2, 3
BL_ERR_WORKSPACE_TOO_SMALL, BL_ERR_CUDA, BL_ERR_DEVICE_TIMEOUT, BL_ERR_BAD_CODE = 4, 5, 6, 7
BL_ERR_SCRATCH_LIMIT = 8
BL_F32, BL_BF16, BL_I8, BL_I32 = 0, 1, 2, 3
BL_PACK_I2, BL_PACK_T5, BL_PACK_B1 = 0, 1, 2
BL_WS_HEADER_BYTES = 256

# (name, restype, argtypes) of every exported entry point
_P, _I64, _I, _F, _SZ = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t
SIGNATURES = {
    "bitlinear_packed_row_bytes": (_I64, [_I64, _I]),
    "bitlinear_quantize_weights_workspace_bytes": (_SZ, [_I64, _I64]),
    "bitlinear_forward_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I, _I]),
    "bitlinear_workspace_init": (_I, [_P, _SZ, _P]),
    "bitlinear_quantize_weights": (_I, [_P, _I, _I64, _I64, _F, _I, _P, _P, _P, _P, _SZ, _P]),
    "bitlinear_absmean": (_I, [_P, _I, _I64, _I64, _P, _P, _SZ, _P]),
    "bitlinear_absmean_noalloc": (_I, [_P, _I, _I64, _I64, _P, _P]),
    "bitlinear_ternarize_pack": (_I, [_P, _I, _I64, _I64, _P, _F, _I, _P, _P, _P]),
    "bitlinear_pack": (_I, [_P, _I64, _I64, _I, _P, _P, _SZ, _P]),
    "bitlinear_binarize_weights_workspace_bytes": (_SZ, [_I64, _I64]),
    "bitlinear_binarize_weights": (_I, [_P, _I, _I64, _I64, _P, _P, _P, _P, _P, _SZ, _P]),
    "bitlinear_quantize_acts": (_I, [_P, _I, _I64, _I64, _P, _P, _P]),
    "bitlinear_layernorm_quantize_acts": (_I, [_P, _I, _P, _P, _F, _I64, _I64, _P, _P, _P, _P]),
    "bitlinear_forward": (_I, [_P, _I, _P, _I64, _I64, _P, _I, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_forward_grouped_workspace_bytes": (_SZ, [_I64, _I64, _P, _I64, _I, _I]),
    "bitlinear_forward_grouped": (_I, [_P, _I, _P, _I64, _P, _I64, _P, _I, _P, _I64, _P, _I, _P, _SZ, _P]),
    "bitlinear_backward_dx_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I]),
    "bitlinear_backward_dx": (_I, [_P, _I, _P, _I64, _I64, _P, _I, _I64, _P, _P, _SZ, _P]),
    "bitlinear_backward_dw": (_I, [_P, _I, _P, _P, _P, _I64, _I64, _I64, _P, _P]),
    "bitlinear_selftest_wait_timeout": (_I, [_P, _SZ, _P]),
    "bitlinear_device_status": (_I, [_P, _P]),
    "bitlinear_status_string": (C.c_char_p, [_I]),
    "bitlinear_version": (_I, []),
}

_lib = None
_lock = threading.Lock()


class BitLinearError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> C.CDLL:
    """Load the CUDA library (raises if it is missing: there is no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it first "
                                   "(python -m bitlinear_b1_fwd_b200.build)")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().bitlinear_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != BL_OK:
        raise BitLinearError(status, where)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


_DT = {torch.float32: BL_F32, torch.bfloat16: BL_BF16, torch.int8: BL_I8, torch.int32: BL_I32}


def dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


# --- size queries -----------------------------------------------------------

def bitlinear_packed_row_bytes(K: int, fmt: int) -> int:
    return int(lib().bitlinear_packed_row_bytes(K, fmt))


def bitlinear_quantize_weights_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_quantize_weights_workspace_bytes(N, K))


def bitlinear_binarize_weights_workspace_bytes(N: int, K: int) -> int:
    return int(lib().bitlinear_binarize_weights_workspace_bytes(N, K))


def bitlinear_forward_workspace_bytes(M: int, N: int, K: int, fmt: int, xdt: int) -> int:
    return int(lib().bitlinear_forward_workspace_bytes(M, N, K, fmt, xdt))


def _rows_array(group_rows):
    rows = [int(r) for r in group_rows]
    return (C.c_int64 * len(rows))(*rows), len(rows)


def bitlinear_forward_grouped_workspace_bytes(M: int, group_rows, K: int, fmt: int, xdt: int) -> int:
    arr, n = _rows_array(group_rows)
    return int(lib().bitlinear_forward_grouped_workspace_bytes(M, n, arr, K, fmt, xdt))


# --- entry points -------------------------------------------------------------

def bitlinear_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib().bitlinear_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_workspace_init")


def bitlinear_quantize_weights(W, eps, fmt, packed, codes, gamma, ws, stream=None) -> None:
    _contig(W, packed, codes, gamma, ws)
    N, K = W.shape
    _check(lib().bitlinear_quantize_weights(_ptr(W), dtype_code(W), N, K, float(eps), fmt, _ptr(packed),
                                            _ptr(codes), _ptr(gamma), _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_quantize_weights")


def bitlinear_absmean(W, gamma, ws, stream=None) -> None:
    _contig(W, gamma, ws)
    N, K = W.shape
    _check(lib().bitlinear_absmean(_ptr(W), dtype_code(W), N, K, _ptr(gamma), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "bitlinear_absmean")


def bitlinear_absmean_noalloc(W, gamma, stream=None) -> None:
    """gamma of W without a workspace (the library's fixed device scratch)."""
    _contig(W, gamma)
    N, K = W.shape
    _check(lib().bitlinear_absmean_noalloc(_ptr(W), dtype_code(W), N, K, _ptr(gamma), _stream(stream)),
           "bitlinear_absmean_noalloc")


def bitlinear_ternarize_pack(W, gamma, eps, fmt, packed, codes, stream=None) -> None:
    _contig(W, packed, codes, gamma)
    N, K = W.shape
    _check(lib().bitlinear_ternarize_pack(_ptr(W), dtype_code(W), N, K, _ptr(gamma), float(eps), fmt,
                                          _ptr(packed), _ptr(codes), _stream(stream)),
           "bitlinear_ternarize_pack")


def bitlinear_pack(codes, fmt, packed, ws, stream=None) -> None:
    _contig(codes, packed, ws)
    N, K = codes.shape
    _check(lib().bitlinear_pack(_ptr(codes), N, K, fmt, _ptr(packed), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "bitlinear_pack")


def bitlinear_quantize_acts(x, xq, scale, stream=None) -> None:
    _contig(x, xq, scale)
    M, K = x.shape
    _check(lib().bitlinear_quantize_acts(_ptr(x), dtype_code(x), M, K, _ptr(xq), _ptr(scale),
                                         _stream(stream)), "bitlinear_quantize_acts")


def bitlinear_layernorm_quantize_acts(x, ln_w, ln_b, eps, xq, scale, y=None, stream=None) -> None:
    """LayerNorm of each token (y: optional bf16 output), then per-token INT8."""
    _contig(x, ln_w, ln_b, xq, scale, y)
    M, K = x.shape
    _check(lib().bitlinear_layernorm_quantize_acts(_ptr(x), dtype_code(x), _ptr(ln_w), _ptr(ln_b), float(eps), M, K,
                                                   _ptr(y), _ptr(xq), _ptr(scale), _stream(stream)),
           "bitlinear_layernorm_quantize_acts")


def bitlinear_binarize_weights(W, packed, codes, beta, alpha, ws, stream=None) -> None:
    _contig(W, packed, codes, beta, alpha, ws)
    N, K = W.shape
    _check(lib().bitlinear_binarize_weights(_ptr(W), dtype_code(W), N, K, _ptr(packed), _ptr(codes), _ptr(beta),
                                            _ptr(alpha), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_binarize_weights")


def bitlinear_forward(packed, fmt, gamma, N, K, x, scale, y, ws, stream=None) -> None:
    _contig(packed, gamma, x, scale, y, ws)
    M = x.shape[0]
    _check(lib().bitlinear_forward(_ptr(packed), fmt, _ptr(gamma), N, K, _ptr(x), dtype_code(x),
                                   _ptr(scale), M, _ptr(y), dtype_code(y), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_forward")


def bitlinear_forward_grouped(packed, fmt, gammas, group_rows, K, x, scale, y, ws, stream=None) -> None:
    _contig(packed, gammas, x, scale, y, ws)
    M = x.shape[0]
    arr, n = _rows_array(group_rows)
    _check(lib().bitlinear_forward_grouped(_ptr(packed), fmt, _ptr(gammas), n, arr, K, _ptr(x), dtype_code(x),
                                           _ptr(scale), M, _ptr(y), dtype_code(y), _ptr(ws),
                                           ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_forward_grouped")


def bitlinear_backward_dx_workspace_bytes(M: int, N: int, K: int, fmt: int) -> int:
    return int(lib().bitlinear_backward_dx_workspace_bytes(M, N, K, fmt))


def bitlinear_backward_dx(packed, fmt, gamma, N, K, dy, dx, ws, stream=None) -> None:
    _contig(packed, gamma, dy, dx, ws)
    M = dy.shape[0]
    _check(lib().bitlinear_backward_dx(_ptr(packed), fmt, _ptr(gamma), N, K, _ptr(dy), dtype_code(dy), M, _ptr(dx),
                                       _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_backward_dx")


def bitlinear_backward_dw(dy, xq, scale, gamma, dw, stream=None) -> None:
    _contig(dy, xq, scale, gamma, dw)
    M, N = dy.shape
    K = xq.shape[1]
    _check(lib().bitlinear_backward_dw(_ptr(dy), dtype_code(dy), _ptr(xq), _ptr(scale), _ptr(gamma), M, N, K,
                                       _ptr(dw), _stream(stream)),
           "bitlinear_backward_dw")


def bitlinear_device_status(ws, stream=None) -> int:
    """Synchronize and return (and clear) the workspace's device status."""
    return int(lib().bitlinear_device_status(_ptr(ws), _stream(stream)))


def bitlinear_selftest_wait_timeout(ws, stream=None) -> None:
    _check(lib().bitlinear_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "bitlinear_selftest_wait_timeout")


def bitlinear_version() -> int:
    return int(lib().bitlinear_version())


# --- convenience layer (allocation through torch, then the calls above) ----------

class BitLinear:
    """A BitLinear layer holding packed ternary weights and gamma on the GPU.

    ``BitLinear.from_weight(W)`` runs steps 1-3 once; calling the layer on
    activations x [M, K] (fp32 / bf16) runs steps 4-6 and returns y [M, N].
    """

    def __init__(self, packed, gamma, N, K, fmt=BL_PACK_I2):
        self.packed, self.gamma, self.N, self.K, self.fmt = packed, gamma, N, K, fmt
        self._ws = None

    @classmethod
    def from_weight(cls, W: torch.Tensor, fmt: int = BL_PACK_I2, eps: float = 1e-5, stream=None):
        N, K = W.shape
        dev = W.device
        packed = torch.empty((N, bitlinear_packed_row_bytes(K, fmt)), dtype=torch.uint8, device=dev)
        gamma = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.zeros(bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=dev)
        bitlinear_quantize_weights(W, eps, fmt, packed, None, gamma, ws, stream)
        return cls(packed, gamma, N, K, fmt)

    def workspace(self, M: int, xdt: int) -> torch.Tensor:
        need = bitlinear_forward_workspace_bytes(M, self.N, self.K, self.fmt, xdt)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=self.packed.device)
        return self._ws

    def __call__(self, x: torch.Tensor, out_dtype=torch.bfloat16, stream=None):
        M = x.shape[0]
        y = torch.empty((M, self.N), dtype=out_dtype, device=x.device)
        scale = torch.empty(M, dtype=torch.float32, device=x.device)
        ws = self.workspace(M, dtype_code(x))
        bitlinear_forward(self.packed, self.fmt, self.gamma, self.N, self.K, x, scale, y, ws, stream)
        return y
