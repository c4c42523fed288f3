"""The C ABI on the CPU: the library builds and loads, exports every function
that include/bitlinear.h declares, and rejects bad arguments on the host
before any CUDA call (no compute runs here)."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bitlinear.h")


@pytest.fixture(scope="module")
def bl():
    from bitlinear_b1_fwd_b200 import build, binding
    build.build()
    return binding


def declared_functions():
    text = open(HEADER).read()
    names = re.findall(r"^(?:BL_API\s+)?(?:const\s+)?\w+\s*\*?\s*(bitlinear_\w+)\s*\(", text, flags=re.M)
    unmarked = re.findall(r"^(?!BL_API)(?:const\s+)?\w+\s*\*?\s*(bitlinear_\w+)\s*\(", text, flags=re.M)
    assert not unmarked, f"declared without BL_API (not exported): {unmarked}"
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("bitlinear_quantize_weights", "bitlinear_pack", "bitlinear_quantize_acts",
                     "bitlinear_forward"):
        assert required in names


def test_library_exports_every_declared_symbol(bl):
    L = bl.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) <= set(bl.SIGNATURES)
    assert bl.bitlinear_version() >= 100


def test_row_bytes_match_oracle(bl, orc):
    for K in (1, 4, 5, 63, 64, 65, 256, 3200, 8192, 8640, 28672, 1 << 20):
        for fmt in (0, 1, 2):
            assert bl.bitlinear_packed_row_bytes(K, fmt) == orc.packed_row_bytes(K, fmt)
    assert bl.bitlinear_packed_row_bytes(0, 0) == -1
    assert bl.bitlinear_packed_row_bytes(5, 7) == -1
    assert bl.bitlinear_packed_row_bytes((1 << 20) + 1, 0) == -1


def test_workspace_sizes(bl):
    assert bl.bitlinear_quantize_weights_workspace_bytes(512, 256) == 256 + 256   # 16 chunks
    assert bl.bitlinear_quantize_weights_workspace_bytes(8640, 3200) == 256 + 3375 * 8 + (256 - 3375 * 8 % 256)
    assert bl.bitlinear_quantize_weights_workspace_bytes(0, 5) == 0
    assert bl.bitlinear_forward_workspace_bytes(1, 8640, 3200, 0, 1) >= bl.BL_WS_HEADER_BYTES
    assert bl.bitlinear_forward_workspace_bytes(1, 8640, 0, 0, 1) == 0


def test_onebit_workspace_sizes(bl):
    # two fp64 partial sums per 8192-element chunk
    assert bl.bitlinear_binarize_weights_workspace_bytes(512, 256) == 256 + 256
    assert bl.bitlinear_binarize_weights_workspace_bytes(8640, 3200) == 256 + (2 * 3375 * 8 + 255) // 256 * 256
    assert bl.bitlinear_binarize_weights_workspace_bytes(0, 5) == 0
    # decode of 1-bit rows up to 4096 bytes needs only the header; longer rows a 2-bit copy
    assert bl.bitlinear_forward_workspace_bytes(1, 8192, 28672, 2, 1) == bl.BL_WS_HEADER_BYTES
    assert bl.bitlinear_forward_workspace_bytes(1, 300, 40000, 2, 1) == 256 + (300 * 10000 + 255) // 256 * 256
    # the tensor-core path transcodes 1-bit weights like base-3 ones
    assert bl.bitlinear_forward_workspace_bytes(64, 256, 1024, 2, 2) == bl.bitlinear_forward_workspace_bytes(64, 256, 1024, 1, 2)


def test_backward_workspace_sizes(bl):
    # header + fp64 partials [ceil(N / 64)][min(M, 2)][K], + a 2-bit copy for base 3 / 1-bit
    assert bl.bitlinear_backward_dx_workspace_bytes(1, 512, 256, 0) == 256 + 8 * 1 * 256 * 8
    assert bl.bitlinear_backward_dx_workspace_bytes(5, 777, 1000, 0) == 256 + (13 * 2 * 1000 * 8 + 255) // 256 * 256
    assert bl.bitlinear_backward_dx_workspace_bytes(1, 512, 256, 1) == 256 + 512 * 64 + 8 * 256 * 8
    assert bl.bitlinear_backward_dx_workspace_bytes(1, 0, 256, 0) == 0


def test_status_strings(bl):
    for s in range(8):
        assert bl.status_string(s).startswith("BL_")
    assert "unknown" in bl.status_string(99)


def test_host_validation_without_gpu(bl):
    """Each call returns its error code before launching anything."""
    L = bl.lib()
    p = C.c_void_p(1 << 20)            # an aligned, never-dereferenced address
    odd = C.c_void_p((1 << 20) + 4)    # 4-byte aligned only
    null = None
    # quantize_weights
    assert L.bitlinear_quantize_weights(null, 0, 4, 4, 1e-5, 0, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 2, 4, 4, 1e-5, 0, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 4, 4, 0.0, 0, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 4, 4, float("nan"), 0, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 4, 4, 1e-5, 3, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 4, 0, 1e-5, 0, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 0, 4, 1e-5, 0, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 4, (1 << 20) + 1, 1e-5, 0, p, null, p, p, 1 << 30, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 1 << 13, 1 << 20, 1e-5, 0, p, null, p, p, 1 << 30, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, 4, 4, 1e-5, 0, null, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(odd, 0, 4, 4, 1e-5, 0, p, null, p, p, 4096, null) == bl.BL_ERR_MISALIGNED
    assert L.bitlinear_quantize_weights(p, 0, 4, 4, 1e-5, 0, p, null, p, p, 100, null) == bl.BL_ERR_WORKSPACE_TOO_SMALL
    # the 1-bit format is not a ternary format
    assert L.bitlinear_quantize_weights(p, 0, 4, 4, 1e-5, 2, p, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_ternarize_pack(p, 0, 4, 4, p, 1e-5, 2, p, null, null) == bl.BL_ERR_INVALID_VALUE
    # binarize_weights
    assert L.bitlinear_binarize_weights(p, 0, 4, 4, null, null, p, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_binarize_weights(p, 0, 4, 4, p, null, null, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_binarize_weights(p, 2, 4, 4, p, null, p, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_binarize_weights(p, 0, 0, 4, p, null, p, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_binarize_weights(odd, 0, 4, 4, p, null, p, p, p, 4096, null) == bl.BL_ERR_MISALIGNED
    assert L.bitlinear_binarize_weights(p, 0, 4, 4, p, null, p, p, p, 100, null) == bl.BL_ERR_WORKSPACE_TOO_SMALL
    # ternarize_pack
    assert L.bitlinear_ternarize_pack(p, 0, 4, 4, null, 1e-5, 0, p, null, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_ternarize_pack(p, 0, 4, 4, p, -1.0, 0, p, null, null) == bl.BL_ERR_INVALID_VALUE
    # pack
    assert L.bitlinear_pack(p, 4, 4, 0, p, p, 10, null) == bl.BL_ERR_WORKSPACE_TOO_SMALL
    assert L.bitlinear_pack(null, 0, 4, 0, null, null, 0, null) == bl.BL_OK
    assert L.bitlinear_pack(odd, 4, 4, 0, p, p, 4096, null) == bl.BL_ERR_MISALIGNED
    assert L.bitlinear_pack(p, 4, 4, 3, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_pack(p, 0, 4, 0, p, p, 4096, null) == bl.BL_OK          # empty: nothing to do
    # quantize_acts
    assert L.bitlinear_quantize_acts(p, 2, 4, 4, p, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_acts(p, 1, 4, 0, p, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_acts(odd, 1, 4, 4, p, p, null) == bl.BL_ERR_MISALIGNED
    assert L.bitlinear_quantize_acts(p, 1, 0, 4, p, p, null) == bl.BL_OK
    # forward
    args = lambda **kw: [kw.get(k, v) for k, v in dict(
        packed=p, fmt=0, gamma=p, N=4, K=4, x=p, xdt=1, scale=p, M=1, y=p, ydt=1, ws=p,
        ws_bytes=4096, stream=null).items()]
    assert L.bitlinear_forward(*args(packed=null)) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(*args(fmt=5)) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(*args(xdt=3)) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(*args(ydt=2)) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(*args(M=-1)) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(*args(K=0)) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(*args(y=odd)) == bl.BL_ERR_MISALIGNED
    assert L.bitlinear_forward(*args(ws_bytes=8)) == bl.BL_ERR_WORKSPACE_TOO_SMALL
    assert L.bitlinear_forward(*args(M=0)) == bl.BL_OK
    assert L.bitlinear_forward(*args(N=0)) == bl.BL_OK
    assert L.bitlinear_forward(*args(M=0, x=null, y=null, scale=null, ws=null)) == bl.BL_OK
    # STE backward
    assert L.bitlinear_backward_dx(p, 0, p, 4, 4, p, 2, 1, p, p, 1 << 20, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dx(p, 5, p, 4, 4, p, 0, 1, p, p, 1 << 20, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dx(null, 0, p, 4, 4, p, 0, 1, p, p, 1 << 20, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dx(p, 0, p, 4, 4, odd, 0, 1, p, p, 1 << 20, null) == bl.BL_ERR_MISALIGNED
    assert L.bitlinear_backward_dx(p, 0, p, 4, 4, p, 0, 1, p, p, 8, null) == bl.BL_ERR_WORKSPACE_TOO_SMALL
    assert L.bitlinear_backward_dx(null, 0, null, 4, 4, null, 0, 0, null, null, 0, null) == bl.BL_OK
    assert L.bitlinear_backward_dw(p, 3, p, p, p, 1, 4, 4, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dw(p, 0, p, p, p, 1, 0, 4, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dw(p, 0, p, p, p, 1, 4, 4, null, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dw(p, 0, p, p, p, 1, 4, 4, odd, null) == bl.BL_ERR_MISALIGNED
    # workspace helpers
    assert L.bitlinear_workspace_init(null, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_device_status(null, null) == bl.BL_ERR_INVALID_VALUE


def test_size_limits_without_gpu(bl):
    """Rows and tokens stay below 2^31 (the kernels count them, and the work
    items of a row, in 32 bits): one past the limit is rejected on the host;
    at the limit the arguments pass every host check and the call reaches the
    CUDA runtime, which has no device here (BL_ERR_CUDA)."""
    L = bl.lib()
    p = C.c_void_p(1 << 20)
    null = None
    top, over = (1 << 31) - 1, 1 << 31
    big = 1 << 62
    # N at K = 1, where N K <= 2^32 alone would allow up to 2^32 rows
    assert L.bitlinear_pack(p, over, 1, 0, p, p, 4096, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_pack(p, top, 1, 0, p, p, 4096, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_quantize_weights(p, 0, over, 1, 1e-5, 0, p, null, p, p, big, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_weights(p, 0, top, 1, 1e-5, 0, p, null, p, p, big, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_binarize_weights(p, 0, over, 1, p, null, p, p, p, big, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dw(p, 1, p, p, p, 1, over, 1, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dw(p, 1, p, p, p, 1, top, 1, p, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_forward(p, 0, p, over, 1, p, 1, p, 1, p, 1, p, big, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward_workspace_bytes(1, over, 1, 0, 1) == 0
    assert L.bitlinear_quantize_weights_workspace_bytes(over, 1) == 0
    # M, tokens
    assert L.bitlinear_quantize_acts(p, 1, over, 16, p, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_quantize_acts(p, 1, top, 16, p, p, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_layernorm_quantize_acts(p, 1, p, p, 1e-5, over, 16, p, p, p, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(p, 0, p, 64, 16, p, 1, p, over, p, 1, p, big, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_forward(p, 0, p, 64, 16, p, 1, p, top, p, 1, p, big, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_forward_workspace_bytes(over, 64, 16, 0, 1) == 0
    assert L.bitlinear_forward_workspace_bytes(top, 64, 16, 0, 1) > top * 16
    assert L.bitlinear_backward_dx(p, 0, p, 64, 16, p, 1, over, p, p, big, null) == bl.BL_ERR_INVALID_VALUE
    assert L.bitlinear_backward_dx_workspace_bytes(over, 64, 16, 0) == 0
    assert L.bitlinear_backward_dw(p, 1, p, p, p, over, 64, 16, p, null) == bl.BL_ERR_INVALID_VALUE
    # typical shapes pass the host checks too
    assert L.bitlinear_forward(p, 0, p, 8640, 3200, p, 1, p, 1, p, 1, p, 1 << 30, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_forward(p, 0, p, 8640, 3200, p, 1, p, 4096, p, 1, p, 1 << 34, null) == bl.BL_ERR_CUDA
    assert L.bitlinear_backward_dx(p, 0, p, 8640, 3200, p, 1, 1, p, p, 1 << 30, null) == bl.BL_ERR_CUDA


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from bitlinear_b1_fwd_b200 import binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        binding.lib()


def _prototypes():
    """name -> (return type, [parameter types]) for every BL_API function."""
    text = re.sub(r"/\*.*?\*/", " ", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"BL_API\s+([^;]*?)\b(bitlinear_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.S):
        ret, name, params = " ".join(m.group(1).split()), m.group(2), " ".join(m.group(3).split())
        if params in ("", "void"):
            types = []
        else:
            types = [re.sub(r"\s*\b\w+$", "", p.strip()).strip() if not p.strip().endswith("*") else p.strip()
                     for p in params.split(",")]
        out[name] = (ret, types)
    return out


def _ctype_of(c_type: str):
    t = c_type.replace("const ", "").strip()
    if "*" in t:
        return C.c_char_p if t.startswith("char") else C.c_void_p
    return {"int64_t": C.c_int64, "size_t": C.c_size_t, "int": C.c_int, "float": C.c_float,
            "bl_status": C.c_int}[t]


def test_binding_signatures_match_the_header(bl):
    """Every ctypes signature has the header's parameter count, widths and
    return type (a mismatch would pass wrong values silently)."""
    protos = _prototypes()
    assert set(protos) == set(declared_functions())
    for name, (ret, params) in protos.items():
        res, args = bl.SIGNATURES[name]
        assert len(args) == len(params), (name, params, args)
        for i, (p, a) in enumerate(zip(params, args)):
            assert _ctype_of(p) == a, (name, i, p, a)
        assert _ctype_of(ret) == res, (name, ret, res)
