"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
on numpy inputs and compare with the oracle by the tolerances of the spec
(integers bit-exact; fp32 within 1e-6 relative; bf16 within 1 ulp)."""
import numpy as np
import torch

from bitlinear_b1_fwd_b200 import binding as B


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def quantize_weights(W: np.ndarray, fmt: int, eps: float = 1e-5, codes: bool = True):
    Wd = dev(W)
    N, K = W.shape
    packed = torch.full((N, B.bitlinear_packed_row_bytes(K, fmt)), 0xAB, dtype=torch.uint8, device="cuda")
    cd = torch.full((N, K), 77, dtype=torch.int8, device="cuda") if codes else None
    gamma = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    B.bitlinear_quantize_weights(Wd, eps, fmt, packed, cd, gamma, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    return (np.float32(gamma.item()), host(cd) if codes else None, host(packed))


def forward(packed: np.ndarray, fmt: int, gamma: np.float32, N: int, K: int, x: np.ndarray,
            ydt: int, scale: np.ndarray | None = None):
    """Run bitlinear_forward; x float32 / bf16 bits (quantized inside) or int8 with scale."""
    M = x.shape[0]
    xd = dev(x)
    sd = dev(scale) if scale is not None else torch.full((M,), -1.0, dtype=torch.float32, device="cuda")
    tdt = {B.BL_F32: torch.float32, B.BL_BF16: torch.bfloat16, B.BL_I32: torch.int32}[ydt]
    y = torch.empty((M, N), dtype=tdt, device="cuda")
    if y.numel():
        y.view(torch.uint8).fill_(0xCD)
    g = torch.tensor([float(gamma)], dtype=torch.float32, device="cuda")
    ws = torch.zeros(max(256, B.bitlinear_forward_workspace_bytes(M, N, K, fmt, B.dtype_code(xd))),
                     dtype=torch.uint8, device="cuda")
    B.bitlinear_forward(dev(packed), fmt, g, N, K, xd, sd, y, ws)
    torch.cuda.synchronize()
    assert B.bitlinear_device_status(ws) == B.BL_OK
    return host(y), host(sd)


def assert_f32_rel(y: np.ndarray, ref: np.ndarray, rel: float = 1e-6):
    y = y.astype(np.float64)
    ref = ref.astype(np.float64)
    bad = np.abs(y - ref) > rel * np.abs(ref)
    assert not bad.any(), f"{bad.sum()} fp32 outputs off by more than {rel} relative; first at {np.argwhere(bad)[:3].tolist()}"


def bf16_ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between bf16 bit patterns."""
    def ordered(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def assert_bf16_ulp(y_bits: np.ndarray, ref_bits: np.ndarray, ulp: int = 1):
    d = bf16_ulp_distance(y_bits, ref_bits)
    assert (d <= ulp).all(), f"{(d > ulp).sum()} bf16 outputs more than {ulp} ulp apart"
