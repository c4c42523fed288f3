"""The allocation-free absmean entry point.

bitlinear_absmean_noalloc serves callers that cannot allocate device memory
when they need gamma (their device memory belongs to another runtime or pool,
or they may not call cudaMalloc / cudaFree after start-up); its partial sums
live in a fixed device array owned by the library.  These tests call it
through the C ABI and check that it gives exactly the gamma of the regular
entry point, which takes a caller-allocated workspace, on two calls in a row
(the second call reuses the array the first one left behind), and, where the
weights are small enough to copy to the host, the oracle's gamma too.  One case
queues both calls on a caller's stream behind a long kernel, with no host
synchronization between them (the path real callers take).  This file is
collected last so that a failure here stops a -x run only after every other
test has run.
"""
import numpy as np
import pytest
import torch

from bitlinear_b1_fwd_b200 import binding as B
from bitlinear_b1_fwd_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from bitlinear_b1_fwd_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _gamma_with_workspace(W):
    N, K = W.shape
    g = torch.full((1,), -1.0, dtype=torch.float32, device=W.device)
    ws = torch.zeros(B.bitlinear_quantize_weights_workspace_bytes(N, K), dtype=torch.uint8, device=W.device)
    B.bitlinear_absmean(W, g, ws)
    torch.cuda.synchronize()
    return g.item()


def _as_device(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(a).cuda()


@pytest.mark.parametrize("shape,bf16", [((8640, 3200), False), ((333, 1001), True), ((1, 5), False),
                                        ((32768, 8192), True)])
def test_noalloc_gamma_matches_workspace_entry(shape, bf16):
    if shape[0] * shape[1] > (1 << 24):
        # at the size limit: a seeded device generator (both sides run on the GPU)
        gen = torch.Generator(device="cuda").manual_seed(7000 + shape[0])
        Wd = torch.randn(shape, generator=gen, device="cuda").mul_(0.02)
        Wd = Wd.to(torch.bfloat16) if bf16 else Wd
    else:
        W = synth.normal_f32(7000 + shape[0], shape, 0.02)
        Wd = _as_device(synth.to_bf16_bits(W) if bf16 else W)
    want = _gamma_with_workspace(Wd)
    if shape[0] * shape[1] <= (1 << 24):     # cheap to copy: the oracle's gamma as well
        import oracle
        W_host = synth.to_bf16_bits(W) if bf16 else W
        assert np.float32(want).view(np.uint32) == oracle.gamma(W_host).view(np.uint32)
    for _ in range(2):                       # two calls in a row share the array
        g = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        B.bitlinear_absmean_noalloc(Wd, g)
        torch.cuda.synchronize()
        assert np.float32(g.item()).view(np.uint32) == np.float32(want).view(np.uint32)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    W = torch.zeros((4, 4), dtype=torch.float32, device="cuda")
    g = torch.zeros(1, dtype=torch.float32, device="cuda")
    st = B.lib().bitlinear_absmean_noalloc(W.data_ptr(), B.BL_F32, 1 << 15, (1 << 13) + 1, g.data_ptr(), None)
    assert st == B.BL_ERR_SCRATCH_LIMIT
    assert "scratch" in B.status_string(st)


def test_noalloc_on_a_caller_stream_behind_a_long_kernel():
    """Two calls queued on a non-default stream right after a kernel that runs
    for a while, with no host synchronization between them: the header reset
    and both reductions keep stream order, and each gamma is bit-equal to the
    workspace entry point's."""
    W = synth.normal_f32(7100, (2000, 3000), 0.02)
    Wd = _as_device(W)
    want = _gamma_with_workspace(Wd)
    st = torch.cuda.Stream()
    g1 = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    g2 = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    with torch.cuda.stream(st):
        torch.cuda._sleep(20_000_000)  # about 10 ms of spinning on this stream
        B.bitlinear_absmean_noalloc(Wd, g1, stream=st)
        B.bitlinear_absmean_noalloc(Wd, g2, stream=st)
    st.synchronize()
    for g in (g1, g2):
        assert np.float32(g.item()).view(np.uint32) == np.float32(want).view(np.uint32)
