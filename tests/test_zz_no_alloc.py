"""The fused layer that allocates nothing (w4a4_linear_fused_noalloc).

Some callers cannot allocate device memory when they run the layer: a plug-in
whose host framework owns all device memory and hands a custom op only its
inputs and outputs, or a serving loop that must not call cudaMalloc once it
runs.  The fused layer needs scratch memory between its two kernels (the
packed activation and its scales); this entry point keeps it in a fixed
8 MiB array inside the library instead of a caller workspace.

The test calls it through the C ABI, twice in a row, and checks both outputs
against the workspace entry w4a4_linear_fused on the same operands (the same
kernels, so the outputs must be bit-identical).  It lives in a file of its
own that pytest collects last, and it passes both alone in a fresh process
and after the other tests.
"""

import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _operands(w4, M, N, K, g, seed, act=0):
    cfg = workloads.Linear("no-alloc", M=M, K=K, N=N, g=g, seed=seed, act=act)
    x, W, b = cfg.make()
    Wq, sw = w4.quantize_weight(W.cuda(), g)
    return x.cuda(), Wq, sw, b.cuda()


def _call(lib, x, Wq, sw, b, y, g, act):
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    M, K = x.shape
    N = Wq.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.w4a4_linear_fused_noalloc(P(x), x.stride(0), P(Wq), P(sw), P(b), P(y), y.stride(0), M, N, K, g, act,
                                         stream)


@pytest.mark.parametrize("M,N,K,g,act", [
    (1, 3072, 3072, 128, 0),       # tiny-M CUDA-core GEMM
    (16, 12288, 3072, 128, 0),     # small-M split-K GEMM
    (64, 3072, 12288, 128, 1),     # small-M, GELU input
    (300, 392, 512, 64, 0),        # tcgen05 GEMM, ragged tiles
    (4608, 3072, 3072, 128, 0),    # the square layer: 7.1 MB of the 8 MiB scratch
])
def test_no_alloc_matches_workspace_entry(cuda_lib, M, N, K, g, act):
    lib = cuda_lib.load_library()
    x, Wq, sw, b = _operands(cuda_lib, M, N, K, g, seed=M + N, act=act)
    want = cuda_lib.linear_fused(x, Wq, sw, b, g, act).view(torch.int16)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call(lib, x, Wq, sw, b, y, g, act) == 0
        torch.cuda.synchronize()
        # the same kernels on the same operands: bit-identical outputs
        assert torch.equal(y.view(torch.int16), want)
    assert cuda_lib.last_device_error() == 0


def test_no_alloc_back_to_back_shapes_and_size_limit(cuda_lib):
    """Two calls with different shapes back to back on one stream reuse the
    scratch; each matches the workspace entry.  A shape whose packed
    activation does not fit the scratch is refused before any launch."""
    lib = cuda_lib.load_library()
    a = _operands(cuda_lib, 4608, 3072, 3072, 128, seed=11)
    c = _operands(cuda_lib, 8, 5120, 5120, 128, seed=12)
    ya = torch.empty(4608, 3072, dtype=torch.bfloat16, device="cuda")
    yc = torch.empty(8, 5120, dtype=torch.bfloat16, device="cuda")
    assert _call(lib, *a, ya, 128, 0) == 0
    assert _call(lib, *c, yc, 128, 0) == 0
    torch.cuda.synchronize()
    assert torch.equal(ya.view(torch.int16), cuda_lib.linear_fused(*a, 128, 0).view(torch.int16))
    assert torch.equal(yc.view(torch.int16), cuda_lib.linear_fused(*c, 128, 0).view(torch.int16))
    x = torch.zeros(4608, 12288, dtype=torch.bfloat16, device="cuda")
    Wq = torch.zeros(256, 6144, dtype=torch.int8, device="cuda")
    sw = torch.ones(256, dtype=torch.float32, device="cuda")
    y = torch.empty(4608, 256, dtype=torch.bfloat16, device="cuda")
    assert _call(lib, x, Wq, sw, torch.zeros(256, dtype=torch.bfloat16, device="cuda"), y, 128, 0) == 2
    assert cuda_lib.last_device_error() == 0
