"""The small-M linear that allocates nothing (w4a4_linear_noalloc).

Some callers cannot allocate device memory when they run the layer -- a
plug-in whose host framework owns all device memory and gives a custom op no
scratch, or a decode loop that must not call cudaMalloc after start-up.  The
small-M kernel reduces its K slices on chip, so this entry point needs no
scratch at all.  The test calls it through the C ABI, twice in a row, and
checks it against w4a4_linear on the same operands.  It lives in a file of
its own that pytest collects last, and it passes both alone in a fresh
process and after the other tests.
"""

import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _operands(w4, M, N, K, seed):
    cfg = workloads.Linear("no-alloc", M=M, K=K, N=N, g=128, seed=seed)
    x, W, b = cfg.make()
    Xq, sx = w4.quantize_activation(x.cuda(), cfg.g)
    Wq, sw = w4.quantize_weight(W.cuda(), cfg.g)
    return Xq, sx, Wq, sw, b.cuda()


def _call(lib, Xq, sx, Wq, sw, b, y):
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    M, Kh = Xq.shape
    N = Wq.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.w4a4_linear_noalloc(P(Xq), P(sx), P(Wq), P(sw), P(b), P(y), M, N, 2 * Kh, y.stride(0), stream)


@pytest.mark.parametrize("M,N,K", [(8, 3072, 3072), (16, 392, 3072), (1, 5120, 5120), (33, 1024, 1024), (2, 3072, 3072), (3, 4096, 4096)])
def test_no_alloc_matches_workspace_entry(cuda_lib, M, N, K):
    lib = cuda_lib.load_library()
    Xq, sx, Wq, sw, b = _operands(cuda_lib, M, N, K, seed=M + N)
    want = cuda_lib.linear(Xq, sx, Wq, sw, b).view(torch.int16)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call(lib, Xq, sx, Wq, sw, b, y) == 0
        torch.cuda.synchronize()
        # same kernel, same operands: the outputs are bit-identical
        assert torch.equal(y.view(torch.int16), want)
    assert cuda_lib.last_device_error() == 0


def test_no_alloc_large_k_and_shape_limit(cuda_lib):
    lib = cuda_lib.load_library()
    # 64 rows, K = 12288: eight K slices per weight tile, all reduced on chip
    M, N, K = 64, 3072, 12288
    Xq, sx, Wq, sw, b = _operands(cuda_lib, M, N, K, seed=5)
    y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    assert _call(lib, Xq, sx, Wq, sw, b, y) == 0
    assert torch.equal(y.view(torch.int16), cuda_lib.linear(Xq, sx, Wq, sw, b).view(torch.int16))
    Xq65, sx65, _, _, _ = _operands(cuda_lib, 65, 256, 256, seed=6)
    Wq2, sw2 = cuda_lib.quantize_weight(workloads.make_weight(256, 256, 6).cuda(), 128)
    y2 = torch.zeros(65, 256, dtype=torch.bfloat16, device="cuda")
    assert _call(lib, Xq65, sx65, Wq2, sw2, torch.zeros(256, dtype=torch.bfloat16, device="cuda"), y2) == 2
