"""Layer chains: the fused layer with the requantising epilogue for the layer
after it (w4a4_linear_fused_requant), against the oracle's two passes
(oracle.chain_requant: the per-tile partial amax of rotate(GELU(y)), the row
scale from their maximum, the codes), through the C ABI.

y must equal the plain fused layer bit for bit.  The next layer's codes and
scales are compared with the oracle quantising the GPU's own y, so that only
the requantisation is measured, with the register quantiser's bounds
(parity.scale_rtol and the rounding-boundary window): both passes form GELU
as the activation kernel does (t times Phi(t) from its table) and sum the
rotation in fp32 along butterflies of depth log2 g (within chunks of 32 in
registers, then across chunks), only in another order."""

import numpy as np
import pytest
import torch

import oracle as orc
import workloads
from parity import check_packed, scale_rtol, to_np_bits

pytestmark = pytest.mark.gpu

BLOCK = 256   # the GEMM's output tile width: the epilogue's amax blocks


def _chain_scale_ok(gpu_scale, ref_scale, g):
    tol = scale_rtol(g, 1)
    gs = gpu_scale.astype(np.float64)
    rs = ref_scale.astype(np.float64)
    zero = rs == 0
    assert np.all(gs[zero] == 0)
    rel = np.abs(gs[~zero] - rs[~zero]) / rs[~zero]
    assert np.all(rel <= tol), f"scale rel diff {rel.max():.3g} > {tol:.3g}"


def _run(cuda_lib, M, K, N, g, g_next, seed, rows=None):
    cfg = workloads.Linear("chain", M=M, K=K, N=N, g=g, seed=seed)
    x, W, b = cfg.make()
    xc = x.cuda()
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), g)
    bc = b.cuda()
    y_plain = cuda_lib.linear_fused(xc, Wq, sw, bc, g)
    y, xq, sx = cuda_lib.linear_fused_requant(xc, Wq, sw, bc, g, 0, g_next)
    torch.cuda.synchronize()
    assert cuda_lib.last_device_error() == 0
    assert torch.equal(y.view(torch.int16), y_plain.view(torch.int16)), "y differs from the plain fused layer"
    sel = np.arange(M) if rows is None else np.asarray(rows)
    yb = to_np_bits(y.cpu()[torch.as_tensor(sel)])
    ref = orc.chain_requant(yb, g_next, BLOCK, act=1)
    assert np.array_equal(ref["scale_from_partials"], ref["scale"])
    xq_s, sx_s = xq.cpu()[torch.as_tensor(sel)], sx.cpu()[torch.as_tensor(sel)]
    _chain_scale_ok(sx_s.numpy(), ref["scale"], g_next)
    # codes: identical to the oracle's except within its rounding-boundary
    # window (the scales were checked above)
    check_packed(xq_s, torch.from_numpy(ref["scale"]), ref, f"chain {M}x{K}->{N} g_next={g_next}", g_next)
    return y, xq, sx, ref


@pytest.mark.parametrize("M,K,N,g_next", [
    (300, 1024, 512, 128),     # two row tiles (the second ragged), two column tiles
    (700, 512, 384, 64),       # the last column tile half past N
    (129, 256, 768, 256),      # a group of 256 fills a whole tile
    (513, 3072, 1280, 128),
])
def test_requant_epilogue_matches_oracle(cuda_lib, M, K, N, g_next):
    _run(cuda_lib, M, K, N, 128, g_next, seed=M + N)


def test_requant_epilogue_full_size_sampled(cuda_lib):
    """The MLP up layer 4608x3072 -> 12288 feeding its down layer (g = 128):
    sampled rows against the oracle, every row against the one-pass
    activation kernel on the same y."""
    up = workloads.MLP_UP
    rng = np.random.default_rng(7)
    rows = sorted(set(rng.choice(up.M, size=36, replace=False).tolist()) | {0, 255, 256, up.M - 1})
    y, xq, sx, _ = _run(cuda_lib, up.M, up.K, up.N, up.g, 128, seed=up.seed, rows=rows)
    xq1, sx1 = cuda_lib.quantize_activation(y, 128, 1)
    a, b = sx.cpu().numpy().astype(np.float64), sx1.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(a - b) / b) <= 2 * scale_rtol(128, 1)
    q0, q1 = orc.unpack_int4(xq.cpu().numpy()), orc.unpack_int4(xq1.cpu().numpy())
    diff = q0 != q1
    assert diff.sum() <= 1e-5 * diff.size and np.all(np.abs(q0[diff].astype(int) - q1[diff]) == 1)


def test_requant_chain_feeds_the_down_layer(cuda_lib):
    """The down layer from the chained codes equals the down layer that
    quantises GELU(y) itself, up to the codes' rounding-boundary flips."""
    M, K, N, Nd = 600, 1024, 1024, 512
    up = workloads.Linear("chain up", M=M, K=K, N=N, g=128, seed=21)
    x, W, b = up.make()
    Wd = workloads.make_weight(Nd, N, seed=22)
    bd = workloads.make_bias(Nd, seed=23)
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), 128)
    Wdq, swd = cuda_lib.quantize_weight(Wd.cuda(), 128)
    y, xq, sx = cuda_lib.linear_fused_requant(x.cuda(), Wq, sw, b.cuda(), 128, 0, 128)
    y2 = cuda_lib.linear(xq, sx, Wdq, swd, bd.cuda())
    y2_ref = cuda_lib.linear_fused(y, Wdq, swd, bd.cuda(), 128, 1)
    a = y2.float().cpu().numpy()
    r = y2_ref.float().cpu().numpy()
    assert np.linalg.norm(a - r) <= 1e-3 * np.linalg.norm(r)


def test_requant_small_batch_uses_the_one_pass_kernel(cuda_lib):
    """Batches routed to the weight-streaming kernels run the layer and the
    activation kernel: the codes equal the one-pass kernel's exactly."""
    M, K, N = 16, 3072, 1024
    cfg = workloads.Linear("chain small", M=M, K=K, N=N, g=128, seed=31)
    x, W, b = cfg.make()
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), 128)
    y, xq, sx = cuda_lib.linear_fused_requant(x.cuda(), Wq, sw, b.cuda(), 128, 0, 128)
    xq1, sx1 = cuda_lib.quantize_activation(y, 128, 1)
    assert torch.equal(xq, xq1) and torch.equal(sx, sx1)


def test_requant_epilogue_gelu_input_and_strided_output(cuda_lib):
    """A chain link inside a chain: a GELU input (act = 1, g = 64) and y
    written into a column slice of a wider buffer (row stride N + 64); the
    padding columns keep their values and the codes still match the oracle."""
    M, K, N, g, g_next = 257, 512, 640, 64, 128
    cfg = workloads.Linear("chain gelu", M=M, K=K, N=N, g=g, seed=41, act=1)
    x, W, b = cfg.make()
    xc = x.cuda()
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), g)
    wide = workloads.make_activation(M, N + 64, seed=42).cuda()
    pad = wide[:, N:].clone()
    y, xq, sx = cuda_lib.linear_fused_requant(xc, Wq, sw, b.cuda(), g, 1, g_next, out=wide[:, :N])
    assert torch.equal(wide[:, N:].view(torch.int16), pad.view(torch.int16))
    y_plain = cuda_lib.linear_fused(xc, Wq, sw, b.cuda(), g, 1)
    assert torch.equal(y.contiguous().view(torch.int16), y_plain.view(torch.int16))
    ref = orc.chain_requant(to_np_bits(y.cpu()), g_next, BLOCK, act=1)
    _chain_scale_ok(sx.cpu().numpy(), ref["scale"], g_next)
    check_packed(xq.cpu(), torch.from_numpy(ref["scale"]), ref, "chain gelu strided", g_next)
    assert cuda_lib.last_device_error() == 0
