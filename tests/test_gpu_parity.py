"""GPU parity of the CUDA path against the CPU oracle, called through the C ABI
(via the thin binding).  Sizes span several tiles and ragged tails; the full
workloads are checked on sampled rows, which the oracle computes one by one
(rows of the layer are independent)."""

import numpy as np
import pytest
import torch

import oracle as orc
import workloads
from parity import (E2E_REL_L2, check_epilogue_exact, check_packed, rel_l2, to_np_bits)

pytestmark = pytest.mark.gpu


def _codes(shape, seed, lo=-7, hi=7):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, shape, generator=g, dtype=torch.int8).numpy()


def _packed_cuda(q):
    return torch.from_numpy(orc.pack_int4(q)).cuda()


# --------------------------------------------------------------------------
# K1: rotate + quantise + pack
# --------------------------------------------------------------------------

def _tc_applies(K, g, act):
    """Shapes the tensor-core rotation (quantiser path 2) takes."""
    return act == 0 and g in (64, 128) and K // g <= 128


_QUANT_CASES = [
    (16, 256, 128, 0), (333, 3072, 128, 0), (333, 3072, 64, 0), (333, 3072, 256, 0),
    (67, 12288, 128, 0), (67, 12288, 256, 1), (130, 5120, 64, 1), (1, 128, 128, 0), (5, 13824, 128, 0),
    # tensor-core tiles of whole rows per 128 lanes: 5 x 24, 1 x 96, 3 x 40, 1 x 108, 2 x 48 lanes
    (777, 3072, 128, 0), (520, 12288, 128, 0), (513, 5120, 128, 0), (1000, 13824, 128, 0), (600, 3072, 64, 0),
    (700, 256, 128, 0),
    # one group per row (up to 128 rows per tile) and 128 groups per row (one row per tile)
    (40000, 128, 128, 0), (512, 8192, 64, 0),
]


@pytest.mark.parametrize("M,K,g,act,path", [c + (p,) for c in _QUANT_CASES for p in (1, 2)
                                            if p == 1 or _tc_applies(c[1], c[2], c[3])])
def test_quantize_activation_parity(cuda_lib, M, K, g, act, path):
    """Both activation kernels -- 1: register butterflies, 2: tensor cores --
    against the oracle, chosen per call."""
    x = workloads.make_activation(M, K, seed=M + K + g, outlier_frac=0.005, outlier_scale=30.0)
    Xq, sx = cuda_lib.quantize_activation(x.cuda(), g, act, path=path)
    ref = orc.quantize_activation(workloads.bf16_bits(x), g, act)
    check_packed(Xq, sx, ref, f"x {M}x{K} g{g} act{act} path{path}", g, path)


@pytest.mark.parametrize("M,K,act,path", [(4608, 3072, 0, 1), (4608, 3072, 0, 2), (4608, 12288, 0, 1),
                                          (4608, 12288, 0, 2), (4608, 12288, 1, 1)])
def test_quantize_activation_full_size(cuda_lib, M, K, act, path):
    """Every row of the M = 4608 layers' activations (the square / MLP-up
    input, and the MLP-down input with GELU) against the oracle, through the
    kernel the layers run (path 1: the routing picks it at 4608 rows) and
    through the tensor-core one.  At 4608 x 12288 each CTA of the register
    kernel walks about eleven one-row tiles, so its shared-memory ring and
    its row-amax slots wrap several times."""
    g = 128
    if path == 1:
        assert cuda_lib.quantize_activation_kernel(M, K, g, act) == 1   # what the fused layer runs here
    x = workloads.make_activation(M, K, seed=K + act, outlier_frac=0.005, outlier_scale=30.0)
    if act == 1:
        x = (x.float() * 3.0).to(torch.bfloat16)   # spread the GELU input over both tails
    Xq, sx = cuda_lib.quantize_activation(x.cuda(), g, act, path=path)
    ref = orc.quantize_activation(workloads.bf16_bits(x), g, act)
    check_packed(Xq, sx, ref, f"x {M}x{K} act{act} path{path}", g, path)


@pytest.mark.parametrize("M,path", [(70, 1), (700, 1), (70, 2), (700, 2)])
def test_quantize_activation_strided_rows(cuda_lib, M, path):
    K, g = 1024, 128
    wide = workloads.make_activation(M, K + 64, seed=3, outlier_frac=0.01, outlier_scale=20.0).cuda()
    x = wide[:, :K]
    Xq, sx = cuda_lib.quantize_activation(x, g, path=path)
    ref = orc.quantize_activation(workloads.bf16_bits(wide.cpu()[:, :K].contiguous()), g)
    check_packed(Xq, sx, ref, "strided x", g, path)


@pytest.mark.parametrize("N,K,g", [(392, 512, 128), (128, 256, 64), (200, 3072, 256), (64, 12288, 128)])
def test_quantize_weight_parity(cuda_lib, N, K, g):
    W = workloads.make_weight(N, K, seed=N + K)
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), g)
    ref = orc.quantize_weight(W.numpy(), g)
    check_packed(Wq, sw, ref, f"W {N}x{K} g{g}", g)


@pytest.mark.parametrize("path", [1, 2])
def test_quantize_zero_rows(cuda_lib, path):
    x = workloads.make_activation(40, 512, seed=9)
    x[[0, 7, 39]] = 0
    Xq, sx = cuda_lib.quantize_activation(x.cuda(), 128, path=path)
    sx = sx.cpu()
    assert sx[0] == 0 and sx[7] == 0 and sx[39] == 0
    assert torch.all(Xq.cpu()[[0, 7, 39]] == 0)
    check_packed(Xq, sx, orc.quantize_activation(workloads.bf16_bits(x), 128), "zero rows", 128, path)


def _one_hot_rows(t_bits, K=128):
    """Rows of K bf16 elements whose only nonzero is t in column 0 (bits)."""
    xb = np.zeros((t_bits.size, K), dtype=np.uint16)
    xb[:, 0] = t_bits
    return xb


def test_gelu_every_finite_bf16_input(cuda_lib):
    """Every finite bf16 value t, alone in a 128-element row (g = 64, GELU on).
    The first group rotates to GELU(t)/8 in every position and the second to
    zeros, so the row scale sx = fl(fl(|GELU(t)| / 8) / 7) exposes the GELU
    of each input; every code of the first group is 7 times the sign of
    GELU(t) (0 where it is zero), every other code 0.  This reaches every
    entry of the device's Phi table and both clamped ends (|t| < 2^-12 and
    |t| >= 8, up to the largest bf16 values of either sign)."""
    bits = np.arange(65536, dtype=np.uint32)
    t_bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)   # Inf and NaN left out
    xb = _one_hot_rows(t_bits)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    Xq, sx = cuda_lib.quantize_activation(x.cuda(), 64, 1)
    ref = orc.quantize_activation(xb, 64, 1)
    sx_g = sx.cpu().numpy().astype(np.float64)
    sx_r = ref["scale"].astype(np.float64)
    # The device forms fl(t * fl(Phi(t))) against the oracle's correctly
    # rounded GELU (about an ulp apart); below |t| = 2^-12 the entry of 2^-12
    # stands in (< 3e-8 absolute on GELU, < 6e-10 on sx); where 1 + erf
    # cancels in double precision (t < -5.6) both sides are below 1e-14.
    tol = 4.0 * 2.0 ** -24 * sx_r + 6e-10
    bad = np.flatnonzero(np.abs(sx_g - sx_r) > tol)
    assert bad.size == 0, (f"{bad.size} inputs off, first t bits {t_bits[bad[:5]].tolist()}: "
                           f"sx {sx_g[bad[:5]].tolist()} vs {sx_r[bad[:5]].tolist()}")
    # the clamped top: GELU(t) = t for t >= 8 and -0 for t <= -8
    big = ((t_bits.astype(np.uint32) >> 7) & 0xFF) >= 130
    neg = (t_bits >> 15) == 1
    assert np.all(sx_g[big & neg] == 0.0)
    assert np.all(sx_g[big & ~neg] == sx_r[big & ~neg])
    # codes: 7 times the sign wherever the oracle's GELU is clearly nonzero
    q_g = orc.unpack_int4(Xq.cpu().numpy())
    clear = sx_r > 1e-12
    assert np.array_equal(q_g[clear], ref["q"][clear])
    assert np.all(q_g[sx_g == 0] == 0)


# --------------------------------------------------------------------------
# K2 / K3: integer GEMM, bit-exact
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(300, 392, 416), (128, 256, 128), (129, 520, 3072), (65, 8, 32),
                                   (1000, 1032, 640), (256, 512, 12288)])
def test_gemm_tc_exact(cuda_lib, M, N, K):
    qa, qb = _codes((M, K), 1 + M), _codes((N, K), 2 + N)
    acc = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=0).cpu().numpy()
    want = orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb))
    assert np.array_equal(acc, want)


def test_gemm_tc_extremes(cuda_lib):
    K = 12288
    qa = np.full((130, K), 7, np.int8)
    qa[1::2] = -7
    qb = np.full((264, K), 7, np.int8)
    qb[::3] = -7
    acc = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=0).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb)))
    assert np.abs(acc).max() == 49 * K


@pytest.mark.parametrize("M", [1, 8, 16, 17, 33, 64])
@pytest.mark.parametrize("N,K", [(392, 3072), (3072, 12288), (128, 128)])
def test_gemm_smallm_exact(cuda_lib, M, N, K):
    qa, qb = _codes((M, K), 5 + M), _codes((N, K), 6 + N)
    acc = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=1).cpu().numpy()
    want = orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb))
    assert np.array_equal(acc, want)
    # same operands through the tensor-core kernel
    acc0 = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=0).cpu().numpy()
    assert np.array_equal(acc0, want)


@pytest.mark.parametrize("M", [1, 2, 3, 4])
@pytest.mark.parametrize("N,K", [(8, 32), (392, 3072), (3072, 12288), (1000, 24576), (12288, 3072), (4744, 256)])
def test_gemm_tiny_m_exact(cuda_lib, M, N, K):
    """The CUDA-core weight-streaming kernel (gemm_s32 path 3): ragged row
    groups of 1, 2 and 4 rows per warp step, K from one 16-byte chunk per row
    up to the largest widened activation that fits (4 x 24576 bytes)."""
    qa, qb = _codes((M, K), 15 + M), _codes((N, K), 16 + N)
    acc = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=3).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb)))


def test_gemm_tiny_m_extremes(cuda_lib):
    """+-7 everywhere reaches the +-49 K bound of the accumulator."""
    K, N = 24576, 24
    qa = np.full((4, K), 7, dtype=np.int8)
    qa[1] = -7
    qb = np.full((N, K), 7, dtype=np.int8)
    qb[::2] = -7
    acc = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=3).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb)))
    assert np.abs(acc).max() == 49 * K


@pytest.mark.parametrize("M,K,g", [(1, 3072, 128), (1, 12288, 128), (2, 6144, 64), (3, 4096, 256),
                                   (4, 3072, 128), (1, 256, 256), (4, 1024, 64), (2, 2048, 128)])
def test_fused_tiny_m_matches_separate_calls(cuda_lib, M, K, g):
    """For a few rows the fused entry (the tiny-M kernel streaming its weights
    into L2 while the activations are quantised) gives outputs, codes and
    scales bit-identical to the activation kernel followed by the linear
    entry, with strided activation rows and an all-zero row."""
    N = 1000 + 8 * M   # ragged row groups
    cfg = workloads.Linear("tiny fused", M=M, K=K, N=N, g=g, seed=40 + M + K // 256)
    x, W, b = cfg.make()
    if M > 1:
        x[1] = 0   # scale 0, codes 0, y = bias
    wide = torch.zeros(M, K + 64, dtype=torch.bfloat16)
    wide[:, :K] = x
    xs = wide.cuda()[:, :K]
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), g)
    bc = b.cuda()
    assert cuda_lib.linear_kernel(M, N, K) == 3
    y1 = cuda_lib.linear_fused(xs, Wq, sw, bc, g)
    nbytes = cuda_lib.load_library().w4a4_fused_workspace_bytes(M, N, K)
    ws = cuda_lib.workspace(nbytes, xs.device, "fused")
    codes = ws[: M * K // 2].view(torch.int8).view(M, K // 2).clone()
    off = (M * K // 2 + 255) // 256 * 256
    scales = ws[off: off + 4 * M].view(torch.float32).clone()
    Xq, sx = cuda_lib.quantize_activation(xs, g)
    y2 = cuda_lib.linear(Xq, sx, Wq, sw, bc)
    assert torch.equal(codes, Xq)
    assert torch.equal(scales.view(torch.int32), sx.view(torch.int32))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    ref = orc.quantize_activation(workloads.bf16_bits(x), g)
    check_packed(codes, scales, ref, f"fused tiny {M}x{K} g{g}", g)


def test_full_size_paths_agree(cuda_lib):
    """At the square layer's size the tensor-core kernel's accumulators equal
    an exact fp64 product on the GPU (integers below 2^53), and its bf16
    outputs equal the same epilogue steps in torch, on every element."""
    M, N, K = 4608, 3072, 3072
    x = workloads.make_activation(M, K, seed=M + 5, outlier_frac=0.005, outlier_scale=30.0).cuda()
    W = workloads.make_weight(N, K, seed=N + 5).cuda()
    b = workloads.make_bias(N, seed=N).cuda()
    Xq, sx = cuda_lib.quantize_activation(x, 128)
    Wq, sw = cuda_lib.quantize_weight(W, 128)
    acc0 = cuda_lib.gemm_s32(Xq, Wq, path=0)
    qa = torch.from_numpy(orc.unpack_int4(Xq.cpu().numpy())).cuda().double()
    qb = torch.from_numpy(orc.unpack_int4(Wq.cpu().numpy())).cuda().double()
    ref = (qa @ qb.T).round().to(torch.int32)
    assert torch.equal(acc0, ref)
    y = cuda_lib.linear(Xq, sx, Wq, sw, b)
    want = (((ref.float() * sx[:, None]) * sw[None, :]) + b.float()[None, :]).to(torch.bfloat16)
    assert torch.equal(y.view(torch.int16), want.view(torch.int16))


# --------------------------------------------------------------------------
# Rank-one epilogue and the whole layer
# --------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K,g,bias", [(300, 392, 512, 128, True), (16, 392, 3072, 128, True),
                                          (64, 3072, 3072, 64, False), (513, 264, 1024, 256, False)])
def test_linear_epilogue_exact(cuda_lib, M, N, K, g, bias):
    x = workloads.make_activation(M, K, seed=M, outlier_frac=0.005, outlier_scale=30.0)
    W = workloads.make_weight(N, K, seed=N)
    b = workloads.make_bias(N, seed=N) if bias else None
    Xq, sx = cuda_lib.quantize_activation(x.cuda(), g)
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), g)
    y = cuda_lib.linear(Xq, sx, Wq, sw, b.cuda() if bias else None)
    acc = orc.gemm_s32(Xq.cpu().numpy(), Wq.cpu().numpy())
    check_epilogue_exact(y, acc, sx.cpu().numpy(), sw.cpu().numpy(),
                         workloads.bf16_bits(b) if bias else None, f"linear {M}x{K}->{N}")


_wq_cache = {}


def _oracle_weight(W, g):
    key = (tuple(W.shape), g, float(W[0, 0]), float(W[-1, -1]), float(W.sum()))
    if key not in _wq_cache:
        _wq_cache[key] = orc.quantize_weight(W.numpy(), g)
    return _wq_cache[key]


def _oracle_layer(cfg, x, W, b, rows=None):
    """Pure-oracle layer on (a sample of) the rows."""
    wq = _oracle_weight(W, cfg.g)
    xb = workloads.bf16_bits(x if rows is None else x[rows])
    return wq, orc.linear(xb, wq["packed"], wq["scale"], workloads.bf16_bits(b) if b is not None else None,
                          cfg.g, cfg.act)


def _check_layer(cuda_lib, cfg, x, W, b, rows=None, y=None):
    xc, Wc = x.cuda(), W.cuda()
    bc = b.cuda() if b is not None else None
    Wq, sw = cuda_lib.quantize_weight(Wc, cfg.g)
    if y is None:
        y = cuda_lib.linear_fused(xc, Wq, sw, bc, cfg.g, cfg.act)
    Xq, sx = cuda_lib.quantize_activation(xc, cfg.g, cfg.act)
    wref, ref = _oracle_layer(cfg, x, W, b, rows)
    check_packed(Wq, sw, wref, f"{cfg.name} weights", cfg.g)
    sel = slice(None) if rows is None else torch.as_tensor(rows)
    xa = orc.quantize_activation(workloads.bf16_bits(x if rows is None else x[rows]), cfg.g, cfg.act)
    path = cuda_lib.quantize_activation_kernel(cfg.M, cfg.K, cfg.g, cfg.act)
    check_packed(Xq.cpu()[sel], sx.cpu()[sel], xa, f"{cfg.name} activations", cfg.g, path)
    # the fused output equals the oracle epilogue on the GPU's own operands
    acc = orc.gemm_s32(Xq.cpu()[sel].numpy(), Wq.cpu().numpy())
    check_epilogue_exact(y.cpu()[sel], acc, sx.cpu()[sel].numpy(), sw.cpu().numpy(),
                         workloads.bf16_bits(b) if b is not None else None, cfg.name)
    err = rel_l2(to_np_bits(y.cpu()[sel]), ref["y32"])
    assert err <= E2E_REL_L2, f"{cfg.name}: relative L2 error {err:.3g}"
    return y


def test_tiny_layer(cuda_lib):
    cfg = workloads.TINY
    x, W, b = cfg.make()
    _check_layer(cuda_lib, cfg, x, W, b)


@pytest.mark.parametrize("M,K,N,g", [(333, 1024, 520, 128), (130, 3072, 264, 64), (700, 2048, 1024, 256)])
def test_medium_layers(cuda_lib, M, K, N, g):
    cfg = workloads.Linear("medium", M=M, K=K, N=N, g=g, seed=M)
    x, W, b = cfg.make()
    _check_layer(cuda_lib, cfg, x, W, b)


def _sample_rows(M, n=48, seed=0):
    g = np.random.default_rng(seed)
    rows = set(g.choice(M, size=n - 4, replace=False).tolist()) | {0, 1, M - 2, M - 1}
    return sorted(rows)


def test_square_full_size_sampled(cuda_lib):
    cfg = workloads.SQUARE
    x, W, b = cfg.make()
    _check_layer(cuda_lib, cfg, x, W, b, rows=_sample_rows(cfg.M))


def test_mlp_pair_full_size_sampled(cuda_lib):
    up, down = workloads.MLP_UP, workloads.MLP_DOWN
    x, Wu, bu = up.make()
    _, Wd, bd = down.make()
    rows = _sample_rows(up.M, 24, seed=1)
    yu = _check_layer(cuda_lib, up, x, Wu, bu, rows=rows)
    # the down layer reads GELU(up output), applied inside the activation kernel
    _check_layer(cuda_lib, down, yu.cpu(), Wd, bd, rows=rows)


@pytest.mark.parametrize("cfg", workloads.small_m_sweep(), ids=lambda c: c.name)
def test_small_m_sweep(cuda_lib, cfg):
    x, W, b = cfg.make()
    _check_layer(cuda_lib, cfg, x, W, b)


# --------------------------------------------------------------------------
# Edge cases
# --------------------------------------------------------------------------

def test_zero_rows_give_bias(cuda_lib):
    cfg = workloads.Linear("zero rows", M=80, K=512, N=264, g=128, seed=4)
    x, W, b = cfg.make()
    x[[3, 50]] = 0
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), 128)
    y = cuda_lib.linear_fused(x.cuda(), Wq, sw, b.cuda(), 128).cpu()
    assert torch.equal(y[3].view(torch.int16), b.view(torch.int16))
    assert torch.equal(y[50].view(torch.int16), b.view(torch.int16))


def test_empty_batch_is_a_no_op(cuda_lib):
    W = workloads.make_weight(256, 512, seed=1).cuda()
    Wq, sw = cuda_lib.quantize_weight(W, 128)
    x = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    y = cuda_lib.linear_fused(x, Wq, sw, None, 128)
    assert y.shape == (0, 256)


def test_repeat_calls_share_workspace_deterministically(cuda_lib):
    # alternating shapes on one cached workspace keep giving bit-identical
    # results, and the fused and two-call paths agree
    outs = {}
    for rep in range(3):
        for (M, N, K) in ((8, 3072, 12288), (64, 392, 3072), (300, 392, 512), (16, 3072, 3072)):
            cfg = workloads.Linear("r", M=M, K=K, N=N, g=128, seed=M)
            x, W, b = cfg.make()
            Wq, sw = cuda_lib.quantize_weight(W.cuda(), 128)
            y1 = cuda_lib.linear_fused(x.cuda(), Wq, sw, b.cuda(), 128)
            Xq, sx = cuda_lib.quantize_activation(x.cuda(), 128)
            y2 = cuda_lib.linear(Xq, sx, Wq, sw, b.cuda())
            assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
            key = (M, N, K)
            if key in outs:
                assert torch.equal(outs[key], y1.view(torch.int16))
            outs[key] = y1.view(torch.int16).clone()


def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    lib = cuda_lib.load_library()
    assert cuda_lib.last_device_error() == 0
    stream = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert lib.w4a4_debug_wait_timeout(2000, ctypes.c_void_p(stream)) == 0
    assert cuda_lib.last_device_error() == 8          # W4A4_ERR_TIMEOUT, then cleared
    assert cuda_lib.last_device_error() == 0
    # the context is still usable
    cfg = workloads.TINY
    x, W, b = cfg.make()
    _check_layer(cuda_lib, cfg, x, W, b)


@pytest.mark.parametrize("kernel", ["quant_butterfly", "quant_tensor_core", "gemm_tc", "gemm_small_m",
                                    "fused_square", "lora", "requant_chain"])
def test_product_kernel_waits_expire_and_context_survives(cuda_lib, kernel):
    """With a wait limit of a few nanoseconds the product kernels' waits on
    their copy rings, widened stages, accumulators and cluster peers expire
    wherever they would have to wait: each kernel must record
    W4A4_ERR_TIMEOUT, stop every role, let its copies and MMAs drain, free
    its tensor memory and exit (its outputs are then undefined).  With the
    default limit back, the same context runs the layer correctly."""
    g = 128
    big = workloads.make_activation(4608, 3072, seed=77, outlier_frac=0.005, outlier_scale=30.0).cuda()
    Wbig = workloads.make_weight(3072, 3072, seed=78).cuda()
    Wq, sw = cuda_lib.quantize_weight(Wbig, g)
    Wk = workloads.make_weight(3072, 12288, seed=79).cuda()
    Wqk, swk = cuda_lib.quantize_weight(Wk, g)
    Xq, sx = cuda_lib.quantize_activation(big, g)
    x16 = workloads.make_activation(16, 12288, seed=80).cuda()
    Xq16, sx16 = cuda_lib.quantize_activation(x16, g)
    gen = torch.Generator().manual_seed(81)
    A = (torch.randn(64, 3072, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    B = (torch.randn(3072, 64, generator=gen) * 0.02).to(torch.bfloat16).cuda()
    ylora = torch.zeros(4608, 3072, dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    assert cuda_lib.last_device_error() == 0
    runs = {
        "quant_butterfly": lambda: cuda_lib.quantize_activation(big, g, path=1),
        "quant_tensor_core": lambda: cuda_lib.quantize_activation(big, g, path=2),
        "gemm_tc": lambda: cuda_lib.linear(Xq[:1000].contiguous(), sx[:1000].contiguous(), Wq, sw),
        "gemm_small_m": lambda: cuda_lib.linear(Xq16, sx16, Wqk, swk),
        "fused_square": lambda: cuda_lib.linear_fused(big, Wq, sw, None, g),
        "lora": lambda: cuda_lib.lora_add(big, A, B, 0.25, ylora),
        # the GEMM instance with the requantising epilogue (its second pass
        # has no waits and runs on whatever the aborted GEMM left)
        "requant_chain": lambda: cuda_lib.linear_fused_requant(big, Wq, sw, None, g, 0, 128),
    }
    if kernel == "gemm_small_m":
        assert cuda_lib.linear_kernel(16, 3072, 12288) == 1
    try:
        cuda_lib.debug_set_wait_limit(5)
        runs[kernel]()
        status = cuda_lib.last_device_error()
    finally:
        cuda_lib.debug_set_wait_limit(0)
    assert status == 8                                  # W4A4_ERR_TIMEOUT, then cleared
    assert cuda_lib.last_device_error() == 0
    cfg = workloads.TINY
    x, W, b = cfg.make()
    _check_layer(cuda_lib, cfg, x, W, b)
    y = cuda_lib.linear_fused(big, Wq, sw, None, g)     # and the full layer again
    assert torch.equal(y.view(torch.int16), cuda_lib.linear(Xq, sx, Wq, sw).view(torch.int16))
    assert cuda_lib.last_device_error() == 0


@pytest.mark.parametrize("n_rows,path", [(300, 1), (600, 1), (300, 2), (600, 2)])
def test_quantize_exact_ties_follow_round_half_even(cuda_lib, n_rows, path):
    """Rows built from the hand-derived tie fixture: every rotated value is an
    exact multiple of 1/2 or 1/4, so many codes sit exactly on a rounding
    boundary.  The kernel must decide all of them as round-half-even of the
    fp32 quotient, with no boundary tolerance."""
    import os
    import scipy.linalg
    from test_oracle_pins import _read_golden_ties
    g, cases = _read_golden_ties()
    Hs = scipy.linalg.hadamard(g).astype(np.float64) / 8.0
    rows = []
    for c in cases:
        r = np.zeros(g)
        r[:len(c["r"])] = c["r"]
        rows.append(Hs @ r)
    # K = 128 (two groups of 64): pair the cases, and repeat with permuted
    # group order and signs so the rows span several CTAs and lanes
    base = [np.concatenate([rows[0], rows[1]]), np.concatenate([rows[1], -rows[0]])]
    X = np.stack([base[i % 2] * (1 if (i // 2) % 2 == 0 else -1) for i in range(n_rows)])
    xb = orc.f32_to_bf16_bits(X.astype(np.float32))
    assert np.array_equal(orc.bf16_bits_to_f32(xb).astype(np.float64), X)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
    Xq, sx = cuda_lib.quantize_activation(x, g, path=path)
    ref = orc.quantize_activation(xb, g)
    assert np.array_equal(Xq.cpu().numpy(), ref["packed"])
    assert np.array_equal(sx.cpu().numpy(), ref["scale"])
    assert np.sum(orc.boundary_window(ref["v"], 0.0)) > 1000   # the ties are really there


def test_block_stack_chain_one_quantised_activation(cuda_lib):
    """One transformer block of the stack workload at reduced width: q, k and
    v read one quantised activation (identical to three fused calls), out
    reads v's output, up reads out's, down reads GELU(up); every layer of the
    chain matches the oracle on its GPU input."""
    M, D, F, g = 300, 1024, 2816, 128
    x = workloads.make_activation(M, D, seed=21, outlier_frac=0.005, outlier_scale=30.0)
    shapes = {"q": (D, D), "k": (D, D), "v": (D, D), "out": (D, D), "up": (D, F), "down": (F, D)}
    Ws = {nm: workloads.make_weight(N, K, seed=30 + i) for i, (nm, (K, N)) in enumerate(shapes.items())}
    bs = {nm: workloads.make_bias(N, seed=40 + i) for i, (nm, (K, N)) in enumerate(shapes.items())}
    Wq = {nm: cuda_lib.quantize_weight(W.cuda(), g) for nm, W in Ws.items()}
    xc = x.cuda()
    Xq, sx = cuda_lib.quantize_activation(xc, g)
    qkv = {}
    for nm in ("q", "k", "v"):
        qkv[nm] = cuda_lib.linear(Xq, sx, Wq[nm][0], Wq[nm][1], bs[nm].cuda())
        fused = cuda_lib.linear_fused(xc, Wq[nm][0], Wq[nm][1], bs[nm].cuda(), g)
        assert torch.equal(qkv[nm].view(torch.int16), fused.view(torch.int16))
    rows = _sample_rows(M, 24, seed=5)
    cfg = lambda nm, act=0: workloads.Linear(f"stack {nm}", M=M, K=shapes[nm][0], N=shapes[nm][1], g=g, act=act)
    for nm in ("q", "k", "v"):
        _check_layer(cuda_lib, cfg(nm), x, Ws[nm], bs[nm], rows=rows, y=qkv[nm])
    y_out = _check_layer(cuda_lib, cfg("out"), qkv["v"].cpu(), Ws["out"], bs["out"], rows=rows)
    y_up = _check_layer(cuda_lib, cfg("up"), y_out.cpu(), Ws["up"], bs["up"], rows=rows)
    y_down = _check_layer(cuda_lib, cfg("down", act=1), y_up.cpu(), Ws["down"], bs["down"], rows=rows)
    assert torch.isfinite(y_down.float()).all()


@pytest.mark.parametrize("M,N,K", [(300, 392, 416), (128, 256, 128), (129, 520, 3072), (65, 8, 32), (1000, 1032, 640)])
def test_gemm_legacy_mma_sync_exact(cuda_lib, M, N, K):
    """The warp-level mma.m16n8k64.s4 comparison kernel gives the same int32
    accumulators as the oracle."""
    qa, qb = _codes((M, K), 51 + M), _codes((N, K), 52 + N)
    acc = cuda_lib.gemm_s32(_packed_cuda(qa), _packed_cuda(qb), path=2).cpu().numpy()
    assert np.array_equal(acc, orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb)))
