"""Dynamic LoRA on the W4A4 layer against the oracle (page "Comfy-INT4-HIPtest
README", LoRA modes: Dynamic; page "ComfyUI-INT4-Fast", Dynamic LoRA
Patching), through the C ABI.

The oracle forms the delta in float64 in the rotated basis and rounds the
layer's output once; the kernels form t = x A^T with fp32 accumulation,
round t to bf16, accumulate t B^T in fp32 and add scale * delta to the
bf16 output of the layer with one fused multiply-add before the bf16
rounding.  The bound below follows those steps."""

import ctypes

import numpy as np
import pytest
import torch

import oracle as orc
import workloads
from parity import E2E_REL_L2, rel_l2, to_np_bits

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def _ulp_bf16(v):
    """Spacing of bf16 numbers around |v| (2^-7 relative, floored at the
    smallest normal's spacing)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def _lora_inputs(N, K, r, seed):
    gen = torch.Generator().manual_seed(seed)
    A = (torch.randn(r, K, generator=gen) * 0.02).to(torch.bfloat16)
    B = (torch.randn(N, r, generator=gen) * 0.02).to(torch.bfloat16)
    return A, B


def _bound(xb, A, B, scale, t_ref, y_ref32, base32):
    """Elementwise bound on |y_gpu - y_oracle|: the two bf16 roundings of
    the kernel path (the layer's output, then the sum) against the oracle's
    one, t rounded to bf16 (2^-8 relative, with its fp32 accumulation error
    K u sum|x A| on top), and delta's fp32 accumulation (r u sum|t B|)."""
    x = np.abs(orc.bf16_bits_to_f32(xb).astype(np.float64))
    Aa = np.abs(orc.bf16_bits_to_f32(workloads.bf16_bits(A)).astype(np.float64))
    Ba = np.abs(orc.bf16_bits_to_f32(workloads.bf16_bits(B)).astype(np.float64))
    K = x.shape[1]
    r = Aa.shape[0]
    t_err = 2.0 ** -8 * np.abs(t_ref) + 2 * K * U * (x @ Aa.T)
    d_err = abs(scale) * (t_err @ Ba.T + 2 * r * U * (np.abs(t_ref) @ Ba.T))
    return _ulp_bf16(y_ref32) + _ulp_bf16(base32) + d_err + 1e-30


@pytest.mark.parametrize("M,K,N,r,rows", [
    (300, 1024, 392, 16, None), (16, 3072, 12288, 32, None), (1, 256, 8, 48, None), (700, 5120, 264, 64, None),
    (129, 3072, 520, 32, None),
    (4608, 3072, 3072, 64, "sample"),     # the square layer, sampled rows
])
def test_fused_lora_matches_oracle(cuda_lib, M, K, N, r, rows):
    cfg = workloads.Linear("lora", M=M, K=K, N=N, g=128, seed=M + r)
    x, W, b = cfg.make()
    A, B = _lora_inputs(N, K, r, seed=K + r)
    scale = 16.0 / r
    xc = x.cuda()
    Wq, sw = cuda_lib.quantize_weight(W.cuda(), cfg.g)
    base = cuda_lib.linear_fused(xc, Wq, sw, b.cuda(), cfg.g)
    y = cuda_lib.linear_fused_lora(xc, Wq, sw, b.cuda(), A.cuda(), B.cuda(), scale, cfg.g)
    # the two-step form (layer, then the in-place update) runs the same kernels
    y2 = cuda_lib.lora_add(xc, A.cuda(), B.cuda(), scale, base.clone())
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    sel = np.arange(M) if rows is None else np.array(sorted(set(np.random.default_rng(0).choice(M, 40, replace=False)) | {0, M - 1}))
    xb = workloads.bf16_bits(x[torch.as_tensor(sel)])
    wq = orc.quantize_weight(W.numpy(), cfg.g)
    ref = orc.linear_lora(xb, wq["packed"], wq["scale"], workloads.bf16_bits(b), cfg.g,
                          orc.bf16_bits_to_f32(workloads.bf16_bits(A)), orc.bf16_bits_to_f32(workloads.bf16_bits(B)),
                          scale)
    got = orc.bf16_bits_to_f32(to_np_bits(y.cpu()[torch.as_tensor(sel)])).astype(np.float64)
    # the layer part is the one the other tests pin bit for bit: take it from
    # the GPU's own base output so that only the LoRA path is measured here
    base_sel = orc.bf16_bits_to_f32(to_np_bits(base.cpu()[torch.as_tensor(sel)])).astype(np.float64)
    want = base_sel + ref["delta"]
    tol = _bound(xb, A, B, scale, ref["t"], want, base_sel)
    bad = np.abs(got - want) > tol
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} outputs off; worst excess "
                           f"{np.max(np.abs(got - want) - tol):.3g}")
    # end to end against the pure oracle (its own quantised layer plus delta)
    err = rel_l2(to_np_bits(y.cpu()[torch.as_tensor(sel)]), ref["y32"])
    assert err <= E2E_REL_L2, err
    # the update is really there: the delta moves the outputs measurably
    assert np.linalg.norm(got - base_sel) > 0.1 * np.linalg.norm(ref["delta"])
    assert cuda_lib.last_device_error() == 0


def test_lora_with_a_zero_update_leaves_y_unchanged(cuda_lib):
    M, K, N, r = 333, 1024, 264, 32
    x = workloads.make_activation(M, K, seed=5).cuda()
    y = workloads.make_activation(M, N, seed=6).cuda()
    A, B = _lora_inputs(N, K, r, seed=7)
    y0 = y.clone()
    cuda_lib.lora_add(x, A.cuda(), torch.zeros_like(B).cuda(), 1.0, y)
    assert torch.equal(y.view(torch.int16), y0.view(torch.int16))
    cuda_lib.lora_add(x, A.cuda(), B.cuda(), 0.0, y)
    assert torch.equal(y.view(torch.int16), y0.view(torch.int16))


def test_lora_down_projection_rows_are_independent(cuda_lib):
    """t of a row does not depend on the other rows (ragged M against the
    128-row tiles and the K slices of a cluster): rows of a 515-row batch
    equal the same rows computed alone."""
    M, K, N, r = 515, 3072, 392, 64
    x = workloads.make_activation(M, K, seed=8).cuda()
    A, B = _lora_inputs(N, K, r, seed=9)
    y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    cuda_lib.lora_add(x, A.cuda(), B.cuda(), 0.5, y)
    for m0, m1 in ((0, 1), (127, 130), (512, 515)):
        yy = torch.zeros(m1 - m0, N, dtype=torch.bfloat16, device="cuda")
        cuda_lib.lora_add(x[m0:m1].contiguous(), A.cuda(), B.cuda(), 0.5, yy)
        assert torch.equal(yy.view(torch.int16), y[m0:m1].view(torch.int16))


@pytest.mark.parametrize("M,N", [(200, 264), (129, 8)])
def test_lora_into_a_strided_y_keeps_the_padding(cuda_lib, M, N):
    """y with a row stride above N (a column slice of a wider buffer): the
    update lands in the N columns only, equal to the update of a compact y,
    and the padding columns keep their values."""
    K, r = 1024, 32
    x = workloads.make_activation(M, K, seed=11).cuda()
    A, B = _lora_inputs(N, K, r, seed=12)
    wide = workloads.make_activation(M, N + 72, seed=13).cuda()
    pad0 = wide[:, N:].clone()
    compact = wide[:, :N].clone()
    cuda_lib.lora_add(x, A.cuda(), B.cuda(), 0.75, wide[:, :N])
    cuda_lib.lora_add(x, A.cuda(), B.cuda(), 0.75, compact)
    assert torch.equal(wide[:, :N].view(torch.int16), compact.view(torch.int16))
    assert torch.equal(wide[:, N:].view(torch.int16), pad0.view(torch.int16))
    assert cuda_lib.last_device_error() == 0


def test_lora_add_with_k_not_a_multiple_of_the_chunk(cuda_lib):
    """w4a4_lora_add accepts any K % 8 == 0: the last 64-element chunk of x
    and A is partly past K (zero-filled by the copies).  With no rotation
    group to speak of, the reference is the plain product the header states,
    t = x A^T, then y += scale * t B^T, in float64."""
    M, K, N, r = 300, 1000, 264, 48
    x = workloads.make_activation(M, K, seed=51)
    A, B = _lora_inputs(N, K, r, seed=52)
    y0 = workloads.make_activation(M, N, seed=53)
    y = y0.clone().cuda()
    scale = 0.5
    cuda_lib.lora_add(x.cuda(), A.cuda(), B.cuda(), scale, y)
    xb = workloads.bf16_bits(x)
    xf = orc.bf16_bits_to_f32(xb).astype(np.float64)
    Af = orc.bf16_bits_to_f32(workloads.bf16_bits(A)).astype(np.float64)
    Bf = orc.bf16_bits_to_f32(workloads.bf16_bits(B)).astype(np.float64)
    t_ref = xf @ Af.T
    base = orc.bf16_bits_to_f32(workloads.bf16_bits(y0)).astype(np.float64)
    want = base + scale * (t_ref @ Bf.T)
    got = orc.bf16_bits_to_f32(to_np_bits(y.cpu())).astype(np.float64)
    tol = _bound(xb, A, B, scale, t_ref, want, base)
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{int(bad.sum())} outputs off; worst excess {np.max(np.abs(got - want) - tol):.3g}"
    assert cuda_lib.last_device_error() == 0
