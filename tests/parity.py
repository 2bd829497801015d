"""Comparison helpers for the GPU parity tests (test infrastructure).

The criteria follow the layer's written tolerances:
  * packed codes: identical, except codes whose oracle pre-rounding value
    lies within 1e-6 relative of a rounding boundary, and such codes are at
    most 1e-5 of all codes;
  * scales: the kernels sum the rotation in fp32, the oracle in fp64, so the
    scales agree only to the error bound of that summation (scale_rtol);
  * int32 accumulators: bit-exact on identical packed operands;
  * rank-one epilogue: both sides round the same fp32 steps in the same order,
    so the bf16 outputs recomputed from the GPU's own operands are bit-exact;
  * end to end against the pure oracle: relative L2 error <= 1e-2.
"""

import math

import numpy as np
import torch

import oracle as orc

U32 = 2.0 ** -24      # unit roundoff of fp32 (round to nearest)
BOUNDARY_REL = 1e-6
BOUNDARY_FRAC = 1e-5
E2E_REL_L2 = 1e-2


def to_np_bits(t):
    """bf16 torch tensor (any device) -> uint16 numpy bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def scale_rtol(g, path=1):
    """Relative bound on |s_gpu - s_oracle| / s_oracle for group size g.

    Each rotated value u_i = sum_j H[i,j] x_j of a group is summed by the
    kernel in fp32 along a tree of depth d, so |fl(u_i) - u_i| <= d u sum_j |x_j|
    (u = 2^-24, to first order).  By Cauchy-Schwarz sum_j |x_j| <= sqrt(g) |x|_2,
    and by Parseval (H H^T = g I) the group's largest |u_i| is at least |x|_2,
    so every error is at most d sqrt(g) u times that group's -- hence the row's
    -- largest |u|: the row amax moves by at most d sqrt(g) u relative.  Five
    more roundings separate the two sides (the kernel's 1/sqrt(g) constant
    and product, the oracle's fp32 rotated value, and the two divisions by
    7).  Path 1 (butterflies): d = log2(g).  Path 2 (tensor cores): each MMA
    sums 16 products, in an order the hardware does not document (taken as
    sequential, depth 16), and g/16 such partial sums accumulate in fp32:
    d = 16 + g/16.
    """
    d = math.log2(g) if path == 1 else 16 + g / 16
    return (d * math.sqrt(g) + 5) * U32


def check_packed(gpu_packed, gpu_scale, ref, what="", g=128, path=1):
    """Compare GPU packed codes and scales against an oracle quantisation
    dict (g and path give the scale bound, see scale_rtol)."""
    gp = gpu_packed.detach().cpu().numpy()
    gs = gpu_scale.detach().cpu().numpy()
    assert gp.shape == ref["packed"].shape, what
    rs = ref["scale"]
    rel = np.abs(gs.astype(np.float64) - rs) / np.maximum(np.abs(rs.astype(np.float64)), 1e-30)
    zero = rs == 0
    assert np.all(gs[zero] == 0), f"{what}: zero rows must keep scale 0"
    tol = scale_rtol(g, path)
    assert np.all(rel[~zero] <= tol), f"{what}: scale max rel diff {rel[~zero].max():.3g} > {tol:.3g}"
    qg = orc.unpack_int4(gp)
    qr = ref["q"]
    mism = qg != qr
    n = int(mism.sum())
    if n:
        window = orc.boundary_window(ref["v"], BOUNDARY_REL)
        outside = mism & ~window
        assert not outside.any(), (
            f"{what}: {int(outside.sum())} codes differ away from a rounding boundary; "
            f"first at {np.argwhere(outside)[0].tolist()}")
        assert n <= max(1, BOUNDARY_FRAC * qg.size), f"{what}: {n} boundary flips of {qg.size}"
        assert np.all(np.abs(qg[mism].astype(int) - qr[mism].astype(int)) == 1)
    return n


def check_epilogue_exact(y_gpu, acc, sx, sw, bias_bits, what=""):
    """bf16 outputs must equal the oracle epilogue on the same operands."""
    _, want = orc.epilogue(acc, sx, sw, bias_bits)
    got = to_np_bits(y_gpu)
    diff = got != want
    assert not diff.any(), f"{what}: {int(diff.sum())} outputs differ, first at {np.argwhere(diff)[0].tolist()}"


def rel_l2(y_gpu_bits, y_ref32):
    y = orc.bf16_bits_to_f32(y_gpu_bits).astype(np.float64)
    r = y_ref32.astype(np.float64)
    return float(np.linalg.norm(y - r) / max(np.linalg.norm(r), 1e-30))
