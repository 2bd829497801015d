"""ConvRot W4A4 linear, written out step by step on the CPU (numpy, fp64 where
the method leaves the precision open).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Product code never
imports this module.

The steps follow the "Description" section of the page "[PR #63]
int4_tensorwise: W4A4 layout (+ConvRot) with fused CUDA kernels" in its own
order: rotate (ConvRot, a blockwise Walsh-Hadamard transform), quantise each
row to signed int4 with one fp32 scale per row, pack two nibbles per byte
low-nibble-first into an [R, K/2] int8 container, multiply the integer codes
with int32 accumulation, and dequantise with the rank-one epilogue
acc * sx[m] * sw[n] (+ bias).

Array conventions: bf16 tensors travel as their raw 16-bit patterns in
``numpy.uint16`` arrays so that both sides see identical bits; packed int4
data is ``numpy.int8``; scales are ``numpy.float32``.
"""

import numpy as np
from scipy.special import erf as _erf

# ---------------------------------------------------------------------------
# bf16 <-> fp32.  bf16 is the top half of an IEEE binary32 pattern, so the
# widening is exact; the narrowing rounds to nearest, ties to even.
# ---------------------------------------------------------------------------


def bf16_bits_to_f32(bits):
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def f32_to_bf16_bits(x):
    """Round float32 values to bf16 (round to nearest, ties to even).

    Returns the uint16 bit patterns.  NaN inputs become a quiet NaN.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded = np.where(nan, np.uint16(0x7FC0), rounded)
    return rounded


# ---------------------------------------------------------------------------
# ConvRot: blockwise Walsh-Hadamard rotation.
# ---------------------------------------------------------------------------


def sylvester_hadamard(g):
    """The g x g Walsh-Hadamard matrix in natural (Sylvester) order,
    H[i, j] = (-1)^popcount(i & j), as int64.

    The pages name a "Hadamard ConvRot" with a configurable group size and a
    radix-4 FHT but print no matrix; natural order without random signs is
    what an unmodified fast Walsh-Hadamard transform computes, and it is used
    for activations and weights alike.
    """
    if g < 1 or (g & (g - 1)) != 0:
        raise ValueError("group size must be a power of two")
    idx = np.arange(g, dtype=np.int64)
    anded = idx[:, None] & idx[None, :]
    parity = np.zeros_like(anded)
    t = anded.copy()
    while np.any(t):
        parity ^= t & 1
        t >>= 1
    return np.where(parity == 1, -1, 1).astype(np.int64)


def rotate_rows(X, g):
    """Rotate every row of X in contiguous groups of g columns.

    For group b of row m: u[m, b*g + i] = sum_j H[i, j] * X[m, b*g + j],
    a dense O(g^2) sum in float64 (exact for bf16 inputs, and for fp32
    inputs up to float64 rounding); then r = float32(u / sqrt(g)).

    Returns (u as float64, r as float32).
    """
    X = np.asarray(X, dtype=np.float64)
    R, K = X.shape
    if K % g != 0:
        raise ValueError("K must be a multiple of the group size")
    H = sylvester_hadamard(g).astype(np.float64)
    u = (X.reshape(R, K // g, g) @ H.T).reshape(R, K)
    r = (u / np.sqrt(np.float64(g))).astype(np.float32)
    return u, r


def gelu_f32(t):
    """GELU with the exact error function, 0.5*t*(1 + erf(t/sqrt(2))),
    evaluated in float64 on float32 inputs and rounded once to float32.

    Not on the pages: the MLP workload feeds the down projection with the
    GELU of the up projection's bf16 output.
    """
    t64 = np.asarray(t, dtype=np.float32).astype(np.float64)
    return (0.5 * t64 * (1.0 + _erf(t64 / np.sqrt(2.0)))).astype(np.float32)


# ---------------------------------------------------------------------------
# Symmetric per-row int4 quantisation and low-nibble-first packing.
# ---------------------------------------------------------------------------


def quantize_rows(r):
    """Per-row symmetric int4 quantisation of float32 rows.

    s[m] = max_k |r[m, k]| / 7 (float32 division); v = r / s (float32
    division); q = clamp(round_half_even(v), -7, 7).  An all-zero row has
    s = 0 and q = 0.

    Returns (q as int8 [R, K], s as float32 [R], v as float32 [R, K]).
    """
    r = np.asarray(r, dtype=np.float32)
    amax = np.max(np.abs(r), axis=1)
    s = (amax / np.float32(7.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        v = (r / s[:, None]).astype(np.float32)
    q = np.clip(np.rint(v), -7, 7)
    q = np.where(s[:, None] > 0, q, 0).astype(np.int8)
    v = np.where(s[:, None] > 0, v, np.float32(0)).astype(np.float32)
    return q, s, v


def pack_int4(q):
    """Pack int4 codes two per byte: element 2j in the low nibble, 2j+1 in
    the high nibble, each as a 4-bit two's-complement value."""
    q = np.asarray(q, dtype=np.int16)
    if q.shape[-1] % 2 != 0:
        raise ValueError("the packed dimension must be even")
    lo = q[..., 0::2] & 0xF
    hi = q[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8).view(np.int8)


def unpack_int4(p):
    """Inverse of pack_int4: every byte yields (low nibble, high nibble),
    each sign-extended from 4 bits."""
    b = np.asarray(p, dtype=np.int8).astype(np.int16)
    hi = b >> 4                      # arithmetic shift keeps the sign
    lo = b & 0xF
    lo = lo - 16 * (lo >= 8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def boundary_window(v, rel=1e-6):
    """True where a pre-rounding value v lies within rel*|v| of a rounding
    boundary k + 1/2; such elements may legitimately round either way when
    the rotation is summed in a different order."""
    v = np.asarray(v, dtype=np.float64)
    d = np.abs(v - (np.floor(v) + 0.5))
    return d <= rel * np.abs(v)


def quantize_weight(W, g):
    """Offline weight preparation: rotate the fp32 rows of W [N, K] with the
    blockwise Hadamard, quantise each row, pack.

    Returns a dict with packed [N, K/2] int8, scales float32 [N], the codes
    and the pre-rounding values.
    """
    W = np.asarray(W, dtype=np.float32)
    _, r = rotate_rows(W, g)
    q, s, v = quantize_rows(r)
    return {"packed": pack_int4(q), "scale": s, "q": q, "v": v, "r": r}


def quantize_activation(x_bits, g, act=0):
    """Run-time activation preparation from bf16 rows x [M, K]: optional exact
    GELU (act=1), blockwise Hadamard rotation, per-row quantisation, pack."""
    xf = bf16_bits_to_f32(x_bits)
    if act == 1:
        xf = gelu_f32(xf)
    elif act != 0:
        raise ValueError("act must be 0 (none) or 1 (gelu)")
    _, r = rotate_rows(xf, g)
    q, s, v = quantize_rows(r)
    return {"packed": pack_int4(q), "scale": s, "q": q, "v": v, "r": r}


# ---------------------------------------------------------------------------
# Integer GEMM and the rank-one epilogue.
# ---------------------------------------------------------------------------


def gemm_s32(xq_packed, wq_packed):
    """acc[m, n] = sum_k qx[m, k] * qw[n, k] over the unpacked int4 codes.

    The product runs as a float64 matrix product of small integers, which is
    exact while |acc| < 2^53; the page bounds |acc| by 49*K, far below that
    and below 2^31, and both bounds are asserted.
    """
    a = unpack_int4(xq_packed).astype(np.float64)
    b = unpack_int4(wq_packed).astype(np.float64)
    if a.shape[1] != b.shape[1]:
        raise ValueError("inner dimensions differ")
    acc = np.rint(a @ b.T).astype(np.int64)
    K = a.shape[1]
    if acc.size and np.max(np.abs(acc)) > 49 * K:
        raise AssertionError("accumulator exceeds the 49*K bound")
    assert 49 * K < 2 ** 31
    return acc.astype(np.int32)


def epilogue(acc, sx, sw, bias_bits=None):
    """Rank-one dequantisation: y = float(acc) * sx[m] * sw[n] (+ bias[n]),
    each step a separately rounded float32 operation in that order, then one
    round-to-nearest-even to bf16.

    Returns (y as float32 before the bf16 rounding, y as bf16 bits).
    """
    t = np.asarray(acc, dtype=np.int64).astype(np.float32)
    t = (t * np.asarray(sx, dtype=np.float32)[:, None]).astype(np.float32)
    t = (t * np.asarray(sw, dtype=np.float32)[None, :]).astype(np.float32)
    if bias_bits is not None:
        t = (t + bf16_bits_to_f32(bias_bits)[None, :]).astype(np.float32)
    return t, f32_to_bf16_bits(t)


def linear(x_bits, wq_packed, sw, bias_bits, g, act=0):
    """The whole layer: quantise the activation, integer GEMM, epilogue."""
    xa = quantize_activation(x_bits, g, act)
    acc = gemm_s32(xa["packed"], wq_packed)
    y32, ybits = epilogue(acc, xa["scale"], sw, bias_bits)
    return {"xq": xa["packed"], "sx": xa["scale"], "v": xa["v"],
            "acc": acc, "y32": y32, "y_bits": ybits}


# ---------------------------------------------------------------------------
# Dynamic LoRA.  Page "Comfy-INT4-HIPtest README", section "LoRA modes": the
# Dynamic mode keeps the LoRA matrices separate and applies their deltas at
# inference time.  Page "ComfyUI-INT4-Fast" (features list, "Dynamic LoRA
# Patching"): the LoRA down projection is rotated with the same Hadamard
# transform as the layer, so that it stays coherent with the rotated basis.
# ---------------------------------------------------------------------------


def lora_delta(x_bits, A, B, g, scale, act=0):
    """The LoRA delta of one layer in the rotated basis, in float64:
    t = x_rot A_rot^T (the rotated activation against the rotated down
    projection A [r, K]), delta = scale * t B^T (B [N, r], the up
    projection).  x_rot and A_rot are the rows rotated blockwise exactly as
    the layer rotates them (u / sqrt(g), not rounded); the activation is the
    layer's input, i.e. GELU(x) when act = 1.

    Returns (t [M, r], delta [M, N]), both float64."""
    xf = bf16_bits_to_f32(x_bits)
    if act == 1:
        xf = gelu_f32(xf)
    elif act != 0:
        raise ValueError("act must be 0 (none) or 1 (gelu)")
    sg = np.sqrt(np.float64(g))
    ux, _ = rotate_rows(xf.astype(np.float64), g)
    ua, _ = rotate_rows(np.asarray(A, dtype=np.float64), g)
    t = (ux / sg) @ (ua / sg).T
    delta = np.float64(scale) * (t @ np.asarray(B, dtype=np.float64).T)
    return t, delta


def linear_lora(x_bits, wq_packed, sw, bias_bits, g, A, B, scale, act=0):
    """The layer with a dynamic LoRA: the W4A4 layer's fp32 output (the
    rank-one epilogue of `linear`) plus the fp32-rounded delta, then one
    round-to-nearest-even to bf16."""
    base = linear(x_bits, wq_packed, sw, bias_bits, g, act)
    t, delta = lora_delta(x_bits, A, B, g, scale, act)
    y32 = (base["y32"] + delta.astype(np.float32)).astype(np.float32)
    out = dict(base)
    out.update({"t": t, "delta": delta, "base_y32": base["y32"], "y32": y32, "y_bits": f32_to_bf16_bits(y32)})
    return out


# ---------------------------------------------------------------------------
# Layer chains.  The down layer of an MLP quantises GELU of the up layer's
# bf16 output (the pages' activation pass -- page "[PR #63] int4_tensorwise:
# W4A4 layout (+ConvRot) with fused CUDA kernels", Description: rotate, then
# one int4 scale per row -- applied to that output).  A requantising epilogue
# splits it in two: the producing layer's column tiles each report, per row,
# the amax of the rotated values in their columns; the row scale is the max
# of those over the row, divided by 7, and the codes follow from it.
# ---------------------------------------------------------------------------


def requant_partials(y_bits, g, block_cols, act=1):
    """Per-row amax of the rotated next-layer activation r = rotate(GELU(y))
    (GELU only for act = 1) over each block of `block_cols` consecutive
    columns (a multiple of g, so that no rotation group straddles blocks;
    the last block may be narrower).  float32 [R, ceil(K / block_cols)]."""
    if block_cols % g != 0:
        raise ValueError("column blocks must hold whole rotation groups")
    xf = bf16_bits_to_f32(y_bits)
    if act == 1:
        xf = gelu_f32(xf)
    elif act != 0:
        raise ValueError("act must be 0 (none) or 1 (gelu)")
    _, r = rotate_rows(xf, g)
    R, K = r.shape
    nb = -(-K // block_cols)
    out = np.zeros((R, nb), dtype=np.float32)
    for b in range(nb):
        out[:, b] = np.max(np.abs(r[:, b * block_cols:(b + 1) * block_cols]), axis=1)
    return out


def chain_requant(y_bits, g, block_cols, act=1):
    """The next layer's packed codes and row scales from the producing
    layer's bf16 output, by the two passes: the row amax as the max of the
    block partials, s = amax / 7 (float32), codes = quantise(r / s).  Equal
    to quantize_activation(y_bits, g, act) by construction (the max of the
    block maxima is the row maximum); returned with the partials."""
    parts = requant_partials(y_bits, g, block_cols, act)
    amax = np.max(parts, axis=1).astype(np.float32)
    out = dict(quantize_activation(y_bits, g, act))
    out["partials"] = parts
    out["amax"] = amax
    out["scale_from_partials"] = (amax / np.float32(7.0)).astype(np.float32)
    return out
