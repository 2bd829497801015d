"""Pins for the CPU oracle: each check compares it with something other than
itself -- a library routine, a closed form, brute force, or a hand-derived
fixture -- so that a dropped term, a wrong sign or index, a swapped nibble or a
transposed operand in the oracle fails at least one of them."""

import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as orc
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Hadamard matrix and the blockwise rotation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("g", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_is_orthogonal(g):
    H = orc.sylvester_hadamard(g)
    assert np.array_equal(H @ H.T, g * np.eye(g, dtype=np.int64))
    assert np.array_equal(H, H.T)


@pytest.mark.parametrize("g", [2, 4, 16, 64, 128, 256])
def test_hadamard_matches_scipy_and_recursion(g):
    H = orc.sylvester_hadamard(g)
    assert np.array_equal(H, scipy.linalg.hadamard(g))
    # independent recursive construction H_2n = [[H, H], [H, -H]]
    R = np.array([[1]], dtype=np.int64)
    while R.shape[0] < g:
        R = np.block([[R, R], [R, -R]])
    assert np.array_equal(H, R)


def _fwht_python(v):
    """In-place radix-2 butterflies written out in pure Python."""
    a = list(v)
    h = 1
    while h < len(a):
        for i in range(0, len(a), 2 * h):
            for j in range(i, i + h):
                x, y = a[j], a[j + h]
                a[j], a[j + h] = x + y, x - y
        h *= 2
    return a


@pytest.mark.parametrize("g", [4, 8, 64])
def test_rotation_matches_bruteforce_fwht(g):
    rng = np.random.default_rng(5)
    X = rng.integers(-9, 10, size=(3, 2 * g)).astype(np.float64)
    u, r = orc.rotate_rows(X, g)
    for m in range(3):
        for b in range(2):
            want = _fwht_python(X[m, b * g:(b + 1) * g].tolist())
            assert u[m, b * g:(b + 1) * g].tolist() == want
    assert np.array_equal(r, (u / math.sqrt(g)).astype(np.float32))


@pytest.mark.parametrize("g", [64, 128, 256])
def test_rotation_preserves_the_product(g):
    # (x R)(W R)^T = x W^T for the orthogonal blockwise R = diag(H/sqrt(g))
    rng = np.random.default_rng(7)
    K = 2 * g
    x = rng.standard_normal((5, K))
    W = rng.standard_normal((3, K))
    ux, _ = orc.rotate_rows(x, g)
    uw, _ = orc.rotate_rows(W, g)
    lhs = (ux / math.sqrt(g)) @ (uw / math.sqrt(g)).T
    rhs = x @ W.T
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(rhs)) * K


def test_rotation_is_an_involution():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 256))
    u1, _ = orc.rotate_rows(x, 128)
    u2, _ = orc.rotate_rows(u1 / math.sqrt(128), 128)
    assert np.allclose(u2 / math.sqrt(128), x, rtol=0, atol=1e-13)


def test_rotation_groups_are_contiguous_and_independent():
    # a spike in group 1 must only touch group 1, spread as +-1/sqrt(g)
    g = 64
    x = np.zeros((1, 3 * g))
    x[0, g + 5] = 8.0
    _, r = orc.rotate_rows(x, g)
    assert np.all(r[0, :g] == 0) and np.all(r[0, 2 * g:] == 0)
    assert np.all(np.abs(r[0, g:2 * g]) == np.float32(1.0))


# --------------------------------------------------------------------------
# bf16 conversions
# --------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    # exact ties: low 16 bits = 0x8000 with even and odd kept parts
    ties = (np.arange(1000, dtype=np.uint32) << np.uint32(16) | np.uint32(0x8000)).view(np.float32)
    v = np.concatenate([v, ties, -ties, np.float32([0.0, -0.0, 1e-40, np.inf, -np.inf])])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.f32_to_bf16_bits(v)
    assert np.array_equal(got, want)
    back = orc.bf16_bits_to_f32(want)
    assert np.array_equal(back, torch.from_numpy(want.view(np.int16)).view(torch.bfloat16).float().numpy())


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------

def test_pack_hand_vector():
    # (q0, q1) = (1, -2): low nibble 0x1, high nibble 0xE
    p = orc.pack_int4(np.array([[1, -2]], dtype=np.int8))
    assert p.view(np.uint8)[0, 0] == 0xE1
    assert orc.unpack_int4(p).tolist() == [[1, -2]]


def test_pack_roundtrip_exhaustive():
    allbytes = np.arange(256, dtype=np.uint8).view(np.int8).reshape(1, 256)
    q = orc.unpack_int4(allbytes)
    assert q.min() == -8 and q.max() == 7
    assert np.array_equal(orc.pack_int4(q), allbytes)
    # every in-range pair survives pack/unpack; unpacking follows the
    # arithmetic-shift definition of a signed nibble
    pairs = np.array([(a, b) for a in range(-7, 8) for b in range(-7, 8)], dtype=np.int8)
    assert len(pairs) == 225
    q2 = orc.unpack_int4(orc.pack_int4(pairs.reshape(1, -1))).reshape(-1, 2)
    assert np.array_equal(q2, pairs)
    for byte in range(256):
        s8 = byte - 256 if byte >= 128 else byte
        lo = ((byte & 0xF) ^ 8) - 8
        hi = s8 >> 4
        assert q[0, 2 * byte] == lo and q[0, 2 * byte + 1] == hi


# --------------------------------------------------------------------------
# Quantiser
# --------------------------------------------------------------------------

def _read_golden_ties():
    cases, g, cur = [], None, None
    with open(os.path.join(GOLDEN, "quant_ties_g64.txt")) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "g":
                g = int(vals[0])
            elif key == "case":
                cur = {"name": vals[0]}
            elif key == "r":
                cur["r"] = [float(v) for v in vals]
            elif key == "scale":
                cur["scale"] = float(vals[0])
            elif key == "q":
                cur["q"] = [int(v) for v in vals]
            elif key == "packed":
                cur["packed"] = [int(v, 16) for v in vals]
            elif key == "end":
                cases.append(cur)
    return g, cases


def test_quantiser_golden_ties():
    g, cases = _read_golden_ties()
    assert g == 64 and len(cases) == 2
    Hs = scipy.linalg.hadamard(g).astype(np.float64) / 8.0
    for c in cases:
        r = np.zeros(g)
        r[:len(c["r"])] = c["r"]
        x = Hs @ r
        xb = orc.f32_to_bf16_bits(x.astype(np.float32))
        assert np.array_equal(orc.bf16_bits_to_f32(xb).astype(np.float64), x), "fixture x not exact in bf16"
        out = orc.quantize_activation(xb.reshape(1, g), g)
        assert out["scale"][0] == np.float32(c["scale"])
        q = np.zeros(g, dtype=np.int8)
        q[:len(c["q"])] = c["q"]
        assert np.array_equal(out["q"][0], q), c["name"]
        pk = np.zeros(g // 2, dtype=np.uint8)
        pk[:len(c["packed"])] = c["packed"]
        assert np.array_equal(out["packed"][0].view(np.uint8), pk), c["name"]


def test_quantiser_invariants_random():
    x, w, _ = workloads.Linear("t", M=64, K=512, N=32, g=128, seed=11).make()
    for rows, g in ((workloads.bf16_bits(x), 128), (None, 64)):
        if rows is None:
            out = orc.quantize_weight(w.numpy(), g)
        else:
            out = orc.quantize_activation(rows, g)
        q, s, r = out["q"], out["scale"], out["r"]
        assert np.abs(q).max() <= 7
        amax = np.abs(r).max(axis=1)
        assert np.array_equal(s, (amax / np.float32(7)).astype(np.float32))
        arg = np.abs(r).argmax(axis=1)
        assert np.all(np.abs(q[np.arange(len(q)), arg]) == 7)
        err = np.abs(r.astype(np.float64) - q * s[:, None].astype(np.float64))
        assert np.all(err <= s[:, None] * 0.5 * (1 + 1e-6))
        # sign is preserved wherever the code is nonzero
        assert np.all(np.sign(q[q != 0]) == np.sign(r[q != 0]))


def test_quantiser_zero_row_and_scale_invariance():
    x = np.zeros((2, 128), dtype=np.float32)
    x[1, 3] = 5.0
    q, s, _ = orc.quantize_rows(x)
    assert s[0] == 0 and np.all(q[0] == 0)
    # codes are invariant to scaling a row by a power of two
    rng = np.random.default_rng(3)
    r = rng.standard_normal((4, 256)).astype(np.float32)
    q1, s1, _ = orc.quantize_rows(r)
    q2, s2, _ = orc.quantize_rows(r * np.float32(8))
    assert np.array_equal(q1, q2) and np.array_equal(s2, s1 * 8)


def test_boundary_window():
    v = np.array([0.5, 2.5000001, 2.51, -3.5, 3.0, 6.4999], dtype=np.float32)
    got = orc.boundary_window(v)
    assert got.tolist() == [True, True, False, True, False, False]


# --------------------------------------------------------------------------
# Integer GEMM
# --------------------------------------------------------------------------

def test_gemm_bruteforce_small():
    rng = np.random.default_rng(4)
    for (M, N, K) in ((1, 1, 2), (3, 5, 8), (7, 2, 64), (16, 9, 30)):
        qa = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
        qb = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
        acc = orc.gemm_s32(orc.pack_int4(qa), orc.pack_int4(qb))
        for m in range(M):
            for n in range(N):
                want = 0
                for k in range(K):
                    want += int(qa[m, k]) * int(qb[n, k])
                assert acc[m, n] == want


def test_gemm_extremes_reach_the_bound():
    K = 12288
    seven = np.full((2, K), 7, dtype=np.int8)
    acc = orc.gemm_s32(orc.pack_int4(seven), orc.pack_int4(np.stack([seven[0], -seven[0]])))
    assert acc[0, 0] == 49 * K and acc[0, 1] == -49 * K


# --------------------------------------------------------------------------
# Epilogue
# --------------------------------------------------------------------------

def test_epilogue_identity_is_bf16_of_acc():
    acc = np.arange(-256, 257, dtype=np.int32).reshape(1, -1)
    y32, yb = orc.epilogue(acc, np.ones(1, np.float32), np.ones(acc.shape[1], np.float32))
    want = torch.from_numpy(acc.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(yb, want)
    assert np.array_equal(y32, acc.astype(np.float32))


def test_epilogue_closed_form():
    rng = np.random.default_rng(9)
    acc = rng.integers(-50000, 50000, size=(6, 10)).astype(np.int32)
    sx = rng.uniform(0.01, 2, 6).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, 10).astype(np.float32)
    bias = orc.f32_to_bf16_bits(rng.standard_normal(10).astype(np.float32) * 0.01)
    y32, yb = orc.epilogue(acc, sx, sw, bias)
    exact = (acc.astype(np.float64) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
             + orc.bf16_bits_to_f32(bias)[None, :].astype(np.float64))
    assert np.all(np.abs(y32 - exact) <= 4 * np.spacing(np.abs(exact).astype(np.float32)) + 1e-12)
    # one round-to-nearest-even to bf16: within half a bf16 ulp of y32
    yf = orc.bf16_bits_to_f32(yb).astype(np.float64)
    ulp = np.abs(y32).astype(np.float64) * 2.0 ** -7
    assert np.all(np.abs(yf - y32) <= 0.5 * ulp * (1 + 1e-9) + 1e-30)


# --------------------------------------------------------------------------
# GELU
# --------------------------------------------------------------------------

def test_gelu_matches_math_erf_and_torch():
    vals = np.array([-6.0, -3.0, -1.0, -0.5, -1e-3, 0.0, 1e-3, 0.5, 1.0, 2.5, 7.0], dtype=np.float32)
    got = orc.gelu_f32(vals)
    for v, gv in zip(vals.tolist(), got.tolist()):
        want = 0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0)))
        assert abs(gv - want) <= 1e-7 * max(abs(want), 1e-30) + 1e-45
    t = torch.nn.functional.gelu(torch.from_numpy(vals).double(), approximate="none").float().numpy()
    assert np.array_equal(got, t)


def test_gelu_saturates_at_both_ends():
    """GELU(t) = t Phi(t): for large positive t Phi rounds to 1 and the value
    is t itself; for large negative t it underflows to -0, up to the largest
    bf16 magnitudes (3.39e38)."""
    pos = np.array([16.0, 1e3, 1e30, 3.3895e38], dtype=np.float32)
    assert np.array_equal(orc.gelu_f32(pos), pos)
    neg = orc.gelu_f32(-pos)
    assert np.all(neg == 0.0) and np.all(np.signbit(neg))


@pytest.mark.parametrize("t", [1.0, -1.0, 2.5])
def test_activation_with_gelu_applies_gelu_before_the_rotation(t):
    """A one-hot row (t in column 0, g = 64): GELU first turns t into
    G = GELU(t), and the rotation then spreads G / 8 over the 64 outputs of
    the first group (every entry of the first Hadamard column is +1, and
    1/sqrt(64) = 1/8 is exact), so sx = fl(fl(G / 8) / 7) and the first
    group's codes are all 7 * sign(G).  Rotating first would give
    GELU(t / 8) instead: a different scale."""
    G = np.float32(0.5 * t * (1.0 + math.erf(t / math.sqrt(2.0))))
    want_s = np.float32(np.float32(G / np.float32(8.0)) / np.float32(7.0))
    xb = np.zeros((1, 128), dtype=np.uint16)
    xb[0, 0] = orc.f32_to_bf16_bits(np.array([t], dtype=np.float32))[0]
    out = orc.quantize_activation(xb, 64, act=1)
    assert out["scale"][0] == abs(want_s)
    q = out["q"][0]
    assert np.all(q[:64] == 7 * int(np.sign(G))) and np.all(q[64:] == 0)
    # the other order is measurably different
    other = np.float32(0.5 * (t / 8) * (1.0 + math.erf((t / 8) / math.sqrt(2.0))))
    assert abs(np.float32(other / np.float32(7.0)) - abs(want_s)) > 1e-3 * abs(want_s)


def test_activation_with_gelu_two_hot_row():
    """Two inputs a, b in the columns 0 and 1 of a 64-group: after GELU the
    rotation gives G(a) + G(b) on even outputs and G(a) - G(b) on odd ones
    (Hadamard columns 0 and 1), divided by 8."""
    a, b = 1.5, -0.75
    Ga = 0.5 * a * (1.0 + math.erf(a / math.sqrt(2.0)))
    Gb = 0.5 * b * (1.0 + math.erf(b / math.sqrt(2.0)))
    xb = np.zeros((1, 64), dtype=np.uint16)
    xb[0, :2] = orc.f32_to_bf16_bits(np.array([a, b], dtype=np.float32))
    out = orc.quantize_activation(xb, 64, act=1)
    Ga32, Gb32 = np.float64(np.float32(Ga)), np.float64(np.float32(Gb))
    even, odd = (Ga32 + Gb32) / 8, (Ga32 - Gb32) / 8
    assert np.allclose(out["r"][0, 0::2], even, rtol=1e-7, atol=0)
    assert np.allclose(out["r"][0, 1::2], odd, rtol=1e-7, atol=0)
    assert out["scale"][0] == np.float32(np.float32(max(abs(even), abs(odd))) / np.float32(7.0))


# --------------------------------------------------------------------------
# The whole layer
# --------------------------------------------------------------------------

def test_linear_tiny_against_full_precision_and_rotation_helps():
    """Information plus a sanity claim of the pages: on inputs with outlier
    channels the rotated W4A4 layer is closer to the full-precision product
    than per-row int4 without the rotation."""
    cfg = workloads.TINY
    x, w, _ = cfg.make()
    xb = workloads.bf16_bits(x)
    wq = orc.quantize_weight(w.numpy(), cfg.g)
    out = orc.linear(xb, wq["packed"], wq["scale"], None, cfg.g)
    ref = orc.bf16_bits_to_f32(xb).astype(np.float64) @ w.numpy().astype(np.float64).T
    rot_err = np.linalg.norm(out["y32"] - ref) / np.linalg.norm(ref)
    # the same layer with the rotation switched off (g = 1 makes H = [1])
    wq1 = orc.quantize_weight(w.numpy(), 1)
    out1 = orc.linear(xb, wq1["packed"], wq1["scale"], None, 1)
    plain_err = np.linalg.norm(out1["y32"] - ref) / np.linalg.norm(ref)
    assert rot_err < plain_err
    assert rot_err < 0.3


def test_linear_zero_activation_gives_bias():
    xb = np.zeros((3, 128), dtype=np.uint16)
    w = workloads.make_weight(8, 128, 0).numpy()
    wq = orc.quantize_weight(w, 64)
    bias = workloads.bf16_bits(workloads.make_bias(8, 0))
    out = orc.linear(xb, wq["packed"], wq["scale"], bias, 64)
    assert np.array_equal(out["y_bits"], np.broadcast_to(bias, (3, 8)))


# --------------------------------------------------------------------------
# Dynamic LoRA
# --------------------------------------------------------------------------

def _lora_case(M=5, K=256, N=24, r=8, g=64, seed=3):
    gen = np.random.default_rng(seed)
    x = workloads.make_activation(M, K, seed=seed, outlier_frac=0.02, outlier_scale=10.0)
    A = gen.standard_normal((r, K)).astype(np.float32) * 0.05
    B = gen.standard_normal((N, r)).astype(np.float32) * 0.05
    return workloads.bf16_bits(x), A, B


@pytest.mark.parametrize("g", [64, 128, 256])
def test_lora_rotated_delta_equals_the_unrotated_one(g):
    """(H/sqrt(g))^2 = I: the rotated activation against the rotated down
    projection gives x A^T, so the rotated delta equals the plain LoRA delta
    (float64, 1e-12).  Rotating A with another group size, or not at all,
    breaks this."""
    xb, A, B = _lora_case(K=512, g=g)
    t, delta = orc.lora_delta(xb, A, B, g, 0.75)
    x = orc.bf16_bits_to_f32(xb).astype(np.float64)
    t_plain = x @ A.astype(np.float64).T
    assert np.allclose(t, t_plain, rtol=1e-12, atol=1e-12 * np.abs(t_plain).max())
    d_plain = 0.75 * t_plain @ B.astype(np.float64).T
    assert np.allclose(delta, d_plain, rtol=1e-12, atol=1e-12 * np.abs(d_plain).max())
    # a down projection rotated with the wrong group size is not coherent
    _, ua = orc.rotate_rows(A.astype(np.float64), g // 2)
    ux, _ = orc.rotate_rows(x, g)
    wrong = (ux / np.sqrt(g)) @ (ua / np.sqrt(g // 2)).T
    assert not np.allclose(wrong, t_plain, rtol=1e-3)


def test_lora_delta_brute_force():
    """Tiny case written out with explicit Hadamard sums in Python."""
    xb, A, B = _lora_case(M=2, K=128, N=3, r=2, g=64, seed=9)
    t, delta = orc.lora_delta(xb, A, B, 64, 2.0)
    x = orc.bf16_bits_to_f32(xb).astype(np.float64)
    H = scipy.linalg.hadamard(64)

    def rot(v):
        out = []
        for b0 in range(0, len(v), 64):
            for i in range(64):
                out.append(sum(H[i][j] * float(v[b0 + j]) for j in range(64)) / 8.0)
        return out

    for m in range(2):
        xr = rot(x[m])
        for j in range(2):
            ar = rot(A[j].astype(np.float64))
            assert abs(t[m, j] - sum(a * b for a, b in zip(xr, ar))) <= 1e-12 * max(1.0, abs(t[m, j]))
        for n in range(3):
            want = 2.0 * sum(t[m, j] * float(B[n, j]) for j in range(2))
            assert abs(delta[m, n] - want) <= 1e-12 * max(1.0, abs(want))


def test_lora_zero_update_gives_the_base_layer():
    xb, A, B = _lora_case()
    w = workloads.make_weight(24, 256, 0).numpy()
    wq = orc.quantize_weight(w, 64)
    bias = workloads.bf16_bits(workloads.make_bias(24, 0))
    base = orc.linear(xb, wq["packed"], wq["scale"], bias, 64)
    for Bz, s in ((np.zeros_like(B), 1.0), (B, 0.0)):
        out = orc.linear_lora(xb, wq["packed"], wq["scale"], bias, 64, A, Bz, s)
        assert np.array_equal(out["y_bits"], base["y_bits"])
    out = orc.linear_lora(xb, wq["packed"], wq["scale"], bias, 64, A, B, 1.0)
    assert not np.array_equal(out["y_bits"], base["y_bits"])
    assert np.array_equal(out["y32"], (base["y32"] + out["delta"].astype(np.float32)).astype(np.float32))


def test_lora_with_gelu_input_uses_gelu_of_x():
    xb, A, B = _lora_case()
    t1, _ = orc.lora_delta(xb, A, B, 64, 1.0, act=1)
    xg = orc.gelu_f32(orc.bf16_bits_to_f32(xb)).astype(np.float64)
    assert np.allclose(t1, xg @ A.astype(np.float64).T, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# Layer chains: the requantising epilogue's two passes
# --------------------------------------------------------------------------

def test_requant_partials_hand_case():
    """One nonzero input t per row, in different column blocks: after GELU
    the rotation spreads G = GELU(t) over its 128-group as +-G / sqrt(128),
    so that block's partial is fl(|G| / sqrt(128)) (the oracle rounds the
    float64 sum u / sqrt(g) once), every other block's partial is 0, and the
    row scale from the partials is that value / 7."""
    g, bc, K = 128, 256, 768
    ts = [1.25, -0.5, 3.0]
    xb = np.zeros((3, K), dtype=np.uint16)
    for i, (t, col) in enumerate(zip(ts, [5, 300, 767])):
        xb[i, col] = orc.f32_to_bf16_bits(np.array([t], dtype=np.float32))[0]
    parts = orc.requant_partials(xb, g, bc, act=1)
    assert parts.shape == (3, 3)
    for i, (t, col) in enumerate(zip(ts, [5, 300, 767])):
        G = np.float64(np.float32(0.5 * t * (1.0 + math.erf(t / math.sqrt(2.0)))))
        want = np.float32(abs(G) / math.sqrt(128.0))
        for b in range(3):
            assert parts[i, b] == (want if b == col // bc else 0.0)
    out = orc.chain_requant(xb, g, bc, act=1)
    assert np.array_equal(out["scale_from_partials"], out["scale"])


def test_requant_partials_brute_force():
    """Small random rows: every partial equals a loop over the block's
    groups with scipy's dense Hadamard matrix and math.erf per element."""
    import scipy.linalg
    rng = np.random.default_rng(5)
    g, bc, K, R = 64, 192, 448, 4     # the last block is 64 wide
    x = (rng.standard_normal((R, K)) * 2).astype(np.float32)
    xb = orc.f32_to_bf16_bits(x)
    xf = orc.bf16_bits_to_f32(xb).astype(np.float64)
    H = scipy.linalg.hadamard(g).astype(np.float64)
    parts = orc.requant_partials(xb, g, bc, act=1)
    assert parts.shape == (R, 3)
    for m in range(R):
        z = np.array([np.float32(0.5 * v * (1.0 + math.erf(v / math.sqrt(2.0)))) for v in xf[m]], dtype=np.float64)
        for b in range(3):
            best = 0.0
            for k0 in range(b * bc, min(K, (b + 1) * bc), g):
                r = (H @ z[k0:k0 + g]) / math.sqrt(g)
                best = max(best, float(np.max(np.abs(r.astype(np.float32)))))
            assert abs(parts[m, b] - best) <= 2e-7 * best


@pytest.mark.parametrize("g,bc", [(64, 256), (128, 256), (256, 256), (128, 384)])
def test_chain_requant_equals_the_layer_quantiser(g, bc):
    """The two passes give exactly the one-pass quantisation of GELU(y):
    the max of the block partials is the row amax, so the scales (and with
    them the codes) agree bit for bit; and dropping a block's partial (a
    tile that did not report) changes the scale of the rows whose maximum
    sits in it."""
    rng = np.random.default_rng(g + bc)
    K = 1536
    y = (rng.standard_normal((6, K)) * rng.uniform(0.2, 4.0, size=(6, 1))).astype(np.float32)
    yb = orc.f32_to_bf16_bits(y)
    out = orc.chain_requant(yb, g, bc, act=1)
    assert np.array_equal(out["scale_from_partials"], out["scale"])
    one = orc.quantize_activation(yb, g, act=1)
    assert np.array_equal(out["packed"], one["packed"]) and np.array_equal(out["scale"], one["scale"])
    arg = np.argmax(out["partials"], axis=1)
    dropped = out["partials"].copy()
    dropped[np.arange(6), arg] = 0.0
    assert np.all(np.max(dropped, axis=1) < out["amax"])
