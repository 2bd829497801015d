"""Host-only checks of the C ABI: the library loads, exports every symbol
the header declares, and rejects invalid arguments before touching a GPU."""

import ctypes
import os
import re

import pytest

import w4a4_hadamard_rotated_b200 as w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a4.h")

NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(1 << 20)          # never dereferenced: every call below fails validation first
MISALIGNED = ctypes.c_void_p((1 << 20) + 2)


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(w4a4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return w4.load_library()


def test_every_declared_symbol_is_exported_and_bound(lib):
    syms = declared_symbols()
    assert len(syms) >= 10
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) == set(w4.SIGNATURES), "binding and header disagree"


def test_status_strings(lib):
    for code, name in w4.STATUS_NAMES.items():
        assert lib.w4a4_status_string(code).decode().startswith(name)
    assert b"unknown" in lib.w4a4_status_string(99)
    assert lib.w4a4_version() >= 100


def test_quantize_activation_rejects_bad_arguments(lib):
    q = lib.w4a4_quantize_activation
    assert q(NULL, 4, 256, 256, 128, 0, FAKE, FAKE, NULL) == 1            # null x
    assert q(FAKE, 4, 256, 256, 96, 0, FAKE, FAKE, NULL) == 3             # bad g
    assert q(FAKE, 4, 384, 384, 256, 0, FAKE, FAKE, NULL) == 3            # g does not divide K
    assert q(FAKE, 4, 200, 200, 64, 0, FAKE, FAKE, NULL) == 2             # K % 128
    assert q(FAKE, 4, 256, 128, 128, 0, FAKE, FAKE, NULL) == 2            # ldx < K
    assert q(FAKE, -1, 256, 256, 128, 0, FAKE, FAKE, NULL) == 2           # M < 0
    assert q(FAKE, 4, 256, 256, 128, 2, FAKE, FAKE, NULL) == 9            # act
    assert q(MISALIGNED, 4, 256, 256, 128, 0, FAKE, FAKE, NULL) == 4      # x alignment
    assert q(FAKE, 4, 256, 260, 128, 0, FAKE, FAKE, NULL) == 4            # ldx % 8
    assert q(FAKE, 4, 49152 + 128, 49280, 128, 0, FAKE, FAKE, NULL) == 2  # K too large


def test_quantize_weight_rejects_bad_arguments(lib):
    q = lib.w4a4_quantize_weight
    assert q(FAKE, 8, 256, 256, 128, NULL, FAKE, NULL) == 1
    assert q(FAKE, 0, 256, 256, 128, FAKE, FAKE, NULL) == 2
    assert q(FAKE, 8, 256, 254, 128, FAKE, FAKE, NULL) == 2
    assert q(FAKE, 8, 256, 258, 128, FAKE, FAKE, NULL) == 4


def test_linear_rejects_bad_arguments(lib):
    f = lib.w4a4_linear
    args = lambda **kw: [kw.get(k, v) for k, v in (
        ("xq", FAKE), ("sx", FAKE), ("wq", FAKE), ("sw", FAKE), ("bias", NULL), ("y", FAKE),
        ("M", 128), ("N", 256), ("K", 256), ("ldy", 256), ("ws", NULL), ("wsb", 0), ("st", NULL))]
    assert f(*args(xq=NULL)) == 1
    assert f(*args(sw=NULL)) == 1
    assert f(*args(N=12)) == 2              # N % 8
    assert f(*args(K=48)) == 2              # K % 32
    assert f(*args(K=0)) == 2
    assert f(*args(M=-3)) == 2
    assert f(*args(ldy=128)) == 2           # ldy < N
    assert f(*args(ldy=260)) == 4           # ldy % 8
    assert f(*args(y=MISALIGNED)) == 4
    assert f(*args(bias=MISALIGNED)) == 4


def test_fused_rejects_bad_arguments(lib):
    f = lib.w4a4_linear_fused
    base = dict(x=FAKE, ldx=256, wq=FAKE, sw=FAKE, bias=NULL, y=FAKE, ldy=256, M=100, N=256, K=256,
                g=128, act=0, ws=NULL, wsb=0, st=NULL)
    call = lambda **kw: f(*({**base, **kw}).values())
    assert call(x=NULL) == 1
    assert call(g=32) == 3
    assert call(K=320) == 2
    assert call(act=5) == 9
    assert call(ldx=250) == 2
    # every other argument is valid: the missing workspace is what fails
    assert call() == 5


def test_gemm_s32_rejects_bad_arguments(lib):
    f = lib.w4a4_gemm_s32
    assert f(FAKE, FAKE, FAKE, 128, 256, 256, 256, 4, NULL, 0, NULL) == 9      # path
    assert f(FAKE, FAKE, FAKE, 5, 256, 256, 256, 3, NULL, 0, NULL) == 2        # tiny-M path, M > 4
    assert f(FAKE, FAKE, FAKE, 4, 256, 32768, 256, 3, NULL, 0, NULL) == 2      # tiny-M path, M*K > 96 KB
    assert f(FAKE, FAKE, FAKE, 65, 256, 256, 256, 1, NULL, 0, NULL) == 2       # small-M path, M > 64
    assert f(FAKE, FAKE, FAKE, 16, 256, 256, 254, 0, NULL, 0, NULL) == 2       # ldc < N


def test_linear_kernel_selection(lib):
    """Which GEMM kernel the linear entries run (a pure host function)."""
    f = lib.w4a4_linear_kernel
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int64] * 3
    assert f(1, 3072, 3072) == 3          # one row: CUDA-core weight streaming
    assert f(1, 3072, 13824) == 3
    assert f(2, 3072, 6144) == 3          # M * K <= 12288
    assert f(4, 12288, 3072) == 3
    assert f(4, 5120, 5120) == 1          # more work per weight byte: split-K tensor cores
    assert f(16, 12288, 3072) == 1
    assert f(64, 3072, 12288) == 1
    assert f(65, 3072, 3072) == 0         # tcgen05 GEMM
    assert f(4608, 3072, 3072) == 0


def test_workspace_sizes_are_host_functions(lib):
    # no kernel of the linear needs scratch memory
    for shape in ((0, 256, 256), (4608, 3072, 3072), (16, 3072, 3072), (64, 3072, 12288), (1, 12288, 3072)):
        assert lib.w4a4_workspace_bytes(*shape) == 0
    # the fused entry keeps the packed activation and its scales: [Xq][sx], 256-byte rounded
    assert lib.w4a4_fused_workspace_bytes(4608, 3072, 3072) == 4608 * 1536 + 4608 * 4
    assert lib.w4a4_fused_workspace_bytes(16, 3072, 3072) == 16 * 1536 + 256
    assert lib.w4a4_fused_workspace_bytes(0, 3072, 3072) == 0


def test_debug_timeout_rejects_bad_limit(lib):
    assert lib.w4a4_debug_wait_timeout(0, NULL) == 9
    assert lib.w4a4_debug_wait_timeout(10_000_000, NULL) == 9


def test_binding_refuses_host_tensors():
    """No host fallback: every compute call of the binding rejects tensors
    that are not on a CUDA device before calling the library."""
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    W = torch.zeros(8, 128, dtype=torch.float32)
    q = torch.zeros(4, 64, dtype=torch.int8)
    qw = torch.zeros(8, 64, dtype=torch.int8)
    s4, s8 = torch.ones(4), torch.ones(8)
    calls = [
        lambda: w4.quantize_weight(W),
        lambda: w4.quantize_activation(x),
        lambda: w4.linear(q, s4, qw, s8),
        lambda: w4.linear_fused(x, qw, s8),
        lambda: w4.gemm_s32(q, qw),
        lambda: w4.linear_fused_noalloc(x, qw, s8),
    ]
    for call in calls:
        with pytest.raises(TypeError, match="CUDA tensor"):
            call()


def test_missing_library_fails_loudly():
    saved = w4._lib
    try:
        w4._lib = None
        with pytest.raises(RuntimeError, match="missing"):
            w4.load_library(os.path.join(ROOT, "no_such_dir", "libw4a4.so"))
    finally:
        w4._lib = saved


def test_product_code_never_touches_the_oracle():
    """The package and the C++/CUDA sources neither import nor name the
    oracle (it is test infrastructure only)."""
    pkg = os.path.join(ROOT, "w4a4_hadamard_rotated_b200")
    for dirpath, _, names in os.walk(pkg):
        for n in names:
            if n.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, n)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), n
                assert "w4a4_oracle" not in text, n


def test_fused_noalloc_rejects_bad_arguments_and_oversized_shapes(lib):
    """The fused entry without a workspace checks its arguments like the fused
    entry, and refuses shapes whose packed activation and scales do not fit
    its fixed 8 MiB scratch, all before any CUDA call."""
    f = lib.w4a4_linear_fused_noalloc
    base = dict(x=FAKE, ldx=3072, wq=FAKE, sw=FAKE, bias=NULL, y=FAKE, ldy=3072, M=4608, N=3072, K=3072,
                g=128, act=0, st=NULL)
    call = lambda **kw: f(*({**base, **kw}).values())
    assert call(x=NULL) == 1
    assert call(wq=NULL) == 1
    assert call(g=32) == 3
    assert call(act=5) == 9
    assert call(ldx=250) == 2
    assert call(y=MISALIGNED) == 4
    # round256(M * K/2) + round256(4 M) <= 8 MiB: at K = 3072 that is M <= 5447
    assert call(M=5448) == 2
    assert call(M=4608, K=12288, ldx=12288) == 2
    assert call(M=32760, K=5120, ldx=5120, N=5120, ldy=5120) == 2


def test_quantize_activation_path_rejects_bad_arguments(lib):
    q = lib.w4a4_quantize_activation_path
    assert q(FAKE, 4, 256, 256, 128, 0, FAKE, FAKE, 3, NULL) == 9            # unknown path
    assert q(FAKE, 4, 256, 256, 128, 0, FAKE, FAKE, -1, NULL) == 9
    assert q(FAKE, 4, 256, 256, 128, 1, FAKE, FAKE, 2, NULL) == 2            # tensor cores: no GELU
    assert q(FAKE, 4, 512, 512, 256, 0, FAKE, FAKE, 2, NULL) == 2            # tensor cores: g <= 128
    assert q(FAKE, 4, 16384, 16384, 64, 0, FAKE, FAKE, 2, NULL) == 2         # tensor cores: K / g <= 128
    assert q(NULL, 4, 256, 256, 128, 0, FAKE, FAKE, 1, NULL) == 1            # the common checks still apply


def test_quantize_activation_kernel_routing(lib):
    """Which activation kernel the entries run (a pure host function): the
    register butterflies below 8192 rows and wherever the tensor-core form
    does not apply, the tensor cores from 8192 rows up."""
    f = lib.w4a4_quantize_activation_kernel
    assert f(4608, 3072, 128, 0) == 1      # the M = 4608 layers
    assert f(4608, 12288, 128, 1) == 1
    assert f(8192, 3072, 128, 0) == 2
    assert f(32760, 5120, 128, 0) == 2     # the block stack
    assert f(32760, 5120, 256, 0) == 1     # g = 256: butterflies only
    assert f(32760, 13824, 128, 1) == 1    # GELU input: butterflies only
    assert f(4608, 3000, 128, 0) == 0      # invalid shape


def test_debug_wait_limit_rejects_bad_values(lib):
    assert lib.w4a4_debug_set_wait_limit(-1) == 9
    assert lib.w4a4_debug_set_wait_limit(3_000_000_000) == 9
    assert lib.w4a4_debug_set_wait_limit(0) == 0       # the default (2 s)


def test_lora_entries_reject_bad_arguments(lib):
    f = lib.w4a4_lora_add
    base = dict(x=FAKE, ldx=256, A=FAKE, B=FAKE, r=32, scale=1.0, y=FAKE, ldy=256, M=10, N=256, K=256,
                ws=NULL, wsb=0, st=NULL)
    call = lambda **kw: f(*({**base, **kw}).values())
    assert call(A=NULL) == 1
    assert call(r=24) == 2                 # r in {16, 32, 48, 64}
    assert call(r=128) == 2
    assert call(N=100) == 2
    assert call(ldx=100) == 2
    assert call(y=MISALIGNED) == 4
    assert call(scale=float("nan")) == 9
    g = lib.w4a4_linear_fused_lora
    gb = dict(x=FAKE, ldx=256, wq=FAKE, sw=FAKE, bias=NULL, A=FAKE, B=FAKE, r=32, scale=1.0, y=FAKE, ldy=256,
              M=10, N=256, K=256, g=128, ws=NULL, wsb=0, st=NULL)
    gcall = lambda **kw: g(*({**gb, **kw}).values())
    assert gcall(B=NULL) == 1
    assert gcall(g=96) == 3
    assert gcall(r=8) == 2
    # [t: M x 64 bf16][partials: slices x M x 64 fp32]; 36 row tiles take 8 K slices
    assert lib.w4a4_lora_workspace_bytes(4608, 3072) == 4608 * 128 + 8 * 4608 * 256
    # one row tile: up to 32 slices, at least one 64-element chunk each (K = 256: 4 slices)
    assert lib.w4a4_lora_workspace_bytes(3, 256) == 512 + 4 * 3 * 256
    # 48 chunks over at most 32 slices: 2 chunks per slice, so 24 slices
    assert lib.w4a4_lora_workspace_bytes(16, 3072) == 2048 + 24 * 16 * 256
    assert lib.w4a4_fused_lora_workspace_bytes(16, 3072, 3072) == (16 * 1536 + 256) + lib.w4a4_lora_workspace_bytes(16, 3072)


def test_fused_requant_rejects_bad_arguments(lib):
    f = lib.w4a4_linear_fused_requant
    base = dict(x=FAKE, ldx=256, wq=FAKE, sw=FAKE, bias=NULL, y=FAKE, ldy=512, M=10, N=512, K=256, g=128, act=0,
                g_next=128, xq=FAKE, sx=FAKE, ws=NULL, wsb=0, st=NULL)
    call = lambda **kw: f(*({**base, **kw}).values())
    assert call(xq=NULL) == 1
    assert call(sx=NULL) == 1
    assert call(g_next=96) == 3            # the next layer's group
    assert call(N=384, ldy=384, g_next=256) == 3   # N % g_next
    assert call(N=264, ldy=264) == 2       # N is the next layer's K: a multiple of 128
    assert call(xq=MISALIGNED) == 4
    assert call(g=96) == 3                 # this layer's own arguments as for w4a4_linear_fused
    # [packed x][sx][row amax slots], each rounded up to 256 bytes
    assert lib.w4a4_fused_requant_workspace_bytes(4608, 12288, 3072) == \
        lib.w4a4_fused_workspace_bytes(4608, 12288, 3072) + 4608 * 4
    assert lib.w4a4_fused_requant_workspace_bytes(3, 256, 256) == (512 + 256) + 256
    assert lib.w4a4_fused_requant_workspace_bytes(0, 256, 256) == 0
