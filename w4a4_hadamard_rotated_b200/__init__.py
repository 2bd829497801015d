"""B200 (sm_100a) ConvRot W4A4 linear layer.

A thin Python binding over the C ABI in ``include/w4a4.h`` (``libw4a4.so``
next to this file).  The binding only marshals arguments: it checks tensor
dtypes, devices and layouts, allocates outputs with PyTorch, and passes raw
device pointers plus the current CUDA stream to the library.  Every step of
the layer runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback, and every call raises if the library is missing or not built.

Functions keep the C names without the ``w4a4_`` prefix:
  quantize_weight(W, g)                      -> (Wq [N, K/2] int8, sw [N] fp32)
  quantize_activation(x, g, act=0)           -> (Xq [M, K/2] int8, sx [M] fp32)
  linear(Xq, sx, Wq, sw, bias=None)          -> y [M, N] bf16
  linear_fused(x, Wq, sw, bias=None, g, act) -> y [M, N] bf16
  gemm_s32(Xq, Wq, path=0)                   -> acc [M, N] int32
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libw4a4.so")

OK = 0
STATUS_NAMES = {0: "W4A4_OK", 1: "W4A4_ERR_NULL", 2: "W4A4_ERR_SHAPE", 3: "W4A4_ERR_GROUP",
                4: "W4A4_ERR_ALIGN", 5: "W4A4_ERR_WORKSPACE", 6: "W4A4_ERR_DEVICE",
                7: "W4A4_ERR_CUDA", 8: "W4A4_ERR_TIMEOUT", 9: "W4A4_ERR_ARG"}

# Every symbol the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t
SIGNATURES = {
    "w4a4_status_string": (ctypes.c_char_p, [_I]),
    "w4a4_version": (_I, []),
    "w4a4_quantize_weight": (_I, [_P, _I64, _I64, _I64, _I, _P, _P, _P]),
    "w4a4_quantize_activation": (_I, [_P, _I64, _I64, _I64, _I, _I, _P, _P, _P]),
    "w4a4_quantize_activation_path": (_I, [_P, _I64, _I64, _I64, _I, _I, _P, _P, _I, _P]),
    "w4a4_quantize_activation_kernel": (_I, [_I64, _I64, _I, _I]),
    "w4a4_linear": (_I, [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "w4a4_linear_fused": (_I, [_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _P, _SZ, _P]),
    "w4a4_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "w4a4_linear_kernel": (_I, [_I64, _I64, _I64]),
    "w4a4_fused_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "w4a4_gemm_s32": (_I, [_P, _P, _P, _I64, _I64, _I64, _I64, _I, _P, _SZ, _P]),
    "w4a4_linear_fused_noalloc": (_I, [_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _P]),

    "w4a4_lora_workspace_bytes": (_SZ, [_I64, _I64]),
    "w4a4_lora_add": (_I, [_P, _I64, _P, _P, _I, ctypes.c_float, _P, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "w4a4_fused_lora_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "w4a4_linear_fused_lora": (_I, [_P, _I64, _P, _P, _P, _P, _P, _I, ctypes.c_float, _P, _I64, _I64, _I64, _I64,
                                    _I, _P, _SZ, _P]),
    "w4a4_fused_requant_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "w4a4_linear_fused_requant": (_I, [_P, _I64, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I, _I, _I, _P, _P, _P, _SZ,
                                       _P]),
    "w4a4_last_device_error": (_I, [_P]),
    "w4a4_debug_wait_timeout": (_I, [_I64, _P]),
    "w4a4_debug_set_wait_limit": (_I, [_I64]),
}

_lib = None


class W4A4Error(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        name = STATUS_NAMES.get(status, f"status {status}")
        super().__init__(f"{what}: {name}")


def load_library(path=LIB_PATH):
    """Load libw4a4.so (once) and declare its C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with __graft_entry__.build() "
                           "(or python w4a4_hadamard_rotated_b200/build.py)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(status, what):
    if status != OK:
        raise W4A4Error(status, what)


def _stream(t):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need_cuda(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _need_out(t, dtype, shape, name, device):
    """An output or operand tensor: on the same CUDA device, the given dtype
    and shape, contiguous (the library takes raw pointers and fixed strides)."""
    _need_cuda(t, dtype, name)
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need_rows(t, dtype, rows, cols, name, device):
    """A 2-D output with `rows` x `cols` and a contiguous inner dimension (its
    row stride is passed to the library)."""
    _need_cuda(t, dtype, name)
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dim() != 2 or tuple(t.shape) != (rows, cols) or t.stride(1) != 1:
        raise ValueError(f"{name} must be a [{rows}, {cols}] tensor with a contiguous inner dimension")


def _bits(t):
    """View a bf16 tensor as its raw 16-bit patterns (no copy)."""
    return t.view(torch.int16)


# Workspaces (the fused entry's packed activation and scales) are cached per
# (purpose, device, stream) and grown on demand.
_workspaces = {}


def linear_kernel(M, N, K):
    """The GEMM kernel linear() and linear_fused() run for this shape, as
    gemm_s32's path number (0 tcgen05 GEMM, 1 small-M split-K, 3 tiny-M
    CUDA-core)."""
    return int(load_library().w4a4_linear_kernel(M, N, K))


def workspace(nbytes, device, kind="linear"):
    key = (kind, device.index if device.index is not None else torch.cuda.current_device(),
           torch.cuda.current_stream(device).cuda_stream)
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
        _workspaces[key] = buf
    return buf


def quantize_weight(W, g=128):
    """Rotate + quantise fp32 weights W [N, K] -> (Wq [N, K/2] int8, sw [N] fp32)."""
    lib = load_library()
    _need_cuda(W, torch.float32, "W")
    if W.dim() != 2 or W.stride(1) != 1:
        raise ValueError("W must be a 2-D tensor with a contiguous inner dimension")
    N, K = W.shape
    Wq = torch.empty(N, K // 2, dtype=torch.int8, device=W.device)
    sw = torch.empty(N, dtype=torch.float32, device=W.device)
    _check(lib.w4a4_quantize_weight(_ptr(W), N, K, W.stride(0), g, _ptr(Wq), _ptr(sw), _stream(W)),
           "w4a4_quantize_weight")
    return Wq, sw


def quantize_activation(x, g=128, act=0, out=None, path=None):
    """Rotate + quantise bf16 activations x [M, K] -> (Xq [M, K/2] int8, sx [M] fp32).
    path: None or 0 = the library's routing, 1 = the register-butterfly
    kernel, 2 = the tensor-core kernel (w4a4_quantize_activation_path)."""
    lib = load_library()
    _need_cuda(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D tensor with a contiguous inner dimension")
    M, K = x.shape
    if out is None:
        Xq = torch.empty(M, K // 2, dtype=torch.int8, device=x.device)
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    else:
        Xq, sx = out
        _need_out(Xq, torch.int8, (M, K // 2), "Xq", x.device)
        _need_out(sx, torch.float32, (M,), "sx", x.device)
    if path is None:
        st = lib.w4a4_quantize_activation(_ptr(x), M, K, x.stride(0), g, act, _ptr(Xq), _ptr(sx), _stream(x))
    else:
        st = lib.w4a4_quantize_activation_path(_ptr(x), M, K, x.stride(0), g, act, _ptr(Xq), _ptr(sx), path,
                                               _stream(x))
    _check(st, "w4a4_quantize_activation")
    return Xq, sx


def quantize_activation_kernel(M, K, g=128, act=0):
    """Which kernel quantize_activation() runs for this shape: 1 (register
    butterflies) or 2 (tensor cores)."""
    return int(load_library().w4a4_quantize_activation_kernel(M, K, g, act))


def _check_packed_operands(Xq, Wq):
    _need_cuda(Xq, torch.int8, "Xq")
    _need_cuda(Wq, torch.int8, "Wq")
    if Xq.dim() != 2 or Wq.dim() != 2 or Xq.shape[1] != Wq.shape[1]:
        raise ValueError("Xq [M, K/2] and Wq [N, K/2] must be 2-D with the same packed width")
    if not Xq.is_contiguous() or not Wq.is_contiguous():
        raise ValueError("Xq and Wq must be contiguous (rows of K/2 bytes)")
    if Wq.device != Xq.device:
        raise ValueError("Xq and Wq must be on the same device")


def linear(Xq, sx, Wq, sw, bias=None, out=None):
    """y [M, N] bf16 from quantised operands (int32 GEMM + rank-one epilogue)."""
    lib = load_library()
    _check_packed_operands(Xq, Wq)
    M, Kh = Xq.shape
    N = Wq.shape[0]
    K = 2 * Kh
    dev = Xq.device
    _need_out(sx, torch.float32, (M,), "sx", dev)
    _need_out(sw, torch.float32, (N,), "sw", dev)
    if bias is not None:
        _need_out(bias, torch.bfloat16, (N,), "bias", dev)
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    _need_rows(y, torch.bfloat16, M, N, "out", dev)
    nbytes = lib.w4a4_workspace_bytes(M, N, K)
    ws = workspace(nbytes, Xq.device) if nbytes else None
    _check(lib.w4a4_linear(_ptr(Xq), _ptr(sx), _ptr(Wq), _ptr(sw), _ptr(bias), _ptr(y), M, N, K, y.stride(0),
                           _ptr(ws), nbytes, _stream(Xq)), "w4a4_linear")
    return y


def _check_fused_operands(x, Wq, sw, bias):
    _need_cuda(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D tensor with a contiguous inner dimension")
    M, K = x.shape
    _need_cuda(Wq, torch.int8, "Wq")
    if Wq.dim() != 2 or Wq.shape[1] * 2 != K or not Wq.is_contiguous() or Wq.device != x.device:
        raise ValueError("Wq must be a contiguous [N, K/2] int8 tensor on x's device")
    N = Wq.shape[0]
    _need_out(sw, torch.float32, (N,), "sw", x.device)
    if bias is not None:
        _need_out(bias, torch.bfloat16, (N,), "bias", x.device)
    return M, K, N


def linear_fused(x, Wq, sw, bias=None, g=128, act=0, out=None):
    """y [M, N] bf16 = the whole layer from bf16 activations x [M, K]."""
    lib = load_library()
    M, K, N = _check_fused_operands(x, Wq, sw, bias)
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _need_rows(y, torch.bfloat16, M, N, "out", x.device)
    nbytes = lib.w4a4_fused_workspace_bytes(M, N, K)
    ws = workspace(nbytes, x.device, "fused") if nbytes else None
    _check(lib.w4a4_linear_fused(_ptr(x), x.stride(0), _ptr(Wq), _ptr(sw), _ptr(bias), _ptr(y), y.stride(0),
                                 M, N, K, g, act, _ptr(ws), nbytes, _stream(x)), "w4a4_linear_fused")
    return y


def gemm_s32(Xq, Wq, path=0, out=None):
    """Raw int32 accumulators acc [M, N] (path 0: tcgen05 kernel, 1: small-M
    kernel, 2: the warp-level mma.sync comparison kernel, 3: the tiny-M
    CUDA-core kernel, M <= 4)."""
    lib = load_library()
    _check_packed_operands(Xq, Wq)
    M, Kh = Xq.shape
    N = Wq.shape[0]
    K = 2 * Kh
    acc = out if out is not None else torch.empty(M, N, dtype=torch.int32, device=Xq.device)
    _need_rows(acc, torch.int32, M, N, "out", Xq.device)
    _check(lib.w4a4_gemm_s32(_ptr(Xq), _ptr(Wq), _ptr(acc), M, N, K, acc.stride(0), path, None, 0,
                             _stream(Xq)), "w4a4_gemm_s32")
    return acc


def linear_fused_noalloc(x, Wq, sw, bias=None, g=128, act=0, out=None):
    """The fused layer without a workspace: its scratch is a fixed 8 MiB array
    inside the library (see w4a4_linear_fused_noalloc in the header; calls
    that overlap on the GPU race on it)."""
    lib = load_library()
    M, K, N = _check_fused_operands(x, Wq, sw, bias)
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _need_rows(y, torch.bfloat16, M, N, "out", x.device)
    _check(lib.w4a4_linear_fused_noalloc(_ptr(x), x.stride(0), _ptr(Wq), _ptr(sw), _ptr(bias), _ptr(y), y.stride(0),
                                         M, N, K, g, act, _stream(x)), "w4a4_linear_fused_noalloc")
    return y


def _check_lora(A, B, K, N, device):
    _need_cuda(A, torch.bfloat16, "A")
    _need_cuda(B, torch.bfloat16, "B")
    if A.dim() != 2 or A.shape[1] != K or not A.is_contiguous() or A.device != device:
        raise ValueError("A must be a contiguous [r, K] bf16 tensor on the activation's device")
    r = A.shape[0]
    if B.dim() != 2 or tuple(B.shape) != (N, r) or not B.is_contiguous() or B.device != device:
        raise ValueError("B must be a contiguous [N, r] bf16 tensor on the activation's device")
    return r


def lora_add(x, A, B, scale, y):
    """Dynamic LoRA update in place: y += scale * (x A^T) B^T (see
    w4a4_lora_add; the rotated form of the pages equals it)."""
    lib = load_library()
    _need_cuda(x, torch.bfloat16, "x")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a 2-D tensor with a contiguous inner dimension")
    M, K = x.shape
    N = y.shape[1]
    _need_rows(y, torch.bfloat16, M, N, "y", x.device)
    r = _check_lora(A, B, K, N, x.device)
    nbytes = lib.w4a4_lora_workspace_bytes(M, K)
    ws = workspace(nbytes, x.device, "lora") if nbytes else None
    _check(lib.w4a4_lora_add(_ptr(x), x.stride(0), _ptr(A), _ptr(B), r, float(scale), _ptr(y), y.stride(0),
                             M, N, K, _ptr(ws), nbytes, _stream(x)), "w4a4_lora_add")
    return y


def linear_fused_requant(x, Wq, sw, bias=None, g=128, act=0, g_next=128, out=None, xq_next=None, sx_next=None):
    """The fused layer y = layer(x) together with the next layer's quantised
    input from GELU(y) (w4a4_linear_fused_requant): returns (y [M, N] bf16,
    Xq_next [M, N/2] int8, sx_next [M] fp32)."""
    lib = load_library()
    M, K, N = _check_fused_operands(x, Wq, sw, bias)
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _need_rows(y, torch.bfloat16, M, N, "out", x.device)
    if N % 2 != 0:
        raise ValueError("N must be even")
    xq = xq_next if xq_next is not None else torch.empty(M, N // 2, dtype=torch.int8, device=x.device)
    sx = sx_next if sx_next is not None else torch.empty(M, dtype=torch.float32, device=x.device)
    _need_out(xq, torch.int8, (M, N // 2), "xq_next", x.device)
    _need_out(sx, torch.float32, (M,), "sx_next", x.device)
    nbytes = lib.w4a4_fused_requant_workspace_bytes(M, N, K)
    ws = workspace(nbytes, x.device, "fused_requant") if nbytes else None
    _check(lib.w4a4_linear_fused_requant(_ptr(x), x.stride(0), _ptr(Wq), _ptr(sw), _ptr(bias), _ptr(y), y.stride(0),
                                         M, N, K, g, act, g_next, _ptr(xq), _ptr(sx), _ptr(ws), nbytes, _stream(x)),
           "w4a4_linear_fused_requant")
    return y, xq, sx


def linear_fused_lora(x, Wq, sw, bias, A, B, scale, g=128, out=None):
    """The fused layer plus its Dynamic LoRA update (w4a4_linear_fused_lora)."""
    lib = load_library()
    M, K, N = _check_fused_operands(x, Wq, sw, bias)
    r = _check_lora(A, B, K, N, x.device)
    y = out if out is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _need_rows(y, torch.bfloat16, M, N, "out", x.device)
    nbytes = lib.w4a4_fused_lora_workspace_bytes(M, N, K)
    ws = workspace(nbytes, x.device, "fused_lora") if nbytes else None
    _check(lib.w4a4_linear_fused_lora(_ptr(x), x.stride(0), _ptr(Wq), _ptr(sw), _ptr(bias), _ptr(A), _ptr(B), r,
                                      float(scale), _ptr(y), y.stride(0), M, N, K, g, _ptr(ws), nbytes,
                                      _stream(x)), "w4a4_linear_fused_lora")
    return y


def debug_set_wait_limit(limit_ns):
    """Test hook: the bounded-wait limit of every kernel launched afterwards
    (0 restores the default of 2 s); see w4a4_debug_set_wait_limit."""
    _check(load_library().w4a4_debug_set_wait_limit(int(limit_ns)), "w4a4_debug_set_wait_limit")


def last_device_error(device=None):
    """Synchronise the current stream and return (and clear) the device status."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    return lib.w4a4_last_device_error(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
