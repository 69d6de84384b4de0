"""ctypes binding of libnvfp4qad.so.

Argument marshalling only: each function checks that the tensors it is given
are CUDA tensors of the right dtype, allocates outputs with torch (device
memory is torch's job here), and calls the C entry point of the same name on
torch's current stream.  Every computation happens in the library's kernels.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))

# enums of include/nvfp4qad.h
BF16, F32 = 0, 1
DYNAMIC, FROZEN_GLOBAL, FROZEN_ALL = 0, 1, 2
SCALES_ROWMAJOR, SCALES_MMA = 0, 1

_STATUS = {0: "OK", 1: "ERR_ARG", 2: "ERR_SHAPE", 3: "ERR_ALIGN", 4: "ERR_DTYPE", 5: "ERR_CUDA",
           6: "ERR_TIMEOUT", 7: "ERR_DEVICE", 8: "ERR_WORKSPACE", 9: "ERR_UNSUPPORTED"}

_lib = None


class TensorRef(ctypes.Structure):
    """nvfp4_tensor_ref of include/nvfp4qad.h."""
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("ld_x", ctypes.c_int64), ("tensor_scale", ctypes.c_void_p), ("block_scales", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("ld_out", ctypes.c_int64)]


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib().nvfp4_status_string(status).decode() if _lib is not None else _STATUS.get(status, "?")
        super().__init__(f"{what}: {msg} ({status})")


def library_path() -> str:
    return os.environ.get("NVFP4QAD_LIB", os.path.join(HERE, "libnvfp4qad.so"))


def lib() -> ctypes.CDLL:
    """Load libnvfp4qad.so (built in-tree by nvfp4_quantization_aware_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(f"libnvfp4qad.so not found at {path}; build it with "
                          f"`python nvfp4_quantization_aware_b200/build.py` (there is no CPU fallback)")
    L = ctypes.CDLL(path)
    i64, f32, p, sz, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    L.nvfp4_status_string.argtypes = [i32]
    L.nvfp4_status_string.restype = ctypes.c_char_p
    L.nvfp4_abi_version.restype = i32
    L.nvfp4_mma_scales_bytes.argtypes = [i64, i64]
    L.nvfp4_mma_scales_bytes.restype = sz
    L.nvfp4_device_error.argtypes = [p, ctypes.POINTER(ctypes.c_int32)]
    L.nvfp4_device_error.restype = i32
    L.nvfp4_quantize_workspace_size.argtypes = [i64, i64, i32]
    L.nvfp4_quantize_workspace_size.restype = sz
    L.nvfp4_fake_quant_workspace_size.argtypes = [i64, i64, i32]
    L.nvfp4_fake_quant_workspace_size.restype = sz
    L.nvfp4_quantize.argtypes = [p, i32, i64, i64, i64, i32, p, p, i32, p, i64, p, sz, p]
    L.nvfp4_quantize.restype = i32
    L.nvfp4_fake_quant.argtypes = [p, i32, i64, i64, i64, i32, p, p, p, i64, p, sz, p]
    L.nvfp4_fake_quant.restype = i32
    L.nvfp4_dequantize.argtypes = [p, i64, p, i32, p, i64, i64, p, i32, i64, p]
    L.nvfp4_dequantize.restype = i32
    L.nvfp4_launch_count.restype = ctypes.c_uint64
    L.nvfp4_grouped_workspace_size.argtypes = [i32]
    L.nvfp4_grouped_workspace_size.restype = sz
    L.nvfp4_quantize_grouped.argtypes = [i32, ctypes.POINTER(TensorRef), i32, i32, i32, p, sz, p]
    L.nvfp4_quantize_grouped.restype = i32
    L.nvfp4_fake_quant_grouped.argtypes = [i32, ctypes.POINTER(TensorRef), i32, i32, p, sz, p]
    L.nvfp4_fake_quant_grouped.restype = i32
    L.nvfp4_selftest_division.argtypes = [p, p, p]
    L.nvfp4_selftest_division.restype = i32
    if hasattr(L, "nvfp4_gemm_w4a4"):
        L.nvfp4_gemm_workspace_size.argtypes = [i64, i64, i64]
        L.nvfp4_gemm_workspace_size.restype = sz
        L.nvfp4_gemm_w4a4.argtypes = [p, p, p, p, p, p, i64, i64, i64, p, i64, p, sz, p]
        L.nvfp4_gemm_w4a4.restype = i32
    if hasattr(L, "qad_kl_fwd_bwd"):
        L.qad_kl_workspace_size.argtypes = [i64, i64, i32]
        L.qad_kl_workspace_size.restype = sz
        L.qad_kl_fwd_bwd.argtypes = [p, p, i32, i64, i64, i64, f32, p, p, p, i64, f32, p, sz, p]
        L.qad_kl_fwd_bwd.restype = i32
    _lib = L
    return L


# ------------------------------------------------------------------ helpers

def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise NVFP4Error(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}; expected bfloat16 or float32")


def _cuda2d(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with a contiguous last dimension")


def _workspace(nbytes: int, device) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def mma_scales_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4_mma_scales_bytes(rows, cols))


def nvfp4_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib().nvfp4_launch_count())


def nvfp4_device_error() -> tuple[int, int]:
    """Synchronize the current stream and read/clear the device error word.
    Returns (status, word)."""
    word = ctypes.c_int32(0)
    st = lib().nvfp4_device_error(ctypes.c_void_p(_stream(torch.device("cuda"))), ctypes.byref(word))
    return int(st), int(word.value)


# ------------------------------------------------------------------ quantize

def nvfp4_quantize(x: torch.Tensor, mode: int = DYNAMIC, tensor_scale: torch.Tensor | None = None,
                   block_scales: torch.Tensor | None = None, layout: int = SCALES_ROWMAJOR,
                   codes: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """Quantize x [rows, cols] (bf16/f32, CUDA) to NVFP4.

    Returns (codes uint8 [rows, cols/2], block_scales uint8, tensor_scale f32 [1]).
    block_scales is [rows, cols/16] (ROWMAJOR) or flat nvfp4_mma_scales_bytes
    (MMA).  DYNAMIC writes tensor_scale; FROZEN_* read it; FROZEN_ALL reads
    block_scales (ROWMAJOR)."""
    _cuda2d(x, "x")
    L = lib()
    rows, cols = x.shape
    dev = x.device
    if tensor_scale is None:
        if mode != DYNAMIC:
            raise ValueError("frozen modes need tensor_scale")
        tensor_scale = torch.empty(1, dtype=torch.float32, device=dev)
    if block_scales is None:
        if mode == FROZEN_ALL:
            raise ValueError("FROZEN_ALL needs block_scales")
        block_scales = (torch.empty(rows, cols // 16, dtype=torch.uint8, device=dev) if layout == SCALES_ROWMAJOR
                        else torch.empty(mma_scales_bytes(rows, cols), dtype=torch.uint8, device=dev))
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    need = int(L.nvfp4_quantize_workspace_size(rows, cols, mode))
    if workspace is None:
        workspace = _workspace(need, dev)
    ld_codes = codes.stride(0) if codes.dim() == 2 else cols // 2
    st = L.nvfp4_quantize(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), mode, _ptr(tensor_scale),
                          _ptr(block_scales), layout, _ptr(codes), ld_codes, _ptr(workspace),
                          0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "nvfp4_quantize")
    return codes, block_scales, tensor_scale


def _refs(xs, tensor_scales, block_scales, outs):
    arr = (TensorRef * len(xs))()
    for i, x in enumerate(xs):
        _cuda2d(x, f"tensor {i}")
        o = outs[i]
        arr[i] = TensorRef(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), tensor_scales[i].data_ptr(),
                           None if block_scales[i] is None else block_scales[i].data_ptr(), o.data_ptr(),
                           o.stride(0) if o.dim() == 2 else x.shape[1] // 2)
    return arr


def nvfp4_quantize_grouped(xs, mode: int = DYNAMIC, tensor_scales=None, block_scales=None,
                           layout: int = SCALES_ROWMAJOR, codes=None, workspace: torch.Tensor | None = None):
    """Quantize a list of tensors (same dtype, same mode) in grouped launches.
    Returns (codes list, block_scales list, tensor_scales [n] f32)."""
    L = lib()
    n = len(xs)
    if n == 0:
        return [], [], None
    dev = xs[0].device
    dt = _dtype_code(xs[0])
    if any(_dtype_code(x) != dt for x in xs):
        raise TypeError("all tensors of a group must share a dtype")
    if tensor_scales is None:
        if mode != DYNAMIC:
            raise ValueError("frozen modes need tensor_scales")
        tensor_scales = torch.empty(n, dtype=torch.float32, device=dev)
    ts_list = [tensor_scales[i:i + 1] for i in range(n)] if isinstance(tensor_scales, torch.Tensor) else list(tensor_scales)
    if block_scales is None:
        if mode == FROZEN_ALL:
            raise ValueError("FROZEN_ALL needs block_scales")
        block_scales = [(torch.empty(x.shape[0], x.shape[1] // 16, dtype=torch.uint8, device=dev)
                         if layout == SCALES_ROWMAJOR else
                         torch.empty(mma_scales_bytes(*x.shape), dtype=torch.uint8, device=dev)) for x in xs]
    if codes is None:
        codes = [torch.empty(x.shape[0], x.shape[1] // 2, dtype=torch.uint8, device=dev) for x in xs]
    arr = _refs(xs, ts_list, block_scales, codes)
    need = int(L.nvfp4_grouped_workspace_size(mode))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.nvfp4_quantize_grouped(n, arr, dt, mode, layout, _ptr(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "nvfp4_quantize_grouped")
    return codes, block_scales, tensor_scales


def nvfp4_fake_quant_grouped(xs, mode: int = DYNAMIC, tensor_scales=None, block_scales=None, outs=None,
                             workspace: torch.Tensor | None = None):
    """Fake-quantize a list of tensors in grouped launches; returns the outputs."""
    L = lib()
    n = len(xs)
    if n == 0:
        return []
    dev = xs[0].device
    dt = _dtype_code(xs[0])
    if tensor_scales is None:
        if mode != DYNAMIC:
            raise ValueError("frozen modes need tensor_scales")
        tensor_scales = torch.empty(n, dtype=torch.float32, device=dev)
    ts_list = [tensor_scales[i:i + 1] for i in range(n)] if isinstance(tensor_scales, torch.Tensor) else list(tensor_scales)
    if block_scales is None:
        if mode == FROZEN_ALL:
            raise ValueError("FROZEN_ALL needs block_scales")
        block_scales = [None] * n
    if outs is None:
        outs = [torch.empty_like(x) for x in xs]
    arr = _refs(xs, ts_list, block_scales, outs)
    need = int(L.nvfp4_grouped_workspace_size(mode))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.nvfp4_fake_quant_grouped(n, arr, dt, mode, _ptr(workspace),
                                    0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "nvfp4_fake_quant_grouped")
    return outs


def nvfp4_fake_quant(x: torch.Tensor, mode: int = DYNAMIC, tensor_scale: torch.Tensor | None = None,
                     block_scales: torch.Tensor | None = None, out: torch.Tensor | None = None,
                     return_scales: bool = False, workspace: torch.Tensor | None = None):
    """y = dequantize(quantize(x)) in one pass, same dtype as x.  With
    return_scales, also returns (block_scales [rows, cols/16], tensor_scale)."""
    _cuda2d(x, "x")
    L = lib()
    rows, cols = x.shape
    dev = x.device
    if tensor_scale is None:
        if mode != DYNAMIC:
            raise ValueError("frozen modes need tensor_scale")
        tensor_scale = torch.empty(1, dtype=torch.float32, device=dev)
    if block_scales is None:
        if mode == FROZEN_ALL:
            raise ValueError("FROZEN_ALL needs block_scales")
        if return_scales:
            block_scales = torch.empty(rows, cols // 16, dtype=torch.uint8, device=dev)
    y = torch.empty_like(x) if out is None else out
    _cuda2d(y, "out")
    need = int(L.nvfp4_fake_quant_workspace_size(rows, cols, mode))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.nvfp4_fake_quant(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), mode, _ptr(tensor_scale),
                            _ptr(block_scales), _ptr(y), y.stride(0), _ptr(workspace),
                            0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "nvfp4_fake_quant")
    if return_scales:
        return y, block_scales, tensor_scale
    return y


def nvfp4_dequantize(codes: torch.Tensor, block_scales: torch.Tensor, tensor_scale: torch.Tensor, cols: int,
                     layout: int = SCALES_ROWMAJOR, out_dtype=torch.bfloat16, out: torch.Tensor | None = None):
    """out [rows, cols] = value(codes) * (float(s_b) * s_g)."""
    _cuda2d(codes, "codes")
    rows = codes.shape[0]
    dev = codes.device
    if out is None:
        out = torch.empty(rows, cols, dtype=out_dtype, device=dev)
    st = lib().nvfp4_dequantize(_ptr(codes), codes.stride(0), _ptr(block_scales), layout, _ptr(tensor_scale),
                                rows, cols, _ptr(out), _dtype_code(out), out.stride(0), _stream(dev))
    _check(st, "nvfp4_dequantize")
    return out


def nvfp4_selftest_division(device="cuda") -> tuple[int, int]:
    """Run the library's division self-test; returns (mismatches, first)."""
    buf = torch.zeros(2, dtype=torch.int64, device=device)
    st = lib().nvfp4_selftest_division(_ptr(buf), buf.data_ptr() + 8, _stream(buf.device))
    _check(st, "nvfp4_selftest_division")
    vals = buf.cpu().tolist()
    return int(vals[0]), int(vals[1]) & 0xFFFFFFFFFFFFFFFF


# ------------------------------------------------------------------ GEMM

def nvfp4_gemm_w4a4(a_codes: torch.Tensor, a_scales_mma: torch.Tensor, a_tensor_scale: torch.Tensor,
                    b_codes: torch.Tensor, b_scales_mma: torch.Tensor, b_tensor_scale: torch.Tensor,
                    out: torch.Tensor | None = None, workspace: torch.Tensor | None = None) -> torch.Tensor:
    """C [M, N] bf16 = (s_gA s_gB) * A^ @ B^T; A codes [M, K/2], B codes [N, K/2],
    scales in the MMA layout."""
    _cuda2d(a_codes, "a_codes")
    _cuda2d(b_codes, "b_codes")
    L = lib()
    M, K2 = a_codes.shape
    N = b_codes.shape[0]
    K = 2 * K2
    if b_codes.shape[1] != K2:
        raise ValueError("A and B must have the same K")
    dev = a_codes.device
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    need = int(L.nvfp4_gemm_workspace_size(M, N, K))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.nvfp4_gemm_w4a4(_ptr(a_codes), _ptr(a_scales_mma), _ptr(a_tensor_scale), _ptr(b_codes),
                           _ptr(b_scales_mma), _ptr(b_tensor_scale), M, N, K, _ptr(out), out.stride(0),
                           _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "nvfp4_gemm_w4a4")
    return out


# ------------------------------------------------------------------ KL

def qad_kl_fwd_bwd(teacher: torch.Tensor, student: torch.Tensor, temperature: float = 1.0,
                   want_grad: bool = True, grad_scale: float | None = None, want_row_kl: bool = False,
                   dlogits: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """KL(p_teacher || p_student) over the vocabulary, mean over rows, and the
    gradient w.r.t. the student logits in one pass.
    Returns (loss f32 [1], row_kl f32 [rows] or None, dlogits or None)."""
    _cuda2d(teacher, "teacher")
    _cuda2d(student, "student")
    if teacher.shape != student.shape or teacher.dtype != student.dtype or teacher.stride() != student.stride():
        raise ValueError("teacher and student must have the same shape, dtype and strides")
    L = lib()
    rows, V = teacher.shape
    dev = teacher.device
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    row_kl = torch.empty(rows, dtype=torch.float32, device=dev) if want_row_kl else None
    if want_grad and dlogits is None:
        dlogits = torch.empty_like(student)
    if not want_grad:
        dlogits = None
    if grad_scale is None:
        grad_scale = 1.0 / rows if rows > 0 else 1.0
    need = int(L.qad_kl_workspace_size(rows, V, _dtype_code(teacher)))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.qad_kl_fwd_bwd(_ptr(teacher), _ptr(student), _dtype_code(teacher), rows, V, teacher.stride(0),
                          float(temperature), _ptr(loss), _ptr(row_kl), _ptr(dlogits),
                          dlogits.stride(0) if dlogits is not None else V, float(grad_scale), _ptr(workspace),
                          0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "qad_kl_fwd_bwd")
    return loss, row_kl, dlogits
