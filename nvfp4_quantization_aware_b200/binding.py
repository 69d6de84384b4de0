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


class MoeShape(ctypes.Structure):
    """qad_moe_shape of include/nvfp4qad.h."""
    _fields_ = [("tokens", ctypes.c_int), ("hidden", ctypes.c_int), ("ffn", ctypes.c_int),
                ("experts", ctypes.c_int), ("topk", ctypes.c_int), ("save_act", ctypes.c_int)]


class MoeWeights(ctypes.Structure):
    """qad_moe_weights of include/nvfp4qad.h."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "gate_ts", "up_ts", "down_ts", "gate_sb", "up_sb", "down_sb",
        "gate_sb_mma", "up_sb_mma", "down_sb_mma", "x_ts", "a_ts")]


# qad_moe_buffer of include/nvfp4qad.h: name -> (index, dtype, shape given (T, H, F, G, k, R))
MOE_BUFFERS = {
    "seg_len": (0, torch.int32, lambda T, H, F, G, k, R: (G,)),
    "seg_off": (1, torch.int32, lambda T, H, F, G, k, R: (G + 1,)),
    "row_token": (2, torch.int32, lambda T, H, F, G, k, R: (R,)),
    "row_weight": (3, torch.float32, lambda T, H, F, G, k, R: (R,)),
    "slot_row": (4, torch.int32, lambda T, H, F, G, k, R: (T, k)),
    "x_codes": (5, torch.uint8, lambda T, H, F, G, k, R: (R, H // 2)),
    "x_scales": (6, torch.uint8, lambda T, H, F, G, k, R: (R * H // 16,)),
    "x_hat": (7, torch.bfloat16, lambda T, H, F, G, k, R: (R, H)),
    "wg_codes": (8, torch.uint8, lambda T, H, F, G, k, R: (G * F, H // 2)),
    "wu_codes": (9, torch.uint8, lambda T, H, F, G, k, R: (G * F, H // 2)),
    "wd_codes": (10, torch.uint8, lambda T, H, F, G, k, R: (G * H, F // 2)),
    "h_gate": (11, torch.bfloat16, lambda T, H, F, G, k, R: (R, F)),
    "h_up": (12, torch.bfloat16, lambda T, H, F, G, k, R: (R, F)),
    "a_codes": (13, torch.uint8, lambda T, H, F, G, k, R: (R, F // 2)),
    "a_scales": (14, torch.uint8, lambda T, H, F, G, k, R: (R * F // 16,)),
    "a_hat": (15, torch.bfloat16, lambda T, H, F, G, k, R: (R, F)),
    "act": (16, torch.bfloat16, lambda T, H, F, G, k, R: (R, F)),
    "y_rows": (17, torch.bfloat16, lambda T, H, F, G, k, R: (R, H)),
    "dy_rows": (18, torch.bfloat16, lambda T, H, F, G, k, R: (R, H)),
    "wd_hat": (19, torch.bfloat16, lambda T, H, F, G, k, R: (G * H, F)),
    "da": (20, torch.bfloat16, lambda T, H, F, G, k, R: (R, F)),
    "dgu": (21, torch.bfloat16, lambda T, H, F, G, k, R: (R, 2 * F)),
    "wgu_hat": (22, torch.bfloat16, lambda T, H, F, G, k, R: (G * 2 * F, H)),
    "dx_rows": (23, torch.bfloat16, lambda T, H, F, G, k, R: (R, H)),
}


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
    L.nvfp4_fault_inject.argtypes = [i64]
    L.nvfp4_fault_inject.restype = None
    L.nvfp4_selftest_timeout.argtypes = [i64, p]
    L.nvfp4_selftest_timeout.restype = i32
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
    L.nvfp4_quantize_fake_quant_grouped.argtypes = [i32, ctypes.POINTER(TensorRef), ctypes.POINTER(p),
                                                    ctypes.POINTER(i64), i32, i32, i32, p, sz, p]
    L.nvfp4_quantize_fake_quant_grouped.restype = i32
    L.nvfp4_fake_quant_grouped.restype = i32
    L.nvfp4_tensor_amax_grouped.argtypes = [i32, ctypes.POINTER(TensorRef), i32, p, p]
    L.nvfp4_tensor_amax_grouped.restype = i32
    L.nvfp4_global_scale_from_amax.argtypes = [p, i32, p, p]
    L.nvfp4_global_scale_from_amax.restype = i32
    L.nvfp4_calibrate_mse.argtypes = [p, i32, i64, i64, i64, p, p, p, p]
    L.nvfp4_calibrate_mse.restype = i32
    L.nvfp4_calibrate_mse_grouped.argtypes = [i32, ctypes.POINTER(TensorRef), i32, ctypes.POINTER(p), p]
    L.nvfp4_calibrate_mse_grouped.restype = i32
    L.nvfp4_selftest_division.argtypes = [p, p, p]
    L.nvfp4_selftest_division.restype = i32
    L.nvfp4_gemm_workspace_size.argtypes = [i64, i64, i64]
    L.nvfp4_gemm_workspace_size.restype = sz
    L.nvfp4_gemm_w4a4.argtypes = [p, p, p, p, p, p, i64, i64, i64, p, i64, p, sz, p]
    L.nvfp4_gemm_w4a4.restype = i32
    L.nvfp4_gemm_w4a4_grouped.argtypes = [i32, p, p, p, i64, p, p, p, p, p, i64, i64, p, i64, p, sz, p]
    L.nvfp4_gemm_w4a4_grouped.restype = i32
    L.nvfp4_gemm_bf16_grouped.argtypes = [i32, i32, p, i32, i64, i64, i64, p, i32, i64, i64, i64, p, p, i64, i64,
                                          i64, p, i64, p]
    L.nvfp4_gemm_bf16_grouped.restype = i32
    L.nvfp4_gemm_w4a16.argtypes = [p, i64, p, p, p, i64, i64, i64, p, i64, p]
    L.nvfp4_gemm_w4a16.restype = i32
    L.nvfp4_probe_fp4_mma.argtypes = [i64, i32, ctypes.POINTER(ctypes.c_double), p]
    L.nvfp4_probe_fp4_mma.restype = i32
    L.qad_kl_workspace_size.argtypes = [i64, i64, i32]
    L.qad_kl_workspace_size.restype = sz
    L.qad_kl_fwd_bwd.argtypes = [p, p, i32, i64, i64, i64, f32, p, p, p, i64, f32, p, sz, p]
    L.qad_kl_fwd_bwd.restype = i32
    L.qad_kl_topk_fwd_bwd.argtypes = [p, p, i32, i64, i64, i64, i64, f32, p, p, p, i64, f32, p, sz, p]
    L.qad_kl_topk_fwd_bwd.restype = i32
    L.qad_kl_topp_workspace_size.argtypes = [i64, i64, i32]
    L.qad_kl_topp_workspace_size.restype = sz
    L.qad_kl_topp_fwd_bwd.argtypes = [p, p, i32, i64, i64, i64, f32, f32, p, p, p, i64, f32, p, p, sz, p]
    L.qad_kl_topp_fwd_bwd.restype = i32
    # MoE layer step
    L.nvfp4_moe_rows_capacity.argtypes = [i32, i32, i32]
    L.nvfp4_moe_rows_capacity.restype = i64
    L.nvfp4_moe_route.argtypes = [p, p, i32, i32, i32, p, p, p, p, p, i64, p]
    L.nvfp4_moe_route.restype = i32
    L.nvfp4_moe_gather_quantize.argtypes = [p, i64, p, p, i32, p, i64, i64, p, p, p, p]
    L.nvfp4_moe_gather_quantize.restype = i32
    L.nvfp4_moe_swiglu_quantize.argtypes = [p, p, i64, p, p, i32, p, i64, i64, p, p, p, p, p]
    L.nvfp4_moe_swiglu_quantize.restype = i32
    L.nvfp4_moe_combine.argtypes = [p, i64, p, p, i32, i32, p, i32, p, p]
    L.nvfp4_moe_combine.restype = i32
    L.nvfp4_moe_scale_rows.argtypes = [p, i64, p, p, p, i32, i64, p, p]
    L.nvfp4_moe_scale_rows.restype = i32
    L.nvfp4_moe_swiglu_backward.argtypes = [p, p, p, i64, p, p, i32, i64, p, p]
    L.nvfp4_moe_swiglu_backward.restype = i32
    L.nvfp4_moe_gather_sum.argtypes = [p, i64, p, i32, i32, p, i32, p, p]
    L.nvfp4_moe_gather_sum.restype = i32
    L.nvfp4_moe_router_grad.argtypes = [p, p, i64, p, i32, i32, p, p]
    L.nvfp4_moe_router_grad.restype = i32
    L.nvfp4_scales_to_mma.argtypes = [p, i64, i64, p, p]
    L.nvfp4_scales_to_mma.restype = i32
    shp, wts = ctypes.POINTER(MoeShape), ctypes.POINTER(MoeWeights)
    L.qad_moe_workspace_size.argtypes = [shp]
    L.qad_moe_workspace_size.restype = sz
    L.qad_moe_rows_capacity.argtypes = [shp]
    L.qad_moe_rows_capacity.restype = i64
    L.qad_moe_workspace_buffer.argtypes = [shp, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.qad_moe_workspace_buffer.restype = i32
    L.qad_moe_forward.argtypes = [shp, wts, p, p, p, p, p, sz, p]
    L.qad_moe_forward.restype = i32
    L.qad_moe_backward.argtypes = [shp, wts, p, p, p, p, p, p, p, sz, p]
    L.qad_moe_backward.restype = i32
    L.qad_moe_expert_forward.argtypes = [shp, wts, p, p, p, p, sz, p]
    L.qad_moe_expert_forward.restype = i32
    L.qad_moe_expert_backward.argtypes = [shp, wts, p, p, p, p, p, p, sz, p]
    L.qad_moe_expert_backward.restype = i32
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


def nvfp4_fault_inject(nth: int) -> None:
    """Arm the library's host-side fault injection: the nth outermost call of
    an exported operation from now fails with NVFP4_ERR_CUDA before launching
    (0 disarms)."""
    lib().nvfp4_fault_inject(int(nth))


def nvfp4_selftest_timeout(limit_cycles: int, device="cuda") -> None:
    """Launch the bounded-wait self-test kernel (a wait that nothing ends,
    expiring after limit_cycles); nvfp4_device_error() then reports it."""
    _check(lib().nvfp4_selftest_timeout(int(limit_cycles), _stream(torch.device(device))), "nvfp4_selftest_timeout")


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


def nvfp4_quantize_fake_quant_grouped(xs, mode: int, tensor_scales, block_scales, codes=None, ys=None,
                                      workspace: torch.Tensor | None = None):
    """Codes (ROWMAJOR block scales) and fake-quant values of a list of
    tensors in one pass; returns (codes list, ys list)."""
    L = lib()
    n = len(xs)
    dev = xs[0].device
    dt = _dtype_code(xs[0])
    ts_list = [tensor_scales[i:i + 1] for i in range(n)] if isinstance(tensor_scales, torch.Tensor) else list(tensor_scales)
    if codes is None:
        codes = [torch.empty(x.shape[0], x.shape[1] // 2, dtype=torch.uint8, device=dev) for x in xs]
    if ys is None:
        ys = [torch.empty_like(x) for x in xs]
    arr = _refs(xs, ts_list, block_scales, codes)
    yp = (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys])
    ld = (ctypes.c_int64 * n)(*[y.stride(0) for y in ys])
    need = int(L.nvfp4_grouped_workspace_size(mode))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.nvfp4_quantize_fake_quant_grouped(n, arr, yp, ld, dt, mode, SCALES_ROWMAJOR, _ptr(workspace),
                                             0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "nvfp4_quantize_fake_quant_grouped")
    return codes, ys


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


def nvfp4_gemm_w4a4_grouped(a_codes: torch.Tensor, a_scales_mma: torch.Tensor, a_tensor_scales: torch.Tensor,
                            a_row_offsets: torch.Tensor, a_rows: torch.Tensor, b_codes: torch.Tensor,
                            b_scales_mma: torch.Tensor, b_tensor_scales: torch.Tensor, N: int,
                            out: torch.Tensor | None = None) -> torch.Tensor:
    """Grouped W4A4 GEMM: group g multiplies A rows [off[g], off[g] + rows[g]) by
    B rows [g N, (g+1) N).  a_codes [rows_total, K/2]; b_codes [groups * N, K/2];
    a_row_offsets int32 [groups + 1], a_rows int32 [groups] (device)."""
    _cuda2d(a_codes, "a_codes")
    _cuda2d(b_codes, "b_codes")
    groups = a_rows.numel()
    rows_total, K2 = a_codes.shape
    dev = a_codes.device
    if out is None:
        out = torch.empty(rows_total, N, dtype=torch.bfloat16, device=dev)
    st = lib().nvfp4_gemm_w4a4_grouped(groups, _ptr(a_codes), _ptr(a_scales_mma), _ptr(a_tensor_scales), rows_total,
                                       _ptr(a_row_offsets), _ptr(a_rows), _ptr(b_codes), _ptr(b_scales_mma),
                                       _ptr(b_tensor_scales), N, 2 * K2, _ptr(out), out.stride(0), None, 0,
                                       _stream(dev))
    _check(st, "nvfp4_gemm_w4a4_grouped")
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


# ------------------------------------------------------------------ BF16 grouped GEMM

def nvfp4_gemm_bf16_grouped(mode: int, a: torch.Tensor, b: torch.Tensor, seg_off: torch.Tensor,
                            seg_len: torch.Tensor, M: int, N: int, K: int, out: torch.Tensor | None = None,
                            a_mn_major: bool = False, b_mn_major: bool = False):
    """C = A B^T per group, bf16.  An operand is K-major (stored rows x K) or
    MN-major (stored K x rows).  mode 0: A's M range in 128-aligned segments,
    B of group g = N indices [g N, (g+1) N) (K-major) or K indices
    [g K, (g+1) K) (MN-major); mode 1: group g reduces over K indices
    [seg_off[g], seg_off[g] + seg_len[g]), C of group g = rows [g M, (g+1) M)."""
    _cuda2d(a, "a")
    _cuda2d(b, "b")
    groups = seg_len.numel()
    dev = a.device
    if out is None:
        rows = (a.shape[1] if a_mn_major else a.shape[0]) if mode == 0 else groups * M
        out = torch.empty(rows, N, dtype=torch.bfloat16, device=dev)
    st = lib().nvfp4_gemm_bf16_grouped(mode, groups, _ptr(a), int(a_mn_major), a.shape[0], a.shape[1], a.stride(0),
                                       _ptr(b), int(b_mn_major), b.shape[0], b.shape[1], b.stride(0), _ptr(seg_off),
                                       _ptr(seg_len), M, N, K, _ptr(out), out.stride(0), _stream(dev))
    _check(st, "nvfp4_gemm_bf16_grouped")
    return out


def nvfp4_gemm_w4a16(a: torch.Tensor, b_codes: torch.Tensor, b_scales: torch.Tensor, b_tensor_scale: torch.Tensor,
                     out: torch.Tensor | None = None) -> torch.Tensor:
    """C = A W^T with A bf16 [M, K] and W NVFP4 (codes [N, K/2], ROWMAJOR block
    scales [N, K/16], tensor scale [1]) dequantized inside the GEMM; bf16 [M, N]."""
    _cuda2d(a, "a")
    _cuda2d(b_codes, "b_codes")
    if a.dtype != torch.bfloat16:
        raise TypeError("a must be bfloat16")
    M, K = a.shape
    N = b_codes.shape[0]
    if b_codes.shape[1] * 2 != K or not b_codes.is_contiguous() or not b_scales.is_contiguous():
        raise ValueError("b_codes must be contiguous [N, K/2] and b_scales contiguous [N, K/16]")
    if b_scales.numel() != N * (K // 16) or b_tensor_scale.dtype != torch.float32:
        raise ValueError("b_scales must hold N * K/16 bytes and b_tensor_scale be float32")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    st = lib().nvfp4_gemm_w4a16(_ptr(a), a.stride(0), _ptr(b_codes), _ptr(b_scales), _ptr(b_tensor_scale), M, N, K,
                                _ptr(out), out.stride(0), _stream(a.device))
    _check(st, "nvfp4_gemm_w4a16")
    return out


def nvfp4_probe_fp4_mma(iters: int, ctas: int, stream: torch.cuda.Stream | None = None) -> float:
    """Launch the dense FP4 MMA throughput probe; returns the flop of the launch
    (the caller times it with CUDA events on the same stream)."""
    flop = ctypes.c_double(0.0)
    s = (stream or torch.cuda.current_stream()).cuda_stream
    _check(lib().nvfp4_probe_fp4_mma(iters, ctas, ctypes.byref(flop), s), "nvfp4_probe_fp4_mma")
    return flop.value


def nvfp4_scales_to_mma(block_scales: torch.Tensor, rows: int, cols: int) -> torch.Tensor:
    """ROWMAJOR block scales [rows, cols/16] -> MMA layout (flat uint8)."""
    out = torch.empty(mma_scales_bytes(rows, cols), dtype=torch.uint8, device=block_scales.device)
    st = lib().nvfp4_scales_to_mma(_ptr(block_scales), rows, cols, _ptr(out), _stream(block_scales.device))
    _check(st, "nvfp4_scales_to_mma")
    return out


# ------------------------------------------------------------------ MoE layer step

class MoeLayerStep:
    """Holds the C structs and the workspace of qad_moe_forward / qad_moe_backward
    for one layer shape.  Tensors are kept referenced so the raw pointers in
    the structs stay valid."""

    def __init__(self, tokens: int, hidden: int, ffn: int, experts: int, topk: int, weights: dict,
                 save_act: bool = False, device="cuda"):
        self.shape = MoeShape(tokens, hidden, ffn, experts, topk, 1 if save_act else 0)
        L = lib()
        self.ws_bytes = int(L.qad_moe_workspace_size(ctypes.byref(self.shape)))
        if self.ws_bytes == 0:
            raise NVFP4Error(2, "qad_moe_workspace_size")
        self.rows_cap = int(L.qad_moe_rows_capacity(ctypes.byref(self.shape)))
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=device)
        self._keep = dict(weights)
        self.weights = MoeWeights(**{n: weights[n].data_ptr() for n, _ in MoeWeights._fields_})
        self.device = torch.device(device)

    def buffer(self, name: str) -> torch.Tensor:
        """A view of one workspace buffer (see MOE_BUFFERS)."""
        idx, dtype, shape_fn = MOE_BUFFERS[name]
        off, nb = ctypes.c_size_t(0), ctypes.c_size_t(0)
        _check(lib().qad_moe_workspace_buffer(ctypes.byref(self.shape), idx, ctypes.byref(off), ctypes.byref(nb)),
               "qad_moe_workspace_buffer")
        s = self.shape
        shape = shape_fn(s.tokens, s.hidden, s.ffn, s.experts + 1, s.topk, self.rows_cap)
        raw = self.workspace[off.value:off.value + nb.value]
        return raw.view(dtype).view(*shape)

    def forward(self, x: torch.Tensor, expert_ids: torch.Tensor, combine_weights: torch.Tensor,
                y: torch.Tensor | None = None) -> torch.Tensor:
        if y is None:
            y = torch.empty_like(x)
        st = lib().qad_moe_forward(ctypes.byref(self.shape), ctypes.byref(self.weights), _ptr(x), _ptr(expert_ids),
                                   _ptr(combine_weights), _ptr(y), _ptr(self.workspace), self.ws_bytes,
                                   _stream(self.device))
        _check(st, "qad_moe_forward")
        return y

    def backward(self, dy: torch.Tensor, dx=None, dw_gate=None, dw_up=None, dw_down=None, d_combine=None,
                 want_combine_grad: bool = True):
        s = self.shape
        G, H, F = s.experts + 1, s.hidden, s.ffn
        dev = self.device
        dx = torch.empty_like(dy) if dx is None else dx
        dw_gate = torch.empty(G * F, H, dtype=torch.bfloat16, device=dev) if dw_gate is None else dw_gate
        dw_up = torch.empty(G * F, H, dtype=torch.bfloat16, device=dev) if dw_up is None else dw_up
        dw_down = torch.empty(G * H, F, dtype=torch.bfloat16, device=dev) if dw_down is None else dw_down
        if want_combine_grad and d_combine is None:
            d_combine = torch.empty(s.tokens, s.topk, dtype=torch.float32, device=dev)
        st = lib().qad_moe_backward(ctypes.byref(self.shape), ctypes.byref(self.weights), _ptr(dy), _ptr(dx),
                                    _ptr(dw_gate), _ptr(dw_up), _ptr(dw_down), _ptr(d_combine),
                                    _ptr(self.workspace), self.ws_bytes, _stream(dev))
        _check(st, "qad_moe_backward")
        return dx, dw_gate, dw_up, dw_down, d_combine


class MoeExpertStep:
    """qad_moe_expert_forward / qad_moe_expert_backward: the expert FFNs of
    `experts` experts (one expert-parallel rank's, or the shared expert alone
    with experts = 1) on a set of rows, each row routed to one of them.  The
    number of rows may change from call to call; the workspace grows when it
    must."""

    def __init__(self, hidden: int, ffn: int, experts: int, weights: dict, device="cuda"):
        self.hidden, self.ffn, self.experts = hidden, ffn, experts
        self._keep = dict(weights)
        self.weights = MoeWeights(**{n: weights[n].data_ptr() for n, _ in MoeWeights._fields_})
        self.device = torch.device(device)
        self.workspace = torch.empty(0, dtype=torch.uint8, device=self.device)
        self.shape = None

    def _shape(self, rows: int) -> MoeShape:
        shape = MoeShape(rows, self.hidden, self.ffn, self.experts, 1, 0)
        need = int(lib().qad_moe_workspace_size(ctypes.byref(shape)))
        if need == 0:
            raise NVFP4Error(2, "qad_moe_workspace_size")
        if self.workspace.numel() < need:
            self.workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
        self.shape = shape
        return shape

    def forward(self, x: torch.Tensor, expert_ids: torch.Tensor, y: torch.Tensor | None = None) -> torch.Tensor:
        """y[r] = E_{expert_ids[r]}(x[r]) for the rows x [n, hidden] (bf16)."""
        if y is None:
            y = torch.empty_like(x)
        if x.shape[0] == 0:
            self.shape = None
            return y
        shape = self._shape(x.shape[0])
        st = lib().qad_moe_expert_forward(ctypes.byref(shape), ctypes.byref(self.weights), _ptr(x), _ptr(expert_ids),
                                          _ptr(y), _ptr(self.workspace), self.workspace.numel(), _stream(self.device))
        _check(st, "qad_moe_expert_forward")
        return y

    def backward(self, dy: torch.Tensor, dx=None, dw_gate=None, dw_up=None, dw_down=None):
        """After forward on the same rows: dy [n, hidden] the rows' output
        gradients (combine weight applied).  Returns (dx, dw_gate, dw_up, dw_down)."""
        E, H, F = self.experts, self.hidden, self.ffn
        dev = self.device
        dx = torch.empty_like(dy) if dx is None else dx
        dw_gate = torch.empty(E * F, H, dtype=torch.bfloat16, device=dev) if dw_gate is None else dw_gate
        dw_up = torch.empty(E * F, H, dtype=torch.bfloat16, device=dev) if dw_up is None else dw_up
        dw_down = torch.empty(E * H, F, dtype=torch.bfloat16, device=dev) if dw_down is None else dw_down
        if dy.shape[0] == 0:
            for t in (dw_gate, dw_up, dw_down):
                t.zero_()
            return dx, dw_gate, dw_up, dw_down
        if self.shape is None or self.shape.tokens != dy.shape[0]:
            raise ValueError("backward needs the forward of the same rows first")
        st = lib().qad_moe_expert_backward(ctypes.byref(self.shape), ctypes.byref(self.weights), _ptr(dy), _ptr(dx),
                                           _ptr(dw_gate), _ptr(dw_up), _ptr(dw_down), _ptr(self.workspace),
                                           self.workspace.numel(), _stream(dev))
        _check(st, "qad_moe_expert_backward")
        return dx, dw_gate, dw_up, dw_down


def qad_kl_topk_fwd_bwd(teacher: torch.Tensor, student: torch.Tensor, k: int, temperature: float = 1.0,
                        want_grad: bool = True, grad_scale: float | None = None, want_row_kl: bool = False,
                        dlogits: torch.Tensor | None = None, workspace: torch.Tensor | None = None):
    """KL over the teacher's top-k entries of each row (both softmaxes
    renormalised on that set; gradient zero elsewhere).
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
    st = L.qad_kl_topk_fwd_bwd(_ptr(teacher), _ptr(student), _dtype_code(teacher), rows, V, teacher.stride(0), int(k),
                               float(temperature), _ptr(loss), _ptr(row_kl), _ptr(dlogits),
                               dlogits.stride(0) if dlogits is not None else V, float(grad_scale), _ptr(workspace),
                               0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "qad_kl_topk_fwd_bwd")
    return loss, row_kl, dlogits


def qad_kl_topp_fwd_bwd(teacher: torch.Tensor, student: torch.Tensor, p: float, temperature: float = 1.0,
                        want_grad: bool = True, grad_scale: float | None = None, want_row_kl: bool = False,
                        want_row_k: bool = False, dlogits: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None):
    """KL over the teacher's top-p set of each row (the shortest prefix of the
    top-k order whose teacher probability reaches p; p >= 1: the whole row).
    Returns (loss f32 [1], row_kl f32 [rows] or None, dlogits or None,
    row_k int64 [rows] (|S| per row) or None)."""
    _cuda2d(teacher, "teacher")
    _cuda2d(student, "student")
    if teacher.shape != student.shape or teacher.dtype != student.dtype or teacher.stride() != student.stride():
        raise ValueError("teacher and student must have the same shape, dtype and strides")
    L = lib()
    rows, V = teacher.shape
    dev = teacher.device
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    row_kl = torch.empty(rows, dtype=torch.float32, device=dev) if want_row_kl else None
    row_k = torch.empty(rows, dtype=torch.int64, device=dev) if want_row_k else None
    if want_grad and dlogits is None:
        dlogits = torch.empty_like(student)
    if not want_grad:
        dlogits = None
    if grad_scale is None:
        grad_scale = 1.0 / rows if rows > 0 else 1.0
    need = int(L.qad_kl_topp_workspace_size(rows, V, _dtype_code(teacher)))
    if workspace is None:
        workspace = _workspace(need, dev)
    st = L.qad_kl_topp_fwd_bwd(_ptr(teacher), _ptr(student), _dtype_code(teacher), rows, V, teacher.stride(0),
                               float(p), float(temperature), _ptr(loss), _ptr(row_kl), _ptr(dlogits),
                               dlogits.stride(0) if dlogits is not None else V, float(grad_scale), _ptr(row_k),
                               _ptr(workspace), 0 if workspace is None else workspace.numel(), _stream(dev))
    _check(st, "qad_kl_topp_fwd_bwd")
    return loss, row_kl, dlogits, row_k


# ------------------------------------------------------------------ MSE calibration

def nvfp4_calibrate_mse(x: torch.Tensor, tensor_scale: torch.Tensor, want_err: bool = False):
    """Block scales (ROWMAJOR uint8 [rows, cols/16]) minimising each block's
    squared fake-quantization error for the given tensor scale; with
    want_err, also the least error per block (f32)."""
    _cuda2d(x, "x")
    rows, cols = x.shape
    sb = torch.empty(rows, cols // 16, dtype=torch.uint8, device=x.device)
    err = torch.empty(rows, cols // 16, dtype=torch.float32, device=x.device) if want_err else None
    st = lib().nvfp4_calibrate_mse(_ptr(x), _dtype_code(x), rows, cols, x.stride(0), _ptr(tensor_scale), _ptr(sb),
                                   _ptr(err), _stream(x.device))
    _check(st, "nvfp4_calibrate_mse")
    return (sb, err) if want_err else sb


def nvfp4_calibrate_mse_grouped(xs, tensor_scales, block_scales=None):
    """Grouped form over a list of tensors (one tensor scale each)."""
    n = len(xs)
    dev = xs[0].device
    ts_list = [tensor_scales[i:i + 1] for i in range(n)] if isinstance(tensor_scales, torch.Tensor) else list(tensor_scales)
    if block_scales is None:
        block_scales = [torch.empty(x.shape[0], x.shape[1] // 16, dtype=torch.uint8, device=dev) for x in xs]
    dummy = [torch.empty(0, dtype=torch.uint8, device=dev)] * n
    arr = (TensorRef * n)()
    for i, x in enumerate(xs):
        _cuda2d(x, f"tensor {i}")
        arr[i] = TensorRef(x.data_ptr(), x.shape[0], x.shape[1], x.stride(0), ts_list[i].data_ptr(),
                           block_scales[i].data_ptr(), None, 0)
    st = lib().nvfp4_calibrate_mse_grouped(n, arr, _dtype_code(xs[0]), None, _stream(dev))
    _check(st, "nvfp4_calibrate_mse_grouped")
    return block_scales
