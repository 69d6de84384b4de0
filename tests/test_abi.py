"""The C-ABI library loads and exports every function declared in
include/*.h; host-side argument validation returns its status before any
CUDA call (no GPU needed)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from nvfp4_quantization_aware_b200 import build
    build.build()
    import nvfp4_quantization_aware_b200 as Q
    return Q.lib()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b([a-z_][a-z0-9_]*)\s*\(", text):
            name = m.group(1)
            if name.startswith(("nvfp4_", "qad_")) and not name.endswith("_t"):
                names.add(name)
    return names


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ["nvfp4_quantize", "nvfp4_fake_quant", "nvfp4_dequantize", "nvfp4_gemm_w4a4",
                     "qad_kl_fwd_bwd", "nvfp4_status_string"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    path = lib._name
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = _declared_functions() - exported
    assert not missing, missing
    for name in _declared_functions():
        assert hasattr(lib, name)


def test_status_strings_and_version(lib):
    assert lib.nvfp4_abi_version() == 1
    for st in range(10):
        s = lib.nvfp4_status_string(st)
        assert s and s.startswith(b"NVFP4")


def test_validation_before_launch(lib):
    # cols not a multiple of 16 -> ERR_SHAPE; bad dtype -> ERR_DTYPE; NULL x -> ERR_ARG.
    p = ctypes.c_void_p(16)
    assert lib.nvfp4_quantize(p, 0, 4, 40, 40, 0, p, p, 0, p, 20, p, 4096, None) == 2
    assert lib.nvfp4_quantize(p, 7, 4, 32, 32, 0, p, p, 0, p, 16, p, 4096, None) == 4
    assert lib.nvfp4_quantize(None, 0, 4, 32, 32, 0, p, p, 0, p, 16, p, 4096, None) == 1
    # unaligned x -> ERR_ALIGN; missing workspace in DYNAMIC -> ERR_WORKSPACE
    assert lib.nvfp4_quantize(ctypes.c_void_p(18), 0, 4, 32, 32, 0, p, p, 0, p, 16, p, 4096, None) == 3
    assert lib.nvfp4_quantize(p, 0, 4, 32, 32, 0, p, p, 0, p, 16, None, 0, None) == 8
    # FROZEN_ALL with MMA layout is rejected
    assert lib.nvfp4_quantize(p, 0, 4, 32, 32, 2, p, p, 1, p, 16, None, 0, None) == 1
    assert lib.nvfp4_fake_quant(p, 0, 4, 32, 32, 2, p, None, p, 32, None, 0, None) == 1
    assert lib.nvfp4_dequantize(p, 16, p, 0, p, 4, 33, p, 0, 33, None) == 2


def test_mma_scales_bytes(lib):
    import oracle as O
    for rows, cols in [(1, 16), (128, 64), (129, 80), (8192, 4096)]:
        assert lib.nvfp4_mma_scales_bytes(rows, cols) == O.swizzled_scale_bytes(rows, cols)


def test_workspace_queries(lib):
    assert lib.nvfp4_quantize_workspace_size(100, 64, 0) >= 4
    assert lib.nvfp4_quantize_workspace_size(100, 64, 1) == 0
    assert lib.nvfp4_quantize_workspace_size(100, 64, 2) == 0


def test_fault_injection_fails_the_nth_call_before_launch(lib):
    """Armed with n = 2, the second outermost call returns NVFP4_ERR_CUDA (5)
    without validating or launching; the calls around it are unaffected and
    the arming is spent after one failure."""
    p = ctypes.c_void_p(16)
    bad_cols = lambda: lib.nvfp4_quantize(p, 0, 4, 40, 40, 0, p, p, 0, p, 20, p, 4096, None)
    lib.nvfp4_fault_inject.argtypes = [ctypes.c_int64]
    lib.nvfp4_fault_inject(2)
    try:
        assert bad_cols() == 2          # 1st: validated as usual (ERR_SHAPE)
        assert bad_cols() == 5          # 2nd: injected ERR_CUDA before validation
        assert bad_cols() == 2          # disarmed again
        lib.nvfp4_fault_inject(1)
        assert lib.nvfp4_dequantize(p, 16, p, 0, p, 4, 33, p, 0, 33, None) == 5  # any exported operation
        assert lib.nvfp4_dequantize(p, 16, p, 0, p, 4, 33, p, 0, 33, None) == 2
    finally:
        lib.nvfp4_fault_inject(0)
    assert bad_cols() == 2


def test_fault_injection_from_the_environment():
    """NVFP4QAD_FAIL_AT=n arms the injection when the library loads."""
    code = ("import ctypes, nvfp4_quantization_aware_b200 as Q; L = Q.lib(); p = ctypes.c_void_p(16); "
            "r = [L.nvfp4_quantize(p, 0, 4, 40, 40, 0, p, p, 0, p, 20, p, 4096, None) for _ in range(4)]; print(r)")
    env = dict(os.environ, NVFP4QAD_FAIL_AT="3", PYTHONPATH=ROOT)
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, env=env, check=True).stdout
    assert out.strip() == "[2, 2, 5, 2]"


def test_timeout_selftest_rejects_unbounded_limits(lib):
    lib.nvfp4_selftest_timeout.argtypes = [ctypes.c_int64, ctypes.c_void_p]
    assert lib.nvfp4_selftest_timeout(0, None) == 1
    assert lib.nvfp4_selftest_timeout((1 << 32) + 1, None) == 1


def test_topp_validates_before_any_launch(lib):
    """Argument checks of qad_kl_topp_fwd_bwd return before touching the GPU."""
    import nvfp4_quantization_aware_b200 as Q
    L = Q.lib()
    p = ctypes.c_void_p(64)
    ws = ctypes.c_void_p(256)
    need = L.qad_kl_topp_workspace_size(4, 100, 0)
    assert need == L.qad_kl_workspace_size(4, 100, 0) + 4 * 8
    assert L.qad_kl_topp_workspace_size(0, 100, 0) == 0
    call = lambda top_p, T=1.0, row_k=None, wsb=need, dtype=0: L.qad_kl_topp_fwd_bwd(
        p, p, dtype, 4, 100, 100, top_p, T, p, None, None, 100, 1.0, row_k, ws, wsb, None)
    assert call(0.0) == 1                      # top_p must be > 0
    assert call(-0.5) == 1
    assert call(float("nan")) == 1
    assert call(0.9, T=0.0) == 1               # temperature > 0
    assert call(0.9, dtype=7) == 4             # dtype
    assert call(0.9, wsb=need - 1) == 8        # workspace too small
    assert call(0.9, row_k=ctypes.c_void_p(68)) == 3  # row_k not 8-byte aligned
