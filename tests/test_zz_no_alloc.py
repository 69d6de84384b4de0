"""The allocation-free KL entry point (qad_kl_fwd_bwd_noalloc) against the
regular one (qad_kl_fwd_bwd), called through the C ABI.

qad_kl_fwd_bwd_noalloc is for callers that cannot allocate device memory when
they compute the loss (for example inside a framework whose caching allocator
already holds the device budget, or with a fixed memory plan): it keeps its
per-row scratch in a static device array of the library instead of taking a
workspace.  This file runs last (pytest collects it after the others) and
must also pass on its own in a fresh process, where its first call is the one
that looks up the array's device address.
"""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
MAX_ROWS = 65536  # NVFP4_KL_NOALLOC_MAX_ROWS in include/nvfp4qad.h


def _noalloc_fn():
    L = Q.lib()
    f = L.qad_kl_fwd_bwd_noalloc
    p, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    f.argtypes = [p, p, i32, i64, i64, i64, f32, p, p, p, i64, f32, p]
    f.restype = i32
    return f


def _call_noalloc(t, s, T=1.0):
    f = _noalloc_fn()
    rows, V = t.shape
    loss = torch.empty(1, dtype=torch.float32, device=DEV)
    row_kl = torch.empty(rows, dtype=torch.float32, device=DEV)
    grad = torch.empty_like(s)
    st = f(t.data_ptr(), s.data_ptr(), Q.BF16 if t.dtype == torch.bfloat16 else Q.F32, rows, V, t.stride(0),
           T, loss.data_ptr(), row_kl.data_ptr(), grad.data_ptr(), grad.stride(0), 1.0 / rows,
           torch.cuda.current_stream().cuda_stream)
    assert st == 0, st
    return loss, row_kl, grad


def _compare(t, s, T=1.0):
    loss_n, row_n, grad_n = _call_noalloc(t, s, T)
    loss_r, row_r, grad_r = Q.qad_kl_fwd_bwd(t, s, temperature=T, want_row_kl=True)
    torch.cuda.synchronize()
    lr = float(loss_r.cpu()[0])
    assert abs(float(loss_n.cpu()[0]) - lr) <= 1e-4 * abs(lr)
    rr = row_r.double().cpu().numpy()
    assert np.allclose(row_n.double().cpu().numpy(), rr, rtol=1e-4, atol=1e-6)
    gr = grad_r.double().cpu().numpy()
    err = np.linalg.norm(grad_n.double().cpu().numpy() - gr) / np.linalg.norm(gr)
    assert err <= 1e-3, err


def test_noalloc_matches_workspace_entry_point_twice():
    # two calls in a row on different inputs, the larger first: the shared
    # scratch keeps the first call's 100 row values, so a second call that
    # read a slot at or beyond its own 48 rows, or left one of its rows
    # unwritten, would return a different loss or per-row KL
    t1, s1 = S.logits_pair(100, 8192, seed=12, device=DEV, dtype=torch.float32, boost=None, teacher_std=4.0,
                           noise_std=0.5)
    _compare(t1, s1, T=1.5)
    t2, s2 = S.logits_pair(48, 131072, seed=11, device=DEV, dtype=torch.bfloat16)
    _compare(t2, s2)


def test_noalloc_rejects_rows_beyond_the_maximum():
    f = _noalloc_fn()
    dummy = torch.empty(16, dtype=torch.float32, device=DEV)
    p = dummy.data_ptr()
    st = f(p, p, Q.F32, MAX_ROWS + 1, 16, 16, 1.0, p, None, None, 16, 1.0, None)
    assert st == 2  # NVFP4_ERR_SHAPE, returned before any launch
