"""Guard bands around every output: each output is a strided view into a
larger buffer filled with a canary byte, on ragged shapes (rows not a
multiple of 128, row strides wider than the rows, unaligned vector paths),
and after the call every byte outside the view must still hold the canary.
The results inside the views must equal those of the same call on plain
contiguous outputs, bit for bit."""
import pytest
import torch

import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
CANARY = 0xA5
PAD = 256  # bytes before and after


def _guarded(rows, cols, ld, dtype):
    """(buffer bytes, view [rows, cols] with row stride ld) inside a canary-filled buffer."""
    esz = torch.empty(0, dtype=dtype).element_size()
    nbytes = 2 * PAD + rows * ld * esz
    buf = torch.full((nbytes,), CANARY, dtype=torch.uint8, device=DEV)
    inner = buf[PAD:PAD + rows * ld * esz].view(dtype).view(rows, ld)
    return buf, inner[:, :cols]


def _outside_intact(buf, rows, cols, ld, dtype):
    esz = torch.empty(0, dtype=dtype).element_size()
    b = buf.cpu()
    ok = bool((b[:PAD] == CANARY).all()) and bool((b[PAD + rows * ld * esz:] == CANARY).all())
    body = b[PAD:PAD + rows * ld * esz].view(rows, ld * esz)
    ok &= bool((body[:, cols * esz:] == CANARY).all())
    return ok


@pytest.mark.parametrize("rows,cols", [(129, 160), (1, 16), (300, 1040)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_quantize_and_fake_quant_write_only_their_views(rows, cols, dtype):
    x = S.weights(rows, cols, seed=rows + cols, device=DEV).to(dtype)
    ref_c, ref_s, ref_t = Q.nvfp4_quantize(x, Q.DYNAMIC)
    ldc = cols // 2 + 12  # codes rows 12 bytes wider (a multiple of 4)
    cbuf, codes = _guarded(rows, cols // 2, ldc, torch.uint8)
    sbuf = torch.full((2 * PAD + rows * (cols // 16),), CANARY, dtype=torch.uint8, device=DEV)
    sb = sbuf[PAD:PAD + rows * (cols // 16)].view(rows, cols // 16)
    c, s, t = Q.nvfp4_quantize(x, Q.DYNAMIC, block_scales=sb, codes=codes)
    torch.cuda.synchronize()
    assert torch.equal(c, ref_c) and torch.equal(s, ref_s) and torch.equal(t, ref_t)
    assert _outside_intact(cbuf, rows, cols // 2, ldc, torch.uint8)
    assert bool((sbuf[:PAD] == CANARY).all()) and bool((sbuf[PAD + rows * (cols // 16):] == CANARY).all())
    # MMA-layout scales: the whole padded layout is written, nothing around it
    nm = Q.mma_scales_bytes(rows, cols)
    mbuf = torch.full((2 * PAD + nm,), CANARY, dtype=torch.uint8, device=DEV)
    Q.nvfp4_quantize(x, Q.DYNAMIC, block_scales=mbuf[PAD:PAD + nm], layout=Q.SCALES_MMA)
    torch.cuda.synchronize()
    assert bool((mbuf[:PAD] == CANARY).all()) and bool((mbuf[PAD + nm:] == CANARY).all())
    # fake-quant and dequantize into views 8 elements wider than the rows
    ref_y = Q.nvfp4_fake_quant(x, Q.DYNAMIC)
    ybuf, y = _guarded(rows, cols, cols + 8, dtype)
    Q.nvfp4_fake_quant(x, Q.DYNAMIC, out=y)
    dbuf, d = _guarded(rows, cols, cols + 8, dtype)
    Q.nvfp4_dequantize(ref_c, ref_s, ref_t, cols, out_dtype=dtype, out=d)
    torch.cuda.synchronize()
    assert torch.equal(y, ref_y) and torch.equal(d, ref_y)
    assert _outside_intact(ybuf, rows, cols, cols + 8, dtype)
    assert _outside_intact(dbuf, rows, cols, cols + 8, dtype)


@pytest.mark.parametrize("M,N,ldc", [(129, 256, 264), (128, 384, 386), (1, 128, 130), (300, 512, 512)])
def test_gemm_writes_only_its_output_view(M, N, ldc):
    K = 512
    x = S.activations(M, K, seed=M, device=DEV)
    w = S.weights(N, K, seed=N, device=DEV)
    a = Q.nvfp4_quantize(x, Q.DYNAMIC, layout=Q.SCALES_MMA)
    b = Q.nvfp4_quantize(w, Q.DYNAMIC, layout=Q.SCALES_MMA)
    ref = Q.nvfp4_gemm_w4a4(*a, *b)
    buf, out = _guarded(M, N, ldc, torch.bfloat16)
    Q.nvfp4_gemm_w4a4(*a, *b, out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert _outside_intact(buf, M, N, ldc, torch.bfloat16)


@pytest.mark.parametrize("loss", ["kl", "topk", "topp"])
@pytest.mark.parametrize("V,ld", [(1003, 1016), (40000, 40008), (131072, 131080)])
def test_kl_losses_write_only_their_gradient_view(loss, V, ld):
    rows = 3
    t, s = S.logits_pair(rows, V, seed=V, device=DEV, dtype=torch.bfloat16)
    call = {"kl": lambda g: Q.qad_kl_fwd_bwd(t, s, dlogits=g),
            "topk": lambda g: Q.qad_kl_topk_fwd_bwd(t, s, 100, dlogits=g),
            "topp": lambda g: Q.qad_kl_topp_fwd_bwd(t, s, 0.9, dlogits=g)}[loss]
    ref = call(None)[2]
    buf, g = _guarded(rows, V, ld, torch.bfloat16)
    call(g)
    torch.cuda.synchronize()
    assert torch.equal(g, ref)
    assert _outside_intact(buf, rows, V, ld, torch.bfloat16)
