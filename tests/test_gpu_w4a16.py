"""GPU parity of the weight-only NVFP4 GEMM (W4A16) against the oracle.

The weights are quantized by the oracle on the host and uploaded (codes,
row-major block scales, tensor scale), so the GPU kernel and the oracle
multiply the same NVFP4 weights; the activations are the same bf16 bits on
both sides.  The oracle dequantizes the weights to bf16 and sums exact
products in float64.  Bar: relative Frobenius error <= 1e-3 against the
oracle rounded to bf16 (fp32 accumulation of up to K products of bf16
values, then one bf16 rounding of the output).
"""
import numpy as np
import pytest
import torch

import oracle as O
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S

pytestmark = pytest.mark.gpu
DEV = "cuda"
GEMM_RTOL = 1e-3


def _rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _bf16_round(c):
    return O.bf16_bits_to_f32(O.bf16_round(c)).astype(np.float64)


def _oracle_weights(w):
    codes, sb, sg = O.quantize(w.float().cpu().numpy(), O.DYNAMIC)
    dev = (torch.from_numpy(codes).to(DEV), torch.from_numpy(sb).to(DEV),
           torch.tensor([sg], dtype=torch.float32, device=DEV))
    return (codes, sb, sg), dev


def _check_clean():
    torch.cuda.synchronize()
    st, word = Q.nvfp4_device_error()
    assert st == 0 and word == 0


def _run(x, w, rows=None):
    (codes, sb, sg), (dc, dsb, dsg) = _oracle_weights(w)
    c = Q.nvfp4_gemm_w4a16(x, dc, dsb, dsg)
    _check_clean()
    a = x.float().cpu().numpy()
    K = x.shape[1]
    if rows is None:
        ref = O.gemm_w4a16(a, codes, sb, sg, K)
        got = c.double().cpu().numpy()
    else:
        ref = O.gemm_w4a16(a[rows], codes, sb, sg, K)
        got = c[torch.as_tensor(rows, device=DEV)].double().cpu().numpy()
    err = _rel_fro(got, _bf16_round(ref))
    assert err <= GEMM_RTOL, err
    return c


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (127, 100, 192), (129, 256, 320), (200, 300, 1024),
                                   (64, 520, 256), (256, 512, 576), (3, 1000, 2048), (5, 1002, 1024),
                                   (130, 4096, 4096), (1, 256, 8192), (300, 257, 128)])
def test_ragged_shapes(M, N, K):
    x = S.activations(M, K, seed=M + K, device=DEV)
    w = S.weights(N, K, seed=N + K, device=DEV)
    _run(x, w)


def test_full_size_sampled_rows():
    # the benchmarked shape: 8192 x 4096 activations, 4096 x 4096 weights
    M, N, K = 8192, 4096, 4096
    x = S.channel_scaled_activations(M, K, seed=0, device=DEV)
    w = S.weights(N, K, seed=1, device=DEV)
    rows = np.random.default_rng(5).choice(M, 48, replace=False)
    rows.sort()
    _run(x, w, rows=rows)


def test_matches_bf16_gemm_on_fake_quant_weights():
    # same tiles, same K order: the dequantize-in-mainloop product equals the
    # BF16 GEMM of the fake-quantized weights bit for bit
    M, N, K = 384, 768, 1024
    x = S.activations(M, K, seed=11, device=DEV)
    w = S.weights(N, K, seed=12, device=DEV)
    codes, sb, ts = Q.nvfp4_quantize(w, Q.DYNAMIC)
    c = Q.nvfp4_gemm_w4a16(x, codes, sb, ts)
    w_hat = Q.nvfp4_fake_quant(w, Q.DYNAMIC)
    off = torch.tensor([0, M], dtype=torch.int32, device=DEV)
    ln = torch.tensor([M], dtype=torch.int32, device=DEV)
    ref = Q.nvfp4_gemm_bf16_grouped(0, x, w_hat, off, ln, M, N, K)
    _check_clean()
    assert torch.equal(c, ref)


def test_all_ones_closed_form():
    M, N, K = 130, 260, 512
    x = torch.ones(M, K, dtype=torch.bfloat16, device=DEV)
    codes = torch.full((N, K // 2), 0x22, dtype=torch.uint8, device=DEV)   # two codes of 1.0
    sb = torch.full((N, K // 16), 0x38, dtype=torch.uint8, device=DEV)      # E4M3 1.0
    ts = torch.tensor([0.25], device=DEV)
    c = Q.nvfp4_gemm_w4a16(x, codes, sb, ts)
    _check_clean()
    assert torch.equal(c, torch.full((M, N), K * 0.25, dtype=torch.bfloat16, device=DEV))


def test_strided_output_and_activations():
    M, N, K = 200, 384, 512
    big = S.activations(M, K + 64, seed=3, device=DEV)
    x = big[:, 64:]                                  # lda = K + 64
    w = S.weights(N, K, seed=4, device=DEV)
    (codes, sb, sg), (dc, dsb, dsg) = _oracle_weights(w)
    out = torch.full((M, N + 8), 7.0, dtype=torch.bfloat16, device=DEV)
    Q.nvfp4_gemm_w4a16(x, dc, dsb, dsg, out=out[:, :N])
    _check_clean()
    assert torch.all(out[:, N:] == 7.0)
    ref = O.gemm_w4a16(x.float().cpu().numpy(), codes, sb, sg, K)
    assert _rel_fro(out[:, :N].double().cpu().numpy(), _bf16_round(ref)) <= GEMM_RTOL


def test_bad_arguments_are_rejected():
    x = torch.zeros(4, 96, dtype=torch.bfloat16, device=DEV)   # K % 64 != 0
    codes = torch.zeros(8, 48, dtype=torch.uint8, device=DEV)
    sb = torch.zeros(8, 6, dtype=torch.uint8, device=DEV)
    ts = torch.ones(1, device=DEV)
    with pytest.raises(RuntimeError):
        Q.nvfp4_gemm_w4a16(x, codes, sb, ts)
