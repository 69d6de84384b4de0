"""GPU parity of the W4A4 block-scaled FP4 GEMM against the oracle.

The GPU quantizes both operands (codes + MMA-layout scales, bit-exact with
the oracle by the quantize tests) and runs the tcgen05 GEMM; the oracle
quantizes the same host bits itself and sums the exact products in float64.
Bar: relative Frobenius error <= 1e-3 against the oracle rounded to bf16.
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


def _gpu_operand(x):
    codes, sf, ts = Q.nvfp4_quantize(x, Q.DYNAMIC, layout=Q.SCALES_MMA)
    return codes, sf, ts


def _oracle_operand(x):
    return O.quantize(x.float().cpu().numpy(), O.DYNAMIC)


def _bf16_round(c):
    return O.bf16_bits_to_f32(O.bf16_round(c)).astype(np.float64)


def _run(x, w, rows=None):
    a = _gpu_operand(x)
    b = _gpu_operand(w)
    c = Q.nvfp4_gemm_w4a4(*a, *b)
    torch.cuda.synchronize()
    st, word = Q.nvfp4_device_error()
    assert st == 0 and word == 0
    ca, sa, ga = _oracle_operand(x)
    cb, sb, gb = _oracle_operand(w)
    K = x.shape[1]
    if rows is None:
        ref = O.gemm_w4a4(ca, sa, ga, cb, sb, gb, K)
        got = c.double().cpu().numpy()
    else:
        ref = O.gemm_w4a4_rows(ca, sa, ga, cb, sb, gb, K, rows)
        got = c[torch.as_tensor(rows, device=DEV)].double().cpu().numpy()
    err = _rel_fro(got, _bf16_round(ref))
    assert err <= GEMM_RTOL, err
    return c, ref


def test_tiny_qad_linear():
    d = S.tiny_qad_linear(seed=0, device=DEV)
    _run(d["x"], d["w"])


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (127, 100, 192), (129, 256, 320), (200, 300, 1024),
                                   (64, 520, 256), (256, 512, 576), (3, 1000, 2048), (5, 1002, 1024),
                                   (130, 4096, 4096), (1, 256, 8192),
                                   # more tiles than resident CTAs (several per CTA), long K
                                   (2304, 2560, 576), (300, 520, 4096)])
def test_ragged_shapes(M, N, K):
    x = S.activations(M, K, seed=M + K, device=DEV)
    w = S.weights(N, K, seed=N + K, device=DEV)
    _run(x, w)


def test_all_ones_closed_form():
    # q = 1.0 everywhere, s_b = 1.0, s_g = 1/448*... -> C = K * s_gA * s_gB exactly
    M, N, K = 130, 260, 512
    a_codes = torch.full((M, K // 2), 0x22, dtype=torch.uint8, device=DEV)  # two codes of 1.0
    b_codes = torch.full((N, K // 2), 0x22, dtype=torch.uint8, device=DEV)
    a_sf = torch.full((Q.mma_scales_bytes(M, K),), 0x38, dtype=torch.uint8, device=DEV)
    b_sf = torch.full((Q.mma_scales_bytes(N, K),), 0x38, dtype=torch.uint8, device=DEV)
    ta = torch.tensor([0.5], device=DEV)
    tb = torch.tensor([0.25], device=DEV)
    c = Q.nvfp4_gemm_w4a4(a_codes, a_sf, ta, b_codes, b_sf, tb)
    assert torch.all(c.float() == K * 0.125)


def test_integer_operands_exact():
    # small integer E2M1 values with power-of-two block scales: every partial
    # sum is exact in fp32, so the bf16-rounded result equals the oracle's
    rng = np.random.default_rng(0)
    M, N, K = 64, 128, 256
    int_codes = np.array([0, 2, 4, 5, 6, 10, 12, 13], np.uint8)
    qa = rng.choice(int_codes, (M, K))
    qb = rng.choice(int_codes, (N, K))
    pack = lambda q: (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    sa = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (M, K // 16))
    sb = rng.choice(np.array([0x30, 0x38, 0x40], np.uint8), (N, K // 16))
    c = Q.nvfp4_gemm_w4a4(torch.from_numpy(pack(qa)).to(DEV), torch.from_numpy(O.swizzle_scales(sa, K)).to(DEV),
                          torch.ones(1, device=DEV), torch.from_numpy(pack(qb)).to(DEV),
                          torch.from_numpy(O.swizzle_scales(sb, K)).to(DEV), torch.ones(1, device=DEV))
    ref = O.gemm_w4a4(pack(qa), sa, 1.0, pack(qb), sb, 1.0, K)
    assert np.array_equal(c.float().cpu().numpy(), _bf16_round(ref).astype(np.float32))


def test_w4a4_gemm_decode_shape():
    d = S.w4a4_gemm(128, seed=0, device=DEV)
    _run(d["x"], d["w"])


@pytest.mark.parametrize("M", [1, 127, 128, 129, 256])
def test_w4a4_gemm_small_m_split_k(M):
    """Decode-sized batches against a 4096 x 4096 weight run the split-K
    kernel (clusters of CTAs along K, partials added in rank order through
    distributed shared memory); parity as for every other shape."""
    d = S.w4a4_gemm(M, seed=M, device=DEV)
    rows = None if M <= 129 else np.concatenate([[0, 127, 128, 255], np.arange(1, 255, 9)])
    c1, _ = _run(d["x"], d["w"], rows=rows)
    # deterministic: the fixed rank order of the partial sums gives the same bits every call
    a = _gpu_operand(d["x"])
    b = _gpu_operand(d["w"])
    c2 = Q.nvfp4_gemm_w4a4(*a, *b)
    assert torch.equal(c1.view(torch.int16), c2.view(torch.int16))


def test_w4a4_gemm_prefill_shape_sampled():
    d = S.w4a4_gemm(8192, seed=0, device=DEV)
    rows = np.sort(np.random.default_rng(1).choice(8192, 96, replace=False))
    rows = np.concatenate([[0, 127, 128, 8191], rows])
    _run(d["x"], d["w"], rows=rows)


def test_matches_cublaslt_nvfp4():
    # library cross-check of the MMA scale layout: torch._scaled_mm on FP4
    # operands with the same swizzled E4M3 scales (cuBLASLt), tensor scales
    # applied outside.
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("torch has no float4 dtype")
    M, N, K = 256, 512, 1024
    x = S.activations(M, K, seed=3, device=DEV)
    w = S.weights(N, K, seed=4, device=DEV)
    ac, asf, ats = _gpu_operand(x)
    bc, bsf, bts = _gpu_operand(w)
    ours = Q.nvfp4_gemm_w4a4(ac, asf, ats, bc, bsf, bts).float()
    try:
        ref = torch._scaled_mm(ac.view(torch.float4_e2m1fn_x2), bc.view(torch.float4_e2m1fn_x2).t(),
                               asf.view(torch.float8_e4m3fn), bsf.view(torch.float8_e4m3fn),
                               out_dtype=torch.float32)
    except Exception as e:  # pragma: no cover - depends on the torch/cuBLASLt build
        pytest.skip(f"torch._scaled_mm has no NVFP4 path here: {e}")
    ref = ref * (ats * bts)
    err = float((ours - ref).norm() / ref.norm())
    assert err <= 2 * GEMM_RTOL, err


def _grouped_case(rows, N, K, seed):
    """Builds a grouped problem: segments padded to 128 rows, stacked B."""
    groups = len(rows)
    offs = [0]
    for r in rows:
        offs.append(offs[-1] + (r + 127) // 128 * 128)
    total = max(offs[-1], 128)
    xs = [S.activations(r, K, seed=seed + g, device=DEV) for g, r in enumerate(rows)]
    ws = [S.weights(N, K, seed=seed + 100 + g, device=DEV) for g in range(groups)]
    a_codes = torch.zeros(total, K // 2, dtype=torch.uint8, device=DEV)
    a_sf = torch.zeros(Q.mma_scales_bytes(total, K), dtype=torch.uint8, device=DEV)
    a_ts = torch.empty(groups, device=DEV)
    kchunks = K // 64
    for g, x in enumerate(xs):
        if rows[g] == 0:
            a_ts[g] = 1.0
            continue
        c, sf, ts = Q.nvfp4_quantize(x, layout=Q.SCALES_MMA)
        a_codes[offs[g]:offs[g] + rows[g]] = c
        seg = (offs[g + 1] - offs[g]) // 128 * kchunks * 512
        a_sf[offs[g] // 128 * kchunks * 512: offs[g] // 128 * kchunks * 512 + sf.numel()] = sf
        a_ts[g] = ts[0]
    bc, bsf, bts = Q.nvfp4_quantize_grouped(ws, Q.DYNAMIC, layout=Q.SCALES_MMA)
    b_codes = torch.cat(bc)
    b_sf = torch.cat(bsf)
    off_t = torch.tensor(offs, dtype=torch.int32, device=DEV)
    rows_t = torch.tensor(rows, dtype=torch.int32, device=DEV)
    return xs, ws, offs, a_codes, a_sf, a_ts, off_t, rows_t, b_codes, b_sf, bts


@pytest.mark.parametrize("rows,N,K", [([200, 0, 128, 1, 300], 384, 512), ([192] * 7 + [4096], 1024, 2048)])
def test_grouped_gemm_matches_oracle_per_group(rows, N, K):
    xs, ws, offs, a_codes, a_sf, a_ts, off_t, rows_t, b_codes, b_sf, bts = _grouped_case(rows, N, K, seed=len(rows))
    c = Q.nvfp4_gemm_w4a4_grouped(a_codes, a_sf, a_ts, off_t, rows_t, b_codes, b_sf, bts, N)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error()[0] == 0
    for g, r in enumerate(rows):
        if r == 0:
            continue
        ca, sa, ga = _oracle_operand(xs[g])
        cb, sb, gb = _oracle_operand(ws[g])
        sel = np.arange(r) if r <= 512 else np.sort(np.random.default_rng(g).choice(r, 256, replace=False))
        ref = O.gemm_w4a4_rows(ca, sa, ga, cb, sb, gb, K, sel)
        got = c[offs[g]:offs[g] + r][torch.as_tensor(sel, device=DEV)].double().cpu().numpy()
        err = _rel_fro(got, _bf16_round(ref))
        assert err <= GEMM_RTOL, (g, err)
