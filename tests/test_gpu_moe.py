"""GPU parity of the MoE layer step (qad_moe_forward / qad_moe_backward) and
of its BF16 grouped GEMM against the oracle.

Bars:
  * routing, weight codes, the routed tokens' codes, block scales and
    dequantized rows: bit-exact;
  * the SwiGLU output's codes: bit-exact on every 16-element block whose
    input (the bf16 SwiGLU output) equals the oracle's bit for bit;
  * floating-point outputs (bf16 tensors): relative Frobenius error against
    the oracle <= MOE_RTOL.  Both sides round to bf16 at the same points;
    what remains is the FP32 accumulation of the GPU GEMMs (~1e-6 relative)
    turning into occasional one-ulp bf16 differences (2^-8 relative) and,
    downstream of those, rare one-step E2M1 differences in the quantized
    SwiGLU output.  The largest error measured on the layer shapes below is
    3.3e-4 (dx), so the bar is the GEMM's 1e-3.
  * BF16 grouped GEMM: relative Frobenius error <= 1e-3 against float64
    products rounded to bf16.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import moe as OM
import nvfp4_quantization_aware_b200 as Q
from nvfp4_quantization_aware_b200 import synthetic as S
from moe_cases import f64, oracle_layer, remap_unused

pytestmark = pytest.mark.gpu
DEV = "cuda"
MOE_RTOL = 1e-3
GEMM_RTOL = 1e-3


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _bf(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _gpu_weights(d: dict, device=DEV):
    """Frozen weight scales from the library's DYNAMIC quantization of the
    calibration weights, the master weights, and the activation scales."""
    out = {}
    for k in ("gate", "up", "down"):
        w0 = d["w0_" + k].to(device)
        G, rows, cols = w0.shape
        _, sbs, ts = Q.nvfp4_quantize_grouped([w0[g] for g in range(G)], Q.DYNAMIC)
        sb = torch.cat(sbs).contiguous()
        out["w_" + k] = d["w_" + k].to(device).reshape(G * rows, cols).contiguous()
        out[k + "_ts"] = ts
        out[k + "_sb"] = sb
        out[k + "_sb_mma"] = Q.nvfp4_scales_to_mma(sb, G * rows, cols)
    out["x_ts"] = d["x_ts"].to(device)
    out["a_ts"] = d["a_ts"].to(device)
    return out


def _run_step(d, save_act=True):
    T, H = d["x"].shape
    G, F, _ = d["w_gate"].shape
    k = d["ids"].shape[1]
    w = _gpu_weights(d)
    step = Q.MoeLayerStep(T, H, F, G - 1, k, w, save_act=save_act)
    x, ids, cw, dy = (d[n].to(DEV) for n in ("x", "ids", "combine", "dy"))
    y = step.forward(x, ids, cw)
    grads = step.backward(dy)
    torch.cuda.synchronize()
    st, word = Q.nvfp4_device_error()
    assert st == 0 and word == 0
    return step, w, y, grads


def _small_case(seed=0, tokens=200, hidden=256, ffn=256, experts=8, topk=2, unused=3):
    d = S.moe_layer(seed=seed, tokens=tokens, hidden=hidden, ffn=ffn, experts=experts, topk=topk)
    if unused is not None:
        d["ids"] = remap_unused(d["ids"], unused, experts)
    return d


@pytest.mark.parametrize("case", [dict(), dict(seed=1, tokens=130, hidden=512, ffn=256, experts=5, topk=3,
                                             unused=None)])
def test_moe_step_matches_oracle(case):
    d = _small_case(**case)
    step, w, y, (dx, dwg, dwu, dwd, dcw) = _run_step(d)
    L = oracle_layer(d)
    ref = OM.layer_step(L, f64(d["dy"]))
    E = L.experts
    G = E + 1
    T, H = L.x.shape
    F = L.w_gate.shape[1]

    # routing (exact)
    seg_len = step.buffer("seg_len").cpu().numpy()
    seg_off = step.buffer("seg_off").cpu().numpy()
    row_token = step.buffer("row_token").cpu().numpy()
    row_weight = step.buffer("row_weight").cpu().numpy()
    slot_row = step.buffer("slot_row").cpu().numpy()
    off = 0
    for g, (t, j) in enumerate(ref["segments"]):
        assert seg_len[g] == len(t) and seg_off[g] == off
        assert np.array_equal(row_token[off:off + len(t)], t)
        pad = (len(t) + 127) // 128 * 128
        assert np.all(row_token[off + len(t):off + pad] == -1)
        if j is not None:
            assert np.array_equal(row_weight[off:off + len(t)], L.cw[t, j].astype(np.float32))
            assert np.array_equal(slot_row[t, j], off + np.arange(len(t)))
        off += pad
    assert seg_off[G] == off

    # weight codes (exact)
    for kind, buf in (("gate", "wg_codes"), ("up", "wu_codes"), ("down", "wd_codes")):
        codes = step.buffer(buf).cpu().numpy()
        rows = codes.shape[0] // G
        for g in range(G):
            assert np.array_equal(codes[g * rows:(g + 1) * rows], L.weight(kind, g)[0]), (kind, g)

    # dequantized weights the backward uses (exact)
    wd_hat = step.buffer("wd_hat").view(torch.int16).cpu().numpy().view(np.uint16)
    wgu_hat = step.buffer("wgu_hat").view(torch.int16).cpu().numpy().view(np.uint16)
    for g in range(G):
        assert np.array_equal(wd_hat[g * H:(g + 1) * H], O.bf16_round(L.weight("down", g)[3])), g
        assert np.array_equal(wgu_hat[2 * g * F:2 * g * F + F], O.bf16_round(L.weight("gate", g)[3])), g
        assert np.array_equal(wgu_hat[2 * g * F + F:2 * (g + 1) * F], O.bf16_round(L.weight("up", g)[3])), g

    # routed rows: codes, MMA scales, dequantized rows (exact); padding zero
    xc = step.buffer("x_codes").cpu().numpy()
    xs = step.buffer("x_scales").cpu().numpy()
    xh = step.buffer("x_hat").view(torch.int16).cpu().numpy().view(np.uint16)
    R = xc.shape[0]
    want_c = np.zeros_like(xc)
    want_sb = np.zeros((R, H // 16), np.uint8)
    want_h = np.zeros_like(xh)
    for g in range(G):
        st = ref["groups"][g]["fwd"]
        if st is None:
            continue
        o, n = seg_off[g], seg_len[g]
        want_c[o:o + n], want_sb[o:o + n] = st["x_codes"], st["x_sb"]
        want_h[o:o + n] = O.bf16_round(st["x_hat"])
    assert np.array_equal(xc, want_c)
    assert np.array_equal(xs, O.swizzle_scales(want_sb, H))
    assert np.array_equal(xh, want_h)

    # gate / up products, SwiGLU output (tolerance), its codes (exact where the inputs agree)
    # rows past the last segment are never written: only segment rows are read
    hg, hu, act = step.buffer("h_gate"), step.buffer("h_up"), step.buffer("act")
    act_bits = act.view(torch.int16).cpu().numpy().view(np.uint16)
    ac = step.buffer("a_codes").cpu().numpy()
    compared = total = 0
    for g in range(G):
        st = ref["groups"][g]["fwd"]
        if st is None:
            continue
        o, n = seg_off[g], seg_len[g]
        assert _rel(_bf(hg[o:o + n]), st["h_gate"]) <= MOE_RTOL
        assert _rel(_bf(hu[o:o + n]), st["h_up"]) <= MOE_RTOL
        a_ref_bits = O.bf16_round(st["a"])
        assert _rel(O.bf16_bits_to_f32(act_bits[o:o + n]).astype(np.float64), st["a"]) <= MOE_RTOL
        same = np.all((act_bits[o:o + n] == a_ref_bits).reshape(n, F // 16, 16), axis=2)
        got_c = ac[o:o + n].reshape(n, F // 16, 8)
        want_c = st["a_codes"].reshape(n, F // 16, 8)
        assert np.array_equal(got_c[same], want_c[same]), g
        compared += int(same.sum())
        total += same.size
    assert compared >= 0.98 * total, (compared, total)

    # layer outputs and gradients (tolerance)
    assert _rel(_bf(y), ref["y"]) <= MOE_RTOL
    assert _rel(_bf(dx), ref["dx"]) <= MOE_RTOL
    dcw_g = dcw.cpu().numpy().astype(np.float64)
    assert _rel(dcw_g, ref["d_combine"]) <= MOE_RTOL
    dwg, dwu, dwd = _bf(dwg), _bf(dwu), _bf(dwd)
    for g in range(G):
        b = ref["groups"][g]["bwd"]
        sl_f, sl_h = slice(g * F, (g + 1) * F), slice(g * H, (g + 1) * H)
        if b is None:
            assert not dwg[sl_f].any() and not dwu[sl_f].any() and not dwd[sl_h].any()
            continue
        assert _rel(dwg[sl_f], b["dW_gate"]) <= MOE_RTOL, g
        assert _rel(dwu[sl_f], b["dW_up"]) <= MOE_RTOL, g
        assert _rel(dwd[sl_h], b["dW_down"]) <= MOE_RTOL, g


@pytest.mark.slow
def test_moe_step_full_size_sampled():
    # 4096 tokens x 2048 hidden, 128 routed experts + 1 shared, top-6, FFN
    # 1024, in the launch configuration the benchmark times; the oracle
    # checks sampled tokens (their 7 experts) and the weight gradients of
    # sampled experts (all of their rows).
    d = S.moe_layer(seed=0, device=DEV)
    step, w, y, (dx, dwg, dwu, dwd, dcw) = _run_step(d, save_act=False)
    dh = {k: v.cpu() for k, v in d.items()}
    ids = dh["ids"].numpy()
    tok = [0, 1234, 4095]
    experts = [int(ids[1234, 0]), int(ids[77, 2])]
    groups = sorted(set(ids[tok].ravel().tolist()) | set(experts) | {128})
    L = oracle_layer(dh, groups=groups)
    G, F, H = 129, 1024, 2048
    # routing (exact)
    seg_len = step.buffer("seg_len").cpu().numpy()
    segs = OM.route(L.ids, 128)
    assert np.array_equal(seg_len, [len(t) for t, _ in segs])
    for kind, buf in (("gate", "wg_codes"), ("up", "wu_codes"), ("down", "wd_codes")):
        codes = step.buffer(buf)
        rows = codes.shape[0] // G
        for g in experts + [128]:
            assert np.array_equal(codes[g * rows:(g + 1) * rows].cpu().numpy(), L.weight(kind, g)[0]), (kind, g)
    dy = f64(dh["dy"])
    y_g, dx_g, dcw_g = _bf(y), _bf(dx), dcw.cpu().numpy()
    for t in tok:
        yt = np.zeros(H)
        dxt = np.zeros(H)
        for j in range(6):
            e = int(ids[t, j])
            st = OM.expert_forward(L, e, L.x[t:t + 1])
            dyp = OM.to_bf16(L.cw[t, j] * dy[t:t + 1])
            dxt += OM.expert_backward(L, e, st, dyp)["dX"][0]
            yt += L.cw[t, j] * st["y"][0]
            assert abs(dcw_g[t, j] - float(dy[t] @ st["y"][0])) <= MOE_RTOL * np.linalg.norm(dy[t]) * \
                np.linalg.norm(st["y"][0])
        st = OM.expert_forward(L, 128, L.x[t:t + 1])
        yt += st["y"][0]
        dxt += OM.expert_backward(L, 128, st, OM.to_bf16(dy[t:t + 1]))["dX"][0]
        assert _rel(y_g[t], OM.to_bf16(yt)) <= MOE_RTOL, t
        assert _rel(dx_g[t], OM.to_bf16(dxt)) <= MOE_RTOL, t
    dwg, dwu, dwd = dwg.cpu(), dwu.cpu(), dwd.cpu()
    for e in experts:
        t, j = segs[e]
        st = OM.expert_forward(L, e, L.x[t])
        b = OM.expert_backward(L, e, st, OM.to_bf16(L.cw[t, j][:, None] * dy[t]))
        assert _rel(_bf(dwg[e * F:(e + 1) * F]), b["dW_gate"]) <= MOE_RTOL, e
        assert _rel(_bf(dwu[e * F:(e + 1) * F]), b["dW_up"]) <= MOE_RTOL, e
        assert _rel(_bf(dwd[e * H:(e + 1) * H]), b["dW_down"]) <= MOE_RTOL, e


# ------------------------------------------------------------------ BF16 grouped GEMM

def _segments(lens, align=128):
    off = [0]
    for n in lens:
        off.append(off[-1] + (n + align - 1) // align * align)
    return off


MAJORS = [(False, False), (False, True), (True, False), (True, True)]


def _padded(x: torch.Tensor) -> torch.Tensor:
    """x on the device in a buffer whose row stride is a multiple of 8 elements."""
    rows, cols = x.shape
    buf = torch.zeros(rows, (cols + 7) // 8 * 8, dtype=x.dtype, device=DEV)
    buf[:, :cols] = x.to(DEV)
    return buf[:, :cols]


@pytest.mark.parametrize("a_mn,b_mn", MAJORS)
@pytest.mark.parametrize("lens,N,K", [([200, 0, 128, 1, 300], 256, 192), ([192] * 5 + [700], 512, 1024),
                                      ([5], 768, 64)])
def test_bf16_grouped_gemm_m_segments(lens, N, K, a_mn, b_mn):
    g = torch.Generator().manual_seed(len(lens) + N)
    off = _segments(lens)
    R = max(off[-1], 128)
    G = len(lens)
    a = torch.randn(R, K, generator=g).to(torch.bfloat16)                 # logical A [R x K]
    b = (torch.randn(G, N, K, generator=g) * 0.1).to(torch.bfloat16)      # logical B_g [N x K]
    a_st = a.t().contiguous() if a_mn else a
    b_st = b.transpose(1, 2).reshape(G * K, N).contiguous() if b_mn else b.reshape(G * N, K)
    c = Q.nvfp4_gemm_bf16_grouped(0, a_st.to(DEV), b_st.to(DEV), torch.tensor(off, dtype=torch.int32, device=DEV),
                                  torch.tensor(lens, dtype=torch.int32, device=DEV), 0, N, K,
                                  a_mn_major=a_mn, b_mn_major=b_mn)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error()[0] == 0
    a64, b64 = a.double(), b.double()
    for i, n in enumerate(lens):
        if n == 0:
            continue
        want = (a64[off[i]:off[i] + n] @ b64[i].T).to(torch.bfloat16).double().numpy()
        assert _rel(c[off[i]:off[i] + n].double().cpu().numpy(), want) <= GEMM_RTOL, i


@pytest.mark.parametrize("a_mn,b_mn", MAJORS)
@pytest.mark.parametrize("lens,M,N", [([200, 0, 128, 1, 300], 256, 512), ([192] * 4, 1024, 256), ([64], 130, 260)])
def test_bf16_grouped_gemm_k_segments(lens, M, N, a_mn, b_mn):
    g = torch.Generator().manual_seed(len(lens) + M)
    off = _segments(lens)
    R = max(off[-1], 128)
    a = torch.zeros(M, R)
    b = torch.zeros(N, R)
    for i, n in enumerate(lens):
        a[:, off[i]:off[i] + n] = torch.randn(M, n, generator=g)
        b[:, off[i]:off[i] + n] = torch.randn(N, n, generator=g) * 0.1
    a, b = a.to(torch.bfloat16), b.to(torch.bfloat16)
    # MN-major storage: the M / N index contiguous, rows padded to 16 bytes
    a_st = _padded(a.t()) if a_mn else a.to(DEV)
    b_st = _padded(b.t()) if b_mn else b.to(DEV)
    c = Q.nvfp4_gemm_bf16_grouped(1, a_st, b_st, torch.tensor(off, dtype=torch.int32, device=DEV),
                                  torch.tensor(lens, dtype=torch.int32, device=DEV), M, N, 0,
                                  a_mn_major=a_mn, b_mn_major=b_mn)
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error()[0] == 0
    a64, b64 = a.double(), b.double()
    for i, n in enumerate(lens):
        got = c[i * M:(i + 1) * M].double().cpu().numpy()
        if n == 0:
            assert not got.any()
            continue
        want = (a64[:, off[i]:off[i] + n] @ b64[:, off[i]:off[i] + n].T).to(torch.bfloat16).double().numpy()
        assert _rel(got, want) <= GEMM_RTOL, i


def test_quantize_fake_quant_grouped_matches_oracle():
    G, rows, cols = 3, 136, 96
    w = [S.weights(rows, cols, seed=g) for g in range(G)]
    wd = [x.to(DEV) for x in w]
    _, sbs, ts = Q.nvfp4_quantize_grouped(wd, Q.DYNAMIC)
    ys = [torch.zeros(rows, cols + 8, dtype=torch.bfloat16, device=DEV)[:, 8:] for _ in range(G)]
    codes, ys = Q.nvfp4_quantize_fake_quant_grouped(wd, Q.FROZEN_ALL, ts, sbs, ys=ys)
    for g in range(G):
        oc, osb, osg = O.quantize(w[g].float().numpy(), O.DYNAMIC)
        _, bits, _, _ = O.fake_quant(w[g].float().numpy(), O.FROZEN_ALL, s_g=osg, s_b=osb)
        assert np.array_equal(codes[g].cpu().numpy(), oc), g
        assert np.array_equal(ys[g].contiguous().view(torch.int16).cpu().numpy().view(np.uint16), bits), g


def test_scales_to_mma_matches_oracle_swizzle():
    sb = torch.randint(0, 127, (300, 20), dtype=torch.uint8, generator=torch.Generator().manual_seed(1))
    got = Q.nvfp4_scales_to_mma(sb.to(DEV), 300, 320).cpu().numpy()
    assert np.array_equal(got, O.swizzle_scales(sb.numpy(), 320))


def test_route_marks_out_of_range_ids():
    ids = torch.tensor([[0, 1], [5, 1], [2, -1]], dtype=torch.int32, device=DEV)
    cw = torch.full((3, 2), 0.5, device=DEV)
    E = 4
    R = int(Q.lib().nvfp4_moe_rows_capacity(3, 2, E))
    seg_len = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    seg_off = torch.empty(E + 2, dtype=torch.int32, device=DEV)
    row_token = torch.empty(R, dtype=torch.int32, device=DEV)
    row_weight = torch.empty(R, device=DEV)
    slot_row = torch.empty(3, 2, dtype=torch.int32, device=DEV)
    st = Q.lib().nvfp4_moe_route(ids.data_ptr(), cw.data_ptr(), 3, 2, E, seg_len.data_ptr(), seg_off.data_ptr(),
                                 row_token.data_ptr(), row_weight.data_ptr(), slot_row.data_ptr(), R,
                                 torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    err = Q.nvfp4_device_error()
    assert err == (7, 3)
    assert seg_len.cpu().tolist() == [1, 2, 1, 0, 3]
    s = slot_row.cpu().numpy()
    assert s[1, 0] == -1 and s[2, 1] == -1
    assert s[0, 0] == 0 and s[0, 1] == 128 and s[1, 1] == 129 and s[2, 0] == 256


# ------------------------------------------------------------------ combine / gather-sum at any width

def _combine_case(tokens, topk, cols, experts, seed, dyadic):
    """A row buffer of expert outputs, each token's slot rows (distinct rows,
    some slots routed nowhere) and the shared rows after the routed ones."""
    g = torch.Generator().manual_seed(seed)
    shared_base = tokens * topk + 5
    rows = shared_base + tokens
    if dyadic:
        # small multiples of 1/8 and power-of-two weights: every binary32 sum is exact
        y = (torch.randint(-64, 65, (rows, cols), generator=g).float() / 8).to(torch.bfloat16)
        w = 2.0 ** torch.randint(-3, 2, (tokens, topk), generator=g).float()
    else:
        y = torch.randn(rows, cols, generator=g).to(torch.bfloat16)
        w = torch.rand(tokens, topk, generator=g)
    slot = torch.randperm(shared_base, generator=g)[:tokens * topk].reshape(tokens, topk).to(torch.int32)
    slot[torch.rand(tokens, topk, generator=g) < 0.1] = -1
    seg_off = torch.zeros(experts + 2, dtype=torch.int32)
    seg_off[experts:] = shared_base
    return y, w, slot, seg_off, shared_base


@pytest.mark.parametrize("cols", [8, 40, 264, 2048])
@pytest.mark.parametrize("dyadic", [True, False])
def test_combine_and_gather_sum_any_width(cols, dyadic):
    """cols need only be a multiple of 8; widths whose 16-byte vectors do not
    fill whole warps exercise the lanes with no vector."""
    tokens, topk, experts = 37, 6, 4
    y, w, slot, seg_off, base = _combine_case(tokens, topk, cols, experts, seed=cols, dyadic=dyadic)
    yd, wd, sd, od = y.to(DEV), w.to(DEV), slot.to(DEV), seg_off.to(DEV)
    out = torch.empty(tokens, cols, dtype=torch.bfloat16, device=DEV)
    dx = torch.empty(tokens, cols, dtype=torch.bfloat16, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    assert Q.lib().nvfp4_moe_combine(yd.data_ptr(), cols, sd.data_ptr(), wd.data_ptr(), tokens, topk, od.data_ptr(),
                                     experts, out.data_ptr(), stream) == 0
    assert Q.lib().nvfp4_moe_gather_sum(yd.data_ptr(), cols, sd.data_ptr(), tokens, topk, od.data_ptr(), experts,
                                        dx.data_ptr(), stream) == 0
    torch.cuda.synchronize()
    assert Q.nvfp4_device_error() == (0, 0)
    y64, s_np = _bf(y), slot.numpy()
    want_out = OM.combine_rows(y64, s_np, w.double().numpy(), base)
    want_dx = OM.gather_sum_rows(y64, s_np, base)
    if dyadic:
        assert np.array_equal(_bf(out), want_out)
        assert np.array_equal(_bf(dx), want_dx)
    else:
        assert _rel(_bf(out), want_out) <= MOE_RTOL
        assert _rel(_bf(dx), want_dx) <= MOE_RTOL
