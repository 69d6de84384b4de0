// moe_step.cu -- one training step of the QAD student's MoE layer as a fixed
// sequence of this library's kernels on one stream (host code only).
//
// Forward (W4A4 NVFP4 with frozen scales: Qwen3.6-35B-A3B W4A4 tutorial,
// "2. PTQ"; Nemotron 3.5 Lightning NVFP4 article, "量化尺度处理策略"):
//   route -> quantize the master weights with their frozen scales ->
//   gather + quantize the routed tokens (frozen tensor scale, block scales
//   from the data) -> grouped W4A4 GEMMs gate and up -> SwiGLU + quantize ->
//   grouped W4A4 GEMM down -> weighted combine with the shared expert.
// Backward (straight-through estimator: every quantizer passes its gradient
// unchanged, so gradients are plain BF16 products with the dequantized
// operands the forward used):
//   dY_g = w * dy  ->  dA = dY_g W^_down  ->  SwiGLU backward -> [dG | dU]
//   (every product reads the forward's buffers in place: the BF16 GEMM takes
//   MN-major operands, and the forward's weight quantizer also writes W^)
//   dX_g = [dG | dU] [W^_gate; W^_up]  -> dx = sum over the token's experts
//   dW_down = dY_g^T A^,  dW_gate = dG^T X^,  dW_up = dU^T X^,
//   d(combine weight) = <dy, y_expert>.
#include <cstring>

#include "moe_internal.cuh"

namespace {

struct Layout {
  int64_t rows_cap;
  size_t off[QAD_MOE_NUM_BUFFERS];
  size_t bytes[QAD_MOE_NUM_BUFFERS];
  size_t total;
};

bool shape_ok(const qad_moe_shape* s) {
  return s && s->tokens >= 1 && s->topk >= 1 && s->experts >= 1 && s->experts + 1 <= 256 && s->hidden >= 256 &&
         s->hidden % 256 == 0 && s->ffn >= 256 && s->ffn % 256 == 0 && s->topk <= s->experts && s->topk <= 32 &&
         (int64_t)s->tokens * s->topk <= (1 << 26) && (int64_t)(s->experts + 1) * s->hidden * s->ffn * 2 < (1ll << 40);
}

Layout layout_of(const qad_moe_shape& s) {
  Layout L;
  const int64_t G = s.experts + 1, T = s.tokens, H = s.hidden, F = s.ffn;
  const int64_t R = nvfp4_moe_rows_capacity(s.tokens, s.topk, s.experts);
  L.rows_cap = R;
  size_t* b = L.bytes;
  b[QAD_MOE_SEG_LEN] = 4 * G;
  b[QAD_MOE_SEG_OFF] = 4 * (G + 1);
  b[QAD_MOE_ROW_TOKEN] = 4 * R;
  b[QAD_MOE_ROW_WEIGHT] = 4 * R;
  b[QAD_MOE_SLOT_ROW] = 4 * T * s.topk;
  b[QAD_MOE_X_CODES] = R * H / 2;
  b[QAD_MOE_X_SCALES] = nvfp4_mma_scales_bytes(R, H);
  b[QAD_MOE_X_HAT] = 2 * R * H;
  b[QAD_MOE_WG_CODES] = G * F * H / 2;
  b[QAD_MOE_WU_CODES] = G * F * H / 2;
  b[QAD_MOE_WD_CODES] = G * H * F / 2;
  b[QAD_MOE_H_GATE] = 2 * R * F;
  b[QAD_MOE_H_UP] = 2 * R * F;
  b[QAD_MOE_A_CODES] = R * F / 2;
  b[QAD_MOE_A_SCALES] = nvfp4_mma_scales_bytes(R, F);
  b[QAD_MOE_A_HAT] = 2 * R * F;
  b[QAD_MOE_ACT] = s.save_act ? 2 * R * F : 0;
  b[QAD_MOE_Y_ROWS] = 2 * R * H;
  b[QAD_MOE_DY_ROWS] = 2 * R * H;
  b[QAD_MOE_WD_HAT] = 2 * G * H * F;
  b[QAD_MOE_DA] = 2 * R * F;
  b[QAD_MOE_DGU] = 2 * R * 2 * F;
  b[QAD_MOE_WGU_HAT] = 2 * G * 2 * F * H;
  b[QAD_MOE_DX_ROWS] = 2 * R * H;
  size_t o = 0;
  for (int i = 0; i < QAD_MOE_NUM_BUFFERS; ++i) {
    L.off[i] = o;
    o += (b[i] + 255) / 256 * 256;
  }
  L.total = o;
  return L;
}

template <typename T>
T* at(void* ws, const Layout& L, int id) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + L.off[id]);
}

#define QAD_TRY(call)                        \
  do {                                       \
    const nvfp4_status st_ = (call);         \
    if (st_ != NVFP4_OK) return st_;         \
  } while (0)

nvfp4_status weights_ok(const qad_moe_weights* w) {
  if (!w || !w->w_gate || !w->w_up || !w->w_down || !w->gate_ts || !w->up_ts || !w->down_ts || !w->gate_sb ||
      !w->up_sb || !w->down_sb || !w->gate_sb_mma || !w->up_sb_mma || !w->down_sb_mma || !w->x_ts || !w->a_ts)
    return NVFP4_ERR_ARG;
  return NVFP4_OK;
}

}  // namespace

extern "C" {

size_t qad_moe_workspace_size(const qad_moe_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return layout_of(*shape).total;
}

nvfp4_status qad_moe_workspace_buffer(const qad_moe_shape* shape, int buffer, size_t* offset, size_t* bytes) {
  if (!shape_ok(shape)) return NVFP4_ERR_SHAPE;
  if (buffer < 0 || buffer >= QAD_MOE_NUM_BUFFERS || !offset || !bytes) return NVFP4_ERR_ARG;
  const Layout L = layout_of(*shape);
  *offset = L.off[buffer];
  *bytes = L.bytes[buffer];
  return NVFP4_OK;
}

int64_t qad_moe_rows_capacity(const qad_moe_shape* shape) {
  if (!shape_ok(shape)) return 0;
  return layout_of(*shape).rows_cap;
}

}  // extern "C"

namespace {

// The layer step; without `shared` there is no shared expert (group E holds
// no rows and its weights are not read), combine_weights may be NULL (weight
// 1), and G below counts the routed experts only.
nvfp4_status moe_forward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* x,
                         const int32_t* expert_ids, const float* combine_weights, void* y, void* workspace,
                         size_t workspace_bytes, void* stream, bool shared) {
  if (!shape_ok(shape)) return NVFP4_ERR_SHAPE;
  QAD_TRY(weights_ok(w));
  if (!x || !expert_ids || (shared && !combine_weights) || !y) return NVFP4_ERR_ARG;
  const qad_moe_shape& s = *shape;
  const Layout L = layout_of(s);
  if (!workspace || workspace_bytes < L.total) return NVFP4_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) || ((uintptr_t)x & 15u) || ((uintptr_t)y & 15u) || ((uintptr_t)w->w_gate & 15u) ||
      ((uintptr_t)w->w_up & 15u) || ((uintptr_t)w->w_down & 15u))
    return NVFP4_ERR_ALIGN;
  const int G = s.experts + (shared ? 1 : 0);
  const int64_t H = s.hidden, F = s.ffn, R = L.rows_cap;
  int32_t* seg_len = at<int32_t>(workspace, L, QAD_MOE_SEG_LEN);
  int32_t* seg_off = at<int32_t>(workspace, L, QAD_MOE_SEG_OFF);
  int32_t* row_token = at<int32_t>(workspace, L, QAD_MOE_ROW_TOKEN);
  float* row_weight = at<float>(workspace, L, QAD_MOE_ROW_WEIGHT);
  int32_t* slot_row = at<int32_t>(workspace, L, QAD_MOE_SLOT_ROW);

  // 1. routing: segments and the permutation
  QAD_TRY(nvfp4::moe::route(expert_ids, combine_weights, s.tokens, s.topk, s.experts, shared, seg_len, seg_off,
                            row_token, row_weight, slot_row, R, stream));
  // 2. master weights -> NVFP4 codes with their frozen scales, and the bf16
  //    dequantized weights the backward multiplies with (one call, 3G tensors):
  //    W^_gate / W^_up of group g interleaved as rows [2gF, 2gF + F) / [2gF + F,
  //    2(g+1)F) of one stack, W^_down as its own stack
  {
    const __nv_bfloat16* wg = static_cast<const __nv_bfloat16*>(w->w_gate);
    const __nv_bfloat16* wu = static_cast<const __nv_bfloat16*>(w->w_up);
    const __nv_bfloat16* wd = static_cast<const __nv_bfloat16*>(w->w_down);
    uint8_t* cg = at<uint8_t>(workspace, L, QAD_MOE_WG_CODES);
    uint8_t* cu = at<uint8_t>(workspace, L, QAD_MOE_WU_CODES);
    uint8_t* cd = at<uint8_t>(workspace, L, QAD_MOE_WD_CODES);
    __nv_bfloat16* hgu = at<__nv_bfloat16>(workspace, L, QAD_MOE_WGU_HAT);
    __nv_bfloat16* hd = at<__nv_bfloat16>(workspace, L, QAD_MOE_WD_HAT);
    nvfp4_tensor_ref refs[3 * 256];
    void* ys[3 * 256];
    int64_t lds[3 * 256];
    for (int g = 0; g < G; ++g) {
      nvfp4_tensor_ref& a = refs[g];
      a.x = wg + (int64_t)g * F * H; a.rows = F; a.cols = H; a.ld_x = H;
      a.tensor_scale = const_cast<float*>(w->gate_ts + g);
      a.block_scales = const_cast<uint8_t*>(w->gate_sb + (int64_t)g * F * (H / 16));
      a.out = cg + (int64_t)g * F * (H / 2); a.ld_out = H / 2;
      ys[g] = hgu + (int64_t)g * 2 * F * H; lds[g] = H;
      nvfp4_tensor_ref& b = refs[G + g];
      b = a;
      b.x = wu + (int64_t)g * F * H;
      b.tensor_scale = const_cast<float*>(w->up_ts + g);
      b.block_scales = const_cast<uint8_t*>(w->up_sb + (int64_t)g * F * (H / 16));
      b.out = cu + (int64_t)g * F * (H / 2);
      ys[G + g] = hgu + (int64_t)g * 2 * F * H + F * H; lds[G + g] = H;
      nvfp4_tensor_ref& d = refs[2 * G + g];
      d.x = wd + (int64_t)g * H * F; d.rows = H; d.cols = F; d.ld_x = F;
      d.tensor_scale = const_cast<float*>(w->down_ts + g);
      d.block_scales = const_cast<uint8_t*>(w->down_sb + (int64_t)g * H * (F / 16));
      d.out = cd + (int64_t)g * H * (F / 2); d.ld_out = F / 2;
      ys[2 * G + g] = hd + (int64_t)g * H * F; lds[2 * G + g] = F;
    }
    QAD_TRY(nvfp4_quantize_fake_quant_grouped(3 * G, refs, ys, lds, NVFP4_BF16, NVFP4_FROZEN_ALL,
                                              NVFP4_SCALES_ROWMAJOR, nullptr, 0, stream));
  }
  // 3. gather the routed tokens and quantize them (frozen s_g per expert)
  QAD_TRY(nvfp4_moe_gather_quantize(x, H, row_token, seg_off, G, w->x_ts, R, H,
                                    at<uint8_t>(workspace, L, QAD_MOE_X_CODES),
                                    at<uint8_t>(workspace, L, QAD_MOE_X_SCALES),
                                    at<void>(workspace, L, QAD_MOE_X_HAT), stream));
  // 4. gate and up projections (grouped W4A4)
  QAD_TRY(nvfp4_gemm_w4a4_grouped(G, at<uint8_t>(workspace, L, QAD_MOE_X_CODES),
                                  at<uint8_t>(workspace, L, QAD_MOE_X_SCALES), w->x_ts, R, seg_off, seg_len,
                                  at<uint8_t>(workspace, L, QAD_MOE_WG_CODES), w->gate_sb_mma, w->gate_ts, F, H,
                                  at<void>(workspace, L, QAD_MOE_H_GATE), F, nullptr, 0, stream));
  QAD_TRY(nvfp4_gemm_w4a4_grouped(G, at<uint8_t>(workspace, L, QAD_MOE_X_CODES),
                                  at<uint8_t>(workspace, L, QAD_MOE_X_SCALES), w->x_ts, R, seg_off, seg_len,
                                  at<uint8_t>(workspace, L, QAD_MOE_WU_CODES), w->up_sb_mma, w->up_ts, F, H,
                                  at<void>(workspace, L, QAD_MOE_H_UP), F, nullptr, 0, stream));
  // 5. SwiGLU and quantize the down projection's input
  QAD_TRY(nvfp4_moe_swiglu_quantize(at<void>(workspace, L, QAD_MOE_H_GATE), at<void>(workspace, L, QAD_MOE_H_UP), F,
                                    row_token, seg_off, G, w->a_ts, R, F, at<uint8_t>(workspace, L, QAD_MOE_A_CODES),
                                    at<uint8_t>(workspace, L, QAD_MOE_A_SCALES), at<void>(workspace, L, QAD_MOE_A_HAT),
                                    s.save_act ? at<void>(workspace, L, QAD_MOE_ACT) : nullptr, stream));
  // 6. down projection
  QAD_TRY(nvfp4_gemm_w4a4_grouped(G, at<uint8_t>(workspace, L, QAD_MOE_A_CODES),
                                  at<uint8_t>(workspace, L, QAD_MOE_A_SCALES), w->a_ts, R, seg_off, seg_len,
                                  at<uint8_t>(workspace, L, QAD_MOE_WD_CODES), w->down_sb_mma, w->down_ts, H, F,
                                  at<void>(workspace, L, QAD_MOE_Y_ROWS), H, nullptr, 0, stream));
  // 7. combine
  return nvfp4::moe::combine(at<void>(workspace, L, QAD_MOE_Y_ROWS), H, slot_row, combine_weights, s.tokens, s.topk,
                             seg_off, s.experts, shared, y, stream);
}

nvfp4_status moe_backward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* dy, void* dx,
                          void* dw_gate, void* dw_up, void* dw_down, float* d_combine, void* workspace,
                          size_t workspace_bytes, void* stream, bool shared) {
  if (!shape_ok(shape)) return NVFP4_ERR_SHAPE;
  QAD_TRY(weights_ok(w));
  if (!dy || !dx || !dw_gate || !dw_up || !dw_down) return NVFP4_ERR_ARG;
  const qad_moe_shape& s = *shape;
  const Layout L = layout_of(s);
  if (!workspace || workspace_bytes < L.total) return NVFP4_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 255u) || ((uintptr_t)dy & 15u) || ((uintptr_t)dx & 15u) || ((uintptr_t)dw_gate & 15u) ||
      ((uintptr_t)dw_up & 15u) || ((uintptr_t)dw_down & 15u))
    return NVFP4_ERR_ALIGN;
  const int G = s.experts + (shared ? 1 : 0);
  const int64_t H = s.hidden, F = s.ffn, R = L.rows_cap;
  int32_t* seg_len = at<int32_t>(workspace, L, QAD_MOE_SEG_LEN);
  int32_t* seg_off = at<int32_t>(workspace, L, QAD_MOE_SEG_OFF);
  int32_t* row_token = at<int32_t>(workspace, L, QAD_MOE_ROW_TOKEN);
  float* row_weight = at<float>(workspace, L, QAD_MOE_ROW_WEIGHT);
  int32_t* slot_row = at<int32_t>(workspace, L, QAD_MOE_SLOT_ROW);
  void* dyp = at<void>(workspace, L, QAD_MOE_DY_ROWS);
  void* da = at<void>(workspace, L, QAD_MOE_DA);
  __nv_bfloat16* dgu = at<__nv_bfloat16>(workspace, L, QAD_MOE_DGU);
  void* dxp = at<void>(workspace, L, QAD_MOE_DX_ROWS);
  const void* xhat = at<void>(workspace, L, QAD_MOE_X_HAT);
  const void* ahat = at<void>(workspace, L, QAD_MOE_A_HAT);
  const void* wd_hat = at<void>(workspace, L, QAD_MOE_WD_HAT);    // [G H x F]
  const void* wgu_hat = at<void>(workspace, L, QAD_MOE_WGU_HAT);  // [G 2F x H]

  // dY of each routed row: combine weight times the token's output gradient
  QAD_TRY(nvfp4_moe_scale_rows(dy, H, row_token, row_weight, seg_off, G, R, dyp, stream));
  // dA = dY W^_down: A = dY rows (K-major, K = H), B_g[f][h] = W^_down_g[h][f]
  // (MN-major, the stack's K rows g H .. g H + H - 1)
  QAD_TRY(nvfp4_gemm_bf16_grouped(0, G, dyp, 0, R, H, H, wd_hat, 1, (int64_t)G * H, F, F, seg_off, seg_len, 0, F, H,
                                  da, F, stream));
  // SwiGLU backward -> [dG | dU]
  QAD_TRY(nvfp4_moe_swiglu_backward(da, at<void>(workspace, L, QAD_MOE_H_GATE), at<void>(workspace, L, QAD_MOE_H_UP), F,
                                    row_token, seg_off, G, R, dgu, stream));
  // dX rows = [dG | dU] [W^_gate; W^_up]: B_g[h][k] = W^_gu_g[k][h] (MN-major,
  // K rows 2 g F .. 2 (g+1) F - 1), then the sum over each token's experts
  QAD_TRY(nvfp4_gemm_bf16_grouped(0, G, dgu, 0, R, 2 * F, 2 * F, wgu_hat, 1, (int64_t)G * 2 * F, H, H, seg_off,
                                  seg_len, 0, H, 2 * F, dxp, H, stream));
  QAD_TRY(nvfp4::moe::gather_sum(dxp, H, slot_row, s.tokens, s.topk, seg_off, s.experts, shared, dx, stream));
  // weight gradients, reduced over each expert's rows (K-segments, both
  // operands MN-major: the row buffers as they are)
  //   dW_down_g[h][f] = sum_r dY[r][h] A^[r][f]
  QAD_TRY(nvfp4_gemm_bf16_grouped(1, G, dyp, 1, R, H, H, ahat, 1, R, F, F, seg_off, seg_len, H, F, 0, dw_down, F,
                                  stream));
  //   dW_gate_g[f][h] = sum_r dG[r][f] X^[r][h],  dW_up_g likewise with dU
  QAD_TRY(nvfp4_gemm_bf16_grouped(1, G, dgu, 1, R, F, 2 * F, xhat, 1, R, H, H, seg_off, seg_len, F, H, 0, dw_gate, H,
                                  stream));
  QAD_TRY(nvfp4_gemm_bf16_grouped(1, G, dgu + F, 1, R, F, 2 * F, xhat, 1, R, H, H, seg_off, seg_len, F, H, 0, dw_up,
                                  H, stream));
  // gradient of the combine weights
  if (d_combine)
    QAD_TRY(nvfp4_moe_router_grad(dy, at<void>(workspace, L, QAD_MOE_Y_ROWS), H, slot_row, s.tokens, s.topk, d_combine,
                                  stream));
  return NVFP4_OK;
}

}  // namespace

extern "C" {

nvfp4_status qad_moe_forward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* x,
                             const int32_t* expert_ids, const float* combine_weights, void* y, void* workspace,
                             size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("qad_moe_forward");
  return moe_forward(shape, w, x, expert_ids, combine_weights, y, workspace, workspace_bytes, stream, true);
}

nvfp4_status qad_moe_backward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* dy, void* dx,
                              void* dw_gate, void* dw_up, void* dw_down, float* d_combine, void* workspace,
                              size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("qad_moe_backward");
  return moe_backward(shape, w, dy, dx, dw_gate, dw_up, dw_down, d_combine, workspace, workspace_bytes, stream, true);
}

nvfp4_status qad_moe_expert_forward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* x,
                                    const int32_t* expert_ids, void* y, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  NVFP4_ENTRY("qad_moe_expert_forward");
  if (!shape || shape->topk != 1) return NVFP4_ERR_SHAPE;
  return moe_forward(shape, w, x, expert_ids, nullptr, y, workspace, workspace_bytes, stream, false);
}

nvfp4_status qad_moe_expert_backward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* dy, void* dx,
                                     void* dw_gate, void* dw_up, void* dw_down, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("qad_moe_expert_backward");
  if (!shape || shape->topk != 1) return NVFP4_ERR_SHAPE;
  return moe_backward(shape, w, dy, dx, dw_gate, dw_up, dw_down, nullptr, workspace, workspace_bytes, stream, false);
}

}  // extern "C"
