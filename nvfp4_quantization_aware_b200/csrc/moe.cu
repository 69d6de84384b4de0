// moe.cu -- kernels of the QAD student's MoE layer step around the grouped
// GEMMs: routing into per-expert segments, NVFP4 quantization of the routed
// activations and of the SwiGLU output, the weighted combine, and the
// straight-through backward pieces.
//
// The layer is the pages' MoE block: 128 routed experts plus one shared
// expert, 6 routed experts per token (Nemotron-3-Nano-30B NVFP4 article, "Was
// ist Nemotron-Nano-3-30B-A3B-NVFP4?"), expert FFNs with down/gate/up
// projections quantized W4A4 NVFP4 with frozen scales (Qwen3.6-35B-A3B W4A4
// tutorial, "2. PTQ"; Nemotron 3.5 Lightning NVFP4 article, "量化尺度处理策略").
//
// Layout.  Group g < E is routed expert g, group E the shared expert.  The
// routed (token, slot) pairs are permuted into R rows: group g owns rows
// [off[g], off[g] + len[g]), off[g] a multiple of 128; rows past len[g] up to
// the next segment are padding (token -1) and every kernel writes zeros
// there, which the K-segmented weight-gradient GEMMs rely on.  Within a
// segment rows are in increasing (token, slot) order, so every result is
// deterministic.
#include "moe_internal.cuh"
#include "quant_common.cuh"

namespace nvfp4 {
namespace moe {

constexpr int kMaxGroups = 256;

// Group owning permuted row r: last g with off[g] <= r (off in shared memory).
NVFP4_DEV int group_of_row(const int32_t* s_off, int groups, int r) {
  int lo = 0, hi = groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_off[mid] <= r) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

NVFP4_DEV int pad128(int n) { return (n + 127) & ~127; }

// ------------------------------------------------------------------ routing

// len[e] = number of assignments routed to expert e (one block per expert);
// len[E] = T for the shared expert.
// The last block marks assignments with an id outside [0, experts) (slot
// -1, device error word kErrExpertId); they are routed nowhere.
// shared_rows: rows of the shared expert's segment (tokens, or 0 when the
// layer has no shared expert, e.g. the rows an expert-parallel rank received).
__global__ void route_count_kernel(const int32_t* __restrict__ ids, int assignments, int experts, int shared_rows,
                                   int32_t* __restrict__ len, int32_t* __restrict__ slot_row) {
  const int e = blockIdx.x;
  if (e == experts) {
    if (threadIdx.x == 0) len[e] = shared_rows;
    for (int i = threadIdx.x; i < assignments; i += blockDim.x) {
      const int id = __ldg(ids + i);
      if (id < 0 || id >= experts) {
        slot_row[i] = -1;
        report_error(kErrExpertId);
      }
    }
    return;
  }
  int c = 0;
  for (int i = threadIdx.x; i < assignments; i += blockDim.x) c += (__ldg(ids + i) == e);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
  __shared__ int part[32];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += part[w];
    len[e] = tot;
  }
}

// Segment offsets and the permutation (one block of 1024 threads per group).
// Ranks within a group come from an in-order block scan, so row order is the
// (token, slot) order.
__global__ void __launch_bounds__(1024) route_scatter_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ weights, int tokens, int topk, int experts,
    const int32_t* __restrict__ len, int32_t* __restrict__ off, int32_t* __restrict__ row_token,
    float* __restrict__ row_weight, int32_t* __restrict__ slot_row, int rows_cap) {
  const int e = blockIdx.x;
  const int groups = experts + 1;
  __shared__ int s_off;
  __shared__ int warp_sum[32];
  if (threadIdx.x == 0) {
    int o = 0;
    for (int g = 0; g < e; ++g) o += pad128(__ldg(len + g));
    s_off = o;
    if (e == experts) {
      // the last block also publishes the whole offset table
      int q = 0;
      for (int g = 0; g < groups; ++g) {
        off[g] = q;
        q += pad128(__ldg(len + g));
      }
      off[groups] = q;
      if (q > rows_cap) report_error(kErrRowsCapacity);
    }
  }
  __syncthreads();
  const int base = s_off;
  const int n = __ldg(len + e);
  if (base + pad128(n) > rows_cap) return;  // reported above
  if (e == experts) {
    for (int t = threadIdx.x; t < n; t += blockDim.x) {  // n = tokens, or 0 without a shared expert
      row_token[base + t] = t;
      row_weight[base + t] = 1.0f;
    }
  } else {
    const int assignments = tokens * topk;
    int running = 0;
    for (int a0 = 0; a0 < assignments; a0 += blockDim.x) {
      const int a = a0 + threadIdx.x;
      const bool hit = a < assignments && __ldg(ids + a) == e;
      const unsigned ballot = __ballot_sync(0xFFFFFFFFu, hit);
      const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
      if (lane == 0) warp_sum[w] = __popc(ballot);
      __syncthreads();
      int before = 0;
      for (int i = 0; i < w; ++i) before += warp_sum[i];
      int chunk_total = 0;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) chunk_total += warp_sum[i];
      if (hit) {
        const int r = base + running + before + __popc(ballot & ((1u << lane) - 1u));
        row_token[r] = a / topk;
        row_weight[r] = weights ? __ldg(weights + a) : 1.0f;
        slot_row[a] = r;
      }
      running += chunk_total;
      __syncthreads();
    }
  }
  for (int r = base + n + threadIdx.x; r < base + pad128(n); r += blockDim.x) {
    row_token[r] = -1;
    row_weight[r] = 0.0f;
  }
}

// ------------------------------------------------------------------ quantize routed rows

struct QuantRowsArgs {
  const __nv_bfloat16* src;   // gather: x [T][cols]; activation: h_gate [R][cols]
  const __nv_bfloat16* src2;  // activation: h_up [R][cols]
  int64_t ld_src;
  const int32_t* row_token;   // [rows_cap]
  const int32_t* off;         // [groups + 1]
  int groups;
  const float* ts;            // frozen tensor scale per group
  int rows_cap, cols;
  uint8_t* codes;             // [rows_cap][cols / 2]
  uint8_t* scales_mma;        // MMA layout of [rows_cap][cols]
  __nv_bfloat16* xhat;        // [rows_cap][cols] dequantized (may be NULL)
  __nv_bfloat16* act;         // activation kernel: the bf16 SwiGLU output before quantization (may be NULL)
  int64_t kchunks;
};

// One warp per 512-column chunk of a permuted row, one lane per 16-element
// block (FROZEN_GLOBAL: the group's tensor scale is given, block scales are
// computed).  GATHER: the row is x[row_token[r]].  Otherwise the row is the
// SwiGLU a = silu(h_gate) * h_up, rounded to bf16 before quantization.
template <bool GATHER>
__global__ void __launch_bounds__(256) quant_rows_kernel(QuantRowsArgs a) {
  __shared__ int32_t s_off[kMaxGroups + 1];
  for (int i = threadIdx.x; i <= a.groups; i += blockDim.x) s_off[i] = __ldg(a.off + i);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int cpr = a.cols / 512 + ((a.cols % 512) ? 1 : 0);
  const int64_t total = (int64_t)a.rows_cap * cpr;
  const int end_rows = s_off[a.groups];
  for (int64_t c = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); c < total; c += (int64_t)gridDim.x * 8) {
    const int r = (int)(c / cpr);
    const int col = (int)(c - (int64_t)r * cpr) * 512 + lane * 16;
    if (col >= a.cols) continue;
    const int tok = r < end_rows ? __ldg(a.row_token + r) : -1;
    float v[16];
    uint32_t lo = 0, hi = 0, sb = 0;
    float d = 0.f;
    if (tok >= 0) {
      const int g = group_of_row(s_off, a.groups, r);
      const float sg = __ldg(a.ts + g);
      if (GATHER) {
        Block16<__nv_bfloat16> in;
        in.load(a.src + (int64_t)tok * a.ld_src + col, false);
        in.to_f32(v);
      } else {
        Block16<__nv_bfloat16> hg, hu;
        hg.load(a.src + (int64_t)r * a.ld_src + col, false);
        hu.load(a.src2 + (int64_t)r * a.ld_src + col, false);
        float gv[16], uv[16];
        hg.to_f32(gv);
        hu.to_f32(uv);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float s = gv[i] / (1.0f + expf(-gv[i]));  // silu
          v[i] = __bfloat162float(__float2bfloat16_rn(s * uv[i]));
        }
        if (a.act) Block16<__nv_bfloat16>::store(a.act + (int64_t)r * a.cols + col, v, false);
      }
      sb = encode_block16<true>(v, sg, __fmul_rn(6.0f, sg), false, 0u, lo, hi, d);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.f;
      if (!GATHER && a.act) Block16<__nv_bfloat16>::store(a.act + (int64_t)r * a.cols + col, v, false);
    }
    uint8_t* dst = a.codes + (int64_t)r * (a.cols / 2) + col / 2;
    st_stream_u32(dst, lo);
    st_stream_u32(dst + 4, hi);
    a.scales_mma[mma_scale_offset(r, col >> 4, a.kchunks)] = (uint8_t)sb;
    if (a.xhat) {
      float o[16];
      if (tok >= 0) decode_block16(lo, hi, d, o);
      else
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = 0.f;
      Block16<__nv_bfloat16>::store(a.xhat + (int64_t)r * a.cols + col, o, false);
    }
  }
}

// ------------------------------------------------------------------ combine / gathers

// out[t] = sum_j w[t, j] y[slot_row[t, j]] + y[shared_base + t]   (FP32 sum in
// the fixed order j = 0..k-1, then the shared expert)
// (without `shared` the shared expert's term is left out; NULL weights are 1)
__global__ void combine_kernel(const __nv_bfloat16* __restrict__ y, int cols, const int32_t* __restrict__ slot_row,
                               const float* __restrict__ weights, int tokens, int topk,
                               const int32_t* __restrict__ off, int experts, int shared,
                               __nv_bfloat16* __restrict__ out) {
  // one warp per token: its slot rows and weights are read once, the lanes
  // stride over the row's 16-byte vectors
  const int lane = threadIdx.x & 31;
  const int vpr = cols / 8;
  const int shared_base = __ldg(off + experts);
  const int warps = (int)(gridDim.x * blockDim.x / 32);
  for (int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) / 32); t < tokens; t += warps) {
    const int my_r = lane < topk ? __ldg(slot_row + (int64_t)t * topk + lane) : -1;
    const float my_w = lane < topk ? (weights ? __ldg(weights + (int64_t)t * topk + lane) : 1.0f) : 0.0f;
    // warp-uniform trip count: every lane takes part in every shuffle; only
    // the loads and the store are predicated on the lane's vector
    for (int vb = 0; vb < vpr; vb += 32) {
      const int vc = vb + lane;
      const bool act = vc < vpr;
      const int c = vc * 8;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int j = 0; j < topk; ++j) {
        const int r = __shfl_sync(0xFFFFFFFFu, my_r, j);
        const float w = __shfl_sync(0xFFFFFFFFu, my_w, j);
        if (r < 0 || !act) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(y + (int64_t)r * cols + c);
        acc[0] = fmaf(w, bf16lo_to_f32(v.x), acc[0]); acc[1] = fmaf(w, bf16hi_to_f32(v.x), acc[1]);
        acc[2] = fmaf(w, bf16lo_to_f32(v.y), acc[2]); acc[3] = fmaf(w, bf16hi_to_f32(v.y), acc[3]);
        acc[4] = fmaf(w, bf16lo_to_f32(v.z), acc[4]); acc[5] = fmaf(w, bf16hi_to_f32(v.z), acc[5]);
        acc[6] = fmaf(w, bf16lo_to_f32(v.w), acc[6]); acc[7] = fmaf(w, bf16hi_to_f32(v.w), acc[7]);
      }
      if (!act) continue;
      if (shared) {
        const uint4 v = *reinterpret_cast<const uint4*>(y + (int64_t)(shared_base + t) * cols + c);
        acc[0] += bf16lo_to_f32(v.x); acc[1] += bf16hi_to_f32(v.x);
        acc[2] += bf16lo_to_f32(v.y); acc[3] += bf16hi_to_f32(v.y);
        acc[4] += bf16lo_to_f32(v.z); acc[5] += bf16hi_to_f32(v.z);
        acc[6] += bf16lo_to_f32(v.w); acc[7] += bf16hi_to_f32(v.w);
      }
      *reinterpret_cast<uint4*>(out + (int64_t)t * cols + c) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                     pack_bf16x2(acc[6], acc[7]));
    }
  }
}

// dyp[r] = row_weight[r] * dy[row_token[r]] (zero on padding rows)
__global__ void scale_rows_kernel(const __nv_bfloat16* __restrict__ dy, int cols, const int32_t* __restrict__ row_token,
                                  const float* __restrict__ row_weight, const int32_t* __restrict__ off, int groups,
                                  int rows_cap, __nv_bfloat16* __restrict__ dyp) {
  // one warp per row: its token and weight are read once, the lanes stride
  // over the row's 16-byte vectors
  const int lane = threadIdx.x & 31;
  const int vpr = cols / 8;
  const int end_rows = __ldg(off + groups);
  const int warps = (int)(gridDim.x * blockDim.x / 32);
  for (int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) / 32); r < rows_cap; r += warps) {
    const int t = r < end_rows ? __ldg(row_token + r) : -1;
    const float w = t >= 0 ? __ldg(row_weight + r) : 0.0f;
    __nv_bfloat16* drow = dyp + (int64_t)r * cols;
    const __nv_bfloat16* srow = dy + (int64_t)(t >= 0 ? t : 0) * cols;
    for (int vc = lane; vc < vpr; vc += 32) {
      uint4 o = make_uint4(0, 0, 0, 0);
      if (t >= 0) {
        const uint4 v = *reinterpret_cast<const uint4*>(srow + vc * 8);
        o = make_uint4(pack_bf16x2(w * bf16lo_to_f32(v.x), w * bf16hi_to_f32(v.x)),
                       pack_bf16x2(w * bf16lo_to_f32(v.y), w * bf16hi_to_f32(v.y)),
                       pack_bf16x2(w * bf16lo_to_f32(v.z), w * bf16hi_to_f32(v.z)),
                       pack_bf16x2(w * bf16lo_to_f32(v.w), w * bf16hi_to_f32(v.w)));
      }
      *reinterpret_cast<uint4*>(drow + vc * 8) = o;
    }
  }
}

// SwiGLU backward: with s = sigmoid(g), silu(g) = g s,
//   dg = da * u * s * (1 + g (1 - s)),  du = da * silu(g);
// written as dgu[r] = [dg | du] (zero on padding rows).  s comes from the
// hardware exponential and a fast reciprocal (relative error ~1e-6; these
// gradients feed no rounding decision), one warp per row.
__global__ void swiglu_bwd_kernel(const __nv_bfloat16* __restrict__ da, const __nv_bfloat16* __restrict__ hg,
                                  const __nv_bfloat16* __restrict__ hu, int cols, const int32_t* __restrict__ row_token,
                                  const int32_t* __restrict__ off, int groups, int rows_cap,
                                  __nv_bfloat16* __restrict__ dgu) {
  const int lane = threadIdx.x & 31;
  const int end_rows = __ldg(off + groups);
  const int vpr = cols / 8;
  const int warps = (int)(gridDim.x * blockDim.x / 32);
  for (int r = (int)((blockIdx.x * blockDim.x + threadIdx.x) / 32); r < rows_cap; r += warps) {
    const int t = r < end_rows ? __ldg(row_token + r) : -1;
    for (int vc = lane; vc < vpr; vc += 32) {
      const int c = vc * 8;
      uint4 og = make_uint4(0, 0, 0, 0), ou = make_uint4(0, 0, 0, 0);
      if (t >= 0) {
        const int64_t e = (int64_t)r * cols + c;
        const uint4 G = ld_stream_v4(hg + e), U = ld_stream_v4(hu + e), D = ld_stream_v4(da + e);
        const uint32_t gw[4] = {G.x, G.y, G.z, G.w}, uw[4] = {U.x, U.y, U.z, U.w}, dw[4] = {D.x, D.y, D.z, D.w};
        uint32_t rg[4], ru[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float dg2[2], du2[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float g = h ? bf16hi_to_f32(gw[k]) : bf16lo_to_f32(gw[k]);
            const float u = h ? bf16hi_to_f32(uw[k]) : bf16lo_to_f32(uw[k]);
            const float d = h ? bf16hi_to_f32(dw[k]) : bf16lo_to_f32(dw[k]);
            const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
            dg2[h] = d * u * sg * (1.0f + g * (1.0f - sg));
            du2[h] = d * g * sg;
          }
          rg[k] = pack_bf16x2(dg2[0], dg2[1]);
          ru[k] = pack_bf16x2(du2[0], du2[1]);
        }
        og = make_uint4(rg[0], rg[1], rg[2], rg[3]);
        ou = make_uint4(ru[0], ru[1], ru[2], ru[3]);
      }
      st_stream_v4(dgu + (int64_t)r * 2 * cols + c, og);
      st_stream_v4(dgu + (int64_t)r * 2 * cols + cols + c, ou);
    }
  }
}

// dx[t] = sum_j dxp[slot_row[t, j]] + dxp[shared_base + t]   (fixed order)
__global__ void gather_sum_kernel(const __nv_bfloat16* __restrict__ dxp, int cols, const int32_t* __restrict__ slot_row,
                                  int tokens, int topk, const int32_t* __restrict__ off, int experts, int shared,
                                  __nv_bfloat16* __restrict__ dx) {
  // one warp per token (its slot rows read once), lanes over 16-byte vectors
  const int lane = threadIdx.x & 31;
  const int vpr = cols / 8;
  const int shared_base = __ldg(off + experts);
  const int warps = (int)(gridDim.x * blockDim.x / 32);
  for (int t = (int)((blockIdx.x * blockDim.x + threadIdx.x) / 32); t < tokens; t += warps) {
    const int my_r = lane < topk ? __ldg(slot_row + (int64_t)t * topk + lane) : -1;
    // warp-uniform trip count (all lanes shuffle); loads and store predicated
    for (int vb = 0; vb < vpr; vb += 32) {
      const int vc = vb + lane;
      const bool act = vc < vpr;
      const int c = vc * 8;
      float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      for (int j = 0; j < topk + shared; ++j) {
        const int rj = __shfl_sync(0xFFFFFFFFu, my_r, j < topk ? j : 0);
        const int r = j < topk ? rj : shared_base + t;
        if (r < 0 || !act) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(dxp + (int64_t)r * cols + c);
        acc[0] += bf16lo_to_f32(v.x); acc[1] += bf16hi_to_f32(v.x);
        acc[2] += bf16lo_to_f32(v.y); acc[3] += bf16hi_to_f32(v.y);
        acc[4] += bf16lo_to_f32(v.z); acc[5] += bf16hi_to_f32(v.z);
        acc[6] += bf16lo_to_f32(v.w); acc[7] += bf16hi_to_f32(v.w);
      }
      if (!act) continue;
      *reinterpret_cast<uint4*>(dx + (int64_t)t * cols + c) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                     pack_bf16x2(acc[6], acc[7]));
    }
  }
}

// dw[t, j] = <dy[t], y[slot_row[t, j]]>  (one warp per assignment, FP32)
__global__ void router_grad_kernel(const __nv_bfloat16* __restrict__ dy, const __nv_bfloat16* __restrict__ y,
                                   int cols, const int32_t* __restrict__ slot_row, int assignments, int topk,
                                   float* __restrict__ dw) {
  const int lane = threadIdx.x & 31;
  for (int a = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); a < assignments;
       a += gridDim.x * (blockDim.x >> 5)) {
    const int t = a / topk;
    const int r = __ldg(slot_row + a);
    float acc = 0.f;
    if (r < 0) {
      if (lane == 0) dw[a] = 0.f;
      continue;
    }
    for (int c = lane * 8; c < cols; c += 256) {
      const uint4 p = *reinterpret_cast<const uint4*>(dy + (int64_t)t * cols + c);
      const uint4 q = *reinterpret_cast<const uint4*>(y + (int64_t)r * cols + c);
      acc = fmaf(bf16lo_to_f32(p.x), bf16lo_to_f32(q.x), acc); acc = fmaf(bf16hi_to_f32(p.x), bf16hi_to_f32(q.x), acc);
      acc = fmaf(bf16lo_to_f32(p.y), bf16lo_to_f32(q.y), acc); acc = fmaf(bf16hi_to_f32(p.y), bf16hi_to_f32(q.y), acc);
      acc = fmaf(bf16lo_to_f32(p.z), bf16lo_to_f32(q.z), acc); acc = fmaf(bf16hi_to_f32(p.z), bf16hi_to_f32(q.z), acc);
      acc = fmaf(bf16lo_to_f32(p.w), bf16lo_to_f32(q.w), acc); acc = fmaf(bf16hi_to_f32(p.w), bf16hi_to_f32(q.w), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) dw[a] = acc;
  }
}

// Row-major block scales [rows][cols/16] -> the MMA scale layout (padding 0).
__global__ void scales_to_mma_kernel(const uint8_t* __restrict__ sb, int64_t rows, int64_t cols,
                                     uint8_t* __restrict__ out) {
  const int64_t nblk = cols / 16;
  const int64_t kchunks = (nblk + 3) / 4;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t total = rows_pad * kchunks * 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / (kchunks * 4), kb = i - r * (kchunks * 4);
    out[mma_scale_offset(r, kb, kchunks)] = (r < rows && kb < nblk) ? __ldg(sb + r * nblk + kb) : (uint8_t)0;
  }
}

static int sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n = 148;
  }
  return n;
}

static nvfp4_status done(int launches) {
  count_launches(launches);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace moe
}  // namespace nvfp4

using namespace nvfp4;
using namespace nvfp4::moe;

extern "C" {

int64_t nvfp4_moe_rows_capacity(int tokens, int topk, int experts) {
  const int64_t r = (int64_t)tokens * topk + 127ll * experts + ((int64_t)tokens + 127) / 128 * 128;
  return (r + 127) / 128 * 128;
}

}  // extern "C"

namespace nvfp4 {
namespace moe {

nvfp4_status route(const int32_t* expert_ids, const float* combine_weights, int tokens, int topk, int experts,
                   bool shared, int32_t* seg_len, int32_t* seg_off, int32_t* row_token, float* row_weight,
                   int32_t* slot_row, int64_t rows_cap, void* stream) {
  if (tokens < 1 || topk < 1 || experts < 1 || experts + 1 > kMaxGroups) return NVFP4_ERR_SHAPE;
  if (rows_cap < nvfp4_moe_rows_capacity(tokens, topk, experts) || rows_cap > 0x7FFFFFFF) return NVFP4_ERR_SHAPE;
  if (!expert_ids || (shared && !combine_weights) || !seg_len || !seg_off || !row_token || !row_weight || !slot_row)
    return NVFP4_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  route_count_kernel<<<experts + 1, 1024, 0, s>>>(expert_ids, tokens * topk, experts, shared ? tokens : 0, seg_len,
                                                  slot_row);
  route_scatter_kernel<<<experts + 1, 1024, 0, s>>>(expert_ids, combine_weights, tokens, topk, experts, seg_len,
                                                    seg_off, row_token, row_weight, slot_row, (int)rows_cap);
  return done(2);
}

nvfp4_status combine(const void* y, int64_t cols, const int32_t* slot_row, const float* combine_weights, int tokens,
                     int topk, const int32_t* seg_off, int experts, bool shared, void* out, void* stream) {
  if (cols < 8 || cols % 8 || tokens < 1 || topk < 1 || topk > 32) return NVFP4_ERR_SHAPE;
  if (!y || !slot_row || (shared && !combine_weights) || !seg_off || !out) return NVFP4_ERR_ARG;
  if (((uintptr_t)y & 15u) || ((uintptr_t)out & 15u)) return NVFP4_ERR_ALIGN;
  combine_kernel<<<sms() * 8, 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<const __nv_bfloat16*>(y), (int)cols,
                                                              slot_row, combine_weights, tokens, topk, seg_off, experts,
                                                              shared ? 1 : 0, reinterpret_cast<__nv_bfloat16*>(out));
  return done(1);
}

nvfp4_status gather_sum(const void* dxp, int64_t cols, const int32_t* slot_row, int tokens, int topk,
                        const int32_t* seg_off, int experts, bool shared, void* dx, void* stream) {
  if (cols < 8 || cols % 8 || tokens < 1 || topk < 1 || topk > 32) return NVFP4_ERR_SHAPE;
  if (!dxp || !slot_row || !seg_off || !dx) return NVFP4_ERR_ARG;
  if (((uintptr_t)dxp & 15u) || ((uintptr_t)dx & 15u)) return NVFP4_ERR_ALIGN;
  gather_sum_kernel<<<sms() * 8, 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<const __nv_bfloat16*>(dxp), (int)cols,
                                                                 slot_row, tokens, topk, seg_off, experts,
                                                                 shared ? 1 : 0, reinterpret_cast<__nv_bfloat16*>(dx));
  return done(1);
}

}  // namespace moe
}  // namespace nvfp4

extern "C" {

nvfp4_status nvfp4_moe_route(const int32_t* expert_ids, const float* combine_weights, int tokens, int topk,
                             int experts, int32_t* seg_len, int32_t* seg_off, int32_t* row_token, float* row_weight,
                             int32_t* slot_row, int64_t rows_cap, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_route");
  return moe::route(expert_ids, combine_weights, tokens, topk, experts, true, seg_len, seg_off, row_token, row_weight,
                    slot_row, rows_cap, stream);
}

static nvfp4_status quant_rows(bool gather, const void* src, const void* src2, int64_t ld_src, const int32_t* row_token,
                               const int32_t* seg_off, int groups, const float* ts, int64_t rows_cap, int64_t cols,
                               uint8_t* codes, uint8_t* scales_mma, void* xhat, void* act, void* stream) {
  if (groups < 1 || groups > kMaxGroups || rows_cap < 128 || rows_cap % 128 || rows_cap > 0x7FFFFFFF || cols < 64 ||
      cols % 64 || cols > 0x7FFFFFFF || ld_src < cols)
    return NVFP4_ERR_SHAPE;
  if (!src || (!gather && !src2) || !row_token || !seg_off || !ts || !codes || !scales_mma) return NVFP4_ERR_ARG;
  if (((uintptr_t)src & 15u) || (ld_src * 2) % 16 || ((uintptr_t)codes & 3u) || (cols / 2) % 4 ||
      (src2 && ((uintptr_t)src2 & 15u)) || (xhat && ((uintptr_t)xhat & 15u)) || (act && ((uintptr_t)act & 15u)))
    return NVFP4_ERR_ALIGN;
  QuantRowsArgs a;
  a.src = reinterpret_cast<const __nv_bfloat16*>(src);
  a.src2 = reinterpret_cast<const __nv_bfloat16*>(src2);
  a.ld_src = ld_src;
  a.row_token = row_token;
  a.off = seg_off;
  a.groups = groups;
  a.ts = ts;
  a.rows_cap = (int)rows_cap;
  a.cols = (int)cols;
  a.codes = codes;
  a.scales_mma = scales_mma;
  a.xhat = reinterpret_cast<__nv_bfloat16*>(xhat);
  a.act = reinterpret_cast<__nv_bfloat16*>(act);
  a.kchunks = (cols / 16 + 3) / 4;
  const int grid = sms() * 4;
  if (gather) quant_rows_kernel<true><<<grid, 256, 0, (cudaStream_t)stream>>>(a);
  else quant_rows_kernel<false><<<grid, 256, 0, (cudaStream_t)stream>>>(a);
  return done(1);
}

nvfp4_status nvfp4_moe_gather_quantize(const void* x, int64_t ld_x, const int32_t* row_token, const int32_t* seg_off,
                                       int groups, const float* tensor_scales, int64_t rows_cap, int64_t cols,
                                       uint8_t* codes, uint8_t* scales_mma, void* xhat, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_gather_quantize");
  return quant_rows(true, x, nullptr, ld_x, row_token, seg_off, groups, tensor_scales, rows_cap, cols, codes,
                    scales_mma, xhat, nullptr, stream);
}

nvfp4_status nvfp4_moe_swiglu_quantize(const void* h_gate, const void* h_up, int64_t ld_h, const int32_t* row_token,
                                       const int32_t* seg_off, int groups, const float* tensor_scales, int64_t rows_cap,
                                       int64_t cols, uint8_t* codes, uint8_t* scales_mma, void* ahat, void* act,
                                       void* stream) {
  NVFP4_ENTRY("nvfp4_moe_swiglu_quantize");
  return quant_rows(false, h_gate, h_up, ld_h, row_token, seg_off, groups, tensor_scales, rows_cap, cols, codes,
                    scales_mma, ahat, act, stream);
}

nvfp4_status nvfp4_moe_combine(const void* y, int64_t cols, const int32_t* slot_row, const float* combine_weights,
                               int tokens, int topk, const int32_t* seg_off, int experts, void* out, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_combine");
  if (!combine_weights) return NVFP4_ERR_ARG;
  return moe::combine(y, cols, slot_row, combine_weights, tokens, topk, seg_off, experts, true, out, stream);
}

nvfp4_status nvfp4_moe_scale_rows(const void* dy, int64_t cols, const int32_t* row_token, const float* row_weight,
                                  const int32_t* seg_off, int groups, int64_t rows_cap, void* dyp, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_scale_rows");
  if (cols < 8 || cols % 8 || rows_cap < 1 || groups < 1) return NVFP4_ERR_SHAPE;
  if (!dy || !row_token || !row_weight || !seg_off || !dyp) return NVFP4_ERR_ARG;
  if (((uintptr_t)dy & 15u) || ((uintptr_t)dyp & 15u)) return NVFP4_ERR_ALIGN;
  scale_rows_kernel<<<sms() * 8, 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<const __nv_bfloat16*>(dy), (int)cols,
                                                                 row_token, row_weight, seg_off, groups, (int)rows_cap,
                                                                 reinterpret_cast<__nv_bfloat16*>(dyp));
  return done(1);
}

nvfp4_status nvfp4_moe_swiglu_backward(const void* da, const void* h_gate, const void* h_up, int64_t cols,
                                       const int32_t* row_token, const int32_t* seg_off, int groups, int64_t rows_cap,
                                       void* dgu, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_swiglu_backward");
  if (cols < 8 || cols % 8 || rows_cap < 1 || groups < 1) return NVFP4_ERR_SHAPE;
  if (!da || !h_gate || !h_up || !row_token || !seg_off || !dgu) return NVFP4_ERR_ARG;
  if (((uintptr_t)da & 15u) || ((uintptr_t)h_gate & 15u) || ((uintptr_t)h_up & 15u) || ((uintptr_t)dgu & 15u))
    return NVFP4_ERR_ALIGN;
  swiglu_bwd_kernel<<<sms() * 8, 256, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(da), reinterpret_cast<const __nv_bfloat16*>(h_gate),
      reinterpret_cast<const __nv_bfloat16*>(h_up), (int)cols, row_token, seg_off, groups, (int)rows_cap,
      reinterpret_cast<__nv_bfloat16*>(dgu));
  return done(1);
}

nvfp4_status nvfp4_moe_gather_sum(const void* dxp, int64_t cols, const int32_t* slot_row, int tokens, int topk,
                                  const int32_t* seg_off, int experts, void* dx, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_gather_sum");
  return moe::gather_sum(dxp, cols, slot_row, tokens, topk, seg_off, experts, true, dx, stream);
}

nvfp4_status nvfp4_moe_router_grad(const void* dy, const void* y, int64_t cols, const int32_t* slot_row, int tokens,
                                   int topk, float* dw, void* stream) {
  NVFP4_ENTRY("nvfp4_moe_router_grad");
  if (cols < 8 || cols % 8 || tokens < 1 || topk < 1) return NVFP4_ERR_SHAPE;
  if (!dy || !y || !slot_row || !dw) return NVFP4_ERR_ARG;
  if (((uintptr_t)dy & 15u) || ((uintptr_t)y & 15u)) return NVFP4_ERR_ALIGN;
  router_grad_kernel<<<sms() * 8, 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<const __nv_bfloat16*>(dy),
                                                                  reinterpret_cast<const __nv_bfloat16*>(y), (int)cols,
                                                                  slot_row, tokens * topk, topk, dw);
  return done(1);
}

nvfp4_status nvfp4_scales_to_mma(const uint8_t* block_scales, int64_t rows, int64_t cols, uint8_t* out, void* stream) {
  NVFP4_ENTRY("nvfp4_scales_to_mma");
  if (rows < 1 || cols < 16 || cols % 16) return NVFP4_ERR_SHAPE;
  if (!block_scales || !out) return NVFP4_ERR_ARG;
  scales_to_mma_kernel<<<sms() * 8, 256, 0, (cudaStream_t)stream>>>(block_scales, rows, cols, out);
  return done(1);
}

}  // extern "C"
