// quantize.cu -- NVFP4 quantize / fake-quantize / dequantize for sm_100a.
//
// NVFP4 (Nemotron-3-Nano-30B NVFP4 article, "NVFP4-Format und warum es
// wichtig ist?"): E2M1 elements in blocks of 16 along the contiguous
// dimension, one E4M3 scale per block, one FP32 scale per tensor.  Scale
// modes (Nemotron 3.5 Lightning NVFP4 article, "量化尺度处理策略"): dynamic
// (recomputed from the max on every call) or frozen (passed in).
//
// Work decomposition.  These kernels stream HBM: every input byte is read
// once per pass and every output byte written once.  A lane owns one whole
// 16-element block (32 bytes of bf16, one 256-bit load), so the block max and
// the block scale are computed once per block without any shuffle, and a warp
// covers a 512-element chunk of a row.  Chunks are numbered row-major per
// tensor; chunk -> (row, column) uses a precomputed multiply-shift divider.
// Each warp takes kUnroll consecutive chunks per iteration so that several
// independent loads per lane are in flight.  Grids are persistent: exactly the
// resident capacity of the GPU (SM count x resident CTAs), grid-striding.
//
// Dynamic mode is two launches per group in stream order: group_amax_kernel
// folds each tensor's max |x| into a workspace word (max is exact, so any
// order gives the same s_g), then the encode kernel derives s_g = amax / 2688.
// The encode is bound by instruction issue rather than by HBM, so re-reading
// the inputs from L2 instead of HBM gains nothing: groups are cut only by the
// number of tensors a launch holds.
#include <cooperative_groups.h>

#include "quant_common.cuh"

namespace cg = cooperative_groups;

namespace nvfp4 {

constexpr int kThreads = 256;           // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;              // chunks per warp per iteration (dequantize)
constexpr int kChunk = 256;             // elements per warp per chunk (dequantize: 8 per lane)
constexpr int kQUnroll = 2;             // chunks per warp per iteration (encode)
constexpr int kQChunk = 512;            // elements per warp per chunk (amax / encode: 16 per lane)

template <typename T>
NVFP4_DEV void store8(T* p, const float (&v)[8]);

template <>
NVFP4_DEV void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]);
  w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]);
  w.w = pack_bf16x2(v[6], v[7]);
  st_stream_v4(p, w);
}

template <>
NVFP4_DEV void store8<float>(float* p, const float (&v)[8]) {
  st_stream_v4(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                             __float_as_uint(v[3])));
  st_stream_v4(p + 4, make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                                 __float_as_uint(v[7])));
}

// Chunk geometry shared by every kernel of this file.
struct Geom {
  int64_t rows, cols, ld;       // input (elements)
  int64_t chunks_per_row;       // ceil(cols / 256)
  int64_t total_chunks;         // rows * chunks_per_row
  NVFP4_DEV void locate(int64_t chunk, int lane, int64_t& row, int64_t& col) const {
    row = chunk / chunks_per_row;
    col = (chunk - row * chunks_per_row) * kChunk + lane * 8;
  }
};

NVFP4_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// ------------------------------------------------------------------ tensor groups
//
// One launch processes a group of up to kMaxGroup tensors (e.g. the 128
// experts of a MoE layer), each with its own FP32 tensor scale.  Their chunks
// are numbered consecutively: tensor i owns [chunk0_i, chunk0_{i+1}).  The
// table travels by value as a __grid_constant__ kernel parameter, read with
// warp-uniform indices.

constexpr int kMaxGroup = 144;

struct GTensor {
  const void* x;        // input, row stride ld_x elements
  uint8_t* codes;       // Out::Codes: packed codes, row stride ld_out bytes
  void* y;              // Out::Fake / Out::Both: dequantized output, row stride ld_y elements
  uint8_t* sb;          // block scales: read (FROZEN_ALL, row-major) or written if non-NULL
  float* ts;            // tensor scale: written (DYNAMIC) or read
  int64_t ld_x, ld_out, ld_y;
  int64_t cols;
  int64_t rows;
  int64_t chunk0;       // first chunk of this tensor in the group
  int64_t kchunks;      // ceil(cols / 64), MMA scale layout
  FastDiv cpr;          // chunks per row = ceil(cols / 512)
};

struct GroupArgs {
  GTensor t[kMaxGroup];
  int n;
  int mode;             // nvfp4_scale_mode
  int layout;           // nvfp4_scale_layout of written block scales
  int64_t total_chunks;
  unsigned* amax;       // DYNAMIC: n words holding max |x| as float bits (zeroed first)
  unsigned* amax_part;  // DYNAMIC, one tensor: per-CTA maxima of the amax launch (or NULL)
  int amax_grid;        // CTAs of that launch (entries of amax_part)
  int x_wide;           // every input row start is 32-byte aligned: 256-bit loads
  int out_wide;         // codes rows 8-byte aligned (8-byte stores)
  int y_wide;           // y rows 32-byte aligned (256-bit stores)
};

// Advance `t` to the tensor owning `chunk` (chunks are visited in increasing
// order by every warp, so the cursor only moves forward).
NVFP4_DEV int find_tensor(const GroupArgs& a, int64_t chunk, int t) {
  while (t + 1 < a.n && chunk >= a.t[t + 1].chunk0) ++t;
  return t;
}

// Row and first column of this lane's block for a chunk of tensor g.
NVFP4_DEV void chunk_pos(const GTensor& g, int64_t chunk, int lane, int64_t& row, int64_t& col) {
  const uint32_t c = (uint32_t)(chunk - g.chunk0);
  const uint32_t r = fastdiv(c, g.cpr);
  row = r;
  col = (int64_t)(c - r * g.cpr.d) * kQChunk + lane * 16;
}

// ------------------------------------------------------------------ amax

// Per-tensor max |x| of a group.  Each CTA takes one contiguous range of
// chunks, so it touches one or two tensors; its warps walk the range in
// increasing order keeping a running max per tensor, fold it into a
// shared-memory table when the tensor changes, and the CTA finally folds the
// table into the global words with one atomicMax on the float bits per tensor
// it touched (|x| >= 0 compares like its bit pattern; max is exact, so the
// order of the atomics does not matter).
// Running max |x| of one lane.  bf16: the magnitudes' bit patterns compare
// like their values, so two 16-bit lanes of a word are folded at once
// (unsigned 16x2 max of the words with the sign bits cleared).
template <typename T>
struct LaneMax;

template <>
struct LaneMax<__nv_bfloat16> {
  uint32_t m2 = 0u;
  NVFP4_DEV void reset() { m2 = 0u; }
  NVFP4_DEV void add(const Block16<__nv_bfloat16>& b) {
#pragma unroll
    for (int i = 0; i < 8; ++i) m2 = __vmaxu2(m2, b.w[i] & 0x7FFF7FFFu);
  }
  NVFP4_DEV float value() const { return fmaxf(bf16lo_to_f32(m2), bf16hi_to_f32(m2)); }
};

template <>
struct LaneMax<float> {
  float m = 0.0f;
  NVFP4_DEV void reset() { m = 0.0f; }
  NVFP4_DEV void add(const Block16<float>& b) {
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(__uint_as_float(b.w[i])));
  }
  NVFP4_DEV float value() const { return m; }
};

constexpr int kAmaxUnroll = 4;  // chunks per warp per iteration (amax)

// Per-tensor maxima of |x| over chunks [c_begin, c_end) into s_max (shared,
// one word per tensor of the group, zeroed by the caller): warps take
// kAmaxUnroll consecutive chunks at a time.
template <typename T>
NVFP4_DEV void amax_range(const GroupArgs& a, int64_t c_begin, int64_t c_end, unsigned* s_max) {
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  int cur = 0;
  int mt = -1;      // tensor of the running max
  LaneMax<T> m;     // running max of this lane
  for (int64_t c0 = c_begin + wid * kAmaxUnroll; c0 < c_end; c0 += kWarps * kAmaxUnroll) {
    Block16<T> in[kAmaxUnroll];
    int tid[kAmaxUnroll];
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      const int64_t c = c0 + u;
      in[u].zero();
      tid[u] = -1;
      if (c < c_end) {
        cur = find_tensor(a, c, cur);
        const GTensor& g = a.t[cur];
        int64_t row, col;
        chunk_pos(g, c, lane, row, col);
        tid[u] = cur;
        if (col < g.cols) in[u].load(reinterpret_cast<const T*>(g.x) + row * g.ld_x + col, a.x_wide != 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kAmaxUnroll; ++u) {
      if (tid[u] < 0) continue;  // warp-uniform
      if (tid[u] != mt) {         // warp-uniform: flush the previous tensor's max
        const float w = warp_max(m.value());
        if (lane == 0 && mt >= 0 && w > 0.0f) atomicMax(s_max + mt, __float_as_uint(w));
        m.reset();
        mt = tid[u];
      }
      m.add(in[u]);
    }
  }
  const float w = warp_max(m.value());
  if (lane == 0 && mt >= 0 && w > 0.0f) atomicMax(s_max + mt, __float_as_uint(w));
}

// With amax_part (a single tensor) every CTA writes its maximum to its own
// entry instead, so nothing has to be cleared before the launch; the encode
// kernel folds the entries.
template <typename T>
__global__ void __launch_bounds__(kThreads) group_amax_kernel(const __grid_constant__ GroupArgs a) {
  __shared__ unsigned s_max[kMaxGroup];
  for (int i = threadIdx.x; i < a.n; i += kThreads) s_max[i] = 0u;
  __syncthreads();
  griddep_wait();
  const int64_t per_cta = (a.total_chunks + gridDim.x - 1) / gridDim.x;
  const int64_t c_begin = (int64_t)blockIdx.x * per_cta;
  const int64_t c_end = c_begin + per_cta < a.total_chunks ? c_begin + per_cta : a.total_chunks;
  amax_range<T>(a, c_begin, c_end, s_max);
  __syncthreads();
  if (a.amax_part != nullptr) {
    if (threadIdx.x == 0) a.amax_part[blockIdx.x] = s_max[0];
    return;
  }
  for (int i = threadIdx.x; i < a.n; i += kThreads)
    if (s_max[i] != 0u) atomicMax(a.amax + i, s_max[i]);
}

// ------------------------------------------------------------------ encode

enum class Out { Codes, Fake, Both };  // Both: codes and the fake-quant values

// s_g of tensor t: amax / (6 * 448) in DYNAMIC mode, else the given scale.
NVFP4_DEV float tensor_scale_of(const GroupArgs& a, int t) {
  if (a.mode == NVFP4_DYNAMIC) return __fdiv_rn(__uint_as_float(__ldcg(a.amax + t)), 2688.0f);
  return __ldg(a.t[t].ts);
}

// Encode one 16-element block of tensor g at (row, col) and write its
// outputs: block scale s_b = E4M3(max|x| / (6 s_g)) (or the frozen one),
// d = s_b s_g, codes E2M1(x / d), and per OUT the packed codes and / or the
// dequantized values.
template <typename T, Out OUT>
NVFP4_DEV void emit_block(const GroupArgs& a, const GTensor& g, int64_t row, int64_t col, const float (&v)[16],
                          float sg, float denom6, bool frozen_all, uint32_t sb_frozen) {
  uint32_t lo, hi;
  float d;
  const uint32_t sb = encode_block16<sizeof(T) == 2>(v, sg, denom6, frozen_all, sb_frozen, lo, hi, d);
  if (OUT != Out::Fake) {
    uint8_t* dst = g.codes + row * g.ld_out + (col >> 1);
    if (a.out_wide) {
      st_stream_v2(dst, lo, hi);
    } else {
      st_stream_u32(dst, lo);
      st_stream_u32(dst + 4, hi);
    }
  }
  if (OUT != Out::Codes) {
    float o[16];
    decode_block16(lo, hi, d, o);
    Block16<T>::store(reinterpret_cast<T*>(g.y) + row * g.ld_y + col, o, a.y_wide != 0);
  }
  if (!frozen_all && g.sb != nullptr) {
    const int64_t kb = col >> 4;
    const int64_t off = (a.layout == NVFP4_SCALES_MMA) ? mma_scale_offset(row, kb, g.kchunks)
                                                       : row * (g.cols >> 4) + kb;
    g.sb[off] = (uint8_t)sb;
  }
}

// Warps take groups of kQUnroll consecutive chunks, grid-striding (the
// chunks in flight at any time form one dense front through memory).  The
// position of a group's first chunk costs one division; the rest of the
// group follows by increments.
// The encode loop over the group's chunks, warps `warp` of `nwarps`
// striding; SgOf(t) gives tensor t's scale s_g.
template <typename T, Out OUT, typename SgOf>
NVFP4_DEV void encode_range(const GroupArgs& a, int64_t warp, int64_t nwarps, SgOf sg_of) {
  const int lane = threadIdx.x & 31;
  const bool frozen_all = a.mode == NVFP4_FROZEN_ALL;
  int cur = 0;
  int sg_t = -1;  // tensor whose scale is cached below
  float sg = 0.0f, denom6 = 0.0f;
  for (int64_t c0 = warp * kQUnroll; c0 < a.total_chunks; c0 += nwarps * kQUnroll) {
    cur = find_tensor(a, c0, cur);
    int t = cur;
    uint32_t row, ci;
    {
      const uint32_t local = (uint32_t)(c0 - a.t[t].chunk0);
      row = fastdiv(local, a.t[t].cpr);
      ci = local - row * a.t[t].cpr.d;
    }
    Block16<T> in[kQUnroll];
    uint32_t sb_in[kQUnroll];
    int tid[kQUnroll];
    int64_t row_[kQUnroll], col_[kQUnroll];
#pragma unroll
    for (int u = 0; u < kQUnroll; ++u) {
      in[u].zero();
      sb_in[u] = 0u;
      tid[u] = -1;
      row_[u] = 0;
      col_[u] = 0;
      if (c0 + u < a.total_chunks) {
        const GTensor& g = a.t[t];
        const int64_t col = (int64_t)ci * kQChunk + lane * 16;
        tid[u] = t;
        row_[u] = row;
        col_[u] = col;
        if (col < g.cols) {
          in[u].load(reinterpret_cast<const T*>(g.x) + (int64_t)row * g.ld_x + col, a.x_wide != 0);
          if (frozen_all) sb_in[u] = (uint32_t)__ldg(g.sb + (int64_t)row * (g.cols >> 4) + (col >> 4));
        }
        // next chunk: along the row, then the next row, then the next tensor
        if (++ci == g.cpr.d) {
          ci = 0;
          if (++row == (uint32_t)g.rows) {
            row = 0;
            ++t;
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kQUnroll; ++u) {
      const int tu = tid[u];
      if (tu < 0) continue;  // warp-uniform: past the end of the group
      const GTensor& g = a.t[tu];
      const int64_t row_u = row_[u], col = col_[u];
      if (col >= g.cols) continue;  // this lane's block lies past the row end
      if (tu != sg_t) {
        sg = sg_of(tu);
        denom6 = __fmul_rn(6.0f, sg);
        sg_t = tu;
      }
      float v[16];
      in[u].to_f32(v);
      emit_block<T, OUT>(a, g, row_u, col, v, sg, denom6, frozen_all, sb_in[u]);
    }
  }
}

template <typename T, Out OUT>
__global__ void __launch_bounds__(kThreads) group_encode_kernel(const __grid_constant__ GroupArgs a) {
  griddep_wait();
  if (a.mode == NVFP4_DYNAMIC && a.amax_part != nullptr) {
    // one tensor: its max is the max of the amax launch's per-CTA entries
    __shared__ unsigned s_warp[kWarps];
    unsigned m = 0u;
    for (int i = threadIdx.x; i < a.amax_grid; i += kThreads) m = max(m, __ldcg(a.amax_part + i));
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = m;
    __syncthreads();
    m = s_warp[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) m = max(m, s_warp[w]);
    const float sg = __fdiv_rn(__uint_as_float(m), 2688.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.t[0].ts = sg;
    encode_range<T, OUT>(a, (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5), (int64_t)gridDim.x * kWarps,
                         [&](int) { return sg; });
    return;
  }
  if (a.mode == NVFP4_DYNAMIC && blockIdx.x == 0)
    for (int i = threadIdx.x; i < a.n; i += kThreads) *a.t[i].ts = tensor_scale_of(a, i);
  encode_range<T, OUT>(a, (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5), (int64_t)gridDim.x * kWarps,
                       [&](int t) { return tensor_scale_of(a, t); });
}

// Dynamic scales for a small group in one launch: one cluster of
// kSmallCluster CTAs takes each tensor's max |x| over its share of the chunks,
// pushes the per-tensor maxima into every peer through distributed shared
// memory, and after one cluster barrier every CTA holds the tensors' amax and
// encodes its share (the second read of a small group comes from L2).  Same
// results as the amax + encode launches; no workspace words and no clearing
// launch.
constexpr int kSmallCluster = 8;
// At most 256 chunks (128K elements) take this path: eight CTAs keep too few
// loads in flight for more (a 1M-element tensor measured 34 us this way and
// ~12 us as amax + encode launches over the whole GPU; 64K elements: 5 us vs 12).
constexpr int64_t kSmallChunks = 256;

template <typename T, Out OUT>
__global__ void __launch_bounds__(kThreads) group_small_dynamic_kernel(const __grid_constant__ GroupArgs a) {
  __shared__ unsigned s_max[kMaxGroup];
  __shared__ unsigned peer_max[kSmallCluster][kMaxGroup];  // written by every CTA of the cluster
  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  for (int i = threadIdx.x; i < a.n; i += kThreads) s_max[i] = 0u;
  __syncthreads();
  const int64_t per_cta = (a.total_chunks + csize - 1) / csize;
  const int64_t c_begin = (int64_t)crank * per_cta;
  const int64_t c_end = c_begin + per_cta < a.total_chunks ? c_begin + per_cta : a.total_chunks;
  amax_range<T>(a, c_begin, c_end, s_max);
  __syncthreads();
  for (int i = threadIdx.x; i < a.n * csize; i += kThreads) {
    const int r = i / a.n, t = i - r * a.n;
    cluster.map_shared_rank(&peer_max[0][0], r)[crank * kMaxGroup + t] = s_max[t];
  }
  cluster.sync();  // every peer's maxima are here; no CTA writes a peer after this point
  for (int i = threadIdx.x; i < a.n; i += kThreads) {
    unsigned m = peer_max[0][i];
    for (int r = 1; r < csize; ++r) m = max(m, peer_max[r][i]);
    s_max[i] = m;
    if (crank == 0) *a.t[i].ts = __fdiv_rn(__uint_as_float(m), 2688.0f);
  }
  __syncthreads();
  encode_range<T, OUT>(a, (int64_t)crank * kWarps + (threadIdx.x >> 5), (int64_t)csize * kWarps,
                       [&](int t) { return __fdiv_rn(__uint_as_float(s_max[t]), 2688.0f); });
}

// ------------------------------------------------------------------ MSE calibration
//
// Frozen-scale QAD starts from MSE-calibrated scales (Nemotron 3.5 Lightning
// NVFP4 article, "量化尺度处理策略").  With each tensor's s_g given, a
// block's E4M3 scale is the code c (all 127 finite non-negative codes) whose
// fake quantization has the least squared error
//   err(c) = sum_i (x_i - value(q_i) d)^2,  d = value(c) s_g,  q_i = E2M1(x_i / d),
// binary32 operations rounded once, accumulated in element order with FMA,
// ties to the smaller code.  Codes whose d makes every quotient round to 0
// (max|x| / d <= 1/4) reproduce code 0's error exactly (x - (+-0) = x), so
// the search stops at the first of them.  One lane per block; the tensor's
// GTensor.y receives the least error per block (f32, rows x cols/16) when set.
template <typename T>
__global__ void __launch_bounds__(kThreads) group_calib_kernel(const __grid_constant__ GroupArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  int cur = 0;
  for (int64_t c = warp; c < a.total_chunks; c += nwarps) {
    cur = find_tensor(a, c, cur);
    const GTensor& g = a.t[cur];
    int64_t row, col;
    chunk_pos(g, c, lane, row, col);
    if (col >= g.cols) continue;
    Block16<T> in;
    in.load(reinterpret_cast<const T*>(g.x) + row * g.ld_x + col, a.x_wide != 0);
    float v[16];
    in.to_f32(v);
    const float sg = __ldg(g.ts);
    float amax = 0.0f, err0 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      amax = fmaxf(amax, fabsf(v[i]));
      err0 = __fmaf_rn(v[i], v[i], err0);  // code 0 (d = 0): every x^ is 0
    }
    uint32_t best = 0u;
    float best_err = err0;
    for (uint32_t code = 1; code < 127u; ++code) {
      const float d = __fmul_rn(e4m3_decode(code), sg);
      if (d == 0.0f) continue;  // same error as code 0 (a tie: the smaller code stays)
      const bool fast = sizeof(T) == 2 && block_scale_in_fast_range(d);
      const float r = fast ? __frcp_rn(d) : 0.0f;
      const float qmax = fast ? div_by_block_scale(amax, d, r) : __fdiv_rn(amax, d);
      if (qmax <= 0.25f) break;  // this code and every larger one: all quotients round to 0
      float q[16];
      if (fast) {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = div_by_block_scale(v[i], d, r);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], d);
      }
      float q0[8], q1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        q0[i] = q[i];
        q1[i] = q[8 + i];
      }
      float xh[16];
      decode_block16(e2m1x8_encode(q0), e2m1x8_encode(q1), d, xh);
      float err = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float diff = __fsub_rn(v[i], xh[i]);
        err = __fmaf_rn(diff, diff, err);
      }
      if (err < best_err) {
        best_err = err;
        best = code;
      }
    }
    const int64_t kb = col >> 4;
    g.sb[row * (g.cols >> 4) + kb] = (uint8_t)best;
    if (g.y) reinterpret_cast<float*>(g.y)[row * (g.cols >> 4) + kb] = best_err;
  }
}

// s_g[i] = amax[i] / 2688 (the DYNAMIC tensor scale from a given max).
__global__ void global_scale_kernel(const float* __restrict__ amax, int n, float* __restrict__ s_g) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    s_g[i] = __fdiv_rn(amax[i], 2688.0f);
}

// Zero the padding bytes of an MMA-layout scale array (rows beyond `rows`,
// blocks beyond cols/16).  One thread per padded (row, block) slot.
__global__ void zero_mma_padding_kernel(uint8_t* __restrict__ s, int64_t rows, int64_t nblk,
                                        int64_t rows_pad, int64_t kchunks) {
  const int64_t kb_pad = kchunks * 4;
  const int64_t total = rows_pad * kb_pad;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / kb_pad, kb = i - r * kb_pad;
    if (r >= rows || kb >= nblk) s[mma_scale_offset(r, kb, kchunks)] = 0;
  }
}

// ------------------------------------------------------------------ dequantize

template <typename TO>
__global__ void __launch_bounds__(kThreads)
    dequant_kernel(const uint8_t* __restrict__ codes, int64_t ld_codes, const uint8_t* __restrict__ sbs,
                   int layout, int64_t kchunks, const float* __restrict__ tensor_scale, Geom g,
                   TO* __restrict__ out, int64_t ld_out) {
  const float sg = __ldg(tensor_scale);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  const int64_t nblk = g.cols >> 4;
  for (int64_t c0 = warp * kUnroll; c0 < g.total_chunks; c0 += nwarps * kUnroll) {
    uint32_t w[kUnroll], sb[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t row, col;
      g.locate(c0 + u, lane, row, col);
      const bool ok = (c0 + u < g.total_chunks) && col < g.cols;
      w[u] = ok ? __ldg(reinterpret_cast<const uint32_t*>(codes + row * ld_codes + (col >> 1))) : 0u;
      const int64_t kb = col >> 4;
      sb[u] = ok ? (uint32_t)__ldg(sbs + (layout == NVFP4_SCALES_MMA ? mma_scale_offset(row, kb, kchunks)
                                                                     : row * nblk + kb))
                 : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t row, col;
      g.locate(c0 + u, lane, row, col);
      if (!((c0 + u < g.total_chunks) && col < g.cols)) continue;
      const float d = __fmul_rn(e4m3_decode(sb[u]), sg);
      float o[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float lo, hi;
        e2m1x2_decode((w[u] >> (8 * j)) & 0xFF, lo, hi);
        o[2 * j] = __fmul_rn(lo, d);
        o[2 * j + 1] = __fmul_rn(hi, d);
      }
      store8<TO>(out + row * ld_out + col, o);
    }
  }
}

// ------------------------------------------------------------------ self-test

// Compares div_by_block_scale with __fdiv_rn for every divisor significand
// (d = 1 + i * 2^-23, i < 2^23) against every bf16 significand of x (128 of
// them, both signs), with x scaled by 2^k for k in [-4, 3] so that the
// quotient spans [2^-5, 2^4) -- every quotient the E2M1 rounding can resolve.
// Counts mismatching quotients (bitwise) into *mismatches and records one of
// them as (d significand << 16) | ((k + 8) << 8) | x index.
__global__ void selftest_division_kernel(unsigned long long* mismatches, unsigned long long* first) {
  const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;  // divisor significand
  if (i >= (1u << 23)) return;
  const float d = __uint_as_float(0x3F800000u | i);
  const float r = __frcp_rn(d);
  unsigned long long bad = 0;
  for (int k = -4; k <= 3; ++k) {
    for (int s = 0; s < 256; ++s) {
      const uint32_t sign = (s & 128) ? 0x80000000u : 0u;
      const uint32_t bits = sign | ((uint32_t)(127 + k) << 23) | ((uint32_t)(s & 127) << 16);
      const float x = __uint_as_float(bits);
      const float q_fast = div_by_block_scale(x, d, r);
      const float q_ref = __fdiv_rn(x, d);
      if (__float_as_uint(q_fast) != __float_as_uint(q_ref)) {
        ++bad;
        atomicCAS(first, ~0ull, ((unsigned long long)i << 16) | ((unsigned long long)(k + 8) << 8) | (unsigned long long)s);
      }
    }
  }
  // signed zeros
  for (int sgn = 0; sgn < 2; ++sgn) {
    const float x = sgn ? -0.0f : 0.0f;
    if (__float_as_uint(div_by_block_scale(x, d, r)) != __float_as_uint(__fdiv_rn(x, d))) {
      ++bad;
      atomicCAS(first, ~0ull, ((unsigned long long)i << 16) | 0xFF00ull | (unsigned long long)sgn);
    }
  }
  if (bad) atomicAdd(mismatches, bad);
}

// ------------------------------------------------------------------ host side

static int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

static Geom make_geom(int64_t rows, int64_t cols, int64_t ld) {
  Geom g;
  g.rows = rows;
  g.cols = cols;
  g.ld = ld;
  g.chunks_per_row = (cols + kChunk - 1) / kChunk;
  g.total_chunks = rows * g.chunks_per_row;
  return g;
}

// Persistent grid: enough CTAs to cover the work, at most 8 per SM.
static int grid_for(const Geom& g) {
  const int64_t per_cta = (int64_t)kWarps * kUnroll;
  int64_t need = (g.total_chunks + per_cta - 1) / per_cta;
  int64_t cap = (int64_t)sm_count() * 8;
  if (need > cap) need = cap;
  return need < 1 ? 1 : (int)need;
}

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static nvfp4_status check_common(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x) {
  if (dtype != NVFP4_BF16 && dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  if (rows < 0 || cols < 0 || cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (ld_x < cols) return NVFP4_ERR_SHAPE;
  if (rows > 0 && cols > 0) {
    if (!x) return NVFP4_ERR_ARG;
    const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
    if (!aligned16(x) || (ld_x * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  }
  return NVFP4_OK;
}

static nvfp4_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

constexpr size_t kDynamicWorkspace = 1024;  // 256 amax words, >= kMaxGroup
// What the size queries ask for: the amax words, then one word per CTA of a
// single tensor's amax launch (that path needs no clearing launch).  A
// workspace of only kDynamicWorkspace bytes still works (clear + atomics).
constexpr size_t kDynamicWorkspacePart = 8192;
constexpr int kMaxAmaxGrid = (int)((kDynamicWorkspacePart - kDynamicWorkspace) / sizeof(unsigned));

// Validate one tensor of a (possibly grouped) quantize / fake-quant call.
template <Out OUT>
static nvfp4_status check_tensor(const nvfp4_tensor_ref& r, nvfp4_dtype dtype, nvfp4_scale_mode mode,
                                 nvfp4_scale_layout layout) {
  nvfp4_status st = check_common(r.x, dtype, r.rows, r.cols, r.ld_x);
  if (st != NVFP4_OK) return st;
  if (!r.tensor_scale) return NVFP4_ERR_ARG;
  if (mode == NVFP4_FROZEN_ALL && layout != NVFP4_SCALES_ROWMAJOR) return NVFP4_ERR_ARG;
  if (r.rows == 0 || r.cols == 0) return NVFP4_OK;
  if (mode == NVFP4_FROZEN_ALL && !r.block_scales) return NVFP4_ERR_ARG;
  if (!r.out) return NVFP4_ERR_ARG;
  if (OUT != Out::Fake) {
    if (!r.block_scales) return NVFP4_ERR_ARG;
    if (r.ld_out < r.cols / 2) return NVFP4_ERR_SHAPE;
    if ((r.ld_out % 4) != 0 || ((uintptr_t)r.out & 3u) != 0) return NVFP4_ERR_ALIGN;
  } else {
    if (r.ld_out < r.cols) return NVFP4_ERR_SHAPE;
    const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
    if (!aligned16(r.out) || (r.ld_out * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  }
  return NVFP4_OK;
}

// The fake-quant output of an Out::Both call (y, ld_y elements of dtype).
static nvfp4_status check_y(const nvfp4_tensor_ref& r, const void* y, int64_t ld_y, nvfp4_dtype dtype) {
  if (r.rows == 0 || r.cols == 0) return NVFP4_OK;
  if (!y) return NVFP4_ERR_ARG;
  if (ld_y < r.cols) return NVFP4_ERR_SHAPE;
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  if (!aligned16(y) || (ld_y * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

// Resident CTAs per SM of a kernel (256 threads, no dynamic shared memory),
// looked up once per kernel and cached by the kernel's address.
static int resident_per_sm(const void* fn) {
  static const void* keys[16] = {};
  static int vals[16] = {};
  for (int i = 0; i < 16; ++i) {
    if (keys[i] == fn) return vals[i];
    if (keys[i] == nullptr) {
      int v = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, fn, kThreads, 0) != cudaSuccess || v <= 0) v = 1;
      keys[i] = fn;
      vals[i] = v;
      return v;
    }
  }
  return 1;
}

// Persistent grid for a group: at most the resident capacity of the GPU, so
// every CTA of the grid-stride loop runs in the same wave.
static int resident_grid(const void* fn, int64_t total_chunks) {
  const int64_t per_cta = (int64_t)kWarps * kQUnroll;
  int64_t need = (total_chunks + per_cta - 1) / per_cta;
  const int64_t cap = (int64_t)sm_count() * resident_per_sm(fn);
  if (need > cap) need = cap;
  return need < 1 ? 1 : (int)need;
}

// Launch the kernels of one group.  In DYNAMIC mode `amax` points at this
// group's n zeroed words of the workspace.
// One launch: a single cluster of kSmallCluster CTAs (DYNAMIC, small group).
template <Out OUT, typename T>
static nvfp4_status launch_small_dynamic(const GroupArgs& a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSmallCluster);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSmallCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, group_small_dynamic_kernel<T, OUT>, a) != cudaSuccess) return NVFP4_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

// DYNAMIC groups this small take the one-launch cluster path.
static bool small_dynamic(const GroupArgs& a) { return a.mode == NVFP4_DYNAMIC && a.total_chunks <= kSmallChunks; }

// The encode launch of a DYNAMIC group follows its amax launch as a
// programmatic dependent launch: it may be scheduled while the amax launch
// drains and waits (griddepcontrol.wait) before touching memory.
template <typename K>
static nvfp4_status launch_dependent(K kernel, int grid, const GroupArgs& a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, a) != cudaSuccess) return NVFP4_ERR_CUDA;
  count_launches(1);
  return launch_status();
}

template <Out OUT>
static nvfp4_status launch_group(GroupArgs& a, nvfp4_dtype dtype, unsigned* amax, unsigned* amax_part,
                                 cudaStream_t s) {
  if (a.n == 0 || a.total_chunks == 0) return NVFP4_OK;
  if (small_dynamic(a))
    return dtype == NVFP4_BF16 ? launch_small_dynamic<OUT, __nv_bfloat16>(a, s) : launch_small_dynamic<OUT, float>(a, s);
  a.amax_part = nullptr;
  a.amax_grid = 0;
  if (a.mode == NVFP4_DYNAMIC) {
    a.amax = amax;
    const void* fn = dtype == NVFP4_BF16 ? (const void*)group_amax_kernel<__nv_bfloat16> : (const void*)group_amax_kernel<float>;
    const int grid = resident_grid(fn, a.total_chunks);
    if (a.n == 1 && amax_part != nullptr && grid <= kMaxAmaxGrid) {
      a.amax_part = amax_part;
      a.amax_grid = grid;
    }
    if (dtype == NVFP4_BF16)
      group_amax_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(a);
    else
      group_amax_kernel<float><<<grid, kThreads, 0, s>>>(a);
    count_launches(1);
    if (launch_status() != NVFP4_OK) return NVFP4_ERR_CUDA;
    if (dtype == NVFP4_BF16)
      return launch_dependent(group_encode_kernel<__nv_bfloat16, OUT>,
                              resident_grid((const void*)group_encode_kernel<__nv_bfloat16, OUT>, a.total_chunks), a, s);
    return launch_dependent(group_encode_kernel<float, OUT>,
                            resident_grid((const void*)group_encode_kernel<float, OUT>, a.total_chunks), a, s);
  }
  if (dtype == NVFP4_BF16)
    group_encode_kernel<__nv_bfloat16, OUT>
        <<<resident_grid((const void*)group_encode_kernel<__nv_bfloat16, OUT>, a.total_chunks), kThreads, 0, s>>>(a);
  else
    group_encode_kernel<float, OUT>
        <<<resident_grid((const void*)group_encode_kernel<float, OUT>, a.total_chunks), kThreads, 0, s>>>(a);
  count_launches(1);
  return launch_status();
}

// Quantize or fake-quantize a list of tensors: validation of every tensor
// first, then one (FROZEN) or two (DYNAMIC) launches per group.
template <Out OUT>
static nvfp4_status run_tensors(int n, const nvfp4_tensor_ref* refs, nvfp4_dtype dtype, nvfp4_scale_mode mode,
                                nvfp4_scale_layout layout, void* ws, size_t ws_bytes, cudaStream_t s,
                                void* const* ys = nullptr, const int64_t* ld_ys = nullptr) {
  if (n < 0 || (n > 0 && !refs)) return NVFP4_ERR_ARG;
  if (OUT == Out::Both && n > 0 && (!ys || !ld_ys)) return NVFP4_ERR_ARG;
  if (mode != NVFP4_DYNAMIC && mode != NVFP4_FROZEN_GLOBAL && mode != NVFP4_FROZEN_ALL) return NVFP4_ERR_ARG;
  if (layout != NVFP4_SCALES_ROWMAJOR && layout != NVFP4_SCALES_MMA) return NVFP4_ERR_ARG;
  if (OUT == Out::Fake && layout != NVFP4_SCALES_ROWMAJOR) return NVFP4_ERR_ARG;
  for (int i = 0; i < n; ++i) {
    nvfp4_status st = check_tensor<OUT>(refs[i], dtype, mode, layout);
    if (st == NVFP4_OK && OUT == Out::Both) st = check_y(refs[i], ys[i], ld_ys[i], dtype);
    if (st != NVFP4_OK) return st;
  }
  if (mode == NVFP4_DYNAMIC) {
    if (!ws || ws_bytes < kDynamicWorkspace) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_ALIGN;
  }
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  GroupArgs a;  // host staging of the kernel parameter (copied at launch)
  a.n = 0;
  a.amax_part = nullptr;
  a.amax_grid = 0;
  a.mode = (int)mode;
  a.layout = (int)layout;
  a.total_chunks = 0;
  a.amax = nullptr;
  a.x_wide = 1;
  a.out_wide = 1;
  a.y_wide = 1;
  // DYNAMIC: every group takes its own amax words from the workspace; the
  // words are cleared once per call, and again whenever they run out.
  unsigned* words = reinterpret_cast<unsigned*>(ws);
  const int nwords = (int)(kDynamicWorkspace / sizeof(unsigned));
  int word_base = nwords;  // forces a clear before the first group
  // A single-tensor group takes per-CTA maxima in the rest of a workspace of
  // kDynamicWorkspacePart bytes instead (no clear needed).
  unsigned* part = ws_bytes >= kDynamicWorkspacePart ? words + nwords : nullptr;
  auto flush = [&]() -> nvfp4_status {
    if (a.n == 0) return NVFP4_OK;
    const int need = a.n;
    const bool use_part = a.n == 1 && part != nullptr;
    if (mode == NVFP4_DYNAMIC && !small_dynamic(a) && !use_part && word_base + need > nwords) {
      if (cudaMemsetAsync(ws, 0, kDynamicWorkspace, s) != cudaSuccess) return NVFP4_ERR_CUDA;
      word_base = 0;
    }
    nvfp4_status st = launch_group<OUT>(a, dtype, words + word_base, use_part ? part : nullptr, s);
    word_base += need;
    return st;
  };
  for (int i = 0; i < n; ++i) {
    const nvfp4_tensor_ref& r = refs[i];
    if (r.rows == 0 || r.cols == 0) {
      if (mode == NVFP4_DYNAMIC && cudaMemsetAsync(r.tensor_scale, 0, sizeof(float), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
      continue;
    }
    if (r.rows * ((r.cols + kQChunk - 1) / kQChunk) > 0xFFFFFFFFll) return NVFP4_ERR_SHAPE;
    if (a.n == kMaxGroup) {
      nvfp4_status st = flush();
      if (st != NVFP4_OK) return st;
      a.n = 0;
      a.total_chunks = 0;
      a.x_wide = 1;
      a.out_wide = 1;
      a.y_wide = 1;
    }
    GTensor& g = a.t[a.n++];
    g.x = r.x;
    g.codes = OUT != Out::Fake ? reinterpret_cast<uint8_t*>(r.out) : nullptr;
    g.y = OUT == Out::Fake ? r.out : (OUT == Out::Both ? ys[i] : nullptr);
    g.ld_y = OUT == Out::Fake ? r.ld_out : (OUT == Out::Both ? ld_ys[i] : 0);
    g.sb = r.block_scales;
    g.ts = r.tensor_scale;
    g.ld_x = r.ld_x;
    g.ld_out = r.ld_out;
    g.cols = r.cols;
    const int64_t cpr = (r.cols + kQChunk - 1) / kQChunk;
    g.cpr = make_fastdiv((uint32_t)cpr);
    g.rows = r.rows;
    g.chunk0 = a.total_chunks;
    g.kchunks = (r.cols / 16 + 3) / 4;
    a.total_chunks += r.rows * cpr;
    // 32-byte rows for 256-bit input loads; 8-byte code rows / 32-byte y rows
    if (((uintptr_t)r.x & 31u) || ((r.ld_x * esz) & 31)) a.x_wide = 0;
    if (OUT != Out::Fake && (((uintptr_t)r.out & 7u) || (r.ld_out & 7))) a.out_wide = 0;
    if (OUT != Out::Codes && (((uintptr_t)g.y & 31u) || ((g.ld_y * esz) & 31))) a.y_wide = 0;
  }
  nvfp4_status st = flush();
  if (st != NVFP4_OK) return st;
  // zero the padding of MMA-layout scale arrays
  if (OUT != Out::Fake && layout == NVFP4_SCALES_MMA && mode != NVFP4_FROZEN_ALL) {
    for (int i = 0; i < n; ++i) {
      const nvfp4_tensor_ref& r = refs[i];
      if (r.rows == 0 || r.cols == 0) continue;
      const int64_t rows_pad = (r.rows + 127) / 128 * 128;
      const int64_t kchunks = (r.cols / 16 + 3) / 4;
      if (rows_pad == r.rows && (r.cols / 16) % 4 == 0) continue;
      const int64_t total = rows_pad * kchunks * 4;
      int64_t blocks = (total + 255) / 256;
      if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
      zero_mma_padding_kernel<<<(int)blocks, 256, 0, s>>>(r.block_scales, r.rows, r.cols / 16, rows_pad, kchunks);
      count_launches(1);
      if (launch_status() != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
  }
  return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_mma_scales_bytes(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0) return 0;
  return (size_t)((rows + 127) / 128 * 128) * (size_t)((cols / 16 + 3) / 4 * 4);
}

size_t nvfp4_quantize_workspace_size(int64_t rows, int64_t cols, nvfp4_scale_mode mode) {
  (void)rows;
  (void)cols;
  return mode == NVFP4_DYNAMIC ? kDynamicWorkspacePart : 0;
}

size_t nvfp4_fake_quant_workspace_size(int64_t rows, int64_t cols, nvfp4_scale_mode mode) {
  return nvfp4_quantize_workspace_size(rows, cols, mode);
}

size_t nvfp4_grouped_workspace_size(nvfp4_scale_mode mode) { return mode == NVFP4_DYNAMIC ? kDynamicWorkspacePart : 0; }

nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                            nvfp4_scale_mode mode, float* tensor_scale, uint8_t* block_scales,
                            nvfp4_scale_layout layout, uint8_t* codes, int64_t ld_codes, void* workspace,
                            size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("nvfp4_quantize");
  nvfp4_tensor_ref r;
  r.x = x;
  r.rows = rows;
  r.cols = cols;
  r.ld_x = ld_x;
  r.tensor_scale = tensor_scale;
  r.block_scales = block_scales;
  r.out = codes;
  r.ld_out = ld_codes;
  return run_tensors<Out::Codes>(1, &r, dtype, mode, layout, workspace, workspace_bytes, (cudaStream_t)stream);
}

nvfp4_status nvfp4_fake_quant(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                              nvfp4_scale_mode mode, float* tensor_scale, uint8_t* block_scales, void* y,
                              int64_t ld_y, void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("nvfp4_fake_quant");
  nvfp4_tensor_ref r;
  r.x = x;
  r.rows = rows;
  r.cols = cols;
  r.ld_x = ld_x;
  r.tensor_scale = tensor_scale;
  r.block_scales = block_scales;
  r.out = y;
  r.ld_out = ld_y;
  return run_tensors<Out::Fake>(1, &r, dtype, mode, NVFP4_SCALES_ROWMAJOR, workspace, workspace_bytes,
                                (cudaStream_t)stream);
}

nvfp4_status nvfp4_quantize_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                    nvfp4_scale_mode mode, nvfp4_scale_layout layout, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("nvfp4_quantize_grouped");
  return run_tensors<Out::Codes>(num_tensors, tensors, dtype, mode, layout, workspace, workspace_bytes,
                                 (cudaStream_t)stream);
}

nvfp4_status nvfp4_quantize_fake_quant_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, void* const* y,
                                               const int64_t* ld_y, nvfp4_dtype dtype, nvfp4_scale_mode mode,
                                               nvfp4_scale_layout layout, void* workspace, size_t workspace_bytes,
                                               void* stream) {
  NVFP4_ENTRY("nvfp4_quantize_fake_quant_grouped");
  return run_tensors<Out::Both>(num_tensors, tensors, dtype, mode, layout, workspace, workspace_bytes,
                                (cudaStream_t)stream, y, ld_y);
}

nvfp4_status nvfp4_calibrate_mse_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                         float* const* block_err, void* stream) {
  NVFP4_ENTRY("nvfp4_calibrate_mse_grouped");
  if (num_tensors < 0 || (num_tensors > 0 && !tensors)) return NVFP4_ERR_ARG;
  if (dtype != NVFP4_BF16 && dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  for (int i = 0; i < num_tensors; ++i) {
    const nvfp4_tensor_ref& r = tensors[i];
    nvfp4_status st = check_common(r.x, dtype, r.rows, r.cols, r.ld_x);
    if (st != NVFP4_OK) return st;
    if (r.rows == 0 || r.cols == 0) continue;
    if (!r.tensor_scale || !r.block_scales) return NVFP4_ERR_ARG;
    if (block_err && block_err[i] && ((uintptr_t)block_err[i] & 3u)) return NVFP4_ERR_ALIGN;
  }
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  cudaStream_t s = (cudaStream_t)stream;
  static GroupArgs a;
  auto launch = [&]() -> nvfp4_status {
    if (a.n == 0 || a.total_chunks == 0) return NVFP4_OK;
    const void* fn = dtype == NVFP4_BF16 ? (const void*)group_calib_kernel<__nv_bfloat16>
                                         : (const void*)group_calib_kernel<float>;
    int64_t grid = (a.total_chunks + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)sm_count() * resident_per_sm(fn);
    if (grid > cap) grid = cap;
    if (dtype == NVFP4_BF16)
      group_calib_kernel<__nv_bfloat16><<<(int)grid, kThreads, 0, s>>>(a);
    else
      group_calib_kernel<float><<<(int)grid, kThreads, 0, s>>>(a);
    count_launches(1);
    return launch_status();
  };
  a.n = 0;
  a.total_chunks = 0;
  a.mode = NVFP4_FROZEN_GLOBAL;
  a.layout = NVFP4_SCALES_ROWMAJOR;
  a.x_wide = 1;
  for (int i = 0; i < num_tensors; ++i) {
    const nvfp4_tensor_ref& r = tensors[i];
    if (r.rows == 0 || r.cols == 0) continue;
    if (r.rows * ((r.cols + kQChunk - 1) / kQChunk) > 0xFFFFFFFFll) return NVFP4_ERR_SHAPE;
    if (a.n == kMaxGroup) {
      nvfp4_status st = launch();
      if (st != NVFP4_OK) return st;
      a.n = 0;
      a.total_chunks = 0;
      a.x_wide = 1;
    }
    GTensor& g = a.t[a.n++];
    g.x = r.x;
    g.codes = nullptr;
    g.y = block_err ? block_err[i] : nullptr;
    g.sb = r.block_scales;
    g.ts = r.tensor_scale;
    g.ld_x = r.ld_x;
    g.ld_out = 0;
    g.ld_y = 0;
    g.cols = r.cols;
    g.rows = r.rows;
    const int64_t cpr = (r.cols + kQChunk - 1) / kQChunk;
    g.cpr = make_fastdiv((uint32_t)cpr);
    g.chunk0 = a.total_chunks;
    g.kchunks = (r.cols / 16 + 3) / 4;
    a.total_chunks += r.rows * cpr;
    if (((uintptr_t)r.x & 31u) || ((r.ld_x * esz) & 31)) a.x_wide = 0;
  }
  return launch();
}

nvfp4_status nvfp4_tensor_amax_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                       float* amax, void* stream) {
  NVFP4_ENTRY("nvfp4_tensor_amax_grouped");
  if (num_tensors < 0 || (num_tensors > 0 && (!tensors || !amax))) return NVFP4_ERR_ARG;
  if (dtype != NVFP4_BF16 && dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  if ((uintptr_t)amax & 3u) return NVFP4_ERR_ALIGN;
  for (int i = 0; i < num_tensors; ++i) {
    nvfp4_status st = check_common(tensors[i].x, dtype, tensors[i].rows, tensors[i].cols, tensors[i].ld_x);
    if (st != NVFP4_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (num_tensors == 0) return NVFP4_OK;
  // max |x| >= 0 compares like its bit pattern: the words start at 0 (= +0.0f)
  if (cudaMemsetAsync(amax, 0, (size_t)num_tensors * sizeof(float), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  static GroupArgs a;
  int first = 0;  // tensor index of a.t[0]
  auto launch = [&]() -> nvfp4_status {
    if (a.n == 0 || a.total_chunks == 0) return NVFP4_OK;
    a.amax = reinterpret_cast<unsigned*>(amax) + first;
    const void* fn = dtype == NVFP4_BF16 ? (const void*)group_amax_kernel<__nv_bfloat16>
                                         : (const void*)group_amax_kernel<float>;
    if (dtype == NVFP4_BF16)
      group_amax_kernel<__nv_bfloat16><<<resident_grid(fn, a.total_chunks), kThreads, 0, s>>>(a);
    else
      group_amax_kernel<float><<<resident_grid(fn, a.total_chunks), kThreads, 0, s>>>(a);
    count_launches(1);
    return launch_status();
  };
  a.n = 0;
  a.total_chunks = 0;
  a.mode = NVFP4_DYNAMIC;
  a.x_wide = 1;
  // tensors map to consecutive words: a group holds consecutive tensors, empty ones included
  for (int i = 0; i < num_tensors; ++i) {
    const nvfp4_tensor_ref& r = tensors[i];
    if (r.rows * ((r.cols + kQChunk - 1) / kQChunk) > 0xFFFFFFFFll) return NVFP4_ERR_SHAPE;
    if (a.n == kMaxGroup) {
      nvfp4_status st = launch();
      if (st != NVFP4_OK) return st;
      first = i;
      a.n = 0;
      a.total_chunks = 0;
      a.x_wide = 1;
    }
    GTensor& g = a.t[a.n++];
    g.x = r.x;
    g.codes = nullptr;
    g.y = nullptr;
    g.sb = nullptr;
    g.ts = nullptr;
    g.ld_x = r.ld_x;
    g.ld_out = 0;
    g.ld_y = 0;
    g.cols = r.cols > 0 ? r.cols : 16;
    g.rows = r.cols > 0 ? r.rows : 0;
    const int64_t cpr = (g.cols + kQChunk - 1) / kQChunk;
    g.cpr = make_fastdiv((uint32_t)cpr);
    g.chunk0 = a.total_chunks;
    g.kchunks = (g.cols / 16 + 3) / 4;
    a.total_chunks += g.rows * cpr;
    if (((uintptr_t)r.x & 31u) || ((r.ld_x * esz) & 31)) a.x_wide = 0;
  }
  return launch();
}

nvfp4_status nvfp4_global_scale_from_amax(const float* amax, int n, float* tensor_scale, void* stream) {
  NVFP4_ENTRY("nvfp4_global_scale_from_amax");
  if (n < 0 || (n > 0 && (!amax || !tensor_scale))) return NVFP4_ERR_ARG;
  if (n == 0) return NVFP4_OK;
  global_scale_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>(amax, n, tensor_scale);
  count_launches(1);
  return launch_status();
}

nvfp4_status nvfp4_calibrate_mse(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                                 const float* tensor_scale, uint8_t* block_scales, float* block_err, void* stream) {
  NVFP4_ENTRY("nvfp4_calibrate_mse");
  nvfp4_tensor_ref r;
  r.x = x;
  r.rows = rows;
  r.cols = cols;
  r.ld_x = ld_x;
  r.tensor_scale = const_cast<float*>(tensor_scale);
  r.block_scales = block_scales;
  r.out = nullptr;
  r.ld_out = 0;
  float* errs[1] = {block_err};
  return nvfp4_calibrate_mse_grouped(1, &r, dtype, errs, stream);
}

nvfp4_status nvfp4_fake_quant_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                      nvfp4_scale_mode mode, void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("nvfp4_fake_quant_grouped");
  return run_tensors<Out::Fake>(num_tensors, tensors, dtype, mode, NVFP4_SCALES_ROWMAJOR, workspace,
                                workspace_bytes, (cudaStream_t)stream);
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, int64_t ld_codes, const uint8_t* block_scales,
                              nvfp4_scale_layout layout, const float* tensor_scale, int64_t rows, int64_t cols,
                              void* out, nvfp4_dtype out_dtype, int64_t ld_out, void* stream) {
  NVFP4_ENTRY("nvfp4_dequantize");
  if (out_dtype != NVFP4_BF16 && out_dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  if (rows < 0 || cols < 0 || cols % 16 != 0 || ld_codes < cols / 2 || ld_out < cols) return NVFP4_ERR_SHAPE;
  if (layout != NVFP4_SCALES_ROWMAJOR && layout != NVFP4_SCALES_MMA) return NVFP4_ERR_ARG;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!codes || !block_scales || !tensor_scale || !out) return NVFP4_ERR_ARG;
  const int64_t esz = out_dtype == NVFP4_BF16 ? 2 : 4;
  if (((uintptr_t)codes & 3u) || (ld_codes % 4) || !aligned16(out) || (ld_out * esz) % 16) return NVFP4_ERR_ALIGN;
  Geom g = make_geom(rows, cols, cols);
  const int grid = grid_for(g);
  const int64_t kchunks = (cols / 16 + 3) / 4;
  cudaStream_t s = (cudaStream_t)stream;
  if (out_dtype == NVFP4_BF16)
    dequant_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(codes, ld_codes, block_scales, (int)layout, kchunks,
                                                            tensor_scale, g, reinterpret_cast<__nv_bfloat16*>(out),
                                                            ld_out);
  else
    dequant_kernel<float><<<grid, kThreads, 0, s>>>(codes, ld_codes, block_scales, (int)layout, kchunks,
                                                    tensor_scale, g, reinterpret_cast<float*>(out), ld_out);
  count_launches(1);
  return launch_status();
}

// Self-test of the per-block division used by the bf16 encode path against
// __fdiv_rn; see selftest_division_kernel.  Both outputs are device words of
// 8 bytes, initialised here: the mismatch count, and one mismatch (or
// all ones when there is none).
nvfp4_status nvfp4_selftest_division(uint64_t* mismatches, uint64_t* first, void* stream) {
  NVFP4_ENTRY("nvfp4_selftest_division");
  if (!mismatches || !first) return NVFP4_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(mismatches, 0, sizeof(uint64_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaMemsetAsync(first, 0xFF, sizeof(uint64_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  selftest_division_kernel<<<(1 << 23) / 256, 256, 0, s>>>(reinterpret_cast<unsigned long long*>(mismatches),
                                                           reinterpret_cast<unsigned long long*>(first));
  count_launches(1);
  return launch_status();
}

}  // extern "C"
