// quantize.cu -- NVFP4 quantize / fake-quantize / dequantize for sm_100a.
//
// NVFP4 (Nemotron-3-Nano-30B NVFP4 article, "NVFP4-Format und warum es
// wichtig ist?"): E2M1 elements in blocks of 16 along the contiguous
// dimension, one E4M3 scale per block, one FP32 scale per tensor.  Scale
// modes (Nemotron 3.5 Lightning NVFP4 article, "量化尺度处理策略"): dynamic
// (recomputed from the max on every call) or frozen (passed in).
//
// Work decomposition.  These kernels stream HBM: every input byte is read
// once per pass with 16-byte non-allocating loads and every output written
// once.  A lane owns 8 consecutive elements (16 B of bf16), so a lane pair
// owns one 16-element block and the block max is one shuffle (lane ^ 1).  A
// warp covers a 256-element chunk of a row; chunks are numbered row-major and
// each warp takes UNROLL consecutive chunks per iteration so that several
// independent 16-byte loads per lane are in flight.  Grids are persistent:
// a multiple of the SM count, grid-striding over chunks.
//
// Dynamic mode is two launches in stream order: amax_partial_kernel writes one
// per-CTA partial max into the workspace, and the encode kernel reduces those
// partials at entry (max is exact, so any order gives the same s_g).
#include "common.cuh"

namespace nvfp4 {

constexpr int kThreads = 256;           // 8 warps per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;              // chunks per warp per iteration
constexpr int kChunk = 256;             // elements per warp per chunk
constexpr int kMaxPartials = 1024;      // amax partials (one per amax CTA)

// ------------------------------------------------------------------ input traits

template <typename T>
struct Lane8;

// bf16: one 16-byte load per lane.
template <>
struct Lane8<__nv_bfloat16> {
  uint4 raw;
  NVFP4_DEV void load(const __nv_bfloat16* p) { raw = ld_stream_v4(p); }
  NVFP4_DEV void zero() { raw = make_uint4(0, 0, 0, 0); }
  NVFP4_DEV void to_f32(float (&v)[8]) const {
    v[0] = bf16lo_to_f32(raw.x); v[1] = bf16hi_to_f32(raw.x);
    v[2] = bf16lo_to_f32(raw.y); v[3] = bf16hi_to_f32(raw.y);
    v[4] = bf16lo_to_f32(raw.z); v[5] = bf16hi_to_f32(raw.z);
    v[6] = bf16lo_to_f32(raw.w); v[7] = bf16hi_to_f32(raw.w);
  }
};

// f32: two 16-byte loads per lane.
template <>
struct Lane8<float> {
  uint4 a, b;
  NVFP4_DEV void load(const float* p) { a = ld_stream_v4(p); b = ld_stream_v4(p + 4); }
  NVFP4_DEV void zero() { a = b = make_uint4(0, 0, 0, 0); }
  NVFP4_DEV void to_f32(float (&v)[8]) const {
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
    v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
  }
};

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

// ------------------------------------------------------------------ amax

// One partial max of |x| per CTA.
template <typename T>
__global__ void __launch_bounds__(kThreads) amax_partial_kernel(const T* __restrict__ x, Geom g,
                                                                float* __restrict__ partial) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  float m = 0.0f;
  for (int64_t c0 = warp * kUnroll; c0 < g.total_chunks; c0 += nwarps * kUnroll) {
    Lane8<T> in[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t row, col;
      g.locate(c0 + u, lane, row, col);
      if (c0 + u < g.total_chunks && col < g.cols) in[u].load(x + row * g.ld + col);
      else in[u].zero();
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float v[8];
      in[u].to_f32(v);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    }
  }
  m = warp_max(m);
  __shared__ float s[kWarps];
  if (lane == 0) s[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kWarps ? s[threadIdx.x] : 0.0f;
    v = warp_max(v);
    if (threadIdx.x == 0) partial[blockIdx.x] = v;
  }
}

// ------------------------------------------------------------------ encode

enum class Out { Codes, Fake };

struct EncodeArgs {
  Geom g;
  int mode;                   // nvfp4_scale_mode
  const float* partial;       // DYNAMIC: amax partials
  int npartial;
  float* tensor_scale;        // DYNAMIC: written by CTA 0; else read
  uint8_t* block_scales;      // FROZEN_ALL: read (row-major); else written if non-NULL
  int scale_layout;           // nvfp4_scale_layout of block_scales (written case)
  int64_t kchunks;            // MMA layout: ceil(cols/64)
  uint8_t* codes;             // Out::Codes
  int64_t ld_codes;
  void* y;                    // Out::Fake
  int64_t ld_y;
};

// Resolve s_g at kernel entry (every CTA): reduce the amax partials in DYNAMIC
// mode, otherwise read the given scale.
NVFP4_DEV float resolve_tensor_scale(const EncodeArgs& a) {
  __shared__ float s_sg;
  if (a.mode == NVFP4_DYNAMIC) {
    if (threadIdx.x < 32) {
      float m = 0.0f;
      for (int i = threadIdx.x; i < a.npartial; i += 32) m = fmaxf(m, a.partial[i]);
      m = warp_max(m);
      if (threadIdx.x == 0) {
        float sg = __fdiv_rn(m, 2688.0f);  // amax / (6 * 448)
        s_sg = sg;
        if (blockIdx.x == 0) *a.tensor_scale = sg;
      }
    }
  } else if (threadIdx.x == 0) {
    s_sg = *a.tensor_scale;
  }
  __syncthreads();
  return s_sg;
}

template <typename T, Out OUT>
__global__ void __launch_bounds__(kThreads) encode_kernel(const T* __restrict__ x, EncodeArgs a) {
  const float sg = resolve_tensor_scale(a);
  const float denom6 = __fmul_rn(6.0f, sg);
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kWarps;
  const Geom& g = a.g;
  const int64_t nblk = g.cols >> 4;
  const bool frozen_all = a.mode == NVFP4_FROZEN_ALL;

  for (int64_t c0 = warp * kUnroll; c0 < g.total_chunks; c0 += nwarps * kUnroll) {
    Lane8<T> in[kUnroll];
    uint32_t sb_in[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t row, col;
      g.locate(c0 + u, lane, row, col);
      const bool ok = (c0 + u < g.total_chunks) && col < g.cols;
      if (ok) in[u].load(x + row * g.ld + col);
      else in[u].zero();
      sb_in[u] = (frozen_all && ok) ? (uint32_t)__ldg(a.block_scales + row * nblk + (col >> 4)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      int64_t row, col;
      g.locate(c0 + u, lane, row, col);
      const bool ok = (c0 + u < g.total_chunks) && col < g.cols;
      float v[8];
      in[u].to_f32(v);
      // ---- block scale
      uint32_t sb;
      if (frozen_all) {
        sb = sb_in[u];
      } else {
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        sb = (sg == 0.0f) ? 0u : e4m3_encode(__fdiv_rn(m, denom6));
      }
      const float d = __fmul_rn(e4m3_decode(sb), sg);
      // ---- element codes
      uint32_t word = 0;
      if (d != 0.0f) {
        float q[8];
        if (sizeof(T) == 2 && block_scale_in_fast_range(d)) {
          const float r = __frcp_rn(d);
#pragma unroll
          for (int i = 0; i < 8; ++i) q[i] = div_by_block_scale(v[i], d, r);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(v[i], d);
        }
        word = e2m1x8_encode(q);
      }
      if (!ok) continue;
      // ---- outputs
      if (OUT == Out::Codes) {
        st_stream_u32(a.codes + row * a.ld_codes + (col >> 1), word);
      } else {
        float o[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float lo, hi;
          e2m1x2_decode((word >> (8 * j)) & 0xFF, lo, hi);
          o[2 * j] = __fmul_rn(lo, d);
          o[2 * j + 1] = __fmul_rn(hi, d);
        }
        store8<T>(reinterpret_cast<T*>(a.y) + row * a.ld_y + col, o);
      }
      if (!frozen_all && a.block_scales != nullptr && (lane & 1) == 0) {
        const int64_t kb = col >> 4;
        const int64_t off = (a.scale_layout == NVFP4_SCALES_MMA) ? mma_scale_offset(row, kb, a.kchunks)
                                                                 : row * nblk + kb;
        a.block_scales[off] = (uint8_t)sb;
      }
    }
  }
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

static int amax_grid(const Geom& g) {
  int gsz = grid_for(g);
  return gsz > kMaxPartials ? kMaxPartials : gsz;
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

// Shared driver of quantize and fake-quant.
template <Out OUT>
static nvfp4_status run_encode(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                               nvfp4_scale_mode mode, float* tensor_scale, uint8_t* block_scales,
                               nvfp4_scale_layout layout, uint8_t* codes, int64_t ld_codes, void* y,
                               int64_t ld_y, void* ws, size_t ws_bytes, cudaStream_t stream) {
  Geom g = make_geom(rows, cols, ld_x);
  EncodeArgs a;
  a.g = g;
  a.mode = (int)mode;
  a.tensor_scale = tensor_scale;
  a.block_scales = block_scales;
  a.scale_layout = (int)layout;
  a.kchunks = (cols / 16 + 3) / 4;
  a.codes = codes;
  a.ld_codes = ld_codes;
  a.y = y;
  a.ld_y = ld_y;
  a.partial = reinterpret_cast<float*>(ws);
  a.npartial = 0;
  if (mode == NVFP4_DYNAMIC) {
    a.npartial = amax_grid(g);
    if (dtype == NVFP4_BF16)
      amax_partial_kernel<__nv_bfloat16><<<a.npartial, kThreads, 0, stream>>>(
          reinterpret_cast<const __nv_bfloat16*>(x), g, reinterpret_cast<float*>(ws));
    else
      amax_partial_kernel<float><<<a.npartial, kThreads, 0, stream>>>(reinterpret_cast<const float*>(x), g,
                                                                      reinterpret_cast<float*>(ws));
    if (launch_status() != NVFP4_OK) return NVFP4_ERR_CUDA;
  }
  const int grid = grid_for(g);
  if (dtype == NVFP4_BF16)
    encode_kernel<__nv_bfloat16, OUT><<<grid, kThreads, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(x), a);
  else
    encode_kernel<float, OUT><<<grid, kThreads, 0, stream>>>(reinterpret_cast<const float*>(x), a);
  if (launch_status() != NVFP4_OK) return NVFP4_ERR_CUDA;
  if (OUT == Out::Codes && layout == NVFP4_SCALES_MMA && mode != NVFP4_FROZEN_ALL) {
    const int64_t rows_pad = (rows + 127) / 128 * 128;
    if (rows_pad != rows || (cols / 16) % 4 != 0) {
      const int64_t total = rows_pad * a.kchunks * 4;
      int64_t blocks = (total + 255) / 256;
      if (blocks > (int64_t)sm_count() * 8) blocks = (int64_t)sm_count() * 8;
      zero_mma_padding_kernel<<<(int)blocks, 256, 0, stream>>>(block_scales, rows, cols / 16, rows_pad,
                                                               a.kchunks);
      if (launch_status() != NVFP4_OK) return NVFP4_ERR_CUDA;
    }
  }
  (void)ws_bytes;
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
  return mode == NVFP4_DYNAMIC ? (size_t)kMaxPartials * sizeof(float) : 0;
}

size_t nvfp4_fake_quant_workspace_size(int64_t rows, int64_t cols, nvfp4_scale_mode mode) {
  return nvfp4_quantize_workspace_size(rows, cols, mode);
}

nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                            nvfp4_scale_mode mode, float* tensor_scale, uint8_t* block_scales,
                            nvfp4_scale_layout layout, uint8_t* codes, int64_t ld_codes, void* workspace,
                            size_t workspace_bytes, void* stream) {
  nvfp4_status st = check_common(x, dtype, rows, cols, ld_x);
  if (st != NVFP4_OK) return st;
  if (mode != NVFP4_DYNAMIC && mode != NVFP4_FROZEN_GLOBAL && mode != NVFP4_FROZEN_ALL) return NVFP4_ERR_ARG;
  if (layout != NVFP4_SCALES_ROWMAJOR && layout != NVFP4_SCALES_MMA) return NVFP4_ERR_ARG;
  if (mode == NVFP4_FROZEN_ALL && layout != NVFP4_SCALES_ROWMAJOR) return NVFP4_ERR_ARG;
  if (!tensor_scale) return NVFP4_ERR_ARG;
  if (ld_codes < cols / 2) return NVFP4_ERR_SHAPE;
  const size_t need = nvfp4_quantize_workspace_size(rows, cols, mode);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return NVFP4_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return NVFP4_ERR_ALIGN;
  if (rows == 0 || cols == 0) {
    if (mode == NVFP4_DYNAMIC)
      return cudaMemsetAsync(tensor_scale, 0, sizeof(float), (cudaStream_t)stream) == cudaSuccess ? NVFP4_OK
                                                                                                : NVFP4_ERR_CUDA;
    return NVFP4_OK;
  }
  if (!block_scales || !codes) return NVFP4_ERR_ARG;
  if ((ld_codes % 4) != 0 || ((uintptr_t)codes & 3u) != 0) return NVFP4_ERR_ALIGN;
  return run_encode<Out::Codes>(x, dtype, rows, cols, ld_x, mode, tensor_scale, block_scales, layout, codes,
                                ld_codes, nullptr, 0, workspace, workspace_bytes, (cudaStream_t)stream);
}

nvfp4_status nvfp4_fake_quant(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                              nvfp4_scale_mode mode, float* tensor_scale, uint8_t* block_scales, void* y,
                              int64_t ld_y, void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4_status st = check_common(x, dtype, rows, cols, ld_x);
  if (st != NVFP4_OK) return st;
  if (mode != NVFP4_DYNAMIC && mode != NVFP4_FROZEN_GLOBAL && mode != NVFP4_FROZEN_ALL) return NVFP4_ERR_ARG;
  if (!tensor_scale) return NVFP4_ERR_ARG;
  if (mode == NVFP4_FROZEN_ALL && !block_scales) return NVFP4_ERR_ARG;
  if (ld_y < cols) return NVFP4_ERR_SHAPE;
  const size_t need = nvfp4_fake_quant_workspace_size(rows, cols, mode);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return NVFP4_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return NVFP4_ERR_ALIGN;
  if (rows == 0 || cols == 0) {
    if (mode == NVFP4_DYNAMIC)
      return cudaMemsetAsync(tensor_scale, 0, sizeof(float), (cudaStream_t)stream) == cudaSuccess ? NVFP4_OK
                                                                                                : NVFP4_ERR_CUDA;
    return NVFP4_OK;
  }
  if (!y) return NVFP4_ERR_ARG;
  const int64_t esz = dtype == NVFP4_BF16 ? 2 : 4;
  if (!aligned16(y) || (ld_y * esz) % 16 != 0) return NVFP4_ERR_ALIGN;
  return run_encode<Out::Fake>(x, dtype, rows, cols, ld_x, mode, tensor_scale, block_scales,
                               NVFP4_SCALES_ROWMAJOR, nullptr, 0, y, ld_y, workspace, workspace_bytes,
                               (cudaStream_t)stream);
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, int64_t ld_codes, const uint8_t* block_scales,
                              nvfp4_scale_layout layout, const float* tensor_scale, int64_t rows, int64_t cols,
                              void* out, nvfp4_dtype out_dtype, int64_t ld_out, void* stream) {
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
  return launch_status();
}

// Self-test of the per-block division used by the bf16 encode path against
// __fdiv_rn; see selftest_division_kernel.  Both outputs are device words of
// 8 bytes, initialised here: the mismatch count, and one mismatch (or
// all ones when there is none).
nvfp4_status nvfp4_selftest_division(uint64_t* mismatches, uint64_t* first, void* stream) {
  if (!mismatches || !first) return NVFP4_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(mismatches, 0, sizeof(uint64_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaMemsetAsync(first, 0xFF, sizeof(uint64_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  selftest_division_kernel<<<(1 << 23) / 256, 256, 0, s>>>(reinterpret_cast<unsigned long long*>(mismatches),
                                                           reinterpret_cast<unsigned long long*>(first));
  return launch_status();
}

}  // extern "C"
