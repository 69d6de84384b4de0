// gemm_bf16.cu -- grouped BF16 GEMMs on the sm_100a tensor cores
// (tcgen05.mma.kind::f16, FP32 accumulation in tensor memory) for the
// backward pass of the QAD student's MoE layer: with the straight-through
// estimator the gradients flow through the dequantized weights and
// activations as plain BF16 products (Nemotron 3.5 Lightning NVFP4 article,
// "QAD的工作原理": the quantized student is trained through simulated
// quantization).
//
// C = A * B^T with A [rows][K] and B [cols][K] both K-major (the contiguous
// dimension is the reduction), bf16 in, bf16 out.  Two ways to group:
//   M-segments  group g owns rows [off[g], off[g] + len[g]) of A and C (off a
//               multiple of 128), B of group g is rows [g N, (g+1) N) of B.
//               Used for dA = dY W_down and dX = dGU [W_gate; W_up].
//   K-segments  group g reduces over columns [off[g], off[g] + len[g]) of A
//               and B (the group's tokens; off and the padded length are
//               multiples of 64, padding holds zeros); C of group g is rows
//               [g M, (g+1) M).  Used for the weight gradients dW = dY^T A.
// Persistent CTAs, 128 x 256 tiles, 4-stage TMA ring (128-byte swizzle),
// 8 epilogue warps, every wait bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "ptx.cuh"

namespace nvfp4 {

namespace bf16gemm {

constexpr int BM = 128, BN = 256;
constexpr int BK = 64;                    // bf16 elements per stage = 128 bytes per row
constexpr int KB = BK / 16;               // MMAs (K = 16) per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB
constexpr int B_BYTES = BN * BK * 2;      // 32 KiB
constexpr int MAX_GROUPS = 256;
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + 1024 + 256 + (2 * MAX_GROUPS + 1) * 4;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int TM_COLS = 256;
// BF16 x BF16 -> F32 (c_format 1 in bits 4-5, a/b format 1 in bits 7-9 / 10-12),
// K-major A and B, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct Params {
  __nv_bfloat16* c;
  int64_t ldc;
  int M, N, K;            // M: rows of A (M-segments: padded total); K: reduction (M-segments)
  int mode;               // 0 = M-segments, 1 = K-segments
  int groups;
  const int32_t* off;     // device [groups + 1]
  const int32_t* len;     // device [groups]
  int c_vec16;
};

struct Tile {
  int g, m0, n0, a_row, b_row, c_row0, row_end;
  int k0, nk;             // first K column and number of K stages
  bool empty;
};

NVFP4_DEV Tile tile_of(int t, const Params& p, const int32_t* s_off, const int32_t* s_len, int num_n, int num_m) {
  Tile tl;
  if (p.mode == 0) {
    const int mt = t / num_n;
    tl.m0 = mt * BM;
    tl.n0 = (t - mt * num_n) * BN;
    int lo = 0, hi = p.groups - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= tl.m0) lo = mid;
      else hi = mid - 1;
    }
    tl.g = lo;
    tl.a_row = tl.m0;
    tl.b_row = lo * p.N + tl.n0;
    tl.c_row0 = 0;
    tl.row_end = s_off[lo] + s_len[lo];
    tl.k0 = 0;
    tl.nk = (p.K + BK - 1) / BK;
    tl.empty = tl.m0 >= tl.row_end;
  } else {
    const int per_g = num_m * num_n;
    tl.g = t / per_g;
    const int r = t - tl.g * per_g;
    const int mt = r / num_n;
    tl.m0 = mt * BM;
    tl.n0 = (r - mt * num_n) * BN;
    tl.a_row = tl.m0;
    tl.b_row = tl.n0;
    tl.c_row0 = tl.g * p.M;
    tl.row_end = p.M;
    tl.k0 = s_off[tl.g];
    tl.nk = (s_len[tl.g] + BK - 1) / BK;
    tl.empty = false;  // an empty segment still writes its zero gradient
  }
  return tl;
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  int32_t* s_off = reinterpret_cast<int32_t*>(smem + STAGES * (A_BYTES + B_BYTES) + 256);
  int32_t* s_len = s_off + MAX_GROUPS + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < p.groups; i += blockDim.x) {
    s_off[i] = __ldg(p.off + i);
    s_len[i] = __ldg(p.len + i);
  }
  if (threadIdx.x == 0) s_off[p.groups] = __ldg(p.off + p.groups);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, EPI_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int num_n = (p.N + BN - 1) / BN;
  const int num_m = (p.mode == 0 ? s_off[p.groups] : p.M + BM - 1) / BM;
  const int num_tiles = p.mode == 0 ? num_m * num_n : p.groups * num_m * num_n;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const Tile tl = tile_of(t, p, s_off, s_len, num_n, num_m);
        if (tl.empty) continue;
        for (int kt = 0; kt < tl.nk; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          mbar_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES));
          tma_load_2d(sA + s * A_BYTES, &tmA, tl.k0 + kt * BK, tl.a_row, &full[s]);
          tma_load_2d(sB + s * B_BYTES, &tmB, tl.k0 + kt * BK, tl.b_row, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, ti = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const Tile tl = tile_of(t, p, s_off, s_len, num_n, num_m);
        if (tl.empty) continue;
        if (!mbar_wait_bounded(acc_empty, ((uint32_t)ti & 1u) ^ 1u)) { *abort_flag = 1; break; }
        tc_fence_after();
        for (int kt = 0; kt < tl.nk; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&full[s], ph)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * B_BYTES);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            // K = 16 bf16 = 32 bytes further along the 128-byte swizzled row
            const uint64_t ad = smem_desc(a_base + kb * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_base + kb * 32, 16, 1024, 2);
            mma_bf16(tmem, ad, bd, IDESC, (kt > 0 || kb > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(acc_full);
        ++ti;
      }
    }
  } else {
    const int sub = warp & 3;
    const int cbase = ((warp - 2) >> 2) * (BN / 2);
    constexpr int HALF = BN / 2;
    int ti = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const Tile tl = tile_of(t, p, s_off, s_len, num_n, num_m);
      if (tl.empty) continue;
      const int par_ti = ti++;
      const bool ok = mbar_wait_bounded(acc_full, (uint32_t)par_ti & 1u);
      if (!ok) *abort_flag = 1;
      if (!ok || *abort_flag) break;
      tc_fence_after();
      uint32_t packed[HALF / 2];
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 64) {
        uint32_t r0[32], r1[32];
        const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + cbase + c0;
        tmem_ld_32x32b_x32(taddr, r0);
        tmem_ld_32x32b_x32(taddr + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          // a K-segment of length 0 issued no MMA: its gradient is zero
          const float f0 = tl.nk > 0 ? __uint_as_float(r0[2 * j]) : 0.f, f1 = tl.nk > 0 ? __uint_as_float(r0[2 * j + 1]) : 0.f;
          const float g0 = tl.nk > 0 ? __uint_as_float(r1[2 * j]) : 0.f, g1 = tl.nk > 0 ? __uint_as_float(r1[2 * j + 1]) : 0.f;
          packed[c0 / 2 + j] = pack_bf16x2(f0, f1);
          packed[c0 / 2 + 16 + j] = pack_bf16x2(g0, g1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int row = tl.m0 + sub * 32 + lane;
      if (row < tl.row_end) {
        __nv_bfloat16* crow = p.c + ((int64_t)tl.c_row0 + row) * p.ldc;
#pragma unroll
        for (int c0 = 0; c0 < HALF; c0 += 32) {
          const int col0 = tl.n0 + cbase + c0;
          if (col0 + 32 <= p.N && p.c_vec16) {
            uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              dst[j] = make_uint4(packed[c0 / 2 + 4 * j], packed[c0 / 2 + 4 * j + 1], packed[c0 / 2 + 4 * j + 2],
                                  packed[c0 / 2 + 4 * j + 3]);
          } else {
            for (int j = 0; j < 32; ++j) {
              if (col0 + j < p.N) {
                const uint32_t w = packed[(c0 + j) >> 1];
                const uint32_t h = (j & 1) ? (w >> 16) : (w & 0xFFFFu);
                crow[col0 + j] = __ushort_as_bfloat16((unsigned short)h);
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(q);
  }
  return fn;
}

// bf16 matrix [rows][cols] with row stride ld elements -> tensor map with a
// box of box_rows x 64 elements (128 bytes), 128-byte swizzle, zero fill.
static bool tmap_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace bf16gemm
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_gemm_bf16_grouped(int mode, int groups, const void* a, int64_t a_rows, int64_t a_cols,
                                                int64_t lda, const void* b, int64_t b_rows, int64_t ldb,
                                                const int32_t* seg_off, const int32_t* seg_len, int64_t M,
                                                int64_t N, int64_t K, void* c, int64_t ldc, void* stream) {
  using namespace bf16gemm;
  if (mode != 0 && mode != 1) return NVFP4_ERR_ARG;
  if (groups < 1 || groups > MAX_GROUPS) return NVFP4_ERR_SHAPE;
  if (!a || !b || !seg_off || !seg_len || !c) return NVFP4_ERR_ARG;
  if (a_rows < 1 || a_cols < 1 || b_rows < 1 || lda < a_cols || ldb < a_cols || N < 1 || ldc < N) return NVFP4_ERR_SHAPE;
  if (mode == 0 && (K < 64 || K % 64 != 0 || K > a_cols || a_rows % 128 != 0 || b_rows < (int64_t)groups * N))
    return NVFP4_ERR_SHAPE;
  if (mode == 1 && (M < 1 || M > a_rows || N > b_rows)) return NVFP4_ERR_SHAPE;
  if (a_rows > 0x7FFFFFFF || b_rows > 0x7FFFFFFF || a_cols > 0x7FFFFFFF || (int64_t)groups * M > 0x7FFFFFFF)
    return NVFP4_ERR_SHAPE;
  if (((uintptr_t)a & 15u) || ((uintptr_t)b & 15u) || (lda * 2) % 16 || (ldb * 2) % 16 || ((uintptr_t)c & 3u))
    return NVFP4_ERR_ALIGN;
  CUtensorMap ta, tb;
  if (!tmap_bf16(&ta, a, a_rows, a_cols, lda, BM) || !tmap_bf16(&tb, b, b_rows, a_cols, ldb, BN)) return NVFP4_ERR_CUDA;
  Params p;
  p.c = reinterpret_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.M = (int)(mode == 0 ? a_rows : M);
  p.N = (int)N;
  p.K = (int)K;
  p.mode = mode;
  p.groups = groups;
  p.off = seg_off;
  p.len = seg_len;
  p.c_vec16 = (((uintptr_t)c & 15u) == 0 && (ldc % 8) == 0) ? 1 : 0;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    attr = true;
  }
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  gemm_bf16_kernel<<<sms, THREADS, SMEM_BYTES, (cudaStream_t)stream>>>(ta, tb, p);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
