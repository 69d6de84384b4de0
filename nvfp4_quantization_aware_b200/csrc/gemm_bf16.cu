// gemm_bf16.cu -- grouped BF16 GEMMs on the sm_100a tensor cores
// (tcgen05.mma.kind::f16, FP32 accumulation in tensor memory) for the
// backward pass of the QAD student's MoE layer: with the straight-through
// estimator the gradients flow through the dequantized weights and
// activations as plain BF16 products (Nemotron 3.5 Lightning NVFP4 article,
// "QAD的工作原理": the quantized student is trained through simulated
// quantization).
//
// C = A * B^T, bf16 in, bf16 out.  Each operand is either K-major (stored
// rows x K, K contiguous) or MN-major (stored K x rows, its M or N index
// contiguous), so that every backward product reads the forward's tensors
// in the layout they already have: no transposes.
//
// Two ways to group:
//   M-segments  group g owns rows [off[g], off[g] + len[g]) of A and C (off a
//               multiple of 128); B of group g is the g-th block of B along
//               its N (K-major B: N rows each) or K (MN-major B: K rows each)
//               dimension.  Used for dA = dY W^_down and
//               dX = [dG | dU] [W^_gate; W^_up].
//   K-segments  group g reduces over K indices [off[g], off[g] + len[g]) of A
//               and B (the group's tokens; off a multiple of 64, padding
//               holds zeros); C of group g is rows [g M, (g+1) M).  Used for
//               the weight gradients dW = dY^T A^.
// Persistent CTAs (one per SM), 128 x 256 tiles, 3-stage TMA ring (128-byte
// swizzle), two accumulators in tensor memory so that the epilogue of one
// tile overlaps the MMAs of the next, 8 epilogue warps that stage their
// 32 x 128 part of the tile in shared memory and write it with TMA stores
// (full 128-byte lines), every wait bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "ptx.cuh"

namespace nvfp4 {

namespace bf16gemm {

constexpr int BM = 128, BN = 256;
constexpr int BK = 64;                    // K per stage: 64 bf16 = 128 bytes
constexpr int KB = BK / 16;               // MMAs (K = 16) per stage
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB
constexpr int B_BYTES = BN * BK * 2;      // 32 KiB
constexpr int MN_ATOM_BYTES = BK * 128;   // MN-major: one 64-wide column block of a stage
constexpr int MAX_GROUPS = 256;
constexpr int EPI_WARPS = 8;
constexpr int STAGE_OUT_BYTES = 32 * 64 * 2;            // one TMA store box: 32 rows x 64 bf16
constexpr int OUT_BYTES = EPI_WARPS * 2 * STAGE_OUT_BYTES; // two boxes per epilogue warp
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + OUT_BYTES + 1024 + 256 + (2 * MAX_GROUPS + 1) * 4;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int ACC_COLS = BN;              // FP32 accumulator columns per tile
constexpr int TM_COLS = 2 * ACC_COLS;     // two accumulators

// BF16 x BF16 -> F32: c_format 1 (bits 4-5), a/b format 1 (bits 7-9, 10-12),
// A / B MN-major flags (bits 15, 16), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
template <bool A_MN, bool B_MN>
constexpr uint32_t idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((A_MN ? 1u : 0u) << 15) | ((B_MN ? 1u : 0u) << 16) |
         ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

struct Params {
  __nv_bfloat16* c;
  int64_t ldc;
  int M, N, K;            // M: rows of C per group (K-segments); K: reduction length (M-segments)
  int mode;               // 0 = M-segments, 1 = K-segments
  int groups;
  const int32_t* off;     // device [groups + 1]
  const int32_t* len;     // device [groups]
  int c_vec16;
  int c_tma;              // write C through the 3-D tensor map (N, rows per group, groups)
};

struct Tile {
  int g, m0, n0;
  int a_mn, a_k, b_mn, b_k;   // operand coordinates of the first stage (MN index, K index)
  int c_row0, row_end;
  int nk;                     // K stages
  bool empty;
};

template <bool B_MN>
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
    tl.a_mn = tl.m0;
    tl.a_k = 0;
    tl.b_mn = B_MN ? tl.n0 : lo * p.N + tl.n0;
    tl.b_k = B_MN ? lo * p.K : 0;
    tl.c_row0 = 0;
    tl.row_end = s_off[lo] + s_len[lo];
    tl.nk = (p.K + BK - 1) / BK;
    tl.empty = tl.m0 >= tl.row_end;
  } else {
    const int per_g = num_m * num_n;
    const int g = t / per_g;
    const int r = t - g * per_g;
    const int mt = r / num_n;
    tl.g = g;
    tl.m0 = mt * BM;
    tl.n0 = (r - mt * num_n) * BN;
    tl.a_mn = tl.m0;
    tl.b_mn = tl.n0;
    tl.a_k = tl.b_k = s_off[g];
    tl.c_row0 = g * p.M;
    tl.row_end = p.M;
    tl.nk = (s_len[g] + BK - 1) / BK;
    tl.empty = false;  // an empty segment still writes its zero gradient
  }
  return tl;
}

// One stage of one operand: ROWS (M or N) x 64 (K) elements into `dst`.
template <bool MN, int ROWS>
NVFP4_DEV void load_operand(uint8_t* dst, const CUtensorMap* map, int mn, int k, uint64_t* bar) {
  if (MN) {
#pragma unroll
    for (int j = 0; j < ROWS / 64; ++j) tma_load_2d(dst + j * MN_ATOM_BYTES, map, mn + 64 * j, k, bar);
  } else {
    tma_load_2d(dst, map, k, mn, bar);
  }
}

// Shared-memory descriptor of K step kb (16 elements) of one operand stage.
//   K-major:  rows of 128 bytes (8-row swizzle atoms, 1024 bytes apart); the
//             K step moves 32 bytes along the swizzled row.
//   MN-major: 64-wide column blocks of BK rows x 128 bytes (MN_ATOM_BYTES
//             apart: the leading-dimension offset); 8-row atoms 1024 bytes
//             apart along K (the stride offset); the K step moves 16 rows.
template <bool MN>
NVFP4_DEV uint64_t operand_desc(uint32_t base, int kb) {
  return MN ? smem_desc(base + kb * 16 * 128, MN_ATOM_BYTES, 1024, 2) : smem_desc(base + kb * 32, 16, 1024, 2);
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sOut = sB + STAGES * B_BYTES;   // 1024-byte aligned: 128-byte swizzle of the store boxes
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + OUT_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  int32_t* s_off = reinterpret_cast<int32_t*>(smem + STAGES * (A_BYTES + B_BYTES) + OUT_BYTES + 256);
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p.c_tma) tma_prefetch_desc(&tmC);
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
        const Tile tl = tile_of<B_MN>(t, p, s_off, s_len, num_n, num_m);
        if (tl.empty) continue;
        for (int kt = 0; kt < tl.nk; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          mbar_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES));
          load_operand<A_MN, BM>(sA + s * A_BYTES, &tmA, tl.a_mn, tl.a_k + kt * BK, &full[s]);
          load_operand<B_MN, BN>(sB + s * B_BYTES, &tmB, tl.b_mn, tl.b_k + kt * BK, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, ti = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const Tile tl = tile_of<B_MN>(t, p, s_off, s_len, num_n, num_m);
        if (tl.empty) continue;
        const int buf = ti & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ((uint32_t)(ti >> 1) & 1u) ^ 1u)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * ACC_COLS);
        for (int kt = 0; kt < tl.nk; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&full[s], ph)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * B_BYTES);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            mma_bf16(acc, operand_desc<A_MN>(a_base, kb), operand_desc<B_MN>(b_base, kb), idesc<A_MN, B_MN>(),
                     (kt > 0 || kb > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[buf]);
        ++ti;
      }
    }
  } else {
    const int sub = warp & 3;                      // TMEM lanes 32 sub .. 32 sub + 31
    const int cbase = ((warp - 2) >> 2) * (BN / 2);
    constexpr int HALF = BN / 2;
    int ti = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const Tile tl = tile_of<B_MN>(t, p, s_off, s_len, num_n, num_m);
      if (tl.empty) continue;
      const int buf = ti & 1;
      const bool ok = mbar_wait_bounded(&acc_full[buf], (uint32_t)(ti >> 1) & 1u);
      ++ti;
      if (!ok) *abort_flag = 1;
      if (!ok || *abort_flag) break;
      tc_fence_after();
      uint32_t packed[HALF / 2];
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 64) {
        uint32_t r0[32], r1[32];
        const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + (uint32_t)(buf * ACC_COLS) + cbase + c0;
        tmem_ld_32x32b_x32(taddr, r0);
        tmem_ld_32x32b_x32(taddr + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          // a K-segment of length 0 issued no MMA: its gradient is zero
          const bool z = tl.nk == 0;
          packed[c0 / 2 + j] = z ? 0u : pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
          packed[c0 / 2 + 16 + j] = z ? 0u : pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (p.c_tma) {
        // stage rows sub*32 .. +31, columns cbase .. cbase+127 as two 32 x 64
        // boxes (row `lane` at 128 bytes per row, 16-byte chunk j at j ^ (row % 8))
        uint8_t* st = sOut + (warp - 2) * 2 * STAGE_OUT_BYTES;
        if (lane == 0) bulk_wait_group_read0();  // the previous tile's boxes have been read
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* v = packed + q * 32 + 4 * j;
            st_shared_v4(st + q * STAGE_OUT_BYTES + lane * 128 + ((j ^ (lane & 7)) << 4), v[0], v[1], v[2], v[3]);
          }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int y = tl.m0 + sub * 32, z = p.mode == 0 ? 0 : tl.g;
          tma_store_3d(&tmC, st, tl.n0 + cbase, y, z);
          tma_store_3d(&tmC, st + STAGE_OUT_BYTES, tl.n0 + cbase + 64, y, z);
          bulk_commit_group();
        }
        continue;
      }
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
    if (p.c_tma && lane == 0) bulk_wait_group0();  // stores complete before the CTA's memory goes away
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
// box of box_rows x 64 columns (128 bytes), 128-byte swizzle, zero fill.
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

// C as a 3-D tensor (N, rows per group, groups), box 64 x 32 x 1, 128-byte
// swizzle: a store never crosses into the next group's rows.
static bool tmap_c(CUtensorMap* m, void* base, int64_t n, int64_t rows, int64_t groups, int64_t ldc) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)n, (cuuint64_t)rows, (cuuint64_t)groups};
  cuuint64_t strides[2] = {(cuuint64_t)(ldc * 2), (cuuint64_t)(ldc * 2 * rows)};
  cuuint32_t box[3] = {64u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool A_MN, bool B_MN>
static nvfp4_status launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const Params& p,
                           cudaStream_t s) {
  // the attribute is per device: set it on every call (cheap)
  if (cudaFuncSetAttribute(gemm_bf16_kernel<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  gemm_bf16_kernel<A_MN, B_MN><<<sms, THREADS, SMEM_BYTES, s>>>(ta, tb, tc, p);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // namespace bf16gemm
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_gemm_bf16_grouped(int mode, int groups, const void* a, int a_mn_major, int64_t a_rows,
                                                int64_t a_cols, int64_t lda, const void* b, int b_mn_major,
                                                int64_t b_rows, int64_t b_cols, int64_t ldb, const int32_t* seg_off,
                                                const int32_t* seg_len, int64_t M, int64_t N, int64_t K, void* c,
                                                int64_t ldc, void* stream) {
  NVFP4_ENTRY("nvfp4_gemm_bf16_grouped");
  using namespace bf16gemm;
  if (mode != 0 && mode != 1) return NVFP4_ERR_ARG;
  if ((a_mn_major != 0 && a_mn_major != 1) || (b_mn_major != 0 && b_mn_major != 1)) return NVFP4_ERR_ARG;
  if (groups < 1 || groups > MAX_GROUPS) return NVFP4_ERR_SHAPE;
  if (!a || !b || !seg_off || !seg_len || !c) return NVFP4_ERR_ARG;
  if (a_rows < 1 || a_cols < 1 || b_rows < 1 || b_cols < 1 || lda < a_cols || ldb < b_cols || N < 1 || ldc < N)
    return NVFP4_ERR_SHAPE;
  if (a_rows > 0x7FFFFFFF || a_cols > 0x7FFFFFFF || b_rows > 0x7FFFFFFF || b_cols > 0x7FFFFFFF)
    return NVFP4_ERR_SHAPE;
  // stored extents: K-major operands are (rows = M or N index, cols = K), MN-major (rows = K, cols = M or N)
  const int64_t a_m = a_mn_major ? a_cols : a_rows, a_k = a_mn_major ? a_rows : a_cols;
  const int64_t b_n = b_mn_major ? b_cols : b_rows, b_k = b_mn_major ? b_rows : b_cols;
  if (mode == 0) {
    if (K < 64 || K % 64 != 0 || K > a_k || a_m % 128 != 0) return NVFP4_ERR_SHAPE;
    if (b_mn_major ? (b_k < (int64_t)groups * K || b_n < N) : (b_n < (int64_t)groups * N || b_k < K))
      return NVFP4_ERR_SHAPE;
    if ((int64_t)groups * K > 0x7FFFFFFF || (int64_t)groups * N > 0x7FFFFFFF) return NVFP4_ERR_SHAPE;
  } else {
    if (M < 1 || M > a_m || N > b_n || a_k != b_k) return NVFP4_ERR_SHAPE;
    if ((int64_t)groups * M > 0x7FFFFFFF) return NVFP4_ERR_SHAPE;
  }
  if (((uintptr_t)a & 15u) || ((uintptr_t)b & 15u) || (lda * 2) % 16 || (ldb * 2) % 16 || ((uintptr_t)c & 3u))
    return NVFP4_ERR_ALIGN;
  CUtensorMap ta, tb;
  if (!tmap_bf16(&ta, a, a_rows, a_cols, lda, a_mn_major ? BK : BM) ||
      !tmap_bf16(&tb, b, b_rows, b_cols, ldb, b_mn_major ? BK : BN))
    return NVFP4_ERR_CUDA;
  Params p;
  p.c = reinterpret_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.M = (int)(mode == 0 ? a_m : M);
  p.N = (int)N;
  p.K = (int)K;
  p.mode = mode;
  p.groups = groups;
  p.off = seg_off;
  p.len = seg_len;
  p.c_vec16 = (((uintptr_t)c & 15u) == 0 && (ldc % 8) == 0) ? 1 : 0;
  // TMA stores need a 16-byte aligned C; in M-segment mode they also write
  // the padding rows of each segment's last 128-row tile
  CUtensorMap tc;
  memset(&tc, 0, sizeof(tc));
  p.c_tma = 0;
  if (p.c_vec16) {
    const bool ok = mode == 0 ? tmap_c(&tc, c, N, a_m, 1, ldc) : tmap_c(&tc, c, N, M, groups, ldc);
    p.c_tma = ok ? 1 : 0;
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (!a_mn_major && !b_mn_major) return launch<false, false>(ta, tb, tc, p, s);
  if (!a_mn_major && b_mn_major) return launch<false, true>(ta, tb, tc, p, s);
  if (a_mn_major && !b_mn_major) return launch<true, false>(ta, tb, tc, p, s);
  return launch<true, true>(ta, tb, tc, p, s);
}
