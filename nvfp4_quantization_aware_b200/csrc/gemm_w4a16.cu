// gemm_w4a16.cu -- weight-only NVFP4 GEMM (W4A16) on the sm_100a tensor cores.
//
// W4A16 keeps the activations in bf16 and only the weights in NVFP4 (the
// Nemotron 3.5 Lightning checkpoint's format).  The Qwen3.6-35B-A3B W4A4
// tutorial (section "为什么目标是 W4A4 而不是 W4A16") contrasts it with W4A4:
// a W4A16 kernel turns the 4-bit weights back into 16-bit values inside its
// main loop and runs a 16-bit MMA, so the FP4 tensor cores stay unused.
//   C = A * W^T,  A bf16 [M][K],  W^ = bf16(value(q) * (s_b * s_g)) [N][K]
// i.e. the bf16 fake-quant weights (the dequantization of nvfp4_dequantize),
// FP32 accumulation, bf16 output.
//
// Persistent CTAs, 128 x 256 tiles, K = 64 per stage, 3 stages.  Warp roles:
//   0      TMA of the A tile (128-byte swizzle)
//   1      tcgen05.mma.kind::f16 issue (one thread), two TMEM accumulators
//   2-9    epilogue (TMA stores through swizzled shared-memory boxes)
//   10-13  dequantizers: per stage they load the 256 x 64 block of FP4 codes
//          and its 256 x 4 block scales from global memory and write the
//          bf16 tile into shared memory in the layout a 128-byte-swizzled
//          TMA load would produce, then arrive on the stage's barrier.
// A stage is full once the A bytes have landed and the four dequantizer
// warps have arrived.  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "ptx.cuh"
#include "quant_common.cuh"

namespace nvfp4 {

namespace w4a16 {

constexpr int BM = 128, BN = 256;
constexpr int BK = 64;
constexpr int KB = BK / 16;
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB
constexpr int B_BYTES = BN * BK * 2;      // 32 KiB
constexpr int EPI_WARPS = 8;
constexpr int DQ_WARPS = 4;
constexpr int THREADS = 64 + 32 * EPI_WARPS + 32 * DQ_WARPS;
constexpr int STAGE_OUT_BYTES = 32 * 64 * 2;
constexpr int OUT_BYTES = EPI_WARPS * 2 * STAGE_OUT_BYTES;
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + OUT_BYTES + 1024 + 256;
constexpr int ACC_COLS = BN;
constexpr int TM_COLS = 2 * ACC_COLS;
// BF16 x BF16 -> F32, K-major A and B, N >> 3, M >> 4
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct Params {
  const uint8_t* b_codes;   // N x K/2
  const uint8_t* b_scales;  // N x K/16, ROWMAJOR
  const float* b_ts;
  __nv_bfloat16* c;
  int64_t ldc;
  int M, N, K;
  int c_vec16, c_tma;
};

// The raw NVFP4 data of the two weight rows (d and d + 128 of the tile) that
// dequantizer thread d turns into bf16 for one stage: 64 codes (8 words,
// low nibble = even element) and the 4 block scales of each row.  Rows past
// N read as code 0 with scale 0, which dequantize to +0.
struct RawRows {
  uint32_t w[2][8];
  uint32_t sw[2];
};

NVFP4_DEV void load_raw(const Params& p, int n0, int kt, int d, RawRows& r) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int n = n0 + d + 128 * h;
    if (n < p.N) {
      const uint8_t* crow = p.b_codes + (int64_t)n * (p.K / 2) + kt * (BK / 2);
      const uint4 c0 = ld_stream_v4(crow), c1 = ld_stream_v4(crow + 16);
      r.w[h][0] = c0.x; r.w[h][1] = c0.y; r.w[h][2] = c0.z; r.w[h][3] = c0.w;
      r.w[h][4] = c1.x; r.w[h][5] = c1.y; r.w[h][6] = c1.z; r.w[h][7] = c1.w;
      r.sw[h] = __ldg(reinterpret_cast<const uint32_t*>(p.b_scales + (int64_t)n * (p.K / 16) + kt * (BK / 16)));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) r.w[h][j] = 0u;
      r.sw[h] = 0u;
    }
  }
}

// Dequantize the two rows and write them into the stage's B tile, laid out as
// a 128-byte-swizzled TMA load of a 256 x 64 bf16 box would: row r occupies
// bytes [128 r, 128 r + 128), its 16-byte chunk j (elements 8j .. 8j+7) at
// chunk position j ^ (r % 8).  Each value is value(q) * (s_b * s_g), two
// binary32 multiplies rounded once each, then rounded to bf16.
NVFP4_DEV void store_rows(const RawRows& raw, uint8_t* sB, int d, float sg) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = d + 128 * h;
    uint8_t* row = sB + r * 128;
#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      const float dd = __fmul_rn(e4m3_decode((raw.sw[h] >> (8 * blk)) & 0xFFu), sg);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j = 2 * blk + half;
        const uint32_t word = raw.w[h][j];
        uint32_t o[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          float v0, v1;
          e2m1x2_decode((word >> (8 * b)) & 0xFFu, v0, v1);
          o[b] = pack_bf16x2(__fmul_rn(v0, dd), __fmul_rn(v1, dd));
        }
        st_shared_v4(row + ((j ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
      }
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmC, Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sOut = sB + STAGES * B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + OUT_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + DQ_WARPS);  // producer arrive (with the A bytes) + each dequantizer warp
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
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
  const int num_m = (p.M + BM - 1) / BM;
  const int num_tiles = num_m * num_n;
  const int nk = p.K / BK;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const int m0 = (t / num_n) * BM;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          mbar_expect_tx(&full[s], (uint32_t)A_BYTES);
          tma_load_2d(sA + s * A_BYTES, &tmA, kt * BK, m0, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int it = 0, ti = 0;
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const int buf = ti & 1;
        if (!mbar_wait_bounded(&acc_empty[buf], ((uint32_t)(ti >> 1) & 1u) ^ 1u)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(buf * ACC_COLS);
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_bounded(&full[s], ph)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * B_BYTES);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
            mma_bf16(acc, smem_desc(a_base + kb * 32, 16, 1024, 2), smem_desc(b_base + kb * 32, 16, 1024, 2), IDESC,
                     (kt > 0 || kb > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[buf]);
        ++ti;
      }
    }
  } else if (warp >= 2 + EPI_WARPS) {
    // ------------------------------------------------------------ dequantizers
    const int d = threadIdx.x - 32 * (2 + EPI_WARPS);  // 0..127
    const float sg = __ldg(p.b_ts);
    // The next stage's codes are loaded before waiting for the current
    // stage's buffer, so their latency overlaps the conversion.
    RawRows cur, nxt;
    int t = blockIdx.x, kt = 0, it = 0;
    if (t < num_tiles) load_raw(p, (t % num_n) * BN, 0, d, cur);
    while (t < num_tiles && !*abort_flag) {
      int t2 = t, kt2 = kt + 1;
      if (kt2 == nk) {
        kt2 = 0;
        t2 += gridDim.x;
      }
      if (t2 < num_tiles) load_raw(p, (t2 % num_n) * BN, kt2, d, nxt);
      const int s = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], ph ^ 1u));  // warp-uniform exit
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      store_rows(cur, sB + s * B_BYTES, d, sg);
      fence_proxy_async_smem();  // the tensor core (async proxy) reads what these threads wrote
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
      cur = nxt;
      t = t2;
      kt = kt2;
      ++it;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;
    const int cbase = ((warp - 2) >> 2) * (BN / 2);
    constexpr int HALF = BN / 2;
    int ti = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int m0 = (t / num_n) * BM, n0 = (t % num_n) * BN;
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
          packed[c0 / 2 + j] = pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
          packed[c0 / 2 + 16 + j] = pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (p.c_tma) {
        uint8_t* st = sOut + (warp - 2) * 2 * STAGE_OUT_BYTES;
        if (lane == 0) bulk_wait_group_read0();
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
          tma_store_3d(&tmC, st, n0 + cbase, m0 + sub * 32, 0);
          tma_store_3d(&tmC, st + STAGE_OUT_BYTES, n0 + cbase + 64, m0 + sub * 32, 0);
          bulk_commit_group();
        }
        continue;
      }
      const int row = m0 + sub * 32 + lane;
      if (row < p.M) {
        __nv_bfloat16* crow = p.c + (int64_t)row * p.ldc;
#pragma unroll
        for (int c0 = 0; c0 < HALF; c0 += 32) {
          const int col0 = n0 + cbase + c0;
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
                crow[col0 + j] = __ushort_as_bfloat16((unsigned short)((j & 1) ? (w >> 16) : (w & 0xFFFFu)));
              }
            }
          }
        }
      }
    }
    if (p.c_tma && lane == 0) bulk_wait_group0();
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

}  // namespace w4a16
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_gemm_w4a16(const void* a, int64_t lda, const uint8_t* b_codes, const uint8_t* b_scales,
                                         const float* b_tensor_scale, int64_t M, int64_t N, int64_t K, void* c,
                                         int64_t ldc, void* stream) {
  using namespace w4a16;
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0 || lda < K || ldc < N) return NVFP4_ERR_SHAPE;
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return NVFP4_ERR_SHAPE;
  if (!a || !b_codes || !b_scales || !b_tensor_scale || !c) return NVFP4_ERR_ARG;
  if (((uintptr_t)a & 15u) || (lda * 2) % 16 || ((uintptr_t)b_codes & 15u) || ((uintptr_t)b_scales & 3u) ||
      ((uintptr_t)c & 3u))
    return NVFP4_ERR_ALIGN;
  auto enc = encode_fn();
  if (!enc) return NVFP4_ERR_CUDA;
  CUtensorMap ta, tc;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(lda * 2)};
    cuuint32_t box[2] = {64u, (cuuint32_t)BM};
    cuuint32_t estr[2] = {1u, 1u};
    if (enc(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return NVFP4_ERR_CUDA;
  }
  Params p;
  p.b_codes = b_codes;
  p.b_scales = b_scales;
  p.b_ts = b_tensor_scale;
  p.c = reinterpret_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.c_vec16 = (((uintptr_t)c & 15u) == 0 && (ldc % 8) == 0) ? 1 : 0;
  p.c_tma = 0;
  memset(&tc, 0, sizeof(tc));
  if (p.c_vec16) {
    cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, 1};
    cuuint64_t strides[2] = {(cuuint64_t)(ldc * 2), (cuuint64_t)(ldc * 2 * M)};
    cuuint32_t box[3] = {64u, 32u, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    p.c_tma = enc(&tc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, c, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(gemm_w4a16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
      return NVFP4_ERR_CUDA;
    attr = true;
  }
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = (int)(((M + BM - 1) / BM) * ((N + BN - 1) / BN));
  gemm_w4a16_kernel<<<tiles < sms ? tiles : sms, THREADS, SMEM_BYTES, (cudaStream_t)stream>>>(ta, tc, p);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
