// gemm_w4a16.cu -- weight-only NVFP4 GEMM (W4A16) on the sm_100a tensor cores.
//
// W4A16 keeps the activations in bf16 and only the weights in NVFP4 (the
// Nemotron 3.5 Lightning checkpoint's format).  The Qwen3.6-35B-A3B W4A4
// tutorial (section "为什么目标是 W4A4 而不是 W4A16") contrasts it with W4A4:
// a W4A16 kernel turns the 4-bit weights back into 16-bit values inside its
// main loop and runs a 16-bit MMA, so the FP4 tensor cores stay unused.
//   C = A * W^T,  A bf16 [M][K],  W^ = bf16(value(q) * (s_b * s_g)) [N][K]
// i.e. the bf16 fake-quant weights, FP32 accumulation, bf16 output.
//
// Persistent CTAs, 256 x 128 tiles (two M = 128 MMAs share each dequantized
// B tile, which halves the dequantization per FLOP against 128-row tiles),
// K = 64 per stage, 3 stages.  Warp roles:
//   0      TMA of the A tile (128-byte swizzle)
//   1      tcgen05.mma.kind::f16 issue (one thread), two TMEM accumulators
//   2-5    epilogue: 64-column chunks through double-buffered swizzled
//          shared-memory boxes and TMA stores
//   6-13   dequantizers, two threads per weight row of the tile (half a row,
//          two blocks, each).  Each thread copies its 16 code bytes and its
//          row's 4 block-scale bytes of a stage into a private 4-deep
//          shared-memory ring with cp.async, several stages ahead, then
//          writes its bf16 half row into the B tile in the layout a
//          128-byte-swizzled TMA load would produce.
// A stage is full once the A bytes have landed and the eight dequantizer
// warps have arrived.  Every wait is bounded.
//
// Dequantization by table lookup.  Within a block all 16 values are
// value(q) * d with d = s_b * s_g and |value(q)| one of 8 magnitudes, so the
// 8 products are formed once per block (binary32 multiply, bf16 rounding,
// the two rounding steps of the fake quantizer) and split into a table of
// their low bytes and one of their high bytes, 8 bytes each.  Each 4-bit code
// then costs byte permutes only: its low 3 bits select the two bytes, its
// sign bit becomes bit 15 of the bf16 (-0 for the negative zero code, as
// value(q) * d gives).  This keeps the per-element work on the integer ALU;
// the conversions (E2M1 -> f16 -> f32 -> bf16 per element) run at a fraction
// of that rate.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "ptx.cuh"
#include "quant_common.cuh"

namespace nvfp4 {

namespace w4a16 {

constexpr int BM = 256, BN = 128;
constexpr int MMA_M = 128;
constexpr int BK = 64;
constexpr int KB = BK / 16;
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;      // 32 KiB
constexpr int B_BYTES = BN * BK * 2;      // 16 KiB
constexpr int EPI_WARPS = 4;
constexpr int DQ_WARPS = 8;
constexpr int DQ_THREADS = 32 * DQ_WARPS;  // == 2 BN: two threads per weight row
constexpr int DQ_FIRST = 64 + 32 * EPI_WARPS;
constexpr int THREADS = DQ_FIRST + DQ_THREADS;
constexpr int RAW_DEPTH = 4;
constexpr int RAW_SLOT = DQ_THREADS * 20;  // 16 code bytes per thread, then the row's 4 scale bytes per thread
constexpr int BOX_BYTES = 32 * 64 * 2;      // one 32-row x 64-column bf16 store box
constexpr int OUT_BYTES = EPI_WARPS * 2 * BOX_BYTES;
constexpr int SMEM_BYTES = STAGES * (A_BYTES + B_BYTES) + RAW_DEPTH * RAW_SLOT + OUT_BYTES + 1024 + 256;
constexpr int ACC_COLS = 2 * BN;  // the two M halves side by side
constexpr int TM_COLS = 2 * ACC_COLS;
// BF16 x BF16 -> F32, K-major A and B, N >> 3, M >> 4
constexpr uint32_t IDESC =
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(MMA_M >> 4) << 24);
static_assert(DQ_THREADS == 2 * BN, "two dequantizer threads per weight row of the tile");
static_assert(BM == 2 * MMA_M, "two MMAs per K step");

struct Params {
  const uint8_t* b_codes;   // N x K/2
  const uint8_t* b_scales;  // N x K/16, ROWMAJOR
  const float* b_ts;
  __nv_bfloat16* c;
  int64_t ldc;
  int M, N, K;
  int c_vec16, c_tma;
};

// Byte tables of one block: the bf16 values of the 8 magnitudes
// {0, 0.5, 1, 1.5, 2, 3, 4, 6} * d, low bytes in lo[0..1], high bytes in hi[0..1].
struct BlockTable {
  uint32_t lo0, lo1, hi0, hi1;
};

NVFP4_DEV BlockTable block_table(float d) {
  const uint32_t w0 = pack_bf16x2(__fmul_rn(0.0f, d), __fmul_rn(0.5f, d));
  const uint32_t w1 = pack_bf16x2(__fmul_rn(1.0f, d), __fmul_rn(1.5f, d));
  const uint32_t w2 = pack_bf16x2(__fmul_rn(2.0f, d), __fmul_rn(3.0f, d));
  const uint32_t w3 = pack_bf16x2(__fmul_rn(4.0f, d), __fmul_rn(6.0f, d));
  BlockTable t;
  t.lo0 = prmt(w0, w1, 0x6420u);
  t.lo1 = prmt(w2, w3, 0x6420u);
  t.hi0 = prmt(w0, w1, 0x7531u);
  t.hi1 = prmt(w2, w3, 0x7531u);
  return t;
}

// Eight codes (one word, element 0 in the low nibble) -> four bf16x2 words.
NVFP4_DEV void decode8(uint32_t cw, const BlockTable& t, uint32_t (&o)[4]) {
  const uint32_t mag = cw & 0x77777777u;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t m = mag >> (16 * h), raw = cw >> (16 * h);
    const uint32_t lo = prmt(t.lo0, t.lo1, m);
    // sign-replicating permute of 0x80 bytes: 0x80 for a positive code, 0xFF
    // for a negative one; its bit 6 moved to bit 7 is the code's sign
    const uint32_t sgn = prmt(0x80808080u, 0x80808080u, raw);
    const uint32_t hi = prmt(t.hi0, t.hi1, m) | ((sgn << 1) & 0x80808080u);
    o[2 * h] = prmt(lo, hi, 0x5140u);
    o[2 * h + 1] = prmt(lo, hi, 0x7362u);
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmC, Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sRaw = sB + STAGES * B_BYTES;
  uint8_t* sOut = sRaw + RAW_DEPTH * RAW_SLOT;
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
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t bd = smem_desc(b_base + kb * 32, 16, 1024, 2);
            const uint32_t accum = (kt > 0 || kb > 0) ? 1u : 0u;
            mma_bf16(acc, smem_desc(a_base + kb * 32, 16, 1024, 2), bd, IDESC, accum);
            mma_bf16(acc + BN, smem_desc(a_base + MMA_M * 128 + kb * 32, 16, 1024, 2), bd, IDESC, accum);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[buf]);
        ++ti;
      }
    }
  } else if (warp >= DQ_FIRST / 32) {
    // ------------------------------------------------------------ dequantizers
    const int d = threadIdx.x - DQ_FIRST;
    const int r = d % BN, part = d / BN;  // weight row of the tile; elements 32 part .. 32 part + 31
    const float sg = __ldg(p.b_ts);
    const int64_t code_ld = p.K / 2, scale_ld = p.K / 16;
    const int my_tiles = (int)blockIdx.x < num_tiles ? (num_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int items = my_tiles * nk;  // (tile, k-stage) pairs in the order the other roles take them
    // copy item i's raw data into ring slot i % RAW_DEPTH (rows past N: zeros, nothing read)
    auto issue = [&](int i) {
      const int t = (int)blockIdx.x + (i / nk) * (int)gridDim.x, kt = i % nk;
      const int n = (t % num_n) * BN + r;
      const bool in = n < p.N;
      const int64_t nn = in ? n : 0;
      uint8_t* slot = sRaw + (i % RAW_DEPTH) * RAW_SLOT;
      cp_async_16(slot + d * 16, p.b_codes + nn * code_ld + kt * (BK / 2) + part * 16, in ? 16u : 0u);
      cp_async_4(slot + DQ_THREADS * 16 + d * 4, p.b_scales + nn * scale_ld + kt * (BK / 16), in ? 4u : 0u);
    };
#pragma unroll
    for (int i = 0; i < RAW_DEPTH - 1; ++i) {
      if (i < items) issue(i);
      cp_async_commit();
    }
    for (int i = 0; i < items; ++i) {
      if (__any_sync(0xFFFFFFFFu, *abort_flag != 0)) break;
      if (i + RAW_DEPTH - 1 < items) issue(i + RAW_DEPTH - 1);
      cp_async_commit();
      cp_async_wait<RAW_DEPTH - 1>();  // item i's copies (this thread's own) have landed
      const uint8_t* slot = sRaw + (i % RAW_DEPTH) * RAW_SLOT;
      const uint4 c4 = *reinterpret_cast<const uint4*>(slot + d * 16);
      const uint32_t sw = *reinterpret_cast<const uint32_t*>(slot + DQ_THREADS * 16 + d * 4) >> (16 * part);
      const int s = i % STAGES;
      const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
      const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&empty[s], ph ^ 1u));  // warp-uniform exit
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
      uint8_t* row = sB + s * B_BYTES + r * 128;
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        const BlockTable tab = block_table(__fmul_rn(e4m3_decode((sw >> (8 * blk)) & 0xFFu), sg));
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 4 * part + 2 * blk + h;  // 16-byte chunk: elements 8j .. 8j+7 of the row
          uint32_t o[4];
          decode8(cw[2 * blk + h], tab, o);
          st_shared_v4(row + ((j ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async_smem();  // the tensor core (async proxy) reads what these threads wrote
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
    }
    cp_async_wait<0>();  // no copy outlives the loop
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;  // TMEM lanes 32 sub .. 32 sub + 31
    uint8_t* st = sOut + (warp - 2) * 2 * BOX_BYTES;
    int ti = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const int m0 = (t / num_n) * BM, n0 = (t % num_n) * BN;
      const int buf = ti & 1;
      const bool ok = mbar_wait_bounded(&acc_full[buf], (uint32_t)(ti >> 1) & 1u);
      ++ti;
      if (!ok) *abort_flag = 1;
      if (!ok || *abort_flag) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < ACC_COLS / 64; ++c) {
        // chunk c: M half c / 2 (rows m0 + 128 (c / 2) ..), columns n0 + 64 (c % 2) ..
        const int orow = m0 + (c >> 1) * MMA_M + sub * 32, ocol = n0 + (c & 1) * 64;
        uint32_t r0[32], r1[32], packed[32];
        const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + (uint32_t)(buf * ACC_COLS) + c * 64;
        tmem_ld_32x32b_x32(taddr, r0);
        tmem_ld_32x32b_x32(taddr + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          packed[j] = pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
          packed[16 + j] = pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
        }
        if (c == ACC_COLS / 64 - 1) {  // the accumulator is free for the tile after next
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        if (p.c_tma) {
          uint8_t* box = st + (c & 1) * BOX_BYTES;
          if (lane == 0) bulk_wait_group_read1();  // the store that last used this box has read it
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(box + lane * 128 + ((j ^ (lane & 7)) << 4), packed[4 * j], packed[4 * j + 1],
                         packed[4 * j + 2], packed[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmC, box, ocol, orow, 0);
            bulk_commit_group();
          }
          continue;
        }
        const int row = orow + lane;
        if (row < p.M) {
          __nv_bfloat16* crow = p.c + (int64_t)row * p.ldc;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int col0 = ocol + 32 * h;
            if (col0 + 32 <= p.N && p.c_vec16) {
              uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(packed[16 * h + 4 * j], packed[16 * h + 4 * j + 1], packed[16 * h + 4 * j + 2],
                                    packed[16 * h + 4 * j + 3]);
            } else {
              for (int j = 0; j < 32; ++j) {
                if (col0 + j < p.N) {
                  const uint32_t w = packed[16 * h + (j >> 1)];
                  crow[col0 + j] = __ushort_as_bfloat16((unsigned short)((j & 1) ? (w >> 16) : (w & 0xFFFFu)));
                }
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

}  // namespace w4a16
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_gemm_w4a16(const void* a, int64_t lda, const uint8_t* b_codes, const uint8_t* b_scales,
                                         const float* b_tensor_scale, int64_t M, int64_t N, int64_t K, void* c,
                                         int64_t ldc, void* stream) {
  NVFP4_ENTRY("nvfp4_gemm_w4a16");
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
    cuuint32_t box[2] = {64u, (cuuint32_t)BM};  // both M halves in one load
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
  // the attribute is per device: set it on every call (cheap)
  if (cudaFuncSetAttribute(gemm_w4a16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = (int)(((M + BM - 1) / BM) * ((N + BN - 1) / BN));
  gemm_w4a16_kernel<<<tiles < sms ? tiles : sms, THREADS, SMEM_BYTES, (cudaStream_t)stream>>>(ta, tc, p);
  count_launches(1);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
