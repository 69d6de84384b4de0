// probe.cu -- dense FP4 tensor-core throughput probe for sm_100a.
//
// The W4A4 GEMM is reported as a fraction of the dense FP4 peak.  The
// datasheet gives a figure; this probe measures what the block-scaled FP4
// MMA sustains on this device: every CTA (one per SM) keeps one 128 x 256
// stage of E2M1 operands (128-byte swizzled, K = 256) and its UE4M3 scales
// resident and issues tcgen05.mma.kind::mxf4nvf4.block_scale back to back
// into a 128 x 256 FP32 accumulator in tensor memory -- the instruction and
// tile shape of the GEMM, without the operand traffic.  The host times the
// launch with CUDA events; flop = 2 * 128 * 256 * 64 per MMA.
#include "ptx.cuh"

namespace nvfp4 {

namespace probe {

constexpr int BM = 128, BN = 256;
constexpr int KB = 4;                 // MMAs (K = 64) per 256-element stage
constexpr int A_BYTES = BM * 128;     // 128 bytes (256 E2M1) per row
constexpr int B_BYTES = BN * 128;
constexpr int THREADS = 128;          // four warps: one per TMEM lane quadrant
// Dynamic shared memory is sized so that no two probe CTAs share an SM (each
// allocates all 512 tensor-memory columns).
constexpr int SMEM_BYTES = 120 * 1024;
constexpr int TM_COLS = 512;
constexpr int TM_SFA = BN;            // 4 * KB columns
constexpr int TM_SFB = BN + 4 * KB;   // 8 * KB columns
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__global__ void __launch_bounds__(THREADS, 1) fp4_mma_probe_kernel(int64_t iters) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + A_BYTES;
  __shared__ uint64_t done;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;

  // operands: a fixed pseudo-random byte pattern (a multiplicative hash of the
  // byte index), so the MMAs see mixed codes rather than zeros
  for (int i = threadIdx.x; i < (A_BYTES + B_BYTES) / 4; i += THREADS)
    reinterpret_cast<uint32_t*>(sA)[i] = (uint32_t)(i + 1) * 2654435761u;
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  fence_proxy_async_smem();  // the MMAs (async proxy) read what these threads wrote
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // every scale 1.0 (UE4M3 0x38), written by each warp into its lane quadrant
  const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
  const uint4 one = make_uint4(0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  for (int c = 0; c < 12 * KB; c += 4) tmem_st_32x32b_x4(lane_base + TM_SFA + c, one);
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (threadIdx.x == 0) {
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    for (int64_t it = 0; it < iters; ++it) {
#pragma unroll
      for (int kb = 0; kb < KB; ++kb)
        mma_fp4_block16(tmem, smem_desc(a_base + kb * 32, 16, 1024, 2), smem_desc(b_base + kb * 32, 16, 1024, 2),
                        IDESC, tmem + TM_SFA + kb * 4, tmem + TM_SFB + kb * 8, (it > 0 || kb > 0) ? 1u : 0u);
    }
    tc_commit(&done);
  }
  __syncwarp();
  if (warp == 0) (void)mbar_wait_bounded(&done, 0);  // the MMAs have completed (bounded)
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

}  // namespace probe
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status nvfp4_probe_fp4_mma(int64_t iters, int ctas, double* flop_per_launch, void* stream) {
  NVFP4_ENTRY("nvfp4_probe_fp4_mma");
  if (iters < 1 || iters > ((int64_t)1 << 40) || ctas < 1 || ctas > 4096) return NVFP4_ERR_ARG;
  // the attribute is per device: set it on every call (cheap)
  if (cudaFuncSetAttribute(probe::fp4_mma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, probe::SMEM_BYTES) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  probe::fp4_mma_probe_kernel<<<ctas, probe::THREADS, probe::SMEM_BYTES, (cudaStream_t)stream>>>(iters);
  count_launches(1);
  if (flop_per_launch)
    *flop_per_launch = 2.0 * probe::BM * probe::BN * 64.0 * probe::KB * (double)iters * (double)ctas;
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// ------------------------------------------------------------------ bounded-wait self-test
//
// Every wait of this library's kernels (on an mbarrier, a TMA transaction, a
// peer) is bounded: when it expires the kernel sets the device error word
// and returns instead of hanging.  This kernel exercises exactly that path:
// one thread waits on an mbarrier that nothing arrives at, with a caller-given
// cycle limit, then reports the expiry the way every other wait does.
namespace nvfp4 {
__global__ void timeout_selftest_kernel(long long limit_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    while (!mbar_try_wait(&bar, 0)) {
      if (clock64() - t0 > limit_cycles) {
        report_error(kErrWaitTimeout);
        break;
      }
    }
  }
}
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_selftest_timeout(int64_t limit_cycles, void* stream) {
  NVFP4_ENTRY("nvfp4_selftest_timeout");
  if (limit_cycles < 1 || limit_cycles > (1ll << 32)) return NVFP4_ERR_ARG;
  nvfp4::timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((long long)limit_cycles);
  nvfp4::count_launches(1);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
