// gemm_w4a4.cu -- W4A4 block-scaled NVFP4 GEMM on the sm_100a tensor cores.
//
// W4A4 quantizes activations as well as weights, so the linear layer is an
// FP4 x FP4 product that runs on the Blackwell FP4 tensor cores (Qwen3.6-35B-A3B
// W4A4 NVFP4 tutorial page, "为什么目标是 W4A4" and "吞吐量"):
//   C[m, n] = (s_gA * s_gB) * sum_k (q_A[m,k] s_bA[m,k/16]) (q_B[n,k] s_bB[n,k/16])
// with E2M1 codes q, UE4M3 block scales s_b per 16 elements of K and FP32
// tensor scales s_g (Nemotron-3-Nano-30B NVFP4 article, "NVFP4-Format und warum
// es wichtig ist?").
//
// Persistent kernel: one CTA per SM walks the 128 x BN output tiles
// (t = blockIdx.x, blockIdx.x + gridDim.x, ...).  Warp roles:
//   warp 0      TMA producer: per K stage (256 elements) the A tile
//               (128 rows x 128 bytes) and B tile (BN rows x 128 bytes) as 2-D
//               tiled TMA loads with 128-byte swizzle, and the stage's block
//               scales as 1-D bulk copies (the MMA scale layout keeps each
//               128-row x 4-block tile contiguous).  No cluster multicast.
//   warp 1      allocates tensor memory, then one thread issues per stage
//               four tcgen05.mma.kind::mxf4nvf4.block_scale (K = 64 each) into
//               an FP32 accumulator in tensor memory; tcgen05.commit releases
//               the stage back to the producer.
//   warps 2-9   epilogue (two per TMEM subpartition, half the columns each):
//               tcgen05.ld of the accumulator, x (s_gA s_gB), bf16 rounding
//               into registers, release of the accumulator to the MMA warp
//               (acc_empty), then the global stores -- which overlap the next
//               tile's MMAs.  Ragged tiles store 32 columns at a time and
//               release at the end.
//   warps 10-13 scale writers, one per TMEM lane quadrant: per stage they
//               move the stage's block scales from shared memory into tensor
//               memory with tcgen05.st, in the layout the block-scaled MMA
//               reads, and arrive on sf_full[stage].  Doing this with
//               tcgen05.cp would put twelve copies per stage in order with
//               the MMAs on the tensor pipe, about a third of the run time.
// A STAGES-deep mbarrier ring between producer and MMA runs across tile
// boundaries, so the next tile's operands stream in while the epilogue drains.
// Tensor memory holds one 128 x BN FP32 accumulator (BN = 256 uses half of the
// 512 columns) plus one set of block scales per ring stage; every wait is
// bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cooperative_groups.h>

#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace nvfp4 {

// 32-byte global store of words w[i0 .. i0 + 7] (address 32-byte aligned).
template <int NW>
NVFP4_DEV void st_global_v8(void* p, const uint32_t (&w)[NW], int i0) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[i0]), "r"(w[i0 + 1]), "r"(w[i0 + 2]),
               "r"(w[i0 + 3]), "r"(w[i0 + 4]), "r"(w[i0 + 5]), "r"(w[i0 + 6]), "r"(w[i0 + 7])
               : "memory");
}

template <int BN_>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int BK = 256;                 // FP4 elements per stage (128 bytes per row)
  static constexpr int KB_PER_STAGE = BK / 64;   // MMAs (K = 64) per stage
  static constexpr int STAGES = 4;
  static constexpr int A_BYTES = BM * BK / 2;
  static constexpr int B_BYTES = BN * BK / 2;
  static constexpr int NB_SFB = BN / 128;        // 128-row scale tiles of B per stage
  static constexpr int SFA_BYTES = 512 * KB_PER_STAGE;
  static constexpr int SFB_BYTES = 512 * KB_PER_STAGE * NB_SFB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int MAX_GROUPS = 256;         // grouped problems: segment table in shared memory
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/ +
                                    (2 * MAX_GROUPS + 1) * 4 /*segment table*/;
  // tensor-memory columns: accumulator, then one set of scales per ring stage
  // (a set is rewritten only after the producer has seen its stage released,
  // i.e. after the MMAs that read it have completed)
  static constexpr int TM_ACC = 0;
  static constexpr int TM_SFA = BN;                                    // STAGES x 4*KB columns
  static constexpr int TM_SFB = BN + STAGES * 4 * KB_PER_STAGE;        // STAGES x 4*KB*NB_SFB columns
  static constexpr int TM_COLS_USED = TM_SFB + STAGES * 4 * KB_PER_STAGE * NB_SFB;
  static constexpr int TM_COLS = TM_COLS_USED <= 256 ? 256 : 512;
  static constexpr int EPI_WARPS = 8;            // two per TMEM subpartition, BN/2 columns each
  static constexpr int SF_WARPS = 4;             // scale writers, one per TMEM subpartition
  static constexpr int THREADS = 64 + 32 * EPI_WARPS + 32 * SF_WARPS;
  // instruction descriptor: E2M1 x E2M1 (format 1), UE4M3 scales, K-major A
  // and B, N >> 3 in bits 17-22, M >> 4 in bits 24-28, dense K = 64.
  static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
};

struct GemmParams {
  const uint8_t* a_sf;   // MMA layout
  const uint8_t* b_sf;
  const float* a_ts;
  const float* b_ts;
  __nv_bfloat16* c;
  int64_t ldc;
  int M, N, K;
  int kchunks;           // K / 64
  int b_rowtiles;        // ceil(N / 128): 128-row scale tiles present for B
  int c_vec16;           // C base 16-byte aligned and ldc % 8 == 0: 16-byte stores
  int c_vec32;           // C base 32-byte aligned and ldc % 16 == 0: 32-byte stores
  int c_vec8;            // C base 8-byte aligned and ldc % 4 == 0: 8-byte stores
  // Grouped problems (groups > 0): group g owns A rows [a_off[g], a_off[g] + a_rows[g]) with
  // a_off[g] a multiple of 128 (device arrays; a_off[groups] is the padded row total), B rows
  // [g * N, (g + 1) * N), tensor scales a_ts[g] and b_ts[g].
  int groups;
  const int32_t* a_off;
  const int32_t* a_rows;
};

// One output tile of the persistent schedule.
struct TileInfo {
  int m0, n0;     // first row of A / C and first column of C
  int b0;         // first row of B
  int g;          // group (0 for a dense problem)
  int row_end;    // rows of A at or beyond this are not part of the problem
  bool empty;     // no valid row (grouped: padding of a segment)
};

// Tile t of the persistent schedule; N fastest, so the CTAs that run at the
// same time share A rows and sweep B (both stay in L2).  For grouped problems
// the group is found by binary search over the segment table in shared memory.
NVFP4_DEV TileInfo tile_info(int t, int num_n, int BM, int BN, const GemmParams& p, const int32_t* s_off,
                             const int32_t* s_rows) {
  TileInfo ti;
  const int mt = t / num_n;
  ti.m0 = mt * BM;
  ti.n0 = (t - mt * num_n) * BN;
  if (p.groups == 0) {
    ti.g = 0;
    ti.b0 = ti.n0;
    ti.row_end = p.M;
    ti.empty = false;
    return ti;
  }
  int lo = 0, hi = p.groups - 1;  // last g with s_off[g] <= m0
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_off[mid] <= ti.m0) lo = mid;
    else hi = mid - 1;
  }
  ti.g = lo;
  ti.b0 = lo * p.N + ti.n0;
  ti.row_end = s_off[lo] + s_rows[lo];
  ti.empty = ti.m0 >= ti.row_end;
  return ti;
}

// Epilogue of one warp for one output tile: drain accumulator columns
// [cbase, cbase + BN/2) of the warp's 32 TMEM lanes (output row `row`),
// multiply by alpha = s_gA s_gB, round to bf16 and store columns
// n0 + cbase ... of the row.  `arrive` (called by every lane after the warp's
// last tcgen05.ld, behind a fence and a warp barrier) hands the accumulator
// back to the MMA issuer: a full-width tile is drained to registers first so
// that its stores overlap the next tile's MMAs; a ragged tile stores 32
// columns at a time and hands back at the end.
template <int BN, class Arrive>
NVFP4_DEV void epilogue_rows(uint32_t tbase, int row, int row_end, int n0, int cbase, const GemmParams& p, float alpha,
                             Arrive arrive) {
  constexpr int HALF = BN / 2;
  __nv_bfloat16* crow = p.c + (int64_t)row * p.ldc;
  if (p.c_vec16 && n0 + BN <= p.N) {
    uint32_t packed[HALF / 2];
#pragma unroll
    for (int c0 = 0; c0 < HALF; c0 += 16) {
      uint32_t r0[16];
      tmem_ld_32x32b_x16(tbase + c0, r0);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        packed[c0 / 2 + j] = pack_bf16x2(__uint_as_float(r0[2 * j]) * alpha, __uint_as_float(r0[2 * j + 1]) * alpha);
    }
    tc_fence_before();
    __syncwarp();
    arrive();
    if (row < row_end) {
      // 32-byte stores write whole L2 sectors and halve the store
      // instructions (the uncoalesced row-per-thread stores compete with
      // the operand traffic in the SM's L1 / shared-memory path)
      if (p.c_vec32) {
        uint8_t* dst = reinterpret_cast<uint8_t*>(crow + n0 + cbase);
#pragma unroll
        for (int j = 0; j < HALF / 16; ++j) st_global_v8(dst + 32 * j, packed, 8 * j);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(crow + n0 + cbase);
#pragma unroll
        for (int j = 0; j < HALF / 8; ++j)
          dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
      }
    }
  } else {
#pragma unroll
    for (int c0 = 0; c0 < HALF; c0 += 32) {
      uint32_t r0[32], packed[16];
      tmem_ld_32x32b_x32(tbase + c0, r0);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        packed[j] = pack_bf16x2(__uint_as_float(r0[2 * j]) * alpha, __uint_as_float(r0[2 * j + 1]) * alpha);
      const int col0 = n0 + cbase + c0;
      if (row < row_end && col0 < p.N) {
        if (col0 + 32 <= p.N && p.c_vec16) {
          uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        } else {
          const int rem = p.N - col0;
          unsigned short* dst = reinterpret_cast<unsigned short*>(crow + col0);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            if (2 * k < rem) dst[2 * k] = (unsigned short)(packed[k] & 0xFFFFu);
            if (2 * k + 1 < rem) dst[2 * k + 1] = (unsigned short)(packed[k] >> 16);
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    arrive();
  }
}

template <int BN>
__global__ void __launch_bounds__(GemmCfg<BN>::THREADS, 1)
    gemm_w4a4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::STAGES * C::A_BYTES;
  uint8_t* sSFA = sB + C::STAGES * C::B_BYTES;
  uint8_t* sSFB = sSFA + C::STAGES * C::SFA_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + C::STAGES * C::SFB_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // MMA -> epilogue: accumulator complete
  uint64_t* acc_empty = acc_full + 1;       // epilogue -> MMA: accumulator drained
  uint64_t* sf_full = acc_empty + 1;        // scale writers -> MMA: stage's scales in tensor memory
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(sf_full + C::STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_slot + 1);
  int32_t* s_off = reinterpret_cast<int32_t*>(smem + C::STAGES * C::STAGE_BYTES + 256);
  int32_t* s_rows = s_off + C::MAX_GROUPS + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_kt = (p.kchunks + C::KB_PER_STAGE - 1) / C::KB_PER_STAGE;
  const int num_n = (p.N + C::BN - 1) / C::BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], C::SF_WARPS);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, C::EPI_WARPS);  // one arrival per epilogue warp
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, C::TM_COLS);
    tmem_relinquish();
  }
  // the set-up above overlaps the previous kernel of the stream under a
  // programmatic dependent launch; global memory only after this point
  griddep_wait();
  for (int i = threadIdx.x; i < p.groups; i += blockDim.x) {
    s_off[i] = __ldg(p.a_off + i);
    s_rows[i] = __ldg(p.a_rows + i);
  }
  if (threadIdx.x == 0 && p.groups > 0) s_off[p.groups] = __ldg(p.a_off + p.groups);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int m_total = p.groups > 0 ? s_off[p.groups] : p.M;
  const int num_tiles = num_n * ((m_total + C::BM - 1) / C::BM);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;  // k-iteration counter across all tiles (ring position)
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        const TileInfo tl = tile_info(t, num_n, C::BM, C::BN, p, s_off, s_rows);
        if (tl.empty) continue;
        const int m0 = tl.m0;
        const int a_tile = m0 / 128;
        int nsfb = 0;
        for (int j = 0; j < C::NB_SFB; ++j)
          if (tl.b0 / 128 + j < p.b_rowtiles) ++nsfb;
        for (int kt = 0; kt < num_kt; ++kt, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
          if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          int nkc = p.kchunks - kt * C::KB_PER_STAGE;
          if (nkc > C::KB_PER_STAGE) nkc = C::KB_PER_STAGE;
          const uint32_t bytes = C::A_BYTES + C::B_BYTES + (uint32_t)nkc * 512u * (1u + (uint32_t)nsfb);
          mbar_expect_tx(&full[s], bytes);
          tma_load_2d(sA + s * C::A_BYTES, &tmA, kt * (C::BK / 2), m0, &full[s]);
          tma_load_2d(sB + s * C::B_BYTES, &tmB, kt * (C::BK / 2), tl.b0, &full[s]);
          const int64_t kc0 = (int64_t)kt * C::KB_PER_STAGE;
          bulk_g2s(sSFA + s * C::SFA_BYTES, p.a_sf + ((int64_t)a_tile * p.kchunks + kc0) * 512,
                   (uint32_t)nkc * 512u, &full[s]);
          for (int j = 0; j < nsfb; ++j)
            bulk_g2s(sSFB + s * C::SFB_BYTES + j * 512 * C::KB_PER_STAGE,
                     p.b_sf + ((int64_t)(tl.b0 / 128 + j) * p.kchunks + kc0) * 512, (uint32_t)nkc * 512u, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t acc = tmem + C::TM_ACC;
      int it = 0;
      int ti = 0;  // tiles done by this CTA
      for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
        if (tile_info(t, num_n, C::BM, C::BN, p, s_off, s_rows).empty) continue;
        // the epilogue must have drained the previous tile's accumulator
        if (!mbar_wait_bounded(acc_empty, ((uint32_t)ti & 1u) ^ 1u)) { *abort_flag = 1; break; }
        tc_fence_after();
        for (int kt = 0; kt < num_kt; ++kt, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
          if (!mbar_wait_bounded(&full[s], ph) || !mbar_wait_bounded(&sf_full[s], ph)) { *abort_flag = 1; break; }
          if (*abort_flag) break;
          tc_fence_after();
          int nkc = p.kchunks - kt * C::KB_PER_STAGE;
          if (nkc > C::KB_PER_STAGE) nkc = C::KB_PER_STAGE;
          const uint32_t sfa_col = tmem + C::TM_SFA + s * 4 * C::KB_PER_STAGE;
          const uint32_t sfb_col = tmem + C::TM_SFB + s * 4 * C::KB_PER_STAGE * C::NB_SFB;
          const uint32_t a_base = smem_u32(sA + s * C::A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * C::B_BYTES);
          for (int kb = 0; kb < nkc; ++kb) {
            // K = 64 FP4 elements = 32 bytes further along the 128-byte swizzled row
            const uint64_t ad = smem_desc(a_base + kb * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(b_base + kb * 32, 16, 1024, 2);
            mma_fp4_block16(acc, ad, bd, C::IDESC, sfa_col + kb * 4, sfb_col + kb * 4 * C::NB_SFB,
                            (kt > 0 || kb > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(acc_full);
        ++ti;
      }
    }
  } else if (warp >= 2 + C::EPI_WARPS) {
    // ------------------------------------------------------------ scale writers
    // Each 512-byte scale tile (128 rows x 4 blocks, MMA layout: row r's 4
    // bytes at 16 (r % 32) + 4 (r / 32)) becomes 4 TMEM columns in which lane
    // L holds bytes [16 (L % 32), 16 (L % 32) + 16) of the tile -- on every
    // subpartition, the image a 32x128b.warpx4 tcgen05.cp would produce.
    const int q = warp & 3;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles && !*abort_flag; t += gridDim.x) {
      if (tile_info(t, num_n, C::BM, C::BN, p, s_off, s_rows).empty) continue;
      bool ok = true;
      for (int kt = 0; kt < num_kt; ++kt, ++it) {
        const int s = it % C::STAGES;
        const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], ph));  // warp-uniform exit
        if (!ok) break;
        int nkc = p.kchunks - kt * C::KB_PER_STAGE;
        if (nkc > C::KB_PER_STAGE) nkc = C::KB_PER_STAGE;
        const uint8_t* a_src = sSFA + s * C::SFA_BYTES + lane * 16;
        const uint8_t* b_src = sSFB + s * C::SFB_BYTES + lane * 16;
        const uint32_t a_col = lane_base + C::TM_SFA + s * 4 * C::KB_PER_STAGE;
        const uint32_t b_col = lane_base + C::TM_SFB + s * 4 * C::KB_PER_STAGE * C::NB_SFB;
        for (int kb = 0; kb < nkc; ++kb) {
          tmem_st_32x32b_x4(a_col + kb * 4, *reinterpret_cast<const uint4*>(a_src + kb * 512));
#pragma unroll
          for (int j = 0; j < C::NB_SFB; ++j)
            tmem_st_32x32b_x4(b_col + kb * 4 * C::NB_SFB + j * 4,
                              *reinterpret_cast<const uint4*>(b_src + j * 512 * C::KB_PER_STAGE + kb * 512));
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[s]);
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;                      // TMEM subpartition this warp may read
    const int cbase = ((warp - 2) >> 2) * (C::BN / 2);  // this warp's half of the columns
    int ti = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      const TileInfo tl = tile_info(t, num_n, C::BM, C::BN, p, s_off, s_rows);
      if (tl.empty) continue;
      const int m0 = tl.m0, n0 = tl.n0;
      const float alpha = __fmul_rn(__ldg(p.a_ts + tl.g), __ldg(p.b_ts + tl.g));
      const int par_ti = ti++;
      const bool ok = mbar_wait_bounded(acc_full, (uint32_t)par_ti & 1u);
      if (!ok) *abort_flag = 1;
      if (!ok || *abort_flag) break;
      tc_fence_after();
      const int row = m0 + sub * 32 + lane;
      const uint32_t tbase = tmem + C::TM_ACC + ((uint32_t)(sub * 32) << 16) + cbase;
      epilogue_rows<C::BN>(tbase, row, tl.row_end, n0, cbase, p, alpha, [&] {
        if (lane == 0) mbar_arrive(acc_empty);
      });
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TM_COLS);
  }
}

// ------------------------------------------------------------------ split-K kernel (few output tiles)
//
// When the output has few tiles -- a decode-sized batch: M of one or two
// 128-row tiles against a large weight -- the persistent kernel leaves most
// SMs idle and each busy SM walks the whole K serially (the per-call FP4
// overhead the Qwen3.6-35B-A3B W4A4 tutorial measures at batch 1, section
// "吞吐量").  Here each 128 x 128 output tile is computed by a cluster of S
// CTAs that split K into S contiguous ranges: every CTA streams its range of
// A and B through a ring with the same producer / MMA / scale-writer roles
// as the persistent kernel, accumulating an FP32 partial tile in tensor
// memory.  CTA r reduces rows [r 128/S, (r+1) 128/S) of the tile: every CTA
// stores its partial of those rows from tensor memory straight into slot
// `rank` of CTA r's receive buffer (distributed shared memory stores, which
// need no reply), and after one cluster barrier CTA r adds the S partials in
// rank order 0..S-1 from its own shared memory, scales by s_gA s_gB and
// stores bf16.  The sum order is fixed, so the result is deterministic; no
// workspace and no second launch.
namespace splitk {
constexpr int BM = 128, BN = 128;
constexpr int BK = 256;                  // FP4 elements per stage (128 bytes per row)
constexpr int KB = BK / 64;              // MMAs (K = 64) per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;     // 16 KiB
constexpr int B_BYTES = BN * BK / 2;     // 16 KiB
constexpr int SF_BYTES = 512 * KB;       // one 128-row scale tile per operand
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + 2 * SF_BYTES;
constexpr int PART_STRIDE = BN + 4;      // floats per partial-tile row in shared memory
constexpr int PART_BYTES = BM * PART_STRIDE * 4;  // receive buffer: S partials of this CTA's BM / S rows
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + PART_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int TM_ACC = 0;                        // 128 lanes x 128 FP32 columns
constexpr int TM_SFA = BN;                       // STAGES x 4 KB columns
constexpr int TM_SFB = BN + STAGES * 4 * KB;     // STAGES x 4 KB columns
constexpr int TM_COLS = 256;
constexpr int EPI_WARPS = 4;                     // one per TMEM subpartition, all 128 columns
constexpr int SF_WARPS = 4;
constexpr int THREADS = 64 + 32 * (EPI_WARPS + SF_WARPS);
constexpr int MAX_SPLIT = 8;                     // portable cluster size
constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(TM_SFB + STAGES * 4 * KB <= TM_COLS, "tensor memory");
}  // namespace splitk

__global__ void __launch_bounds__(splitk::THREADS, 1)
    gemm_w4a4_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                            GemmParams p) {
  using namespace splitk;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SF_BYTES;
  float* recv = reinterpret_cast<float*>(sSFB + STAGES * SF_BYTES);  // [S][BM / S][PART_STRIDE]
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(recv) + PART_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_full = empty + STAGES;
  uint64_t* acc_full = sf_full + STAGES;
  uint64_t* recv_full = acc_full + 1;  // every CTA's partial rows have arrived (transaction bytes)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* stage = reinterpret_cast<float*>(smem);  // [BM][PART_STRIDE]: this CTA's partial, over the drained ring

  cg::cluster_group cluster = cg::this_cluster();
  const int split = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x / split;
  const int num_n = (p.N + BN - 1) / BN;
  const int mt = tile / num_n;
  const int m0 = mt * BM, n0 = (tile - mt * num_n) * BN;
  const int num_kt = (p.kchunks + KB - 1) / KB;
  // contiguous K-stage range of this CTA; split <= num_kt, so none is empty
  const int kt0 = (int)((int64_t)num_kt * rank / split);
  const int kt1 = (int)((int64_t)num_kt * (rank + 1) / split);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], SF_WARPS);
    }
    mbar_init(acc_full, 1);
    mbar_init(recv_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    // the S partial-row blocks this CTA will receive, (BM / S) rows each
    mbar_expect_tx(recv_full, (uint32_t)(BM * PART_STRIDE * 4));
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TM_COLS);
    tmem_relinquish();
  }
  // first half of a cluster barrier: the peers' receive barriers are
  // initialised before any partial is sent (the wait comes just before)
  cluster_arrive();
  griddep_wait();  // global memory only after this point (programmatic dependent launch)
  const float alpha = __fmul_rn(__ldg(p.a_ts), __ldg(p.b_ts));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int kt = kt0; kt < kt1; ++kt) {
        const int it = kt - kt0, s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u)) { *abort_flag = 1; break; }
        if (*abort_flag) break;
        int nkc = p.kchunks - kt * KB;
        if (nkc > KB) nkc = KB;
        mbar_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES) + 2u * (uint32_t)nkc * 512u);
        tma_load_2d(sA + s * A_BYTES, &tmA, kt * (BK / 2), m0, &full[s]);
        tma_load_2d(sB + s * B_BYTES, &tmB, kt * (BK / 2), n0, &full[s]);
        const int64_t kc0 = (int64_t)kt * KB;
        bulk_g2s(sSFA + s * SF_BYTES, p.a_sf + ((int64_t)(m0 / 128) * p.kchunks + kc0) * 512, (uint32_t)nkc * 512u,
                 &full[s]);
        bulk_g2s(sSFB + s * SF_BYTES, p.b_sf + ((int64_t)(n0 / 128) * p.kchunks + kc0) * 512, (uint32_t)nkc * 512u,
                 &full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kt = kt0; kt < kt1 && ok; ++kt) {
        const int it = kt - kt0, s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!mbar_wait_bounded(&full[s], ph) || !mbar_wait_bounded(&sf_full[s], ph) || *abort_flag) {
          ok = false;
          break;
        }
        tc_fence_after();
        int nkc = p.kchunks - kt * KB;
        if (nkc > KB) nkc = KB;
        const uint32_t a_base = smem_u32(sA + s * A_BYTES);
        const uint32_t b_base = smem_u32(sB + s * B_BYTES);
        for (int kb = 0; kb < nkc; ++kb)
          mma_fp4_block16(tmem + TM_ACC, smem_desc(a_base + kb * 32, 16, 1024, 2), smem_desc(b_base + kb * 32, 16, 1024, 2),
                          IDESC, tmem + TM_SFA + s * 4 * KB + kb * 4, tmem + TM_SFB + s * 4 * KB + kb * 4,
                          (it > 0 || kb > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (ok) tc_commit(acc_full);
      else *abort_flag = 1;
    }
  } else if (warp >= 2 + EPI_WARPS) {
    // ------------------------------------------------------------ scale writers
    // the persistent kernel's image: per 512-byte scale tile, 4 TMEM columns in
    // which lane L holds bytes [16 (L % 32), +16) on every subpartition
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    for (int kt = kt0; kt < kt1; ++kt) {
      const int it = kt - kt0, s = it % STAGES;
      const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded(&full[s], ph))) {  // warp-uniform exit
        *abort_flag = 1;
        break;
      }
      int nkc = p.kchunks - kt * KB;
      if (nkc > KB) nkc = KB;
      const uint8_t* a_src = sSFA + s * SF_BYTES + lane * 16;
      const uint8_t* b_src = sSFB + s * SF_BYTES + lane * 16;
      for (int kb = 0; kb < nkc; ++kb) {
        tmem_st_32x32b_x4(lane_base + TM_SFA + s * 4 * KB + kb * 4, *reinterpret_cast<const uint4*>(a_src + kb * 512));
        tmem_st_32x32b_x4(lane_base + TM_SFB + s * 4 * KB + kb * 4, *reinterpret_cast<const uint4*>(b_src + kb * 512));
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[s]);
    }
  } else {
    // ------------------------------------------------------------ partial tile -> shared memory
    // After acc_full every MMA of this CTA has completed, so every TMA load
    // has landed and been read and the ring can be overwritten.
    const int sub = warp & 3;
    const bool ok = mbar_wait_bounded(acc_full, 0u);
    if (!ok) *abort_flag = 1;
    if (ok) {
      tc_fence_after();
      float* prow = stage + (sub * 32 + lane) * PART_STRIDE;
      const uint32_t tbase = tmem + TM_ACC + ((uint32_t)(sub * 32) << 16);
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + c0, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 4) st_shared_v4(prow + c0 + j, r[j], r[j + 1], r[j + 2], r[j + 3]);
      }
    }
    fence_proxy_async_smem();  // the bulk copies below read these writes
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // ---- exchange: rows [q 128/S, (q+1) 128/S) of this CTA's partial go to slot
  // `rank` of CTA q's receive buffer, one bulk shared-to-shared copy per CTA
  const int rows_per = BM / split;  // split divides BM (a power of two up to 8)
  cluster_wait();                   // every CTA's receive barrier is initialised
  if (threadIdx.x == 0) {
    const uint32_t bytes = (uint32_t)(rows_per * PART_STRIDE * 4);
    for (int q = 0; q < split; ++q)
      bulk_s2cluster(cluster_addr(recv + (size_t)rank * rows_per * PART_STRIDE, (uint32_t)q),
                     stage + (size_t)q * rows_per * PART_STRIDE, bytes, cluster_addr(recv_full, (uint32_t)q));
  }
  // ---- reduction of this CTA's rows [rank * rows_per, +rows_per): per row 32
  // groups of 4 columns, each the sum of the S partials in rank order 0..S-1
  {
    const bool arrived = __all_sync(0xFFFFFFFFu, mbar_wait_bounded(recv_full, 0u));
    if (!arrived) *abort_flag = 1;
    const int r0 = rank * rows_per;
    const bool bad = *abort_flag != 0;
    for (int item = threadIdx.x; item < rows_per * (BN / 4); item += THREADS) {
      const int lrow = item / (BN / 4);
      const int col = (item % (BN / 4)) * 4;
      const int grow = m0 + r0 + lrow, gcol = n0 + col;
      if (grow >= p.M || gcol >= p.N) continue;
      float4 acc = *reinterpret_cast<const float4*>(recv + (size_t)lrow * PART_STRIDE + col);
      for (int q = 1; q < split; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(recv + ((size_t)q * rows_per + lrow) * PART_STRIDE + col);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      if (bad) acc = make_float4(__int_as_float(0x7FC00000), __int_as_float(0x7FC00000),
                                 __int_as_float(0x7FC00000), __int_as_float(0x7FC00000));
      const uint32_t lo = pack_bf16x2(acc.x * alpha, acc.y * alpha), hi = pack_bf16x2(acc.z * alpha, acc.w * alpha);
      __nv_bfloat16* dst = p.c + (int64_t)grow * p.ldc + gcol;
      if (gcol + 4 <= p.N && p.c_vec8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(lo, hi);
      } else {
        const uint32_t w[2] = {lo, hi};
        unsigned short* d16 = reinterpret_cast<unsigned short*>(dst);
        for (int j = 0; j < 4 && gcol + j < p.N; ++j) d16[j] = (unsigned short)(w[j >> 1] >> (16 * (j & 1)));
      }
    }
  }
  // every CTA has received all its rows, so every copy out of this CTA's
  // shared memory has completed: now it may exit
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Launch as a programmatic dependent launch (the kernel's set-up may overlap
// the previous kernel of the stream; the kernel waits with griddepcontrol.wait
// before it touches global memory), in clusters of `cluster` CTAs.
template <typename K>
static nvfp4_status launch_pdl(K kernel, int grid, int threads, int smem, int cluster, const CUtensorMap& ta,
                               const CUtensorMap& tb, const GemmParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, ta, tb, p);
  count_launches(1);
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

// Row-major uint8 matrix [rows][row_bytes] -> tensor map with a box of
// box_rows x 128 bytes, 128-byte swizzle, zero fill out of bounds.
static bool make_tmap(CUtensorMap* m, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN>
static nvfp4_status launch_gemm(const uint8_t* a, const uint8_t* b, const GemmParams& p, cudaStream_t s) {
  using C = GemmCfg<BN>;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, a, p.M, p.K / 2, C::BM) || !make_tmap(&tb, b, p.N, p.K / 2, C::BN)) return NVFP4_ERR_CUDA;
  // the attribute is per device: set it on every call (cheap)
  if (cudaFuncSetAttribute(gemm_w4a4_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return NVFP4_ERR_CUDA;
  const int tiles = ((p.N + C::BN - 1) / C::BN) * ((p.M + C::BM - 1) / C::BM);
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = tiles < sms ? tiles : sms;  // persistent: one CTA per SM
  return launch_pdl(gemm_w4a4_kernel<BN>, grid, C::THREADS, C::SMEM_BYTES, 1, ta, tb, p, s);
}

// Split-K dispatch: the output has few 128 x 128 tiles and K is long.  S CTAs
// per tile (one cluster), S = the SMs per tile rounded down to a power of two,
// at most 8 and at most the K stages; S = 1 means the split does not pay and
// the persistent kernel runs.
static int splitk_factor(const GemmParams& p, int sms) {
  const int tiles = ((p.M + splitk::BM - 1) / splitk::BM) * ((p.N + splitk::BN - 1) / splitk::BN);
  const int num_kt = (p.kchunks + splitk::KB - 1) / splitk::KB;
  if (tiles * 2 > sms) return 1;  // the persistent kernel fills the GPU at least as well
  if (num_kt < 8) return 1;       // short K (< 2048): the exchange costs more than the split saves
  int sk = sms / tiles;
  if (sk > splitk::MAX_SPLIT) sk = splitk::MAX_SPLIT;
  if (sk > num_kt) sk = num_kt;
  while (sk & (sk - 1)) --sk;  // a power of two, so that it divides the tile's 128 rows
  return sk;
}

static nvfp4_status launch_gemm_splitk(const uint8_t* a, const uint8_t* b, const GemmParams& p, int split,
                                       cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, a, p.M, p.K / 2, splitk::BM) || !make_tmap(&tb, b, p.N, p.K / 2, splitk::BN))
    return NVFP4_ERR_CUDA;
  if (cudaFuncSetAttribute(gemm_w4a4_splitk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           splitk::SMEM_BYTES) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  const int tiles = ((p.M + splitk::BM - 1) / splitk::BM) * ((p.N + splitk::BN - 1) / splitk::BN);
  return launch_pdl(gemm_w4a4_splitk_kernel, tiles * split, splitk::THREADS, splitk::SMEM_BYTES, split, ta, tb, p, s);
}

template <int BN>
static nvfp4_status launch_gemm_grouped(const uint8_t* a, const uint8_t* b, const GemmParams& p, int64_t b_rows,
                                        cudaStream_t s) {
  using C = GemmCfg<BN>;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, a, p.M, p.K / 2, C::BM) || !make_tmap(&tb, b, b_rows, p.K / 2, C::BN)) return NVFP4_ERR_CUDA;
  if (cudaFuncSetAttribute(gemm_w4a4_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return NVFP4_ERR_CUDA;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return launch_pdl(gemm_w4a4_kernel<BN>, sms, C::THREADS, C::SMEM_BYTES, 1, ta, tb, p, s);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;
}

nvfp4_status nvfp4_gemm_w4a4(const uint8_t* a_codes, const uint8_t* a_scales_mma, const float* a_tensor_scale,
                             const uint8_t* b_codes, const uint8_t* b_scales_mma, const float* b_tensor_scale,
                             int64_t M, int64_t N, int64_t K, void* c, int64_t ldc, void* workspace,
                             size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("nvfp4_gemm_w4a4");
  (void)workspace;
  (void)workspace_bytes;
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0 || ldc < N) return NVFP4_ERR_SHAPE;
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return NVFP4_ERR_SHAPE;
  if (!a_codes || !a_scales_mma || !a_tensor_scale || !b_codes || !b_scales_mma || !b_tensor_scale || !c)
    return NVFP4_ERR_ARG;
  auto a16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };
  if (!a16(a_codes) || !a16(b_codes) || !a16(a_scales_mma) || !a16(b_scales_mma) || ((uintptr_t)c & 3u))
    return NVFP4_ERR_ALIGN;
  GemmParams p;
  p.a_sf = a_scales_mma;
  p.b_sf = b_scales_mma;
  p.a_ts = a_tensor_scale;
  p.b_ts = b_tensor_scale;
  p.c = reinterpret_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.kchunks = (int)(K / 64);
  p.b_rowtiles = (int)((N + 127) / 128);
  p.c_vec16 = (((uintptr_t)c & 15u) == 0 && (ldc % 8) == 0) ? 1 : 0;
  p.c_vec32 = (((uintptr_t)c & 31u) == 0 && (ldc % 16) == 0) ? 1 : 0;
  p.c_vec8 = (((uintptr_t)c & 7u) == 0 && (ldc % 4) == 0) ? 1 : 0;
  p.groups = 0;
  p.a_off = nullptr;
  p.a_rows = nullptr;
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int split = splitk_factor(p, sms);
  if (split > 1) return launch_gemm_splitk(a_codes, b_codes, p, split, (cudaStream_t)stream);
  return launch_gemm<256>(a_codes, b_codes, p, (cudaStream_t)stream);
}

size_t nvfp4_gemm_grouped_workspace_size(int groups, int64_t a_rows_total, int64_t N, int64_t K) {
  (void)groups;
  (void)a_rows_total;
  (void)N;
  (void)K;
  return 0;
}

nvfp4_status nvfp4_gemm_w4a4_grouped(int groups, const uint8_t* a_codes, const uint8_t* a_scales_mma,
                                     const float* a_tensor_scales, int64_t a_rows_total, const int32_t* a_row_offsets,
                                     const int32_t* a_rows, const uint8_t* b_codes, const uint8_t* b_scales_mma,
                                     const float* b_tensor_scales, int64_t N, int64_t K, void* c, int64_t ldc,
                                     void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("nvfp4_gemm_w4a4_grouped");
  (void)workspace;
  (void)workspace_bytes;
  if (groups < 1 || groups > GemmCfg<256>::MAX_GROUPS) return NVFP4_ERR_SHAPE;
  if (a_rows_total < 128 || a_rows_total % 128 != 0 || N < 128 || N % 128 != 0 || K < 64 || K % 64 != 0 || ldc < N)
    return NVFP4_ERR_SHAPE;
  if (a_rows_total > 0x7FFFFFFF || (int64_t)groups * N > 0x7FFFFFFF || K > 0x7FFFFFFF) return NVFP4_ERR_SHAPE;
  if (!a_codes || !a_scales_mma || !a_tensor_scales || !a_row_offsets || !a_rows || !b_codes || !b_scales_mma ||
      !b_tensor_scales || !c)
    return NVFP4_ERR_ARG;
  auto a16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };
  if (!a16(a_codes) || !a16(b_codes) || !a16(a_scales_mma) || !a16(b_scales_mma) || ((uintptr_t)c & 3u))
    return NVFP4_ERR_ALIGN;
  GemmParams p;
  p.a_sf = a_scales_mma;
  p.b_sf = b_scales_mma;
  p.a_ts = a_tensor_scales;
  p.b_ts = b_tensor_scales;
  p.c = reinterpret_cast<__nv_bfloat16*>(c);
  p.ldc = ldc;
  p.M = (int)a_rows_total;
  p.N = (int)N;
  p.K = (int)K;
  p.kchunks = (int)(K / 64);
  p.b_rowtiles = (int)((int64_t)groups * N / 128);
  p.c_vec16 = (((uintptr_t)c & 15u) == 0 && (ldc % 8) == 0) ? 1 : 0;
  p.c_vec32 = (((uintptr_t)c & 31u) == 0 && (ldc % 16) == 0) ? 1 : 0;
  p.c_vec8 = (((uintptr_t)c & 7u) == 0 && (ldc % 4) == 0) ? 1 : 0;
  p.groups = groups;
  p.a_off = a_row_offsets;
  p.a_rows = a_rows;
  return launch_gemm_grouped<256>(a_codes, b_codes, p, (int64_t)groups * N, (cudaStream_t)stream);
}

}  // extern "C"
