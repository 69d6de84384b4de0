/*
 * nvfp4qad.h -- C ABI of libnvfp4qad.so, the B200 (sm_100a) hot path of NVFP4
 * quantization-aware distillation (QAD).
 *
 * What the operations are, and where they are defined:
 *
 *  NVFP4 is a 4-bit floating-point element (E2M1: values 0, 0.5, 1, 1.5, 2,
 *  3, 4, 6 with a sign bit) stored in blocks of 16 consecutive elements, each
 *  block with an E4M3 (FP8) scale, and one FP32 scale per tensor ("two-level
 *  scaling") -- Nemotron-3-Nano-30B NVFP4 article, section "NVFP4-Format und
 *  warum es wichtig ist?" and "Wichtige Erkenntnisse".
 *
 *  QAD runs every student forward pass through simulated (fake) quantization
 *  and trains the student to match a frozen BF16 teacher through a KL
 *  divergence between their output-token distributions -- Nemotron 3.5
 *  Lightning NVFP4 article, section "QAD的工作原理"; Nemotron-3-Nano article,
 *  "Von QAT zu QAD".  Scales are either recomputed from the max every step
 *  (dynamic-scale QAD) or taken from calibration and held fixed (frozen-scale
 *  QAD) -- Nemotron 3.5 Lightning article, "量化尺度处理策略".
 *
 *  W4A4: weights and activations are both NVFP4, so the linear layer is a
 *  block-scaled FP4 x FP4 GEMM on the FP4 tensor cores -- Qwen3.6-35B-A3B
 *  W4A4 NVFP4 tutorial page, "为什么目标是 W4A4".
 *
 * Numerical definitions (identical on every entry point):
 *   per-tensor scale (decode direction)  s_g = amax(|x|) / 2688   (2688 = 6*448)
 *   per-block scale  (E4M3, RNE, saturating at 448)
 *                    s_b = E4M3( max_{block}|x| / (6 * s_g) ),  s_b = 0 if s_g = 0
 *   decode scale     d   = float(s_b) * s_g                     (binary32)
 *   element code     q   = E2M1( x / d )  RNE, |.| >= 6 -> 6, sign kept;
 *                    q   = +0 for every element of a block with d = 0
 *   dequantized      x^  = value(q) * d                         (binary32, then
 *                                                                 bf16 RNE)
 *   Each binary32 operation above is rounded once (no fused multiply-add), so
 *   codes and scales are reproducible bit for bit.
 *
 * Conventions:
 *   - Every function returns nvfp4_status; NVFP4_OK is 0.  Argument checks
 *     run on the host and fail before anything is launched.
 *   - Every pointer argument is a DEVICE pointer owned by the caller, unless
 *     the parameter says "host".  The library never allocates device memory;
 *     scratch is passed as (workspace, workspace_bytes), sized by the
 *     *_workspace_size() query of the same operation.
 *   - Every call is asynchronous on `stream` (a cudaStream_t, passed as
 *     void*; NULL is the legacy default stream) and never synchronizes,
 *     except nvfp4_device_error().
 *   - Matrices are row-major with a row stride `ld` counted in elements of
 *     their own type (bytes for uint8 code arrays).  Quantization blocks run
 *     along the last (contiguous) dimension, so `cols` must be a multiple of
 *     16; base pointers must be 16-byte aligned and ld * element size a
 *     multiple of 16 bytes.
 *   - Inputs must be finite, and logits given to the KL loss above -1e30;
 *     other inputs give NVFP4_OK and unspecified outputs.
 *   - Packed codes: byte j of a row holds element 2j in its low nibble and
 *     element 2j+1 in its high nibble.
 */
#ifndef NVFP4QAD_H
#define NVFP4QAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NVFP4QAD_ABI_VERSION 1

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_ARG = 1,       /* NULL pointer where one is required, bad enum, T <= 0 */
  NVFP4_ERR_SHAPE = 2,     /* negative or unsupported sizes (e.g. cols % 16 != 0) */
  NVFP4_ERR_ALIGN = 3,     /* pointer or row stride not 16-byte aligned           */
  NVFP4_ERR_DTYPE = 4,     /* dtype not supported by this entry point             */
  NVFP4_ERR_CUDA = 5,      /* a CUDA runtime call or launch failed                */
  NVFP4_ERR_TIMEOUT = 6,   /* a bounded device-side wait expired                  */
  NVFP4_ERR_DEVICE = 7,    /* device reported an error word (see nvfp4_device_error) */
  NVFP4_ERR_WORKSPACE = 8, /* workspace missing or smaller than the size query    */
  NVFP4_ERR_UNSUPPORTED = 9 /* no kernel for this device / configuration          */
} nvfp4_status;

typedef enum nvfp4_dtype { NVFP4_BF16 = 0, NVFP4_F32 = 1 } nvfp4_dtype;

/* Scale strategy of the two QAD variants (Nemotron 3.5 Lightning article,
 * "量化尺度处理策略"):
 *   DYNAMIC       s_g and every s_b recomputed from the data on each call
 *                 (dynamic-scale QAD; *tensor_scale is written).
 *   FROZEN_GLOBAL s_g given (a calibrated activation amax / 2688), s_b derived
 *                 per block: activations in frozen-scale QAD, whose blocks are
 *                 per token and cannot be calibrated ahead of time.
 *   FROZEN_ALL    s_g and s_b both given (frozen-scale QAD weights: "only the
 *                 weights are updated"). */
typedef enum nvfp4_scale_mode {
  NVFP4_DYNAMIC = 0,
  NVFP4_FROZEN_GLOBAL = 1,
  NVFP4_FROZEN_ALL = 2
} nvfp4_scale_mode;

/* Block-scale array layout.
 *   ROWMAJOR  uint8 [rows][cols/16], row stride cols/16 bytes.
 *   MMA       the layout the block-scaled tensor-core MMA reads: tiles of 128
 *             rows x 4 blocks (512 bytes), tiles ordered block-index fastest,
 *             row r / block kb of a tile at byte (r%32)*16 + (r/32)*4 + kb;
 *             size nvfp4_mma_scales_bytes(rows, cols); padding bytes (rows
 *             beyond `rows`, blocks beyond cols/16) are written as 0 by the
 *             quantizer and never affect a GEMM output that is stored. */
typedef enum nvfp4_scale_layout { NVFP4_SCALES_ROWMAJOR = 0, NVFP4_SCALES_MMA = 1 } nvfp4_scale_layout;

/* Human-readable name of a status code (static string, never NULL). */
const char* nvfp4_status_string(nvfp4_status status);

/* NVFP4QAD_ABI_VERSION of the loaded library. */
int nvfp4_abi_version(void);

/* Bytes of an MMA-layout block-scale array for a rows x cols tensor:
 * ceil(rows/128)*128 * ceil(cols/64)*4. */
size_t nvfp4_mma_scales_bytes(int64_t rows, int64_t cols);

/* Number of kernels this library has launched in this process so far (host
 * counter, incremented at each launch). */
uint64_t nvfp4_launch_count(void);

/* Synchronize `stream`, then read and clear the library's device error word.
 * *code_out (host, may be NULL) receives the raw word: 0 = none, otherwise a
 * kernel-specific reason (1 = bounded wait expired).  Returns NVFP4_OK,
 * NVFP4_ERR_TIMEOUT when a bounded wait expired, NVFP4_ERR_DEVICE for other
 * words, NVFP4_ERR_CUDA if the synchronization failed. */
nvfp4_status nvfp4_device_error(void* stream, int32_t* code_out);

/* Host-side fault injection (failure-detection tests; the pages' QAD runs are
 * long multi-job trainings, Qwen3.6-35B-A3B W4A4 tutorial, "成本").  After
 * nvfp4_fault_inject(n) with n >= 1, the n-th outermost call of an exported
 * operation from now returns NVFP4_ERR_CUDA before it validates its arguments
 * or launches anything; one failure per arming; n = 0 disarms.  Setting
 * NVFP4QAD_FAIL_AT=n in the environment arms it when the library loads.
 * Operations called by another exported operation (the MoE step's parts) are
 * not counted on their own.  Every exported operation also opens an NVTX
 * range named after itself for the duration of the call. */
void nvfp4_fault_inject(int64_t nth);

/* Self-test of the bounded device waits: one thread waits on an mbarrier that
 * nothing arrives at for limit_cycles SM clock cycles (1 .. 2^32), then sets
 * the device error word to 1, as every expired wait of this library does; the
 * next nvfp4_device_error returns NVFP4_ERR_TIMEOUT and the context stays
 * usable.  NVFP4_ERR_ARG for a limit outside the range. */
nvfp4_status nvfp4_selftest_timeout(int64_t limit_cycles, void* stream);

/* ------------------------------------------------------------------------
 * Quantize (steps: tensor amax [DYNAMIC] -> block scale -> E2M1 encode and
 * pack), NVFP4 definition of the Nemotron-3-Nano article, scale modes of the
 * Nemotron 3.5 Lightning article.
 *
 *   x             rows x cols of `dtype` (bf16 or f32), row stride ld_x elements
 *   mode          see nvfp4_scale_mode
 *   tensor_scale  one float: written in DYNAMIC mode, read otherwise
 *   block_scales  read in FROZEN_ALL mode, written otherwise; layout `layout`
 *                 (FROZEN_ALL requires ROWMAJOR)
 *   codes         rows x cols/2 bytes, row stride ld_codes bytes (>= cols/2)
 *   workspace     >= nvfp4_quantize_workspace_size(rows, cols, mode) bytes,
 *                 16-byte aligned; may be NULL when that size is 0.  Its
 *                 contents on entry do not matter.
 * In DYNAMIC mode two kernels run in stream order (a grid-wide amax, then
 * the encode); no host synchronization and no device-to-host copy happen.
 * rows == 0 is a no-op (DYNAMIC writes s_g = 0).
 * ------------------------------------------------------------------------ */
size_t nvfp4_quantize_workspace_size(int64_t rows, int64_t cols, nvfp4_scale_mode mode);

nvfp4_status nvfp4_quantize(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols,
                            int64_t ld_x, nvfp4_scale_mode mode, float* tensor_scale,
                            uint8_t* block_scales, nvfp4_scale_layout layout, uint8_t* codes,
                            int64_t ld_codes, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Self-test of the encode path's division.  The bf16 encoder divides each
 * element by its block's decode scale d with a correctly rounded reciprocal
 * of d and one FMA correction (Markstein) instead of a full IEEE division per
 * element; this call checks that quotient against IEEE division (CUDA's
 * __fdiv_rn) for every binary32 significand of d and every bf16 significand
 * and sign of x, over the exponent offsets that give quotients in
 * [2^-5, 2^4).  mismatches, first: device, 8 bytes each; on completion
 * *mismatches holds the number of differing quotients (0 expected) and
 * *first one of them encoded as (d significand << 16) | ((k + 8) << 8) | x
 * index, or all ones.  Asynchronous on `stream`. */
nvfp4_status nvfp4_selftest_division(uint64_t* mismatches, uint64_t* first, void* stream);

/* Dense FP4 tensor-core throughput probe (measurement support for the W4A4
 * GEMM's roofline).  Launches `ctas` CTAs (one per SM when ctas <= the SM
 * count; each takes all 512 tensor-memory columns and enough shared memory to
 * keep others off its SM), each issuing `iters` x 4 block-scaled FP4 MMAs
 * (tcgen05.mma.kind::mxf4nvf4, 128 x 256 x 64, UE4M3 scales of 1.0) back to
 * back on one resident shared-memory stage -- the instruction and tile of
 * nvfp4_gemm_w4a4 without its operand traffic.  *flop_per_launch (host,
 * may be NULL) receives 2 * 128 * 256 * 64 * 4 * iters * ctas; the caller
 * times the launch (CUDA events on `stream`).  1 <= iters <= 2^40,
 * 1 <= ctas <= 4096, else NVFP4_ERR_ARG. */
nvfp4_status nvfp4_probe_fp4_mma(int64_t iters, int ctas, double* flop_per_launch, void* stream);

/* ------------------------------------------------------------------------
 * Grouped quantize / fake-quant: one call for a list of tensors that share a
 * dtype and a scale mode, each with its own tensor scale (e.g. the routed and
 * shared expert weights of a MoE layer; one FP32 scale per expert).  Results
 * are identical to calling nvfp4_quantize / nvfp4_fake_quant on each tensor.
 * Kernels are launched per group of tensors (at most 144 tensors per
 * group): one encode launch per group, preceded in DYNAMIC mode by one
 * tensor-max launch.
 * ------------------------------------------------------------------------ */
typedef struct nvfp4_tensor_ref {
  const void* x;          /* device input, rows x cols of the call's dtype */
  int64_t rows, cols;     /* cols % 16 == 0 */
  int64_t ld_x;           /* row stride of x, elements */
  float* tensor_scale;    /* device, one float: written in DYNAMIC mode, read otherwise */
  uint8_t* block_scales;  /* device; quantize: as in nvfp4_quantize; fake-quant: ROWMAJOR,
                             read in FROZEN_ALL, else written when non-NULL */
  void* out;              /* device; quantize: codes (uint8); fake-quant: y (dtype) */
  int64_t ld_out;         /* row stride of out: bytes (codes) or elements (y) */
} nvfp4_tensor_ref;

/* Workspace bytes of a grouped (or single-tensor) call in `mode`; the same
 * workspace serves every group of the call, in stream order. */
size_t nvfp4_grouped_workspace_size(nvfp4_scale_mode mode);

/* tensors: HOST array of num_tensors descriptors (read during the call only).
 * Every descriptor is validated before any launch. */
nvfp4_status nvfp4_quantize_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                    nvfp4_scale_mode mode, nvfp4_scale_layout layout, void* workspace,
                                    size_t workspace_bytes, void* stream);

nvfp4_status nvfp4_fake_quant_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                      nvfp4_scale_mode mode, void* workspace, size_t workspace_bytes,
                                      void* stream);

/* Quantize and fake-quantize in one pass: tensors[i].out receives the codes
 * (as nvfp4_quantize_grouped) and y[i] the dequantized values (as
 * nvfp4_fake_quant_grouped, same dtype as the input, row stride ld_y[i]
 * elements); y and ld_y are HOST arrays of num_tensors entries.  For the
 * weights of a layer whose forward runs on the codes and whose backward
 * needs the dequantized weights. */
nvfp4_status nvfp4_quantize_fake_quant_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, void* const* y,
                                               const int64_t* ld_y, nvfp4_dtype dtype, nvfp4_scale_mode mode,
                                               nvfp4_scale_layout layout, void* workspace,
                                               size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Tensor max and tensor scale as separate steps, for a tensor whose rows are
 * spread over several GPUs: each rank takes the max of its rows, the ranks
 * combine the maxima with an all-reduce(max), and every rank then derives
 * the same s_g = amax / 2688 and quantizes its rows in FROZEN_GLOBAL mode --
 * the same codes and scales as a DYNAMIC call on the whole tensor.
 *   nvfp4_tensor_amax_grouped: amax[i] = max |x_i| (device, num_tensors floats;
 *     0 for an empty tensor); tensors[i].tensor_scale / block_scales / out are
 *     not used.
 *   nvfp4_global_scale_from_amax: tensor_scale[i] = amax[i] / 2688 (binary32
 *     division, as in DYNAMIC mode).
 * ------------------------------------------------------------------------ */
nvfp4_status nvfp4_tensor_amax_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                       float* amax, void* stream);
nvfp4_status nvfp4_global_scale_from_amax(const float* amax, int n, float* tensor_scale, void* stream);

/* ------------------------------------------------------------------------
 * MSE block-scale calibration (the starting scales of frozen-scale QAD,
 * Nemotron 3.5 Lightning article, "量化尺度处理策略": the page names MSE
 * calibration only).  With the tensor scale s_g given, each block's E4M3
 * scale s_b is the code (of the 127 finite non-negative ones) whose fake
 * quantization of the block has the least squared error
 *   err = sum_i (x_i - value(q_i) * d)^2,  d = value(s_b) * s_g,
 *   q_i = E2M1_RNE_sat(x_i / d) (all 0 when d = 0),
 * binary32 operations rounded once, the sum accumulated in element order
 * with FMA; a tie goes to the smaller code.  The result is meant for
 * FROZEN_ALL quantization.
 *   x             rows x cols (bf16 or f32), row stride ld_x
 *   tensor_scale  one float (device, read)
 *   block_scales  rows x cols/16 ROWMAJOR (device, written)
 *   block_err     rows x cols/16 floats (device), the least error, or NULL
 * ------------------------------------------------------------------------ */
nvfp4_status nvfp4_calibrate_mse(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols, int64_t ld_x,
                                 const float* tensor_scale, uint8_t* block_scales, float* block_err,
                                 void* stream);

/* Grouped form: tensors[i].tensor_scale is read, tensors[i].block_scales
 * written (ROWMAJOR), .out / .ld_out unused; block_err: HOST array of
 * num_tensors device pointers (entries may be NULL), or NULL. */
nvfp4_status nvfp4_calibrate_mse_grouped(int num_tensors, const nvfp4_tensor_ref* tensors, nvfp4_dtype dtype,
                                         float* const* block_err, void* stream);

/* ------------------------------------------------------------------------
 * Fake quantization: y = dequantize(quantize(x)) in one pass, the simulated
 * quantization every student forward pass goes through (Nemotron 3.5
 * Lightning article, "QAD的工作原理").  Bitwise equal to nvfp4_quantize
 * followed by nvfp4_dequantize with the same scales.
 *
 *   x, y          rows x cols of `dtype`; y may alias x (same ld) -- the amax
 *                 pass of DYNAMIC mode completes before any element is written
 *   tensor_scale  written in DYNAMIC mode, read otherwise
 *   block_scales  ROWMAJOR; read in FROZEN_ALL mode; otherwise written when
 *                 non-NULL (so a later FROZEN_ALL call can reuse them)
 * The straight-through estimator makes the backward pass the identity
 * (dx = dy), so there is no backward entry point.
 * ------------------------------------------------------------------------ */
size_t nvfp4_fake_quant_workspace_size(int64_t rows, int64_t cols, nvfp4_scale_mode mode);

nvfp4_status nvfp4_fake_quant(const void* x, nvfp4_dtype dtype, int64_t rows, int64_t cols,
                              int64_t ld_x, nvfp4_scale_mode mode, float* tensor_scale,
                              uint8_t* block_scales, void* y, int64_t ld_y, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dequantize: out = value(q) * (float(s_b) * s_g), rounded to out_dtype.
 *   codes         rows x cols/2 bytes, row stride ld_codes
 *   block_scales  layout `layout`
 *   tensor_scale  one float (device)
 *   out           rows x cols of out_dtype, row stride ld_out elements
 * ------------------------------------------------------------------------ */
nvfp4_status nvfp4_dequantize(const uint8_t* codes, int64_t ld_codes, const uint8_t* block_scales,
                              nvfp4_scale_layout layout, const float* tensor_scale, int64_t rows,
                              int64_t cols, void* out, nvfp4_dtype out_dtype, int64_t ld_out,
                              void* stream);

/* ------------------------------------------------------------------------
 * W4A4 GEMM: C = (s_gA * s_gB) * A^ * B^T, with A^ (M x K) and B^ (N x K)
 * the block-scaled NVFP4 operands, FP32 accumulation on the tcgen05
 * block-scaled FP4 tensor cores, bf16 output (RNE).  Qwen3.6-35B-A3B W4A4
 * tutorial, "为什么目标是 W4A4" and "吞吐量".
 *
 *   a_codes        M x K/2 bytes, contiguous (row stride K/2)
 *   a_scales_mma   A's block scales in the MMA layout (nvfp4_mma_scales_bytes(M, K))
 *   a_tensor_scale one float (device)
 *   b_codes        N x K/2 bytes, contiguous
 *   b_scales_mma   B's block scales in the MMA layout (nvfp4_mma_scales_bytes(N, K))
 *   b_tensor_scale one float (device)
 *   c              M x N bf16, row stride ldc elements (>= N)
 * Requires M, N >= 1, K >= 64 and K % 64 == 0.  Tails in M and N are
 * handled (out-of-range rows read as zero, out-of-range outputs not stored).
 * ------------------------------------------------------------------------ */
size_t nvfp4_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

nvfp4_status nvfp4_gemm_w4a4(const uint8_t* a_codes, const uint8_t* a_scales_mma,
                             const float* a_tensor_scale, const uint8_t* b_codes,
                             const uint8_t* b_scales_mma, const float* b_tensor_scale, int64_t M,
                             int64_t N, int64_t K, void* c, int64_t ldc, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Grouped W4A4 GEMM for the experts of a MoE layer (Nemotron-3-Nano article,
 * "Was ist Nemotron-Nano-3-30B-A3B-NVFP4?": 128 routed experts + 1 shared;
 * Qwen3.6 tutorial, "2. PTQ": experts are NVFP4 W4A4).  For every group g:
 *   C[rows of g] = (s_gA[g] * s_gB[g]) * A^_g * B^_g^T
 *
 *   a_codes         a_rows_total x K/2 bytes: the groups' activation rows, each
 *                   group in a segment [a_row_offsets[g], a_row_offsets[g] +
 *                   a_rows[g]) whose start is a multiple of 128 (rows of a
 *                   segment past a_rows[g] are padding and are not stored)
 *   a_scales_mma    MMA-layout block scales of the whole a_codes buffer
 *                   (nvfp4_mma_scales_bytes(a_rows_total, K))
 *   a_tensor_scales groups floats (device), one per group
 *   a_row_offsets   groups + 1 int32 (device); a_row_offsets[groups] is the end
 *                   of the last segment (<= a_rows_total)
 *   a_rows          groups int32 (device): valid rows of each segment
 *   b_codes         groups * N x K/2 bytes: B of group g in rows [g N, (g+1) N)
 *   b_scales_mma    MMA-layout block scales of the stacked B (groups * N rows)
 *   b_tensor_scales groups floats (device)
 *   c               a_rows_total x N bf16, row stride ldc; only valid rows written
 * Requires 1 <= groups <= 256, a_rows_total % 128 == 0, N % 128 == 0,
 * K % 64 == 0.  The segment table is read on the device, so routing results
 * never travel to the host.
 * ------------------------------------------------------------------------ */
size_t nvfp4_gemm_grouped_workspace_size(int groups, int64_t a_rows_total, int64_t N, int64_t K);

nvfp4_status nvfp4_gemm_w4a4_grouped(int groups, const uint8_t* a_codes, const uint8_t* a_scales_mma,
                                     const float* a_tensor_scales, int64_t a_rows_total,
                                     const int32_t* a_row_offsets, const int32_t* a_rows,
                                     const uint8_t* b_codes, const uint8_t* b_scales_mma,
                                     const float* b_tensor_scales, int64_t N, int64_t K, void* c,
                                     int64_t ldc, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Grouped BF16 GEMM on the tcgen05 tensor cores (FP32 accumulation in
 * tensor memory, bf16 output RNE) for the straight-through backward of the
 * MoE layer, whose gradients are plain BF16 products with the dequantized
 * operands (Nemotron 3.5 Lightning article, "QAD的工作原理").  Always
 * C = A * B^T.
 *
 * Operand storage (row-major, a_rows x a_cols with row stride lda elements;
 * b likewise):
 *   *_mn_major = 0  K-major: element (i, k) of the operand at [i][k]
 *   *_mn_major = 1  MN-major: element (i, k) at [k][i]
 * (i is the M index for A, the N index for B.)
 *
 *   mode 0 (M-segments)  A's M range in segments [seg_off[g], seg_off[g] +
 *                        seg_len[g]) with seg_off[g] % 128 == 0 and the M
 *                        extent a multiple of 128; B of group g: N indices
 *                        [g N, (g+1) N) (K-major) or K indices [g K, (g+1) K)
 *                        (MN-major); c: M extent x N (ldc): the segments'
 *                        rows are written (when c is 16-byte aligned with
 *                        ldc % 8 == 0, also the padding rows of each
 *                        segment's last 128-row tile, with A's padding rows
 *                        times B).  K % 64 == 0; M is ignored.
 *   mode 1 (K-segments)  group g reduces over K indices [seg_off[g],
 *                        seg_off[g] + seg_len[g]) of A and B (seg_off[g] % 64
 *                        == 0; K indices up to the next multiple of 64 are
 *                        read and must hold zeros); c: groups * M x N, group g
 *                        in rows [g M, (g+1) M); M <= A's M extent, N <= B's
 *                        N extent, equal K extents; K is ignored.  A group
 *                        with seg_len 0 writes zeros.
 *   seg_off, seg_len     device int32 arrays (groups + 1 and groups entries)
 * 1 <= groups <= 256; a, b 16-byte aligned, lda * 2 and ldb * 2 multiples of
 * 16; c 4-byte aligned.
 * ------------------------------------------------------------------------ */
nvfp4_status nvfp4_gemm_bf16_grouped(int mode, int groups, const void* a, int a_mn_major, int64_t a_rows,
                                     int64_t a_cols, int64_t lda, const void* b, int b_mn_major, int64_t b_rows,
                                     int64_t b_cols, int64_t ldb, const int32_t* seg_off, const int32_t* seg_len,
                                     int64_t M, int64_t N, int64_t K, void* c, int64_t ldc, void* stream);

/* ------------------------------------------------------------------------
 * Weight-only NVFP4 GEMM (W4A16), the format of the Nemotron 3.5 Lightning
 * checkpoint; the Qwen3.6-35B-A3B W4A4 tutorial (section "为什么目标是 W4A4
 * 而不是 W4A16") contrasts it with W4A4: the weights are turned back into
 * 16-bit values in the GEMM's main loop and the product runs at 16 bits.
 *   C[M x N] = A[M x K] * W^[N x K]^T,  FP32 accumulation, bf16 output,
 *   W^[n][k] = bf16(value(q[n][k]) * (value(s_b[n][k/16]) * s_g))
 * (each product a binary32 multiply rounded once, then rounded to bf16:
 * exactly the bf16 fake-quant weights of nvfp4_quantize_fake_quant).
 *   a               bf16, row-major M x K, leading dimension lda (elements)
 *   b_codes         W's E2M1 codes, N x K/2 bytes, row-major, contiguous
 *                   (low nibble = even element)
 *   b_scales        W's E4M3 block scales in NVFP4_SCALES_ROWMAJOR layout
 *                   (N x K/16, contiguous)
 *   b_tensor_scale  device pointer to W's FP32 tensor scale s_g
 *   c               bf16, row-major M x N, leading dimension ldc (elements)
 * K % 64 == 0; a 16-byte aligned with lda * 2 a multiple of 16; b_codes
 * 16-byte aligned; b_scales and c 4-byte aligned.  One kernel launch;
 * NVFP4_ERR_SHAPE / _ARG / _ALIGN on bad arguments (nothing launched).
 * ------------------------------------------------------------------------ */
nvfp4_status nvfp4_gemm_w4a16(const void* a, int64_t lda, const uint8_t* b_codes, const uint8_t* b_scales,
                              const float* b_tensor_scale, int64_t M, int64_t N, int64_t K, void* c, int64_t ldc,
                              void* stream);

/* ------------------------------------------------------------------------
 * MoE layer of the QAD student: 128 routed experts plus one shared expert,
 * top-6 routing (Nemotron-3-Nano-30B NVFP4 article, "Was ist
 * Nemotron-Nano-3-30B-A3B-NVFP4?"), SwiGLU expert FFNs whose weights and
 * activations are NVFP4 (W4A4) with frozen scales (Qwen3.6-35B-A3B W4A4
 * tutorial, "2. PTQ"; Nemotron 3.5 Lightning article, "量化尺度处理策略").
 * For token t with routed experts e_j and combine weights w_j:
 *   y_t = sum_j w_j E_{e_j}(x_t) + E_shared(x_t),
 *   E(x) = Q(a) W^_down^T,  a = silu(Q(x) W^_gate^T) * (Q(x) W^_up^T),
 * Q = NVFP4 fake quantization (weights FROZEN_ALL, x and a FROZEN_GLOBAL
 * with one tensor scale per expert), silu(g) = g / (1 + exp(-g)); the gate
 * and up products are rounded to bf16, a is rounded to bf16 before Q.
 * Backward: straight-through estimator (dQ(v)/dv = identity), BF16 grads.
 *
 * Groups: g < experts is routed expert g; g = experts the shared expert.
 * Routed (token, slot) pairs are permuted into rows: group g owns rows
 * [seg_off[g], seg_off[g] + seg_len[g]), seg_off[g] % 128 == 0, rows in
 * increasing (token, slot) order; rows past seg_len[g] up to the next
 * segment are padding (row_token -1) and hold zeros in every row buffer.
 * ------------------------------------------------------------------------ */

/* Rows of the permutation buffers: tokens*topk + 127*experts +
 * ceil(tokens/128)*128, rounded up to a multiple of 128. */
int64_t nvfp4_moe_rows_capacity(int tokens, int topk, int experts);

/* Routing.  expert_ids, combine_weights: tokens x topk (device).  Outputs
 * (device): seg_len [experts+1], seg_off [experts+2] (seg_off[experts+1] =
 * end of the last segment), row_token / row_weight [rows_cap] (shared rows
 * have weight 1), slot_row [tokens x topk] = the row of each assignment.
 * An id outside [0, experts) is routed nowhere: its slot_row is -1 and the
 * device error word becomes 3.  rows_cap >= nvfp4_moe_rows_capacity(...).
 * Rows in [seg_off[experts+1], rows_cap) are not written by this call. */
nvfp4_status nvfp4_moe_route(const int32_t* expert_ids, const float* combine_weights, int tokens, int topk,
                             int experts, int32_t* seg_len, int32_t* seg_off, int32_t* row_token,
                             float* row_weight, int32_t* slot_row, int64_t rows_cap, void* stream);

/* Gather + FROZEN_GLOBAL quantize: row r of the permutation holds
 * x[row_token[r]] (zeros when row_token[r] < 0 or r >= seg_off[groups]),
 * quantized with tensor scale tensor_scales[group of r].
 *   x        bf16 tokens x cols, row stride ld_x
 *   codes    rows_cap x cols/2 bytes; scales_mma: MMA layout of rows_cap x cols
 *   xhat     bf16 rows_cap x cols, the dequantized rows, or NULL
 * rows_cap % 128 == 0, cols % 64 == 0, 1 <= groups <= 256. */
nvfp4_status nvfp4_moe_gather_quantize(const void* x, int64_t ld_x, const int32_t* row_token,
                                       const int32_t* seg_off, int groups, const float* tensor_scales,
                                       int64_t rows_cap, int64_t cols, uint8_t* codes, uint8_t* scales_mma,
                                       void* xhat, void* stream);

/* SwiGLU + FROZEN_GLOBAL quantize: a = bf16(silu(h_gate) * h_up) in binary32
 * (h_gate, h_up bf16 rows_cap x cols, row stride ld_h; silu through expf),
 * then quantized per row as above.  ahat: dequantized a or NULL; act: a
 * itself (bf16 rows_cap x cols) or NULL.  Padding rows give zeros. */
nvfp4_status nvfp4_moe_swiglu_quantize(const void* h_gate, const void* h_up, int64_t ld_h,
                                       const int32_t* row_token, const int32_t* seg_off, int groups,
                                       const float* tensor_scales, int64_t rows_cap, int64_t cols,
                                       uint8_t* codes, uint8_t* scales_mma, void* ahat, void* act, void* stream);

/* out[t] = bf16( sum_j w[t,j] * y[slot_row[t,j]] + y[seg_off[experts] + t] ),
 * binary32 sums in the order j = 0..topk-1, then the shared expert; y bf16
 * rows x cols (cols % 8 == 0), out bf16 tokens x cols; 1 <= topk <= 32. */
nvfp4_status nvfp4_moe_combine(const void* y, int64_t cols, const int32_t* slot_row, const float* combine_weights,
                               int tokens, int topk, const int32_t* seg_off, int experts, void* out, void* stream);

/* dyp[r] = bf16(row_weight[r] * dy[row_token[r]]), zeros on padding rows and
 * rows >= seg_off[groups]; dy tokens x cols, dyp rows_cap x cols (bf16). */
nvfp4_status nvfp4_moe_scale_rows(const void* dy, int64_t cols, const int32_t* row_token, const float* row_weight,
                                  const int32_t* seg_off, int groups, int64_t rows_cap, void* dyp, void* stream);

/* SwiGLU backward, binary32 with the hardware exponential and a fast
 * reciprocal for s = 1 / (1 + exp(-g)) (relative error ~1e-6),
 *   dG = da * u * s * (1 + g (1 - s)),  dU = da * g * s,
 * written as dgu[r] = [dG | dU] (bf16 rows_cap x 2 cols); da, h_gate, h_up
 * bf16 rows_cap x cols contiguous; zeros on padding rows.  cols % 8 == 0,
 * pointers 16-byte aligned. */
nvfp4_status nvfp4_moe_swiglu_backward(const void* da, const void* h_gate, const void* h_up, int64_t cols,
                                       const int32_t* row_token, const int32_t* seg_off, int groups,
                                       int64_t rows_cap, void* dgu, void* stream);

/* dx[t] = bf16( sum_j dxp[slot_row[t,j]] + dxp[seg_off[experts] + t] ), slots in order
 * j = 0..topk-1 then the shared expert; 1 <= topk <= 32. */
nvfp4_status nvfp4_moe_gather_sum(const void* dxp, int64_t cols, const int32_t* slot_row, int tokens, int topk,
                                  const int32_t* seg_off, int experts, void* dx, void* stream);

/* d_combine[t,j] = sum_c dy[t,c] * y[slot_row[t,j], c]  (binary32; 0 for an
 * assignment routed nowhere): the gradient of the layer w.r.t. its combine
 * weights. */
nvfp4_status nvfp4_moe_router_grad(const void* dy, const void* y, int64_t cols, const int32_t* slot_row, int tokens,
                                   int topk, float* d_combine, void* stream);

/* ROWMAJOR block scales of rows x cols -> the MMA layout (padding 0). */
nvfp4_status nvfp4_scales_to_mma(const uint8_t* block_scales, int64_t rows, int64_t cols, uint8_t* out,
                                 void* stream);

/* Shape of one MoE layer step. */
typedef struct qad_moe_shape {
  int tokens;    /* T >= 1 */
  int hidden;    /* H, % 256 == 0 */
  int ffn;       /* F, % 256 == 0 */
  int experts;   /* routed experts E (group E is the shared expert), E + 1 <= 256 */
  int topk;      /* routed experts per token, <= E and <= 32 */
  int save_act;  /* nonzero: the forward also stores a (pre-quantization) in QAD_MOE_ACT */
} qad_moe_shape;

/* Parameters of the layer (device pointers; group g's block in rows of g). */
typedef struct qad_moe_weights {
  const void* w_gate;          /* bf16 master weights, (E+1) F x H */
  const void* w_up;            /* bf16 (E+1) F x H */
  const void* w_down;          /* bf16 (E+1) H x F */
  const float* gate_ts;        /* frozen tensor scales, E+1 each */
  const float* up_ts;
  const float* down_ts;
  const uint8_t* gate_sb;      /* frozen block scales, ROWMAJOR, of the stacked weights */
  const uint8_t* up_sb;
  const uint8_t* down_sb;
  const uint8_t* gate_sb_mma;  /* the same in the MMA layout (nvfp4_scales_to_mma of the stack) */
  const uint8_t* up_sb_mma;
  const uint8_t* down_sb_mma;
  const float* x_ts;           /* frozen tensor scale of each group's input x, E+1 */
  const float* a_ts;           /* frozen tensor scale of each group's down-projection input a, E+1 */
} qad_moe_weights;

/* Buffers inside the step's workspace (offsets from qad_moe_workspace_buffer;
 * R = qad_moe_rows_capacity).  The forward fills the first group, the
 * backward reads them and fills the rest; a training step is forward then
 * backward with the same workspace and no other call in between. */
enum qad_moe_buffer {
  QAD_MOE_SEG_LEN = 0,  /* int32 [E+1] */
  QAD_MOE_SEG_OFF,      /* int32 [E+2] */
  QAD_MOE_ROW_TOKEN,    /* int32 [R] */
  QAD_MOE_ROW_WEIGHT,   /* f32 [R] */
  QAD_MOE_SLOT_ROW,     /* int32 [T x topk] */
  QAD_MOE_X_CODES,      /* u8 [R x H/2] */
  QAD_MOE_X_SCALES,     /* u8 MMA layout of R x H */
  QAD_MOE_X_HAT,        /* bf16 [R x H] */
  QAD_MOE_WG_CODES,     /* u8 [(E+1) F x H/2] */
  QAD_MOE_WU_CODES,     /* u8 [(E+1) F x H/2] */
  QAD_MOE_WD_CODES,     /* u8 [(E+1) H x F/2] */
  QAD_MOE_H_GATE,       /* bf16 [R x F] */
  QAD_MOE_H_UP,         /* bf16 [R x F] */
  QAD_MOE_A_CODES,      /* u8 [R x F/2] */
  QAD_MOE_A_SCALES,     /* u8 MMA layout of R x F */
  QAD_MOE_A_HAT,        /* bf16 [R x F] */
  QAD_MOE_ACT,          /* bf16 [R x F] (0 bytes unless save_act) */
  QAD_MOE_Y_ROWS,       /* bf16 [R x H] */
  QAD_MOE_DY_ROWS,      /* bf16 [R x H] */
  QAD_MOE_WD_HAT,       /* bf16 [(E+1) H x F]: dequantized W_down (bf16 fake-quant) */
  QAD_MOE_DA,           /* bf16 [R x F] */
  QAD_MOE_DGU,          /* bf16 [R x 2F] */
  QAD_MOE_WGU_HAT,      /* bf16 [(E+1) 2F x H]: dequantized W_gate / W_up of group g in rows 2gF.. / 2gF+F.. */
  QAD_MOE_DX_ROWS,      /* bf16 [R x H] */
  QAD_MOE_NUM_BUFFERS
};

/* 0 for an unsupported shape. */
size_t qad_moe_workspace_size(const qad_moe_shape* shape);
int64_t qad_moe_rows_capacity(const qad_moe_shape* shape);
/* Offset (256-byte aligned) and size of one buffer of the workspace (host outputs). */
nvfp4_status qad_moe_workspace_buffer(const qad_moe_shape* shape, int buffer, size_t* offset, size_t* bytes);

/* Forward.  shape, w: host structs.  x bf16 T x H; expert_ids int32 T x
 * topk; combine_weights f32 T x topk; y bf16 T x H; workspace 256-byte
 * aligned, >= qad_moe_workspace_size(shape). */
nvfp4_status qad_moe_forward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* x,
                             const int32_t* expert_ids, const float* combine_weights, void* y, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Backward of the last forward on this workspace.  dy bf16 T x H; outputs
 * dx bf16 T x H, dw_gate / dw_up bf16 (E+1) F x H, dw_down bf16 (E+1) H x F
 * (gradients w.r.t. the master weights through the straight-through
 * quantizers), d_combine f32 T x topk or NULL. */
nvfp4_status qad_moe_backward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* dy, void* dx,
                              void* dw_gate, void* dw_up, void* dw_down, float* d_combine, void* workspace,
                              size_t workspace_bytes, void* stream);

/* Expert-parallel form: the expert FFNs of this rank's experts on the rows it
 * received from every rank (expert parallelism with EP 4 / 8: Nemotron 3.5
 * Lightning NVFP4 article, training set-up; Qwen3.6-35B-A3B W4A4 tutorial,
 * "3. QAD").  Each received row is one (token, slot) assignment, so
 *   shape->tokens  rows received (>= 1), shape->topk must be 1,
 *   shape->experts this rank's experts E_r; there is no shared expert (it
 *                  runs on each token's home rank: call this with experts = 1
 *                  and every id 0 for it);
 *   expert_ids     [rows] the expert of each row among this rank's experts;
 *   w              the E_r experts' weights and scales as in qad_moe_forward
 *                  (no shared group: gate/up/down, the tensor scales and
 *                  x_ts / a_ts have E_r entries);
 *   y              [rows x hidden] bf16: y[r] = E_{id[r]}(x[r]), not combined
 *                  (the home rank weights and sums the returned rows).
 * Workspace: qad_moe_workspace_size(shape) bytes, as for qad_moe_forward.
 * The results of a row equal those qad_moe_forward computes for the same
 * (token, expert) pair, bit for bit (rows are independent in every step). */
nvfp4_status qad_moe_expert_forward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* x,
                                    const int32_t* expert_ids, void* y, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Backward of qad_moe_expert_forward (after it, same workspace): dy [rows x
 * hidden] is each received row's output gradient, already multiplied by its
 * combine weight on the home rank; dx [rows x hidden] the rows' input
 * gradients; dw_gate / dw_up [E_r F x H], dw_down [E_r H x F] the weight
 * gradients of this rank's experts, reduced over the received rows in row
 * order (sources in rank order keep the single-process order). */
nvfp4_status qad_moe_expert_backward(const qad_moe_shape* shape, const qad_moe_weights* w, const void* dy, void* dx,
                                     void* dw_gate, void* dw_up, void* dw_down, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * KL distillation loss, forward and backward in one pass (Nemotron 3.5
 * Lightning article, "QAD的工作原理"; Nemotron-3-Nano article, "Von QAT zu
 * QAD"; full-vocabulary form of the loss in the Qwen3.6 tutorial, section 3).
 * With p = softmax(z / T) per row:
 *   row_kl[i]   = sum_v p_t[i,v] * (log p_t[i,v] - log p_s[i,v])
 *   *loss       = (1/rows) * sum_i row_kl[i]       (fixed summation order)
 *   dlogits[i,v]= grad_scale * (p_s[i,v] - p_t[i,v]) / T
 * (forward KL(teacher || student), mean over tokens, no T^2 factor).
 *
 *   teacher, student  rows x vocab of `dtype`, row stride ld elements
 *   temperature       T > 0
 *   loss              one float (device), required
 *   row_kl            rows floats (device) or NULL
 *   dlogits           rows x vocab of `dtype`, row stride ld_grad, or NULL
 *                     (forward only)
 *   grad_scale        multiplier of the gradient; 1/rows gives the gradient
 *                     of *loss
 *   workspace         >= qad_kl_workspace_size(rows, vocab, dtype) bytes
 * Each logit is read from memory once; probabilities are never stored.
 * ------------------------------------------------------------------------ */
size_t qad_kl_workspace_size(int64_t rows, int64_t vocab, nvfp4_dtype dtype);

nvfp4_status qad_kl_fwd_bwd(const void* teacher, const void* student, nvfp4_dtype dtype,
                            int64_t rows, int64_t vocab, int64_t ld, float temperature,
                            float* loss, float* row_kl, void* dlogits, int64_t ld_grad,
                            float grad_scale, void* workspace, size_t workspace_bytes,
                            void* stream);

/* ------------------------------------------------------------------------
 * Top-k KL distillation loss (Qwen3.6-35B-A3B W4A4 tutorial, section "3.
 * QAD": --logit_kl_topk 4096): per row, S = the teacher's k largest logits
 * (among equal logits the smaller vocabulary index first; k >= vocab selects
 * the whole row), both softmaxes renormalised over S:
 *   row_kl[i]    = sum_{v in S} p_t^S (log p_t^S - log p_s^S)
 *   *loss        = (1/rows) * sum_i row_kl[i]
 *   dlogits[i,v] = grad_scale * (p_s^S[v] - p_t^S[v]) / T on S, 0 elsewhere
 * Arguments as qad_kl_fwd_bwd, plus k >= 1 (NVFP4_ERR_ARG otherwise); same
 * workspace (qad_kl_workspace_size).  S is found by a radix select over the
 * teacher logits held on chip; each logit is read from memory once.
 * ------------------------------------------------------------------------ */
nvfp4_status qad_kl_topk_fwd_bwd(const void* teacher, const void* student, nvfp4_dtype dtype,
                                 int64_t rows, int64_t vocab, int64_t ld, int64_t k, float temperature,
                                 float* loss, float* row_kl, void* dlogits, int64_t ld_grad,
                                 float grad_scale, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Top-p KL distillation loss (Qwen3.6-35B-A3B W4A4 tutorial, section "5.
 * 评估": its recommendation for the next QAD run, after the runs that hit the
 * output-length cap, is to select the teacher's top-p entries instead of the
 * top-k ones).  Per row, S = the shortest prefix of the teacher's entries in
 * decreasing logit order (equal logits: smaller vocabulary index first) whose
 * teacher probability softmax(z_t / T) sums to at least top_p; top_p >= 1
 * selects the whole row.  The loss and gradient over S are those of
 * qad_kl_topk_fwd_bwd with k = |S|.
 * Arguments as qad_kl_topk_fwd_bwd with top_p (> 0, NVFP4_ERR_ARG otherwise)
 * in place of k, plus:
 *   row_k       device int64 [rows] or NULL: receives |S| of every row
 *   workspace   >= qad_kl_topp_workspace_size(rows, vocab, dtype) bytes,
 *               16-byte aligned
 * The probabilities are summed in 64-bit fixed point (the largest logit of a
 * row weighs 2^40; exponentials from the hardware ex2), so |S| does not
 * depend on the order of the additions; against a float64 computation it can
 * differ only where the cumulative probability lies within ~1e-6 of top_p.
 * Three launches: a pass over the teacher logits that finds |S| (a radix
 * select whose buckets hold probability mass; for top_p >= 1 a fill), the
 * top-k loss kernel with that k per row, and the mean over the rows.
 * ------------------------------------------------------------------------ */
size_t qad_kl_topp_workspace_size(int64_t rows, int64_t vocab, nvfp4_dtype dtype);

nvfp4_status qad_kl_topp_fwd_bwd(const void* teacher, const void* student, nvfp4_dtype dtype,
                                 int64_t rows, int64_t vocab, int64_t ld, float top_p, float temperature,
                                 float* loss, float* row_kl, void* dlogits, int64_t ld_grad,
                                 float grad_scale, int64_t* row_k, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* ------------------------------------------------------------------------
 * qad_kl_fwd_bwd without a workspace argument, for callers that cannot
 * allocate device memory when they compute the loss (a framework whose
 * caching allocator holds the device budget, a fixed pre-planned memory
 * layout, or a path where a possibly synchronizing cudaMalloc is not
 * acceptable).  The method described on the pages has no counterpart of
 * this; it is a deployment convenience.
 *
 * Same arguments and results as qad_kl_fwd_bwd, minus the workspace.  The
 * per-row scratch is a static device array inside the library, of
 * NVFP4_KL_NOALLOC_MAX_ROWS floats (256 KiB), held on every GPU that loads
 * the library until the process exits; nothing is allocated by the call.
 *   - rows > NVFP4_KL_NOALLOC_MAX_ROWS returns NVFP4_ERR_SHAPE before any
 *     launch.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture.  Calls made outside a
 *     capture look the address up again, so after a cudaDeviceReset the
 *     first call must again come before any capture.
 *   - All calls on a device share the array and each call overwrites it: two
 *     calls that can run at the same time on the GPU (different streams,
 *     without ordering between them) race and may return wrong losses.
 *     Order them on one stream or with events.
 * ------------------------------------------------------------------------ */
#define NVFP4_KL_NOALLOC_MAX_ROWS 65536

nvfp4_status qad_kl_fwd_bwd_noalloc(const void* teacher, const void* student, nvfp4_dtype dtype,
                                    int64_t rows, int64_t vocab, int64_t ld, float temperature,
                                    float* loss, float* row_kl, void* dlogits, int64_t ld_grad,
                                    float grad_scale, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4QAD_H */
