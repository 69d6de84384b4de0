// kl.cu -- KL-divergence distillation loss and its gradient for sm_100a.
//
// The student is trained to match the frozen teacher's output-token
// distribution with a KL divergence (Nemotron 3.5 Lightning NVFP4 article,
// "QAD的工作原理"; Nemotron-3-Nano article, "Von QAT zu QAD").  Per row:
//   KL = sum_v p_t (log p_t - log p_s),  p = softmax(z / T),
//   dz_s = grad_scale * (p_s - p_t) / T.
// The full-vocabulary form is computed; the Qwen3.6 tutorial (section 3)
// explains why materialising [seq, vocab] fp32 probabilities is what makes it
// expensive, and this kernel never stores them.
//
// Design.  One thread-block cluster per row, C CTAs (C <= 8), each holding a
// contiguous slice of the row's teacher and student logits in shared memory:
//   1. a TMA bulk copy (cp.async.bulk, completion on an mbarrier) brings the
//      two slices from HBM into shared memory -- the only HBM read of the
//      logits;
//   2. slice max of both rows -> exchanged through distributed shared memory;
//   3. slice sums S_t, S_s and X = sum e_t (w_t - w_s) -> exchanged;
//   4. dLogits from the on-chip slice, 16-byte stores.
// Work is in the log2 domain: w = z * log2(e) / T, e = 2^(w - max w).  Per-row
// KL goes to the workspace; a second one-CTA kernel sums the rows in a fixed
// order (in double) into the mean, so the loss is deterministic.
#include <cooperative_groups.h>

#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace nvfp4 {

constexpr int kKlThreads = 512;
constexpr int kKlWarps = kKlThreads / 32;
constexpr int kKlMaxCluster = 8;
NVFP4_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T>
struct KlElem;
template <>
struct KlElem<__nv_bfloat16> {
  static constexpr int kVec = 8;  // elements per 16 bytes
  NVFP4_DEV static void unpack(const uint4& r, float (&v)[8]) {
    v[0] = bf16lo_to_f32(r.x); v[1] = bf16hi_to_f32(r.x); v[2] = bf16lo_to_f32(r.y); v[3] = bf16hi_to_f32(r.y);
    v[4] = bf16lo_to_f32(r.z); v[5] = bf16hi_to_f32(r.z); v[6] = bf16lo_to_f32(r.w); v[7] = bf16hi_to_f32(r.w);
  }
  NVFP4_DEV static uint4 pack(const float (&v)[8]) {
    return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                      pack_bf16x2(v[6], v[7]));
  }
  NVFP4_DEV static float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  NVFP4_DEV static void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};
template <>
struct KlElem<float> {
  static constexpr int kVec = 4;
  NVFP4_DEV static void unpack(const uint4& r, float (&v)[4]) {
    v[0] = __uint_as_float(r.x); v[1] = __uint_as_float(r.y); v[2] = __uint_as_float(r.z); v[3] = __uint_as_float(r.w);
  }
  NVFP4_DEV static uint4 pack(const float (&v)[4]) {
    return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
  }
  NVFP4_DEV static float load1(const float* p) { return *p; }
  NVFP4_DEV static void store1(float* p, float v) { *p = v; }
};

struct KlArgs {
  const void* teacher;
  const void* student;
  int64_t rows, vocab, ld;
  int64_t slice;          // elements per CTA (multiple of the 16-byte vector)
  float a;                // log2(e) / T
  float gscale;           // grad_scale / T
  float* row_kl;          // workspace, rows floats
  void* dlogits;          // may be NULL
  int64_t ld_grad;
};

// Block-wide reduction of NV values (sum or max) into warp 0's lane 0..NV-1
// results broadcast through shared memory.
template <int NV, bool MAX>
NVFP4_DEV void block_reduce(float (&v)[NV], float* scratch /* [kKlWarps][NV] */) {
#pragma unroll
  for (int i = 0; i < NV; ++i)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float w = __shfl_xor_sync(0xFFFFFFFFu, v[i], o);
      v[i] = MAX ? fmaxf(v[i], w) : v[i] + w;
    }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < NV; ++i) scratch[warp * NV + i] = v[i];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float acc = scratch[i];
    for (int w = 1; w < kKlWarps; ++w) acc = MAX ? fmaxf(acc, scratch[w * NV + i]) : acc + scratch[w * NV + i];
    v[i] = acc;
  }
  __syncthreads();
}

// Stand-in for positions of the shared-memory slice that hold no logit (the
// alignment pad before and after the slice): exp underflows to 0 and it never
// wins the max while the slice holds at least one real logit.
constexpr float kPadLogit = -1.0e30f;

template <typename T>
__global__ void __launch_bounds__(kKlThreads) kl_row_kernel(KlArgs args) {
  using E = KlElem<T>;
  constexpr int V8 = E::kVec;        // elements per 16-byte vector
  constexpr int ESZ = (int)sizeof(T);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint64_t bar;
  __shared__ float red[kKlWarps * 3];
  __shared__ float xchg[8];  // [0..1] slice max (t, s); [2..4] slice sums (S_t, S_s, Y)
  __shared__ int s_ok;

  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int64_t row = blockIdx.x / csize;
  const int64_t v0 = (int64_t)crank * args.slice;
  int64_t v1 = v0 + args.slice;
  if (v1 > args.vocab) v1 = args.vocab;
  const int n = v1 > v0 ? (int)(v1 - v0) : 0;

  const T* gt = reinterpret_cast<const T*>(args.teacher) + row * args.ld + v0;
  const T* gs = reinterpret_cast<const T*>(args.student) + row * args.ld + v0;
  // Teacher and student rows share one stride, so they share an alignment:
  // `head` logits precede the first 16-byte boundary; in shared memory the
  // slice starts `off` slots in so that the bulk-copied interior lands on a
  // 16-byte boundary too.
  int head = (int)(((16u - ((uint32_t)(uintptr_t)gt & 15u)) & 15u) / ESZ);
  if (head > n) head = n;
  const int off = (V8 - head % V8) % V8;
  const int nint = (n - head) / V8 * V8;      // bulk-copied interior
  const int tail0 = head + nint;              // first tail logit
  const int nslots = off + n;
  const int nvec = (nslots + V8 - 1) / V8;    // vectors covering the slice
  const int cap = nvec * V8;                  // slots actually used

  T* st = reinterpret_cast<T*>(smem_raw);
  T* ss = st + args.slice + 2 * V8;

  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    s_ok = 1;
  }
  __syncthreads();
  if (threadIdx.x == 0 && nint > 0) {
    mbar_expect_tx(&bar, (uint32_t)(2 * nint * ESZ));
    bulk_g2s(st + off + head, gt + head, (uint32_t)(nint * ESZ), &bar);
    bulk_g2s(ss + off + head, gs + head, (uint32_t)(nint * ESZ), &bar);
  }
  // head, tail and pad slots with plain accesses (disjoint from the bulk copy)
  for (int j = threadIdx.x; j < cap; j += kKlThreads) {
    const int i = j - off;  // logit index inside the slice
    if (i >= 0 && i < head) {
      st[j] = gt[i];
      ss[j] = gs[i];
    } else if (i >= tail0 && i < n) {
      st[j] = gt[i];
      ss[j] = gs[i];
    } else if (i < 0 || i >= n) {
      E::store1(st + j, kPadLogit);
      E::store1(ss + j, kPadLogit);
    }
  }
  if (nint > 0 && !mbar_wait_bounded(&bar, 0)) s_ok = 0;
  __syncthreads();
  const bool ok = s_ok != 0;

  const uint4* vt = reinterpret_cast<const uint4*>(st);
  const uint4* vs = reinterpret_cast<const uint4*>(ss);

  // ---- pass 1: slice max of z_t and z_s
  float mx[2] = {-INFINITY, -INFINITY};
  if (ok) {
    for (int k = threadIdx.x; k < nvec; k += kKlThreads) {
      float zt[V8], zs[V8];
      E::unpack(vt[k], zt);
      E::unpack(vs[k], zs);
#pragma unroll
      for (int j = 0; j < V8; ++j) {
        mx[0] = fmaxf(mx[0], zt[j]);
        mx[1] = fmaxf(mx[1], zs[j]);
      }
    }
  }
  block_reduce<2, true>(mx, red);
  if (threadIdx.x == 0) {
    xchg[0] = mx[0];
    xchg[1] = mx[1];
  }
  cluster.sync();
  float Mt = -INFINITY, Ms = -INFINITY;
  for (int r = 0; r < csize; ++r) {
    const float* peer = cluster.map_shared_rank(xchg, r);
    Mt = fmaxf(Mt, peer[0]);
    Ms = fmaxf(Ms, peer[1]);
  }
  // log2 domain: w = z * a with a = log2(e) / T > 0, so max w = max(z) * a;
  // d = w - max w <= 0 is formed by one FMA per logit.
  const float a = args.a;
  const float Wt = Mt * a, Ws = Ms * a;

  // ---- pass 2: S_t = sum 2^d_t, S_s = sum 2^d_s, Y = sum 2^d_t (d_t - d_s)
  float sums[3] = {0.f, 0.f, 0.f};
  if (ok) {
    for (int k = threadIdx.x; k < nvec; k += kKlThreads) {
      float zt[V8], zs[V8];
      E::unpack(vt[k], zt);
      E::unpack(vs[k], zs);
#pragma unroll
      for (int j = 0; j < V8; ++j) {
        const float dt = fmaf(zt[j], a, -Wt), ds = fmaf(zs[j], a, -Ws);
        const float et = ex2(dt), es = ex2(ds);
        sums[0] += et;
        sums[1] += es;
        sums[2] = fmaf(et, dt - ds, sums[2]);
      }
    }
  }
  block_reduce<3, false>(sums, red);
  if (threadIdx.x == 0) {
    xchg[2] = sums[0];
    xchg[3] = sums[1];
    xchg[4] = sums[2];
  }
  cluster.sync();
  float St = 0.f, Ss = 0.f, Y = 0.f;
  for (int r = 0; r < csize; ++r) {
    const float* peer = cluster.map_shared_rank(xchg, r);
    St += peer[2];
    Ss += peer[3];
    Y += peer[4];
  }
  if (crank == 0 && threadIdx.x == 0) {
    // KL = sum p_t (log p_t - log p_s) = ln2 * (Y / S_t + log2(S_s / S_t)):
    // the max shifts cancel, so only O(1) terms are combined.
    const float kl = 0.69314718055994531f * (Y / St + log2f(Ss / St));
    args.row_kl[row] = ok ? kl : __int_as_float(0x7FC00000);
  }

  // ---- pass 3: dLogits = gscale * (p_s - p_t), p = 2^(w - max w - log2 S)
  if (args.dlogits != nullptr && ok) {
    const float g = args.gscale;
    const float Lt = Wt + __log2f(St), Ls = Ws + __log2f(Ss);
    T* gout = reinterpret_cast<T*>(args.dlogits) + row * args.ld_grad + v0 - off;  // slot j -> gout[j]
    const bool vec_ok = (((uintptr_t)gout) & 15u) == 0;
    for (int k = threadIdx.x; k < nvec; k += kKlThreads) {
      float zt[V8], zs[V8], o[V8];
      E::unpack(vt[k], zt);
      E::unpack(vs[k], zs);
#pragma unroll
      for (int j = 0; j < V8; ++j) {
        const float pt = ex2(fmaf(zt[j], a, -Lt));
        const float ps = ex2(fmaf(zs[j], a, -Ls));
        o[j] = g * (ps - pt);
      }
      const int j0 = k * V8;
      if (vec_ok && j0 >= off && j0 + V8 <= nslots) {
        st_stream_v4(gout + j0, E::pack(o));
      } else {
#pragma unroll
        for (int j = 0; j < V8; ++j)
          if (j0 + j >= off && j0 + j < nslots) E::store1(gout + j0 + j, o[j]);
      }
    }
  }
  // keep this CTA's shared memory alive until every peer has read it
  cluster.sync();
}

// loss = mean of row_kl in a fixed order (double accumulation); optionally
// copies the per-row values to the caller's buffer.
__global__ void __launch_bounds__(1024) kl_mean_kernel(const float* __restrict__ row_kl, int64_t rows,
                                                       float* __restrict__ loss, float* __restrict__ row_out) {
  __shared__ double part[1024];
  double acc = 0.0;
  const int64_t per = (rows + 1023) / 1024;
  const int64_t r0 = (int64_t)threadIdx.x * per;
  for (int64_t r = r0; r < r0 + per && r < rows; ++r) {
    const float v = row_kl[r];
    acc += (double)v;
    if (row_out) row_out[r] = v;
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) *loss = rows > 0 ? (float)(part[0] / (double)rows) : 0.0f;
}

// ------------------------------------------------------------------ host

struct KlPlan {
  int cluster;
  int64_t slice;      // elements per CTA
  size_t smem;        // dynamic shared memory per CTA
};

static bool kl_plan(int64_t vocab, int esz, KlPlan& p) {
  const int vec = 16 / esz;
  const size_t soft_budget = 64 * 1024;   // two slices; lets 3 CTAs share an SM
  const size_t hard_budget = 200 * 1024;  // one CTA per SM
  for (int c = 1; c <= kKlMaxCluster; c *= 2) {
    int64_t slice = (vocab + c - 1) / c;
    slice = (slice + vec - 1) / vec * vec;
    const size_t bytes = (size_t)(slice + 2 * vec) * esz * 2;
    if (bytes <= soft_budget || (c == kKlMaxCluster && bytes <= hard_budget)) {
      p.cluster = c;
      p.slice = slice;
      p.smem = bytes;
      return true;
    }
  }
  return false;
}

template <typename T>
static cudaError_t launch_kl(const KlArgs& a, const KlPlan& p, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(kl_row_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.rows * p.cluster));
  cfg.blockDim = dim3(kKlThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kl_row_kernel<T>, a);
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t qad_kl_workspace_size(int64_t rows, int64_t vocab, nvfp4_dtype dtype) {
  (void)vocab;
  (void)dtype;
  return rows > 0 ? (size_t)((rows * sizeof(float) + 15) / 16 * 16) : 0;
}

nvfp4_status qad_kl_fwd_bwd(const void* teacher, const void* student, nvfp4_dtype dtype, int64_t rows,
                            int64_t vocab, int64_t ld, float temperature, float* loss, float* row_kl,
                            void* dlogits, int64_t ld_grad, float grad_scale, void* workspace,
                            size_t workspace_bytes, void* stream) {
  if (dtype != NVFP4_BF16 && dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  if (!(temperature > 0.0f) || !loss) return NVFP4_ERR_ARG;
  if (rows < 0 || vocab <= 0 || ld < vocab) return NVFP4_ERR_SHAPE;
  if (dlogits && ld_grad < vocab) return NVFP4_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (rows == 0) return cudaMemsetAsync(loss, 0, sizeof(float), s) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
  if (!teacher || !student) return NVFP4_ERR_ARG;
  if (rows > 0x7FFFFFFFll / kKlMaxCluster) return NVFP4_ERR_SHAPE;
  const int esz = dtype == NVFP4_BF16 ? 2 : 4;
  auto a16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  if (((uintptr_t)teacher ^ (uintptr_t)student) & 15u) return NVFP4_ERR_ALIGN;  // same alignment
  if (((uintptr_t)teacher | (uintptr_t)student) % esz) return NVFP4_ERR_ALIGN;
  if (dlogits && ((uintptr_t)dlogits % esz)) return NVFP4_ERR_ALIGN;
  const size_t need = qad_kl_workspace_size(rows, vocab, dtype);
  if (!workspace || workspace_bytes < need) return NVFP4_ERR_WORKSPACE;
  if (!a16(workspace)) return NVFP4_ERR_ALIGN;
  KlPlan plan;
  if (!kl_plan(vocab, esz, plan)) return NVFP4_ERR_UNSUPPORTED;
  KlArgs args;
  args.teacher = teacher;
  args.student = student;
  args.rows = rows;
  args.vocab = vocab;
  args.ld = ld;
  args.slice = plan.slice;
  args.a = 1.4426950408889634f / temperature;
  args.gscale = grad_scale / temperature;
  args.row_kl = reinterpret_cast<float*>(workspace);
  args.dlogits = dlogits;
  args.ld_grad = ld_grad;
  cudaError_t e = dtype == NVFP4_BF16 ? launch_kl<__nv_bfloat16>(args, plan, s) : launch_kl<float>(args, plan, s);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  kl_mean_kernel<<<1, 1024, 0, s>>>(args.row_kl, rows, loss, row_kl);
  count_launches(2);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------------------ allocation-free variant
//
// Some callers cannot allocate device memory at the point where they need the
// loss: code running inside a framework whose caching allocator already owns
// the device memory budget, callers with a fixed, pre-planned memory layout,
// and code paths where a cudaMalloc (which may synchronize the device) is not
// acceptable.  qad_kl_fwd_bwd_noalloc serves them: its per-row scratch lives
// in the file-scope array below, which every GPU that loads this library keeps
// until the process exits (kKlNoAllocMaxRows floats = 256 KiB per device).

namespace nvfp4 {

constexpr int64_t kKlNoAllocMaxRows = 65536;
static __device__ __align__(256) float g_kl_noalloc_rows[kKlNoAllocMaxRows];

// Device address of g_kl_noalloc_rows, looked up once per device.  In host
// code the array's name only stands for the symbol; the address a kernel may
// use comes from cudaGetSymbolAddress with that device current.
constexpr int kKlNoAllocMaxDevices = 64;
static void* g_kl_noalloc_ptr[kKlNoAllocMaxDevices] = {};

static nvfp4_status kl_noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (dev < 0 || dev >= kKlNoAllocMaxDevices) return NVFP4_ERR_UNSUPPORTED;
  if (g_kl_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kl_noalloc_rows) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
    g_kl_noalloc_ptr[dev] = p;
  }
  *out = g_kl_noalloc_ptr[dev];
  return NVFP4_OK;
}

}  // namespace nvfp4

extern "C" nvfp4_status qad_kl_fwd_bwd_noalloc(const void* teacher, const void* student, nvfp4_dtype dtype,
                                               int64_t rows, int64_t vocab, int64_t ld, float temperature,
                                               float* loss, float* row_kl, void* dlogits, int64_t ld_grad,
                                               float grad_scale, void* stream) {
  if (rows > nvfp4::kKlNoAllocMaxRows) return NVFP4_ERR_SHAPE;
  void* scratch = nullptr;
  nvfp4_status st = nvfp4::kl_noalloc_scratch(&scratch);
  if (st != NVFP4_OK) return st;
  // every row's slot is written before it is read, so nothing needs clearing
  return qad_kl_fwd_bwd(teacher, student, dtype, rows, vocab, ld, temperature, loss, row_kl, dlogits, ld_grad,
                        grad_scale, scratch, (size_t)nvfp4::kKlNoAllocMaxRows * sizeof(float), stream);
}
