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
//   2. one online pass over the slice keeps, per thread, running maxima of
//      both rows and the sums S_t = sum 2^d_t, S_s = sum 2^d_s and
//      Y = sum 2^d_t (d_t - d_s) relative to those maxima (rescaled when a
//      maximum grows), merged across the CTA and then pushed into every peer's
//      shared memory: one cluster barrier per row;
//   3. dLogits from the on-chip slice, 16-byte stores.
// The element arithmetic of the bf16 path uses the paired binary32
// operations of sm_100 (two logits per instruction) and the MUFU unit for
// all four exponentials per logit pair: the kernel is bound by instruction
// issue and the MUFU unit together, and a polynomial exponential on the FMA
// pipe measured slower than the MUFU one.
// Work is in the log2 domain: w = z * log2(e) / T, d = w - max w.  Per-row KL
// goes to the workspace; a second one-CTA kernel sums the rows in a fixed
// order (in double) into the mean, so the loss is deterministic.
#include <cooperative_groups.h>

#include <atomic>

#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace nvfp4 {

constexpr int kKlThreads = 256;
constexpr int kKlWarps = kKlThreads / 32;
constexpr int kKlMaxCluster = 8;
NVFP4_DEV float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for x <= 0 on the FMA and integer pipes only (no conversion
// instruction, which would share the MUFU/XU pipe): x = n + f with
// n = rint(x) taken from the low mantissa bits of x + 1.5 * 2^23, f in
// [-1/2, 1/2]; 2^f by a degree-5 polynomial (least-squares fit of 2^f on
// 2000 Chebyshev nodes of [-1/2, 1/2], coefficients rounded to binary32;
// maximum relative error 1.8e-7 over the interval); 2^n applied by adding n
// to the exponent field (the magic constant's own bits shift out of the
// 32-bit word).  x is clamped at -126 so that the result stays normal.
NVFP4_DEV float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;      // 1.5 * 2^23: rounds x to an integer in the low bits
  const float f = x - (t - 12582912.0f);
  float p = 0.0013400432653725147f;
  p = fmaf(p, f, 0.009676037356257439f);
  p = fmaf(p, f, 0.05550327152013779f);
  p = fmaf(p, f, 0.2402210682630539f);
  p = fmaf(p, f, 0.6931471824645996f);
  p = fmaf(p, f, 1.0000001192092896f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// ---- paired binary32 arithmetic (sm_100 .f32x2: two lanes per instruction,
// each rounded like the scalar operation); a pair is a 64-bit register with
// the first element in the low half.
typedef unsigned long long f32x2;

NVFP4_DEV f32x2 pair(float lo, float hi) {
  return ((f32x2)__float_as_uint(hi) << 32) | (f32x2)__float_as_uint(lo);
}
NVFP4_DEV float lo_of(f32x2 v) { return __uint_as_float((uint32_t)(v & 0xFFFFFFFFull)); }
NVFP4_DEV float hi_of(f32x2 v) { return __uint_as_float((uint32_t)(v >> 32)); }
NVFP4_DEV f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
NVFP4_DEV f32x2 add2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
NVFP4_DEV f32x2 sub2(f32x2 a, f32x2 b) {
  f32x2 r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// the two bf16 of a word (element 2i low) as a pair of floats
NVFP4_DEV f32x2 bf16x2_pair(uint32_t w) {
  return ((f32x2)(w & 0xFFFF0000u) << 32) | (f32x2)(w << 16);
}
NVFP4_DEV f32x2 ex2_pair(f32x2 x) { return pair(ex2(lo_of(x)), ex2(hi_of(x))); }

// Running softmax statistics of a (teacher, student) pair of rows, in the
// log2 domain, relative to the running maxima mt and ms:
//   St = sum 2^(w_t - mt), Ss = sum 2^(w_s - ms),
//   Y  = sum 2^(w_t - mt) ((w_t - mt) - (w_s - ms)).
struct KlStats {
  float mt, ms, St, Ss, Y;
};

// Empty statistics whose maxima sit at the pad value (scaled by a): merging
// them into real statistics scales them by 2^(pad a - max) = 0.
NVFP4_DEV void stats_init(KlStats& s, float pad_w) {
  s.mt = pad_w;
  s.ms = pad_w;
  s.St = s.Ss = s.Y = 0.f;
}

// Re-express `a` relative to new maxima (Mt, Ms) >= (a.mt, a.ms): the terms
// scale by 2^(m - M) and every d shifts by (M - m).
NVFP4_DEV void stats_rebase(KlStats& a, float Mt, float Ms) {
  const float ft = ex2(a.mt - Mt), fs = ex2(a.ms - Ms);
  const float c = (Mt - a.mt) - (Ms - a.ms);
  a.Y = ft * fmaf(-c, a.St, a.Y);
  a.St *= ft;
  a.Ss *= fs;
  a.mt = Mt;
  a.ms = Ms;
}

NVFP4_DEV KlStats stats_merge(KlStats a, KlStats b) {
  const float Mt = fmaxf(a.mt, b.mt), Ms = fmaxf(a.ms, b.ms);
  stats_rebase(a, Mt, Ms);
  stats_rebase(b, Mt, Ms);
  a.St += b.St;
  a.Ss += b.Ss;
  a.Y += b.Y;
  return a;
}

NVFP4_DEV KlStats stats_shfl_xor(const KlStats& a, int o) {
  KlStats b;
  b.mt = __shfl_xor_sync(0xFFFFFFFFu, a.mt, o);
  b.ms = __shfl_xor_sync(0xFFFFFFFFu, a.ms, o);
  b.St = __shfl_xor_sync(0xFFFFFFFFu, a.St, o);
  b.Ss = __shfl_xor_sync(0xFFFFFFFFu, a.Ss, o);
  b.Y = __shfl_xor_sync(0xFFFFFFFFu, a.Y, o);
  return b;
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
  // max of the 8 logits of a vector (exact: bf16 max on packed pairs)
  NVFP4_DEV static float vmax(const uint4& r) {
    __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&r.x);
    __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&r.y);
    __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(&r.z);
    __nv_bfloat162 d = *reinterpret_cast<const __nv_bfloat162*>(&r.w);
    __nv_bfloat162 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
    return fmaxf(__low2float(m), __high2float(m));
  }
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
  NVFP4_DEV static float vmax(const uint4& r) {
    return fmaxf(fmaxf(__uint_as_float(r.x), __uint_as_float(r.y)), fmaxf(__uint_as_float(r.z), __uint_as_float(r.w)));
  }
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
  int64_t topk;           // top-k kernel: entries of the teacher's top set per row
  const int64_t* topk_rows = nullptr;  // top-k kernel: a k per row instead (device), when set
};

// Stand-in for positions of the shared-memory slice that hold no logit (the
// alignment pad before and after the slice).  A power of two, so that its
// product with a = log2(e) / T is exact and d = fma(pad, a, -pad * a) is 0;
// it is below every logit the kernel accepts (logits must exceed -1e30), so
// it never wins a max that a real logit takes part in, and 2^(pad a - max)
// underflows to 0.
constexpr float kPadLogit = -0x1p100f;

// Geometry of a CTA's slice of one row in shared memory: slot j holds logit
// v0 + j - off for off <= j < nslots; the other slots of [0, cap) hold the
// pad value.
struct KlSliceGeom {
  int off, nslots, nvec, cap;
};

// Stages the slice [v0, v0 + n) of row `row` of the teacher and the student
// into st / ss (the teacher only when ss is null; then, on request, the
// student's interior is prefetched into L2): the 16-byte-aligned interior by
// TMA bulk copies (completion on `bar`, bounded wait; *s_ok = 0 if it
// expired), the head and tail by plain loads.  Called by every thread of the
// CTA (contains barriers).
template <typename T, int NT = kKlThreads>
NVFP4_DEV KlSliceGeom kl_stage_slice(const KlArgs& args, int64_t row, int64_t v0, int n, T* st, T* ss,
                                     uint64_t* bar_, int* s_ok_, bool prefetch_student = false) {
  using E = KlElem<T>;
  constexpr int V8 = E::kVec;
  constexpr int ESZ = (int)sizeof(T);
  uint64_t& bar = *bar_;
  int& s_ok = *s_ok_;
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

  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    s_ok = 1;
  }
  __syncthreads();
  if (threadIdx.x == 0 && nint > 0) {
    mbar_expect_tx(&bar, (uint32_t)((ss != nullptr ? 2 : 1) * nint * ESZ));
    bulk_g2s(st + off + head, gt + head, (uint32_t)(nint * ESZ), &bar);
    if (ss != nullptr) bulk_g2s(ss + off + head, gs + head, (uint32_t)(nint * ESZ), &bar);
    if (ss == nullptr && prefetch_student) bulk_prefetch_l2(gs + head, (uint32_t)(nint * ESZ));
  }
  // head and tail logits with plain loads, pad slots with the pad value; all
  // disjoint from the bulk-copied interior [off + head, off + tail0)
  for (int j = threadIdx.x; j < off + head; j += NT) {  // pad, then head
    const int i = j - off;
    if (i < 0) {
      E::store1(st + j, kPadLogit);
      if (ss != nullptr) E::store1(ss + j, kPadLogit);
    } else {
      st[j] = gt[i];
      if (ss != nullptr) ss[j] = gs[i];
    }
  }
  for (int j = off + tail0 + threadIdx.x; j < cap; j += NT) {  // tail, then pad
    const int i = j - off;
    if (i < n) {
      st[j] = gt[i];
      if (ss != nullptr) ss[j] = gs[i];
    } else {
      E::store1(st + j, kPadLogit);
      if (ss != nullptr) E::store1(ss + j, kPadLogit);
    }
  }
  if (nint > 0 && !mbar_wait_bounded(&bar, 0)) s_ok = 0;
  __syncthreads();

  KlSliceGeom g;
  g.off = off;
  g.nslots = nslots;
  g.nvec = nvec;
  g.cap = cap;
  return g;
}

template <typename T>
__global__ void __launch_bounds__(kKlThreads, 6) kl_row_kernel(KlArgs args) {
  using E = KlElem<T>;
  constexpr int V8 = E::kVec;        // elements per 16-byte vector
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint64_t bar;
  __shared__ float warp_max[2][kKlWarps];
  __shared__ float warp_sum[3][kKlWarps];
  __shared__ KlStats peer_stats[kKlMaxCluster];  // written by every CTA of the cluster
  __shared__ int s_ok;

  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int64_t row = blockIdx.x / csize;
  const int64_t v0 = (int64_t)crank * args.slice;
  int64_t v1 = v0 + args.slice;
  if (v1 > args.vocab) v1 = args.vocab;
  const int n = v1 > v0 ? (int)(v1 - v0) : 0;

  // The teacher slice is staged in shared memory; the student slice is
  // prefetched into L2 and read from global memory in both passes (slot j
  // holds logit v0 + j - off of the row), which halves the shared memory of
  // a CTA and so doubles the CTAs an SM holds.
  T* st = reinterpret_cast<T*>(smem_raw);
  const T* gs = reinterpret_cast<const T*>(args.student) + row * args.ld + v0;
  const KlSliceGeom geo = kl_stage_slice<T>(args, row, v0, n, st, nullptr, &bar, &s_ok, true);
  const int off = geo.off, nslots = geo.nslots, nvec = geo.nvec;
  const bool ok = s_ok != 0;
  const int kfirst = (off + V8 - 1) / V8;  // vectors [kfirst, klast) hold no pad slot
  const int klast = nslots / V8;

  const uint4* vt = reinterpret_cast<const uint4*>(st);
  // the student's vector k, pad value outside the slice; interior vectors are
  // 16-byte aligned in global memory as in shared memory
  auto svec = [&](int k) -> uint4 {
    if (k >= kfirst && k < klast) return __ldg(reinterpret_cast<const uint4*>(gs + (k * V8 - off)));
    float z[V8];
#pragma unroll
    for (int e = 0; e < V8; ++e) {
      const int j = k * V8 + e;
      z[e] = (j >= off && j < nslots) ? E::load1(gs + (j - off)) : kPadLogit;
    }
    return E::pack(z);
  };
  const float a = args.a;  // log2(e) / T > 0

  // ---- online statistics over this thread's vectors; the running maxima are
  // kept on the raw logits (a > 0, so max w = a * max z) and d = z a - max w
  // is one FMA
  KlStats my;
  stats_init(my, kPadLogit * a);
  float zmt = kPadLogit, zms = kPadLogit;  // running max of the raw logits
  if (ok) {
    for (int k = threadIdx.x; k < nvec; k += kKlThreads) {
      const uint4 rt = vt[k], rs = svec(k);
      const float lt = E::vmax(rt), ls = E::vmax(rs);
      if (lt > zmt || ls > zms) {
        zmt = fmaxf(zmt, lt);
        zms = fmaxf(zms, ls);
        stats_rebase(my, zmt * a, zms * a);
      }
      const float nMt = -my.mt, nMs = -my.ms;
      if constexpr (sizeof(T) == 2) {
        // two logits of each row per paired operation; the pair sums are
        // folded into the thread's statistics once per vector
        const uint32_t wt[4] = {rt.x, rt.y, rt.z, rt.w}, ws[4] = {rs.x, rs.y, rs.z, rs.w};
        const f32x2 A = pair(a, a), NT = pair(nMt, nMt), NS = pair(nMs, nMs);
        f32x2 St2 = 0ull, Ss2 = 0ull, Y2 = 0ull;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const f32x2 dt = fma2(bf16x2_pair(wt[j]), A, NT), ds = fma2(bf16x2_pair(ws[j]), A, NS);
          const f32x2 et = ex2_pair(dt), es = ex2_pair(ds);
          St2 = add2(St2, et);
          Ss2 = add2(Ss2, es);
          Y2 = fma2(et, sub2(dt, ds), Y2);
        }
        my.St += lo_of(St2) + hi_of(St2);
        my.Ss += lo_of(Ss2) + hi_of(Ss2);
        my.Y += lo_of(Y2) + hi_of(Y2);
      } else {
        float zt[V8], zs[V8];
        E::unpack(rt, zt);
        E::unpack(rs, zs);
#pragma unroll
        for (int j = 0; j < V8; ++j) {
          const float dt = fmaf(zt[j], a, nMt), ds = fmaf(zs[j], a, nMs);
          const float et = ex2(dt), es = ex2(ds);
          my.St += et;
          my.Ss += es;
          my.Y = fmaf(et, dt - ds, my.Y);
        }
      }
    }
  }
  // ---- merge over the CTA, then push to every CTA of the cluster: the CTA's
  // maxima first (a max butterfly, no exponentials), then every thread
  // rebases its sums to them once and the sums are added by a butterfly and
  // in warp order
  {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    float Mt = my.mt, Ms = my.ms;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Mt = fmaxf(Mt, __shfl_xor_sync(0xFFFFFFFFu, Mt, o));
      Ms = fmaxf(Ms, __shfl_xor_sync(0xFFFFFFFFu, Ms, o));
    }
    if (lane == 0) {
      warp_max[0][wid] = Mt;
      warp_max[1][wid] = Ms;
    }
    __syncthreads();
    Mt = warp_max[0][0];
    Ms = warp_max[1][0];
#pragma unroll
    for (int w = 1; w < kKlWarps; ++w) {
      Mt = fmaxf(Mt, warp_max[0][w]);
      Ms = fmaxf(Ms, warp_max[1][w]);
    }
    stats_rebase(my, Mt, Ms);
    float sum_t = my.St, sum_s = my.Ss, sum_y = my.Y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sum_t += __shfl_xor_sync(0xFFFFFFFFu, sum_t, o);
      sum_s += __shfl_xor_sync(0xFFFFFFFFu, sum_s, o);
      sum_y += __shfl_xor_sync(0xFFFFFFFFu, sum_y, o);
    }
    if (lane == 0) {
      warp_sum[0][wid] = sum_t;
      warp_sum[1][wid] = sum_s;
      warp_sum[2][wid] = sum_y;
    }
    __syncthreads();
    if ((int)threadIdx.x < csize) {
      KlStats c;
      c.mt = Mt;
      c.ms = Ms;
      c.St = c.Ss = c.Y = 0.f;
      for (int w = 0; w < kKlWarps; ++w) {
        c.St += warp_sum[0][w];
        c.Ss += warp_sum[1][w];
        c.Y += warp_sum[2][w];
      }
      cluster.map_shared_rank(peer_stats, (int)threadIdx.x)[crank] = c;
    }
  }
  cluster.sync();  // all pushes visible; no CTA reads a peer after this point
  __shared__ KlStats row_stats_sh;
  if (threadIdx.x == 0) {  // one thread merges the peers (in rank order) for the whole CTA
    KlStats m = peer_stats[0];
    for (int r = 1; r < csize; ++r) m = stats_merge(m, peer_stats[r]);
    row_stats_sh = m;
  }
  __syncthreads();
  const KlStats row_stats = row_stats_sh;
  const float Wt = row_stats.mt, Ws = row_stats.ms, St = row_stats.St, Ss = row_stats.Ss;
  if (crank == 0 && threadIdx.x == 0) {
    // KL = sum p_t (log p_t - log p_s) = ln2 * (Y / S_t + log2(S_s / S_t))
    const float kl = 0.69314718055994531f * (row_stats.Y / St + log2f(Ss / St));
    args.row_kl[row] = ok ? kl : __int_as_float(0x7FC00000);
  }

  // ---- dLogits = gscale * (p_s - p_t), p = 2^(w - max w - log2 S); for
  // gscale > 0 the factor goes into the exponent: g p = 2^(w - L + log2 g)
  if (args.dlogits != nullptr && ok) {
    const float g = args.gscale;
    const bool fold = g > 0.0f;
    const float lg = fold ? __log2f(g) : 0.0f;
    const float Lt = Wt + __log2f(St) - lg, Ls = Ws + __log2f(Ss) - lg;
    const float gm = fold ? 1.0f : g;
    T* gout = reinterpret_cast<T*>(args.dlogits) + row * args.ld_grad + v0 - off;  // slot j -> gout[j]
    const bool vec_ok = (((uintptr_t)gout) & 15u) == 0;
    for (int k = threadIdx.x; k < nvec; k += kKlThreads) {
      float o[V8];
      if constexpr (sizeof(T) == 2) {
        const uint4 rt = vt[k], rs = svec(k);
        const uint32_t wt[4] = {rt.x, rt.y, rt.z, rt.w}, ws[4] = {rs.x, rs.y, rs.z, rs.w};
        const f32x2 A = pair(a, a), NLt = pair(-Lt, -Lt), NLs = pair(-Ls, -Ls), G = pair(gm, gm);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const f32x2 pt = ex2_pair(fma2(bf16x2_pair(wt[j]), A, NLt));
          const f32x2 ps = ex2_pair(fma2(bf16x2_pair(ws[j]), A, NLs));
          f32x2 d = sub2(ps, pt);
          if (!fold) d = fma2(d, G, 0ull);
          o[2 * j] = lo_of(d);
          o[2 * j + 1] = hi_of(d);
        }
      } else {
        float zt[V8], zs[V8];
        E::unpack(vt[k], zt);
        E::unpack(svec(k), zs);
#pragma unroll
        for (int j = 0; j < V8; ++j) {
          const float pt = exp2_poly(fmaf(zt[j], a, -Lt));
          const float ps = ex2(fmaf(zs[j], a, -Ls));
          o[j] = fold ? ps - pt : gm * (ps - pt);
        }
      }
      const int j0 = k * V8;
      if (vec_ok && k >= kfirst && k < klast) {
        st_stream_v4(gout + j0, E::pack(o));
      } else {
#pragma unroll
        for (int j = 0; j < V8; ++j)
          if (j0 + j >= off && j0 + j < nslots) E::store1(gout + j0 + j, o[j]);
      }
    }
  }
}

// ------------------------------------------------------------------ top-k KL
//
// The distillation loss restricted to the teacher's top-k vocabulary entries
// of each row (Qwen3.6-35B-A3B W4A4 tutorial, section "3. QAD":
// --logit_kl_topk 4096), both softmaxes renormalised over that set S, ties
// broken by the smaller vocabulary index; the gradient is zero outside S.
// Same cluster-per-row layout as kl_row_kernel.  S is found by a radix
// select over order-preserving integer keys of the teacher logits held in
// shared memory: one digit per pass (9 + 7 bits for bf16, 4 x 8 for f32),
// each pass a CTA histogram (shared-memory atomics) summed over the
// cluster through distributed shared memory; that yields the k-th key tau
// and how many keys equal to tau belong to S.  The last pass's per-CTA
// counts of keys equal to tau give, in rank order, how many of them each
// CTA contributes; the one CTA where that number is neither none nor all
// ranks its own in index order.  The statistics and the gradient then run
// over S only.

template <typename T>
struct KlKey;
template <>
struct KlKey<__nv_bfloat16> {
  static constexpr int kBits = 16;
  static constexpr int kPerWord = 2;
  NVFP4_DEV static uint32_t key(uint32_t w, int h) {  // element h of a 32-bit word
    const uint32_t u = h ? (w >> 16) : (w & 0xFFFFu);
    return (u & 0x8000u) ? (~u & 0xFFFFu) : (u | 0x8000u);
  }
};
// Both order-preserving keys of a word of two bf16 (element 0 in the low
// half): positive values get the sign bit set, negative ones all 16 bits
// flipped -- the same map as KlKey<__nv_bfloat16>::key, two at a time.
NVFP4_DEV uint32_t bf16x2_keys(uint32_t w) {
  const uint32_t m = ((w >> 15) & 0x00010001u) * 0xFFFFu;  // 0xFFFF in each half whose sign is set
  return w ^ (m | 0x80008000u);
}

template <>
struct KlKey<float> {
  static constexpr int kBits = 32;
  static constexpr int kPerWord = 1;
  NVFP4_DEV static uint32_t key(uint32_t w, int) { return (w & 0x80000000u) ? ~w : (w | 0x80000000u); }
};

// bf16 keys are selected in two digits of 9 and 7 bits; the first digit is
// the sign and exponent, so its bucket at the k-th key holds one binade.  The
// first pass also keeps each 16-byte vector's largest key, so that the
// second digit and the final selection read only the vectors that can hold a
// key of the bucket (or of S): each warp lists those of its vectors with a
// ballot and works through the list with all lanes.  f32 keys take four
// 8-bit digits over the whole slice.
constexpr int kTopkThreads = 256;
constexpr int kTopkWarps = kTopkThreads / 32;

// The digit whose bucket holds the remaining-th largest key of a histogram
// of `bins` counts (cluster totals in hist): an inclusive scan of the
// bucket counts from the largest digit down over the CTA's threads
// (kTopkThreads, each owning bins / kTopkThreads or one bucket).  Every
// thread returns (digit, keys to take from its bucket, keys in its bucket).
NVFP4_DEV void topk_find_digit(const unsigned* hist, int bins, unsigned remaining, unsigned* warp_tot,
                               unsigned* s_digit, unsigned* s_remaining, unsigned* s_count) {
  const int t = (int)threadIdx.x, lane = t & 31, wid = t >> 5;
  const int per = bins > kTopkThreads ? bins / kTopkThreads : 1;
  const int b_hi = bins - 1 - t * per;  // this thread's buckets: b_hi, b_hi - 1, ..., b_hi - per + 1
  unsigned mine = 0u;
  if (b_hi >= 0)
    for (int i = 0; i < per; ++i) mine += hist[b_hi - i];
  unsigned x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  unsigned before = x - mine;
  for (int w = 0; w < wid; ++w) before += warp_tot[w];
  if (b_hi >= 0 && before < remaining && remaining <= before + mine) {
    unsigned cum = before;
    for (int i = 0; i < per; ++i) {
      const int b = b_hi - i;
      if (cum + hist[b] >= remaining) {
        *s_digit = (unsigned)b;
        *s_remaining = remaining - cum;
        *s_count = hist[b];
        break;
      }
      cum += hist[b];
    }
  }
  __syncthreads();
}

// Sums the CTA histograms (hist[0..bins)) over the cluster: every CTA pushes
// its counts into slot crank of each peer's rbuf ([csize][stride], 16-byte
// vectors), then, after the cluster barrier, adds the csize rows into hist.
// rbuf keeps the per-CTA rows.
NVFP4_DEV void topk_cluster_hist(cg::cluster_group& cluster, unsigned* hist, unsigned* rbuf, int stride, int bins,
                                 int csize, int crank) {
  const int q4 = bins / 4;
  const uint4* h4 = reinterpret_cast<const uint4*>(hist);
  for (int i = (int)threadIdx.x; i < csize * q4; i += kTopkThreads) {
    const int r = i / q4, b4 = i - r * q4;
    reinterpret_cast<uint4*>(cluster.map_shared_rank(rbuf, r) + crank * stride)[b4] = h4[b4];
  }
  cluster.sync();
  for (int b = (int)threadIdx.x; b < bins; b += kTopkThreads) {
    unsigned tot = 0u;
    for (int r = 0; r < csize; ++r) tot += rbuf[r * stride + b];
    hist[b] = tot;
  }
  __syncthreads();
}

// Appends to this warp's list (list[kw0 ...], in index order) its vectors k
// in [kw0, kw0 + W) with pred(k); returns the list length.  Warp-uniform.
template <typename P>
NVFP4_DEV unsigned topk_warp_list(unsigned* list, int kw0, int W, int nvec, P pred) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  unsigned len = 0u;
  for (int kb = kw0; kb < kw0 + W && kb < nvec; kb += 32) {
    const int k = kb + lane;
    const bool in = k < nvec && k < kw0 + W && pred(k);
    const unsigned b = __ballot_sync(0xFFFFFFFFu, in);
    if (in) list[kw0 + len + __popc(b & lt_mask)] = (unsigned)k;
    len += __popc(b);
  }
  __syncwarp();
  return len;
}

template <typename T>
__global__ void __launch_bounds__(kTopkThreads) kl_topk_row_kernel(KlArgs args) {
  using E = KlElem<T>;
  using Kf = KlKey<T>;
  constexpr int V8 = E::kVec;
  constexpr bool BF = sizeof(T) == 2;
  constexpr int PASSES = BF ? 2 : 4;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint64_t bar;
  __shared__ int s_ok;
  __shared__ __align__(16) unsigned hist[512];
  // cluster exchange of the histograms: one buffer per pass parity, written
  // by every CTA of the cluster; the even passes' buffer (512 counts per
  // CTA) lies over the vector lists and the selection mask, which are not in
  // use before the second digit
  __shared__ __align__(16) unsigned recv_b[kKlMaxCluster][256];
  __shared__ unsigned warp_sum[kTopkWarps];
  __shared__ unsigned s_digit, s_remaining, s_count;
  __shared__ KlStats warp_stats[kTopkWarps];
  __shared__ KlStats peer_stats[kKlMaxCluster];

  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int64_t row = blockIdx.x / csize;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t v0 = (int64_t)crank * args.slice;
  int64_t v1 = v0 + args.slice;
  if (v1 > args.vocab) v1 = args.vocab;
  const int n = v1 > v0 ? (int)(v1 - v0) : 0;

  // Only the teacher slice is staged; the few student logits of S are read
  // from global memory (slot j holds logit v0 + j - off of the row).
  T* st = reinterpret_cast<T*>(smem_raw);
  const T* gs = reinterpret_cast<const T*>(args.student) + row * args.ld + v0;
  const int nvec_max = (int)((args.slice + 2 * V8) / V8);
  // bf16: largest valid key of each vector (0 when it has none)
  uint16_t* vmax = reinterpret_cast<uint16_t*>(st + args.slice + 2 * V8);
  unsigned* vlist = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(vmax) + (nvec_max * 2 + 15) / 16 * 16);
  uint8_t* sel_mask = reinterpret_cast<uint8_t*>(vlist + nvec_max);  // bit e: element e of the vector is in S
  unsigned* recv_a = vlist;                                          // [csize][512], first digit only
  // the student's slice is prefetched into L2: the statistics and gradient
  // passes read the vectors holding members of S, which cover most of its lines
  const KlSliceGeom geo = kl_stage_slice<T, kTopkThreads>(args, row, v0, n, st, nullptr, &bar, &s_ok, true);
  const int off = geo.off, nslots = geo.nslots, nvec = geo.nvec;
  const int kfirst = (off + V8 - 1) / V8;  // vectors [kfirst, klast) hold no pad slot
  const int klast = nslots / V8;
  const bool ok = s_ok != 0;
  const uint32_t* wt = reinterpret_cast<const uint32_t*>(st);  // words of the teacher slice
  const uint4* vt = reinterpret_cast<const uint4*>(st);
  constexpr int WPV = 16 / 4;                                   // words per 16-byte vector
  // Warp w owns vectors [w W, (w + 1) W) for its lists, so that index order
  // is (warp, list position) order.
  const int W = ((nvec + kTopkWarps - 1) / kTopkWarps + 31) / 32 * 32;
  const int kw0 = wid * W;

  // ---- radix select of the k-th largest key over the row
  int64_t kreq = args.topk_rows != nullptr ? args.topk_rows[row] : args.topk;
  if (kreq < 1) kreq = 1;
  const uint32_t kk = (uint32_t)(kreq < args.vocab ? kreq : args.vocab);
  uint32_t prefix = 0, remaining = kk;
  for (int p = 0; p < PASSES; ++p) {
    // digit p: bf16 bits [15:7] then [6:0]; f32 8 bits at a time from the top
    const int dbits = BF ? (p == 0 ? 9 : 7) : 8;
    const int shift = BF ? (p == 0 ? 7 : 0) : Kf::kBits - 8 * (p + 1);
    const int bins = 1 << dbits;
    for (int b = (int)threadIdx.x; b < bins; b += kTopkThreads) hist[b] = 0u;
    __syncthreads();
    if (BF && p == 1) {
      // the vectors whose largest key reaches bucket `prefix`; keys outside
      // the bucket are counted in a lane's own spare bin (128 + lane), so
      // that every lane adds and no two lanes collide there
      const uint32_t base = prefix << 7;
      const unsigned len =
          topk_warp_list(vlist, kw0, W, nvec, [&](int k) { return ok && (uint32_t)vmax[k] >= base; });
      for (unsigned i = lane; i < len; i += 32) {
        const int k = (int)vlist[kw0 + i];
        const uint4 v = vt[k];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
        const bool interior = k >= kfirst && k < klast;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t k2 = bf16x2_keys(w4[q]);
          const int j0 = k * V8 + 2 * q;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t key = h ? (k2 >> 16) : (k2 & 0xFFFFu);
            const bool in = (key >> 7) == prefix && (interior || (j0 + h >= off && j0 + h < nslots));
            atomicAdd(&hist[in ? (key & 0x7Fu) : 128u + (unsigned)lane], 1u);
          }
        }
      }
    } else if (ok) {
      for (int k = (int)threadIdx.x; k < nvec; k += kTopkThreads) {
        if (BF && k >= kfirst && k < klast) {  // interior bf16 vector, first digit: every key counts
          const uint4 v = vt[k];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t k2 = bf16x2_keys(w4[q]);
            atomicAdd(&hist[(k2 & 0xFFFFu) >> 7], 1u);
            atomicAdd(&hist[k2 >> 23], 1u);
          }
          const uint32_t m = __vmaxu2(__vmaxu2(bf16x2_keys(w4[0]), bf16x2_keys(w4[1])),
                                      __vmaxu2(bf16x2_keys(w4[2]), bf16x2_keys(w4[3])));
          vmax[k] = (uint16_t)max(m & 0xFFFFu, m >> 16);
          continue;
        }
        // edge vectors (and f32): one key at a time
        uint32_t vm = 0u;
#pragma unroll
        for (int q = 0; q < WPV; ++q) {
          const uint32_t w = wt[k * WPV + q];
#pragma unroll
          for (int h = 0; h < Kf::kPerWord; ++h) {
            const int j = k * V8 + q * Kf::kPerWord + h;  // slot
            const uint32_t key = Kf::key(w, h);
            const bool in_slice = j >= off && j < nslots;
            if (in_slice) vm = max(vm, key);
            if (in_slice && (p == 0 || (key >> (shift + dbits)) == prefix))
              atomicAdd(&hist[(key >> shift) & (uint32_t)(bins - 1)], 1u);
          }
        }
        if (BF && p == 0) vmax[k] = (uint16_t)vm;
      }
    }
    __syncthreads();
    // the cluster's totals (the buffers alternate, so that no CTA writes a
    // peer's buffer of the previous digit while that peer still reads it)
    if (p & 1)
      topk_cluster_hist(cluster, hist, &recv_b[0][0], 256, bins, csize, crank);
    else
      topk_cluster_hist(cluster, hist, recv_a, 512, bins, csize, crank);
    topk_find_digit(hist, bins, remaining, warp_sum, &s_digit, &s_remaining, &s_count);
    prefix = (prefix << dbits) | s_digit;
    remaining = s_remaining;  // keys equal to the prefix so far still to take
    __syncthreads();          // hist, s_* are rewritten by the next pass
  }
  const uint32_t tau = prefix;
  const uint32_t m_ties = remaining;  // keys == tau that belong to S

  // ---- this CTA's share of the ties: the last digit's per-CTA counts (the
  // odd passes' buffer, last written in the final pass) in rank order
  const unsigned last_digit = BF ? (tau & 0x7Fu) : (tau & 0xFFu);
  unsigned cta_off = 0u;
  for (int r = 0; r < crank; ++r) cta_off += recv_b[r][last_digit];
  const unsigned n_mine = recv_b[crank][last_digit];
  const unsigned take = m_ties > cta_off ? min(m_ties - cta_off, n_mine) : 0u;

  // ---- the vectors that can hold a key of S (bf16: largest key >= tau)
  unsigned len = topk_warp_list(vlist, kw0, W, nvec, [&](int k) {
    sel_mask[k] = 0u;
    return ok && (!BF || (uint32_t)vmax[k] >= tau);
  });
  // ---- their selection masks.  Keys above tau are in S; keys equal to tau
  // are when this CTA takes all of its ties, none when it takes none, and in
  // the one CTA that takes some of them (CTA-uniform), the first `take` in
  // index order: a first pass keeps each listed vector's tie bits in its list
  // entry (bits 24..31; vector indices stay below 2^16), a scan over the warps
  // gives each warp's first rank, and a second pass adds the ties below
  // `take`.  Either way the list ends up holding (in place, in order) the
  // vectors with a selected element.
  const bool split_ties = take != 0u && take != n_mine;
  const bool all_ties = take == n_mine;
  const unsigned lt_mask = (1u << lane) - 1u;
  unsigned list_len = 0u, ties_before = 0u;
  for (unsigned ib = 0; ib < len; ib += 32) {  // warp-uniform trip count
    const unsigned i = ib + lane;
    const int k = i < len ? (int)vlist[kw0 + i] : -1;
    unsigned gt = 0u, eq = 0u;
    if (k >= 0) {
      const uint4 v = vt[k];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      if (BF && k >= kfirst && k < klast) {
#pragma unroll
        for (int q = 0; q < WPV; ++q) {
          const uint32_t k2 = bf16x2_keys(w4[q]);
          const uint32_t k0 = k2 & 0xFFFFu, k1 = k2 >> 16;
          gt |= ((k0 > tau ? 1u : 0u) | (k1 > tau ? 2u : 0u)) << (2 * q);
          eq |= ((k0 == tau ? 1u : 0u) | (k1 == tau ? 2u : 0u)) << (2 * q);
        }
      } else {
#pragma unroll
        for (int q = 0; q < WPV; ++q)
#pragma unroll
          for (int h = 0; h < Kf::kPerWord; ++h) {
            const int e = q * Kf::kPerWord + h;
            const int j = k * V8 + e;
            const uint32_t key = Kf::key(w4[q], h);
            const bool valid = j >= off && j < nslots;
            gt |= (valid && key > tau ? 1u : 0u) << e;
            eq |= (valid && key == tau ? 1u : 0u) << e;
          }
      }
    }
    if (split_ties) {
      if (k >= 0) {
        sel_mask[k] = (uint8_t)gt;
        vlist[kw0 + i] = (unsigned)k | (eq << 24);
      }
      ties_before += __reduce_add_sync(0xFFFFFFFFu, (unsigned)__popc(eq));
    } else {
      const unsigned mask = gt | (all_ties ? eq : 0u);
      if (k >= 0) sel_mask[k] = (uint8_t)mask;
      const unsigned b = __ballot_sync(0xFFFFFFFFu, mask != 0u);  // every lane has read its entry
      if (mask != 0u) vlist[kw0 + list_len + __popc(b & lt_mask)] = (unsigned)k;
      list_len += __popc(b);
    }
  }
  if (split_ties) {  // CTA-uniform
    if (lane == 0) warp_sum[wid] = ties_before;
    __syncthreads();
    unsigned rank = 0u;  // ties of this CTA in the warps before this one
    for (int w = 0; w < wid; ++w) rank += warp_sum[w];
    for (unsigned ib = 0; ib < len; ib += 32) {
      const unsigned i = ib + lane;
      const unsigned entry = i < len ? vlist[kw0 + i] : 0u;
      const int k = i < len ? (int)(entry & 0xFFFFFFu) : -1;
      unsigned eq = entry >> 24;
      const unsigned c = (unsigned)__popc(eq);
      unsigned x = c;  // inclusive scan of the tie counts over the lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xFFFFFFFFu, x, o);
        if (lane >= o) x += y;
      }
      const unsigned first = rank + x - c;  // rank of this vector's first tie
      unsigned mask = 0u;
      if (k >= 0) {
        mask = sel_mask[k];
        for (unsigned r = first; r < take && eq != 0u; ++r) {  // its ties ranked below `take`
          mask |= eq & (0u - eq);
          eq &= eq - 1u;
        }
        sel_mask[k] = (uint8_t)mask;
      }
      rank += __shfl_sync(0xFFFFFFFFu, x, 31);
      const unsigned b = __ballot_sync(0xFFFFFFFFu, mask != 0u);  // every lane has read its entry
      if (mask != 0u) vlist[kw0 + list_len + __popc(b & lt_mask)] = (unsigned)k;
      list_len += __popc(b);
    }
  }
  unsigned* sel_list = vlist;
  __syncthreads();
  // ---- online statistics over S (other slots read as the pad value)
  // the student's vector k (pad value outside the slice); interior vectors
  // are 16-byte aligned in global memory as in shared memory
  auto student_vec = [&](int k, float (&zs)[V8]) {
    if (k >= kfirst && k < klast) {
      E::unpack(__ldg(reinterpret_cast<const uint4*>(gs + (k * V8 - off))), zs);
    } else {
#pragma unroll
      for (int e = 0; e < V8; ++e) {
        const int j = k * V8 + e;
        zs[e] = (j >= off && j < nslots) ? E::load1(gs + (j - off)) : kPadLogit;
      }
    }
  };
  const float a = args.a;
  KlStats my;
  stats_init(my, kPadLogit * a);
  float zmt = kPadLogit, zms = kPadLogit;
  if (ok) {
    for (unsigned i = lane; i < list_len; i += 32) {  // only this warp's vectors with a selected element
      const int k = (int)sel_list[kw0 + i];
      const unsigned mask = sel_mask[k];
      float zt[V8], zs[V8];
      E::unpack(vt[k], zt);
      student_vec(k, zs);
      float lt = kPadLogit, ls = kPadLogit;
#pragma unroll
      for (int e = 0; e < V8; ++e) {
        if (!((mask >> e) & 1u)) {
          zt[e] = kPadLogit;
          zs[e] = kPadLogit;
        }
        lt = fmaxf(lt, zt[e]);
        ls = fmaxf(ls, zs[e]);
      }
      if (lt > zmt || ls > zms) {
        zmt = fmaxf(zmt, lt);
        zms = fmaxf(zms, ls);
        stats_rebase(my, zmt * a, zms * a);
      }
      const float nMt = -my.mt, nMs = -my.ms;
#pragma unroll
      for (int e = 0; e < V8; ++e) {
        const float dt = fmaf(zt[e], a, nMt), ds = fmaf(zs[e], a, nMs);
        const float et = ex2(dt), es = ex2(ds);
        my.St += et;
        my.Ss += es;
        my.Y = fmaf(et, dt - ds, my.Y);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) my = stats_merge(my, stats_shfl_xor(my, o));
  if (lane == 0) warp_stats[wid] = my;
  __syncthreads();
  if (threadIdx.x < csize) {
    KlStats c = warp_stats[0];
    for (int w = 1; w < kTopkWarps; ++w) c = stats_merge(c, warp_stats[w]);
    cluster.map_shared_rank(peer_stats, (int)threadIdx.x)[crank] = c;
  }
  cluster.sync();  // all pushes visible; no CTA touches a peer after this point
  KlStats rs_ = peer_stats[0];
  for (int r = 1; r < csize; ++r) rs_ = stats_merge(rs_, peer_stats[r]);
  const float Wt = rs_.mt, Ws = rs_.ms, St = rs_.St, Ss = rs_.Ss;
  if (crank == 0 && threadIdx.x == 0) {
    const float kl = 0.69314718055994531f * (rs_.Y / St + log2f(Ss / St));
    args.row_kl[row] = ok ? kl : __int_as_float(0x7FC00000);
  }

  // ---- dLogits: gscale (p_s^S - p_t^S) on S, 0 elsewhere
  if (args.dlogits != nullptr && ok) {
    const float g = args.gscale;
    const float Lt = Wt + __log2f(St), Ls = Ws + __log2f(Ss);
    T* gout = reinterpret_cast<T*>(args.dlogits) + row * args.ld_grad + v0 - off;  // slot j -> gout[j]
    const bool vec_ok = (((uintptr_t)gout) & 15u) == 0;
    auto store_vec = [&](int k, const float (&o)[V8]) {
      const int j0 = k * V8;
      if (vec_ok && k >= kfirst && k < klast) {
        st_stream_v4(gout + j0, E::pack(o));
      } else {
#pragma unroll
        for (int e = 0; e < V8; ++e)
          if (j0 + e >= off && j0 + e < nslots) E::store1(gout + j0 + e, o[e]);
      }
    };
    // vectors with a selected element: this warp's list
    for (unsigned i = lane; i < list_len; i += 32) {
      const int k = (int)sel_list[kw0 + i];
      const unsigned mask = sel_mask[k];
      float zt[V8], zs[V8], o[V8];
      E::unpack(vt[k], zt);
      student_vec(k, zs);
#pragma unroll
      for (int e = 0; e < V8; ++e) {
        const float pt = ex2(fmaf(zt[e], a, -Lt)), ps = ex2(fmaf(zs[e], a, -Ls));
        o[e] = ((mask >> e) & 1u) ? g * (ps - pt) : 0.0f;
      }
      store_vec(k, o);
    }
    // the rest: zeros
    for (int k = (int)threadIdx.x; k < nvec; k += kTopkThreads) {
      if (sel_mask[k] != 0u) continue;
      float o[V8];
#pragma unroll
      for (int e = 0; e < V8; ++e) o[e] = 0.0f;
      store_vec(k, o);
    }
  }
}

// ------------------------------------------------------------------ top-p set size
//
// The Qwen3.6-35B-A3B W4A4 tutorial (section "5. 评估", on the runs that hit
// the output-length cap) suggests selecting the teacher's top-p entries
// instead of the top-k ones.  Per row, S is the shortest prefix of the top-k
// order (decreasing teacher logit, equal logits by smaller index) whose
// teacher probability at temperature T reaches p; the loss over S is the
// top-k loss with k = |S|.  kl_topp_count_kernel finds |S| for every row with
// the top-k kernel's cluster layout (teacher slice staged; the student is not
// read) and a radix select over the same keys in which a bucket counts
// teacher probability mass instead of entries.  The mass of a logit is
// 2^((z - max z) a) in fixed point (2^40 for the largest logit), summed as
// integers, so that the sums, and therefore the chosen set, do not depend on
// the order of the additions.  A CTA's bucket sums are kept as two 32-bit
// words (low word by a 32-bit atomic that returns the old value, the carry
// and the high bits of the mass by a second, rare one); the cluster sums are
// 64-bit.

constexpr float kToppScale = 0x1p40f;

// the logit whose order-preserving key is `key` (inverse of KlKey<T>::key)
template <typename T>
NVFP4_DEV float topp_key_value(uint32_t key);
template <>
NVFP4_DEV float topp_key_value<__nv_bfloat16>(uint32_t key) {
  const uint32_t u = (key & 0x8000u) ? (key & 0x7FFFu) : (~key & 0xFFFFu);
  return __uint_as_float(u << 16);
}
template <>
NVFP4_DEV float topp_key_value<float>(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// fixed-point teacher mass of a logit, mw = a * (largest logit)
NVFP4_DEV unsigned long long topp_mass(float z, float a, float mw) {
  return (unsigned long long)__float2ull_rn(ex2(fmaf(z, a, -mw)) * kToppScale);
}

constexpr int kToppThreads = 512;  // two CTAs of 16 warps per SM (64 registers a thread)
constexpr int kToppWarps = kToppThreads / 32;

// The bucket (largest digit first) in which the cumulative mass reaches
// `need` >= 1: thread t owns bins / kToppThreads buckets (or one) from the
// top; returns through s_* the digit and the mass of the buckets above it,
// and s_found = 0 when the buckets together hold less than `need`.
NVFP4_DEV void topp_find_bucket(const unsigned long long* hm, int bins, unsigned long long need,
                                unsigned long long* warp_m, unsigned* s_digit, unsigned long long* s_before_m,
                                int* s_found) {
  const int t = (int)threadIdx.x, lane = t & 31, wid = t >> 5;
  const int per = bins > kToppThreads ? bins / kToppThreads : 1;
  const int b_hi = bins - 1 - t * per;
  unsigned long long mine = 0ull;
  if (b_hi >= 0)
    for (int i = 0; i < per; ++i) mine += hm[b_hi - i];
  unsigned long long x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_m[wid] = x;
  if (t == 0) *s_found = 0;
  __syncthreads();
  unsigned long long before = x - mine;
  for (int w = 0; w < wid; ++w) before += warp_m[w];
  if (b_hi >= 0 && before < need && need <= before + mine) {
    unsigned long long cm = before;
    for (int i = 0; i < per; ++i) {
      const int b = b_hi - i;
      if (cm + hm[b] >= need) {
        *s_digit = (unsigned)b;
        *s_before_m = cm;
        *s_found = 1;
        break;
      }
      cm += hm[b];
    }
  }
  __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kToppThreads, 2) kl_topp_count_kernel(KlArgs args, float top_p, int64_t* row_k) {
  using E = KlElem<T>;
  using Kf = KlKey<T>;
  constexpr int V8 = E::kVec;
  constexpr bool BF = sizeof(T) == 2;
  constexpr int PASSES = BF ? 2 : 4;
  constexpr int WPV = 4;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __shared__ uint64_t bar;
  __shared__ int s_ok, s_found;
  __shared__ unsigned long long hist_m[512];   // cluster sums
  __shared__ unsigned hist_lo[512], hist_hi[512];  // this CTA's sums: low word, high bits and carries
  __shared__ unsigned recv_max[kKlMaxCluster];
  __shared__ unsigned warp_u[2][kToppWarps];
  __shared__ unsigned long long warp_m[kToppWarps];
  __shared__ unsigned s_digit;
  __shared__ unsigned long long s_before_m, s_P;

  cg::cluster_group cluster = cg::this_cluster();
  const int csize = (int)cluster.num_blocks();
  const int crank = (int)cluster.block_rank();
  const int64_t row = blockIdx.x / csize;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t v0 = (int64_t)crank * args.slice;
  int64_t v1 = v0 + args.slice;
  if (v1 > args.vocab) v1 = args.vocab;
  const int n = v1 > v0 ? (int)(v1 - v0) : 0;

  T* st = reinterpret_cast<T*>(smem_raw);
  const int nvec_max = (int)((args.slice + 2 * V8) / V8);
  // bf16: high byte of each vector's largest valid key (0 when it has none)
  uint8_t* vtop = reinterpret_cast<uint8_t*>(st + args.slice + 2 * V8);
  // cluster exchange of the CTA histograms ([csize][512] low words, then
  // [csize][512] high words), later of the CTA counts; then the warps'
  // vector lists ([nvec_max])
  unsigned* recv_lo = reinterpret_cast<unsigned*>(vtop + (nvec_max + 15) / 16 * 16);
  unsigned* recv_hi = recv_lo + csize * 512;
  unsigned* vlist = recv_hi + csize * 512;
  const KlSliceGeom geo = kl_stage_slice<T, kToppThreads>(args, row, v0, n, st, nullptr, &bar, &s_ok);
  const int off = geo.off, nslots = geo.nslots, nvec = geo.nvec;
  const bool ok = s_ok != 0;
  const uint32_t* wt = reinterpret_cast<const uint32_t*>(st);
  const uint4* vt = reinterpret_cast<const uint4*>(st);
  const int kfirst = (off + V8 - 1) / V8;  // vectors [kfirst, klast) hold no pad slot
  const int klast = nslots / V8;
  const float a = args.a;
  const int W = ((nvec + kToppWarps - 1) / kToppWarps + 31) / 32 * 32;  // warp w lists vectors [w W, (w+1) W)
  const int kw0 = wid * W;

  // ---- largest key of the row (and of every vector)
  uint32_t mk = 0u;
  if (ok)
    for (int k = (int)threadIdx.x; k < nvec; k += kToppThreads) {
      uint32_t vm = 0u;
      if (BF && k >= kfirst && k < klast) {  // interior bf16 vector: keys two at a time
        const uint4 v = vt[k];
        const uint32_t m2 = __vmaxu2(__vmaxu2(bf16x2_keys(v.x), bf16x2_keys(v.y)),
                                     __vmaxu2(bf16x2_keys(v.z), bf16x2_keys(v.w)));
        vm = max(m2 & 0xFFFFu, m2 >> 16);
        mk = max(mk, vm);
        vtop[k] = (uint8_t)(vm >> 8);
        continue;
      }
#pragma unroll
      for (int q = 0; q < WPV; ++q) {
        const uint32_t w = wt[k * WPV + q];
#pragma unroll
        for (int h = 0; h < Kf::kPerWord; ++h) {
          const int j = k * V8 + q * Kf::kPerWord + h;
          if (j >= off && j < nslots) vm = max(vm, Kf::key(w, h));
        }
      }
      mk = max(mk, vm);
      if (BF) vtop[k] = (uint8_t)(vm >> 8);
    }
  mk = __reduce_max_sync(0xFFFFFFFFu, mk);
  if (lane == 0) warp_u[0][wid] = mk;
  __syncthreads();
  if ((int)threadIdx.x < csize) {
    uint32_t c = warp_u[0][0];
    for (int w = 1; w < kToppWarps; ++w) c = max(c, warp_u[0][w]);
    cluster.map_shared_rank(recv_max, (int)threadIdx.x)[crank] = c;
  }
  cluster.sync();
  uint32_t kmax = recv_max[0];
  for (int r = 1; r < csize; ++r) kmax = max(kmax, recv_max[r]);
  const float mw = topp_key_value<T>(kmax) * a;

  // ---- radix select on mass: the key tau at which the cumulative mass from
  // the top reaches P = ceil(p * total mass)
  uint32_t prefix = 0u;
  unsigned long long above_m = 0ull, P = 0ull;
  bool found = true;
  for (int p = 0; p < PASSES && found; ++p) {
    const int dbits = BF ? (p == 0 ? 9 : 7) : 8;
    const int shift = BF ? (p == 0 ? 7 : 0) : Kf::kBits - 8 * (p + 1);
    const int bins = 1 << dbits;
    for (int b = (int)threadIdx.x; b < bins; b += kToppThreads) {
      hist_lo[b] = 0u;
      hist_hi[b] = 0u;
    }
    __syncthreads();
    auto add_mass = [&](unsigned b, float z) {
      const unsigned long long q = topp_mass(z, a, mw);
      const unsigned qlo = (unsigned)q, qhi = (unsigned)(q >> 32);
      const unsigned old = atomicAdd(&hist_lo[b], qlo);
      const unsigned up = qhi + (old + qlo < old ? 1u : 0u);  // high bits + carry
      if (up != 0u) atomicAdd(&hist_hi[b], up);
    };
    auto add_key = [&](uint32_t key) { add_mass((key >> shift) & (uint32_t)(bins - 1), topp_key_value<T>(key)); };
    auto vector_keys = [&](int k, bool match) {
#pragma unroll
      for (int q = 0; q < WPV; ++q) {
        const uint32_t w = wt[k * WPV + q];
#pragma unroll
        for (int h = 0; h < Kf::kPerWord; ++h) {
          const int j = k * V8 + q * Kf::kPerWord + h;
          const uint32_t key = Kf::key(w, h);
          if (j >= off && j < nslots && (!match || (key >> (shift + dbits)) == prefix)) add_key(key);
        }
      }
    };
    if (ok) {
      if (BF && p == 1) {
        // only the vectors whose largest key can lie in bucket `prefix`
        const uint32_t top = prefix >> 1;
        const unsigned len =
            topk_warp_list(vlist, kw0, W, nvec, [&](int k) { return (uint32_t)vtop[k] >= top; });
        for (unsigned i = lane; i < len; i += 32) {
          const int k = (int)vlist[kw0 + i];
          if (BF && k >= kfirst && k < klast) {  // interior bf16 vector: two keys at a time
            const uint4 v = vt[k];
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t k2 = bf16x2_keys(w4[q]);
              if (((k2 & 0xFFFFu) >> 7) == prefix) add_mass(k2 & 0x7Fu, __uint_as_float(w4[q] << 16));
              if ((k2 >> 23) == prefix) add_mass((k2 >> 16) & 0x7Fu, __uint_as_float(w4[q] & 0xFFFF0000u));
            }
            continue;
          }
          vector_keys(k, true);
        }
      } else {
        for (int k = (int)threadIdx.x; k < nvec; k += kToppThreads) {
          if (BF && p == 0 && k >= kfirst && k < klast) {  // interior bf16 vector, first digit
            const uint4 v = vt[k];
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint32_t k2 = bf16x2_keys(w4[q]);
              add_mass((k2 & 0xFFFFu) >> 7, __uint_as_float(w4[q] << 16));
              add_mass(k2 >> 23, __uint_as_float(w4[q] & 0xFFFF0000u));
            }
            continue;
          }
          vector_keys(k, p > 0);
        }
      }
    }
    __syncthreads();
    for (int i = (int)threadIdx.x; i < csize * bins; i += kToppThreads) {
      const int r = i / bins, b = i - r * bins;
      cluster.map_shared_rank(recv_lo, r)[crank * 512 + b] = hist_lo[b];
      cluster.map_shared_rank(recv_hi, r)[crank * 512 + b] = hist_hi[b];
    }
    cluster.sync();
    for (int b = (int)threadIdx.x; b < bins; b += kToppThreads) {
      unsigned long long tm = 0ull;
      for (int r = 0; r < csize; ++r) tm += ((unsigned long long)recv_hi[r * 512 + b] << 32) | recv_lo[r * 512 + b];
      hist_m[b] = tm;
    }
    cluster.sync();  // every CTA has read its buffers before a peer writes them again
    if (p == 0) {
      if (threadIdx.x == 0) {
        unsigned long long tot = 0ull;
        for (int b = 0; b < bins; ++b) tot += hist_m[b];
        const unsigned long long need = (unsigned long long)ceil((double)top_p * (double)tot);
        s_P = need > 0ull ? need : 1ull;
      }
      __syncthreads();
      P = s_P;
    }
    topp_find_bucket(hist_m, bins, P - above_m, warp_m, &s_digit, &s_before_m, &s_found);
    found = s_found != 0;
    if (found) {
      above_m += s_before_m;
      prefix = (prefix << dbits) | s_digit;
    }
    __syncthreads();  // hist_*, s_* are rewritten by the next digit
  }
  // ---- keys above tau and equal to tau, counted over the row (found is the
  // same in every CTA of the cluster)
  unsigned n_gt = 0u, n_eq = 0u;
  if (found) {
    const uint32_t tau = prefix;
    unsigned c_gt = 0u, c_eq = 0u;
    if (ok)
      for (int k = (int)threadIdx.x; k < nvec; k += kToppThreads) {
        if (BF && (uint32_t)vtop[k] < (tau >> 8)) continue;  // no key of this vector reaches tau
        if (BF && k >= kfirst && k < klast) {  // interior bf16 vector: two keys at a time
          const uint4 v = vt[k];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t k2 = bf16x2_keys(w4[q]);
            const uint32_t k0 = k2 & 0xFFFFu, k1 = k2 >> 16;
            c_gt += (k0 > tau ? 1u : 0u) + (k1 > tau ? 1u : 0u);
            c_eq += (k0 == tau ? 1u : 0u) + (k1 == tau ? 1u : 0u);
          }
          continue;
        }
#pragma unroll
        for (int q = 0; q < WPV; ++q) {
          const uint32_t w = wt[k * WPV + q];
#pragma unroll
          for (int h = 0; h < Kf::kPerWord; ++h) {
            const int j = k * V8 + q * Kf::kPerWord + h;
            const uint32_t key = Kf::key(w, h);
            const bool in = j >= off && j < nslots;
            c_gt += (in && key > tau) ? 1u : 0u;
            c_eq += (in && key == tau) ? 1u : 0u;
          }
        }
      }
    c_gt = __reduce_add_sync(0xFFFFFFFFu, c_gt);
    c_eq = __reduce_add_sync(0xFFFFFFFFu, c_eq);
    if (lane == 0) {
      warp_u[0][wid] = c_gt;
      warp_u[1][wid] = c_eq;
    }
    __syncthreads();
    if ((int)threadIdx.x < csize) {
      unsigned g = 0u, e = 0u;
      for (int w = 0; w < kToppWarps; ++w) {
        g += warp_u[0][w];
        e += warp_u[1][w];
      }
      cluster.map_shared_rank(recv_lo, (int)threadIdx.x)[crank] = g;
      cluster.map_shared_rank(recv_hi, (int)threadIdx.x)[crank] = e;
    }
    cluster.sync();
    for (int r = 0; r < csize; ++r) {
      n_gt += recv_lo[r];
      n_eq += recv_hi[r];
    }
  }
  if (crank == 0 && threadIdx.x == 0) {
    int64_t m = args.vocab;
    if (found && ok) {
      const unsigned long long q_tau = topp_mass(topp_key_value<T>(prefix), a, mw);
      unsigned long long r = q_tau > 0ull ? (P - above_m + q_tau - 1ull) / q_tau : (unsigned long long)n_eq;
      if (r < 1ull) r = 1ull;
      if (r > n_eq) r = n_eq;
      m = (int64_t)n_gt + (int64_t)r;
    }
    row_k[row] = m;
  }
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
  const size_t smem = p.smem / 2;  // the teacher's slice only
  cudaError_t e = cudaFuncSetAttribute(kl_row_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.rows * p.cluster));
  cfg.blockDim = dim3(kKlThreads);
  cfg.dynamicSmemBytes = smem;
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

template <typename T>
static cudaError_t launch_kl_topk(const KlArgs& a, const KlPlan& p, cudaStream_t s) {
  const int vec = 16 / (int)sizeof(T);
  const size_t nvec_max = (size_t)((p.slice + 2 * vec) / vec);
  // the teacher slice, the per-vector largest key (u16), then the vector
  // lists (u32) and the selection mask (u8), or, over them, the cluster's
  // 512-count histograms
  size_t tail = nvec_max * 4 + (nvec_max + 3) / 4 * 4;
  if (tail < (size_t)p.cluster * 512 * 4) tail = (size_t)p.cluster * 512 * 4;
  const size_t smem = p.smem / 2 + (nvec_max * 2 + 15) / 16 * 16 + tail;  // the teacher's slice only
  cudaError_t e = cudaFuncSetAttribute(kl_topk_row_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.rows * p.cluster));
  cfg.blockDim = dim3(kTopkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kl_topk_row_kernel<T>, a);
}

template <typename T>
static cudaError_t launch_kl_topp_count(const KlArgs& a, const KlPlan& p, float top_p, int64_t* row_k,
                                        cudaStream_t s) {
  // the teacher slice, the vector tops (u8), the two exchange buffers
  // ([cluster][512] u32 each) and the vector lists (u32)
  const int vec = 16 / (int)sizeof(T);
  const size_t nvec_max = (size_t)((p.slice + 2 * vec) / vec);
  const size_t smem = p.smem / 2 + (nvec_max + 15) / 16 * 16 + (size_t)p.cluster * 512 * 8 + nvec_max * 4;
  cudaError_t e =
      cudaFuncSetAttribute(kl_topp_count_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.rows * p.cluster));
  cfg.blockDim = dim3(kToppThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kl_topp_count_kernel<T>, a, top_p, row_k);
}

// every entry of k[0..n) = v
__global__ void fill_i64_kernel(int64_t* k, int64_t n, int64_t v) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    k[i] = v;
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
  NVFP4_ENTRY("qad_kl_fwd_bwd");
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
  args.topk = vocab;
  cudaError_t e = dtype == NVFP4_BF16 ? launch_kl<__nv_bfloat16>(args, plan, s) : launch_kl<float>(args, plan, s);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  kl_mean_kernel<<<1, 1024, 0, s>>>(args.row_kl, rows, loss, row_kl);
  count_launches(2);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

nvfp4_status qad_kl_topk_fwd_bwd(const void* teacher, const void* student, nvfp4_dtype dtype, int64_t rows,
                                 int64_t vocab, int64_t ld, int64_t k, float temperature, float* loss,
                                 float* row_kl, void* dlogits, int64_t ld_grad, float grad_scale, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("qad_kl_topk_fwd_bwd");
  if (dtype != NVFP4_BF16 && dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  if (!(temperature > 0.0f) || !loss || k < 1) return NVFP4_ERR_ARG;
  if (rows < 0 || vocab <= 0 || ld < vocab) return NVFP4_ERR_SHAPE;
  if (dlogits && ld_grad < vocab) return NVFP4_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (rows == 0) return cudaMemsetAsync(loss, 0, sizeof(float), s) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
  if (!teacher || !student) return NVFP4_ERR_ARG;
  if (rows > 0x7FFFFFFFll / kKlMaxCluster) return NVFP4_ERR_SHAPE;
  const int esz = dtype == NVFP4_BF16 ? 2 : 4;
  if (((uintptr_t)teacher ^ (uintptr_t)student) & 15u) return NVFP4_ERR_ALIGN;
  if (((uintptr_t)teacher | (uintptr_t)student) % esz) return NVFP4_ERR_ALIGN;
  if (dlogits && ((uintptr_t)dlogits % esz)) return NVFP4_ERR_ALIGN;
  const size_t need = qad_kl_workspace_size(rows, vocab, dtype);
  if (!workspace || workspace_bytes < need) return NVFP4_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 15u) != 0) return NVFP4_ERR_ALIGN;
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
  args.topk = k;
  cudaError_t e =
      dtype == NVFP4_BF16 ? launch_kl_topk<__nv_bfloat16>(args, plan, s) : launch_kl_topk<float>(args, plan, s);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  kl_mean_kernel<<<1, 1024, 0, s>>>(args.row_kl, rows, loss, row_kl);
  count_launches(2);
  return cudaGetLastError() == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}

size_t qad_kl_topp_workspace_size(int64_t rows, int64_t vocab, nvfp4_dtype dtype) {
  return rows > 0 ? qad_kl_workspace_size(rows, vocab, dtype) + (size_t)rows * sizeof(int64_t) : 0;
}

nvfp4_status qad_kl_topp_fwd_bwd(const void* teacher, const void* student, nvfp4_dtype dtype, int64_t rows,
                                 int64_t vocab, int64_t ld, float top_p, float temperature, float* loss,
                                 float* row_kl, void* dlogits, int64_t ld_grad, float grad_scale, int64_t* row_k,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_ENTRY("qad_kl_topp_fwd_bwd");
  if (dtype != NVFP4_BF16 && dtype != NVFP4_F32) return NVFP4_ERR_DTYPE;
  if (!(temperature > 0.0f) || !loss || !(top_p > 0.0f)) return NVFP4_ERR_ARG;
  if (rows < 0 || vocab <= 0 || ld < vocab) return NVFP4_ERR_SHAPE;
  if (dlogits && ld_grad < vocab) return NVFP4_ERR_SHAPE;
  cudaStream_t s = (cudaStream_t)stream;
  if (rows == 0) return cudaMemsetAsync(loss, 0, sizeof(float), s) == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
  if (!teacher || !student) return NVFP4_ERR_ARG;
  if (rows > 0x7FFFFFFFll / kKlMaxCluster) return NVFP4_ERR_SHAPE;
  const int esz = dtype == NVFP4_BF16 ? 2 : 4;
  if (((uintptr_t)teacher ^ (uintptr_t)student) & 15u) return NVFP4_ERR_ALIGN;
  if (((uintptr_t)teacher | (uintptr_t)student) % esz) return NVFP4_ERR_ALIGN;
  if (dlogits && ((uintptr_t)dlogits % esz)) return NVFP4_ERR_ALIGN;
  if (row_k && ((uintptr_t)row_k % sizeof(int64_t))) return NVFP4_ERR_ALIGN;
  const size_t need = qad_kl_topp_workspace_size(rows, vocab, dtype);
  if (!workspace || workspace_bytes < need) return NVFP4_ERR_WORKSPACE;
  if (((uintptr_t)workspace & 15u) != 0) return NVFP4_ERR_ALIGN;
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
  args.topk = vocab;
  int64_t* ks = row_k ? row_k
                      : reinterpret_cast<int64_t*>(static_cast<uint8_t*>(workspace) +
                                                   qad_kl_workspace_size(rows, vocab, dtype));
  cudaError_t e;
  if (top_p >= 1.0f) {  // the whole row
    const int64_t blocks = (rows + 255) / 256 < 1024 ? (rows + 255) / 256 : 1024;
    fill_i64_kernel<<<(unsigned)blocks, 256, 0, s>>>(ks, rows, vocab);
    e = cudaGetLastError();
  } else {
    e = dtype == NVFP4_BF16 ? launch_kl_topp_count<__nv_bfloat16>(args, plan, top_p, ks, s)
                            : launch_kl_topp_count<float>(args, plan, top_p, ks, s);
  }
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  args.topk_rows = ks;
  e = dtype == NVFP4_BF16 ? launch_kl_topk<__nv_bfloat16>(args, plan, s) : launch_kl_topk<float>(args, plan, s);
  if (e != cudaSuccess) return NVFP4_ERR_CUDA;
  kl_mean_kernel<<<1, 1024, 0, s>>>(args.row_kl, rows, loss, row_kl);
  count_launches(3);
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

// Device address of g_kl_noalloc_rows per device.  In host code the array's
// name only stands for the symbol; the address a kernel may use comes from
// cudaGetSymbolAddress with that device current.  The first call on a device
// looks it up; later calls outside a stream capture look it up again (cheap,
// and correct after a cudaDeviceReset reloaded the module), calls inside a
// capture use the cached value.
constexpr int kKlNoAllocMaxDevices = 64;
static std::atomic<void*> g_kl_noalloc_ptr[kKlNoAllocMaxDevices];

static nvfp4_status kl_noalloc_scratch(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (dev < 0 || dev >= kKlNoAllocMaxDevices) return NVFP4_ERR_UNSUPPORTED;
  void* p = g_kl_noalloc_ptr[dev].load(std::memory_order_acquire);
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusActive;
  const bool capturing = cudaStreamIsCapturing(stream, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
  if (p == nullptr || !capturing) {
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_kl_noalloc_rows) != cudaSuccess || q == nullptr) return NVFP4_ERR_CUDA;
    g_kl_noalloc_ptr[dev].store(q, std::memory_order_release);
    p = q;
  }
  *out = p;
  return NVFP4_OK;
}

}  // namespace nvfp4

extern "C" nvfp4_status qad_kl_fwd_bwd_noalloc(const void* teacher, const void* student, nvfp4_dtype dtype,
                                               int64_t rows, int64_t vocab, int64_t ld, float temperature,
                                               float* loss, float* row_kl, void* dlogits, int64_t ld_grad,
                                               float grad_scale, void* stream) {
  NVFP4_ENTRY("qad_kl_fwd_bwd_noalloc");
  if (rows > nvfp4::kKlNoAllocMaxRows) return NVFP4_ERR_SHAPE;
  void* scratch = nullptr;
  nvfp4_status st = nvfp4::kl_noalloc_scratch((cudaStream_t)stream, &scratch);
  if (st != NVFP4_OK) return st;
  // every row's slot is written before it is read, so nothing needs clearing
  return qad_kl_fwd_bwd(teacher, student, dtype, rows, vocab, ld, temperature, loss, row_kl, dlogits, ld_grad,
                        grad_scale, scratch, (size_t)nvfp4::kKlNoAllocMaxRows * sizeof(float), stream);
}
