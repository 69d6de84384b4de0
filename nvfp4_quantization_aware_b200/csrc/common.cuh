// common.cuh -- shared device helpers for the sm_100a kernels of libnvfp4qad.
//
// Format conversions use the sm_100a PTX conversion instructions (cvt with
// .e2m1x2 / .e4m3x2 and .satfinite), all round-to-nearest-even.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "nvfp4qad.h"

#define NVFP4_DEV __device__ __forceinline__

namespace nvfp4 {

// Device error word, read and cleared by nvfp4_device_error().
extern __device__ int g_device_error;

constexpr int kErrWaitTimeout = 1;
constexpr int kErrRowsCapacity = 2;   // routed rows exceed the permutation buffer
constexpr int kErrExpertId = 3;       // an expert id outside [0, experts)

NVFP4_DEV void report_error(int code) { atomicCAS(&g_device_error, 0, code); }

// Programmatic dependent launch: a kernel launched with the programmatic
// stream serialization attribute may start while the previous kernel of the
// stream is finishing; it must execute this before it reads or writes any
// global memory that kernel may touch (a no-op for a normal launch).
NVFP4_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host-side count of kernel launches (nvfp4_launch_count).
void count_launches(int n);

// Entry of an exported operation: an NVTX range named after it for the
// duration of the call (nested calls nest), and the host-side fault-injection
// point -- when armed (nvfp4_fault_inject, or NVFP4QAD_FAIL_AT=n in the
// environment at load time) the n-th outermost entry returns NVFP4_ERR_CUDA
// before it validates or launches anything.
struct EntryScope {
  explicit EntryScope(const char* name);
  ~EntryScope();
  bool inject;  // this entry is the armed one
};
#define NVFP4_ENTRY(name)                         \
  ::nvfp4::EntryScope nvfp4_entry_scope_(name);   \
  if (nvfp4_entry_scope_.inject) return NVFP4_ERR_CUDA

// ---------------------------------------------------------------- loads/stores

// 16-byte streaming load that bypasses L1 allocation (each byte is read once).
NVFP4_DEV uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

NVFP4_DEV void st_stream_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

NVFP4_DEV void st_stream_u32(void* p, uint32_t v) {
  asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- bf16 helpers

NVFP4_DEV float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
NVFP4_DEV float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two floats -> packed bf16x2 (lo in bits 0..15), round to nearest even.
NVFP4_DEV uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------- E4M3

// Non-negative float -> E4M3 byte, RNE, saturating to 448.
NVFP4_DEV uint32_t e4m3_encode(float t) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
  return (uint32_t)(r & 0xFF);
}

// E4M3 byte -> float (exact: every E4M3 value is an f16 value).
NVFP4_DEV float e4m3_decode(uint32_t code) {
  uint32_t h2;
  uint16_t in = (uint16_t)(code & 0xFF);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// ---------------------------------------------------------------- E2M1

// Two floats -> one byte of two E2M1 codes (lo nibble from `lo`), RNE,
// saturating to +-6.
NVFP4_DEV uint32_t e2m1x2_encode(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Eight floats -> 32-bit word of eight E2M1 codes (element i in nibble i).
NVFP4_DEV uint32_t e2m1x8_encode(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// One byte of two E2M1 codes -> the two values as floats (exact).
NVFP4_DEV void e2m1x2_decode(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.u8.u32 b, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(h2)
      : "r"(byte));
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  lo = __low2float(h);
  hi = __high2float(h);
}

// ---------------------------------------------------------------- division

// Correctly rounded quotient x / d for a divisor shared by a whole block,
// from r = RN(1/d) (computed once per block with __frcp_rn) and Markstein's
// FMA correction: q0 = RN(x r); the remainder x - q0 d is exact through the
// FMA; q = RN(q0 + (x - q0 d) r).  The remainder is formed as -(q0 d - x) so
// that both negations are free FMA operand modifiers and x = -0 yields -0
// (q0 = -0, q0 d - x = +0, -(+0) r + q0 = -0).  Used only when d lies in
// [2^-90, 2^90]; the library's self-test (nvfp4_selftest_division) compares
// it with __fdiv_rn for every bf16 significand and sign of x (and +-0)
// against every binary32 significand of d.
NVFP4_DEV float div_by_block_scale(float x, float d, float r) {
  const float q0 = __fmul_rn(x, r);
  const float e = __fmaf_rn(q0, d, -x);
  return __fmaf_rn(-e, r, q0);
}

NVFP4_DEV bool block_scale_in_fast_range(float d) {
  return d >= 0x1p-90f && d <= 0x1p90f;
}

// Byte offset of block scale (row, kb) in the MMA scale layout (tiles of 128
// rows x 4 blocks, block index fastest; inside a tile (r%32)*16+(r/32)*4+kb).
NVFP4_DEV int64_t mma_scale_offset(int64_t row, int64_t kb, int64_t kchunks) {
  int64_t tile = (row >> 7) * kchunks + (kb >> 2);
  int32_t rr = (int32_t)(row & 127);
  return tile * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + (kb & 3);
}

}  // namespace nvfp4
