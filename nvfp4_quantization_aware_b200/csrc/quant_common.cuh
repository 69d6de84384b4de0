// quant_common.cuh -- device helpers shared by the NVFP4 encode kernels
// (quantize.cu and the MoE gather/activation quantizers in moe.cu): 256-bit
// streaming IO, a 16-element block held by one lane, a multiply-shift divider,
// and the per-block encode (block scale, division, E2M1 packing).
#pragma once

#include "common.cuh"

namespace nvfp4 {

// Unsigned 32-bit division by a run-time invariant divisor through one
// multiply-high and two shifts (Granlund & Montgomery, "Division by Invariant
// Integers using Multiplication", 1994, section 4): for d >= 1 with
// l = ceil(log2 d), m = floor(2^32 (2^l - d) / d) + 1,
//   q = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0),  t = mulhi(m, n),
// exact for every 32-bit n.
struct FastDiv {
  uint32_t d, m, s1, s2;
};

static FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (1ull << l) < d) ++l;
  FastDiv f;
  f.d = d;
  f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
  f.s1 = l < 1 ? l : 1;
  f.s2 = l > 0 ? l - 1 : 0;
  return f;
}

NVFP4_DEV uint32_t fastdiv(uint32_t n, const FastDiv& f) {
  const uint32_t t = __umulhi(f.m, n);
  return (t + ((n - t) >> f.s1)) >> f.s2;
}

// 32-byte (256-bit) streaming load and store.
NVFP4_DEV void ld_stream_v8(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

NVFP4_DEV void st_stream_v8(void* p, const uint32_t (&r)[8]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]),
               "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

NVFP4_DEV void st_stream_v2(void* p, uint32_t a, uint32_t b) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1,%2};" ::"l"(p), "r"(a), "r"(b) : "memory");
}

// One 16-element block held by a lane.
template <typename T>
struct Block16;

template <>
struct Block16<__nv_bfloat16> {
  uint32_t w[8];
  // wide: the address is 32-byte aligned (one 256-bit load); else 16-byte
  NVFP4_DEV void load(const __nv_bfloat16* p, bool wide) {
    if (wide) {
      ld_stream_v8(p, w);
    } else {
      const uint4 a = ld_stream_v4(p), b = ld_stream_v4(p + 8);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
  }
  NVFP4_DEV void zero() {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = 0u;
  }
  NVFP4_DEV void to_f32(float (&v)[16]) const {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = bf16lo_to_f32(w[i]);
      v[2 * i + 1] = bf16hi_to_f32(w[i]);
    }
  }
  NVFP4_DEV static void store(__nv_bfloat16* p, const float (&v)[16], bool wide) {
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    if (wide) {
      st_stream_v8(p, o);
    } else {
      st_stream_v4(p, make_uint4(o[0], o[1], o[2], o[3]));
      st_stream_v4(p + 8, make_uint4(o[4], o[5], o[6], o[7]));
    }
  }
};

template <>
struct Block16<float> {
  uint32_t w[16];
  NVFP4_DEV void load(const float* p, bool wide) {
    if (wide) {
      uint32_t a[8], b[8];
      ld_stream_v8(p, a);
      ld_stream_v8(p + 8, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        w[i] = a[i];
        w[8 + i] = b[i];
      }
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 a = ld_stream_v4(p + 4 * j);
        w[4 * j] = a.x; w[4 * j + 1] = a.y; w[4 * j + 2] = a.z; w[4 * j + 3] = a.w;
      }
    }
  }
  NVFP4_DEV void zero() {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = 0u;
  }
  NVFP4_DEV void to_f32(float (&v)[16]) const {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(w[i]);
  }
  NVFP4_DEV static void store(float* p, const float (&v)[16], bool wide) {
    uint32_t a[8], b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[i] = __float_as_uint(v[i]);
      b[i] = __float_as_uint(v[8 + i]);
    }
    if (wide) {
      st_stream_v8(p, a);
      st_stream_v8(p + 8, b);
    } else {
      st_stream_v4(p, make_uint4(a[0], a[1], a[2], a[3]));
      st_stream_v4(p + 4, make_uint4(a[4], a[5], a[6], a[7]));
      st_stream_v4(p + 8, make_uint4(b[0], b[1], b[2], b[3]));
      st_stream_v4(p + 12, make_uint4(b[4], b[5], b[6], b[7]));
    }
  }
};

// ------------------------------------------------------------------ input traits

template <typename T>
struct Lane8;

// bf16: one 16-byte load per lane.
template <>
struct Lane8<__nv_bfloat16> {
  uint4 raw;
  NVFP4_DEV void load(const __nv_bfloat16* p) { raw = ld_stream_v4(p); }
  NVFP4_DEV void zero() { raw = make_uint4(0, 0, 0, 0); }
  NVFP4_DEV void to_f32(float (&v)[8]) const {
    v[0] = bf16lo_to_f32(raw.x); v[1] = bf16hi_to_f32(raw.x);
    v[2] = bf16lo_to_f32(raw.y); v[3] = bf16hi_to_f32(raw.y);
    v[4] = bf16lo_to_f32(raw.z); v[5] = bf16hi_to_f32(raw.z);
    v[6] = bf16lo_to_f32(raw.w); v[7] = bf16hi_to_f32(raw.w);
  }
};

// f32: two 16-byte loads per lane.
template <>
struct Lane8<float> {
  uint4 a, b;
  NVFP4_DEV void load(const float* p) { a = ld_stream_v4(p); b = ld_stream_v4(p + 4); }
  NVFP4_DEV void zero() { a = b = make_uint4(0, 0, 0, 0); }
  NVFP4_DEV void to_f32(float (&v)[8]) const {
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
    v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
  }
};


// Encode one 16-element block with tensor scale sg (denom6 = 6 * sg, rounded):
// returns the E4M3 block scale (computed, or `sb_frozen` when frozen) and the
// 16 codes in (lo, hi) (element i in nibble i of lo for i < 8, of hi else),
// and the decode scale d through `d_out`.
template <bool BF16_IN>
NVFP4_DEV uint32_t encode_block16(const float (&v)[16], float sg, float denom6, bool frozen, uint32_t sb_frozen,
                                  uint32_t& lo, uint32_t& hi, float& d_out) {
  uint32_t sb;
  if (frozen) {
    sb = sb_frozen;
  } else {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
    sb = (sg == 0.0f) ? 0u : e4m3_encode(__fdiv_rn(m, denom6));
  }
  const float d = __fmul_rn(e4m3_decode(sb), sg);
  lo = 0;
  hi = 0;
  if (d != 0.0f) {
    float q[16];
    if (BF16_IN && block_scale_in_fast_range(d)) {
      const float r = __frcp_rn(d);
#pragma unroll
      for (int i = 0; i < 16; ++i) q[i] = div_by_block_scale(v[i], d, r);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) q[i] = __fdiv_rn(v[i], d);
    }
    float q0[8], q1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q0[i] = q[i];
      q1[i] = q[8 + i];
    }
    lo = e2m1x8_encode(q0);
    hi = e2m1x8_encode(q1);
  }
  d_out = d;
  return sb;
}

// Dequantize the 16 codes of a block with decode scale d (binary32 products).
NVFP4_DEV void decode_block16(uint32_t lo, uint32_t hi, float d, float (&o)[16]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t word = j < 4 ? lo : hi;
    float a0, a1;
    e2m1x2_decode((word >> (8 * (j & 3))) & 0xFF, a0, a1);
    o[2 * j] = __fmul_rn(a0, d);
    o[2 * j + 1] = __fmul_rn(a1, d);
  }
}

}  // namespace nvfp4
