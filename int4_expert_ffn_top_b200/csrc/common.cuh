// Device helpers shared by the routed-expert kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

constexpr int kGroup = 64;

// Bytes of one row record: codes, then in/64 fp16 scales, then in/64 fp16 biases, padded to 16.
__host__ __device__ constexpr int qrow_bytes(int in, int bits) { return (in * bits / 8 + 4 * (in / 64) + 15) / 16 * 16; }

// Position of element j of an fp16 vector stored in pair order (per 8-block: (v_j, v_{j+4})).
MOE_DEV int pair_pos(int j) { return (j & ~7) + ((j & 3) << 1) + ((j >> 2) & 1); }

MOE_DEV uint32_t lop_and_or(uint32_t a, uint32_t b, uint32_t c) {
  // (a & b) | c in one LOP3
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

MOE_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

MOE_DEV __half2 as_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
MOE_DEV uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// d = a*b + c with fp16 a, b and fp32 c, d: the product of two fp16 values is
// exact in fp32, so each step rounds once, like an fp32 FMA on exact operands.
MOE_DEV float fma_mix(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}

// Both halves of two half2 registers: acc += a.x*b.x + a.y*b.y (two roundings).
MOE_DEV float dot2_mix(uint32_t a, uint32_t b, float acc) {
  acc = fma_mix(static_cast<uint16_t>(a & 0xffffu), static_cast<uint16_t>(b & 0xffffu), acc);
  acc = fma_mix(static_cast<uint16_t>(a >> 16), static_cast<uint16_t>(b >> 16), acc);
  return acc;
}

// One packed int4 word (nibble j at bits 4j) -> four half2 holding (q_j - 8,
// q_{j+4} - 8) for j = 0..3.  OR-ing a nibble into the mantissa of fp16 1024.0
// (0x6400) yields exactly 1024 + q (IEEE-754 binary16, ulp 1 on [1024, 2048));
// a nibble at bits 4..7 yields 1024 + 16q, scaled back by an exact 1/16.  The
// results are small integers, exact in fp16.
MOE_DEV void int4_word_to_h2(uint32_t w, uint32_t (&o)[4]) {
  const uint32_t kMagic = 0x64006400u;
  const uint32_t lo0 = lop_and_or(w, 0x000F000Fu, kMagic);
  const uint32_t hi0 = lop_and_or(w, 0x00F000F0u, kMagic);
  const uint32_t w8 = w >> 8;
  const uint32_t lo1 = lop_and_or(w8, 0x000F000Fu, kMagic);
  const uint32_t hi1 = lop_and_or(w8, 0x00F000F0u, kMagic);
  const __half2 k1032 = __half2half2(__ushort_as_half(0x6408));   // 1032
  const __half2 k16th = __half2half2(__ushort_as_half(0x2C00));   // 1/16
  const __half2 km72 = __half2half2(__ushort_as_half(0xD480));    // -72
  o[0] = h2_bits(__hsub2(as_h2(lo0), k1032));
  o[1] = h2_bits(__hfma2(as_h2(hi0), k16th, km72));
  o[2] = h2_bits(__hsub2(as_h2(lo1), k1032));
  o[3] = h2_bits(__hfma2(as_h2(hi1), k16th, km72));
}

// One packed 8-bit word (byte j at bits 8j) -> two half2 holding (q0-128, q1-128)
// and (q2-128, q3-128); same magic-exponent construction (1024 + q exact for q < 1024).
MOE_DEV void int8_word_to_h2(uint32_t w, uint32_t (&o)[2]) {
  const uint32_t kHi = 0x64646464u;
  const __half2 k1152 = __half2half2(__ushort_as_half(0x6480));   // 1152
  o[0] = h2_bits(__hsub2(as_h2(prmt(w, kHi, 0x4140u)), k1152));
  o[1] = h2_bits(__hsub2(as_h2(prmt(w, kHi, 0x4342u)), k1152));
}

// 32 nibbles (one 16-byte chunk = half a group) dotted with 32 activations held
// as 16 half2 in "pair order" (for each 8-block: (u_j, u_{j+4}), j = 0..3).
// Two independent accumulation chains (words 0-1 and 2-3), added at the end.
MOE_DEV float dot_chunk_int4(const uint4& wq, const uint4* up, float acc) {
  const uint32_t ws[4] = {wq.x, wq.y, wq.z, wq.w};
  float a2[2] = {acc, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t q[4];
    int4_word_to_h2(ws[i], q);
    const uint4 u = up[i];
    float& a = a2[i >> 1];
    a = dot2_mix(q[0], u.x, a);
    a = dot2_mix(q[1], u.y, a);
    a = dot2_mix(q[2], u.z, a);
    a = dot2_mix(q[3], u.w, a);
  }
  return a2[0] + a2[1];
}

// 16 bytes (a quarter group) of an 8-bit matrix dotted with 16 activations held
// as 8 half2 in natural order.
MOE_DEV float dot_chunk_int8(const uint4& wq, const uint4* up, float acc) {
  const uint32_t ws[4] = {wq.x, wq.y, wq.z, wq.w};
  const uint4 u0 = up[0], u1 = up[1];
  const uint32_t us[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t q[2];
    int8_word_to_h2(ws[i], q);
    acc = dot2_mix(q[0], us[2 * i], acc);
    acc = dot2_mix(q[1], us[2 * i + 1], acc);
  }
  return acc;
}

// 8 fp16 weights (one 16-byte chunk) dotted with 8 activations as 4 half2 (natural order).
MOE_DEV float dot_chunk_f16(const uint4& w, const uint4& u, float acc) {
  acc = dot2_mix(w.x, u.x, acc);
  acc = dot2_mix(w.y, u.y, acc);
  acc = dot2_mix(w.z, u.z, acc);
  acc = dot2_mix(w.w, u.w, acc);
  return acc;
}

MOE_DEV uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Device-side status report into an optional error word: the first nonzero status wins.
MOE_DEV void report(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Largest finite fp16 value: bf16 activations above it in magnitude (or not finite) cannot be
// multiplied as fp16 (moe_status MOE_ERR_RANGE).
constexpr float kF16Max = 65504.0f;

MOE_DEV float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }
MOE_DEV float bf16_bits_to_float(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// bf16 -> fp16 bit pattern (exact for |x| in fp16's normal range; rounds below it).
MOE_DEV uint16_t bf16_to_f16_bits(uint16_t b) {
  return __half_as_ushort(__float2half_rn(bf16_bits_to_float(b)));
}

// SiLU and sigmoid through the hardware reciprocal (__fdividef, <= 2 ulp): the
// IEEE division would inline a long slow path at every call site.
MOE_DEV float silu(float x) { return __fdividef(x, 1.0f + expf(-x)); }
MOE_DEV float sigmoid(float x) { return __fdividef(1.0f, 1.0f + expf(-x)); }

template <int SEG>
MOE_DEV float seg_reduce(float v) {
#pragma unroll
  for (int o = SEG / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

MOE_DEV float warp_reduce(float v) { return seg_reduce<32>(v); }

MOE_DEV float seg_reduce_dyn(float v, int seg) {
  for (int o = seg / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace moe
