// Device helpers shared by the decode kernels: number formats, streaming loads, packed
// fp32x2 arithmetic, and the dot product of one 16-byte chunk of packed codes with staged
// activations (see decode.cu for the arithmetic).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace moe {

__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf1(uint16_t v) { return __uint_as_float(((uint32_t)v) << 16); }

__device__ __forceinline__ uint16_t f2bf(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

// 16-byte streaming load that bypasses L1 (weights are read once per call).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ uint16_t ld_u16(const void* p) {
  return __ldg(reinterpret_cast<const unsigned short*>(p));
}

// Packed fp32x2 arithmetic (sm_100).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(a)),
        "l"(reinterpret_cast<const unsigned long long&>(b)),
        "l"(reinterpret_cast<const unsigned long long&>(c)));
  return d;
}

// Two masked code fields (each < 2^23) -> their exact integer values as a float pair.
__device__ __forceinline__ float2 codes2(uint32_t m0, uint32_t m1) {
  float2 v = make_float2(__uint_as_float(m0 | 0x4B000000u), __uint_as_float(m1 | 0x4B000000u));
  const float2 off = make_float2(-8388608.0f, -8388608.0f);
  float2 d;
  asm("add.f32x2 %0, %1, %2;"
      : "=l"(reinterpret_cast<unsigned long long&>(d))
      : "l"(reinterpret_cast<const unsigned long long&>(v)),
        "l"(reinterpret_cast<const unsigned long long&>(off)));
  return d;
}

__device__ __forceinline__ uint32_t word_of(const uint4& q, int i) {
  return i == 0 ? q.x : i == 1 ? q.y : i == 2 ? q.z : q.w;
}

// Bit position (within its field's shifted word) at which code j of a 16-byte chunk is read:
// int4 nibble n of a word is read at bit 4n for n <= 4 and at bit 4(n-3) after >> 12; int8
// byte n at bit 8n for n <= 1 and at bit 8(n-2) after >> 16.
template <int BITS>
__device__ __forceinline__ int code_shift(int j) {
  if constexpr (BITS == 4) {
    const int n = j & 7;
    return 4 * (n <= 4 ? n : n - 3);
  } else {
    return 8 * (j & 1);
  }
}

// Scale applied to the activation of code j of a 16-byte chunk when it is staged, so
// that (code field value) * (staged activation) == q_j * x_j exactly: 2^-shift.
template <int BITS>
__device__ __forceinline__ float stage_scale(int j) {
  return __int_as_float((127 - code_shift<BITS>(j)) << 23);
}

// Exact inverse of stage_scale: 2^shift.
template <int BITS>
__device__ __forceinline__ float stage_unscale(int j) {
  return __int_as_float((127 + code_shift<BITS>(j)) << 23);
}

// One 16-byte chunk of one code row against staged activations.
// x4[v * ns], v < 32/BITS*... holds 4 consecutive (pre-scaled) activations.
template <int BITS>
__device__ __forceinline__ float dot_chunk(const uint4& q, const float4* x4, int ns) {
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
  if constexpr (BITS == 4) {
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t w = word_of(q, wi), wh = w >> 12;
      const float4 xa = x4[(2 * wi) * ns], xb = x4[(2 * wi + 1) * ns];
      a0 = ffma2(codes2(w & 0xFu, w & 0xF0u), make_float2(xa.x, xa.y), a0);
      a1 = ffma2(codes2(w & 0xF00u, w & 0xF000u), make_float2(xa.z, xa.w), a1);
      a0 = ffma2(codes2(w & 0xF0000u, wh & 0xF00u), make_float2(xb.x, xb.y), a0);
      a1 = ffma2(codes2(wh & 0xF000u, wh & 0xF0000u), make_float2(xb.z, xb.w), a1);
    }
  } else {
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t w = word_of(q, wi), wh = w >> 16;
      const float4 xa = x4[wi * ns];
      a0 = ffma2(codes2(w & 0xFFu, w & 0xFF00u), make_float2(xa.x, xa.y), a0);
      a1 = ffma2(codes2(wh & 0xFFu, wh & 0xFF00u), make_float2(xa.z, xa.w), a1);
    }
  }
  return (a0.x + a0.y) + (a1.x + a1.y);
}

// The codes of one 32-bit word of a chunk as float pairs, in the pairing the dot products
// above use: int4 (c0, c1), (c2, c3), (c4, c5), (c6, c7); int8 (c0, c1), (c2, c3) in out[0..1].
template <int BITS>
__device__ __forceinline__ void codes_of_word(uint32_t w, float2 out[4]) {
  if constexpr (BITS == 4) {
    const uint32_t wh = w >> 12;
    out[0] = codes2(w & 0xFu, w & 0xF0u);
    out[1] = codes2(w & 0xF00u, w & 0xF000u);
    out[2] = codes2(w & 0xF0000u, wh & 0xF00u);
    out[3] = codes2(wh & 0xF000u, wh & 0xF0000u);
  } else {
    const uint32_t wh = w >> 16;
    out[0] = codes2(w & 0xFFu, w & 0xFF00u);
    out[1] = codes2(wh & 0xFFu, wh & 0xFF00u);
  }
}

// Two code rows (gate and up) sharing the same activations.
template <int BITS>
__device__ __forceinline__ void dot_chunk2(const uint4& qa, const uint4& qb, const float4* x4, int ns,
                                           float& da, float& db) {
  float2 a0 = make_float2(0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
  if constexpr (BITS == 4) {
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t wa = word_of(qa, wi), wah = wa >> 12;
      const uint32_t wb = word_of(qb, wi), wbh = wb >> 12;
      const float4 xa = x4[(2 * wi) * ns], xb = x4[(2 * wi + 1) * ns];
      const float2 x01 = make_float2(xa.x, xa.y), x23 = make_float2(xa.z, xa.w);
      const float2 x45 = make_float2(xb.x, xb.y), x67 = make_float2(xb.z, xb.w);
      a0 = ffma2(codes2(wa & 0xFu, wa & 0xF0u), x01, a0);
      a1 = ffma2(codes2(wa & 0xF00u, wa & 0xF000u), x23, a1);
      a0 = ffma2(codes2(wa & 0xF0000u, wah & 0xF00u), x45, a0);
      a1 = ffma2(codes2(wah & 0xF000u, wah & 0xF0000u), x67, a1);
      b0 = ffma2(codes2(wb & 0xFu, wb & 0xF0u), x01, b0);
      b1 = ffma2(codes2(wb & 0xF00u, wb & 0xF000u), x23, b1);
      b0 = ffma2(codes2(wb & 0xF0000u, wbh & 0xF00u), x45, b0);
      b1 = ffma2(codes2(wbh & 0xF000u, wbh & 0xF0000u), x67, b1);
    }
  } else {
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t wa = word_of(qa, wi), wah = wa >> 16;
      const uint32_t wb = word_of(qb, wi), wbh = wb >> 16;
      const float4 xa = x4[wi * ns];
      const float2 x01 = make_float2(xa.x, xa.y), x23 = make_float2(xa.z, xa.w);
      a0 = ffma2(codes2(wa & 0xFFu, wa & 0xFF00u), x01, a0);
      a1 = ffma2(codes2(wah & 0xFFu, wah & 0xFF00u), x23, a1);
      b0 = ffma2(codes2(wb & 0xFFu, wb & 0xFF00u), x01, b0);
      b1 = ffma2(codes2(wbh & 0xFFu, wbh & 0xFF00u), x23, b1);
    }
  }
  da = (a0.x + a0.y) + (a1.x + a1.y);
  db = (b0.x + b0.y) + (b1.x + b1.y);
}

// Stages `rows` vectors of K activations (fp32 or bf16 source) into the chunk-interleaved
// shared layout: float4 v of chunk c of vector r at s4[(r*V4 + v)*NC + c] (consecutive lanes
// read consecutive 16-byte words), and the chunk sums at sums[r*NC + c].  Threads
// tid = 0..nthreads-1 of the block take part.
template <int BITS, int K, typename Load>
__device__ __forceinline__ void stage_vectors(float4* s4, float* sums, int rows, int tid, int nthreads, Load load) {
  constexpr int CC = 128 / BITS, NC = K / CC, V4 = CC / 4;
  for (int i = tid; i < rows * NC; i += nthreads) {
    const int r = i / NC, c = i - r * NC;
    float sum = 0.f;
#pragma unroll
    for (int v = 0; v < V4; ++v) {
      const float4 f = load(r, c * CC + 4 * v);
      sum += (f.x + f.y) + (f.z + f.w);
      const int j = 4 * v;
      s4[(r * V4 + v) * NC + c] =
          make_float4(f.x * stage_scale<BITS>(j), f.y * stage_scale<BITS>(j + 1),
                      f.z * stage_scale<BITS>(j + 2), f.w * stage_scale<BITS>(j + 3));
    }
    sums[r * NC + c] = sum;
  }
}

}  // namespace moe
