// quant_math.cuh — per-element arithmetic of the dynamic quantisers, shared
// by the standalone quantisation kernels and the GEMM's fused activation
// prologue so that both produce the same codes and scales bit for bit:
//   scale = amax / Qmax (correctly rounded fp32 division), 1 for amax = 0;
//   code  = round-to-nearest-even(x / scale) (correctly rounded division),
//           saturating: e4m3 to +-448, int8 to [-127, 127].
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace qg {

__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ float absmax8(const float (&x)[8]) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
  return m;
}

// Two e4m3 codes: `lo` goes to the low byte (the lower K index).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Eight e2m1 codes -> 32 bits, element 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
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
// Exact decode of one e4m3 code (every e4m3 value is an f16 value).
__device__ __forceinline__ float dec_e4m3(uint32_t code) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(code & 0xFF)));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

// Codes of 8 values against one scale: 8 bytes (e4m3 or int8), each the
// correctly rounded quotient x / s rounded once more to the format.
template <bool INT8>
__device__ __forceinline__ uint2 quant8(const float (&x)[8], float s) {
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t acc = 0;
    if constexpr (INT8) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        int q = __float2int_rn(__fdiv_rn(x[4 * h + i], s));
        q = max(-127, min(127, q));
        acc |= ((uint32_t)(q & 0xFF)) << (8 * i);
      }
    } else {
      const uint32_t a = cvt_e4m3x2(__fdiv_rn(x[4 * h + 0], s), __fdiv_rn(x[4 * h + 1], s));
      const uint32_t b = cvt_e4m3x2(__fdiv_rn(x[4 * h + 2], s), __fdiv_rn(x[4 * h + 3], s));
      acc = a | (b << 16);
    }
    w[h] = acc;
  }
  return make_uint2(w[0], w[1]);
}

// Scale of a row or group from its amax.
template <bool INT8>
__device__ __forceinline__ float scale_of_amax(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, INT8 ? 127.f : 448.f) : 1.f;
}

}  // namespace qg
