// nvfp4.cuh -- NVFP4 block quantisation on the device.
//
// NVFP4 is the 4-bit tier of the Blackwell low-precision recipes (the
// Megatron Core MoE technical summary, sections 2.4 and 3, runs the expert
// GEMMs in FP8/FP4 and lists an NVFP4 recipe; the format itself is NVIDIA's):
//   elements  E2M1 (OCP MX v1.0 section 5.3.3: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6),
//             two per byte, element 2i in the low nibble of byte i;
//   blocks    16 consecutive elements along K share one positive E4M3 scale
//             s = e4m3((amax / 6) * G), nearest-even, at most 448;
//   tensor    an fp32 encode scale G per tensor: 6 * 448 / amax(tensor) for a
//             weight matrix (so its largest block scale is 448), 1 for
//             activations, whose amax is not known when they are produced.
//   element i = e2m1(v_i * (G / s)) (nearest-even, saturating at 6; 0 when s == 0),
//   decoded value = code * s / G.
// Every step is one IEEE fp32 operation in that order, so the codes do not
// depend on contraction or on the compiler.
#pragma once

#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace nvq {

// Value of a non-negative E4M3 code (exact).
MOE_DEV float e4m3_pos_value(uint8_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  if (e == 0) return (float)m * 0.001953125f;  // subnormal: m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Block scale byte: (amax / 6) * G, rounded to E4M3.
MOE_DEV uint8_t scale_byte(float amax, float G) {
  const float s = __fmul_rn(__fdiv_rn(amax, 6.0f), G);
  return (uint8_t)__nv_cvt_float_to_fp8(s, __NV_SATFINITE, __NV_E4M3);
}

// Element multiplier G / s of a block with scale byte sb (0 for a zero scale).
MOE_DEV float elem_mult(uint8_t sb, float G) {
  const float sd = e4m3_pos_value(sb);
  return sd > 0.f ? __fdiv_rn(G, sd) : 0.f;
}

// Eight values times r -> eight E2M1 codes in one 32-bit word (element 2i in the low nibble of byte i).
MOE_DEV uint32_t pack8(const float* v, float r) {
  uint32_t w = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_fp4x2_storage_t b =
        __nv_cvt_float2_to_fp4x2(make_float2(__fmul_rn(v[2 * i], r), __fmul_rn(v[2 * i + 1], r)), __NV_E2M1,
                                 cudaRoundNearest);
    w |= (uint32_t)b << (8 * i);
  }
  return w;
}

// One 16-block: scale byte and the eight packed bytes (two words).
MOE_DEV uint8_t quant16(const float* v, float G, uint32_t& w0, uint32_t& w1) {
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) am = fmaxf(am, fabsf(v[i]));
  const uint8_t sb = scale_byte(am, G);
  const float r = elem_mult(sb, G);
  w0 = pack8(v, r);
  w1 = pack8(v + 8, r);
  return sb;
}

}  // namespace nvq
