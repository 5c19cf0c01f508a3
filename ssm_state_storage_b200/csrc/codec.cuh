// codec.cuh -- FP8 E4M3 and NVFP4 (E2M1 + E4M3 block scale + fp32 tile scale)
// conversions for the low-precision read copy of the checkpoint.
//
// Element formats: OCP Microscaling Formats (MX) v1.0, sections 5.3 (E4M3) and
// 5.3.3 (E2M1).  Encoding uses the sm_100a cvt instructions with round to
// nearest even and saturation to the largest finite value.  NVFP4 tile
// quantisation, every step one correctly rounded fp32 operation:
//   s_g  = amax(tile) / 2688  (= 6 * 448; 1 for an all-zero tile)
//   s_b  = E4M3(amax(16-element block) / (6 * s_g))
//   code = E2M1(x / (s_b * s_g))      (0 when s_b * s_g == 0)
//   x'   = E2M1value(code) * s_b * s_g
// The low-precision copy serves reads only; the fp32 checkpoint carries the
// recurrence [sitech.ge, "NVIDIA ו-Dao AI Lab הציגו ReplaySSM…", §Bounding
// quantisation error].
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

namespace rssm {

// E4M3 code of v (low byte).
__device__ __forceinline__ uint32_t e4m3_encode(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// E4M3 code -> value, decoded from the bit fields (bias 7, subnormals at
// exponent field 0).  NaN codes do not occur in a saturating encode.
__device__ __forceinline__ float e4m3_decode(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
  float mag = (e == 0) ? __int2float_rn((int)m) * 0.001953125f  // m * 2^-9
                       : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (c & 0x80u) ? -mag : mag;
}

// Two E2M1 codes packed in one byte: lo in bits 0-3, hi in bits 4-7.
__device__ __forceinline__ uint32_t e2m1x2_encode(float lo, float hi) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// E2M1 code (4 bits) -> value: magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_decode(uint32_t c) {
  const uint32_t e = (c >> 1) & 3u, m = c & 1u;
  float mag = (e == 0) ? 0.5f * (float)m : __uint_as_float(((e + 126u) << 23) | (m << 22));
  return (c & 8u) ? -mag : mag;
}

// Two E4M3 codes (bits 0-7 and 8-15 of `two`) -> their values, by the
// hardware conversion to f16x2 (every E4M3 value is exact in f16); the low
// byte lands in .x.
__device__ __forceinline__ float2 e4m3x2_decode(uint32_t two) {
  uint32_t h2;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}"
      : "=r"(h2)
      : "r"(two));
  return __half22float2(*reinterpret_cast<const __half2 *>(&h2));
}

// Two E2M1 codes packed in one byte (lo nibble first) -> their values, by
// the hardware conversion to f16x2 (exact).
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte) {
  uint32_t h2;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}"
      : "=r"(h2)
      : "r"(byte));
  return __half22float2(*reinterpret_cast<const __half2 *>(&h2));
}

__device__ __forceinline__ float nvfp4_tile_scale(float amax) {
  return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Block scale code for a 16-element block with absolute maximum bmax.
__device__ __forceinline__ uint32_t nvfp4_block_code(float bmax, float sg) {
  return e4m3_encode(__fdiv_rn(bmax, __fmul_rn(6.0f, sg)));
}

// Element step d = s_b * s_g.
__device__ __forceinline__ float nvfp4_step(uint32_t sb_code, float sg) {
  return __fmul_rn(e4m3_decode(sb_code), sg);
}

__device__ __forceinline__ uint32_t nvfp4_pack2(float x0, float x1, float d) {
  if (!(d > 0.0f)) return 0u;
  return e2m1x2_encode(__fdiv_rn(x0, d), __fdiv_rn(x1, d));
}

__device__ __forceinline__ float nvfp4_value(uint32_t code, float d_sb, float sg) {
  // e2m1 * s_b is exact in fp32; the product with s_g is rounded once.
  return __fmul_rn(e2m1_decode(code) * d_sb, sg);
}

}  // namespace rssm
