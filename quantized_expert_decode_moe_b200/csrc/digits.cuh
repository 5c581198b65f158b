// Digit blocks: activations (x, or the SwiGLU outputs a) written once per call
// as exact fixed-point digit planes for the integer dot products of the
// digit-block layer kernels (mx.cu). Shared by those kernels and the decode
// router (kernels.cu), which writes x's blocks as a side job.
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "kernels.cuh"

namespace qmoe {

// 2^n for n in [-149, 127], from its bits (subnormal below 2^-126)
__device__ __forceinline__ float mx_pow2(int n) {
  return n >= -126 ? __int_as_float((n + 127) << 23) : __int_as_float(1 << (n + 149));
}

// ---- digit blocks (the layer kernels): a 32-value block of x or a as 22-bit fixed point with
// its own power of two, X = rint(v 2^p), max |v| 2^p < 2^22, split exactly into three balanced
// signed 8-bit digits (three 32-byte planes), then the factor 2^-(p+1) as a float at byte 96
// (the 1/2 undoes the MXFP4 codes' 2 e2m1; the affine kernels double it back) and the exact
// sum of the block's X as an int32 at byte 100 (|sum| <= 2^27; the affine bias term). bf16
// values within 2^-14 of the block's largest are exact, others round within 2^-23 of it.
// Within a plane the digits follow the order in which the matrix codes expand to bytes
// (mx_dig_pos). Written once per call: x's by the decode router (route_logits_kernel) or by
// mx_digits_kernel, a's by the gate/up kernel.
constexpr int kMxDig = 112;   // bytes per digit block (96 digits, the factor, the sum, padding to 16)

// Byte of element k (0..31) of a block within a digit plane. MXFP4: element order (a half-word
// of codes expands to elements 8i..8i+3). 4-bit: per 8 elements, the even ones then the odd
// ones (the low and the high nibbles of a code word, masked). 2-bit: per 16 elements, stride 4
// (code word w shifted by 2j and masked holds elements j, j+4, j+8, j+12).
__device__ __forceinline__ int mx_dig_pos(int k, int codec) {
  if (codec == kCodecQ4) return (k & ~7) | ((k & 1) << 2) | ((k >> 1) & 3);
  if (codec == kCodecQ2) return (k & ~15) | ((k & 3) << 2) | ((k >> 2) & 3);
  return k;
}

// The digit block of 32 values held one per lane (lane k: value k), written to o; the whole warp
// calls it. The block's largest magnitude by warp shuffles, each lane's three digit bytes stored
// directly, the factor and the padding by lane 0.
__device__ __forceinline__ void mx_digit_lanes(float v, int lane, uint8_t* o, int codec) {
  const float m = warp_max(fabsf(v));
  int p = 0;
  if (m > 0.f) {   // m = f 2^E, f in [0.5, 1); below 2^-126 treated as 2^-126
    const int E = m >= 0x1p-126f ? (int)((__float_as_uint(m) >> 23) & 0xFFu) - 126 : -125;
    p = 22 - E;
  }
  const int X = __float2int_rn(v * mx_pow2(p / 2) * mx_pow2(p - p / 2));   // |X| <= 2^22
  const int d0 = ((X + 128) & 255) - 128;
  const int X1 = (X - d0) / 256;
  const int d1 = ((X1 + 128) & 255) - 128;
  const int d2 = (X1 - d1) / 256;
  const int at = mx_dig_pos(lane, codec);
  o[at] = (uint8_t)(d0 & 255);
  o[32 + at] = (uint8_t)(d1 & 255);
  o[64 + at] = (uint8_t)(d2 & 255);
  const int sum = __reduce_add_sync(0xffffffffu, X);
  if (lane == 0)
    *(uint4*)(o + 96) = make_uint4(__float_as_uint(-p - 1 >= -149 ? mx_pow2(-p - 1) : 0.f), (uint32_t)sum, 0u, 0u);
}

}  // namespace qmoe
