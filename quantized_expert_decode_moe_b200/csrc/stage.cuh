// Staging helpers of the decode kernels (sm_100a): windows of per-row scale
// and bias arrays for bulk copies, activation chunk loads for the operand
// tables, and the SwiGLU activation.
#pragma once

#include "common.cuh"

namespace qmoe {

// 16-byte aligned window of rows [r0, r0+n) of a per-row array of SRB bytes
// per row; `pre` = offset of row r0 inside the window. The window ends inside
// the array: its size R*SRB is a multiple of 16 (R a multiple of 16, SRB of 4).
__host__ __device__ __forceinline__ unsigned sb_window(int r0, int n, int SRB, int& pre) {
  const unsigned o = (unsigned)r0 * (unsigned)SRB, e = o + (unsigned)n * (unsigned)SRB;
  const unsigned oa = o & ~15u, ea = (e + 15u) & ~15u;
  pre = (int)(o - oa);
  return ea - oa;
}
__host__ __device__ __forceinline__ int sb_region(int rows, int SRB) { return (rows * SRB + 32 + 15) & ~15; }

__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + expf(-z)); }

// Loads the table builder's elements of chunk q of a bf16 vector.
template <int BITS>
__device__ __forceinline__ void load_chunk_bf16(const uint16_t* x, int q, float (&v)[TabTraits<BITS>::kEPT]) {
  constexpr int EPT = TabTraits<BITS>::kEPT;
  const uint4* p = (const uint4*)(x + (size_t)q * EPT);
#pragma unroll
  for (int u = 0; u < EPT / 8; ++u) {
    const uint4 r = __ldcg(p + u);
    const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[8 * u + 2 * i] = bf16lo(w4[i]); v[8 * u + 2 * i + 1] = bf16hi(w4[i]); }
  }
}
template <int BITS>
__device__ __forceinline__ void load_chunk_f32(const float* a, int q, float (&v)[TabTraits<BITS>::kEPT]) {
  constexpr int EPT = TabTraits<BITS>::kEPT;
  const float4* p = (const float4*)(a + (size_t)q * EPT);
#pragma unroll
  for (int u = 0; u < EPT / 4; ++u) {
    const float4 r = __ldcg(p + u);
    v[4 * u] = r.x; v[4 * u + 1] = r.y; v[4 * u + 2] = r.z; v[4 * u + 3] = r.w;
  }
}

// 16 bytes of scale or bias data (4 spans x a bf16 pair) at p: one 16-byte
// load when the per-row arrays keep 16-byte alignment, else four 4-byte loads.
__device__ __forceinline__ uint4 lds_chunk(const unsigned char* p, bool al16) {
  if (al16) return *(const uint4*)p;
  const uint32_t* q = (const uint32_t*)p;
  return make_uint4(q[0], q[1], q[2], q[3]);
}
__device__ __forceinline__ uint32_t chunk_word(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

}  // namespace qmoe
