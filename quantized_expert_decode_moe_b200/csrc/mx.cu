// MXFP4 expert matrices: the third codec. The page on running a 300B MoE from
// a 32 GB laptop ("300b on 32gb MoE-streaming findings + optimisations")
// streams MXFP4 experts; the format is read as the OCP Microscaling (MX) v1.0
// definition: FP4 E2M1 elements (sign, two exponent bits with bias 1, one
// mantissa bit; values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their negatives), one
// E8M0 scale 2^(byte - 127) per 32 consecutive k (byte 0xFF is NaN). Codes use
// the 4-bit packing (element k of a row in word k/8 at bits 4(k%8), LSB first),
// scales are uint8 [R][K/32].
//
// Two entry points:
//  * mx_gemv_kernel: y = W x (decode). A warp per row, a lane per 32-element
//    block: the 16 code bytes of the block in one load. A code's magnitude
//    field f, shifted to bit 22 of an fp32 word, is |v| 2^-126 exactly (f = 1,
//    the subnormal E2M1 value 0.5, lands on the fp32 subnormal 2^-127), and its
//    sign bit goes to bit 31: three integer operations per element, then
//    packed fp32x2 FMAs against x staged per block as x 2^s (the block's
//    largest |x| brought near 2^50, so every product is a normal float); the
//    block sum times 2^(126 - s) and the E8M0 scale 2^(byte - 127).
//  * mx_gemm_kernel: Y = X W^T for many tokens on the tcgen05 tensor cores,
//    kind::mxf4 with block scaling: the weight codes go from HBM to shared
//    memory unchanged (TMA tiles of 16 bytes x 128 rows, i.e. one MX block of
//    128 rows) and the MMA applies the weight's E8M0 scales itself. The bf16
//    activations are written as a sum of kMxTerms E2M1 terms, each with its
//    own E8M0 scale per 32-block (mx_prep_kernel): term j is the residual's
//    block maximum scaled to at most 6, rounded to the nearest E2M1 value, and
//    subtracted exactly (the rounded value lies within a factor of two of the
//    residual, so the fp32 subtraction is exact). Each term cuts the largest
//    residual of a block by a factor of at least four; after five terms it is
//    below 4^-4 / 3 of the block's maximum (about 5e-5 of the output's norm in
//    practice). All terms accumulate into one fp32 accumulator in tensor
//    memory, since each carries its own scales.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "digits.cuh"
#include "kernels.cuh"
#include "sync.cuh"
#include "tc.cuh"

namespace qmoe {

namespace cg = cooperative_groups;

// ------------------------------------------------------------------ mat-vec (decode)
constexpr int kMvWarps = 8;
constexpr int kMvXStride = 36;   // floats per 32-element block of x in shared memory (padded)

// the E8M0 scale 2^(byte - 127); NaN for 0xFF
__device__ __forceinline__ float mx_scale(unsigned byte) {
  return byte == 0xFFu ? __int_as_float(0x7FC00000) : mx_pow2((int)byte - 127);
}

// packed fp32x2 arithmetic (two values in one 64-bit register, the first in the low half)
__device__ __forceinline__ unsigned long long f2_pack(uint32_t lo, uint32_t hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float f2_sum(unsigned long long v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return lo + hi;
}

// element j of a code word as the fp32 bits of |v| 2^-126 with v's sign: the magnitude field
// at bit 22 (field 1, the subnormal value 0.5, is the fp32 subnormal 2^-127), the sign at bit 31
__device__ __forceinline__ uint32_t mx_code_bits(uint32_t w, int j) {
  const uint32_t mag = j <= 5 ? (w << (22 - 4 * j)) : (w >> (4 * j - 22));
  return ((w << (28 - 4 * j)) & 0x80000000u) | (mag & 0x01C00000u);
}

// sum over one 32-element block of e2m1(code_k) x_k; xs: the block as mx_stage_block left it
// (32 values x_k 2^s, then the factor 2^(126 - s) in slot 32)
__device__ __forceinline__ float mx_block_dot(const uint4 c, const float* xs) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  unsigned long long acc = 0ull;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const ulonglong2 xa = *(const ulonglong2*)(xs + 8 * i), xb = *(const ulonglong2*)(xs + 8 * i + 4);
    acc = f2_fma(f2_pack(mx_code_bits(w[i], 0), mx_code_bits(w[i], 1)), xa.x, acc);
    acc = f2_fma(f2_pack(mx_code_bits(w[i], 2), mx_code_bits(w[i], 3)), xa.y, acc);
    acc = f2_fma(f2_pack(mx_code_bits(w[i], 4), mx_code_bits(w[i], 5)), xb.x, acc);
    acc = f2_fma(f2_pack(mx_code_bits(w[i], 6), mx_code_bits(w[i], 7)), xb.y, acc);
  }
  return f2_sum(acc) * xs[32];
}

// Stages one 32-value block: x 2^s, with s the power of two that brings the block's largest |x|
// into [2^50, 2^51) (clamped to [-1, 126], so 2^s and the factor 2^(126 - s) are normal floats),
// then the factor in slot 32. Exact: scaling by powers of two.
__device__ __forceinline__ void mx_stage_block(const float (&v)[32], float* dst) {
  float m = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(v[k]));
  int sc = 0;
  if (m > 0.f) {
    const int e = m >= 0x1p-126f ? (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127 : -127;   // floor(log2 m)
    sc = min(126, max(-1, 50 - e));
  }
  const float up = mx_pow2(sc);
#pragma unroll
  for (int k = 0; k < 32; k += 4)
    *(float4*)(dst + k) = make_float4(v[k] * up, v[k + 1] * up, v[k + 2] * up, v[k + 3] * up);
  dst[32] = mx_pow2(126 - sc);
}
// one block of 32 fp32 / 32 bf16 values from global memory into shared memory
__device__ __forceinline__ void mx_stage_f32(const float* src, float* dst) {
  float v[32];
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 q = __ldg((const float4*)(src + k));
    v[k] = q.x; v[k + 1] = q.y; v[k + 2] = q.z; v[k + 3] = q.w;
  }
  mx_stage_block(v, dst);
}
__device__ __forceinline__ void mx_stage_bf16(const uint16_t* src, float* dst) {
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg((const uint4*)src + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[8 * i + 2 * h] = bf16lo(w[h]);
      v[8 * i + 2 * h + 1] = bf16hi(w[h]);
    }
  }
  mx_stage_block(v, dst);
}

// prmt.b32 in its generic mode: byte n of the result is byte (c >> 4n) & 7 of b:a, or, where bit
// 4n + 3 of c is set, that byte's sign bit replicated; only the low 16 bits of c are read.
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The signed bytes 2 e2m1(code) (-12 .. 12) of the four codes in the low 16 bits of s, given sn =
// s with every code's sign bit flipped. The code itself selects from a byte table of the values
// 2 e2m1 (all below 0x80): a set sign bit turns its byte into 0, so p holds the positive codes'
// values; the flipped codes give the negative codes' magnitudes n; 0x80 - n per byte never
// borrows (n <= 12) and, with the top bit flipped back, is -n as a byte.
__device__ __forceinline__ uint32_t mx_q4(uint32_t s, uint32_t sn) {
  const uint32_t p = prmt_b32(0x03020100u, 0x0C080604u, s);    //  0, 1, 2, 3 | 4, 6, 8, 12
  const uint32_t n = prmt_b32(0x03020100u, 0x0C080604u, sn);
  return p | ((0x80808080u - n) ^ 0x80808080u);
}

// Sum over one 32-element block of e2m1(code_k) x_k, x as a digit block: the integer sums of the
// codes (as 2 e2m1) times each digit plane (dp4a, four products an instruction) combine exactly
// in 32 bits (|sum of 2 e2m1(c) X| <= 32 * 12 * 2^22 < 2^31), then one conversion and the block's
// factor.
__device__ __forceinline__ float mx_block_dot_dig(const uint4 c, const uint8_t* d) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  const uint4* dp = (const uint4*)d;
  const uint4 p0a = dp[0], p0b = dp[1], p1a = dp[2], p1b = dp[3], p2a = dp[4], p2b = dp[5];
  const uint32_t d0[8] = {p0a.x, p0a.y, p0a.z, p0a.w, p0b.x, p0b.y, p0b.z, p0b.w};
  const uint32_t d1[8] = {p1a.x, p1a.y, p1a.z, p1a.w, p1b.x, p1b.y, p1b.z, p1b.w};
  const uint32_t d2[8] = {p2a.x, p2a.y, p2a.z, p2a.w, p2b.x, p2b.y, p2b.z, p2b.w};
  int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t wn = w[i] ^ 0x88888888u;
    const int lo = (int)mx_q4(w[i], wn), hi = (int)mx_q4(w[i] >> 16, wn >> 16);   // elements 8i..8i+3, 8i+4..8i+7
    s0 = __dp4a(lo, (int)d0[2 * i], s0); s0 = __dp4a(hi, (int)d0[2 * i + 1], s0);
    s1 = __dp4a(lo, (int)d1[2 * i], s1); s1 = __dp4a(hi, (int)d1[2 * i + 1], s1);
    s2 = __dp4a(lo, (int)d2[2 * i], s2); s2 = __dp4a(hi, (int)d2[2 * i + 1], s2);
  }
  return (float)(s0 + s1 * 256 + s2 * 65536) * __uint_as_float(((const uint32_t*)d)[24]);
}

// The digit planes of a block as 8 words each.
struct MxPlanes {
  uint32_t d0[8], d1[8], d2[8];
};
__device__ __forceinline__ MxPlanes mx_planes(const uint8_t* d) {
  const uint4* dp = (const uint4*)d;
  const uint4 p0a = dp[0], p0b = dp[1], p1a = dp[2], p1b = dp[3], p2a = dp[4], p2b = dp[5];
  return MxPlanes{{p0a.x, p0a.y, p0a.z, p0a.w, p0b.x, p0b.y, p0b.z, p0b.w},
                  {p1a.x, p1a.y, p1a.z, p1a.w, p1b.x, p1b.y, p1b.z, p1b.w},
                  {p2a.x, p2a.y, p2a.z, p2a.w, p2b.x, p2b.y, p2b.z, p2b.w}};
}

// Sum over one 32-element block of q_k X_k for 4-bit codes q (0..15) and a digit block in the
// 4-bit order: the low and the high nibbles of each code word, masked, are four unsigned bytes
// each (elements 8i + 0, 2, 4, 6 and 8i + 1, 3, 5, 7); exact in 32 bits (32 * 15 * 2^22 < 2^31).
__device__ __forceinline__ int dq4_block_dot(const uint4 c, const uint8_t* d) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  const MxPlanes P = mx_planes(d);
  int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int lo = (int)(w[i] & 0x0F0F0F0Fu), hi = (int)((w[i] >> 4) & 0x0F0F0F0Fu);
    s0 = __dp4a(lo, (int)P.d0[2 * i], s0); s0 = __dp4a(hi, (int)P.d0[2 * i + 1], s0);
    s1 = __dp4a(lo, (int)P.d1[2 * i], s1); s1 = __dp4a(hi, (int)P.d1[2 * i + 1], s1);
    s2 = __dp4a(lo, (int)P.d2[2 * i], s2); s2 = __dp4a(hi, (int)P.d2[2 * i + 1], s2);
  }
  return s0 + s1 * 256 + s2 * 65536;
}

// The same for 2-bit codes (two words per block): word i shifted by 2j and masked holds
// elements 16i + j, + 4, + 8, + 12, the 2-bit order of the digit block.
__device__ __forceinline__ int dq2_block_dot(const uint2 c, const uint8_t* d) {
  const uint32_t w[2] = {c.x, c.y};
  const MxPlanes P = mx_planes(d);
  int s0 = 0, s1 = 0, s2 = 0;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = (int)((w[i] >> (2 * j)) & 0x03030303u);
      s0 = __dp4a(r, (int)P.d0[4 * i + j], s0);
      s1 = __dp4a(r, (int)P.d1[4 * i + j], s1);
      s2 = __dp4a(r, (int)P.d2[4 * i + j], s2);
    }
  return s0 + s1 * 256 + s2 * 65536;
}

// grid ceil(rows K/32 / 8), block 256: the digit blocks of rows of K bf16 values,
// dst[row][K/32][kMxDig], a warp per block. It reads the rows without waiting: under a
// programmatic launch it follows a kernel that triggered its dependents only after its own wait
// (so the rows' writer, two launches back, has completed). It waits for that kernel before it
// exits, so that whatever waits for this one also finds that one complete.
__global__ void __launch_bounds__(256) mx_digits_kernel(const uint16_t* __restrict__ src, int rows, int K,
                                                        uint8_t* __restrict__ dst, int codec) {
  griddep_launch_dependents();
  const size_t wi = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;   // the warp's block
  const int lane = threadIdx.x & 31, nb = K / 32;
  if (wi < (size_t)rows * nb)   // whole warps
    mx_digit_lanes(bf16_to_f32(__ldg(src + (wi / nb) * K + (wi % nb) * 32 + lane)), lane, dst + wi * kMxDig, codec);
  griddep_wait();
}

// grid ceil(R / kMvWarps), block 32 kMvWarps: warp w of CTA b computes row b kMvWarps + w.
__global__ void __launch_bounds__(kMvWarps * 32) mx_gemv_kernel(const uint32_t* __restrict__ q,
                                                                const uint8_t* __restrict__ e, int R, int K,
                                                                const float* __restrict__ x, float* __restrict__ y) {
  extern __shared__ __align__(16) float xs[];   // [K/32][kMvXStride]
  const int nb = K / 32;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) mx_stage_f32(x + 32 * b, xs + b * kMvXStride);
  __syncthreads();
  const int lane = threadIdx.x & 31, r = blockIdx.x * kMvWarps + (threadIdx.x >> 5);
  if (r >= R) return;
  const uint4* qr = (const uint4*)(q + (size_t)r * (K / 8));
  const uint8_t* er = e + (size_t)r * nb;
  float acc = 0.f;
  for (int b0 = 0; b0 < nb; b0 += 4 * 32) {   // four blocks per lane in flight
    uint4 c[4];
    unsigned sb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b = b0 + 32 * u + lane;
      c[u] = b < nb ? __ldg(qr + b) : make_uint4(0u, 0u, 0u, 0u);
      sb[u] = b < nb ? __ldg(er + b) : 0u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b = b0 + 32 * u + lane;
      if (b < nb) acc = fmaf(mx_block_dot(c[u], xs + b * kMvXStride), mx_scale(sb[u]), acc);
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) y[r] = acc;
}

cudaError_t launch_mx_gemv(const uint32_t* q, const uint8_t* e, int R, int K, const float* x, float* y,
                           cudaStream_t s) {
  const size_t sm = sizeof(float) * (size_t)(K / 32) * kMvXStride;
  cudaError_t err = set_func_attr((const void*)mx_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
  if (err != cudaSuccess) return err;
  mx_gemv_kernel<<<(R + kMvWarps - 1) / kMvWarps, kMvWarps * 32, sm, s>>>(q, e, R, K, x, y);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ many tokens (tcgen05 kind::mxf4)
constexpr int kMxTerms = 5;                      // E2M1 terms of an activation block
constexpr int kMxM = 128, kMxN = 128;            // weight rows, tokens per CTA
constexpr int kMxKS = 128;                       // columns per stage: four MX blocks
constexpr int kMxStages = 4;
constexpr int kMxChunk = 128 * 16;               // one MX block (16 bytes of codes) of 128 rows
constexpr int kMxTileA = 4 * kMxChunk;           // 8 KB
constexpr int kMxTileB = kMxTerms * 4 * kMxChunk;   // 40 KB: the terms of 128 tokens
constexpr int kMxSf = 512;                       // scales of 128 rows x 4 blocks
constexpr int kMxStageBytes = kMxTileA + kMxTileB + kMxSf * (1 + kMxTerms);
constexpr int kMxSfCols = 4 * (1 + kMxTerms);    // tensor-memory columns of one stage's scales
constexpr int kMxPrepThreads = 128;
constexpr int kMxSplitMax = 8;                   // column splits of the product at most
constexpr int kMxWaveCtas = 148;                 // CTAs of one wave (one per SM of a B200)

static_assert(kMxStageBytes % 1024 == 0, "stages stay 1 KB aligned");
static_assert(kMxN + kMxStages * kMxSfCols <= 256, "accumulator and scales fit 256 tensor-memory columns");

// Byte offset of a scale in a 512-byte block of 128 rows x 4 blocks: row m =
// m0 + 32 m1 and block j at m0 16 + m1 4 + j. Copied to tensor memory by
// tcgen05.cp 32x128b.warpx4, that puts the four scales of row m0 + 32 m1 in
// column m1 of lane m0 of every 32-lane group, the layout the block-scaled
// MMA reads (scale j of the word selected by the descriptor's scale id).
__host__ __device__ __forceinline__ int mx_sf_off(int m, int j) { return (m & 31) * 16 + (m >> 5) * 4 + j; }

// grid T_pad q + ceil(R nstg / kMxPrepThreads) with q = ceil(4 (K/32) / kMxPrepThreads),
// block kMxPrepThreads.
//  CTA t q + j (t < T_pad): token row t (zeros beyond T). Four adjacent threads take one
//   32-element block b (thread i of the CTA: task j kMxPrepThreads + i, block task / 4, quarter
//   task % 4 = elements 8 quarter .. +7, one code word); the block's maximum per term is reduced
//   over the four with shuffles. Per term the code word goes to
//   bq[(((t/128) nstg + b/4) kMxTerms + term) kMxTileA + (b%4) kMxChunk + (t%128) 16 + 4 quarter]
//   and (quarter 0) the scale byte to bsf[(((t/128) nstg + b/4) kMxTerms + term) 512 + mx_sf_off(t%128, b%4)].
//  CTA T_pad q + s: scale words i = s kMxPrepThreads + thread (row i / nstg, stage
//   i % nstg: the row's four scales of that stage), rearranged into the same
//   512-byte blocks, asf[((row/128) nstg + stage) 512 + mx_sf_off(row%128, 0)].
__global__ void __launch_bounds__(kMxPrepThreads) mx_prep_kernel(const uint16_t* __restrict__ x, int T, int Tpad,
                                                                 const uint8_t* __restrict__ e, int R, int K,
                                                                 uint8_t* __restrict__ bq, uint8_t* __restrict__ bsf,
                                                                 uint8_t* __restrict__ asf) {
  const int nb = K / 32, nstg = K / kMxKS;
  const int q = (4 * nb + kMxPrepThreads - 1) / kMxPrepThreads;
  if ((int)blockIdx.x >= Tpad * q) {   // weight scales: one 4-byte word (4 blocks, K % 128 == 0) per thread
    const size_t i = (size_t)(blockIdx.x - Tpad * q) * kMxPrepThreads + threadIdx.x;
    if (i >= (size_t)R * nstg) return;
    const int r = (int)(i / nstg), g = (int)(i % nstg);
    const uint32_t w = __ldg((const uint32_t*)e + i);
    *(uint32_t*)(asf + ((size_t)(r / kMxM) * nstg + g) * kMxSf + mx_sf_off(r % kMxM, 0)) = w;
    return;
  }
  const int t = blockIdx.x / q, task = (blockIdx.x % q) * kMxPrepThreads + threadIdx.x;
  const int b = task >> 2, qt = task & 3, tt = t / kMxN, rr = t % kMxN;
  // every thread of a group of four takes part in the shuffles; a group past the row's last block
  // has no block (b >= nb) and stores nothing
  const bool in = b < nb;
  float v[8];
  if (in && t < T) {
    const uint4 u = __ldg((const uint4*)(x + (size_t)t * K + 32 * b + 8 * qt));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[2 * h] = bf16lo(w[h]);
      v[2 * h + 1] = bf16hi(w[h]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = 0.f;
  }
  const int g = b / 4, c = b % 4;
#pragma unroll 1
  for (int term = 0; term < kMxTerms; ++term) {
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    // the smallest power 2^u with m <= 6 2^u, no smaller than 2^-127 (every m below 2^-126 takes
    // u = -127): with m = f 2^E, f in [0.5, 1), u = E - 3 if f <= 0.75, else E - 2
    int u = -127;
    if (m >= 0x1p-126f) {
      const uint32_t bits = __float_as_uint(m);
      const int E = (int)((bits >> 23) & 0xFFu) - 126;
      u = max(-127, (bits & 0x7FFFFFu) <= 0x400000u ? E - 3 : E - 2);
    }
    const float down = mx_pow2(-u), up = mx_pow2(u);   // 2^-u, 2^u
    uint32_t code = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      // a = |v| 2^-u in [0, 6] (exact unless it underflows, far below 0.25), rounded to the nearest
      // E2M1 value: from 1 up, one mantissa bit (add half of it to the float's bits, then drop the
      // rest: 1, 1.5, 2, 3, 4, 6; code 2 (exponent + 1) + mantissa bit); below 1, rint(2a) halves
      // (0, 0.5, 1; code = rint(2a))
      const float a = fabsf(v[k] * down);
      const uint32_t rb = (__float_as_uint(a) + 0x200000u) & 0xFFC00000u;
      const int hi_code = (int)(((rb >> 23) - 126u) << 1 | ((rb >> 22) & 1u));
      const int lo_code = __float2int_rn(2.f * a);
      const bool big = a >= 1.f;
      const int idx = big ? hi_code : lo_code;
      const float r = big ? __uint_as_float(rb) : 0.5f * (float)lo_code;
      const bool neg = v[k] < 0.f;
      v[k] -= (neg ? -r : r) * up;   // exact: r has two significant bits and is 0 or within a factor of two of a
      code |= (uint32_t)(idx | (neg ? 8 : 0)) << (4 * k);
    }
    if (in) {
      const size_t blk = ((size_t)tt * nstg + g) * kMxTerms + term;
      *(uint32_t*)(bq + blk * kMxTileA + (size_t)c * kMxChunk + (size_t)rr * 16 + 4 * qt) = code;
      if (qt == 0) bsf[blk * kMxSf + mx_sf_off(rr, c)] = (uint8_t)(u + 127);
    }
  }
}

// grid (R/128, T_pad/128), block 128. Stage u (columns 128u .. 128u+127):
// the weight codes by four TMA tiles (16 bytes x 128 rows each, one MX block,
// at byte c kMxChunk), then the tokens' terms (one bulk copy of kMxTileB) and
// the scales of the weight rows and of the terms (512 bytes each). Thread 0
// loads; thread 32 copies the stage's scales into tensor memory (tcgen05.cp)
// and issues per term two MMAs of K = 64 (blocks 2h, 2h+1: scale id 2h); all
// four warps read the accumulator (lane = weight row) and write Y[t][r].
struct MxSmem {
  uint64_t full[kMxStages], empty[kMxStages], done;
  uint32_t tslot;
  int abort;
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      :: "r"(smem_u32(dst)), "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

// kind::mxf4 instruction descriptor: E2M1 A and B (format 1), both K-major,
// N >> 3 at bit 17, E8M0 scales (bit 23), M >> 4 at bit 24, scale ids of B
// (bits 4-5) and A (bits 29-30), K = 64.
__device__ __forceinline__ uint32_t mx_idesc(int sf_id) {
  return ((uint32_t)sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kMxN >> 3) << 17) | (1u << 23) |
         ((uint32_t)(kMxM >> 4) << 24) | ((uint32_t)sf_id << 29);
}

struct MxGemmParams {
  int R, K, T, splits;
  float* part;         // [splits][T][R] partial products when splits > 1
  const uint8_t* bq;   // the tokens' terms (prep layout)
  const uint8_t* bsf;  // their scales
  const uint8_t* asf;  // the weight scales, rearranged
  float* y;            // [T][R]
  uint32_t* status;
  unsigned long long wait_ns;
};

__global__ void __launch_bounds__(128, 1) mx_gemm_kernel(const __grid_constant__ CUtensorMap wmap, MxGemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  MxSmem& S = *(MxSmem*)(smem + kMxStages * kMxStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int mt = blockIdx.x, nt = blockIdx.y, nstg = p.K / kMxKS;
  const int i0 = (int)((long long)nstg * blockIdx.z / p.splits), n = (int)((long long)nstg * (blockIdx.z + 1) / p.splits) - i0;
  const unsigned long long wait_ns = p.wait_ns;
  uint32_t* status = p.status;
  if (tid == 0) {
    for (int s = 0; s < kMxStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.done, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(&S.tslot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tslot;
  volatile int* abort_flag = &S.abort;

  if (tid == 0) {   // ---------------------------------------------------- loads
    int last[kMxStages];
    for (int s = 0; s < kMxStages; ++s) last[s] = -1;
    for (int u = 0; u < n; ++u) {
      const int slot = u % kMxStages, use = u / kMxStages, g = i0 + u;
      if (use > 0 && !mbar_wait_bounded(&S.empty[slot], (use - 1) & 1, wait_ns, status)) *abort_flag = 1;
      if (*abort_flag) break;
      unsigned char* st = smem + (size_t)slot * kMxStageBytes;
      mbar_expect_tx(&S.full[slot], (unsigned)kMxStageBytes);
      for (int c = 0; c < 4; ++c) tma_load_2d(st + c * kMxChunk, &wmap, g * (kMxKS / 2) + 16 * c, mt * kMxM, &S.full[slot]);
      const size_t bstage = (size_t)nt * nstg + g;
      bulk_g2s(st + kMxTileA, p.bq + bstage * kMxTileB, kMxTileB, &S.full[slot]);
      bulk_g2s(st + kMxTileA + kMxTileB, p.asf + ((size_t)mt * nstg + g) * kMxSf, kMxSf, &S.full[slot]);
      bulk_g2s(st + kMxTileA + kMxTileB + kMxSf, p.bsf + bstage * kMxTerms * kMxSf, kMxTerms * kMxSf, &S.full[slot]);
      last[slot] = use;
    }
    for (int s = 0; s < kMxStages; ++s)   // no copy may land after the CTA has left
      if (last[s] >= 0) mbar_wait_bounded(&S.full[s], last[s] & 1, wait_ns, status);
  } else if (tid == 32) {   // --------------------------------------------- scales to tensor memory, MMAs
    bool started = false;
    for (int u = 0; u < n; ++u) {
      const int slot = u % kMxStages, ph = (u / kMxStages) & 1;
      if (!mbar_wait_bounded(&S.full[slot], ph, wait_ns, status)) *abort_flag = 1;
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + (size_t)slot * kMxStageBytes), b0 = a0 + kMxTileA;
      const uint32_t sf0 = b0 + kMxTileB;
      const uint32_t tsf = tbase + (uint32_t)(kMxN + slot * kMxSfCols);
      for (int i = 0; i < 1 + kMxTerms; ++i)   // weight scales, then each term's: 4 columns each
        tc_cp_sf(tsf + 4 * i, tc_smem_desc(sf0 + i * kMxSf, 128, 128));
#pragma unroll
      for (int term = 0; term < kMxTerms; ++term)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t ad = tc_smem_desc(a0 + 2 * h * kMxChunk, kMxChunk, 128);
          const uint64_t bd = tc_smem_desc(b0 + term * kMxTileA + 2 * h * kMxChunk, kMxChunk, 128);
          const uint32_t sfa = (tsf) | ((uint32_t)(2 * h) << 30);
          const uint32_t sfb = (tsf + 4 * (1 + term)) | ((uint32_t)(2 * h) << 30);
          const uint32_t acc = started ? 1u : 0u;
          asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                       " tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n}\n"
                       :: "r"(tbase), "l"(ad), "l"(bd), "r"(mx_idesc(2 * h)), "r"(acc), "r"(sfa), "r"(sfb)
                       : "memory");
          started = true;
        }
      tc_commit(&S.empty[slot]);
    }
    tc_commit(&S.done);
    mbar_wait_bounded(&S.done, 0, wait_ns, status);
  }
  // -------------------------------------------------------------------- epilogue (all warps)
  __syncwarp();
  bool ok = mbar_wait_bounded(&S.done, 0, wait_ns, status) && !*abort_flag;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  if (ok) {
    const int r = mt * kMxM + tid;
    const uint32_t lane_addr = tbase + ((uint32_t)(warp * 32) << 16);
    float* out = p.splits > 1 ? p.part + (size_t)blockIdx.z * p.T * p.R : p.y;
    for (int c0 = 0; c0 < kMxN; c0 += 16) {
      uint32_t v[16];
      tc_ld16(lane_addr + c0, v);
      tc_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = nt * kMxN + c0 + j;
        if (t < p.T && r < p.R) out[(size_t)t * p.R + r] = __uint_as_float(v[j]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tc_dealloc(tbase, 256);
}

// grid ceil(T R / 4 / 256), block 256: Y = the splits' partial products summed in split order.
__global__ void __launch_bounds__(256) mx_reduce_kernel(const float* __restrict__ part, int splits, size_t n4,
                                                        float* __restrict__ y) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 a = __ldcg((const float4*)part + i);
  for (int q = 1; q < splits; ++q) {
    const float4 b = __ldcg((const float4*)part + (size_t)q * n4 + i);
    a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
  }
  *((float4*)y + i) = a;
}

// ------------------------------------------------------------------ host side
// Workspace of the many-token product: a 256-byte header (status word first),
// then the tokens' terms, their scales and the rearranged weight scales.
struct MxWs {
  size_t bq, bsf, asf, part, total;
  int splits;
};
// Column splits: as many as keep the CTAs within one wave, at most kMxSplitMax, at least two
// stages each; a function of the shape alone, so the workspace size is known without a device.
static int mx_splits(int R, int K, int T) {
  const int tiles = (R / kMxM) * ((T + kMxN - 1) / kMxN), nstg = K / kMxKS;
  int s = kMxWaveCtas / tiles;
  s = s > kMxSplitMax ? kMxSplitMax : s;
  s = s > nstg / 2 ? nstg / 2 : s;
  return s < 1 ? 1 : s;
}
static MxWs mx_ws(int R, int K, int T) {
  const size_t tpad = (size_t)(T + kMxN - 1) / kMxN * kMxN;
  MxWs w;
  w.splits = mx_splits(R, K, T);
  size_t o = 256;
  w.bq = o; o = (o + tpad * (size_t)K / 2 * kMxTerms + 255) / 256 * 256;
  w.bsf = o; o = (o + tpad * (size_t)K / 32 * kMxTerms + 255) / 256 * 256;
  w.asf = o; o = (o + (size_t)R * K / 32 + 255) / 256 * 256;
  w.part = o; o = (o + (w.splits > 1 ? sizeof(float) * w.splits * (size_t)T * R : 0) + 255) / 256 * 256;
  w.total = o;
  return w;
}

size_t mx_gemm_ws_bytes(int R, int K, int T) { return mx_ws(R, K, T).total; }

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
  }
  return fn;
}

cudaError_t launch_mx_gemm(const uint32_t* q, const uint8_t* e, int R, int K, const uint16_t* x, int T, float* y,
                           void* ws, unsigned long long wait_ns, cudaStream_t s) {
  const MxWs W = mx_ws(R, K, T);
  const int tpad = (T + kMxN - 1) / kMxN * kMxN;
  uint8_t* base = (uint8_t*)ws;
  const int nscale = (int)(((size_t)R * (K / kMxKS) + kMxPrepThreads - 1) / kMxPrepThreads);
  const int qrow = (4 * (K / 32) + kMxPrepThreads - 1) / kMxPrepThreads;
  mx_prep_kernel<<<tpad * qrow + nscale, kMxPrepThreads, 0, s>>>(x, T, tpad, e, R, K, base + W.bq, base + W.bsf,
                                                             base + W.asf);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)R};   // bytes of a row, rows
  const cuuint64_t strides[1] = {(cuuint64_t)K / 2};
  const cuuint32_t box[2] = {16, (cuuint32_t)kMxM};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void*)q, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  MxGemmParams p;
  p.R = R; p.K = K; p.T = T; p.splits = W.splits;
  p.part = (float*)(base + W.part);
  p.bq = base + W.bq; p.bsf = base + W.bsf; p.asf = base + W.asf;
  p.y = y;
  p.status = (uint32_t*)ws;
  p.wait_ns = wait_ns;
  const size_t sm = (size_t)kMxStages * kMxStageBytes + sizeof(MxSmem);
  err = set_func_attr((const void*)mx_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (err != cudaSuccess) return err;
  mx_gemm_kernel<<<dim3(R / kMxM, tpad / kMxN, W.splits), 128, sm, s>>>(map, p);
  err = cudaGetLastError();
  if (err != cudaSuccess || W.splits == 1) return err;
  const size_t n4 = (size_t)T * R / 4;   // R % 128 == 0
  mx_reduce_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(p.part, W.splits, n4, y);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ decode layer kernels on digit blocks
// After the router and the top-k (kernels.cu): gate/up with SwiGLU, then down with the weighted
// combine and the residual, then the RMSNorm (kernels.cu), for two kinds of expert matrices:
//  * MXFP4 (kCodecMx): moe_qmat.q the E2M1 codes, scales the E8M0 bytes [R][K/32], biases unused;
//  * affine 4-bit and 2-bit codes (kCodecQ4, kCodecQ2): q the codes, scales and biases bf16
//    [R][K/64], w = q s + b per group of 64 consecutive k.
// A lane takes whole 32-element blocks of a row (16 bytes of codes, 8 for 2-bit codes, and the
// block's scale, or its group's scale and bias) against x or a as digit blocks whose planes
// follow the order in which the codes expand to bytes.
constexpr int kMxLWarps = 8;
constexpr int kMxMaxSlots = kMaxSlots;

template <int CODEC> struct MxBlk;                               // one block's codes and scale words
template <> struct MxBlk<kCodecMx> { uint4 c; unsigned e; };
template <> struct MxBlk<kCodecQ4> { uint4 c; unsigned sb; };   // sb: scale bits | bias bits << 16
template <> struct MxBlk<kCodecQ2> { uint2 c; unsigned sb; };

// Block b of row `row` of a K-column matrix M (nothing read when !in).
template <int CODEC>
__device__ __forceinline__ MxBlk<CODEC> mx_blk_load(const moe_qmat& M, size_t row, int K, int b, bool in);
template <>
__device__ __forceinline__ MxBlk<kCodecMx> mx_blk_load<kCodecMx>(const moe_qmat& M, size_t row, int K, int b, bool in) {
  const size_t at = row * (K / 32) + b;
  return MxBlk<kCodecMx>{in ? __ldg((const uint4*)M.q + at) : make_uint4(0u, 0u, 0u, 0u),
                         in ? (unsigned)__ldg((const uint8_t*)M.scales + at) : 0u};
}
__device__ __forceinline__ unsigned mx_sb_load(const moe_qmat& M, size_t row, int K, int b, bool in) {
  const size_t g = row * (K / 64) + b / 2;
  return in ? (unsigned)__ldg(M.scales + g) | ((unsigned)__ldg(M.biases + g) << 16) : 0u;
}
template <>
__device__ __forceinline__ MxBlk<kCodecQ4> mx_blk_load<kCodecQ4>(const moe_qmat& M, size_t row, int K, int b, bool in) {
  return MxBlk<kCodecQ4>{in ? __ldg((const uint4*)M.q + row * (K / 32) + b) : make_uint4(0u, 0u, 0u, 0u),
                         mx_sb_load(M, row, K, b, in)};
}
template <>
__device__ __forceinline__ MxBlk<kCodecQ2> mx_blk_load<kCodecQ2>(const moe_qmat& M, size_t row, int K, int b, bool in) {
  return MxBlk<kCodecQ2>{in ? __ldg((const uint2*)M.q + row * (K / 32) + b) : make_uint2(0u, 0u),
                         mx_sb_load(M, row, K, b, in)};
}

// The block's share of the row's dot product with the values of digit block d. Affine codes:
// s sum q X + b sum X, both sums exact integers, times 2^-p (twice the stored factor).
__device__ __forceinline__ float mx_blk_value(const MxBlk<kCodecMx>& k, const uint8_t* d) {
  return mx_block_dot_dig(k.c, d) * mx_scale(k.e);
}
__device__ __forceinline__ float mx_affine(int sq, unsigned sb, const uint8_t* d) {
  const float f = 2.f * __uint_as_float(((const uint32_t*)d)[24]);
  const int sx = ((const int*)d)[25];
  return f * fmaf((float)sq, bf16lo(sb), (float)sx * bf16hi(sb));
}
__device__ __forceinline__ float mx_blk_value(const MxBlk<kCodecQ4>& k, const uint8_t* d) {
  return mx_affine(dq4_block_dot(k.c, d), k.sb, d);
}
__device__ __forceinline__ float mx_blk_value(const MxBlk<kCodecQ2>& k, const uint8_t* d) {
  return mx_affine(dq2_block_dot(k.c, d), k.sb, d);
}

// grid (S I / kMxLWarps, T), block 32 kMxLWarps, clusters of kMxGuCluster CTAs: a[t][s][i] =
// silu(G x_t)_i (U x_t)_i for the expert of slot s (slot k = the shared expert), one (slot, row)
// per warp, every lane's 4 blocks of the gate and up rows requested at once; a cluster's warps
// hold the 32 rows of one block of a, which they gather in the shared memory of the cluster's
// first CTA, whose first warp writes the block's digit block to adig.
// Under a programmatic launch the CTA copies x_t's digit blocks (complete once this kernel
// starts: their kernel ran two launches before, and the top-k triggered this launch only after
// its own wait) before waiting for the top-k; then each warp resolves its expert and requests
// its rows.
// 64 registers (4 CTAs per SM): the 512 CTAs of 4 slots x intermediate 1024 run in one wave on
// 148 SMs, which pays for the few spilled bytes.
constexpr int kMxGuCluster = 32 / kMxLWarps;
template <int CODEC>
__global__ void __cluster_dims__(kMxGuCluster, 1, 1) __launch_bounds__(kMxLWarps * 32, 4)
mx_gateup_kernel(MxLayerParams p) {
  extern __shared__ __align__(16) unsigned char xd[];   // x_t's digit blocks, [H/32][kMxDig]
  __shared__ float ablk[32];                             // the cluster's block of a (first CTA)
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int t = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nb = p.H / 32;
  const int item = blockIdx.x * kMxLWarps + warp;   // < S I: the grid is exact
  // first phase of the cluster barrier: passed below once every CTA of the cluster runs, before
  // any writes into the first CTA's shared memory
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  const int sl = item / p.I, i = item % p.I;
  const uint4* xsrc = (const uint4*)(p.xdig + (size_t)t * nb * kMxDig);
  for (int q = threadIdx.x; q < nb * (kMxDig / 16); q += blockDim.x) ((uint4*)xd)[q] = __ldcg(xsrc + q);
  griddep_wait();   // the top-k has completed
  griddep_launch_dependents();
  MxBlk<CODEC> ga[4], ua[4];
  auto load = [&](int b0) {   // the expert's descriptor read again for every chunk of 128 blocks
    const moe_expert* ex = sl < p.k ? p.experts + p.idx[t * p.k + sl] : &p.shared;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b = b0 + 32 * u + lane;
      ga[u] = mx_blk_load<CODEC>(ex->gate, i, p.H, b, b < nb);
      ua[u] = mx_blk_load<CODEC>(ex->up, i, p.H, b, b < nb);
    }
  };
  load(0);
  __syncthreads();
  float2 acc = make_float2(0.f, 0.f);
  for (int b0 = 0;;) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int b = b0 + 32 * u + lane;
      if (b < nb) {
        acc.x += mx_blk_value(ga[u], xd + b * kMxDig);
        acc.y += mx_blk_value(ua[u], xd + b * kMxDig);
      }
    }
    b0 += 4 * 32;
    if (b0 >= nb) break;
    load(b0);
  }
  const float g = warp_sum(acc.x), u = warp_sum(acc.y);
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  if (lane == 0) *cluster.map_shared_rank(&ablk[rank * kMxLWarps + warp], 0) = g / (1.f + expf(-g)) * u;
  cluster.sync();   // the block is complete; nobody touches another CTA's shared memory after this
  if (rank == 0 && warp == 0)   // item is the block's first row
    mx_digit_lanes(ablk[lane], lane, p.adig + (((size_t)t * p.S + sl) * (p.I / 32) + i / 32) * kMxDig, CODEC);
}

// grid (ceil(H / kMxLWarps), T), block 32 kMxLWarps, a hidden row per warp:
// h[t][j] += sum_{s<k} w[t][s] (D_s a[t][s])_j + sg[t] (D_shared a[t][k])_j, in that order.
// Each warp resolves every slot's expert (the selection is complete: the top-k ran before the
// gate/up kernel passed its wait) and requests its row's first blocks, then waits for the digit
// blocks of a[t] and copies them. NS >= S bounds the slots held in registers; with up to 4 slots
// the kernel fits 64 registers, so 4 CTAs per SM hold all 512 CTAs of hidden 4096 in one wave.
template <int CODEC, int NS>
__global__ void __launch_bounds__(kMxLWarps * 32, NS <= 4 ? 4 : 2) mx_down_kernel(MxLayerParams p) {
  extern __shared__ __align__(16) unsigned char ad[];   // a[t][s]'s digit blocks, [S][I/32][kMxDig]
  const int t = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nb = p.I / 32, sstride = nb * kMxDig;
  const int row = blockIdx.x * kMxLWarps + warp;
  const bool has = row < p.H;
  MxBlk<CODEC> c[NS];
  auto load = [&](int b0) {   // every slot's block b0 + lane (descriptors read again per chunk)
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
      const bool in = has && sl < p.S && b0 + lane < nb;
      moe_qmat D{};
      if (in) D = sl < p.k ? p.experts[p.idx[t * p.k + sl]].down : p.shared.down;
      c[sl] = mx_blk_load<CODEC>(D, row, p.I, b0 + lane, in);
    }
  };
  load(0);
  griddep_wait();   // the digit blocks of a are complete
  griddep_launch_dependents();
  const uint4* asrc = (const uint4*)(p.adig + (size_t)t * p.S * sstride);
  for (int qq = threadIdx.x; qq < p.S * sstride / 16; qq += blockDim.x) ((uint4*)ad)[qq] = __ldcg(asrc + qq);
  __syncthreads();
  if (!has) return;
  float y[NS];
#pragma unroll
  for (int sl = 0; sl < NS; ++sl) y[sl] = 0.f;
  for (int b0 = 0;;) {   // every slot's block b0 + lane in flight at once
    const int b = b0 + lane;
#pragma unroll
    for (int sl = 0; sl < NS; ++sl)
      if (sl < p.S && b < nb) y[sl] += mx_blk_value(c[sl], ad + sl * sstride + b * kMxDig);
    b0 += 32;
    if (b0 >= nb) break;
    load(b0);
  }
  float acc = p.h[(size_t)t * p.H + row];
#pragma unroll
  for (int sl = 0; sl < NS; ++sl)
    if (sl < p.S) acc = fmaf(sl < p.k ? p.w[t * p.k + sl] : p.sg[t], warp_sum(y[sl]), acc);
  if (lane == 0) p.h[(size_t)t * p.H + row] = acc;
}

static cudaError_t mx_launch(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                             void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  if (pdl) {
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelExC(&cfg, fn, args);
}

cudaError_t launch_mx_digits(const uint16_t* src, int rows, int K, uint8_t* dst, int codec, cudaStream_t s,
                             bool pdl) {
  const size_t n = (size_t)rows * (K / 32);
  const uint16_t* sp = src;
  void* args[] = {(void*)&sp, &rows, &K, &dst, &codec};
  return mx_launch((const void*)mx_digits_kernel, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, s, pdl, args);
}

// gate/up (writing the digit blocks of a), down
template <int CODEC>
static cudaError_t mx_layer_launch(const MxLayerParams& p, cudaStream_t s, bool pdl) {
  const size_t sg = (size_t)(p.H / 32) * kMxDig;
  const size_t sd = (size_t)p.S * (p.I / 32) * kMxDig;
  const void* gateup = (const void*)mx_gateup_kernel<CODEC>;
  const void* down = p.S <= 2 ? (const void*)mx_down_kernel<CODEC, 2>
                   : p.S <= 4 ? (const void*)mx_down_kernel<CODEC, 4>
                   : p.S <= 6 ? (const void*)mx_down_kernel<CODEC, 6> : (const void*)mx_down_kernel<CODEC, kMxMaxSlots>;
  cudaError_t e = set_func_attr(gateup, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg);
  if (e != cudaSuccess) return e;
  e = set_func_attr(down, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sd);
  if (e != cudaSuccess) return e;
  MxLayerParams q = p;
  void* args[] = {&q};
  // S I / kMxLWarps CTAs: a multiple of the cluster size, since 32 divides I
  e = mx_launch(gateup, dim3(p.S * p.I / kMxLWarps, p.T), dim3(kMxLWarps * 32), sg, s, pdl, args);
  if (e != cudaSuccess) return e;
  return mx_launch(down, dim3((p.H + kMxLWarps - 1) / kMxLWarps, p.T), dim3(kMxLWarps * 32), sd, s, pdl, args);
}

cudaError_t launch_mx_layer(const MxLayerParams& p, cudaStream_t s, bool pdl) {
  switch (p.codec) {
    case kCodecMx: return mx_layer_launch<kCodecMx>(p, s, pdl);
    case kCodecQ4: return mx_layer_launch<kCodecQ4>(p, s, pdl);
    case kCodecQ2: return mx_layer_launch<kCodecQ2>(p, s, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qmoe
