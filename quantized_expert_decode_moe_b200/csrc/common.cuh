// Device building blocks of the quantized MoE expert forward (sm_100a).
//
// Dequantising mat-vec ("FMA-optimised dequant kernel" on the Flash-MoE pages:
// a weight is code*scale + bias, applied as (q*s + b)*x). The pages fold the
// scale and bias into the activation per element, fma(q, s*x, b*x). Here the
// same sum is regrouped once more, per quantisation group g of G=64 elements:
//     sum_k (q_k s + b) x_k = s * sum_k (q_k - z) x_k + (b + z s) * X_g,
// with X_g = sum_{k in g} x_k computed once per vector and z a code offset
// (8 for 4-bit, 2 for 2-bit). The inner sum sum_k (q_k - z) x_k runs on the
// tensor cores: (q - z) is a small integer, exact in fp16, and x is split into
// fp16 hi + lo parts, so an m16n8k16 MMA with fp32 accumulation computes it
// to ~22 bits. The MMA's N=8 columns carry {group 0, group 1} x {hi, lo} of
// one 128-element span, so each group's partial sum comes out separately and
// its scale is applied in fp32 after the MMA.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace qmoe {

constexpr int kSpan = 128;      // k elements per span (two quantisation groups)
constexpr int kGroup = 64;      // quantisation group
constexpr int kWarps = 16;      // warps per CTA of the dequant kernels
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTopK = 8;
constexpr int kMaxSlots = kMaxTopK + 1;

// status word codes latched by kernels (mirrors moe_status)
constexpr uint32_t kStatusDeviceFault = MOE_ERR_DEVICE_FAULT;

// ------------------------------------------------------------------ scalar helpers
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint16_t f32_to_bf16(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}

// fp16 hi part / lo part of a float: v ~= hi + lo to about 22 bits
__device__ __forceinline__ __half half_hi(float v) { return __float2half_rn(v); }
__device__ __forceinline__ __half half_lo(float v) { return __float2half_rn(v - __half2float(__float2half_rn(v))); }

// ------------------------------------------------------------------ memory helpers
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg_stream_v2(const void* p) {
  uint2 r;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ldg_stream_u32(const void* p) {
  uint32_t r;
  asm("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
// coherent (L2) loads of data written by an earlier kernel of the same chain
__device__ __forceinline__ double ldcg_f64(const double* p) { return __ldcg(p); }
__device__ __forceinline__ float ldcg_f32(const float* p) { return __ldcg(p); }
__device__ __forceinline__ int ldcg_i32(const int* p) { return __ldcg(p); }

// Hint HBM -> L2 for [p, p+bytes); only whole 16-byte pieces inside the range.
__device__ __forceinline__ void prefetch_l2_range(const void* p, size_t bytes) {
  uintptr_t a = (uintptr_t)p;
  uintptr_t lo = (a + 15) & ~(uintptr_t)15;
  uintptr_t hi = (a + bytes) & ~(uintptr_t)15;
  while (lo < hi) {
    uint32_t n = (uint32_t)((hi - lo) < 65536 ? (hi - lo) : 65536);
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(lo), "r"(n) : "memory");
    lo += n;
  }
}
// Part `part` of `nparts` of [p, p+bytes), for spreading one prefetch over CTAs.
__device__ __forceinline__ void prefetch_l2_part(const void* p, size_t bytes, int part, int nparts) {
  size_t per = ((bytes + nparts - 1) / nparts + 15) & ~(size_t)15;
  size_t lo = per * (size_t)part;
  if (lo >= bytes) return;
  size_t hi = lo + per < bytes ? lo + per : bytes;
  prefetch_l2_range((const char*)p + lo, hi - lo);
}

// ------------------------------------------------------------------ programmatic dependent launch
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------ tensor-core MMA
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ code unpack (exact fp16 pairs)
// (a & mask) | magic: places a code field in the mantissa of the fp16 1024.
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
  return r;
}
__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// One 4-bit word (codes n0..n7, n_i at bits 4i) -> 4 fp16x2 pairs of (n - 8):
// p[0] = (n0, n4), p[1] = (n1, n5), p[2] = (n2, n6), p[3] = (n3, n7); first element in the low half.
__device__ __forceinline__ void unpack_q4(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t kMagic = 0x64006400u;   // fp16 1024, 1024
  const uint32_t k1032 = 0x64086408u;    // 1024 + 8
  const uint32_t kSixteenth = 0x2C002C00u;
  const uint32_t kMinus72 = 0xD480D480u; // -(64 + 8)
  const uint32_t w2 = w >> 8;
  p[0] = hsub2_u(lop3_and_or(w, 0x000F000Fu, kMagic), k1032);
  p[1] = hfma2_u(lop3_and_or(w, 0x00F000F0u, kMagic), kSixteenth, kMinus72);
  p[2] = hsub2_u(lop3_and_or(w2, 0x000F000Fu, kMagic), k1032);
  p[3] = hfma2_u(lop3_and_or(w2, 0x00F000F0u, kMagic), kSixteenth, kMinus72);
}
// One 2-bit word (codes c0..c15, c_i at bits 2i) -> 8 fp16x2 pairs of (c - 2):
// p[i] = (c_i, c_{i+8}) for i = 0..7.
__device__ __forceinline__ void unpack_q2(uint32_t w, uint32_t (&p)[8]) {
  const uint32_t kMagic = 0x64006400u;
  const uint32_t w2 = w >> 8;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t v = h ? w2 : w;
    p[4 * h + 0] = hsub2_u(lop3_and_or(v, 0x00030003u, kMagic), 0x64026402u);                  // -(1024+2)
    p[4 * h + 1] = hfma2_u(lop3_and_or(v, 0x000C000Cu, kMagic), 0x34003400u, 0xDC08DC08u);      // /4, -(256+2)
    p[4 * h + 2] = hfma2_u(lop3_and_or(v, 0x00300030u, kMagic), 0x2C002C00u, 0xD420D420u);      // /16, -(64+2)
    p[4 * h + 3] = hfma2_u(lop3_and_or(v, 0x00C000C0u, kMagic), 0x24002400u, 0xCC80CC80u);      // /64, -(16+2)
  }
}

template <int BITS> struct QTraits;
template <> struct QTraits<4> {
  static constexpr int kWordsPerThread = 4;  // per row per span: 32 codes
  static constexpr float kZ = 8.f;
  // k offset (within the thread's 32-element window) of element e of pair p
  __host__ __device__ static constexpr int koff(int p, int e) { return 8 * (p >> 2) + (p & 3) + 4 * e; }
};
template <> struct QTraits<2> {
  static constexpr int kWordsPerThread = 2;
  static constexpr float kZ = 2.f;
  __host__ __device__ static constexpr int koff(int p, int e) { return 16 * (p >> 3) + (p & 7) + 8 * e; }
};

// ------------------------------------------------------------------ B-fragment table
// For one vector (one token) x' (prescaled fp32) of length K, the table holds,
// per span s and MMA j (0..7), the two f16x2 B registers of the 8 lanes that
// carry data. Column n = lane>>2 of the MMA is {grp = (n>>1)&1, lo = n&1} for
// n < 4 (columns 4..7 are zero: one token). Lane (g', t) supplies the rows
// k = s*128 + 32t + koff(2j+i, e) of column n; they are nonzero only when the
// thread's 32-element window lies in group grp, i.e. (t>>1) == grp. Those 8
// lanes are stored compactly at c = 2n + (t&1); every other lane reads zeros.
constexpr int kBtabPerSpan = 8 * 8;   // MMAs x live lanes (uint2 each)

__device__ __forceinline__ int btab_lane(int lane) {
  const int n = lane >> 2, t = lane & 3;
  return (n < 4 && ((n >> 1) & 1) == (t >> 1)) ? 2 * n + (t & 1) : -1;
}

template <int BITS>
__device__ __forceinline__ uint2 btab_entry(const float* xs, int s, int j, int c) {
  const int n = c >> 1, t = 2 * ((n >> 1) & 1) + (c & 1);
  const int lo = n & 1;
  const float* w = xs + s * kSpan + 32 * t;
  uint32_t r[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float v0 = w[QTraits<BITS>::koff(2 * j + i, 0)];
    const float v1 = w[QTraits<BITS>::koff(2 * j + i, 1)];
    r[i] = lo ? pack_half2(half_lo(v0), half_lo(v1)) : pack_half2(half_hi(v0), half_hi(v1));
  }
  return make_uint2(r[0], r[1]);
}

// Prescale exponent so that max|x * 2^p| lies in [2^14, 2^15): keeps the fp16
// hi part in range and the lo part meaningful. Exact (power of two).
__device__ __forceinline__ float prescale_for(float amax) {
  if (!(amax > 0.f) || !isfinite(amax)) return 1.f;
  int e = ilogbf(amax);
  int sh = 14 - e;
  sh = sh > 100 ? 100 : (sh < -100 ? -100 : sh);
  return ldexpf(1.f, sh);
}



// ------------------------------------------------------------------ per-warp staging with cp.async
// Each warp stages exactly the units it will compute: every lane issues its
// own 16-byte asynchronous copies (codes) and 4-byte copies (the span's
// bf16x2 scales / biases) for all of the warp's units at once, one commit
// group per unit, so the whole share of the warp is in flight before the
// first MMA. Unit slot layout in shared memory: codes [16 rows][span bytes],
// then scales [16][4 B], biases [16][4 B].
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" :: "r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }
// wait until at most n commit groups of this thread are pending (0 <= n, clamped to 7)
__device__ __forceinline__ void cp_async_wait_dyn(int n) {
  switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    case 6: cp_async_wait<6>(); break;
    default: cp_async_wait<7>(); break;
  }
}

template <int BITS>
struct SpanBytes { static constexpr int v = kSpan * BITS / 8; };   // code bytes of one row over one span
template <int BITS>
struct UnitSmem { static constexpr int bytes = 16 * SpanBytes<BITS>::v + 16 * 4 * 2; };
constexpr int kUnitSlots = 8;   // staged units per warp in flight

// The 16 source rows of one tile: row r (0..15) of codes / scales / biases.
struct RowSrc { const uint32_t* q; const uint16_t* s; const uint16_t* b; };

// What one lane copies for every unit of a tile, as pointers at span 0 and
// shared-memory offsets inside a unit slot (computed once per tile).
template <int BITS>
struct LaneCopy {
  const unsigned char* q0; const unsigned char* q1;   // 16-byte code chunks (q1 unused for 2-bit)
  const unsigned char* sb;                            // 4-byte bf16x2 scale (lanes 0-15) or bias (16-31)
  uint32_t d0, d1, ds;
};

template <int BITS, class RowFn>
__device__ __forceinline__ LaneCopy<BITS> lane_copy(RowFn row, int tile, int lane) {
  constexpr int SB = SpanBytes<BITS>::v;   // 64 (4-bit) or 32 (2-bit)
  constexpr int parts = SB / 16;
  LaneCopy<BITS> L;
  {
    const int c = lane, r = c / parts, q = c % parts;
    L.q0 = (const unsigned char*)row(tile, r).q + q * 16;
    L.d0 = r * SB + q * 16;
  }
  if constexpr (parts == 4) {
    const int c = lane + 32, r = c / parts, q = c % parts;
    L.q1 = (const unsigned char*)row(tile, r).q + q * 16;
    L.d1 = r * SB + q * 16;
  } else {
    L.q1 = nullptr; L.d1 = 0;
  }
  const int r = lane & 15;
  const RowSrc rs = row(tile, r);
  L.sb = (const unsigned char*)(lane < 16 ? rs.s : rs.b);
  L.ds = 16 * SB + (lane < 16 ? 0 : 64) + r * 4;
  return L;
}

template <int BITS>
__device__ __forceinline__ void stage_unit(unsigned char* slot, const LaneCopy<BITS>& L, int span) {
  constexpr int SB = SpanBytes<BITS>::v;
  cp_async16(slot + L.d0, L.q0 + span * SB);
  if constexpr (SB == 64) cp_async16(slot + L.d1, L.q1 + span * SB);
  cp_async4(slot + L.ds, L.sb + span * 4);
}

template <int BITS>
struct Frag {   // one unit's A codes of rows g and g+8, and the span's bf16x2 scales / biases
  uint32_t wa[QTraits<BITS>::kWordsPerThread];
  uint32_t wb[QTraits<BITS>::kWordsPerThread];
  uint32_t sa, sb, ba, bb;
};

template <int BITS>
__device__ __forceinline__ void frag_load(Frag<BITS>& F, const unsigned char* slot, int g, int t) {
  constexpr int W = QTraits<BITS>::kWordsPerThread;
  constexpr int SB = SpanBytes<BITS>::v;
  const unsigned char* c = slot + t * W * 4;
  if constexpr (W == 4) {
    const uint4 va = *(const uint4*)(c + g * SB);
    const uint4 vb = *(const uint4*)(c + (g + 8) * SB);
    F.wa[0] = va.x; F.wa[1] = va.y; F.wa[2] = va.z; F.wa[3] = va.w;
    F.wb[0] = vb.x; F.wb[1] = vb.y; F.wb[2] = vb.z; F.wb[3] = vb.w;
  } else {
    const uint2 va = *(const uint2*)(c + g * SB);
    const uint2 vb = *(const uint2*)(c + (g + 8) * SB);
    F.wa[0] = va.x; F.wa[1] = va.y;
    F.wb[0] = vb.x; F.wb[1] = vb.y;
  }
  const uint32_t* sc = (const uint32_t*)(slot + 16 * SB);
  F.sa = sc[g]; F.sb = sc[g + 8];
  F.ba = sc[16 + g]; F.bb = sc[16 + g + 8];
}

// 8 MMAs over one span, two independent accumulator chains:
// c[0..1] = row g (cols 2t, 2t+1), c[2..3] = row g+8.
template <int BITS>
__device__ __forceinline__ void mma_frag(const Frag<BITS>& F, const uint2* __restrict__ bt, int bl, float (&c)[4]) {
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  float e[4] = {0.f, 0.f, 0.f, 0.f};
  if constexpr (BITS == 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t pa[4], pb[4];
      unpack_q4(F.wa[u], pa);
      unpack_q4(F.wb[u], pb);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = 2 * u + h;
        const uint2 b = bl >= 0 ? bt[j * 8 + bl] : make_uint2(0u, 0u);
        if (h == 0) mma_16816(d, pa[0], pb[0], pa[1], pb[1], b.x, b.y);
        else mma_16816(e, pa[2], pb[2], pa[3], pb[3], b.x, b.y);
      }
    }
  } else {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      uint32_t pa[8], pb[8];
      unpack_q2(F.wa[u], pa);
      unpack_q2(F.wb[u], pb);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int j = 4 * u + h;
        const uint2 b = bl >= 0 ? bt[j * 8 + bl] : make_uint2(0u, 0u);
        if (h & 1) mma_16816(e, pa[2 * h], pb[2 * h], pa[2 * h + 1], pb[2 * h + 1], b.x, b.y);
        else mma_16816(d, pa[2 * h], pb[2 * h], pa[2 * h + 1], pb[2 * h + 1], b.x, b.y);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = d[i] + e[i];
}

// Applies the group scales: thread t (< 2) owns group 2*span + t (hi + lo columns).
template <int BITS>
__device__ __forceinline__ void scale_frag(const Frag<BITS>& F, const float (&c)[4], const float* Xg, int span, int t,
                                           float& acc_a, float& acc_b) {
  if (t < 2) {
    const float xg = Xg[2 * span + t];
    const float s_a = t ? bf16hi(F.sa) : bf16lo(F.sa);
    const float s_b = t ? bf16hi(F.sb) : bf16lo(F.sb);
    const float b_a = t ? bf16hi(F.ba) : bf16lo(F.ba);
    const float b_b = t ? bf16hi(F.bb) : bf16lo(F.bb);
    acc_a = fmaf(s_a, c[0] + c[1], fmaf(fmaf(QTraits<BITS>::kZ, s_a, b_a), xg, acc_a));
    acc_b = fmaf(s_b, c[2] + c[3], fmaf(fmaf(QTraits<BITS>::kZ, s_b, b_b), xg, acc_b));
  }
}

// ------------------------------------------------------------------ split-unit schedule
// Work is a list of U = tiles * nspans units in tile-major order. CTA c owns
// [U*c/nCTA, U*(c+1)/nCTA); warp w owns an even share of that. Host picks nCTA
// so that every CTA range is >= nspans (a tile then meets at most two CTAs, so
// the fp32 atomic sum of at most two partials is order independent) and every
// warp range is <= nspans (a warp then meets at most two tiles).
struct Range { int a, b; };
__device__ __forceinline__ Range cta_range(long long U, int c, int n) {
  return Range{(int)(U * c / n), (int)(U * (c + 1) / n)};
}
__device__ __forceinline__ Range warp_range(Range r, int w) {
  const int L = r.b - r.a;
  return Range{r.a + L * w / kWarps, r.a + L * (w + 1) / kWarps};
}

// Per-CTA partial sums of the (at most two) tiles each warp met.
struct PartialSmem {
  float v[kWarps][2][16];
  int tile[kWarps][2];
};

// Unit loop of one warp: stages up to kUnitSlots units at a time with
// cp.async, then MMAs them in order as they land. Partials go to `ps`.
// (tile, span) of consecutive units are tracked incrementally; the lanes'
// copy sources are recomputed only when the tile changes.
template <int BITS, class RowFn, class BtFn, class XgFn>
__device__ __forceinline__ void run_units(Range wr, int nspans, unsigned char* wslots, RowFn row, BtFn bt_of,
                                          XgFn xg_of, PartialSmem& ps, int warp, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int bl = btab_lane(lane);
  if (lane == 0) { ps.tile[warp][0] = -1; ps.tile[warp][1] = -1; }
  __syncwarp();
  if (wr.a >= wr.b) return;
  int si = 0;
  float acc_a = 0.f, acc_b = 0.f;
  int tile_s = wr.a / nspans, span_s = wr.a - tile_s * nspans;   // staging cursor
  int tile_c = tile_s, span_c = span_s;                           // compute cursor
  LaneCopy<BITS> lc = lane_copy<BITS>(row, tile_s, lane);
  const uint2* bt = bt_of(tile_c);
  const float* xg = xg_of(tile_c);
  for (int u0 = wr.a; u0 < wr.b; u0 += kUnitSlots) {
    const int n = wr.b - u0 < kUnitSlots ? wr.b - u0 : kUnitSlots;
    for (int i = 0; i < n; ++i) {
      stage_unit<BITS>(wslots + i * UnitSmem<BITS>::bytes, lc, span_s);
      cp_async_commit();
      if (++span_s == nspans && u0 + i + 1 < wr.b) { span_s = 0; ++tile_s; lc = lane_copy<BITS>(row, tile_s, lane); }
    }
    for (int i = 0; i < n; ++i) {
      cp_async_wait_dyn(n - 1 - i);
      __syncwarp();
      Frag<BITS> F;
      frag_load<BITS>(F, wslots + i * UnitSmem<BITS>::bytes, g, t);
      float c[4];
      mma_frag<BITS>(F, bt + span_c * kBtabPerSpan, bl, c);
      scale_frag<BITS>(F, c, xg, span_c, t, acc_a, acc_b);
      const bool last = u0 + i + 1 >= wr.b;
      if (++span_c == nspans || last) {
        acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
        acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 1);
        if (t == 0) { ps.v[warp][si][g] = acc_a; ps.v[warp][si][g + 8] = acc_b; }
        if (lane == 0) ps.tile[warp][si] = tile_c;
        si++;
        acc_a = acc_b = 0.f;
        if (!last) { span_c = 0; ++tile_c; bt = bt_of(tile_c); xg = xg_of(tile_c); }
      }
    }
    __syncwarp();
  }
}

// After __syncthreads: sums the partials of every tile the CTA met, in warp
// order (only the warps whose ranges meet the tile), and hands (tile, row,
// value) to `out`.
template <class OutFn>
__device__ __forceinline__ void reduce_partials(Range cr, int nspans, const PartialSmem& ps, OutFn out) {
  if (cr.a >= cr.b) return;
  const int tl = cr.a / nspans, th = (cr.b - 1) / nspans;
  const int n = (th - tl + 1) * 16;
  const int L = cr.b - cr.a;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int tile = tl + i / 16, r = i % 16;
    // warps w with [a + L*w/16, a + L*(w+1)/16) meeting [tile*nspans, (tile+1)*nspans)
    const int lo = tile * nspans - cr.a, hi = (tile + 1) * nspans - cr.a;
    int w0 = lo <= 0 ? 0 : (lo * kWarps) / L;
    if (w0 > 0) --w0;
    float s = 0.f;
    bool any = false;
    for (int w = w0; w < kWarps; ++w) {
      if (L * w / kWarps >= hi) break;
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (ps.tile[w][k] == tile) { s += ps.v[w][k][r]; any = true; }
    }
    if (any) out(tile, r, s);
  }
}

}  // namespace qmoe
