// Device building blocks of the quantized MoE expert forward (sm_100a).
//
// Dequantising mat-vec ("FMA-optimised dequant kernel" on the Flash-MoE pages:
// a weight is code*scale + bias, applied as (q*s + b)*x). The pages fold the
// scale and bias into the activation per element, fma(q, s*x, b*x). Here the
// same sum is regrouped once more, per quantisation group g of G=64 elements:
//     sum_k (q_k s + b) x_k = s * sum_k q_k x_k + b * X_g,
// with X_g = sum_{k in g} x_k computed once per vector. The inner sum
// sum_k q_k x_k runs on the integer tensor cores (m16n8k32, u8 x s8 -> s32):
// the codes are used as unsigned bytes straight from the packed words (one
// AND per four codes), and each activation group is held in fixed point,
// x = X * 2^-p_g with |X| < 2^22, split exactly into three signed 8-bit
// digits. The MMA's N=8 columns carry the digits of the two quantisation
// groups of one 128-element span (columns 0..2 and 4..6), so each group's
// exact integer partial sums come out separately; the group's scale and
// 2^-p_g are applied in fp32 after the MMA.
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
// coherent (L2) loads of data written by an earlier kernel of the same chain
__device__ __forceinline__ float ldcg_f32(const float* p) { return __ldcg(p); }
__device__ __forceinline__ int ldcg_i32(const int* p) { return __ldcg(p); }

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
// D = A (16x32 u8, row) * B (32x8 s8, col) + C, s32 accumulate
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------------------ code bytes for the A operand
// For MMA j (32 k-slots) a thread supplies two registers per row, each four
// unsigned code bytes: slots 4t..4t+3 (half 0) and 16+4t..16+4t+3 (half 1).
// 4-bit: word j of the thread's window, even nibbles (half 0) / odd (half 1).
// 2-bit: word j>>1, crumb fields s, s+4, s+8, s+12 with s = 2(j&1) + half.
template <int BITS>
__device__ __forceinline__ uint32_t code_bytes(const uint32_t* w, int j, int half) {
  if constexpr (BITS == 4) return (half ? (w[j] >> 4) : w[j]) & 0x0F0F0F0Fu;
  else return (w[j >> 1] >> (2 * (2 * (j & 1) + half))) & 0x03030303u;
}

template <int BITS> struct QTraits;
template <> struct QTraits<4> {
  static constexpr int kWordsPerThread = 4;  // per row per span: 32 codes
  // window offset of byte i (0..3) of half h of MMA j
  __host__ __device__ static constexpr int koff(int j, int h, int i) { return 8 * j + 2 * i + h; }
};
template <> struct QTraits<2> {
  static constexpr int kWordsPerThread = 2;
  __host__ __device__ static constexpr int koff(int j, int h, int i) { return 16 * (j >> 1) + 2 * (j & 1) + h + 4 * i; }
};

// ------------------------------------------------------------------ B-fragment table
// For one vector of length K: per quantisation group g a power of two 2^p_g
// with X_k = rint(x_k 2^p_g), |X_k| < 2^22, split as X = d0 + 2^8 d1 + 2^16 d2
// with signed bytes d_i. Per span s and MMA j (0..3) the table holds the two
// B registers (4 s8 each) of the lanes that carry data: MMA column n =
// lane>>2 is {grp = n>>2, digit = n&3 (< 3)}; lane (g', t) supplies the rows
// k = s*128 + 32t + koff(j, h, i) of column n, nonzero only when the thread's
// 32-element window lies in group grp, i.e. (t>>1) == grp. 12 live lanes per
// MMA are stored compactly.
constexpr int kDigits = 3;
constexpr int kBtLanes = 4 * kDigits;          // live lanes per MMA
constexpr int kBtPerSpan = 4 * kBtLanes;       // uint2 entries per span

__device__ __forceinline__ int bt_lane_index(int lane) {
  const int n = lane >> 2, t = lane & 3;
  const int grp = n >> 2, d = n & 3;
  if (d >= kDigits || grp != (t >> 1)) return -1;
  return (grp * kDigits + d) * 2 + (t & 1);
}

// power-of-two prescale of a group with max |x| = m: m * 2^p in [2^21, 2^22)
__device__ __forceinline__ float group_prescale(float m) {
  if (!(m > 0.f) || !isfinite(m)) return 1.f;
  int sh = 21 - ilogbf(m);
  sh = sh > 120 ? 120 : (sh < -120 ? -120 : sh);
  return ldexpf(1.f, sh);
}
__device__ __forceinline__ uint32_t digit_byte(float v, float sc, int d) {
  int X = __float2int_rn(v * sc);
  const int d0 = ((X + 128) & 255) - 128;
  if (d == 0) return (uint32_t)d0 & 255u;
  X = (X - d0) >> 8;
  const int d1 = ((X + 128) & 255) - 128;
  if (d == 1) return (uint32_t)d1 & 255u;
  return (uint32_t)((X - d1) >> 8) & 255u;
}
// entry i (= s * kBtPerSpan + j * kBtLanes + c) of the table of vector xs with
// per-group prescale gsc[g]
template <int BITS>
__device__ __forceinline__ uint2 btab_at(const float* xs, const float* gsc, int i) {
  const int s = i / kBtPerSpan, j = (i % kBtPerSpan) / kBtLanes, c = i % kBtLanes;
  const int gd = c >> 1, grp = gd / kDigits, d = gd % kDigits;
  const int t = 2 * grp + (c & 1);
  const float* w = xs + s * kSpan + 32 * t;
  const float sc = gsc[2 * s + grp];
  uint32_t r[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) v |= digit_byte(w[QTraits<BITS>::koff(j, h, b)], sc, d) << (8 * b);
    r[h] = v;
  }
  return make_uint2(r[0], r[1]);
}
// Per-group prescale gsc[g], its inverse igsc[g] and sums Xg[g] of xs (one warp per group).
__device__ __forceinline__ void group_stats(const float* xs, int ngroups, float* gsc, float* igsc, float* Xg, int warp,
                                            int lane, int nwarps) {
  for (int gi = warp; gi < ngroups; gi += nwarps) {
    const float a = xs[gi * kGroup + lane], b = xs[gi * kGroup + 32 + lane];
    float sum = a + b, m = fmaxf(fabsf(a), fabsf(b));
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (lane == 0) {
      const float sc = group_prescale(m);
      gsc[gi] = sc;
      igsc[gi] = 1.f / sc;
      Xg[gi] = sum;
    }
  }
}

// ------------------------------------------------------------------ B tables from registers
// The table builder's thread holds the EPT consecutive elements that feed its
// own B entries: 8 (4-bit: MMA j of window t takes elements 8j..8j+7) or 16
// (2-bit: MMAs 2jj, 2jj+1 take elements 16jj..16jj+15).
template <int BITS> struct TabTraits { static constexpr int kEPT = BITS == 4 ? 8 : 16; };

// Exponent sh of the power-of-two prescale of a group with max |x| = m:
// m * 2^sh in [2^21, 2^22) for normal m; 0 for zero or non-finite m;
// clamped to [-120, 120].
__device__ __forceinline__ int prescale_shift(float m) {
  const int eb = (int)((__float_as_uint(m) >> 23) & 0xFFu);
  if (eb == 0xFF || !(m > 0.f)) return 0;
  const int sh = 148 - eb;
  return sh > 120 ? 120 : (sh < -120 ? -120 : sh);
}
// signed-digit byte d (0..2) of X = d0 + 2^8 d1 + 2^16 d2, |X| <= 2^22
__device__ __forceinline__ uint32_t sdigit(int X, int d) {
  if (d > 0) X = (X - (int)(signed char)(X & 0xFF)) >> 8;
  if (d > 1) X = (X - (int)(signed char)(X & 0xFF)) >> 8;
  return (uint32_t)X & 0xFFu;
}
template <int EPT>
__device__ __forceinline__ uint32_t pack_digits(const int (&X)[EPT], int o, int st, int d) {
  return sdigit(X[o], d) | (sdigit(X[o + st], d) << 8) | (sdigit(X[o + 2 * st], d) << 16) |
         (sdigit(X[o + 3 * st], d) << 24);
}

// v = elements e0 .. e0+EPT-1 of a vector (e0 a multiple of EPT). The
// 64/EPT threads of a quantisation group are consecutive lanes, and all 32
// lanes of the warp call together (valid = false: no elements, v ignored).
// Writes the thread's B entries into bt (the vector's table) and, from the
// group's first thread, gs[g] = 2^-p_g and gs[ng + g] = X_g (the group sum).
template <int BITS>
__device__ __forceinline__ void build_tables(const float (&v)[TabTraits<BITS>::kEPT], int e0, bool valid, uint2* bt,
                                             float* gs, int ng) {
  constexpr int EPT = TabTraits<BITS>::kEPT, TPG = kGroup / EPT;
  float m = 0.f, sum = 0.f;
#pragma unroll
  for (int i = 0; i < EPT; ++i) { m = fmaxf(m, fabsf(v[i])); sum += v[i]; }
#pragma unroll
  for (int o = 1; o < TPG; o <<= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  if (!valid) return;
  const int sh = prescale_shift(m);
  const int s = e0 / kSpan, w = e0 % kSpan, t = w / 32, grp = t >> 1;
  const int c0 = grp * kDigits * 2 + (t & 1);   // entry of digit d: c0 + 2d
  // Element o of the window enters the MMA as code << (BITS * q) (masked in
  // place, q = its field in the byte), so its fixed point is scaled down by
  // 2^(BITS q): X = rint(x * 2^(sh - BITS q)).
  int X[EPT];
  if constexpr (BITS == 4) {
#pragma unroll
    for (int i = 0; i < EPT; ++i) X[i] = __float2int_rn(v[i] * __uint_as_float((uint32_t)(127 + sh - 4 * (i & 1)) << 23));
    uint2* e = bt + s * kBtPerSpan + ((w % 32) / 8) * kBtLanes + c0;
#pragma unroll
    for (int d = 0; d < kDigits; ++d) e[2 * d] = make_uint2(pack_digits(X, 0, 2, d), pack_digits(X, 1, 2, d));
  } else {
#pragma unroll
    for (int i = 0; i < EPT; ++i) X[i] = __float2int_rn(v[i] * __uint_as_float((uint32_t)(127 + sh - 2 * (i & 3)) << 23));
    const int jj = (w % 32) / 16;
#pragma unroll
    for (int jl = 0; jl < 2; ++jl) {
      uint2* e = bt + s * kBtPerSpan + (2 * jj + jl) * kBtLanes + c0;
#pragma unroll
      for (int d = 0; d < kDigits; ++d)
        e[2 * d] = make_uint2(pack_digits(X, 2 * jl, 4, d), pack_digits(X, 2 * jl + 1, 4, d));
    }
  }
  if (e0 % kGroup == 0) {
    const int g = e0 / kGroup;
    gs[g] = __uint_as_float((uint32_t)(127 - sh) << 23);
    gs[ng + g] = sum;
  }
}

// Code bytes of MMA j, half h, with each field left in place in its byte
// (the B table holds the matching scaled-down digits): 4-bit: low / high
// nibble; 2-bit: field 2(j&1)+h of word j>>1.
template <int BITS>
__device__ __forceinline__ uint32_t code_bytes_m(const uint32_t* w, int j, int half) {
  if constexpr (BITS == 4) return w[j] & (half ? 0xF0F0F0F0u : 0x0F0F0F0Fu);
  else return w[j >> 1] & (0x03030303u << (2 * (2 * (j & 1) + half)));
}

// B operand of one span of a vector, loaded once and reused for every row tile.
struct BFrag {
  uint2 b[4];
  float ip, xg;   // 2^-p of the lane's group; X_g on even lanes (bias term), 0 on odd lanes
};
__device__ __forceinline__ void load_bfrag(BFrag& B, const uint2* bt_span, int bl, const float* gs, int ng, int span,
                                           int t) {
#pragma unroll
  for (int j = 0; j < 4; ++j) B.b[j] = bl >= 0 ? bt_span[j * kBtLanes + bl] : make_uint2(0u, 0u);
  const int gi = 2 * span + (t >> 1);
  B.ip = gs[gi];
  B.xg = (t & 1) ? 0.f : gs[ng + gi];
}
// Lane constants of the epilogue: thread t holds MMA columns 2t, 2t+1 = the
// digits of group t>>1 (t even: d0, d1; t odd: d2).
struct LaneK {
  float m0, m1;   // f = c0 * m0 + c1 * m1
  int shl;        // bf16 of the lane's group: (word << shl) & 0xFFFF0000
};
__device__ __forceinline__ LaneK lane_consts(int t) {
  LaneK K;
  const bool odd = t & 1;
  K.m0 = odd ? 65536.f : 1.f;
  K.m1 = odd ? 0.f : 256.f;
  K.shl = (t >> 1) ? 0 : 16;
  return K;
}
__device__ __forceinline__ float bf16_sel(uint32_t wd, int shl) { return __uint_as_float((wd << shl) & 0xFFFF0000u); }

// One span of one 16-row tile: A codes of rows g (wa) and g+8 (wb), scale and
// bias words of those rows (bf16 pairs of the span's two groups); adds the
// dequantised products to acc_a (row g) and acc_b (row g+8).
template <int BITS>
__device__ __forceinline__ void tile_span(const uint32_t* wa, const uint32_t* wb, uint32_t sa, uint32_t sb, uint32_t ba,
                                          uint32_t bb, const BFrag& B, const LaneK& K, float& acc_a, float& acc_b) {
  int c[4] = {0, 0, 0, 0};
#pragma unroll
  for (int j = 0; j < 4; ++j)
    mma_u8s8(c, code_bytes_m<BITS>(wa, j, 0), code_bytes_m<BITS>(wb, j, 0), code_bytes_m<BITS>(wa, j, 1),
             code_bytes_m<BITS>(wb, j, 1), B.b[j].x, B.b[j].y);
  const float fa = fmaf((float)c[1], K.m1, (float)c[0] * K.m0);
  const float fb = fmaf((float)c[3], K.m1, (float)c[2] * K.m0);
  acc_a = fmaf(bf16_sel(sa, K.shl) * B.ip, fa, fmaf(bf16_sel(ba, K.shl), B.xg, acc_a));
  acc_b = fmaf(bf16_sel(sb, K.shl) * B.ip, fb, fmaf(bf16_sel(bb, K.shl), B.xg, acc_b));
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

// 4 integer MMAs over one span: c[0..1] = row g (cols 2t, 2t+1), c[2..3] = row g+8.
template <int BITS>
__device__ __forceinline__ void mma_frag(const Frag<BITS>& F, const uint2* __restrict__ bt, int bl, int (&c)[4]) {
  c[0] = c[1] = c[2] = c[3] = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint2 b = bl >= 0 ? bt[j * kBtLanes + bl] : make_uint2(0u, 0u);
    mma_u8s8(c, code_bytes<BITS>(F.wa, j, 0), code_bytes<BITS>(F.wb, j, 0), code_bytes<BITS>(F.wa, j, 1),
             code_bytes<BITS>(F.wb, j, 1), b.x, b.y);
  }
}

// Applies the group scales. Thread t holds columns 2t, 2t+1: digits of group
// grp = t>>1 (t even: d0, d1; t odd: d2), so each thread scales its own part;
// the even thread adds the bias term b * X_g. The four threads of a quad are
// summed when the tile is flushed.
__device__ __forceinline__ void scale_frag_i(uint32_t sa, uint32_t sb, uint32_t ba, uint32_t bb, const int (&c)[4],
                                             const float* igsc, const float* Xg, int span, int t, float& acc_a,
                                             float& acc_b) {
  const int grp = t >> 1, gi = 2 * span + grp;
  const bool odd = t & 1;
  const float fa = odd ? 65536.f * (float)c[0] : fmaf(256.f, (float)c[1], (float)c[0]);
  const float fb = odd ? 65536.f * (float)c[2] : fmaf(256.f, (float)c[3], (float)c[2]);
  const float ip = igsc[gi], xg = odd ? 0.f : Xg[gi];
  const float s_a = grp ? bf16hi(sa) : bf16lo(sa);
  const float s_b = grp ? bf16hi(sb) : bf16lo(sb);
  const float b_a = grp ? bf16hi(ba) : bf16lo(ba);
  const float b_b = grp ? bf16hi(bb) : bf16lo(bb);
  acc_a = fmaf(s_a * ip, fa, fmaf(b_a, xg, acc_a));
  acc_b = fmaf(s_b * ip, fb, fmaf(b_b, xg, acc_b));
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

// Rolling per-warp pipeline over the units of a warp range. The range meets
// at most two tiles (host guarantee); the units of each tile form a
// sub-range, and a pass selects which sub-ranges it runs (e.g. the shared
// expert's before the routing is known, the routed ones after). Up to NS
// units (a template argument) are in flight (cp.async, one commit group per
// unit); the oldest is computed when it lands and its slot is refilled.
struct SubRange { int tile, s0, s1, si; };

template <int BITS>
struct WarpPipe {
  SubRange sr[2];
  int n;              // sub-ranges of this pass
  int is, ispan;      // next unit to issue: sub-range index, span
  int cs, cspan;      // next unit to compute
  int issued, computed;
  LaneCopy<BITS> lc;
  int lc_tile;
};

// Sub-ranges of the warp range wr (tile = u / nspans) whose tile satisfies `take`.
template <int BITS, class TakeFn>
__device__ __forceinline__ void pipe_init(WarpPipe<BITS>& P, Range wr, int nspans, TakeFn take) {
  P.n = 0;
  P.is = P.cs = 0;
  P.issued = P.computed = 0;
  P.lc_tile = -1;
  if (wr.a >= wr.b) return;
  const int t0 = wr.a / nspans, t1 = (wr.b - 1) / nspans;
  for (int tile = t0; tile <= t1; ++tile) {
    const int lo = wr.a > tile * nspans ? wr.a - tile * nspans : 0;
    const int hi = wr.b < (tile + 1) * nspans ? wr.b - tile * nspans : nspans;
    if (take(tile)) P.sr[P.n++] = SubRange{tile, lo, hi, tile - t0};
  }
  if (P.n) { P.ispan = P.sr[0].s0; P.cspan = P.sr[0].s0; }
}

// Issues units until NS (<= 8) are in flight or the pass is exhausted.
template <int BITS, int NS, class RowFn>
__device__ __forceinline__ void pipe_issue(WarpPipe<BITS>& P, unsigned char* wslots, RowFn row, int lane) {
  static_assert(NS >= 1 && NS <= 8, "slots per warp");
  while (P.is < P.n && P.issued - P.computed < NS) {
    const SubRange& r = P.sr[P.is];
    if (P.lc_tile != r.tile) { P.lc = lane_copy<BITS>(row, r.tile, lane); P.lc_tile = r.tile; }
    stage_unit<BITS>(wslots + (P.issued % NS) * UnitSmem<BITS>::bytes, P.lc, P.ispan);
    cp_async_commit();
    ++P.issued;
    if (++P.ispan == r.s1 && ++P.is < P.n) P.ispan = P.sr[P.is].s0;
  }
}

// Computes every unit of the pass (issuing more as slots free up); partials of
// each sub-range go to ps.v[warp][si] / ps.tile[warp][si].
// bt_of(tile) gives the B table of the tile's vector, gs_of(tile) a pointer
// G with G[g] = 2^-p_g and G[gstride + g] = X_g for that vector.
template <int BITS, int NS, class RowFn, class BtFn, class GsFn>
__device__ __forceinline__ void pipe_run(WarpPipe<BITS>& P, unsigned char* wslots, RowFn row, BtFn bt_of, GsFn gs_of,
                                         int gstride, PartialSmem& ps, int warp, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int bl = bt_lane_index(lane);
  float acc_a = 0.f, acc_b = 0.f;
  while (P.cs < P.n) {
    pipe_issue<BITS, NS>(P, wslots, row, lane);
    const SubRange& r = P.sr[P.cs];
    cp_async_wait_dyn(P.issued - P.computed - 1);
    __syncwarp();
    Frag<BITS> F;
    frag_load<BITS>(F, wslots + (P.computed % NS) * UnitSmem<BITS>::bytes, g, t);
    int c[4];
    mma_frag<BITS>(F, bt_of(r.tile) + P.cspan * kBtPerSpan, bl, c);
    const float* G = gs_of(r.tile);
    scale_frag_i(F.sa, F.sb, F.ba, F.bb, c, G, G + gstride, P.cspan, t, acc_a, acc_b);
    __syncwarp();   // every lane has read the slot before it is refilled
    ++P.computed;
    if (++P.cspan == r.s1) {
      acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
      acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 1);
      acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 2);
      acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 2);
      if (t == 0) { ps.v[warp][r.si][g] = acc_a; ps.v[warp][r.si][g + 8] = acc_b; }
      if (lane == 0) ps.tile[warp][r.si] = r.tile;
      acc_a = acc_b = 0.f;
      if (++P.cs < P.n) P.cspan = P.sr[P.cs].s0;
    }
  }
}

__device__ __forceinline__ void partials_clear(PartialSmem& ps, int warp, int lane) {
  if (lane == 0) { ps.tile[warp][0] = -1; ps.tile[warp][1] = -1; }
  __syncwarp();
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
