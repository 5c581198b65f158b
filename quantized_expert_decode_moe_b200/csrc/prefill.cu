// Prefill path of the quantized MoE expert forward (T > 8 tokens, sm_100a):
// grouped dequantising GEMMs on the integer tensor cores.
//
// After routing, the (token, rank) pairs are grouped by expert and cut into
// chunks of up to C tokens of one expert (see group_kernel; the shared expert
// takes every token). The products are dense GEMMs of an expert's weight rows
// with a chunk's tokens as the N dimension:
//   gate/up:  a[pair][j] = silu(G_e[j] . x_t) * (U_e[j] . x_t)
//   down:     y[pair][h] = D_e[h] . a[pair]
// with w = q*s + b per group of 64 columns of a row ("Key technologies >
// FMA-optimised dequant kernel" of the Flash-MoE write-up), so
//   W_row . v = sum_g s_g (q_g . v_g) + b_g V_g,   V_g = sum of v over group g.
//
// Arithmetic: the codes enter the tensor cores as they are stored (u8 planes
// masked out of the packed words, no dequantisation); every activation row is
// written once as a 16-bit fixed-point number v = 2^-p (256 d1 + d0) with one
// exponent p per row and two s8 digits (pf_digitize_kernel). One
// mma.sync m16n8k32 (u8 x s8 -> s32) takes 16 weight rows x 32 columns
// against 4 tokens x 2 digits, so per group the integer sums are exact and
// the float work is one scale and one bias term per row, token and group.
//
// Work: an item is (chunk, 16-row block); the items are ordered chunk-major
// and every CTA (one per SM) takes one contiguous range of them, so a CTA
// meets only a few chunks and keeps their B fragments in registers. Each
// item's 16 code rows (padded in shared memory so that the 8 rows a warp
// reads fall in different banks), scales and biases arrive with bulk copies
// into a ring of stages, issued nst items ahead by one warp right after the
// block barrier that frees a stage; the 16 warps each take 1/16 of K and
// their partial sums are added in a fixed order.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace qmoe {

constexpr int kPfWarps = 16;                            // each owns 1/16 of K
constexpr int kPfThreads = kPfWarps * 32;
constexpr int kPfIssuer = kPfWarps - 1;                 // the warp that issues the bulk copies
constexpr int kPfMaxStages = 8;
constexpr int kPfDigitThreads = 256;

// ------------------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ unsigned long long pf_time_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void pf_mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void pf_expect(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void pf_bulk(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void pf_fence_proxy() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ bool pf_try(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait for the phase of parity `parity` of bar; on timeout latches
// MOE_ERR_TIMEOUT (when status is given) and returns false.
__device__ __noinline__ bool pf_wait_slow(uint64_t* bar, unsigned parity, unsigned long long bound_ns,
                                          uint32_t* status) {
  const unsigned long long t0 = pf_time_ns();
  while (!pf_try(bar, parity)) {
    if (pf_time_ns() - t0 > bound_ns) {
      if (status) atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool pf_wait(uint64_t* bar, unsigned parity, unsigned long long bound_ns,
                                        uint32_t* status) {
  if (pf_try(bar, parity)) return true;
  return pf_wait_slow(bar, parity, bound_ns, status);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ------------------------------------------------------------------ digit tables
// Position of the digits of a column inside its group's 128-byte block:
// [t][d][m][h][i] with t the quad lane that supplies it, d the digit (0 high,
// 1 low), m the MMA of the group, h the A register half (a0/a1 or a2/a3) and
// i the byte. Per lane t and MMA m the A side takes one packed word of the
// row: 4-bit word 2t+m (8 columns; low nibbles -> h = 0, high nibbles ->
// h = 1), 2-bit word t (16 columns; field 2m -> h = 0, field 2m+1 -> h = 1).
// So the 16 columns of unit u = 4*group + t fill one 32-byte run; this is the
// slot (m, h, i) -> 8m + 4h + i of column c16 of the unit.
template <int BITS>
__device__ __forceinline__ int pf_digit_slot(int c16) {
  if constexpr (BITS == 4) return (c16 >> 3) * 8 + (c16 & 1) * 4 + ((c16 & 7) >> 1);
  else return ((c16 & 3) >> 1) * 8 + (c16 & 1) * 4 + (c16 >> 2);
}

// One CTA per activation row: p = the largest exponent with max|v| * 2^p <=
// 32639 (so both digits fit s8 after rounding), v' = rint(v * 2^p),
// d1 = floor((v' + 128) / 256), d0 = v' - 256 d1; rs[row] = 2^-p and
// X[row][g] = the fp32 sum of the row's 64 values of group g.
template <int BITS, bool BF16>
__global__ void __launch_bounds__(kPfDigitThreads) pf_digitize_kernel(const void* src, int K, unsigned char* dig,
                                                                      float* X, float* rs) {
  __shared__ uint32_t red[kPfDigitThreads / 32];
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int units = K / 16, ng = K / kGroup;
  auto load16 = [&](int u, float (&v)[16]) {
    if constexpr (BF16) {
      const uint4* s = (const uint4*)((const uint16_t*)src + (size_t)row * K + 16 * u);
      const uint4 a = s[0], b = s[1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) { v[2 * i] = bf16_lo(w[i]); v[2 * i + 1] = bf16_hi(w[i]); }
    } else {
      const float4* s = (const float4*)((const float*)src + (size_t)row * K + 16 * u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = s[i];
        v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
      }
    }
  };
  uint32_t mx = 0;
  for (int u = tid; u < units; u += kPfDigitThreads) {
    float v[16];
    load16(u, v);
#pragma unroll
    for (int i = 0; i < 16; ++i) mx = max(mx, __float_as_uint(fabsf(v[i])));
  }
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  mx = 0;
#pragma unroll
  for (int w = 0; w < kPfDigitThreads / 32; ++w) mx = max(mx, red[w]);
  const float m = __uint_as_float(mx);
  int p = 0;
  if (m > 0.f) {
    const int e = (int)(mx >> 23);   // biased exponent (0 for a subnormal m)
    p = 141 - e;                     // m * 2^p in [2^14, 2^15) for a normal m
    if (p > 126) p = 126;
    if (m * __uint_as_float((uint32_t)(127 + p) << 23) > 32639.f) --p;
  }
  const float sc = __uint_as_float((uint32_t)(127 + p) << 23);
  if (tid == 0) rs[row] = __uint_as_float((uint32_t)(127 - p) << 23);
  for (int base = 0; base < units; base += kPfDigitThreads) {   // uniform trips: the quads shuffle below
    const int u = base + tid;
    const bool live = u < units;   // units is a multiple of 8, so a quad is live or idle as a whole
    float v[16];
    if (live) load16(u, v);
    else {
#pragma unroll
      for (int c = 0; c < 16; ++c) v[c] = 0.f;
    }
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};   // high digits [m][h], then low digits [m][h]
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      s += v[c];
      const int q = __float2int_rn(v[c] * sc);
      const int d1 = (q + 128) >> 8, d0 = q - (d1 << 8);
      const int slot = pf_digit_slot<BITS>(c);
      w[slot >> 2] |= (uint32_t)(d1 & 0xFF) << (8 * (slot & 3));
      w[4 + (slot >> 2)] |= (uint32_t)(d0 & 0xFF) << (8 * (slot & 3));
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (live) {
      uint4* o = (uint4*)(dig + (size_t)row * 2 * K + (size_t)(u >> 2) * 128 + (u & 3) * 32);
      o[0] = make_uint4(w[0], w[1], w[2], w[3]);
      o[1] = make_uint4(w[4], w[5], w[6], w[7]);
      if ((u & 3) == 0) X[(size_t)row * ng + (u >> 2)] = s;
    }
  }
}

// ------------------------------------------------------------------ grouped GEMM geometry
// Shared memory: nst stages of {codes [16][stride], scales [16][ng], biases
// [16][ng]} (stride = row bytes + 8*bits, so the rows a warp reads at one
// column start 8*bits bytes apart in the banks), partial sums [2][16 warps]
// [16 rows][C], output rows [2][C], one barrier per stage.
struct PfGeom { int RB, SRB, stride, nst; size_t stage, sc, bi, part, rows, bars, total; };
__host__ __device__ inline PfGeom pf_geom(int K, int bits, int C, int nst) {
  PfGeom G;
  G.RB = K * bits / 8;
  G.SRB = (K / kGroup) * 2;
  G.stride = G.RB + 8 * bits;
  G.sc = (size_t)16 * G.stride;
  G.bi = G.sc + (size_t)16 * G.SRB;
  G.stage = (G.bi + (size_t)16 * G.SRB + 127) & ~(size_t)127;
  G.nst = nst;
  size_t o = G.stage * nst;
  G.part = o; o += sizeof(float) * 2 * kPfWarps * 16 * C;
  G.rows = o; o += sizeof(int) * 2 * C;
  o = (o + 15) & ~(size_t)15;
  G.bars = o; o += sizeof(uint64_t) * kPfMaxStages;
  G.total = o;
  return G;
}

// activation row of token j of a chunk {e, pos, n}: x row (gate/up) or pair row (down)
__device__ __forceinline__ int pf_in_row(const PrefillParams& p, int4 ch, int j, bool gu) {
  if (ch.x == p.E) return gu ? ch.y + j : p.T * p.k + ch.y + j;
  const int pair = __ldg(p.perm + ch.y + j);
  return gu ? pair / p.k : pair;
}
// output row (pair index; T*k + t for the shared expert)
__device__ __forceinline__ int pf_out_row(const PrefillParams& p, int4 ch, int j) {
  return ch.x == p.E ? p.T * p.k + ch.y + j : __ldg(p.perm + ch.y + j);
}
__device__ __forceinline__ moe_qmat pf_mat(const PrefillParams& p, int e, int which) {   // 0 gate, 1 up, 2 down
  if (e == p.E) return which == 0 ? p.shared.gate : (which == 1 ? p.shared.up : p.shared.down);
  const moe_expert* x = p.experts + e;
  return which == 0 ? x->gate : (which == 1 ? x->up : x->down);
}

// Persistent grouped GEMM (GU: gate/up + SwiGLU -> a; else down -> y).
// GPW: most groups per warp; TILES: 4-token tiles per chunk.
template <int BITS, bool GU, int GPW, int TILES>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_grouped_kernel(PrefillParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int C = 4 * TILES;
  const int K = GU ? p.H : p.I;
  const int R = GU ? p.I / 8 : p.H / 16;   // 16-row blocks per expert
  const int ng = K / kGroup;
  const PfGeom G = pf_geom(K, BITS, C, p.nst);
  const int nst = G.nst;
  uint64_t* full = (uint64_t*)(smem + G.bars);
  float* part = (float*)(smem + G.part);
  int* rows_out = (int*)(smem + G.rows);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long N = (long long)__ldg(p.nchunks) * R;
  const long long lo = N * blockIdx.x / gridDim.x, hi = N * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(hi - lo);
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) pf_mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const unsigned item_bytes = 16u * G.RB + 32u * G.SRB;
  // Copies of local item i into stage i % nst (issuer warp: lane 0 arms the
  // barrier, one lane per copy).
  int icur = -1, ie = 0;
  auto issue = [&](int i) {
    const int st = i % nst;
    const long long item = lo + i;
    const int ci = (int)(item / R), rb = (int)(item - (long long)ci * R);
    if (ci != icur) { icur = ci; ie = __ldg(&p.chunks[ci].x); }
    const int e = ie;
    unsigned char* sb = smem + (size_t)st * G.stage;
    if (lane == 0) pf_expect(&full[st], item_bytes);
    __syncwarp();
    if (GU) {
      if (lane < 16) {   // code rows: gate rows rb*8.. -> 0..7, up rows -> 8..15
        const moe_qmat m = pf_mat(p, e, lane >> 3);
        pf_bulk(sb + (size_t)lane * G.stride, (const char*)m.q + (size_t)(rb * 8 + (lane & 7)) * G.RB, G.RB,
                &full[st]);
      } else if (lane < 20) {   // 16 gate scales, 17 up scales, 18 gate biases, 19 up biases
        const int c = lane - 16;
        const moe_qmat m = pf_mat(p, e, c & 1);
        pf_bulk(sb + (c < 2 ? G.sc : G.bi) + (size_t)(c & 1) * 8 * G.SRB,
                (const char*)(c < 2 ? m.scales : m.biases) + (size_t)rb * 8 * G.SRB, 8u * G.SRB, &full[st]);
      }
    } else if (lane < 18) {   // 16 code rows, then scales and biases
      const moe_qmat m = pf_mat(p, e, 2);
      if (lane < 16)
        pf_bulk(sb + (size_t)lane * G.stride, (const char*)m.q + (size_t)(rb * 16 + lane) * G.RB, G.RB, &full[st]);
      else
        pf_bulk(sb + (lane == 16 ? G.sc : G.bi),
                (const char*)(lane == 16 ? m.scales : m.biases) + (size_t)rb * 16 * G.SRB, 16u * G.SRB, &full[st]);
    }
  };
  if (warp == kPfIssuer)
    for (int i = 0; i < nloc && i < nst; ++i) issue(i);

  const int g = lane >> 2, t = lane & 3;
  const int gpw = (ng + kPfWarps - 1) / kPfWarps;
  const int g0 = warp * gpw;
  const int mg = max(0, min(gpw, ng - g0));   // groups of this warp
  const unsigned char* dig = GU ? p.xd : p.ad;
  const float* Xt = GU ? p.xX : p.aX;
  const float* rst = GU ? p.xrs : p.ars;
  const bool vec_sb = (mg == GPW) && (ng % GPW == 0);   // the warp's scales in one load per row
  uint4 bq[TILES][GPW];
  float xg[TILES][GPW], rsc[TILES];
  int cur = -1, n = 0, orow = -1;
  for (int i = 0; i < nloc; ++i) {
    const int st = i % nst;
    const long long item = lo + i;
    const int ci = (int)(item / R), rb = (int)(item - (long long)ci * R);
    if (ci != cur) {   // new chunk: B fragments and group sums of its tokens
      cur = ci;
      const int4 ch = __ldg(&p.chunks[ci]);
      n = ch.z;
#pragma unroll
      for (int tau = 0; tau < TILES; ++tau) {
        const int jb = 4 * tau + (g >> 1), jc = 4 * tau + t;   // B column g = (token g/2, digit g%2); C token t
        const int rB = jb < n ? pf_in_row(p, ch, jb, GU) : -1;
        const int rC = jc < n ? pf_in_row(p, ch, jc, GU) : -1;
        const unsigned char* db = dig + (size_t)(rB < 0 ? 0 : rB) * 2 * K + (size_t)t * 32 + (g & 1) * 16;
#pragma unroll
        for (int gi = 0; gi < GPW; ++gi) {
          bq[tau][gi] = (rB >= 0 && gi < mg) ? __ldg((const uint4*)(db + (size_t)(g0 + gi) * 128))
                                             : make_uint4(0u, 0u, 0u, 0u);
          xg[tau][gi] = (rC >= 0 && gi < mg) ? __ldg(Xt + (size_t)rC * ng + g0 + gi) : 0.f;
        }
        rsc[tau] = rC >= 0 ? __ldg(rst + rC) : 0.f;
      }
      if (warp == 0 && lane < C) orow = lane < n ? pf_out_row(p, ch, lane) : -1;
    }
    if (warp == 0 && lane < C) rows_out[(i & 1) * C + lane] = orow;
    pf_wait(&full[st], (unsigned)(i / nst) & 1u, p.wait_ns, p.status);
    const unsigned char* sb = smem + (size_t)st * G.stage;
    const uint16_t* ssc = (const uint16_t*)(sb + G.sc);
    const uint16_t* sbi = (const uint16_t*)(sb + G.bi);
    // scales / biases of rows g and g+8 for the warp's groups
    float sA[GPW], sB[GPW], bA[GPW], bB[GPW];
    if (vec_sb) {
      using V = typename std::conditional<GPW == 4, uint2, uint4>::type;
      const V va = *(const V*)(ssc + (size_t)g * ng + g0), vb = *(const V*)(ssc + (size_t)(g + 8) * ng + g0);
      const V wa = *(const V*)(sbi + (size_t)g * ng + g0), wb = *(const V*)(sbi + (size_t)(g + 8) * ng + g0);
      const uint32_t* pa = (const uint32_t*)&va;
      const uint32_t* pb = (const uint32_t*)&vb;
      const uint32_t* qa = (const uint32_t*)&wa;
      const uint32_t* qb = (const uint32_t*)&wb;
#pragma unroll
      for (int h = 0; h < GPW / 2; ++h) {
        sA[2 * h] = bf16_lo(pa[h]); sA[2 * h + 1] = bf16_hi(pa[h]);
        sB[2 * h] = bf16_lo(pb[h]); sB[2 * h + 1] = bf16_hi(pb[h]);
        bA[2 * h] = bf16_lo(qa[h]); bA[2 * h + 1] = bf16_hi(qa[h]);
        bB[2 * h] = bf16_lo(qb[h]); bB[2 * h + 1] = bf16_hi(qb[h]);
      }
    } else {
#pragma unroll
      for (int gi = 0; gi < GPW; ++gi) {
        const int gg = gi < mg ? g0 + gi : 0;
        sA[gi] = bf16_lo(ssc[(size_t)g * ng + gg]); sB[gi] = bf16_lo(ssc[(size_t)(g + 8) * ng + gg]);
        bA[gi] = bf16_lo(sbi[(size_t)g * ng + gg]); bB[gi] = bf16_lo(sbi[(size_t)(g + 8) * ng + gg]);
      }
    }
    float sacc[TILES][2], bacc[TILES][2];
#pragma unroll
    for (int tau = 0; tau < TILES; ++tau) sacc[tau][0] = sacc[tau][1] = bacc[tau][0] = bacc[tau][1] = 0.f;
    const unsigned char* ra = sb + (size_t)g * G.stride;
    const unsigned char* rbp = sb + (size_t)(g + 8) * G.stride;
#pragma unroll
    for (int gi = 0; gi < GPW; ++gi) {
      if (gi < mg) {
        const int grp = g0 + gi;
        uint32_t A[2][4];   // per MMA m: a0 (row g, h 0), a1 (row g+8, h 0), a2 (row g, h 1), a3 (row g+8, h 1)
        if constexpr (BITS == 4) {
          const uint2 ua = *(const uint2*)(ra + grp * 32 + 8 * t), ub = *(const uint2*)(rbp + grp * 32 + 8 * t);
          A[0][0] = ua.x & 0x0F0F0F0Fu; A[0][2] = (ua.x >> 4) & 0x0F0F0F0Fu;
          A[0][1] = ub.x & 0x0F0F0F0Fu; A[0][3] = (ub.x >> 4) & 0x0F0F0F0Fu;
          A[1][0] = ua.y & 0x0F0F0F0Fu; A[1][2] = (ua.y >> 4) & 0x0F0F0F0Fu;
          A[1][1] = ub.y & 0x0F0F0F0Fu; A[1][3] = (ub.y >> 4) & 0x0F0F0F0Fu;
        } else {
          const uint32_t ua = *(const uint32_t*)(ra + grp * 16 + 4 * t);
          const uint32_t ub = *(const uint32_t*)(rbp + grp * 16 + 4 * t);
#pragma unroll
          for (int m = 0; m < 2; ++m) {
            A[m][0] = (ua >> (4 * m)) & 0x03030303u; A[m][2] = (ua >> (4 * m + 2)) & 0x03030303u;
            A[m][1] = (ub >> (4 * m)) & 0x03030303u; A[m][3] = (ub >> (4 * m + 2)) & 0x03030303u;
          }
        }
#pragma unroll
        for (int tau = 0; tau < TILES; ++tau) {
          int c[4] = {0, 0, 0, 0};
          const uint4 b = bq[tau][gi];
          mma_u8s8(c, A[0][0], A[0][1], A[0][2], A[0][3], b.x, b.y);
          mma_u8s8(c, A[1][0], A[1][1], A[1][2], A[1][3], b.z, b.w);
          // columns 2t, 2t+1 of the tile: token t's high- and low-digit sums
          sacc[tau][0] = fmaf(sA[gi], (float)(c[0] * 256 + c[1]), sacc[tau][0]);
          sacc[tau][1] = fmaf(sB[gi], (float)(c[2] * 256 + c[3]), sacc[tau][1]);
          bacc[tau][0] = fmaf(bA[gi], xg[tau][gi], bacc[tau][0]);
          bacc[tau][1] = fmaf(bB[gi], xg[tau][gi], bacc[tau][1]);
        }
      }
    }
    float* pw = part + ((size_t)(i & 1) * kPfWarps + warp) * 16 * C;
#pragma unroll
    for (int tau = 0; tau < TILES; ++tau) {
      pw[g * C + 4 * tau + t] = fmaf(sacc[tau][0], rsc[tau], bacc[tau][0]);
      pw[(g + 8) * C + 4 * tau + t] = fmaf(sacc[tau][1], rsc[tau], bacc[tau][1]);
    }
    pf_fence_proxy();   // this thread's reads of the stage precede the copies that refill it
    __syncthreads();
    if (warp == kPfIssuer && i + nst < nloc) issue(i + nst);   // stage st is free again
    // outputs: the 16 warps' partials added in a fixed order, L lanes per output
    const float* pr = part + (size_t)(i & 1) * kPfWarps * 16 * C;
    const int* ro = rows_out + (i & 1) * C;
    if (GU) {
      constexpr int L = kPfWarps * 32 / (8 * C), PW = kPfWarps / L;   // lanes per output, warps per lane
      const int o = tid / L, s = tid - o * L;   // o = x * 8 + j
      const int x = o >> 3, j = o & 7;
      float gs = 0.f, us = 0.f;
#pragma unroll
      for (int w = 0; w < PW; ++w) {
        const float* pq = pr + (size_t)(s * PW + w) * 16 * C;
        gs += pq[j * C + x];
        us += pq[(8 + j) * C + x];
      }
#pragma unroll
      for (int off = 1; off < L; off <<= 1) {
        gs += __shfl_xor_sync(0xffffffffu, gs, off);
        us += __shfl_xor_sync(0xffffffffu, us, off);
      }
      if (s == 0 && x < n) p.a[(size_t)ro[x] * p.I + rb * 8 + j] = gs / (1.f + expf(-gs)) * us;
    } else {
      constexpr int L = kPfWarps * 32 / (16 * C), PW = kPfWarps / L;
      const int o = tid / L, s = tid - o * L;   // o = x * 16 + r
      const int x = o >> 4, r = o & 15;
      float y = 0.f;
#pragma unroll
      for (int w = 0; w < PW; ++w) y += pr[(size_t)(s * PW + w) * 16 * C + r * C + x];
#pragma unroll
      for (int off = 1; off < L; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
      if (s == 0 && x < n) p.y[(size_t)ro[x] * p.H + rb * 16 + r] = y;
    }
  }
  // every copy this CTA issued has landed before it exits (immediate unless a wait above gave up)
  if (warp == kPfIssuer)
    for (int i = nloc - nst < 0 ? 0 : nloc - nst; i < nloc; ++i)
      pf_wait(&full[i % nst], (unsigned)(i / nst) & 1u, p.wait_ns, nullptr);
}

// ------------------------------------------------------------------ launchers
int pf_chunk_tokens(int H, int I) { return (H > 4096 || I > 4096) ? 4 : 8; }

static cudaError_t pf_prepare(const void* fn, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int BITS, bool GU>
static cudaError_t pf_grouped(const PrefillParams& p, cudaStream_t s) {
  const int K = GU ? p.H : p.I;
  const int C = pf_chunk_tokens(p.H, p.I);
  const int ng = K / kGroup, gpw = (ng + kPfWarps - 1) / kPfWarps;
  int optin = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const size_t fixed = pf_geom(K, BITS, C, 0).total;
  const size_t stage = pf_geom(K, BITS, C, 1).stage;
  if ((size_t)optin < fixed + 2 * stage) return cudaErrorInvalidConfiguration;
  int nst = (int)(((size_t)optin - fixed) / stage);
  if (nst > kPfMaxStages) nst = kPfMaxStages;
  if (gpw > (C == 8 ? 4 : 8)) return cudaErrorInvalidConfiguration;
  PrefillParams q = p;
  q.nst = nst;
  const size_t sm = pf_geom(K, BITS, C, nst).total;
  const void* fn = C == 8 ? (const void*)prefill_grouped_kernel<BITS, GU, 4, 2>
                          : (const void*)prefill_grouped_kernel<BITS, GU, 8, 1>;
  cudaError_t e = pf_prepare(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  return cudaLaunchKernel(fn, dim3(num_sms()), dim3(kPfThreads), args, sm, s);
}

template <int BITS, bool BF16>
static cudaError_t pf_digitize(const void* src, int rows, int K, unsigned char* dig, float* X, float* rs,
                               cudaStream_t s) {
  pf_digitize_kernel<BITS, BF16><<<rows, kPfDigitThreads, 0, s>>>(src, K, dig, X, rs);
  return cudaGetLastError();
}

cudaError_t launch_prefill_gateup(const PrefillParams& p, int bits, cudaStream_t s) {
  cudaError_t e = bits == 4 ? pf_digitize<4, true>(p.x, p.T, p.H, p.xd, p.xX, p.xrs, s)
                            : pf_digitize<2, true>(p.x, p.T, p.H, p.xd, p.xX, p.xrs, s);
  if (e != cudaSuccess) return e;
  return bits == 4 ? pf_grouped<4, true>(p, s) : pf_grouped<2, true>(p, s);
}

cudaError_t launch_prefill_down(const PrefillParams& p, int bits, cudaStream_t s) {
  const int rows = p.T * p.k + (p.has_shared ? p.T : 0);
  cudaError_t e = bits == 4 ? pf_digitize<4, false>(p.a, rows, p.I, p.ad, p.aX, p.ars, s)
                            : pf_digitize<2, false>(p.a, rows, p.I, p.ad, p.aX, p.ars, s);
  if (e != cudaSuccess) return e;
  return bits == 4 ? pf_grouped<4, false>(p, s) : pf_grouped<2, false>(p, s);
}

}  // namespace qmoe
