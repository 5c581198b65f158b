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
// exponent p per 64-value group and two s8 digits (pf_digitize_kernel). One
// mma.sync m16n8k32 (u8 x s8 -> s32) takes 16 weight rows x 32 columns
// against 4 tokens x 2 digits, so per group the integer sums are exact and
// the float work is one scale and one bias term per row, token and group.
//
// Work: an item is (chunk, 16-row block); the items are ordered chunk-major
// and every CTA (one per SM) takes one contiguous range of them, so a CTA
// meets only a few chunks and keeps their B fragments in registers. Each
// item's 16 code rows (padded in shared memory so that the 8 rows a warp
// reads fall in different banks), scales and biases arrive with bulk copies
// into a ring of stages, issued nst items ahead by all warps (one row each)
// right after the block barrier that frees a stage; the 16 warps each take
// 1/16 of K and their partial sums are added in a fixed order.
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace qmoe {

constexpr int kPfWarps = 16;                            // each owns 1/16 of K
constexpr int kPfThreads = kPfWarps * 32;
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

// One CTA per activation row, one exponent per quantisation group g of 64
// values: p_g = the largest exponent with max|v_g| * 2^p_g <= 32639 (so both
// digits fit s8 after rounding), v' = rint(v * 2^p_g), d1 = floor((v' + 128)
// / 256), d0 = v' - 256 d1; rs[row][g] = 2^-p_g and X[row][g] = the fp32 sum
// of the group's values. A group's four 16-value units sit on the four
// threads of a quad, so its maximum and sum are quad reductions. (A group
// exponent keeps 16 bits relative to the group's own maximum: a large value
// elsewhere in the row costs the other groups nothing.)
template <int BITS, bool BF16>
__global__ void __launch_bounds__(kPfDigitThreads) pf_digitize_kernel(const void* src, int K, unsigned char* dig,
                                                                      float* X, float* rs) {
  const int row = blockIdx.x, tid = threadIdx.x;
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
  for (int base = 0; base < units; base += kPfDigitThreads) {   // uniform trips: the quads shuffle below
    const int u = base + tid;
    const bool live = u < units;   // units is a multiple of 4, so a quad is live or idle as a whole
    float v[16];
    if (live) load16(u, v);
    else {
#pragma unroll
      for (int c = 0; c < 16; ++c) v[c] = 0.f;
    }
    uint32_t mx = 0;
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) { mx = max(mx, __float_as_uint(fabsf(v[c]))); s += v[c]; }
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    const float m = __uint_as_float(mx);
    int p = 0;
    if (m > 0.f) {
      const int e = (int)(mx >> 23);   // biased exponent (0 for a subnormal m)
      p = 141 - e;                     // m * 2^p in [2^14, 2^15) for a normal m
      if (p > 126) p = 126;
      if (m * __uint_as_float((uint32_t)(127 + p) << 23) > 32639.f) --p;
    }
    const float sc = __uint_as_float((uint32_t)(127 + p) << 23);
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};   // high digits [m][h], then low digits [m][h]
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int q = __float2int_rn(v[c] * sc);
      const int d1 = (q + 128) >> 8, d0 = q - (d1 << 8);
      const int slot = pf_digit_slot<BITS>(c);
      w[slot >> 2] |= (uint32_t)(d1 & 0xFF) << (8 * (slot & 3));
      w[4 + (slot >> 2)] |= (uint32_t)(d0 & 0xFF) << (8 * (slot & 3));
    }
    if (live) {
      uint4* o = (uint4*)(dig + (size_t)row * 2 * K + (size_t)(u >> 2) * 128 + (u & 3) * 32);
      o[0] = make_uint4(w[0], w[1], w[2], w[3]);
      o[1] = make_uint4(w[4], w[5], w[6], w[7]);
      if ((u & 3) == 0) {
        X[(size_t)row * ng + (u >> 2)] = s;
        rs[(size_t)row * ng + (u >> 2)] = __uint_as_float((uint32_t)(127 - p) << 23);
      }
    }
  }
}

// ------------------------------------------------------------------ grouped GEMM geometry
// An item holds TT = RT * RW tiles of 16 weight rows (gate/up: tile r = 8
// gate rows and the 8 up rows of the same intermediate indices): the 16 warps
// form RT groups of NS = 16 / RT K-slices, and each warp takes RW consecutive
// tiles of its slice. Shared memory: nst stages of {codes [16 TT][stride],
// scales [16 TT][ng], biases [16 TT][ng]} (stride = row bytes + 8*bits, so the
// rows a warp reads at one column start 8*bits bytes apart in the banks;
// gate/up scales and biases are [gate 8 TT][up 8 TT]), partial sums
// [2][NS][16 TT rows][C], output rows [2][C], one barrier per stage.
struct PfGeom { int RB, SRB, stride, nst; size_t stage, sc, bi, part, rows, bars, total; };
__host__ __device__ inline PfGeom pf_geom(int K, int bits, int C, int RT, int RW, int nst) {
  PfGeom G;
  const int TT = RT * RW;   // 16-row tiles per item
  G.RB = K * bits / 8;
  G.SRB = (K / kGroup) * 2;
  G.stride = G.RB + 8 * bits;
  G.sc = (size_t)16 * TT * G.stride;
  G.bi = G.sc + (size_t)16 * TT * G.SRB;
  G.stage = (G.bi + (size_t)16 * TT * G.SRB + 127) & ~(size_t)127;
  G.nst = nst;
  size_t o = G.stage * nst;
  G.part = o; o += sizeof(float) * 2 * kPfWarps * 16 * RW * C;   // [2][NS slices][16 TT rows][C]
  G.rows = o; o += sizeof(int) * 2 * C;
  o = (o + 15) & ~(size_t)15;
  G.bars = o; o += sizeof(uint64_t) * kPfMaxStages;
  G.total = o;
  return G;
}
// row tiles per item: enough that every warp owns up to 4 groups of its K-slice
__host__ __device__ inline int pf_row_tiles(int K) {
  const int ng = K / kGroup;
  return ng >= 64 ? 1 : (ng >= 32 ? 2 : 4);
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
// GPW: most groups per warp; TILES: 4-token tiles per chunk. Warp w takes row
// tile w / NS of the item and K-slice w % NS (NS = 16 / RT slices of ng / NS
// groups each).
template <int BITS, bool GU, int GPW, int TILES>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_grouped_kernel(PrefillParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int C = 4 * TILES;
  const int K = GU ? p.H : p.I;
  const int RT = p.rt;                                 // tile groups per item (1, 2 or 4)
  const int RW = p.rw;                                 // tiles per warp (1 or 2)
  const int TT = RT * RW;                              // 16-row tiles per item
  const int rshift = RT == 1 ? 0 : (RT == 2 ? 1 : 2);
  const int tshift = rshift + (RW == 2 ? 1 : 0);       // log2 TT
  const int NS = kPfWarps >> rshift;                   // K-slices
  const int R = GU ? p.I / (8 * TT) : p.H / (16 * TT); // items per chunk
  const int ng = K / kGroup;
  const PfGeom G = pf_geom(K, BITS, C, RT, RW, p.nst);
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
  const unsigned item_bytes = 16u * TT * G.RB + 32u * TT * G.SRB;
  const int ci0 = (int)(lo / R), rb0 = (int)(lo - (long long)ci0 * R);

  // Copies of the next item to issue (cursor ici, irb) into stage st. Lane 0
  // of warp w copies code rows w, w+16, ... of the item; warps 0-3 (gate/up)
  // or 0-1 (down) also one scale or bias block. The stage's barrier is armed
  // by thread 0 before the block barrier that precedes these copies.
  int ici = ci0, irb = rb0, icur = -1, ie = -1;
  const char* mq = nullptr;    // this warp's code rows (gate/up: gate for warps 0-7, up for 8-15)
  const char* msb = nullptr;   // this warp's scale or bias block (warps 0-3 / 0-1)
  auto issue = [&](int st) {
    if (ici != icur) {
      icur = ici;
      const int e = __ldg(&p.chunks[ici].x);
      if (e != ie) {
        ie = e;
        const moe_qmat m = pf_mat(p, e, GU ? (warp >> 3) : 2);
        mq = (const char*)m.q;
        if (GU && warp < 4) {
          const moe_qmat ms = pf_mat(p, e, warp & 1);
          msb = (const char*)(warp < 2 ? ms.scales : ms.biases);
        } else if (!GU && warp < 2) {
          msb = (const char*)(warp == 0 ? m.scales : m.biases);
        }
      }
    }
    unsigned char* sb = smem + (size_t)st * G.stage;
    for (int r = warp; r < 16 * TT; r += kPfWarps) {
      const int tr = r >> 4, q = r & 15;
      const int src = GU ? irb * 8 * TT + 8 * tr + (q & 7) : irb * 16 * TT + r;
      pf_bulk(sb + (size_t)r * G.stride, mq + (size_t)src * G.RB, G.RB, &full[st]);
    }
    if (GU && warp < 4)   // 0 gate scales, 1 up scales, 2 gate biases, 3 up biases
      pf_bulk(sb + (warp < 2 ? G.sc : G.bi) + (size_t)(warp & 1) * 8 * TT * G.SRB,
              msb + (size_t)irb * 8 * TT * G.SRB, 8u * TT * G.SRB, &full[st]);
    else if (!GU && warp < 2)
      pf_bulk(sb + (warp == 0 ? G.sc : G.bi), msb + (size_t)irb * 16 * TT * G.SRB, 16u * TT * G.SRB, &full[st]);
    if (++irb == R) { irb = 0; ++ici; }
  };
  if (tid == 0)
    for (int i = 0; i < nloc && i < nst; ++i) pf_expect(&full[i], item_bytes);
  __syncthreads();
  if (lane == 0)
    for (int i = 0; i < nloc && i < nst; ++i) issue(i);

  const int g = lane >> 2, t = lane & 3;
  const int tg = warp >> (4 - rshift), ks = warp & (NS - 1);   // tile group, K-slice
  const int gpw = (ng + NS - 1) / NS;
  const int g0 = ks * gpw;
  const int mg = max(0, min(gpw, ng - g0));   // groups of this warp
  const unsigned char* dig = GU ? p.xd : p.ad;
  const float* Xt = GU ? p.xX : p.aX;
  const float* rst = GU ? p.xrs : p.ars;
  const bool vec_sb = (mg == GPW) && (ng % GPW == 0);   // the warp's scales in one load per row
  uint4 bq[TILES][GPW];
  float xg[TILES][GPW], rsg[TILES][GPW];
  int cur = -1, n = 0, orow = -1;
  int ci = ci0, rb = rb0, st = 0;
  unsigned phase = 0;
  for (int i = 0; i < nloc; ++i) {
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
          rsg[tau][gi] = (rC >= 0 && gi < mg) ? __ldg(rst + (size_t)rC * ng + g0 + gi) : 0.f;
        }
      }
      if (warp == 0 && lane < C) orow = lane < n ? pf_out_row(p, ch, lane) : -1;
    }
    if (warp == 0 && lane < C) rows_out[(i & 1) * C + lane] = orow;
    pf_wait(&full[st], phase, p.wait_ns, p.status);
    const unsigned char* sb = smem + (size_t)st * G.stage;
    const uint16_t* ssc = (const uint16_t*)(sb + G.sc);
    const uint16_t* sbi = (const uint16_t*)(sb + G.bi);
    float* pw = part + ((size_t)(i & 1) * NS + ks) * 16 * TT * C;   // part[buf][ks][tile row][token]
#pragma unroll 1
    for (int rr = 0; rr < RW; ++rr) {   // the warp's tiles, one at a time
      const int tr = tg * RW + rr;
      // shared-memory rows of the tile: A rows g (gate / first 8) and g+8 (up / last 8)
      const int crA = 16 * tr + g, crB = 16 * tr + 8 + g;
      const int srA = GU ? 8 * tr + g : crA, srB = GU ? 8 * TT + 8 * tr + g : crB;
      // scales / biases of the warp's two rows for its groups
      float sA[GPW], sB[GPW], bA[GPW], bB[GPW];
      if (vec_sb) {
        using V = typename std::conditional<GPW == 4, uint2, uint4>::type;
        const V va = *(const V*)(ssc + (size_t)srA * ng + g0), vb = *(const V*)(ssc + (size_t)srB * ng + g0);
        const V wa = *(const V*)(sbi + (size_t)srA * ng + g0), wb = *(const V*)(sbi + (size_t)srB * ng + g0);
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
          sA[gi] = sB[gi] = bA[gi] = bB[gi] = 0.f;
          if (gi < mg) {
            const int gg = g0 + gi;
            sA[gi] = bf16_lo(ssc[(size_t)srA * ng + gg]); sB[gi] = bf16_lo(ssc[(size_t)srB * ng + gg]);
            bA[gi] = bf16_lo(sbi[(size_t)srA * ng + gg]); bB[gi] = bf16_lo(sbi[(size_t)srB * ng + gg]);
          }
        }
      }
      float sacc[TILES][2], bacc[TILES][2];
#pragma unroll
      for (int tau = 0; tau < TILES; ++tau) sacc[tau][0] = sacc[tau][1] = bacc[tau][0] = bacc[tau][1] = 0.f;
      const unsigned char* ra = sb + (size_t)crA * G.stride;
      const unsigned char* rbp = sb + (size_t)crB * G.stride;
      // one quantisation group of the warp's K-slice; the groups go in pairs,
      // so two groups' MMA chains share a basic block and interleave
      auto group = [&](int gi) {
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
          sacc[tau][0] = fmaf(sA[gi] * rsg[tau][gi], (float)(c[0] * 256 + c[1]), sacc[tau][0]);
          sacc[tau][1] = fmaf(sB[gi] * rsg[tau][gi], (float)(c[2] * 256 + c[3]), sacc[tau][1]);
          bacc[tau][0] = fmaf(bA[gi], xg[tau][gi], bacc[tau][0]);
          bacc[tau][1] = fmaf(bB[gi], xg[tau][gi], bacc[tau][1]);
        }
      };
#pragma unroll
      for (int gp = 0; gp < GPW; gp += 2) {
        if (gp + 1 < mg) { group(gp); group(gp + 1); }
        else if (gp < mg) group(gp);
      }
#pragma unroll
      for (int tau = 0; tau < TILES; ++tau) {
        pw[crA * C + 4 * tau + t] = sacc[tau][0] + bacc[tau][0];
        pw[crB * C + 4 * tau + t] = sacc[tau][1] + bacc[tau][1];
      }
    }
    if (tid == 0 && i + nst < nloc) pf_expect(&full[st], item_bytes);   // its phase for item i is complete
    __syncthreads();
    if (lane == 0 && i + nst < nloc) {   // stage st is free again: item i + nst
      pf_fence_proxy();   // the block's reads of the stage (ordered by the barrier) precede the refill
      issue(st);
    }
    // outputs: one thread per output adds the NS slices' partials in slice order
    const float* pr = part + (size_t)(i & 1) * NS * 16 * TT * C;
    const int* ro = rows_out + (i & 1) * C;
    const int slice = 16 * TT * C;   // floats per slice
    if (GU) {
      for (int o = tid; o < 8 * TT * C; o += kPfThreads) {   // o = x * 8 TT + jj
        const int x = o >> (3 + tshift), jj = o & (8 * TT - 1);
        const int prow = 16 * (jj >> 3) + (jj & 7);
        const float* pq = pr + prow * C + x;
        float gs = 0.f, us = 0.f;
        for (int w = 0; w < NS; ++w) {
          gs += pq[w * slice];
          us += pq[w * slice + 8 * C];
        }
        if (x < n) p.a[(size_t)ro[x] * p.I + rb * 8 * TT + jj] = gs / (1.f + expf(-gs)) * us;
      }
    } else {
      for (int o = tid; o < 16 * TT * C; o += kPfThreads) {   // o = x * 16 TT + rr
        const int x = o >> (4 + tshift), rr = o & (16 * TT - 1);
        const float* pq = pr + rr * C + x;
        float y = 0.f;
        for (int w = 0; w < NS; ++w) y += pq[w * slice];
        if (x < n) p.y[(size_t)ro[x] * p.H + rb * 16 * TT + rr] = y;
      }
    }
    if (++st == nst) { st = 0; phase ^= 1u; }
    if (++rb == R) { rb = 0; ++ci; }
  }
  // every copy this CTA issued has landed before it exits (immediate unless a wait above gave up)
  if (lane == 0)
    for (int i = nloc - nst < 0 ? 0 : nloc - nst; i < nloc; ++i)
      pf_wait(&full[i % nst], (unsigned)(i / nst) & 1u, p.wait_ns, nullptr);
}

// ------------------------------------------------------------------ grouping by expert
// Exclusive scan of v[0..n) in place (one block); returns the total.
__device__ int block_exclusive_scan(int* v, int n, int* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  int carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int e = base + tid;
    const int x = e < n ? v[e] : 0;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int wv = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wv, o);
        if (lane >= o) wv += y;
      }
      if (lane < nw) warp_tot[lane] = wv;
    }
    __syncthreads();
    if (e < n) v[e] = carry + (warp ? warp_tot[warp - 1] : 0) + incl - x;
    const int tot = warp_tot[nw - 1];
    __syncthreads();
    carry += tot;
  }
  return carry;
}

// Prefill grouping in one CTA: histogram of the chosen experts, exclusive
// scan, then a stable scatter of the flattened (token, rank) pairs by one warp
// that walks them in order 32 at a time (ranks of equal experts from
// __match_any_sync). Also the chunk list of the grouped GEMMs: expert e's
// pairs in runs of `chunk`, then the shared expert's tokens in runs of `chunk`.
__global__ void __launch_bounds__(1024) group_kernel(GroupParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  int* cnt = (int*)smem;            // [E]
  int* fill = cnt + p.E;            // [E]
  int* cb = fill + p.E;             // [E] first chunk of each expert
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = p.T * p.k, C = p.chunk;
  for (int e = tid; e < p.E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int i = tid; i < N; i += blockDim.x) {
    const int e = p.idx[i];
    if (e >= 0 && e < p.E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = tid; e < p.E; e += blockDim.x) {
    p.counts[e] = cnt[e];
    fill[e] = cnt[e];
    cb[e] = C > 0 ? (cnt[e] + C - 1) / C : 0;
  }
  __syncthreads();
  const int total = block_exclusive_scan(fill, p.E, warp_tot);
  const int nrouted = block_exclusive_scan(cb, p.E, warp_tot);
  const bool chunked = p.chunks != nullptr && p.nchunks != nullptr && C > 0;   // the grouped GEMMs' list
  for (int e = tid; e < p.E; e += blockDim.x) {
    p.offsets[e] = fill[e];
    if (chunked)
      for (int c = 0; c * C < cnt[e]; ++c)
        p.chunks[cb[e] + c] = make_int4(e, fill[e] + c * C, min(C, cnt[e] - c * C), 0);
  }
  const int nshared = chunked && p.has_shared ? (p.T + C - 1) / C : 0;
  for (int c = tid; c < nshared; c += blockDim.x)
    p.chunks[nrouted + c] = make_int4(p.E, c * C, min(C, p.T - c * C), 0);
  if (tid == 0) {
    p.offsets[p.E] = total;
    if (chunked) *p.nchunks = nrouted + nshared;
  }
  __syncthreads();
  if (warp == 0) {
    for (int base = 0; base < N; base += 32) {
      const int i = base + lane;
      const bool valid = i < N;
      const int e = valid ? p.idx[i] : -1;
      const unsigned mask = __ballot_sync(0xffffffffu, valid);
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int leader = __ffs(peers) - 1;
      int basepos = 0;
      if (valid && e >= 0 && e < p.E && lane == leader) basepos = fill[e];
      basepos = __shfl_sync(0xffffffffu, basepos, leader);
      if (valid && e >= 0 && e < p.E) p.perm[basepos + rank] = i;
      __syncwarp();
      if (valid && e >= 0 && e < p.E && lane == leader) fill[e] = basepos + __popc(peers & mask);
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------------ launchers
size_t pf_max_chunks(int T, int k, int E, int chunk) {
  // sum over experts of ceil(n_e / chunk) <= min(T*k, T*k / chunk + E), plus the shared expert's
  const size_t pairs = (size_t)T * k;
  const size_t routed = pairs / chunk + (size_t)E < pairs ? pairs / chunk + (size_t)E : pairs;
  return routed + ((size_t)T + chunk - 1) / chunk;
}

cudaError_t launch_group(const GroupParams& p, cudaStream_t s) {
  const size_t sm = sizeof(int) * 3 * (size_t)p.E;
  cudaError_t e = set_func_attr((const void*)group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  GroupParams q = p;
  void* args[] = {&q};
  return cudaLaunchKernel((const void*)group_kernel, dim3(1), dim3(1024), args, sm, s);
}


int pf_chunk_tokens(int H, int I) { return (H > 4096 || I > 4096) ? 4 : 8; }

static cudaError_t pf_prepare(const void* fn, size_t bytes) {
  cudaError_t e = set_func_attr(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  return set_func_attr(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Launch configuration of a grouped kernel (gate/up or down) of a layer shape:
// row tile groups per item, tiles per warp, stages; false when the shape
// cannot run (too many groups per warp, row tiles that do not divide, or
// fewer than two stages in the shared memory of one CTA).
struct PfConfig { int rt, rw, nst; };
static bool pf_config(int H, int I, int bits, bool gu, PfConfig& cf) {
  const int K = gu ? H : I;
  const int C = pf_chunk_tokens(H, I);
  const int RT = C == 8 ? pf_row_tiles(K) : 1;
  const int ng = K / kGroup, NS = kPfWarps / RT, gpw = (ng + NS - 1) / NS;
  if (gpw > (C == 8 ? 4 : 8)) return false;
  const int rows = gu ? I / 8 : H / 16;   // 16-row tiles per expert matrix
  if (rows % RT != 0) return false;
  int optin = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (optin <= 0) optin = 227 * 1024;
  auto stages = [&](int rw) {
    const size_t fixed = pf_geom(K, bits, C, RT, rw, 0).total, stage = pf_geom(K, bits, C, RT, rw, 1).stage;
    if ((size_t)optin < fixed + 2 * stage) return 0;
    const int n = (int)(((size_t)optin - fixed) / stage);
    return n > kPfMaxStages ? kPfMaxStages : n;
  };
  // two tiles per warp where the shapes divide and two stages still fit
  const int RW = (C == 8 && rows % (2 * RT) == 0 && stages(2) >= 2) ? 2 : 1;
  const int nst = stages(RW);
  if (nst < 2) return false;
  cf.rt = RT; cf.rw = RW; cf.nst = nst;
  return true;
}

bool prefill_supported(int H, int I, int bits) {
  PfConfig a, b;
  return pf_config(H, I, bits, true, a) && pf_config(H, I, bits, false, b);
}

template <int BITS, bool GU>
static cudaError_t pf_grouped(const PrefillParams& p, cudaStream_t s) {
  const int K = GU ? p.H : p.I;
  const int C = pf_chunk_tokens(p.H, p.I);
  PfConfig cf;
  if (!pf_config(p.H, p.I, BITS, GU, cf)) return cudaErrorInvalidConfiguration;
  PrefillParams q = p;
  q.nst = cf.nst;
  q.rt = cf.rt;
  q.rw = cf.rw;
  const size_t sm = pf_geom(K, BITS, C, cf.rt, cf.rw, cf.nst).total;
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
