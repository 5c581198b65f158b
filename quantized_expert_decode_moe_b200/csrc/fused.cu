// Fused decode layer (sm_100a): the whole expert forward of one token
// (router -> top-k -> gate/up + SwiGLU -> down -> weighted combine + shared
// gate + residual -> RMSNorm) for one or more consecutive layers, in ONE
// persistent kernel with one CTA per SM.
//
// The Flash-MoE write-up ("Key technologies > Deferred GPU expert compute")
// keeps the combine, normalisation and residual on the device and hands the
// result straight to the next layer. Here every dependency of the layer is a
// grid-wide barrier inside the kernel instead of a kernel boundary:
//   B1  all router logits written        -> every CTA ranks them itself
//   B1s the shared expert's SwiGLU output written (waited on much later)
//   B2  the routed experts' SwiGLU outputs written
//   B3  every CTA's partial sum of squares of h' written -> RMSNorm
// The waits are bounded by %globaltimer (MOE_ERR_TIMEOUT on expiry). The
// grid is one CTA per SM (at most one wave), so all CTAs are resident once
// the previous kernel has left the GPU.
//
// Ownership (CTA c of n): router rows [R c/n, R (c+1)/n) of the E routed rows
// plus the shared-gate row (R = E + 1 with a shared expert); intermediate rows
// [I c/n, I (c+1)/n) (at most 8: one 16-row MMA tile per expert, gate rows
// 0-7, up rows 8-15) of every active expert; hidden rows [H c/n, H (c+1)/n)
// (at most 32: two 16-row tiles) of every active expert's down matrix and of
// h', x_out. No result is summed across CTAs.
//
// Weight streams: the shared expert's rows and the router rows do not depend
// on the routing and are requested at the start (for the layer after the
// first, during the previous layer); the routed experts' gate/up and down
// rows are requested together as soon as the CTA has ranked the logits, so
// the down rows stream while gate/up computes. Per CTA about 75 KB per
// routed expert of one layer of the 512-expert, hidden-4096 shape.
//
// Arithmetic is that of the four-kernel decode chain: codes on the integer
// tensor cores against per-group fixed-point activation digits, scale and
// bias in fp32; the router is the compensated fp32 sum with a certified
// top-k (topk.cuh).
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "stage.cuh"
#include "sync.cuh"
#include "topk.cuh"

namespace qmoe {

constexpr int kFuGuBufs = 3;      // gate/up buffers (the shared expert's is reused by a routed one)
constexpr int kFuGuRows = 8;      // intermediate rows per CTA at most
constexpr int kFuDnRows = 32;     // hidden rows per CTA at most
constexpr int kFuRouteChunks = 4; // 16-byte router chunks per lane per (row, quarter): H <= 4096
constexpr int kFuMaxRouterItems = 256;   // (row, quarter) items per CTA

struct FuLayout {
  int gRB, gSRB, gSBR, gGB;   // gate/up: code bytes per row, scale bytes per row, scale region, buffer bytes
  int dRB, dSRB, dSBR, dGB;   // down: the same
  size_t gu, dn, xs, btab, gs, part, yacc, ysh, hres, wsl, red, slots, ctx, bars, total;
};
__host__ __device__ inline FuLayout fu_layout(int H, int I, int S, int bits) {
  FuLayout L;
  L.gRB = H * bits / 8;
  L.gSRB = H / 32;
  L.gSBR = sb_region(kFuGuRows, L.gSRB);
  L.gGB = (2 * kFuGuRows * L.gRB + 4 * L.gSBR + 127) & ~127;
  L.dRB = I * bits / 8;
  L.dSRB = I / 32;
  L.dSBR = sb_region(kFuDnRows, L.dSRB);
  L.dGB = (kFuDnRows * L.dRB + 2 * L.dSBR + 127) & ~127;
  const int xsp = H / kSpan, asp = S * (I / kSpan);
  const int ngx = H / kGroup, nga = S * (I / kGroup);
  size_t o = 0;
  L.gu = o; o += (size_t)kFuGuBufs * L.gGB;
  L.dn = o; o += (size_t)S * L.dGB;
  L.xs = o; o += (size_t)H * 2;
  L.btab = o; o += sizeof(uint2) * (size_t)(xsp > asp ? xsp : asp) * kBtPerSpan;
  L.gs = o; o += sizeof(float) * 2 * (size_t)(ngx > nga ? ngx : nga);
  o = (o + 15) & ~(size_t)15;
  // partial sums of gate/up (largest), of down, the router's (row, quarter)
  // partials and the top-k scratch share one region (used one after another)
  size_t part = sizeof(float) * kFuGuBufs * kWarps * 16;
  if (part < sizeof(float) * 3 * kFuMaxRouterItems) part = sizeof(float) * 3 * kFuMaxRouterItems;
  if (part < sizeof(TopkSmem)) part = sizeof(TopkSmem);
  L.part = o; o += (part + 15) & ~(size_t)15;
  L.yacc = o; o += sizeof(float) * kFuDnRows;
  L.ysh = o; o += sizeof(float) * kFuDnRows;
  L.hres = o; o += sizeof(float) * kFuDnRows;
  L.wsl = o; o += sizeof(float) * 4 * ((kMaxSlots + 3) / 4);
  L.red = o; o += sizeof(float) * 32;
  o = (o + 15) & ~(size_t)15;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  L.ctx = o; o += 512;   // the CTA's context (FuCtx)
  o = (o + 15) & ~(size_t)15;
  L.bars = o; o += 8 * (kFuGuBufs + kMaxSlots);
  L.total = o;
  return L;
}

// Loads the table builder's elements of chunk q of a bf16 vector in shared memory.
template <int BITS>
__device__ __forceinline__ void load_chunk_bf16_smem(const uint16_t* x, int q, float (&v)[TabTraits<BITS>::kEPT]) {
  constexpr int EPT = TabTraits<BITS>::kEPT;
  const uint4* p = (const uint4*)(x + (size_t)q * EPT);
#pragma unroll
  for (int u = 0; u < EPT / 8; ++u) {
    const uint4 r = p[u];
    const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { v[8 * u + 2 * i] = bf16lo(w4[i]); v[8 * u + 2 * i + 1] = bf16hi(w4[i]); }
  }
}

// ------------------------------------------------------------------ per-CTA context
// Geometry, shared-memory regions and wait state of one CTA, built once at
// the start in shared memory; every phase function reads it from there.
struct FuCtx {
  int H, I, E, k, S, hs, n, c;
  int j0, nj, h0, nh, r0, nr, qn;
  int gpre, dpre;
  unsigned gsbw, dsbw, gu_bytes, dn_bytes;
  int ngx, nspx, nga, nspa, per_a, ntile;
  FuLayout FL;
  unsigned char* gubuf;
  unsigned char* dnbuf;
  uint16_t* xs;
  uint2* btab;
  float* gs;
  float* part;
  float* yacc;
  float* ysh;
  float* hres;
  float* wsl;
  float* red;
  moe_expert* slot_ex;
  uint64_t* gbar;
  uint64_t* dbar;
  uint32_t* status;
  unsigned long long wait_ns;
  int fail;    // a wait ran out (read and written through volatile accesses)
  int go[8];   // thread 0's decision at each arm point
};
static_assert(sizeof(FuCtx) <= 512, "the context region of the layout");
enum { kArmPrologue = 0, kArmRouted = 1, kArmNextGu = 2, kArmNextDn = 3 };

__device__ __forceinline__ bool fu_failed(FuCtx& C) { return *(volatile int*)&C.fail != 0; }
__device__ __forceinline__ void fu_note(FuCtx& C, bool ok) {
  if (!ok) *(volatile int*)&C.fail = 1;
}
// Thread 0 at an arm point: no wait has run out -> arm (and publish the decision for the issuers).
__device__ __forceinline__ bool fu_decide(FuCtx& C, int point) {
  const bool go = !fu_failed(C);
  *(volatile int*)&C.go[point] = go ? 1 : 0;
  return go;
}
__device__ __forceinline__ bool fu_go(FuCtx& C, int point) { return *(volatile int*)&C.go[point] != 0; }

static __device__ __noinline__ void fu_mwait(FuCtx& C, uint64_t* bar, unsigned par) {
  if (fu_failed(C)) return;
  fu_note(C, mbar_wait_bounded(bar, par, C.wait_ns, C.status));
}
static __device__ __noinline__ void fu_gwait(FuCtx& C, GridBar b, unsigned g) {   // thread 0
  if (fu_failed(C)) return;
  fu_note(C, grid_wait(b, g, C.wait_ns, C.status));
}

// ---------------------------------------------------------------- copies
// gate/up rows of expert ex into gate/up buffer b: cp = 0 gate code rows,
// 1 up code rows (row blocks), 2..5 gate scales, up scales, gate biases, up biases
static __device__ __noinline__ void fu_gu_copy(FuCtx& C, const moe_expert& ex, int b, int cp) {
  unsigned char* buf = C.gubuf + (size_t)b * C.FL.gGB;
  fence_proxy_async();
  if (cp < 2) {
    const moe_qmat& m = cp == 0 ? ex.gate : ex.up;
    bulk_g2s(buf + (size_t)cp * kFuGuRows * C.FL.gRB, (const char*)m.q + (size_t)C.j0 * C.FL.gRB,
             (unsigned)C.nj * C.FL.gRB, &C.gbar[b]);
  } else {
    const int w = cp - 2;
    const moe_qmat& m = (w & 1) ? ex.up : ex.gate;
    const uint16_t* src = w < 2 ? m.scales : m.biases;
    bulk_g2s(buf + 2 * kFuGuRows * C.FL.gRB + w * C.FL.gSBR,
             (const char*)src + (((size_t)C.j0 * C.FL.gSRB) & ~(size_t)15), C.gsbw, &C.gbar[b]);
  }
}
// down rows of matrix m into down buffer b: cp = 0 code rows, 1 scales, 2 biases
static __device__ __noinline__ void fu_dn_copy(FuCtx& C, const moe_qmat& m, int b, int cp) {
  unsigned char* buf = C.dnbuf + (size_t)b * C.FL.dGB;
  fence_proxy_async();
  if (cp == 0) {
    bulk_g2s(buf, (const char*)m.q + (size_t)C.h0 * C.FL.dRB, (unsigned)C.nh * C.FL.dRB, &C.dbar[b]);
  } else {
    const uint16_t* src = cp == 1 ? m.scales : m.biases;
    bulk_g2s(buf + kFuDnRows * C.FL.dRB + (cp - 1) * C.FL.dSBR,
             (const char*)src + (((size_t)C.h0 * C.FL.dSRB) & ~(size_t)15), C.dsbw, &C.dbar[b]);
  }
}
// This CTA's router rows of a layer into L2 ahead of their use (one thread).
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" :: "l"(p), "r"(bytes) : "memory");
}
static __device__ __noinline__ void fu_router_prefetch(FuCtx& C, const FuLayer& Ly) {
  const int re = C.r0 + C.nr < C.E ? C.r0 + C.nr : C.E;   // routed rows [r0, re), then the gate row
  if (re > C.r0) prefetch_l2(Ly.router_w + (size_t)C.r0 * C.H, (unsigned)(re - C.r0) * C.H * 2);
  if (C.r0 + C.nr > C.E && Ly.gate_w) prefetch_l2(Ly.gate_w, (unsigned)C.H * 2);
}

// ---------------------------------------------------------------- router
// Logits of this CTA's router rows: items (row, quarter of H), one warp
// each; exact fp32 products summed in fp64, merged per row; bound on the
// distance to the fp64 definition beside each routed logit.
static __device__ __noinline__ void fu_router(FuCtx& C, const FuLayer& Ly, double* logits, float* bound) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nri = C.nr * 4, qn = C.qn, H = C.H, E = C.E;
  const uint4* x4 = (const uint4*)C.xs;
  float* part = C.part;
  for (int it = warp; it < nri; it += kWarps) {
    const int row = C.r0 + (it >> 2), qt = it & 3;
    const uint16_t* src = (row < E ? Ly.router_w + (size_t)row * H : Ly.gate_w) + (size_t)qt * qn * 8;
    uint4 wv[kFuRouteChunks];
#pragma unroll
    for (int i = 0; i < kFuRouteChunks; ++i) {
      const int cc = lane + 32 * i;
      wv[i] = cc < qn ? ldg_stream_v4(src + (size_t)cc * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
    double acc2[2] = {0.0, 0.0};
    float sa = 0.f;
#pragma unroll
    for (int i = 0; i < kFuRouteChunks; ++i) {
      const int ch = lane + 32 * i;
      if (ch < qn) dot8_bf16_f64(wv[i], x4[qt * qn + ch], acc2, sa);
    }
    const double v = warp_sum_f64(acc2[0] + acc2[1]);
    sa = warp_sum(sa);
    if (lane == 0) { ((double*)part)[it] = v; part[2 * kFuMaxRouterItems + it] = sa; }
  }
  __syncthreads();
  if (tid < C.nr) {
    const int row = C.r0 + tid;
    double acc = 0.0;
    float sa = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc += ((const double*)part)[4 * tid + q];
      sa += part[2 * kFuMaxRouterItems + 4 * tid + q];
    }
    const double bias = (row < E && Ly.router_bias) ? (double)Ly.router_bias[row] : 0.0;
    acc += bias;
    logits[row] = acc;
    if (row < E) bound[row] = logit_bound(H, sa, acc, bias);
  }
}

// ---------------------------------------------------------------- routing
// Every CTA ranks the logits itself (certified top-k), then loads the chosen
// experts' pointers and their weights (wsl: routed in rank order, the shared
// gate last). CTA 0 reports the routing.
static __device__ __noinline__ void fu_topk(FuCtx& C, const FuLayer& Ly, const double* logits, const float* bound,
                                            unsigned* rechecks, int32_t* idx_out, float* w_out) {
  const int tid = threadIdx.x;
  TopkSmem& ts = *(TopkSmem*)C.part;
  const RouterRef rr{C.xs, Ly.router_w, Ly.router_bias, C.H};
  block_topk(logits, bound, C.E, C.k, C.hs, rr, ts);
  load_slots(ts, C.k, C.E, Ly.experts, C.slot_ex, C.status);
  if (tid < C.k) C.wsl[tid] = ts.w[tid];
  if (tid == 0) C.wsl[C.S - 1] = C.hs ? ts.sg : 0.f;
  if (C.c == 0 && tid == 0 && ts.rechecked) atomicAdd(rechecks, 1u);
  if (C.c == 0 && tid < C.k) {
    if (idx_out) idx_out[tid] = ts.idx[tid];
    if (w_out) w_out[tid] = ts.w[tid];
  }
}

// ---------------------------------------------------------------- gate/up
// B tables of x (shared memory) for the gate/up MMAs.
template <int BITS>
static __device__ __noinline__ void fu_x_tables(FuCtx& C) {
  constexpr int EPT = TabTraits<BITS>::kEPT;
  const int nq = C.H / EPT, tid = threadIdx.x;
  for (int q0 = 0; q0 < nq; q0 += kThreads) {
    const int q = q0 + tid;
    float v[EPT];
    if (q < nq) load_chunk_bf16_smem<BITS>(C.xs, q, v);
    build_tables<BITS>(v, q * EPT, q < nq, C.btab, C.gs, C.ngx);
  }
}
// MMAs of this warp's spans for the gate/up items [i0, i1) (item it in
// buffer it % 3, at most 3 items), waiting for each buffer's phase of parity
// bit b of gpar: B fragments of a span loaded once for all items; row sums of
// item it to part[(it - i0)][warp][16].
template <int BITS>
static __device__ __noinline__ void fu_gu_compute(FuCtx& C, int i0, int i1, unsigned gpar) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3, qb = lane & ~3;
  const int bl = bt_lane_index(lane);
  const LaneK K = lane_consts(tq);
  constexpr int SB = SpanBytes<BITS>::v;
  constexpr int W = QTraits<BITS>::kWordsPerThread;
  const int gRB = C.FL.gRB, gSRB = C.FL.gSRB, gSBR = C.FL.gSBR, gGB = C.FL.gGB, gpre = C.gpre, ngx = C.ngx;
  const bool al16 = gSRB % 16 == 0;
  const uint2* btab = C.btab;
  const float* gs = C.gs;
  float* part = C.part;
  const int s0 = C.nspx * warp / kWarps, s1 = C.nspx * (warp + 1) / kWarps;
  for (int sp = s0; sp < s1; sp += 2) {
    BFrag B[2];
    load_bfrag(B[0], btab + sp * kBtPerSpan, bl, gs, ngx, sp, tq);
    if (sp + 1 < s1) load_bfrag(B[1], btab + (sp + 1) * kBtPerSpan, bl, gs, ngx, sp + 1, tq);
    for (int it = i0; it < i1; ++it) {
      const int b = it % kFuGuBufs;
      if (sp == s0) fu_mwait(C, &C.gbar[b], (gpar >> b) & 1u);
      const unsigned char* buf = C.gubuf + (size_t)b * gGB;
      // 16-byte chunk of 4 spans' scale (or bias) words; a pair that starts on the last span of a
      // chunk (odd first span of the warp) takes its second span from the next chunk
      const unsigned char* sc = buf + 2 * kFuGuRows * gRB + tq * gSBR + gpre + g * gSRB;
      const uint4 sv0 = lds_chunk(sc + 16 * (sp >> 2), al16);
      const uint4 sv1 = ((sp & 3) == 3 && sp + 1 < s1) ? lds_chunk(sc + 16 * ((sp + 1) >> 2), al16) : sv0;
      float aa = 0.f, ab = 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int s = sp + q;
        if (s < s1) {
          const uint32_t w = chunk_word(q == 0 ? sv0 : sv1, s & 3);
          uint32_t wa[W], wb[W];
          const unsigned char* ra = buf + (size_t)g * gRB + s * SB + tq * W * 4;
          const unsigned char* rb = ra + (size_t)kFuGuRows * gRB;
          if constexpr (W == 4) {
            const uint4 va = *(const uint4*)ra, vb = *(const uint4*)rb;
            wa[0] = va.x; wa[1] = va.y; wa[2] = va.z; wa[3] = va.w;
            wb[0] = vb.x; wb[1] = vb.y; wb[2] = vb.z; wb[3] = vb.w;
          } else {
            const uint2 va = *(const uint2*)ra, vb = *(const uint2*)rb;
            wa[0] = va.x; wa[1] = va.y;
            wb[0] = vb.x; wb[1] = vb.y;
          }
          const uint32_t sa = __shfl_sync(0xffffffffu, w, qb), sb = __shfl_sync(0xffffffffu, w, qb + 1);
          const uint32_t ba = __shfl_sync(0xffffffffu, w, qb + 2), bb = __shfl_sync(0xffffffffu, w, qb + 3);
          tile_span<BITS>(wa, wb, sa, sb, ba, bb, B[q], K, aa, ab);
        }
      }
      aa += __shfl_xor_sync(0xffffffffu, aa, 1);
      ab += __shfl_xor_sync(0xffffffffu, ab, 1);
      aa += __shfl_xor_sync(0xffffffffu, aa, 2);
      ab += __shfl_xor_sync(0xffffffffu, ab, 2);
      float* pt = part + ((size_t)(it - i0) * kWarps + warp) * 16;
      if (tq == 0) {
        if (sp == s0) { pt[g] = aa; pt[8 + g] = ab; }
        else { pt[g] += aa; pt[8 + g] += ab; }
      }
    }
  }
  if (s0 == s1) {
    for (int it = i0; it < i1; ++it)
      if (lane < 16) part[((size_t)(it - i0) * kWarps + warp) * 16 + lane] = 0.f;
  }
}
// a = silu(g) * u of the items [i0, i1) (after a __syncthreads), item i0 + i
// -> slot slot0 + i of a [S][I] (global).
static __device__ __noinline__ void fu_gu_finalize(FuCtx& C, int i0, int i1, int slot0, float* a) {
  const int tid = threadIdx.x, nj = C.nj;
  if (tid < (i1 - i0) * nj) {
    const int i = tid / nj, r = tid - i * nj;
    const float* pt = C.part + (size_t)i * kWarps * 16;
    float gsum = 0.f, usum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) { gsum += pt[w * 16 + r]; usum += pt[w * 16 + 8 + r]; }
    a[(size_t)(slot0 + i) * C.I + C.j0 + r] = silu_f32(gsum) * usum;
  }
}

// ---------------------------------------------------------------- down
// B tables of slots [sl0, sl1) from a (global, written by every CTA).
template <int BITS>
static __device__ __noinline__ void fu_a_tables(FuCtx& C, int sl0, int sl1, const float* a) {
  constexpr int EPT = TabTraits<BITS>::kEPT;
  const int tid = threadIdx.x, I = C.I, nga = C.nga, per_a = C.per_a;
  const int qs = I / EPT, nq = (sl1 - sl0) * qs;
  for (int q0 = 0; q0 < nq; q0 += kThreads) {
    const int q = q0 + tid, sl = sl0 + q / qs, e = (q - (q / qs) * qs) * EPT;
    const bool valid = q < nq;
    float v[EPT];
    if (valid) load_chunk_f32<BITS>(a + (size_t)sl * I, e / EPT, v);
    build_tables<BITS>(v, e, valid, C.btab + (size_t)(valid ? sl : 0) * per_a,
                       C.gs + (size_t)(valid ? sl : 0) * 2 * nga, nga);
  }
}
// Spans [s0, s1) of every row tile of slot sl (down buffer sl): row sums to pt[tile][16].
template <int BITS>
static __device__ __noinline__ void fu_dn_seg(FuCtx& C, int sl, int s0, int s1, float* pt) {
  constexpr int kTiles = kFuDnRows / 16;
  const int lane = threadIdx.x & 31;
  const int dRB = C.FL.dRB, dSRB = C.FL.dSRB, dSBR = C.FL.dSBR, dpre = C.dpre, nga = C.nga, ntile = C.ntile;
  const bool al16 = dSRB % 16 == 0;
  const unsigned char* buf = C.dnbuf + (size_t)sl * C.FL.dGB;
  const int g = lane >> 2, tq = lane & 3, qb = lane & ~3;
  const int bl = bt_lane_index(lane);
  const LaneK K = lane_consts(tq);
  constexpr int SB = SpanBytes<BITS>::v;
  constexpr int W = QTraits<BITS>::kWordsPerThread;
  const uint2* bt = C.btab + (size_t)sl * C.per_a;
  const float* gsl = C.gs + (size_t)sl * 2 * nga;
  float aa[kTiles], ab[kTiles];
  uint4 sv[kTiles];
#pragma unroll
  for (int tl = 0; tl < kTiles; ++tl) { aa[tl] = 0.f; ab[tl] = 0.f; sv[tl] = make_uint4(0u, 0u, 0u, 0u); }
  for (int s = s0; s < s1; ++s) {
    BFrag B;
    load_bfrag(B, bt + s * kBtPerSpan, bl, gsl, nga, s, tq);
#pragma unroll
    for (int tl = 0; tl < kTiles; ++tl) {
      if (tl < ntile) {
        const int r = tl * 16 + g;
        if (s == s0 || (s & 3) == 0)
          sv[tl] = lds_chunk(buf + kFuDnRows * dRB + dpre + (tq >> 1) * dSBR + (r + 8 * (tq & 1)) * dSRB +
                                 16 * (s >> 2), al16);
        const uint32_t w = chunk_word(sv[tl], s & 3);
        uint32_t wa[W], wb[W];
        const unsigned char* ra = buf + (size_t)r * dRB + s * SB + tq * W * 4;
        const unsigned char* rb = ra + (size_t)8 * dRB;
        if constexpr (W == 4) {
          const uint4 va = *(const uint4*)ra, vb = *(const uint4*)rb;
          wa[0] = va.x; wa[1] = va.y; wa[2] = va.z; wa[3] = va.w;
          wb[0] = vb.x; wb[1] = vb.y; wb[2] = vb.z; wb[3] = vb.w;
        } else {
          const uint2 va = *(const uint2*)ra, vb = *(const uint2*)rb;
          wa[0] = va.x; wa[1] = va.y;
          wb[0] = vb.x; wb[1] = vb.y;
        }
        const uint32_t sa = __shfl_sync(0xffffffffu, w, qb), sb = __shfl_sync(0xffffffffu, w, qb + 1);
        const uint32_t ba = __shfl_sync(0xffffffffu, w, qb + 2), bb = __shfl_sync(0xffffffffu, w, qb + 3);
        tile_span<BITS>(wa, wb, sa, sb, ba, bb, B, K, aa[tl], ab[tl]);
      }
    }
  }
#pragma unroll
  for (int tl = 0; tl < kTiles; ++tl) {
    if (tl < ntile) {
      float a = aa[tl], b = ab[tl];
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      b += __shfl_xor_sync(0xffffffffu, b, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      b += __shfl_xor_sync(0xffffffffu, b, 2);
      if (tq == 0) { pt[tl * 16 + g] = a; pt[tl * 16 + 8 + g] = b; }
    }
  }
}
// Down of slots [sl0, sl1): segments (slot, span part) over the warps, each
// waiting for its slot's buffer phase (parity bit sl of dpar); then per
// owned row, in slot order: shared (accumulate = false) ysh = sg * y, routed
// (accumulate = true) yacc += w_slot * y.
template <int BITS>
static __device__ __noinline__ void fu_dn_run(FuCtx& C, int sl0, int sl1, unsigned dpar, bool accumulate) {
  constexpr int kTiles = kFuDnRows / 16;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int ni = sl1 - sl0, nspa = C.nspa;
  int nsplit = kWarps / ni;
  nsplit = nsplit < 1 ? 1 : (nsplit > nspa ? nspa : nsplit);
  const int nseg = ni * nsplit;
  int waited = -1;
  for (int sg = warp; sg < nseg; sg += kWarps) {
    const int itr = sg / nsplit, pr = sg - itr * nsplit;
    const int sl = sl0 + itr;
    if (sl != waited) {
      fu_mwait(C, &C.dbar[sl], (dpar >> sl) & 1u);
      waited = sl;
    }
    fu_dn_seg<BITS>(C, sl, nspa * pr / nsplit, nspa * (pr + 1) / nsplit, C.part + (size_t)sg * kTiles * 16);
  }
  __syncthreads();
  if (tid < C.nh) {
    const int tl = tid >> 4, rr = tid & 15;
    float acc = accumulate ? C.yacc[tid] : 0.f;
    for (int itr = 0; itr < ni; ++itr) {
      const float* pt = C.part + (size_t)itr * nsplit * kTiles * 16 + tl * 16 + rr;
      float y = 0.f;
      for (int pr = 0; pr < nsplit; ++pr) y += pt[pr * kTiles * 16];
      acc = fmaf(C.wsl[sl0 + itr], y, acc);
    }
    if (accumulate) C.yacc[tid] = acc;
    else C.ysh[tid] = acc;
  }
  __syncthreads();
}

// ---------------------------------------------------------------- the kernel
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) fused_decode_kernel(const __grid_constant__ FusedParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  FuCtx& C = *(FuCtx*)(smem + fu_layout(p.H, p.I, p.S, BITS).ctx);
  if (tid == 0) {
    const FuLayout FL = fu_layout(p.H, p.I, p.S, BITS);
    const int H = p.H, I = p.I, E = p.E, n = p.nCTA, c = blockIdx.x;
    C.H = H; C.I = I; C.E = E; C.k = p.k; C.S = p.S; C.hs = p.has_shared; C.n = n; C.c = c;
    C.j0 = (int)((long long)I * c / n); C.nj = (int)((long long)I * (c + 1) / n) - C.j0;
    C.h0 = (int)((long long)H * c / n); C.nh = (int)((long long)H * (c + 1) / n) - C.h0;
    const int R = E + p.has_shared;
    C.r0 = (int)((long long)R * c / n); C.nr = (int)((long long)R * (c + 1) / n) - C.r0;
    C.qn = H / 32;
    C.gsbw = sb_window(C.j0, C.nj, FL.gSRB, C.gpre);
    C.dsbw = sb_window(C.h0, C.nh, FL.dSRB, C.dpre);
    C.gu_bytes = 2u * C.nj * FL.gRB + 4u * C.gsbw;
    C.dn_bytes = (unsigned)C.nh * FL.dRB + 2u * C.dsbw;
    C.ngx = H / kGroup; C.nspx = H / kSpan;
    C.nga = I / kGroup; C.nspa = I / kSpan; C.per_a = C.nspa * kBtPerSpan;
    C.ntile = (C.nh + 15) / 16;
    C.FL = FL;
    C.gubuf = smem + FL.gu; C.dnbuf = smem + FL.dn; C.xs = (uint16_t*)(smem + FL.xs);
    C.btab = (uint2*)(smem + FL.btab); C.gs = (float*)(smem + FL.gs); C.part = (float*)(smem + FL.part);
    C.yacc = (float*)(smem + FL.yacc); C.ysh = (float*)(smem + FL.ysh); C.hres = (float*)(smem + FL.hres);
    C.wsl = (float*)(smem + FL.wsl); C.red = (float*)(smem + FL.red); C.slot_ex = (moe_expert*)(smem + FL.slots);
    C.gbar = (uint64_t*)(smem + FL.bars); C.dbar = C.gbar + kFuGuBufs;
    C.status = p.status; C.wait_ns = p.wait_ns;
    C.fail = 0;
    for (int i = 0; i < 8; ++i) C.go[i] = 0;
    for (int b = 0; b < kFuGuBufs + p.S; ++b) mbar_init(&C.gbar[b], 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int S = C.S, k = C.k, hs = C.hs, n = C.n, H = C.H, nh = C.nh, h0 = C.h0;
  unsigned* hdr = p.hdr;
  const GridBar B1{hdr + 16, hdr + 32}, B1s{hdr + 17, hdr + 40}, B2{hdr + 18, hdr + 48}, B3{hdr + 19, hdr + 56};
  // parity of the latest phase armed on each buffer barrier, and whether copies went out for it (bit b =
  // buffer b). Arming and issuing go together: thread 0 decides (no wait has run out), arms and publishes
  // the decision before a __syncthreads; after it every thread records the new phases and the issuing
  // lanes start the copies. A barrier is armed again only after its previous phase completed (thread 0
  // waited on it, or a __syncthreads separates the arming from every other warp's wait).
  unsigned gpar = 0, dpar = 0, gissued = 0, dissued = 0;
  auto note_gu = [&](int b) { gpar ^= (gissued >> b) & 1u ? (1u << b) : 0u; gissued |= 1u << b; };
  auto note_dn = [&](int b) { dpar ^= (dissued >> b) & 1u ? (1u << b) : 0u; dissued |= 1u << b; };

  // ---------------------------------------------------------------- prologue (layer 0)
  // The weights of layer 0 do not depend on the previous kernel: the shared
  // expert's copies and the router rows' L2 prefetch go out before the
  // dependency wait. x, h and the workspace are touched only after it.
  if (tid == 0 && fu_decide(C, kArmPrologue) && hs) {
    mbar_expect_tx(&C.gbar[0], C.gu_bytes);
    mbar_expect_tx(&C.dbar[S - 1], C.dn_bytes);
  }
  if (tid == 32) fu_router_prefetch(C, p.layer[0]);
  __syncthreads();
  if (fu_go(C, kArmPrologue) && hs) {
    note_gu(0);
    note_dn(S - 1);
    if (lane == 0 && warp < 6) fu_gu_copy(C, p.layer[0].shared, 0, warp);
    if (lane == 0 && warp >= 6 && warp < 9) fu_dn_copy(C, p.layer[0].shared.down, S - 1, warp - 6);
  }
  griddep_wait();
  for (int i = tid; i < H / 8; i += kThreads) ((uint4*)C.xs)[i] = __ldcg((const uint4*)p.x_in + i);
  if (tid < nh) C.hres[tid] = __ldcg(p.h + h0 + tid);
  __syncthreads();

  for (int l = 0; l < p.L; ++l) {
    const FuLayer& Ly = p.layer[l];
    const bool last = l + 1 == p.L;
    // ------------------------------------------------ (A) x tables + router logits
    fu_x_tables<BITS>(C);
    fu_router(C, Ly, p.logits, p.bound);
    if (p.x_rec)
      for (int r = tid; r < nh; r += kThreads) p.x_rec[(size_t)l * H + h0 + r] = C.xs[h0 + r];
    if (p.h_rec)
      for (int r = tid; r < nh; r += kThreads) p.h_rec[(size_t)l * H + h0 + r] = C.hres[r];
    __syncthreads();   // logits written; B tables of x complete
    unsigned g1 = 0, g1s = 0, g2 = 0, g3 = 0;
    if (tid == 0) g1 = grid_arrive(B1, n);
    // ------------------------------------------------ (B) shared gate/up
    if (hs) {
      fu_gu_compute<BITS>(C, 0, 1, gpar);
      fence_proxy_async();
      __syncthreads();
      fu_gu_finalize(C, 0, 1, S - 1, p.a);
      __syncthreads();
      if (tid == 0) g1s = grid_arrive(B1s, n);
    }
    // ------------------------------------------------ (C) routing
    if (tid == 0) fu_gwait(C, B1, g1);
    __syncthreads();
    // every CTA of this kernel is resident (all arrived at B1): a dependent
    // launch may now take the SMs these CTAs leave
    if (l == 0) griddep_launch_dependents();
    fu_topk(C, Ly, p.logits, p.bound, hdr + 4, p.idx_out ? p.idx_out + (size_t)l * k : nullptr,
            p.w_out ? p.w_out + (size_t)l * k : nullptr);
    if (tid == 0 && fu_decide(C, kArmRouted)) {
      for (int r = 0; r < k; ++r) {
        mbar_expect_tx(&C.gbar[(r + hs) % kFuGuBufs], C.gu_bytes);
        mbar_expect_tx(&C.dbar[r], C.dn_bytes);
      }
    }
    __syncthreads();   // slots visible; shared gate/up buffer consumed; barriers armed
    if (fu_go(C, kArmRouted)) {
      for (int r = 0; r < k; ++r) {
        note_gu((r + hs) % kFuGuBufs);
        note_dn(r);
      }
      if (lane == 0) {
        const int ncp = 9 * k;   // 6 gate/up copies per expert, then 3 down copies per expert
        for (int cp = warp; cp < ncp; cp += kWarps) {
          if (cp < 6 * k) fu_gu_copy(C, C.slot_ex[cp / 6], (cp / 6 + hs) % kFuGuBufs, cp % 6);
          else fu_dn_copy(C, C.slot_ex[(cp - 6 * k) / 3].down, (cp - 6 * k) / 3, (cp - 6 * k) % 3);
        }
      }
    }
    // ------------------------------------------------ (D) routed gate/up
    fu_gu_compute<BITS>(C, hs, hs + k, gpar);
    fence_proxy_async();
    __syncthreads();   // every wait on a gate/up buffer is over: buffer 0 may be armed again
    const bool pre_gu = !last && hs;   // the next layer's shared gate/up rows into buffer 0
    if (tid == 0 && fu_decide(C, kArmNextGu) && pre_gu) mbar_expect_tx(&C.gbar[0], C.gu_bytes);
    fu_gu_finalize(C, hs, hs + k, 0, p.a);
    __syncthreads();
    if (tid == 0) g2 = grid_arrive(B2, n);
    if (fu_go(C, kArmNextGu) && pre_gu) {
      note_gu(0);
      if (lane == 0 && warp < 6) fu_gu_copy(C, p.layer[l + 1].shared, 0, warp);
    }
    // ------------------------------------------------ (E) shared down
    if (hs) {
      if (tid == 0) fu_gwait(C, B1s, g1s);
      __syncthreads();
      fu_a_tables<BITS>(C, S - 1, S, p.a);
      __syncthreads();
      fu_dn_run<BITS>(C, S - 1, S, dpar, false);
      fence_proxy_async();
      if (tid == 0 && fu_decide(C, kArmNextDn) && !last) mbar_expect_tx(&C.dbar[S - 1], C.dn_bytes);
      __syncthreads();
      if (fu_go(C, kArmNextDn) && !last) {   // the next layer's shared down rows
        note_dn(S - 1);
        if (lane == 0 && warp >= 6 && warp < 9) fu_dn_copy(C, p.layer[l + 1].shared.down, S - 1, warp - 6);
      }
    }
    if (!last && tid == 32) fu_router_prefetch(C, p.layer[l + 1]);   // the next layer's router rows into L2
    // ------------------------------------------------ (F) routed down + combine
    if (tid == 0) fu_gwait(C, B2, g2);
    __syncthreads();
    fu_a_tables<BITS>(C, 0, k, p.a);
    if (tid < nh) C.yacc[tid] = C.hres[tid];
    __syncthreads();
    fu_dn_run<BITS>(C, 0, k, dpar, true);
    fence_proxy_async();   // the down buffers are refilled by the next layer's copies
    float ss = 0.f;
    if (tid < nh) {
      const float v = hs ? C.yacc[tid] + C.ysh[tid] : C.yacc[tid];
      C.yacc[tid] = v;
      p.hacc[h0 + tid] = v;
      ss = v * v;
    }
    ss = warp_sum(ss);
    if (lane == 0) C.red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kWarps; ++w) t += C.red[w];
      p.gpart[C.c] = t;
      g3 = grid_arrive(B3, n);
    }
    // ------------------------------------------------ (G) RMSNorm
    if (tid == 0) fu_gwait(C, B3, g3);
    __syncthreads();
    if (warp == 0) {   // the CTAs' partials summed in a fixed order (the same in every CTA)
      float t = 0.f;
      for (int q = lane; q < n; q += 32) t += __ldcg(p.gpart + q);
      t = warp_sum(t);
      if (lane == 0) C.red[0] = t;
    }
    __syncthreads();
    const float inv = 1.f / sqrtf(C.red[0] / (float)H + Ly.eps);
    if (last) {
      if (tid < nh) {
        const int j = h0 + tid;
        const float v = C.yacc[tid];
        const float xo = v * inv * bf16_to_f32(Ly.gamma[j]);
        p.h[j] = v;
        p.x_out[j] = f32_to_bf16(xo);
        if (p.x_out_f32) p.x_out_f32[j] = xo;
      }
    } else {
      // every CTA forms the whole next input from h' for its router and tables
      for (int i = tid; i < H / 2; i += kThreads) {
        const float2 v = __ldcg((const float2*)p.hacc + i);
        const uint32_t gw = ((const uint32_t*)Ly.gamma)[i];
        ((uint32_t*)C.xs)[i] = (uint32_t)f32_to_bf16(v.x * inv * bf16lo(gw)) |
                               ((uint32_t)f32_to_bf16(v.y * inv * bf16hi(gw)) << 16);
      }
      if (tid < nh) C.hres[tid] = C.yacc[tid];
      __syncthreads();
    }
  }
  // no bulk copy may still be writing into shared memory when the CTA exits
  __syncthreads();
  if (tid == 0) {
    for (int b = 0; b < kFuGuBufs; ++b)
      if ((gissued >> b) & 1u) mbar_wait_bounded(&C.gbar[b], (gpar >> b) & 1u, p.wait_ns, nullptr);
    for (int b = 0; b < S; ++b)
      if ((dissued >> b) & 1u) mbar_wait_bounded(&C.dbar[b], (dpar >> b) & 1u, p.wait_ns, nullptr);
  }
}

// ------------------------------------------------------------------ diagnostics
// One thread arrives at the first grid barrier of the workspace header as if
// the grid had two CTAs, so the round never completes: its bounded wait runs
// out, latches MOE_ERR_TIMEOUT and the kernel returns. The arrival counter is
// left at 1, as a real timeout can leave it; moe_poll_status clears it.
__global__ void __launch_bounds__(32) selftest_grid_kernel(unsigned* hdr, uint32_t* status,
                                                           unsigned long long bound_ns) {
  if (threadIdx.x == 0) {
    const GridBar b{hdr + 16, hdr + 32};
    const unsigned g = grid_arrive(b, 2u);
    grid_wait(b, g, bound_ns, status);
  }
}

cudaError_t launch_selftest_grid(unsigned* hdr, unsigned long long bound_ns, cudaStream_t s) {
  selftest_grid_kernel<<<1, 32, 0, s>>>(hdr, hdr, bound_ns);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ launcher
size_t fused_smem_bytes(int H, int I, int S, int bits) { return fu_layout(H, I, S, bits).total; }

static int fu_optin_smem() {
  static int v = 0;
  if (!v) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (v <= 0) v = 227 * 1024;
  }
  return v;
}

int fused_ctas(int H, int I) {
  int n = num_sms();
  if (n > I) n = I;
  if (n > H) n = H;
  return n;
}

bool fused_supported(int H, int I, int E, int k, int has_shared, int bits) {
  const int S = k + (has_shared ? 1 : 0);
  if (k > kFuGuBufs || S > kMaxSlots || H > 32 * kFuRouteChunks * 32 || H % kSpan || I % kSpan) return false;
  const int n = fused_ctas(H, I);
  if (n < 1 || (I + n - 1) / n > kFuGuRows || (H + n - 1) / n > kFuDnRows) return false;
  if (4 * ((E + has_shared + n - 1) / n) > kFuMaxRouterItems) return false;
  if (E > kTopkPer * kThreads) return false;
  return fused_smem_bytes(H, I, S, bits) <= (size_t)fu_optin_smem();
}

cudaError_t launch_fused(const FusedParams& p, int bits, cudaStream_t s) {
  const size_t sm = fused_smem_bytes(p.H, p.I, p.S, bits);
  if (sm > (size_t)fu_optin_smem()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)fused_decode_kernel<4> : (const void*)fused_decode_kernel<2>;
  cudaError_t e = set_func_attr(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  if ((e = set_func_attr(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess) return e;
  // the grid-wide barriers need every CTA resident at once: at most one wave
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, sm)) != cudaSuccess) return e;
  if (per_sm < 1 || p.nCTA > per_sm * num_sms()) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nCTA);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = s;
  // Programmatic dependent launch: the launch and the weight prologue overlap
  // the previous kernel's tail; x, h and the workspace are read after
  // griddepcontrol.wait, i.e. after the previous kernel has completed. This
  // kernel lets its own dependents launch only once all of its CTAs are
  // resident (after the first grid barrier), so a dependent CTA never holds
  // an SM that one of this kernel's CTAs still needs.
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  FusedParams q = p;
  void* args[] = {&q};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace qmoe
