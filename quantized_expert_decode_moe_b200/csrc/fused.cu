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
// launch is cooperative, so all CTAs are resident.
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
  size_t gu, dn, xs, btab, gs, part, yacc, ysh, hres, wsl, red, slots, flags, bars, total;
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
  L.flags = o; o += 32;
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

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) fused_decode_kernel(const __grid_constant__ FusedParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = p.H, I = p.I, E = p.E, k = p.k, S = p.S, hs = p.has_shared, n = p.nCTA;
  const FuLayout FL = fu_layout(H, I, S, BITS);
  unsigned char* gubuf = smem + FL.gu;
  unsigned char* dnbuf = smem + FL.dn;
  uint16_t* xs = (uint16_t*)(smem + FL.xs);
  uint2* btab = (uint2*)(smem + FL.btab);
  float* gs = (float*)(smem + FL.gs);
  float* part = (float*)(smem + FL.part);
  TopkSmem& ts = *(TopkSmem*)(smem + FL.part);
  float* yacc = (float*)(smem + FL.yacc);
  float* ysh = (float*)(smem + FL.ysh);
  float* hres = (float*)(smem + FL.hres);
  float* wsl = (float*)(smem + FL.wsl);
  float* red = (float*)(smem + FL.red);
  moe_expert* slot_ex = (moe_expert*)(smem + FL.slots);
  // flags[0]: a wait ran out; flags[point]: thread 0's decision at arm point `point` (one slot per
  // point, so a slot is rewritten only a layer later, long after every thread has read it)
  volatile int* flags = (volatile int*)(smem + FL.flags);
  uint64_t* gbar = (uint64_t*)(smem + FL.bars);
  uint64_t* dbar = gbar + kFuGuBufs;

  const int c = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j0 = (int)((long long)I * c / n), nj = (int)((long long)I * (c + 1) / n) - j0;
  const int h0 = (int)((long long)H * c / n), nh = (int)((long long)H * (c + 1) / n) - h0;
  const int R = E + hs, r0 = (int)((long long)R * c / n), nr = (int)((long long)R * (c + 1) / n) - r0;
  int gpre, dpre;
  const unsigned gsbw = sb_window(j0, nj, FL.gSRB, gpre);
  const unsigned dsbw = sb_window(h0, nh, FL.dSRB, dpre);
  const unsigned gu_bytes = 2u * nj * FL.gRB + 4u * gsbw;
  const unsigned dn_bytes = (unsigned)nh * FL.dRB + 2u * dsbw;
  const int ngx = H / kGroup, nspx = H / kSpan;
  const int nga = I / kGroup, nspa = I / kSpan, per_a = nspa * kBtPerSpan;
  const int ntile = (nh + 15) / 16;
  unsigned* hdr = p.hdr;
  const GridBar B1{hdr + 16, hdr + 32}, B1s{hdr + 17, hdr + 40}, B2{hdr + 18, hdr + 48}, B3{hdr + 19, hdr + 56};
  // parity of the latest phase armed on each buffer barrier, and whether copies went out for it
  unsigned gpar = 0, dpar = 0, gissued = 0, dissued = 0;   // bit b = buffer b

  auto failed = [&]() { return flags[0] != 0; };
  auto note = [&](bool ok) { if (!ok) flags[0] = 1; };
  auto mwait = [&](uint64_t* bar, unsigned par) {
    if (failed()) return;
    note(mbar_wait_bounded(bar, par, p.wait_ns, p.status));
  };
  auto gwait = [&](GridBar b, unsigned g) {   // thread 0
    if (failed()) return;
    note(grid_wait(b, g, p.wait_ns, p.status));
  };

  if (tid == 0) {
    for (int b = 0; b < kFuGuBufs + S; ++b) mbar_init(&gbar[b], 1);
    fence_mbar_init();
    for (int i = 0; i < 8; ++i) flags[i] = 0;
  }
  __syncthreads();

  // ---------------------------------------------------------------- copies
  // gate/up rows of expert ex into gate/up buffer b: c = 0 gate code rows,
  // 1 up code rows (row blocks), 2..5 gate scales, up scales, gate biases, up biases
  auto gu_copy = [&](const moe_expert& ex, int b, int cp) {
    unsigned char* buf = gubuf + (size_t)b * FL.gGB;
    fence_proxy_async();
    if (cp < 2) {
      const moe_qmat& m = cp == 0 ? ex.gate : ex.up;
      bulk_g2s(buf + (size_t)cp * kFuGuRows * FL.gRB, (const char*)m.q + (size_t)j0 * FL.gRB, (unsigned)nj * FL.gRB,
               &gbar[b]);
    } else {
      const int w = cp - 2;
      const moe_qmat& m = (w & 1) ? ex.up : ex.gate;
      const uint16_t* src = w < 2 ? m.scales : m.biases;
      bulk_g2s(buf + 2 * kFuGuRows * FL.gRB + w * FL.gSBR, (const char*)src + (((size_t)j0 * FL.gSRB) & ~(size_t)15),
               gsbw, &gbar[b]);
    }
  };
  // down rows of matrix m into down buffer b: c = 0 code rows, 1 scales, 2 biases
  auto dn_copy = [&](const moe_qmat& m, int b, int cp) {
    unsigned char* buf = dnbuf + (size_t)b * FL.dGB;
    fence_proxy_async();
    if (cp == 0) {
      bulk_g2s(buf, (const char*)m.q + (size_t)h0 * FL.dRB, (unsigned)nh * FL.dRB, &dbar[b]);
    } else {
      const uint16_t* src = cp == 1 ? m.scales : m.biases;
      bulk_g2s(buf + kFuDnRows * FL.dRB + (cp - 1) * FL.dSBR, (const char*)src + (((size_t)h0 * FL.dSRB) & ~(size_t)15),
               dsbw, &dbar[b]);
    }
  };
  // Arming and issuing go together. Thread 0 decides (no wait has run out),
  // publishes the decision in the point's flag and arms the barriers before a
  // __syncthreads; after it every thread reads the decision, records the new
  // phases (so all threads agree on the parity to wait for) and the issuing
  // lanes start the copies. After a failed wait nothing is armed or issued,
  // so no barrier phase waits for copies that never went out. A barrier is
  // armed again only after its previous phase completed (thread 0 waited on
  // it, or a __syncthreads separates the arming from every other warp's wait).
  enum { kArmPrologue = 1, kArmRouted = 2, kArmNextGu = 3, kArmNextDn = 4 };
  auto decide = [&](int point) {   // thread 0
    const bool go = !failed();
    flags[point] = go ? 1 : 0;
    return go;
  };
  auto note_gu = [&](int b) {   // every thread: a new phase armed on gate/up buffer b
    gpar ^= (gissued >> b) & 1u ? (1u << b) : 0u;
    gissued |= 1u << b;
  };
  auto note_dn = [&](int b) {
    dpar ^= (dissued >> b) & 1u ? (1u << b) : 0u;
    dissued |= 1u << b;
  };

  // ---------------------------------------------------------------- router
  // items (row, quarter) of this CTA's router rows; the first item of each
  // warp can be loaded ahead into registers (rw)
  const int nri = nr * 4;
  const int qn = H / 32;   // 16-byte chunks per quarter row
  uint4 rw[kFuRouteChunks];
  auto router_src = [&](const FuLayer& Ly, int it) {
    const int row = r0 + (it >> 2), qt = it & 3;
    const uint16_t* wrow = row < E ? Ly.router_w + (size_t)row * H : Ly.gate_w;
    return wrow + (size_t)qt * qn * 8;
  };
  auto router_load = [&](const FuLayer& Ly, int it, uint4 (&wv)[kFuRouteChunks]) {
    const uint16_t* src = router_src(Ly, it);
#pragma unroll
    for (int i = 0; i < kFuRouteChunks; ++i) {
      const int cc = lane + 32 * i;
      wv[i] = cc < qn ? ldg_stream_v4(src + (size_t)cc * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto router_run = [&](const FuLayer& Ly) {
    const uint4* x4 = (const uint4*)xs;
    for (int it = warp; it < nri; it += kWarps) {
      uint4 wv[kFuRouteChunks];
      if (it == warp) {
#pragma unroll
        for (int i = 0; i < kFuRouteChunks; ++i) wv[i] = rw[i];
      } else {
        router_load(Ly, it, wv);
      }
      const int qt = it & 3;
      float cs[4] = {0.f, 0.f, 0.f, 0.f}, cc[4] = {0.f, 0.f, 0.f, 0.f}, sa = 0.f;
#pragma unroll
      for (int i = 0; i < kFuRouteChunks; ++i) {
        const int ch = lane + 32 * i;
        if (ch < qn) dot8_bf16_comp(wv[i], x4[qt * qn + ch], cs, cc, sa);
      }
      float as_ = cs[0], ac_ = cc[0] + cc[1] + cc[2] + cc[3];
      two_sum_acc(as_, ac_, cs[1]);
      two_sum_acc(as_, ac_, cs[2]);
      two_sum_acc(as_, ac_, cs[3]);
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, as_, o), oc = __shfl_xor_sync(0xffffffffu, ac_, o);
        ac_ += oc;
        two_sum_acc(as_, ac_, os);
      }
      sa = warp_sum(sa);
      if (lane == 0) { part[3 * it] = as_; part[3 * it + 1] = ac_; part[3 * it + 2] = sa; }
    }
    __syncthreads();
    if (tid < nr) {
      const int row = r0 + tid;
      float as_ = part[12 * tid], ac_ = part[12 * tid + 1], sa = part[12 * tid + 2];
#pragma unroll
      for (int q = 1; q < 4; ++q) {
        ac_ += part[12 * tid + 3 * q + 1];
        two_sum_acc(as_, ac_, part[12 * tid + 3 * q]);
        sa += part[12 * tid + 3 * q + 2];
      }
      double acc = (double)as_ + (double)ac_;
      const double bias = (row < E && Ly.router_bias) ? (double)Ly.router_bias[row] : 0.0;
      acc += bias;
      p.logits[row] = acc;
      if (row < E) p.bound[row] = logit_bound(H, sa, acc, bias);
    }
  };

  // ---------------------------------------------------------------- gate/up
  // B tables of x (xs) for the gate/up MMAs
  auto x_tables = [&]() {
    constexpr int EPT = TabTraits<BITS>::kEPT;
    const int nq = H / EPT;
    for (int q0 = 0; q0 < nq; q0 += kThreads) {
      const int q = q0 + tid;
      float v[EPT];
      if (q < nq) load_chunk_bf16_smem<BITS>(xs, q, v);
      build_tables<BITS>(v, q * EPT, q < nq, btab, gs, ngx);
    }
  };
  // MMAs of this warp's spans for the gate/up items [i0, i1) (item it in
  // buffer it % 3, at most 3 items): B fragments of a span loaded once for
  // all items; row sums of item it to part[(it - i0)][warp][16].
  const bool gal16 = FL.gSRB % 16 == 0;
  auto gu_compute = [&](int i0, int i1) {
    const int g = lane >> 2, tq = lane & 3, qb = lane & ~3;
    const int bl = bt_lane_index(lane);
    const LaneK K = lane_consts(tq);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int W = QTraits<BITS>::kWordsPerThread;
    const int s0 = nspx * warp / kWarps, s1 = nspx * (warp + 1) / kWarps;
    for (int sp = s0; sp < s1; sp += 2) {
      BFrag B[2];
      load_bfrag(B[0], btab + sp * kBtPerSpan, bl, gs, ngx, sp, tq);
      if (sp + 1 < s1) load_bfrag(B[1], btab + (sp + 1) * kBtPerSpan, bl, gs, ngx, sp + 1, tq);
      for (int it = i0; it < i1; ++it) {
        const int b = it % kFuGuBufs;
        if (sp == s0) mwait(&gbar[b], (gpar >> b) & 1u);
        const unsigned char* buf = gubuf + (size_t)b * FL.gGB;
        const uint4 sv = lds_chunk(buf + 2 * kFuGuRows * FL.gRB + tq * FL.gSBR + gpre + g * FL.gSRB + 16 * (sp >> 2), gal16);
        float aa = 0.f, ab = 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int s = sp + q;
          if (s < s1) {
            const uint32_t w = chunk_word(sv, s & 3);
            uint32_t wa[W], wb[W];
            const unsigned char* ra = buf + (size_t)g * FL.gRB + s * SB + tq * W * 4;
            const unsigned char* rb = ra + (size_t)kFuGuRows * FL.gRB;
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
  };
  // a = silu(g) * u of items [i0, i1) (after a __syncthreads); item it -> slot slot_of(it)
  auto gu_finalize = [&](int i0, int i1, auto slot_of) {
    if (tid < (i1 - i0) * nj) {
      const int i = tid / nj, r = tid - i * nj;
      const float* pt = part + (size_t)i * kWarps * 16;
      float gsum = 0.f, usum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) { gsum += pt[w * 16 + r]; usum += pt[w * 16 + 8 + r]; }
      p.a[(size_t)slot_of(i0 + i) * I + j0 + r] = silu_f32(gsum) * usum;
    }
  };

  // ---------------------------------------------------------------- down
  // B tables of slots [sl0, sl1) from a (global, written by every CTA)
  auto a_tables = [&](int sl0, int sl1) {
    constexpr int EPT = TabTraits<BITS>::kEPT;
    const int qs = I / EPT, nq = (sl1 - sl0) * qs;
    for (int q0 = 0; q0 < nq; q0 += kThreads) {
      const int q = q0 + tid, sl = sl0 + q / qs, e = (q - (q / qs) * qs) * EPT;
      const bool valid = q < nq;
      float v[EPT];
      if (valid) load_chunk_f32<BITS>(p.a + (size_t)sl * I, e / EPT, v);
      build_tables<BITS>(v, e, valid, btab + (size_t)(valid ? sl : 0) * per_a, gs + (size_t)(valid ? sl : 0) * 2 * nga,
                         nga);
    }
  };
  constexpr int kTiles = kFuDnRows / 16;
  const bool dal16 = FL.dSRB % 16 == 0;
  // spans [s0, s1) of every row tile of slot sl (buffer sl): row sums to pt[tile][16]
  auto dn_seg = [&](int sl, int s0, int s1, float* pt) {
    const unsigned char* buf = dnbuf + (size_t)sl * FL.dGB;
    const int g = lane >> 2, tq = lane & 3, qb = lane & ~3;
    const int bl = bt_lane_index(lane);
    const LaneK K = lane_consts(tq);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int W = QTraits<BITS>::kWordsPerThread;
    const uint2* bt = btab + (size_t)sl * per_a;
    const float* gsl = gs + (size_t)sl * 2 * nga;
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
            sv[tl] = lds_chunk(buf + kFuDnRows * FL.dRB + dpre + (tq >> 1) * FL.dSBR + (r + 8 * (tq & 1)) * FL.dSRB +
                                   16 * (s >> 2), dal16);
          const uint32_t w = chunk_word(sv[tl], s & 3);
          uint32_t wa[W], wb[W];
          const unsigned char* ra = buf + (size_t)r * FL.dRB + s * SB + tq * W * 4;
          const unsigned char* rb = ra + (size_t)8 * FL.dRB;
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
  };
  // slots [sl0, sl1): segments (slot, span part) over the warps; then, per
  // owned row and in slot order, out(row, slot, y)
  auto dn_run = [&](int sl0, int sl1, auto out) {
    const int ni = sl1 - sl0;
    int nsplit = kWarps / ni;
    nsplit = nsplit < 1 ? 1 : (nsplit > nspa ? nspa : nsplit);
    const int nseg = ni * nsplit;
    int waited = -1;
    for (int sg = warp; sg < nseg; sg += kWarps) {
      const int itr = sg / nsplit, pr = sg - itr * nsplit;
      const int sl = sl0 + itr;
      if (sl != waited) {
        mwait(&dbar[sl], (dpar >> sl) & 1u);
        waited = sl;
      }
      dn_seg(sl, nspa * pr / nsplit, nspa * (pr + 1) / nsplit, part + (size_t)sg * kTiles * 16);
    }
    __syncthreads();
    if (tid < nh) {
      const int tl = tid >> 4, rr = tid & 15;
      for (int itr = 0; itr < ni; ++itr) {
        const float* pt = part + (size_t)itr * nsplit * kTiles * 16 + tl * 16 + rr;
        float y = 0.f;
        for (int pr = 0; pr < nsplit; ++pr) y += pt[pr * kTiles * 16];
        out(tid, sl0 + itr, y);
      }
    }
    __syncthreads();
  };

  // ---------------------------------------------------------------- per-layer helpers
  // the shared expert's gate/up rows go to gate/up buffer 0, its down rows to down buffer S-1
  auto shared_gu_issue = [&](const FuLayer& Ly) {
    if (lane == 0 && warp < 6) gu_copy(Ly.shared, 0, warp);
  };
  auto shared_dn_issue = [&](const FuLayer& Ly) {
    if (lane == 0 && warp >= 6 && warp < 9) dn_copy(Ly.shared.down, S - 1, warp - 6);
  };

  // ---------------------------------------------------------------- layer 0 prologue
  {
    const FuLayer& L0 = p.layer[0];
    if (tid == 0 && decide(kArmPrologue) && hs) {
      mbar_expect_tx(&gbar[0], gu_bytes);
      mbar_expect_tx(&dbar[S - 1], dn_bytes);
    }
    if (nri > warp) router_load(L0, warp, rw);
    // x into shared memory, the residual rows into hres
    for (int i = tid; i < H / 8; i += kThreads) ((uint4*)xs)[i] = __ldcg((const uint4*)p.x_in + i);
    if (tid < nh) hres[tid] = __ldcg(p.h + h0 + tid);
    __syncthreads();   // barriers armed, xs and hres visible
    if (flags[kArmPrologue] && hs) {
      note_gu(0);
      note_dn(S - 1);
      shared_gu_issue(L0);
      shared_dn_issue(L0);
    }
  }

  for (int l = 0; l < p.L; ++l) {
    const FuLayer& Ly = p.layer[l];
    const bool last = l + 1 == p.L;
    // ------------------------------------------------ (A) x tables + router logits
    x_tables();
    router_run(Ly);   // ends with the logits of this CTA's rows written
    if (p.x_rec)
      for (int r = tid; r < nh; r += kThreads) p.x_rec[(size_t)l * H + h0 + r] = xs[h0 + r];
    if (p.h_rec)
      for (int r = tid; r < nh; r += kThreads) p.h_rec[(size_t)l * H + h0 + r] = hres[r];
    __syncthreads();   // logits written; B tables of x complete
    unsigned g1 = 0, g1s = 0, g2 = 0, g3 = 0;
    if (tid == 0) g1 = grid_arrive(B1, n);
    // ------------------------------------------------ (B) shared gate/up
    if (hs) {
      gu_compute(0, 1);
      fence_proxy_async();
      __syncthreads();
      gu_finalize(0, 1, [&](int) { return S - 1; });
      __syncthreads();
      if (tid == 0) g1s = grid_arrive(B1s, n);
    }
    // ------------------------------------------------ (C) routing
    if (tid == 0) gwait(B1, g1);
    __syncthreads();
    {
      const RouterRef rr{xs, Ly.router_w, Ly.router_bias, H};
      block_topk(p.logits, p.bound, E, k, hs, rr, ts);
    }
    load_slots(ts, k, E, Ly.experts, slot_ex, p.status);
    if (tid < k) wsl[tid] = ts.w[tid];
    if (tid == 0) wsl[S - 1] = hs ? ts.sg : 0.f;
    if (c == 0 && tid == 0 && ts.rechecked) atomicAdd(hdr + 4, 1u);
    if (c == 0 && tid < k) {
      if (p.idx_out) p.idx_out[(size_t)l * k + tid] = ts.idx[tid];
      if (p.w_out) p.w_out[(size_t)l * k + tid] = ts.w[tid];
    }
    if (tid == 0 && decide(kArmRouted)) {
      for (int r = 0; r < k; ++r) {
        mbar_expect_tx(&gbar[(r + hs) % kFuGuBufs], gu_bytes);
        mbar_expect_tx(&dbar[r], dn_bytes);
      }
    }
    __syncthreads();   // slots visible; shared gate/up buffer consumed; barriers armed
    if (flags[kArmRouted]) {
      for (int r = 0; r < k; ++r) {
        note_gu((r + hs) % kFuGuBufs);
        note_dn(r);
      }
      if (lane == 0) {
        const int ncp = 9 * k;   // 6 gate/up copies per expert, then 3 down copies per expert
        for (int cp = warp; cp < ncp; cp += kWarps) {
          if (cp < 6 * k) gu_copy(slot_ex[cp / 6], (cp / 6 + hs) % kFuGuBufs, cp % 6);
          else dn_copy(slot_ex[(cp - 6 * k) / 3].down, (cp - 6 * k) / 3, (cp - 6 * k) % 3);
        }
      }
    }
    // ------------------------------------------------ (D) routed gate/up
    gu_compute(hs, hs + k);
    fence_proxy_async();
    __syncthreads();   // every wait on a gate/up buffer is over: buffer 0 may be armed again
    const bool pre_gu = !last && hs;   // the next layer's shared gate/up rows into buffer 0
    if (tid == 0 && decide(kArmNextGu) && pre_gu) mbar_expect_tx(&gbar[0], gu_bytes);
    gu_finalize(hs, hs + k, [&](int it) { return it - hs; });
    __syncthreads();
    if (tid == 0) g2 = grid_arrive(B2, n);
    if (flags[kArmNextGu] && pre_gu) {
      note_gu(0);
      shared_gu_issue(p.layer[l + 1]);
    }
    // ------------------------------------------------ (E) shared down
    if (hs) {
      if (tid == 0) gwait(B1s, g1s);
      __syncthreads();
      a_tables(S - 1, S);
      __syncthreads();
      dn_run(S - 1, S, [&](int r, int, float y) { ysh[r] = wsl[S - 1] * y; });
      fence_proxy_async();
      if (tid == 0 && decide(kArmNextDn) && !last) mbar_expect_tx(&dbar[S - 1], dn_bytes);   // the next layer's shared down rows
      __syncthreads();
      if (flags[kArmNextDn] && !last) {
        note_dn(S - 1);
        shared_dn_issue(p.layer[l + 1]);
      }
    }
    if (!last && nri > warp) router_load(p.layer[l + 1], warp, rw);   // the next layer's router rows
    // ------------------------------------------------ (F) routed down + combine
    if (tid == 0) gwait(B2, g2);
    __syncthreads();
    a_tables(0, k);
    __syncthreads();
    if (tid < nh) yacc[tid] = hres[tid];
    dn_run(0, k, [&](int r, int sl, float y) { yacc[r] = fmaf(wsl[sl], y, yacc[r]); });
    fence_proxy_async();   // the down buffers are refilled by the next layer's copies
    float ss = 0.f;
    if (tid < nh) {
      const float v = hs ? yacc[tid] + ysh[tid] : yacc[tid];
      yacc[tid] = v;
      p.hacc[h0 + tid] = v;
      ss = v * v;
    }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int w = 0; w < kWarps; ++w) t += red[w];
      p.gpart[c] = t;
      g3 = grid_arrive(B3, n);
    }
    // ------------------------------------------------ (G) RMSNorm
    if (tid == 0) gwait(B3, g3);
    __syncthreads();
    if (warp == 0) {   // the CTAs' partials summed in a fixed order (the same in every CTA)
      float t = 0.f;
      for (int q = lane; q < n; q += 32) t += __ldcg(p.gpart + q);
      t = warp_sum(t);
      if (lane == 0) red[0] = t;
    }
    __syncthreads();
    const float inv = 1.f / sqrtf(red[0] / (float)H + Ly.eps);
    if (last) {
      if (tid < nh) {
        const int j = h0 + tid;
        const float v = yacc[tid];
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
        ((uint32_t*)xs)[i] = (uint32_t)f32_to_bf16(v.x * inv * bf16lo(gw)) |
                             ((uint32_t)f32_to_bf16(v.y * inv * bf16hi(gw)) << 16);
      }
      if (tid < nh) hres[tid] = yacc[tid];
      __syncthreads();
    }
  }
  // no bulk copy may still be writing into shared memory when the CTA exits
  __syncthreads();
  if (tid == 0) {
    for (int b = 0; b < kFuGuBufs; ++b)
      if ((gissued >> b) & 1u) mbar_wait_bounded(&gbar[b], (gpar >> b) & 1u, p.wait_ns, nullptr);
    for (int b = 0; b < S; ++b)
      if ((dissued >> b) & 1u) mbar_wait_bounded(&dbar[b], (dpar >> b) & 1u, p.wait_ns, nullptr);
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
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess) return e;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, sm)) != cudaSuccess) return e;
  if (per_sm < 1 || p.nCTA > per_sm * num_sms()) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.nCTA);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the grid-wide barriers need it
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  FusedParams q = p;
  void* args[] = {&q};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace qmoe
