// Expert kernels of the decode chain (sm_100a): gate/up + SwiGLU, and down +
// weighted combine + residual, for T <= 8 tokens of one layer.
//
// Work split: every CTA owns whole output rows, so no result is ever summed
// across CTAs. The gate/up kernel's CTA c owns intermediate rows [j0, j1)
// (at most 8) of every chosen expert: for each expert one 16-row MMA tile
// (rows 0-7 = gate rows j0.., rows 8-15 = up rows j0..), all H columns; it
// finishes with a_j = silu(g_j) * u_j. The down kernel's CTA owns hidden rows
// [h0, h1) (at most 32) of every chosen expert and finishes with
// hacc = h + sum_e w_e y_e for those rows.
//
// Weights move with the bulk-copy (TMA) engine: a CTA's rows of one matrix
// are contiguous in memory (row-major codes [R][K*b/32] words, bf16 scales and
// biases [R][K/64]), so each expert costs a handful of cp.async.bulk copies
// into shared memory, completed on an mbarrier (one per buffer).
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "stage.cuh"
#include "sync.cuh"
#include "topk.cuh"

namespace qmoe {

// ------------------------------------------------------------------ gate/up + SwiGLU
constexpr int kGuBufs = 3;      // expert tiles staged per CTA (the shared expert's buffer is reused)
constexpr int kGuMaxRows = 8;   // intermediate rows per CTA

struct GuLayout {
  int RB, P, SRB, SBR, GB;   // code bytes per row, padded row pitch, scale bytes per row, scale region, buffer bytes
  size_t buf, btab, gs, part, slots, topk, bars, total;
};
__host__ __device__ inline GuLayout gu_layout(int H, int bits) {
  GuLayout L;
  L.RB = H * bits / 8;
  L.P = L.RB;   // rows land contiguously (one bulk copy per row block)
  L.SRB = H / 32;
  L.SBR = sb_region(kGuMaxRows, L.SRB);
  L.GB = (2 * kGuMaxRows * L.P + 4 * L.SBR + 127) & ~127;
  size_t o = 0;
  L.buf = o; o += (size_t)kGuBufs * L.GB;
  L.btab = o; o += sizeof(uint2) * (size_t)(H / kSpan) * kBtPerSpan;
  L.gs = o; o += sizeof(float) * 2 * (size_t)(H / kGroup);   // [2^-p_g | X_g]
  o = (o + 15) & ~(size_t)15;
  const size_t part = sizeof(float) * kGuBufs * kWarps * 16;
  L.part = o; L.topk = o;   // the top-k scratch is dead before the partial sums are written
  o += part > sizeof(TopkSmem) ? part : sizeof(TopkSmem);
  o = (o + 15) & ~(size_t)15;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.bars = o; o += 8 * kGuBufs;
  L.total = o;
  return L;
}

// grid (nCTA, T), block 512. Before the dependency wait (this kernel starts
// only after every router CTA has passed its own wait, so x is final): the
// shared expert's copies and the B tables of x. After it: every CTA ranks the
// router's logits itself (the first CTA of each token publishes the selection
// for the down kernel behind a flag), issues the copies of the routed experts
// whose buffers are free, computes the shared expert while they land, stores
// and fences its a, lets the down kernel launch, and computes the routed
// experts.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 2) gateup_decode_kernel(GateUpParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GuLayout L = gu_layout(p.H, BITS);
  unsigned char* bufs = smem + L.buf;
  uint2* btab = (uint2*)(smem + L.btab);
  float* gs = (float*)(smem + L.gs);
  float* part = (float*)(smem + L.part);
  moe_expert* slot_ex = (moe_expert*)(smem + L.slots);
  TopkSmem& ts = *(TopkSmem*)(smem + L.topk);
  uint64_t* bars = (uint64_t*)(smem + L.bars);

  const int t = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I, S = p.S, k = p.k;
  const int ng = H / kGroup, nspans = H / kSpan;
  const int j0 = (int)((unsigned)I * blockIdx.x / gridDim.x);
  const int n = (int)((unsigned)I * (blockIdx.x + 1) / gridDim.x) - j0;
  const int nitems = k + (p.has_shared ? 1 : 0);
  auto item_slot = [&](int it) { return p.has_shared ? (it == 0 ? S - 1 : it - 1) : it; };
  int pre;
  const unsigned sbw = sb_window(j0, n, L.SRB, pre);
  const unsigned item_bytes = 2u * n * L.RB + 4u * sbw;
  bool ok = true;

  auto arm = [&](int it) {   // thread 0, before the barrier that precedes the item's copies
    if (tid == 0) mbar_expect_tx(&bars[it % kGuBufs], item_bytes);
  };
  // copies of item `it` into buffer it % kGuBufs, one per call: c = 0 gate
  // code rows, 1 up code rows (row blocks), 2..5 gate/up scales, gate/up biases
  const int ncp = 6;
  auto issue_ex = [&](const moe_expert& ex, int it, int c) {
    const int b = it % kGuBufs;
    unsigned char* buf = bufs + (size_t)b * L.GB;
    fence_proxy_async();
    if (c < 2) {
      const moe_qmat& m = c == 0 ? ex.gate : ex.up;
      bulk_g2s(buf + (size_t)c * kGuMaxRows * L.P, (const char*)m.q + (size_t)j0 * L.RB, (unsigned)n * L.RB, &bars[b]);
    } else {
      const int w = c - 2;   // 0 gate scales, 1 up scales, 2 gate biases, 3 up biases
      const moe_qmat& m = (w & 1) ? ex.up : ex.gate;
      const uint16_t* src = w < 2 ? m.scales : m.biases;
      bulk_g2s(buf + 2 * kGuMaxRows * L.P + w * L.SBR, (const char*)src + (((size_t)j0 * L.SRB) & ~(size_t)15), sbw,
               &bars[b]);
    }
  };
  auto issue = [&](int it, int c) { issue_ex(slot_ex[item_slot(it)], it, c); };
  // MMAs of this warp's spans [nspans*w/16, nspans*(w+1)/16) for the items
  // [i0, i1) (at most kGuBufs, each one 16-row tile in buffer it % kGuBufs):
  // the B fragments of a span are loaded once for all items. Lane tq of a
  // quad loads 4 spans of one of the row's four scale/bias arrays (gate
  // scales, up scales, gate biases, up biases) and the quad shares them by
  // shuffles. Row sums go to part[(it - i0)][warp][16].
  const bool al16 = L.SRB % 16 == 0;
  auto compute_items = [&](int i0, int i1) {
    const int g = lane >> 2, tq = lane & 3, qb = lane & ~3;
    const int bl = bt_lane_index(lane);
    const LaneK K = lane_consts(tq);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int W = QTraits<BITS>::kWordsPerThread;
    const int s0 = nspans * warp / kWarps, s1 = nspans * (warp + 1) / kWarps;
    for (int sp = s0; sp < s1; sp += 2) {   // span pairs: B fragments loaded once for all items
      BFrag B[2];
      load_bfrag(B[0], btab + sp * kBtPerSpan, bl, gs, ng, sp, tq);
      if (sp + 1 < s1) load_bfrag(B[1], btab + (sp + 1) * kBtPerSpan, bl, gs, ng, sp + 1, tq);
      for (int it = i0; it < i1; ++it) {
        if (sp == s0) ok &= mbar_wait_bounded(&bars[it % kGuBufs], (unsigned)(it / kGuBufs) & 1u, p.wait_ns, p.status);
        const unsigned char* buf = bufs + (size_t)(it % kGuBufs) * L.GB;
        // 16-byte chunk of 4 spans' scale (or bias) words; a pair that starts on the last span of a
        // chunk (odd first span of the warp) takes its second span from the next chunk
        const unsigned char* sc = buf + 2 * kGuMaxRows * L.P + tq * L.SBR + pre + g * L.SRB;
        const uint4 sv0 = lds_chunk(sc + 16 * (sp >> 2), al16);
        const uint4 sv1 = ((sp & 3) == 3 && sp + 1 < s1) ? lds_chunk(sc + 16 * ((sp + 1) >> 2), al16) : sv0;
        float aa = 0.f, ab = 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int s = sp + q;
          if (s < s1) {
            const uint32_t w = chunk_word(q == 0 ? sv0 : sv1, s & 3);
            uint32_t wa[W], wb[W];
            const unsigned char* ra = buf + (size_t)g * L.P + s * SB + tq * W * 4;
            const unsigned char* rb = ra + (size_t)kGuMaxRows * L.P;
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
    if (s0 == s1) {   // no spans: zero contributions
      for (int it = i0; it < i1; ++it)
        if (lane < 16) part[((size_t)(it - i0) * kWarps + warp) * 16 + lane] = 0.f;
    }
  };
  // a = silu(g) * u of the items [i0, i1) from the partial sums (after a barrier)
  auto finalize = [&](int i0, int i1) {
    if (tid < (i1 - i0) * n) {
      const int i = tid / n, r = tid - i * n;
      const float* pt = part + (size_t)i * kWarps * 16;
      float gsum = 0.f, usum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) { gsum += pt[w * 16 + r]; usum += pt[w * 16 + 8 + r]; }
      p.a[((size_t)t * S + item_slot(i0 + i)) * I + j0 + r] = silu_f32(gsum) * usum;
      if (i0 == 0 && p.has_shared) __threadfence();   // the down kernel reads the shared expert's a before its own wait
    }
  };


  if (tid == 0) {
    for (int b = 0; b < kGuBufs; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    if (p.has_shared) slot_ex[S - 1] = p.shared;
  }
  if (p.has_shared) {   // the shared expert's copies go out first, from the kernel parameters
    arm(0);
    if (warp < ncp) {
      asm volatile("bar.sync 1, %0;" :: "r"(ncp * 32) : "memory");   // barriers initialised (warps 0..ncp-1)
      if (lane == 0) issue_ex(p.shared, 0, warp);
    }
  }
  // B tables of x, straight from registers
  {
    constexpr int EPT = TabTraits<BITS>::kEPT;
    const int nq = H / EPT;
    for (int q0 = 0; q0 < nq; q0 += kThreads) {
      const int q = q0 + tid;
      float v[EPT];
      if (q < nq) load_chunk_bf16<BITS>(p.x + (size_t)t * H, q, v);
      build_tables<BITS>(v, q * EPT, q < nq, btab, gs, ng);
    }
  }
  __syncthreads();

  // the router's logits are complete after the wait
  griddep_wait();
  {
    const RouterRef rr{p.x + (size_t)t * H, p.router_w, p.router_bias, H};
    block_topk(p.logits + (size_t)t * (p.E + 1), p.bound + (size_t)t * (p.E + 1), p.E, k, p.has_shared, rr, ts);
  }
  load_slots(ts, k, p.E, p.experts, slot_ex, p.status);
  if (blockIdx.x == 0 && tid == 0 && p.rechecks && ts.rechecked) atomicAdd(p.rechecks, 1u);
  if (blockIdx.x == 0) {   // publish the selection for the down kernel (and the user copies)
    if (tid < k) {
      p.sel_idx[(size_t)t * k + tid] = ts.idx[tid];
      p.sel_w[(size_t)t * k + tid] = ts.w[tid];
      if (p.idx_out) p.idx_out[(size_t)t * k + tid] = ts.idx[tid];
      if (p.w_out) p.w_out[(size_t)t * k + tid] = ts.w[tid];
    }
    if (tid == 0) p.sel_sg[t] = ts.sg;
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      st_release_u32(p.sel_flag + t, 1u);
    }
  }
  // Items: 0 = the shared expert (copies issued before the wait, buffer 0), then the
  // routed ones. The routed items whose buffers are free go out first; the shared
  // expert is computed while they land, and its a is stored (and fenced) before the
  // dependent launch, since the down kernel applies it before its own wait.
  int it0 = 0, issued = 0;   // items [0, issued) have had their copies issued
  if (p.has_shared) {
    const int w1 = nitems < kGuBufs ? nitems : kGuBufs;
    for (int it = 1; it < w1; ++it) arm(it);
    __syncthreads();   // slots loaded
    if (lane == 0)
      for (int c = warp; c < ncp * (w1 - 1); c += kWarps) issue(1 + c / ncp, c % ncp);
    compute_items(0, 1);
    fence_proxy_async();
    __syncthreads();
    finalize(0, 1);
    __syncthreads();   // ... so no thread signals the dependent launch before those stores are fenced
    it0 = 1;
    issued = w1;
  }
  griddep_launch_dependents();
  // routed items in waves of up to kGuBufs; every warp takes its spans of all items of the wave
  for (int w0 = it0; w0 < nitems; w0 += kGuBufs) {
    const int w1 = nitems - w0 < kGuBufs ? nitems : w0 + kGuBufs;
    // after a wait ran out, nothing more is armed or issued (a new phase on a
    // buffer whose copies may still be landing would mix two phases)
    if (!__syncthreads_and(ok)) break;
    const int a0 = issued > w0 ? issued : w0;   // the wave's items not yet issued
    for (int it = a0; it < w1; ++it) arm(it);
    __syncthreads();   // slots loaded (first wave) / previous wave's buffers and partial sums consumed
    if (lane == 0)
      for (int c = warp; c < ncp * (w1 - a0); c += kWarps) issue(a0 + c / ncp, c % ncp);
    issued = w1;
    compute_items(w0, w1);
    fence_proxy_async();
    __syncthreads();
    finalize(w0, w1);
  }
  if (!__syncthreads_and(ok) && tid == 0) {   // drain: no copy may still be landing when the CTA exits
    for (int it = (issued > kGuBufs ? issued - kGuBufs : 0); it < issued; ++it)
      mbar_wait_bounded(&bars[it % kGuBufs], (unsigned)(it / kGuBufs) & 1u, p.wait_ns, nullptr);
  }
}

// ------------------------------------------------------------------ down + weighted combine + residual
constexpr int kDnBufs = 4;      // expert row blocks staged per CTA
constexpr int kDnMaxRows = 32;  // hidden rows per CTA

struct DnLayout {
  int RB, P, SRB, SBR, GB, nsp, ng;
  size_t buf, btab, gs, part, yacc, wsl, slots, topk, bars, total;
};
__host__ __device__ inline DnLayout dn_layout(int I, int S, int bits) {
  DnLayout L;
  L.RB = I * bits / 8;
  L.P = L.RB;   // rows land contiguously (one bulk copy per row block)
  L.SRB = I / 32;
  L.SBR = sb_region(kDnMaxRows, L.SRB);
  L.GB = (kDnMaxRows * L.P + 2 * L.SBR + 127) & ~127;
  L.nsp = I / kSpan;
  L.ng = I / kGroup;
  const int nb = S < kDnBufs ? S : kDnBufs;
  size_t o = 0;
  L.buf = o; o += (size_t)nb * L.GB;
  L.btab = o; o += sizeof(uint2) * (size_t)S * L.nsp * kBtPerSpan;
  L.gs = o; o += sizeof(float) * 2 * (size_t)S * L.ng;     // per slot [2^-p_g | X_g]
  o = (o + 15) & ~(size_t)15;
  const size_t part = sizeof(float) * kWarps * (kDnMaxRows / 16) * 16;   // [segment][tile][16]
  L.part = o; L.topk = o;   // the top-k scratch is dead before the partial sums are written
  o += part > sizeof(TopkSmem) ? part : sizeof(TopkSmem);
  L.yacc = o; o += sizeof(float) * kDnMaxRows;
  L.wsl = o; o += sizeof(float) * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.bars = o; o += 8 * kDnBufs;
  L.total = o;
  return L;
}

// grid (nCTA, T), block 512. This kernel starts once every gate/up CTA has
// passed its dependency wait, so the router's logits, the residual h and the
// shared expert's a are final: before its own wait it ranks the logits,
// starts the copies of its rows of every chosen expert's down matrix and
// applies the shared expert. After the wait it turns the routed experts' a
// into B tables and forms hacc = h + sum_i w_i y_i + sg * y_shared for its rows.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 2) down_decode_kernel(DownParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int S = p.S;
  const DnLayout L = dn_layout(p.I, S, BITS);
  unsigned char* bufs = smem + L.buf;
  uint2* btab = (uint2*)(smem + L.btab);
  float* gs = (float*)(smem + L.gs);
  float* part = (float*)(smem + L.part);
  float* yacc = (float*)(smem + L.yacc);
  float* wsl = (float*)(smem + L.wsl);
  moe_expert* slot_ex = (moe_expert*)(smem + L.slots);
  TopkSmem& ts = *(TopkSmem*)(smem + L.topk);
  uint64_t* bars = (uint64_t*)(smem + L.bars);

  const int t = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I, k = p.k, nsp = L.nsp, ng = L.ng;
  const int nb = S < kDnBufs ? S : kDnBufs;
  const int h0 = (int)((unsigned)H * blockIdx.x / gridDim.x);
  const int n = (int)((unsigned)H * (blockIdx.x + 1) / gridDim.x) - h0;
  const int ntile = (n + 15) / 16;
  const int nitems = S;
  auto item_slot = [&](int it) { return p.has_shared ? (it == 0 ? S - 1 : it - 1) : it; };
  int pre;
  const unsigned sbw = sb_window(h0, n, L.SRB, pre);
  const unsigned item_bytes = (unsigned)n * L.RB + 2u * sbw;
  const int per = nsp * kBtPerSpan;
  bool ok = true;

  // copies of item `it`, one per call: c = 0 code rows, 1 scales, 2 biases (row blocks)
  const int ncp = 3;
  auto issue = [&](int it, int c) {
    const int b = it % nb;
    unsigned char* buf = bufs + (size_t)b * L.GB;
    const moe_qmat& m = slot_ex[item_slot(it)].down;
    fence_proxy_async();
    if (c == 0) {
      bulk_g2s(buf, (const char*)m.q + (size_t)h0 * L.RB, (unsigned)n * L.RB, &bars[b]);
    } else {
      const uint16_t* src = c == 1 ? m.scales : m.biases;
      bulk_g2s(buf + kDnMaxRows * L.P + (c - 1) * L.SBR, (const char*)src + (((size_t)h0 * L.SRB) & ~(size_t)15), sbw,
               &bars[b]);
    }
  };
  // B tables of slots [sl0, sl1) from a
  auto tables = [&](int sl0, int sl1) {
    constexpr int EPT = TabTraits<BITS>::kEPT;
    const int qs = I / EPT, nq = (sl1 - sl0) * qs;
    for (int q0 = 0; q0 < nq; q0 += kThreads) {
      const int q = q0 + tid, sl = sl0 + q / qs, e = (q - (q / qs) * qs) * EPT;
      const bool valid = q < nq;
      float v[EPT];
      if (valid) load_chunk_f32<BITS>(p.a + ((size_t)t * S + sl) * I, e / EPT, v);
      build_tables<BITS>(v, e, valid, btab + (size_t)(valid ? sl : 0) * per, gs + (size_t)(valid ? sl : 0) * 2 * ng, ng);
    }
  };
  // MMAs of spans [s0, s1) of every row tile of item it, the span's B
  // fragments loaded once for the tiles; row sums of tile tl, rows g / g+8
  // to pt[tl][16] (quad-reduced). Lane tq of a quad loads 4 spans of one
  // scale/bias row of each tile (tq = 0 scales of row r, 1 scales of row
  // r+8, 2 biases of row r, 3 biases of row r+8); the quad shares them by
  // shuffles.
  constexpr int kTiles = kDnMaxRows / 16;
  const bool al16 = L.SRB % 16 == 0;
  auto seg_compute = [&](int it, int s0, int s1, float* pt) {
    const int slot = item_slot(it);
    const unsigned char* buf = bufs + (size_t)(it % nb) * L.GB;
    const int g = lane >> 2, tq = lane & 3, qb = lane & ~3;
    const int bl = bt_lane_index(lane);
    const LaneK K = lane_consts(tq);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int W = QTraits<BITS>::kWordsPerThread;
    const uint2* bt = btab + (size_t)slot * per;
    const float* gsl = gs + (size_t)slot * 2 * ng;
    float aa[kTiles], ab[kTiles];
    uint4 sv[kTiles];
#pragma unroll
    for (int tl = 0; tl < kTiles; ++tl) { aa[tl] = 0.f; ab[tl] = 0.f; sv[tl] = make_uint4(0u, 0u, 0u, 0u); }
    for (int s = s0; s < s1; ++s) {
      BFrag B;
      load_bfrag(B, bt + s * kBtPerSpan, bl, gsl, ng, s, tq);
#pragma unroll
      for (int tl = 0; tl < kTiles; ++tl) {
        if (tl < ntile) {
          const int r = tl * 16 + g;
          if (s == s0 || (s & 3) == 0)
            sv[tl] = lds_chunk(buf + kDnMaxRows * L.P + pre + (tq >> 1) * L.SBR + (r + 8 * (tq & 1)) * L.SRB +
                                   16 * (s >> 2), al16);
          const uint32_t w = chunk_word(sv[tl], s & 3);
          uint32_t wa[W], wb[W];
          const unsigned char* ra = buf + (size_t)r * L.P + s * SB + tq * W * 4;
          const unsigned char* rb = ra + (size_t)8 * L.P;
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
  // items [i0, i1) (all staged): segments (item, span part) spread over the
  // warps, each covering all row tiles; then, in item order, yacc += w * y
  auto run = [&](int i0, int i1) {
    const int ni = i1 - i0;
    int nsplit = kWarps / ni;
    nsplit = nsplit < 1 ? 1 : (nsplit > nsp ? nsp : nsplit);
    const int nseg = ni * nsplit;
    int waited = -1;
    for (int sg = warp; sg < nseg; sg += kWarps) {
      const int itr = sg / nsplit, pr = sg - itr * nsplit;
      const int it = i0 + itr;
      if (it != waited) {
        ok &= mbar_wait_bounded(&bars[it % nb], (unsigned)(it / nb) & 1u, p.wait_ns, p.status);
        waited = it;
      }
      seg_compute(it, nsp * pr / nsplit, nsp * (pr + 1) / nsplit, part + (size_t)sg * kTiles * 16);
    }
    fence_proxy_async();
    __syncthreads();
    if (tid < n) {
      const int tl = tid >> 4, rr = tid & 15;
      float acc = yacc[tid];
      for (int itr = 0; itr < ni; ++itr) {
        const float* pt = part + (size_t)itr * nsplit * kTiles * 16 + tl * 16 + rr;
        float y = 0.f;
        for (int pr = 0; pr < nsplit; ++pr) y += pt[pr * kTiles * 16];
        acc = fmaf(wsl[item_slot(i0 + itr)], y, acc);
      }
      yacc[tid] = acc;
    }
  };

  if (tid == 0) {
    for (int b = 0; b < nb; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    for (int b = 0; b < nb; ++b) mbar_expect_tx(&bars[b], item_bytes);   // items 0..nb-1
    if (p.has_shared) slot_ex[S - 1] = p.shared;
  }
  // the selection of the gate/up kernel's first CTA: published behind a flag that the norm
  // kernel clears after this kernel has completed (the wait is bounded)
  if (tid == 0) {
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_u32(p.sel_flag + t) == 0u)
      if (globaltimer_ns() - t0 > p.wait_ns) {
        latch_timeout(p.status);
        break;
      }
  }
  __syncthreads();
  if (tid < k) {
    ts.idx[tid] = __ldcg(p.sel_idx + (size_t)t * k + tid);
    wsl[tid] = __ldcg(p.sel_w + (size_t)t * k + tid);
  }
  if (tid == 0 && p.has_shared) wsl[S - 1] = __ldcg(p.sel_sg + t);
  __syncthreads();
  load_slots(ts, k, p.E, p.experts, slot_ex, p.status);
  if (tid < n) yacc[tid] = __ldcg(p.h + (size_t)t * H + h0 + tid);
  __syncthreads();
  if (lane == 0)
    for (int c = warp; c < ncp * nb; c += kWarps) issue(c / ncp, c % ncp);
  int issued = nb;   // items [0, issued) have their copies in flight or landed
  int it0 = 0;
  if (p.has_shared) {   // the shared expert's a is final: apply it before the wait
    tables(S - 1, S);
    __syncthreads();
    run(0, 1);
    it0 = 1;
  }

  griddep_wait();
  griddep_launch_dependents();
  tables(0, k);
  __syncthreads();
  for (int w0 = it0; w0 < nitems; w0 += nb) {
    const int w1 = nitems - w0 < nb ? nitems : w0 + nb;
    if (issued < w1) {   // refill buffers whose previous items are done
      // after a wait ran out, nothing more is armed or issued
      if (!__syncthreads_and(ok)) break;
      if (tid == 0)
        for (int it = issued; it < w1; ++it) mbar_expect_tx(&bars[it % nb], item_bytes);
      __syncthreads();
      if (lane == 0)
        for (int c = warp; c < ncp * (w1 - issued); c += kWarps) issue(issued + c / ncp, c % ncp);
      issued = w1;
    }
    run(w0, w1);
    __syncthreads();
  }
  if (tid < n) p.hacc[(size_t)t * H + h0 + tid] = yacc[tid];
  if (!__syncthreads_and(ok) && tid == 0) {   // drain: no copy may still be landing when the CTA exits
    for (int it = (issued > nb ? issued - nb : 0); it < issued; ++it)
      mbar_wait_bounded(&bars[it % nb], (unsigned)(it / nb) & 1u, p.wait_ns, nullptr);
  }
}

// ------------------------------------------------------------------ diagnostics
// One warp waits, through the same bounded wait as every kernel above, on an
// mbarrier phase that nothing completes (16 bytes expected, no copy issued):
// the wait gives up after bound_ns, latches MOE_ERR_TIMEOUT in *status and the
// kernel returns. Nothing is in flight when it gives up.
__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t* status, unsigned long long bound_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_expect_tx(&bar, 16);
  }
  __syncthreads();
  mbar_wait_bounded(&bar, 0u, bound_ns, status);
}

// ------------------------------------------------------------------ launchers
static cudaError_t launch_pdl(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
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

static cudaError_t prepare(const void* fn, size_t bytes) {
  cudaError_t e = set_func_attr(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  return set_func_attr(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

static int optin_smem() {
  static int v = 0;
  if (!v) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (v <= 0) v = 227 * 1024;
  }
  return v;
}

size_t gateup_smem_bytes(int H, int bits) { return gu_layout(H, bits).total; }

bool chain_supported(int H, int I, int k, int has_shared, int bits) {
  const int S = k + (has_shared ? 1 : 0);
  return gu_layout(H, bits).total <= (size_t)optin_smem() && dn_layout(I, S, bits).total <= (size_t)optin_smem();
}
size_t down_smem_bytes(int I, int S, int bits) { return dn_layout(I, S, bits).total; }

int gateup_ctas(int I) {
  int n = num_sms();
  const int lo = (I + kGuMaxRows - 1) / kGuMaxRows;
  if (n < lo) n = lo;
  if (n > I) n = I;
  return n;
}
int down_ctas(int H) {
  int n = num_sms();
  const int lo = (H + kDnMaxRows - 1) / kDnMaxRows;
  if (n < lo) n = lo;
  if (n > H) n = H;
  return n;
}

cudaError_t launch_gateup(const GateUpParams& p, int bits, int T, bool pdl, cudaStream_t s) {
  GateUpParams q = p;
  const size_t sm = gateup_smem_bytes(p.H, bits);
  if (sm > (size_t)optin_smem()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)gateup_decode_kernel<4> : (const void*)gateup_decode_kernel<2>;
  cudaError_t e = prepare(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  return launch_pdl(fn, dim3(p.nCTA, T), dim3(kThreads), sm, s, pdl, args);
}

cudaError_t launch_down(const DownParams& p, int bits, int T, bool pdl, cudaStream_t s) {
  DownParams q = p;
  const size_t sm = down_smem_bytes(p.I, p.S, bits);
  if (sm > (size_t)optin_smem()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)down_decode_kernel<4> : (const void*)down_decode_kernel<2>;
  cudaError_t e = prepare(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  return launch_pdl(fn, dim3(p.nCTA, T), dim3(kThreads), sm, s, pdl, args);
}

cudaError_t launch_selftest_wait(uint32_t* status, unsigned long long bound_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, bound_ns);
  return cudaGetLastError();
}

}  // namespace qmoe
