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
#include "topk.cuh"

namespace qmoe {

// ------------------------------------------------------------------ mbarrier and bulk copies
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// orders this thread's earlier generic-proxy accesses of shared memory before its later bulk copies
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
// global -> shared bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned), counted on bar
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Waits for the phase of parity `parity` of bar, for at most bound_ns; on
// timeout latches MOE_ERR_TIMEOUT in *status and returns false.
__device__ __noinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, unsigned long long bound_ns,
                                               uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > bound_ns) {
      if (status) atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

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

// A fragments of one span for MMA rows g (from ra) and g+8 (from rb), t = lane & 3.
template <int BITS>
__device__ __forceinline__ void frag_codes(Frag<BITS>& F, const unsigned char* ra, const unsigned char* rb) {
  if constexpr (BITS == 4) {
    const uint4 va = *(const uint4*)ra, vb = *(const uint4*)rb;
    F.wa[0] = va.x; F.wa[1] = va.y; F.wa[2] = va.z; F.wa[3] = va.w;
    F.wb[0] = vb.x; F.wb[1] = vb.y; F.wb[2] = vb.z; F.wb[3] = vb.w;
  } else {
    const uint2 va = *(const uint2*)ra, vb = *(const uint2*)rb;
    F.wa[0] = va.x; F.wa[1] = va.y;
    F.wb[0] = vb.x; F.wb[1] = vb.y;
  }
}

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

// ------------------------------------------------------------------ gate/up + SwiGLU
constexpr int kGuBufs = 3;      // expert tiles staged per CTA (the shared expert's buffer is reused)
constexpr int kGuMaxRows = 8;   // intermediate rows per CTA

struct GuLayout {
  int RB, SRB, SBR, GB;   // code bytes per row, scale bytes per row, scale region, buffer bytes
  size_t buf, btab, gs, part, slots, topk, bars, total;
};
__host__ __device__ inline GuLayout gu_layout(int H, int bits) {
  GuLayout L;
  L.RB = H * bits / 8;
  L.SRB = H / 32;
  L.SBR = sb_region(kGuMaxRows, L.SRB);
  L.GB = (2 * kGuMaxRows * L.RB + 4 * L.SBR + 127) & ~127;
  size_t o = 0;
  L.buf = o; o += (size_t)kGuBufs * L.GB;
  L.btab = o; o += sizeof(uint2) * (size_t)(H / kSpan) * kBtPerSpan;
  L.gs = o; o += sizeof(float) * 2 * (size_t)(H / kGroup);   // [2^-p_g | X_g]
  o = (o + 15) & ~(size_t)15;
  L.part = o; o += sizeof(float) * kWarps * 16;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.topk = o; o += sizeof(TopkSmem);
  o = (o + 15) & ~(size_t)15;
  L.bars = o; o += 8 * kGuBufs;
  L.total = o;
  return L;
}

// grid (nCTA, T), block 512. Items: the shared expert first (its copies and
// MMAs run before the dependency wait: this kernel starts only after every
// router CTA has passed its own wait, so x is final; its a values are stored
// and fenced before this kernel lets the down kernel launch), then the k
// routed experts, which every CTA ranks itself from the router's logits and
// computes side by side, each on its own group of warps.
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
  const int j0 = (int)((long long)I * blockIdx.x / gridDim.x);
  const int n = (int)((long long)I * (blockIdx.x + 1) / gridDim.x) - j0;
  const int nitems = k + (p.has_shared ? 1 : 0);
  auto item_slot = [&](int it) { return p.has_shared ? (it == 0 ? S - 1 : it - 1) : it; };
  int pre;
  const unsigned sbw = sb_window(j0, n, L.SRB, pre);
  const unsigned item_bytes = 2u * n * L.RB + 4u * sbw;
  bool ok = true;

  auto arm = [&](int it) {   // thread 0, before the barrier that precedes the item's copies
    if (tid == 0) mbar_expect_tx(&bars[it % kGuBufs], item_bytes);
  };
  // copies of item `it` into buffer it % kGuBufs: one copy per thread listed below
  auto issue = [&](int it, int c) {   // c = copy 0..5: gate codes, up codes, gate/up scales, gate/up biases
    const int b = it % kGuBufs;
    unsigned char* buf = bufs + (size_t)b * L.GB;
    const moe_expert& ex = slot_ex[item_slot(it)];
    fence_proxy_async();
    if (c < 2) {
      const moe_qmat& m = c == 0 ? ex.gate : ex.up;
      bulk_g2s(buf + (size_t)c * kGuMaxRows * L.RB, (const char*)m.q + (size_t)j0 * L.RB, (unsigned)n * L.RB, &bars[b]);
    } else {
      const int w = c - 2;   // 0 gate scales, 1 up scales, 2 gate biases, 3 up biases
      const moe_qmat& m = (w & 1) ? ex.up : ex.gate;
      const uint16_t* src = w < 2 ? m.scales : m.biases;
      bulk_g2s(buf + 2 * kGuMaxRows * L.RB + w * L.SBR, (const char*)src + (((size_t)j0 * L.SRB) & ~(size_t)15), sbw,
               &bars[b]);
    }
  };
  // MMAs of spans [s0, s1) of the item in buffer b; row sums of rows g, g+8 returned in acc_a, acc_b (quad-reduced)
  auto compute = [&](int b, int s0, int s1, float& acc_a, float& acc_b) {
    const unsigned char* buf = bufs + (size_t)b * L.GB;
    const int g = lane >> 2, tq = lane & 3;
    const int bl = bt_lane_index(lane);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int WB = QTraits<BITS>::kWordsPerThread * 4;
    const unsigned char* ra = buf + (size_t)g * L.RB + tq * WB;
    const unsigned char* rb = buf + (size_t)(kGuMaxRows + g) * L.RB + tq * WB;
    const unsigned char* sc = buf + 2 * kGuMaxRows * L.RB + pre + g * L.SRB;
    acc_a = 0.f; acc_b = 0.f;
    for (int s = s0; s < s1; ++s) {
      Frag<BITS> F;
      frag_codes<BITS>(F, ra + s * SB, rb + s * SB);
      F.sa = *(const uint32_t*)(sc + s * 4);
      F.sb = *(const uint32_t*)(sc + L.SBR + s * 4);
      F.ba = *(const uint32_t*)(sc + 2 * L.SBR + s * 4);
      F.bb = *(const uint32_t*)(sc + 3 * L.SBR + s * 4);
      int c[4];
      mma_frag<BITS>(F, btab + s * kBtPerSpan, bl, c);
      scale_frag_i(F.sa, F.sb, F.ba, F.bb, c, gs, gs + ng, s, tq, acc_a, acc_b);
    }
    acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
    acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 1);
    acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 2);
    acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 2);
  };
  auto store_a = [&](int it, int i, float gsum, float usum) {
    p.a[((size_t)t * S + item_slot(it)) * I + j0 + i] = silu_f32(gsum) * usum;
  };

  if (tid == 0) {
    for (int b = 0; b < kGuBufs; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    if (p.has_shared) slot_ex[S - 1] = p.shared;
  }
  if (p.has_shared) arm(0);
  __syncthreads();
  if (p.has_shared && warp < 6 && lane == 0) issue(0, warp);
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
  int it0 = 0;
  if (p.has_shared) {   // all warps: spans [nspans*w/16, nspans*(w+1)/16)
    ok &= mbar_wait_bounded(&bars[0], 0, p.wait_ns, p.status);
    float aa, ab;
    compute(0, nspans * warp / kWarps, nspans * (warp + 1) / kWarps, aa, ab);
    if ((lane & 3) == 0) { part[warp * 16 + (lane >> 2)] = aa; part[warp * 16 + 8 + (lane >> 2)] = ab; }
    fence_proxy_async();
    __syncthreads();
    if (tid < n) {
      float gsum = 0.f, usum = 0.f;
      for (int w = 0; w < kWarps; ++w) { gsum += part[w * 16 + tid]; usum += part[w * 16 + 8 + tid]; }
      store_a(0, tid, gsum, usum);
    }
    __threadfence();   // the down kernel reads the shared expert's a before its own dependency wait
    it0 = 1;
  }

  // the router's logits are complete after the wait
  griddep_wait();
  griddep_launch_dependents();
  block_topk(p.logits + (size_t)t * (p.E + 1), p.E, k, p.has_shared, ts);
  load_slots(ts, k, p.E, p.experts, slot_ex, p.status);
  if (blockIdx.x == 0 && tid < k) {
    if (p.idx_out) p.idx_out[(size_t)t * k + tid] = ts.idx[tid];
    if (p.w_out) p.w_out[(size_t)t * k + tid] = ts.w[tid];
  }
  // routed items in waves of up to kGuBufs, each item on its own group of warps
  for (int w0 = it0; w0 < nitems; w0 += kGuBufs) {
    const int nw = nitems - w0 < kGuBufs ? nitems - w0 : kGuBufs;
    for (int i = 0; i < nw; ++i) arm(w0 + i);
    __syncthreads();   // slots loaded (first wave) / previous wave's buffers read
    if (lane == 0)
      for (int c = warp; c < 6 * nw; c += kWarps) issue(w0 + c / 6, c % 6);
    const int wi = warp * nw / kWarps;                       // this warp's item in the wave
    const int wf = (wi * kWarps + nw - 1) / nw;               // first warp of that item
    const int wc = ((wi + 1) * kWarps + nw - 1) / nw - wf;    // warps of that item
    const int it = w0 + wi, r = warp - wf;
    ok &= mbar_wait_bounded(&bars[it % kGuBufs], (unsigned)(it / kGuBufs) & 1u, p.wait_ns, p.status);
    float aa, ab;
    compute(it % kGuBufs, nspans * r / wc, nspans * (r + 1) / wc, aa, ab);
    __syncthreads();   // part of the previous wave is consumed
    if ((lane & 3) == 0) { part[warp * 16 + (lane >> 2)] = aa; part[warp * 16 + 8 + (lane >> 2)] = ab; }
    fence_proxy_async();
    __syncthreads();
    if (tid < nw * n) {
      const int iw = tid / n, i = tid - iw * n;
      const int f = (iw * kWarps + nw - 1) / nw, c = ((iw + 1) * kWarps + nw - 1) / nw - f;
      float gsum = 0.f, usum = 0.f;
      for (int w = f; w < f + c; ++w) { gsum += part[w * 16 + i]; usum += part[w * 16 + 8 + i]; }
      store_a(w0 + iw, i, gsum, usum);
    }
  }
  if (!ok) {   // a copy never landed: give the copies in flight one more bound before leaving
    for (int it = (nitems > kGuBufs ? nitems - kGuBufs : 0); it < nitems; ++it)
      mbar_wait_bounded(&bars[it % kGuBufs], (unsigned)(it / kGuBufs) & 1u, p.wait_ns, nullptr);
  }
}

// ------------------------------------------------------------------ down + weighted combine + residual
constexpr int kDnBufs = 4;      // expert row blocks staged per CTA
constexpr int kDnMaxRows = 32;  // hidden rows per CTA

struct DnLayout {
  int RB, SRB, SBR, GB, nsp, ng;
  size_t buf, btab, gs, part, yacc, wsl, slots, topk, bars, total;
};
__host__ __device__ inline DnLayout dn_layout(int I, int S, int bits) {
  DnLayout L;
  L.RB = I * bits / 8;
  L.SRB = I / 32;
  L.SBR = sb_region(kDnMaxRows, L.SRB);
  L.GB = (kDnMaxRows * L.RB + 2 * L.SBR + 127) & ~127;
  L.nsp = I / kSpan;
  L.ng = I / kGroup;
  const int nb = S < kDnBufs ? S : kDnBufs;
  size_t o = 0;
  L.buf = o; o += (size_t)nb * L.GB;
  L.btab = o; o += sizeof(uint2) * (size_t)S * L.nsp * kBtPerSpan;
  L.gs = o; o += sizeof(float) * 2 * (size_t)S * L.ng;     // per slot [2^-p_g | X_g]
  o = (o + 15) & ~(size_t)15;
  L.part = o; o += sizeof(float) * (size_t)nb * (kDnMaxRows / 16) * L.nsp * 16;
  L.yacc = o; o += sizeof(float) * kDnMaxRows;
  L.wsl = o; o += sizeof(float) * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.topk = o; o += sizeof(TopkSmem);
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
  const int h0 = (int)((long long)H * blockIdx.x / gridDim.x);
  const int n = (int)((long long)H * (blockIdx.x + 1) / gridDim.x) - h0;
  const int ntile = (n + 15) / 16;
  const int nitems = S;
  auto item_slot = [&](int it) { return p.has_shared ? (it == 0 ? S - 1 : it - 1) : it; };
  int pre;
  const unsigned sbw = sb_window(h0, n, L.SRB, pre);
  const unsigned item_bytes = (unsigned)n * L.RB + 2u * sbw;
  const int per = nsp * kBtPerSpan;
  const int ppart = (kDnMaxRows / 16) * nsp * 16;   // floats of part per item
  bool ok = true;

  auto issue = [&](int it, int c) {   // c = 0 codes, 1 scales, 2 biases
    const int b = it % nb;
    unsigned char* buf = bufs + (size_t)b * L.GB;
    const moe_qmat& m = slot_ex[item_slot(it)].down;
    fence_proxy_async();
    if (c == 0) {
      bulk_g2s(buf, (const char*)m.q + (size_t)h0 * L.RB, (unsigned)n * L.RB, &bars[b]);
    } else {
      const uint16_t* src = c == 1 ? m.scales : m.biases;
      bulk_g2s(buf + kDnMaxRows * L.RB + (c - 1) * L.SBR, (const char*)src + (((size_t)h0 * L.SRB) & ~(size_t)15),
               sbw, &bars[b]);
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
  // unit u = (tile, span) of item it: row sums to pt[u][16]
  auto unit = [&](int it, int u, float* pt) {
    const int b = it % nb, slot = item_slot(it);
    const unsigned char* buf = bufs + (size_t)b * L.GB;
    const int g = lane >> 2, tq = lane & 3;
    const int bl = bt_lane_index(lane);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int WB = QTraits<BITS>::kWordsPerThread * 4;
    const int tile = u / nsp, s = u - tile * nsp;
    const int r = tile * 16 + g;
    Frag<BITS> F;
    frag_codes<BITS>(F, buf + (size_t)r * L.RB + s * SB + tq * WB, buf + (size_t)(r + 8) * L.RB + s * SB + tq * WB);
    const unsigned char* sc = buf + kDnMaxRows * L.RB + pre + s * 4;
    F.sa = *(const uint32_t*)(sc + r * L.SRB);
    F.sb = *(const uint32_t*)(sc + (r + 8) * L.SRB);
    F.ba = *(const uint32_t*)(sc + L.SBR + r * L.SRB);
    F.bb = *(const uint32_t*)(sc + L.SBR + (r + 8) * L.SRB);
    int c[4];
    mma_frag<BITS>(F, btab + (size_t)slot * per + s * kBtPerSpan, bl, c);
    const float* gsl = gs + (size_t)slot * 2 * ng;
    float acc_a = 0.f, acc_b = 0.f;
    scale_frag_i(F.sa, F.sb, F.ba, F.bb, c, gsl, gsl + ng, s, tq, acc_a, acc_b);
    acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
    acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 1);
    acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 2);
    acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 2);
    if (tq == 0) { pt[u * 16 + g] = acc_a; pt[u * 16 + 8 + g] = acc_b; }
  };
  // items [i0, i1) (all staged): units spread over the warps, then yacc += w * y
  auto run = [&](int i0, int i1) {
    const int U = ntile * nsp, UT = (i1 - i0) * U;
    int waited = -1;
    for (int x = UT * warp / kWarps; x < UT * (warp + 1) / kWarps; ++x) {
      const int it = i0 + x / U;
      if (it != waited) {
        ok &= mbar_wait_bounded(&bars[it % nb], (unsigned)(it / nb) & 1u, p.wait_ns, p.status);
        waited = it;
      }
      unit(it, x - (it - i0) * U, part + (size_t)(it % nb) * ppart);
    }
    fence_proxy_async();
    __syncthreads();
    if (tid < n) {
      const int tile = tid >> 4, rr = tid & 15;
      float acc = yacc[tid];
      for (int it = i0; it < i1; ++it) {
        const float* pt = part + (size_t)(it % nb) * ppart;
        float y = 0.f;
        for (int s = 0; s < nsp; ++s) y += pt[(tile * nsp + s) * 16 + rr];
        acc = fmaf(wsl[item_slot(it)], y, acc);
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
  block_topk(p.logits + (size_t)t * (p.E + 1), p.E, k, p.has_shared, ts);
  load_slots(ts, k, p.E, p.experts, slot_ex, p.status);
  if (tid < k) wsl[tid] = ts.w[tid];
  if (tid == 0 && p.has_shared) wsl[S - 1] = ts.sg;
  if (tid < n) yacc[tid] = __ldcg(p.h + (size_t)t * H + h0 + tid);
  __syncthreads();
  if (lane == 0)
    for (int c = warp; c < 3 * nb; c += kWarps) issue(c / 3, c % 3);
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
      if (tid == 0)
        for (int it = issued; it < w1; ++it) mbar_expect_tx(&bars[it % nb], item_bytes);
      __syncthreads();
      if (lane == 0)
        for (int c = warp; c < 3 * (w1 - issued); c += kWarps) issue(issued + c / 3, c % 3);
      issued = w1;
    }
    run(w0, w1);
    __syncthreads();
  }
  if (tid < n) p.hacc[(size_t)t * H + h0 + tid] = yacc[tid];
  if (!ok) {
    for (int it = (nitems > nb ? nitems - nb : 0); it < nitems; ++it)
      mbar_wait_bounded(&bars[it % nb], (unsigned)(it / nb) & 1u, p.wait_ns, nullptr);
  }
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
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
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

}  // namespace qmoe
