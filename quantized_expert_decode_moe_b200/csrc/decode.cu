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

// ------------------------------------------------------------------ gate/up + SwiGLU
constexpr int kGuBufs = 2;      // expert tiles in flight per CTA
constexpr int kGuMaxRows = 8;   // intermediate rows per CTA

struct GuLayout {
  int RB, SRB, SBR, GB;   // code bytes per row, scale bytes per row, scale region, buffer bytes
  size_t buf, btab, gsc, gs, part, slots, topk, bars, total;
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
  L.gsc = o; o += sizeof(float) * (size_t)(H / kGroup);
  L.gs = o; o += sizeof(float) * 2 * (size_t)(H / kGroup);   // [2^-p_g | X_g]
  o = (o + 15) & ~(size_t)15;
  L.part = o; o += sizeof(float) * 2 * kWarps * 16;
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
// router CTA has passed its own wait, so x is final), then the k routed
// experts, which every CTA ranks itself from the router's logits.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 2) gateup_decode_kernel(GateUpParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GuLayout L = gu_layout(p.H, BITS);
  unsigned char* bufs = smem + L.buf;
  uint2* btab = (uint2*)(smem + L.btab);
  float* gsc = (float*)(smem + L.gsc);
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

  // the byte count of item `it` on its buffer's barrier (thread 0, before the
  // barrier that precedes the copies; the buffer's previous phase has completed)
  auto arm = [&](int it) {
    if (tid == 0 && n) mbar_expect_tx(&bars[it % kGuBufs], item_bytes);
  };
  // copies of item `it` into buffer it % kGuBufs: lane 0 of warps 0-5, one copy each
  auto issue = [&](int it) {
    if (lane != 0 || warp >= 6 || n == 0) return;
    const int b = it % kGuBufs;
    unsigned char* buf = bufs + (size_t)b * L.GB;
    const moe_expert& ex = slot_ex[item_slot(it)];
    fence_proxy_async();
    if (warp < 2) {
      const moe_qmat& m = warp == 0 ? ex.gate : ex.up;
      bulk_g2s(buf + (size_t)warp * kGuMaxRows * L.RB, (const char*)m.q + (size_t)j0 * L.RB, (unsigned)n * L.RB,
               &bars[b]);
    } else {
      const int w = warp - 2;   // 0 gate scales, 1 up scales, 2 gate biases, 3 up biases
      const moe_qmat& m = (w & 1) ? ex.up : ex.gate;
      const uint16_t* src = w < 2 ? m.scales : m.biases;
      bulk_g2s(buf + 2 * kGuMaxRows * L.RB + w * L.SBR, (const char*)src + (((size_t)j0 * L.SRB) & ~(size_t)15),
               sbw, &bars[b]);
    }
  };
  // MMAs of one item: warp w takes spans [nspans*w/16, nspans*(w+1)/16); row sums to pt[w][16]
  auto compute = [&](int b, float* pt) {
    const unsigned char* buf = bufs + (size_t)b * L.GB;
    const int g = lane >> 2, tq = lane & 3;
    const int bl = bt_lane_index(lane);
    const int s0 = nspans * warp / kWarps, s1 = nspans * (warp + 1) / kWarps;
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int WB = QTraits<BITS>::kWordsPerThread * 4;
    const unsigned char* ra = buf + (size_t)g * L.RB + tq * WB;
    const unsigned char* rb = buf + (size_t)(kGuMaxRows + g) * L.RB + tq * WB;
    const unsigned char* sc = buf + 2 * kGuMaxRows * L.RB + pre + g * L.SRB;
    float acc_a = 0.f, acc_b = 0.f;
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
    if (tq == 0) { pt[warp * 16 + g] = acc_a; pt[warp * 16 + 8 + g] = acc_b; }
  };
  auto finalize = [&](int it, const float* pt) {
    if (tid < n) {
      float gsum = 0.f, usum = 0.f;
      for (int w = 0; w < kWarps; ++w) { gsum += pt[w * 16 + tid]; usum += pt[w * 16 + 8 + tid]; }
      p.a[((size_t)t * S + item_slot(it)) * I + j0 + tid] = silu_f32(gsum) * usum;
    }
  };

  if (tid == 0) {
    for (int b = 0; b < kGuBufs; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    if (p.has_shared) slot_ex[S - 1] = p.shared;
  }
  if (p.has_shared) arm(0);
  __syncthreads();
  if (p.has_shared) issue(0);
  // activation -> fp32 (exact; staged in buffer 1, free until the routed copies), group prescales and sums,
  // B-fragment table
  float* xs = (float*)(bufs + (size_t)1 * L.GB);
  const uint4* xt = (const uint4*)(p.x + (size_t)t * H);
  for (int i = tid; i < H / 8; i += kThreads) {
    const uint4 v = __ldcg(xt + i);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) { xs[8 * i + 2 * q] = bf16lo(w4[q]); xs[8 * i + 2 * q + 1] = bf16hi(w4[q]); }
  }
  __syncthreads();
  group_stats(xs, ng, gsc, gs, gs + ng, warp, lane, kWarps);
  __syncthreads();
  for (int i = tid; i < nspans * kBtPerSpan; i += kThreads) btab[i] = btab_at<BITS>(xs, gsc, i);
  fence_proxy_async();   // buffer 1 (x staging) is refilled by bulk copies later
  __syncthreads();
  int it0 = 0;
  if (p.has_shared) {
    if (n) ok &= mbar_wait_bounded(&bars[0], 0, p.wait_ns, p.status);
    compute(0, part);
    fence_proxy_async();
    __syncthreads();
    finalize(0, part);
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
  for (int it = it0; it < nitems && it < it0 + kGuBufs; ++it) arm(it);
  __syncthreads();
  for (int it = it0; it < nitems && it < it0 + kGuBufs; ++it) issue(it);
  for (int it = it0; it < nitems; ++it) {
    const int b = it % kGuBufs;
    float* pt = part + (it & 1) * kWarps * 16;
    if (n) ok &= mbar_wait_bounded(&bars[b], (unsigned)(it / kGuBufs) & 1u, p.wait_ns, p.status);
    compute(b, pt);
    fence_proxy_async();
    if (it + kGuBufs < nitems) arm(it + kGuBufs);
    __syncthreads();
    if (it + kGuBufs < nitems) issue(it + kGuBufs);
    finalize(it, pt);
  }
  if (!ok) {   // a copy never landed: give the copies in flight one more bound before leaving
    for (int it = (nitems > kGuBufs ? nitems - kGuBufs : 0); it < nitems; ++it)
      if (n) mbar_wait_bounded(&bars[it % kGuBufs], (unsigned)(it / kGuBufs) & 1u, p.wait_ns, nullptr);
  }
}

// ------------------------------------------------------------------ down + weighted combine + residual
constexpr int kDnBufs = 4;      // expert row blocks staged per CTA
constexpr int kDnMaxRows = 32;  // hidden rows per CTA

struct DnLayout {
  int RB, SRB, SBR, GB, nsp, ng;
  size_t buf, as, btab, gsc, gs, part, yacc, wsl, slots, topk, bars, total;
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
  L.as = o; o += sizeof(float) * (size_t)S * I;
  L.btab = o; o += sizeof(uint2) * (size_t)S * L.nsp * kBtPerSpan;
  L.gsc = o; o += sizeof(float) * (size_t)S * L.ng;
  L.gs = o; o += sizeof(float) * 2 * (size_t)S * L.ng;
  o = (o + 15) & ~(size_t)15;
  L.part = o; o += sizeof(float) * 2 * (kDnMaxRows / 16) * L.nsp * 16;
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
// passed its dependency wait, so the router's logits and the residual h are
// final: before its own wait it ranks the logits and starts the copies of its
// rows of every chosen expert's down matrix. After the wait it turns a into
// per-expert B tables and forms hacc = h + sum_i w_i y_i + sg * y_shared for
// its rows.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 2) down_decode_kernel(DownParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int S = p.S;
  const DnLayout L = dn_layout(p.I, S, BITS);
  unsigned char* bufs = smem + L.buf;
  float* as = (float*)(smem + L.as);
  uint2* btab = (uint2*)(smem + L.btab);
  float* gsc = (float*)(smem + L.gsc);
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
  bool ok = true;

  if (tid == 0) {
    for (int b = 0; b < nb; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
    for (int b = 0; b < nb; ++b)
      if (n) mbar_expect_tx(&bars[b], item_bytes);   // items 0..nb-1
    if (p.has_shared) slot_ex[S - 1] = p.shared;
  }
  block_topk(p.logits + (size_t)t * (p.E + 1), p.E, k, p.has_shared, ts);
  load_slots(ts, k, p.E, p.experts, slot_ex, p.status);
  if (tid < k) wsl[tid] = ts.w[tid];
  if (tid == 0 && p.has_shared) wsl[S - 1] = ts.sg;
  if (tid < n) yacc[tid] = __ldcg(p.h + (size_t)t * H + h0 + tid);
  __syncthreads();

  auto issue = [&](int it) {   // lane 0 of warps 0-2, one copy each
    if (lane != 0 || warp >= 3 || n == 0) return;
    const int b = it % nb;
    unsigned char* buf = bufs + (size_t)b * L.GB;
    const moe_qmat& m = slot_ex[item_slot(it)].down;
    fence_proxy_async();
    if (warp == 0) {
      bulk_g2s(buf, (const char*)m.q + (size_t)h0 * L.RB, (unsigned)n * L.RB, &bars[b]);
    } else {
      const uint16_t* src = warp == 1 ? m.scales : m.biases;
      bulk_g2s(buf + kDnMaxRows * L.RB + (warp - 1) * L.SBR, (const char*)src + (((size_t)h0 * L.SRB) & ~(size_t)15),
               sbw, &bars[b]);
    }
  };
  for (int it = 0; it < nb; ++it) issue(it);

  griddep_wait();
  griddep_launch_dependents();
  // a = silu(g) * u of every slot -> per-slot group prescales, sums and B tables
  const float4* ag = (const float4*)(p.a + (size_t)t * S * I);
  for (int i = tid; i < S * I / 4; i += kThreads) ((float4*)as)[i] = __ldcg(ag + i);
  __syncthreads();
  group_stats(as, S * ng, gsc, gs, gs + S * ng, warp, lane, kWarps);   // [slot*ng + g]
  __syncthreads();
  const int per = nsp * kBtPerSpan;
  for (int i = tid; i < S * per; i += kThreads) {
    const int sl = i / per;
    btab[i] = btab_at<BITS>(as + (size_t)sl * I, gsc + (size_t)sl * ng, i - sl * per);
  }
  __syncthreads();

  // units of an item: (tile, span), warp w takes [U*w/16, U*(w+1)/16); row sums to pt[tile][span][16]
  const int U = ntile * nsp;
  auto compute = [&](int b, int slot, float* pt) {
    const unsigned char* buf = bufs + (size_t)b * L.GB;
    const int g = lane >> 2, tq = lane & 3;
    const int bl = bt_lane_index(lane);
    constexpr int SB = SpanBytes<BITS>::v;
    constexpr int WB = QTraits<BITS>::kWordsPerThread * 4;
    const uint2* bt = btab + (size_t)slot * per;
    const float* gsl = gs + (size_t)slot * ng;          // 2^-p_g of this slot
    const float* xgl = gs + (size_t)S * ng + (size_t)slot * ng;   // X_g of this slot
    for (int u = U * warp / kWarps; u < U * (warp + 1) / kWarps; ++u) {
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
      mma_frag<BITS>(F, bt + s * kBtPerSpan, bl, c);
      float acc_a = 0.f, acc_b = 0.f;
      scale_frag_i(F.sa, F.sb, F.ba, F.bb, c, gsl, xgl, s, tq, acc_a, acc_b);
      acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 1);
      acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 1);
      acc_a += __shfl_xor_sync(0xffffffffu, acc_a, 2);
      acc_b += __shfl_xor_sync(0xffffffffu, acc_b, 2);
      if (tq == 0) { pt[u * 16 + g] = acc_a; pt[u * 16 + 8 + g] = acc_b; }
    }
  };
  auto finalize = [&](int slot, const float* pt) {
    if (tid < n) {
      const int tile = tid >> 4, r = tid & 15;
      float y = 0.f;
      for (int s = 0; s < nsp; ++s) y += pt[(tile * nsp + s) * 16 + r];
      yacc[tid] = fmaf(wsl[slot], y, yacc[tid]);
    }
  };
  for (int it = 0; it < nitems; ++it) {
    const int b = it % nb, slot = item_slot(it);
    float* pt = part + (it & 1) * (kDnMaxRows / 16) * nsp * 16;
    if (n) ok &= mbar_wait_bounded(&bars[b], (unsigned)(it / nb) & 1u, p.wait_ns, p.status);
    compute(b, slot, pt);
    fence_proxy_async();
    if (tid == 0 && n && it + nb < nitems) mbar_expect_tx(&bars[b], item_bytes);
    __syncthreads();
    if (it + nb < nitems) issue(it + nb);
    finalize(slot, pt);
  }
  if (tid < n) p.hacc[(size_t)t * H + h0 + tid] = yacc[tid];
  if (!ok) {
    for (int it = (nitems > nb ? nitems - nb : 0); it < nitems; ++it)
      if (n) mbar_wait_bounded(&bars[it % nb], (unsigned)(it / nb) & 1u, p.wait_ns, nullptr);
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
