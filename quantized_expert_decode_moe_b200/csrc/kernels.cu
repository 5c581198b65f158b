// Decode-path kernels of the quantized MoE expert forward (sm_100a):
// router logits, top-k, expert gate/up and down dequant GEMVs, combine +
// residual + RMSNorm, standalone dequant GEMV, and the grouping of routed
// (token, rank) pairs by expert.
#include <math.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace qmoe {

static inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

WsLayout ws_layout(int H, int I, int E, int k, int S, int T) {
  WsLayout L{};
  size_t o = 0;
  L.status = o; o = align256(o + 256);
  L.logits = o; o = align256(o + sizeof(double) * (size_t)T * (E + 1));
  L.gu = o; o = align256(o + sizeof(float) * (size_t)T * S * 2 * I);
  L.y = o; o = align256(o + sizeof(float) * (size_t)T * S * H);
  L.w = o; o = align256(o + sizeof(float) * (size_t)T * k);
  L.sg = o; o = align256(o + sizeof(float) * (size_t)T);
  L.idx = o; o = align256(o + sizeof(int32_t) * (size_t)T * k);
  L.slots = o; o = align256(o + sizeof(moe_expert) * (size_t)T * kMaxSlots);
  L.counts = o; o = align256(o + sizeof(int32_t) * (size_t)E);
  L.offsets = o; o = align256(o + sizeof(int32_t) * (size_t)(E + 1));
  L.perm = o; o = align256(o + sizeof(int32_t) * (size_t)T * k);
  L.total = o;
  return L;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// CTA count for a split-unit kernel: every CTA range >= nspans units (a tile
// meets <= 2 CTAs) and every warp range <= nspans units (a warp meets <= 2 tiles).
int choose_ncta(long long ntiles, int nspans) {
  long long n = num_sms();
  if (n > ntiles) n = ntiles;
  const long long lo = (ntiles + kWarps - 1) / kWarps;
  if (n < lo) n = lo;
  if (n < 1) n = 1;
  return (int)n;
}

// ------------------------------------------------------------------ block reductions
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : 0.f;
  r = warp_max(r);
  return r;
}
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : 0.f;
  r = warp_sum(r);
  return r;
}

// ------------------------------------------------------------------ router logits
constexpr int kRouteWarps = 4;

// s + c += x with the rounding error of the addition kept in c (Knuth's TwoSum).
__device__ __forceinline__ void two_sum_acc(float& s, float& c, float x) {
  const float t = s + x;
  const float bp = t - s;
  c += (s - (t - bp)) + (x - bp);
  s = t;
}
// Dot product of 8 bf16 pairs accumulated as unevaluated sums s[i] + c[i]
// over 4 independent chains: each bf16 x bf16 product is exact in fp32 and
// every addition error is carried, so the sum of the chains holds the dot
// product to about 2^-44 relative to sum |w x|.
__device__ __forceinline__ void dot8_bf16_comp(uint4 w, uint4 x, float (&s)[4], float (&c)[4]) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w}, xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    two_sum_acc(s[i], c[i], bf16lo(wv[i]) * bf16lo(xv[i]));
    two_sum_acc(s[i], c[i], bf16hi(wv[i]) * bf16hi(xv[i]));
  }
}

__device__ void prefetch_expert_part(const moe_expert& ex, int H, int I, int bits, int part, int nparts) {
  const size_t qgu = (size_t)I * H * bits / 8, sgu = (size_t)I * (H / kGroup) * 2;
  const size_t qd = (size_t)H * I * bits / 8, sd = (size_t)H * (I / kGroup) * 2;
  prefetch_l2_part(ex.gate.q, qgu, part, nparts);
  prefetch_l2_part(ex.up.q, qgu, part, nparts);
  prefetch_l2_part(ex.gate.scales, sgu, part, nparts);
  prefetch_l2_part(ex.gate.biases, sgu, part, nparts);
  prefetch_l2_part(ex.up.scales, sgu, part, nparts);
  prefetch_l2_part(ex.up.biases, sgu, part, nparts);
  prefetch_l2_part(ex.down.q, qd, part, nparts);
  prefetch_l2_part(ex.down.scales, sd, part, nparts);
  prefetch_l2_part(ex.down.biases, sd, part, nparts);
}

// grid (ceil(rows / 4), T), block 128: one warp per router row (row E = shared gate).
// Each lane keeps all of its row chunks in flight (up to 16 x 16 bytes).
__global__ void __launch_bounds__(kRouteWarps * 32) route_logits_kernel(RouteParams p) {
  griddep_launch_dependents();
  extern __shared__ __align__(128) unsigned char smem[];
  uint4* xs = (uint4*)smem;   // [H/8]
  const int t = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = p.H / 8;
  const int nrows = p.E + (p.has_shared ? 1 : 0);
  const int e = blockIdx.x * kRouteWarps + warp;
  const uint16_t* wrow = e < p.E ? p.router_w + (size_t)e * p.H : p.gate_w;
  const uint4* xr = (const uint4*)(p.x + (size_t)t * p.H);
  constexpr int kChunks = 16;
  float cs[4] = {0.f, 0.f, 0.f, 0.f}, cc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int c0 = 0; c0 < nch; c0 += 32 * kChunks) {
    uint4 wv[kChunks];
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = c0 + lane + 32 * i;
      wv[i] = (e < nrows && c < nch) ? ldg_stream_v4(wrow + (size_t)c * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (c0 == 0) {
      for (int c = threadIdx.x; c < nch; c += blockDim.x) xs[c] = __ldcg(xr + c);
      if (t == 0) {
        if (p.zero_buf) {
          for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.zero_n; i += (size_t)gridDim.x * blockDim.x)
            p.zero_buf[i] = 0.f;
        }
        if (p.prefetch_shared && p.has_shared && threadIdx.x == 0)
          prefetch_expert_part(p.shared, p.H, p.I, p.bits, blockIdx.x, gridDim.x);
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
      const int c = c0 + lane + 32 * i;
      if (c < nch) dot8_bf16_comp(wv[i], xs[c], cs, cc);
    }
    __syncthreads();
  }
  if (e >= nrows) return;
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
  if (lane == 0) {
    double acc = (double)as_ + (double)ac_;
    if (e < p.E && p.router_bias) acc += (double)p.router_bias[e];
    p.logits[(size_t)t * (p.E + 1) + e] = acc;
  }
}

// ------------------------------------------------------------------ top-k (one CTA per token)
// k largest logits, descending, ties to the lower index; weights = softmax over
// all E renormalised over the chosen k = exp(l_i - l_max) / sum_chosen exp(l_j - l_max).
// Logits are compared through an order-preserving 64-bit integer key of their
// double bits (NaN ranks lowest). Each warp finds the top-k of its slice;
// warp 0 merges the candidates. Exact: every global top-k entry is in its
// slice's top-k.
struct TopkSmem {
  unsigned long long ck[kWarps * kMaxTopK];   // candidate keys
  int ce[kWarps * kMaxTopK];                  // candidate expert ids
  double cl[kWarps * kMaxTopK];               // candidate logits
  double chosen[kMaxTopK];
};

__device__ __forceinline__ unsigned long long order_key(double v) {
  if (isnan(v)) return 0ull;
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ bool better(unsigned long long k, int e, unsigned long long bk, int be) {
  return k > bk || (k == bk && e < be);
}
// warp-wide argmax of (key desc, id asc) with three warp reductions
__device__ __forceinline__ void warp_argmax(unsigned long long& bk, int& be) {
  const unsigned hi = (unsigned)(bk >> 32), lo = (unsigned)bk;
  const unsigned mh = __reduce_max_sync(0xffffffffu, hi);
  const unsigned ml = __reduce_max_sync(0xffffffffu, hi == mh ? lo : 0u);
  const bool cand = hi == mh && lo == ml;
  const unsigned me = __reduce_min_sync(0xffffffffu, cand ? (unsigned)be : 0xffffffffu);
  bk = ((unsigned long long)mh << 32) | ml;
  be = (int)me;
}

// All kThreads threads of the CTA take part. Thread tid holds logits
// e = tid + kThreads * i, i < PER. Results in idx_s / w_s.
template <int kTopkPer>
__device__ void block_topk_n(const double* lg, int E, int k, TopkSmem& ts, int32_t* idx_s, float* w_s) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kNone = 0x7fffffff;
  double lv[kTopkPer];
  int id[kTopkPer];
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) {
    const int e = tid + kThreads * i;
    lv[i] = e < E ? ldcg_f64(lg + e) : 0.0;
    id[i] = e < E ? e : kNone;
  }
  unsigned long long key[kTopkPer];
#pragma unroll
  for (int i = 0; i < kTopkPer; ++i) key[i] = order_key(lv[i]);
  for (int r = 0; r < k; ++r) {   // per-warp top-k of its values
    unsigned long long bk = 0ull;
    int be = kNone, bi = -1;
#pragma unroll
    for (int i = 0; i < kTopkPer; ++i)
      if (id[i] != kNone && better(key[i], id[i], bk, be)) { bk = key[i]; be = id[i]; bi = i; }
    unsigned long long wk = bk;
    int we = be;
    warp_argmax(wk, we);
    const bool mine = bi >= 0 && be == we && we != kNone;
#pragma unroll
    for (int i = 0; i < kTopkPer; ++i)
      if (mine && i == bi) {
        ts.cl[warp * k + r] = lv[i];
        id[i] = kNone;
      }
    if (lane == 0) { ts.ck[warp * k + r] = wk; ts.ce[warp * k + r] = we; }
  }
  __syncthreads();
  if (warp == 0) {   // merge the warps' candidates
    const int nc = kWarps * k;
    constexpr int kC = kWarps * kMaxTopK / 32;
    unsigned long long ck[kC];
    int ce[kC];
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      const int c = lane + 32 * i;
      ck[i] = c < nc ? ts.ck[c] : 0ull;
      ce[i] = c < nc ? ts.ce[c] : kNone;
    }
    for (int r = 0; r < k; ++r) {
      unsigned long long bk = 0ull;
      int be = kNone, bi = -1;
#pragma unroll
      for (int i = 0; i < kC; ++i)
        if (ce[i] != kNone && better(ck[i], ce[i], bk, be)) { bk = ck[i]; be = ce[i]; bi = i; }
      unsigned long long wk = bk;
      int we = be;
      warp_argmax(wk, we);
      if (bi >= 0 && be == we) {
#pragma unroll
        for (int i = 0; i < kC; ++i)
          if (i == bi) { ts.chosen[r] = ts.cl[lane + 32 * i]; ce[i] = kNone; }
        idx_s[r] = we;
      }
    }
    __syncwarp();
    if (lane == 0) {
      float ex[kMaxTopK];
      float z = 0.f;
      for (int r = 0; r < k; ++r) { ex[r] = expf((float)(ts.chosen[r] - ts.chosen[0])); z += ex[r]; }
      for (int r = 0; r < k; ++r) w_s[r] = ex[r] / z;
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void block_topk(const double* lg, int E, int k, TopkSmem& ts, int32_t* idx_s, float* w_s) {
  if (E <= kThreads) block_topk_n<1>(lg, E, k, ts, idx_s, w_s);
  else if (E <= 2 * kThreads) block_topk_n<2>(lg, E, k, ts, idx_s, w_s);
  else if (E <= 4 * kThreads) block_topk_n<4>(lg, E, k, ts, idx_s, w_s);
  else block_topk_n<8>(lg, E, k, ts, idx_s, w_s);
}

__device__ __forceinline__ float sigmoid_f64(double z) { return (float)(1.0 / (1.0 + exp(-z))); }

// grid T, block 512
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkParams p) {
  __shared__ TopkSmem ts;
  __shared__ int32_t idx_s[kMaxTopK];
  __shared__ float w_s[kMaxTopK];
  const int t = blockIdx.x, tid = threadIdx.x;
  const double* lg = p.logits + (size_t)t * (p.E + 1);
  block_topk(lg, p.E, p.k, ts, idx_s, w_s);
  if (tid < p.k) {
    p.idx[(size_t)t * p.k + tid] = idx_s[tid];
    p.w[(size_t)t * p.k + tid] = w_s[tid];
  }
  if (tid == 0 && p.sg) p.sg[t] = p.has_shared ? sigmoid_f64(ldcg_f64(lg + p.E)) : 0.f;
}

// ------------------------------------------------------------------ shared-memory layouts
// [B tables][group sums][...][unit slots: kWarps x kUnitSlots]; the slots are
// last and also hold the activation staging of the prologue.
template <int BITS>
__host__ __device__ inline size_t slots_bytes() { return (size_t)kWarps * kUnitSlots * UnitSmem<BITS>::bytes; }

struct GateUpSmem { size_t btab, xg, ts, ps, red, slots, idx, w, misc, buf, total; };
__host__ __device__ inline GateUpSmem gateup_smem(int H, int nspans, size_t slots) {
  GateUpSmem L{};
  size_t o = 0;
  L.btab = o; o += sizeof(uint2) * (size_t)nspans * kBtabPerSpan;
  L.xg = o; o += sizeof(float) * (size_t)(H / kGroup);
  o = (o + 15) & ~(size_t)15;
  L.ts = o; o += sizeof(TopkSmem);
  L.ps = o; o += sizeof(PartialSmem);
  L.red = o; o += sizeof(float) * 32;
  o = (o + 15) & ~(size_t)15;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  L.idx = o; o += sizeof(int32_t) * kMaxTopK;
  L.w = o; o += sizeof(float) * kMaxTopK;
  L.misc = o; o += sizeof(float) * 4;
  o = (o + 127) & ~(size_t)127;
  L.buf = o;
  const size_t xs = sizeof(float) * (size_t)H;
  o += slots > xs ? slots : xs;
  L.total = o;
  return L;
}

// ------------------------------------------------------------------ expert gate/up (decode)
// grid (nCTA, T), block 512. Units: (slot, tile of 8 intermediate rows, span);
// a tile is 16 MMA rows: rows 0-7 = gate rows j..j+7, rows 8-15 = up rows j..j+7.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) gateup_decode_kernel(GateUpParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GateUpSmem SL = gateup_smem(p.H, p.nspans, slots_bytes<BITS>());
  uint2* btab = (uint2*)(smem + SL.btab);
  float* Xg = (float*)(smem + SL.xg);
  TopkSmem& tsm = *(TopkSmem*)(smem + SL.ts);
  PartialSmem& ps = *(PartialSmem*)(smem + SL.ps);
  float* red = (float*)(smem + SL.red);
  moe_expert* slot_ex = (moe_expert*)(smem + SL.slots);
  int32_t* idx_s = (int32_t*)(smem + SL.idx);
  float* w_s = (float*)(smem + SL.w);
  float* misc = (float*)(smem + SL.misc);
  unsigned char* buf = smem + SL.buf;
  float* xs = (float*)buf;

  griddep_launch_dependents();
  const int t = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I;
  const Range cr = cta_range(p.U, blockIdx.x, p.nCTA);

  // 1) activation -> fp32, prescale, group sums, B-fragment table (independent of routing)
  const uint4* xt = (const uint4*)(p.x + (size_t)t * H);
  float amax = 0.f;
  for (int i0 = 0; i0 < H / 8; i0 += 2 * kThreads) {
    uint4 v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) v[u] = i0 + tid + u * kThreads < H / 8 ? __ldcg(xt + i0 + tid + u * kThreads) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + tid + u * kThreads;
      if (i < H / 8) {
        const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = bf16lo(w4[q]), b = bf16hi(w4[q]);
          xs[8 * i + 2 * q] = a; xs[8 * i + 2 * q + 1] = b;
          amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
        }
      }
    }
  }
  amax = block_max(amax, red);
  const float sc = prescale_for(amax);
  for (int i = tid; i < H; i += kThreads) xs[i] *= sc;
  __syncthreads();
  for (int gi = warp; gi < H / kGroup; gi += kWarps) {
    float v = xs[gi * kGroup + lane] + xs[gi * kGroup + 32 + lane];
    v = warp_sum(v);
    if (lane == 0) Xg[gi] = v;
  }
  for (int i = tid; i < p.nspans * kBtabPerSpan; i += kThreads)
    btab[i] = btab_entry<BITS>(xs, i >> 6, (i >> 3) & 7, i & 7);
  __syncthreads();   // xs is dead from here on: its space holds the unit slots

  // 2) routing decision of this token (needs the router kernel's logits)
  griddep_wait();
  const double* lg = p.logits + (size_t)t * (p.E + 1);
  if (tid == 0) misc[0] = p.has_shared ? sigmoid_f64(ldcg_f64(lg + p.E)) : 0.f;
  block_topk(lg, p.E, p.k, tsm, idx_s, w_s);
  if (tid < p.S) {
    if (tid < p.k) {
      int e = idx_s[tid];
      if (e < 0 || e >= p.E) { atomicExch(p.status, kStatusDeviceFault); e = 0; }
      slot_ex[tid] = p.experts[e];
    } else {
      slot_ex[tid] = p.shared;
    }
  }
  __syncthreads();

  // 3) publish the routing (CTA 0); hint the chosen experts' down weights into L2
  if (blockIdx.x == 0 && warp == kWarps - 1) {
    if (lane < p.k) {
      p.idx_ws[(size_t)t * p.k + lane] = idx_s[lane];
      p.w_ws[(size_t)t * p.k + lane] = w_s[lane];
      if (p.idx_out) p.idx_out[(size_t)t * p.k + lane] = idx_s[lane];
      if (p.w_out) p.w_out[(size_t)t * p.k + lane] = w_s[lane];
    }
    if (lane < p.S) p.slots_ws[(size_t)t * kMaxSlots + lane] = slot_ex[lane];
    if (lane == 0) p.sg_ws[t] = misc[0];
  }
  if (p.prefetch_down && warp == kWarps - 2 && lane < p.k) {
    const moe_expert& ex = slot_ex[lane];
    const size_t qd = (size_t)H * I * BITS / 8, sd = (size_t)H * (I / kGroup) * 2;
    prefetch_l2_part(ex.down.q, qd, blockIdx.x, p.nCTA);
    prefetch_l2_part(ex.down.scales, sd, blockIdx.x, p.nCTA);
    prefetch_l2_part(ex.down.biases, sd, blockIdx.x, p.nCTA);
  }

  // 4) dequant MMAs over this warp's units (staged with cp.async)
  const size_t wpr = (size_t)H * BITS / 32, gpr = (size_t)H / kGroup;
  const Range wr = warp_range(cr, warp);
  auto row = [&](int tile, int r) {
    const moe_expert& ex = slot_ex[tile / p.ntiles];
    const moe_qmat& m = r < 8 ? ex.gate : ex.up;
    const size_t j = (size_t)(tile % p.ntiles) * 8 + (r & 7);
    return RowSrc{m.q + j * wpr, m.scales + j * gpr, m.biases + j * gpr};
  };
  auto bt_of = [&](int) -> const uint2* { return btab; };
  auto xg_of = [&](int) -> const float* { return Xg; };
  run_units<BITS>(wr, p.nspans, buf + (size_t)warp * kUnitSlots * UnitSmem<BITS>::bytes, row, bt_of, xg_of, ps,
                  warp, lane);
  __syncthreads();
  const float inv = 1.f / sc;
  float* gu = p.gu + (size_t)t * p.S * 2 * I;
  reduce_partials(cr, p.nspans, ps, [&](int tile, int r, float v) {
    const int slot = tile / p.ntiles;
    const int j = (tile % p.ntiles) * 8 + (r & 7);
    atomicAdd(gu + ((size_t)slot * 2 + (r >> 3)) * I + j, v * inv);
  });
}

// ------------------------------------------------------------------ expert down (decode)
struct DownSmem { size_t btab, xg, ps, red, slots, sc, amax, buf, total; };
__host__ __device__ inline DownSmem down_smem(int I, int nspans, int nslots, size_t slots) {
  DownSmem L{};
  size_t o = 0;
  L.btab = o; o += sizeof(uint2) * (size_t)nspans * kBtabPerSpan * nslots;
  L.xg = o; o += sizeof(float) * (size_t)(I / kGroup) * nslots;
  o = (o + 15) & ~(size_t)15;
  L.ps = o; o += sizeof(PartialSmem);
  L.red = o; o += sizeof(float) * 32 * kMaxSlots;
  o = (o + 15) & ~(size_t)15;
  L.slots = o; o += sizeof(moe_expert) * kMaxSlots;
  L.sc = o; o += sizeof(float) * kMaxSlots;
  L.amax = o; o += sizeof(float) * kMaxSlots;
  o = (o + 127) & ~(size_t)127;
  L.buf = o;
  const size_t as = sizeof(float) * (size_t)I * nslots;   // activations of the CTA's slots (prologue only)
  o += slots > as ? slots : as;
  L.total = o;
  return L;
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.f + expf(-z)); }

// grid (nCTA, T), block 512. Units: (slot, tile of 16 output rows, span over I).
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) down_decode_kernel(DownParams p, int max_slots) {
  extern __shared__ __align__(128) unsigned char smem[];
  const DownSmem SL = down_smem(p.I, p.nspans, max_slots, slots_bytes<BITS>());
  uint2* btab = (uint2*)(smem + SL.btab);
  float* Xg = (float*)(smem + SL.xg);
  PartialSmem& ps = *(PartialSmem*)(smem + SL.ps);
  float* red = (float*)(smem + SL.red);
  moe_expert* slot_ex = (moe_expert*)(smem + SL.slots);
  float* scs = (float*)(smem + SL.sc);
  float* amx = (float*)(smem + SL.amax);
  unsigned char* buf = smem + SL.buf;
  float* as = (float*)buf;

  griddep_launch_dependents();
  const int t = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I;
  const Range cr = cta_range(p.U, blockIdx.x, p.nCTA);
  const int per_slot = p.ntiles * p.nspans;
  const int slot_lo = cr.a < cr.b ? cr.a / per_slot : 0;
  const int nsl = cr.a < cr.b ? (cr.b - 1) / per_slot - slot_lo + 1 : 0;

  griddep_wait();
  if (tid < p.S) {   // chosen experts as published by the gate/up kernel
    const unsigned long long* s8 = (const unsigned long long*)(p.slots_ws + (size_t)t * kMaxSlots + tid);
    unsigned long long* d8 = (unsigned long long*)(slot_ex + tid);
#pragma unroll
    for (int q = 0; q < (int)(sizeof(moe_expert) / 8); ++q) d8[q] = __ldcg(s8 + q);
  }
  // a = silu(g) * u for every slot of this CTA, all loads in flight at once
  const float* gu = p.gu + (size_t)t * p.S * 2 * I;
  const int nq = I / 4;                         // float4 per slot vector
  float am[kMaxSlots];
#pragma unroll
  for (int q = 0; q < kMaxSlots; ++q) am[q] = 0.f;
  for (int i = tid; i < nsl * nq; i += kThreads) {
    const int li = i / nq, e4 = (i % nq) * 4, sl = slot_lo + li;
    const float4 gv = __ldcg((const float4*)(gu + (size_t)sl * 2 * I + e4));
    const float4 uv = __ldcg((const float4*)(gu + ((size_t)sl * 2 + 1) * I + e4));
    const float a0 = silu_f32(gv.x) * uv.x, a1 = silu_f32(gv.y) * uv.y;
    const float a2 = silu_f32(gv.z) * uv.z, a3 = silu_f32(gv.w) * uv.w;
    float* d = as + (size_t)li * I + e4;
    d[0] = a0; d[1] = a1; d[2] = a2; d[3] = a3;
    const float m = fmaxf(fmaxf(fabsf(a0), fabsf(a1)), fmaxf(fabsf(a2), fabsf(a3)));
#pragma unroll
    for (int q = 0; q < kMaxSlots; ++q) if (q == li) am[q] = fmaxf(am[q], m);
  }
#pragma unroll
  for (int q = 0; q < kMaxSlots; ++q) {
    if (q >= nsl) break;
    const float v = warp_max(am[q]);
    if (lane == 0) red[q * 32 + warp] = v;
  }
  __syncthreads();
  if (tid < nsl) {
    float m = 0.f;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[tid * 32 + w]);
    scs[tid] = prescale_for(m);
  }
  __syncthreads();
  for (int i = tid; i < nsl * I; i += kThreads) as[i] *= scs[i / I];
  __syncthreads();
  for (int gi = warp; gi < nsl * (I / kGroup); gi += kWarps) {
    float v = as[gi * kGroup + lane] + as[gi * kGroup + 32 + lane];
    v = warp_sum(v);
    if (lane == 0) Xg[gi] = v;
  }
  const int per = p.nspans * kBtabPerSpan;
  for (int i = tid; i < nsl * per; i += kThreads) {
    const int li = i / per, j = i % per;
    btab[i] = btab_entry<BITS>(as + (size_t)li * I, j >> 6, (j >> 3) & 7, j & 7);
  }
  __syncthreads();   // activations are dead: their space holds the unit slots

  const size_t wpr = (size_t)I * BITS / 32, gpr = (size_t)I / kGroup;
  const Range wr = warp_range(cr, warp);
  auto row = [&](int tile, int r) {
    const moe_qmat& m = slot_ex[tile / p.ntiles].down;
    const size_t rr = (size_t)(tile % p.ntiles) * 16 + r;
    return RowSrc{m.q + rr * wpr, m.scales + rr * gpr, m.biases + rr * gpr};
  };
  auto bt_of = [&](int tile) -> const uint2* { return btab + (size_t)(tile / p.ntiles - slot_lo) * per; };
  auto xg_of = [&](int tile) -> const float* { return Xg + (size_t)(tile / p.ntiles - slot_lo) * (I / kGroup); };
  run_units<BITS>(wr, p.nspans, buf + (size_t)warp * kUnitSlots * UnitSmem<BITS>::bytes, row, bt_of, xg_of, ps,
                  warp, lane);
  __syncthreads();
  float* y = p.y + (size_t)t * p.S * H;
  reduce_partials(cr, p.nspans, ps, [&](int tile, int r, float v) {
    const int slot = tile / p.ntiles;
    atomicAdd(y + (size_t)slot * H + (size_t)(tile % p.ntiles) * 16 + r, v / scs[slot - slot_lo]);
  });
  (void)amx;
}

// ------------------------------------------------------------------ combine + residual + RMSNorm
// One thread-block cluster of kNormCluster CTAs per token: CTA r combines the
// elements [r*H/8, (r+1)*H/8) of h' = h + sum_i w_i y_i + sg * y_s, the CTAs
// exchange their partial sums of squares through distributed shared memory,
// and each normalises its slice. Spreads the token's ~(k+2)*4*H bytes of
// loads over 8 SMs.
constexpr int kNormCluster = 8;
constexpr int kNormCThreads = 256;
constexpr int kNormCPer = 4;      // elements per thread (H <= 8192)

__global__ void __cluster_dims__(kNormCluster, 1, 1) __launch_bounds__(kNormCThreads)
norm_cluster_kernel(NormParams p) {
  __shared__ float red[kNormCThreads / 32];
  __shared__ float parts[kNormCluster];   // partial sums of squares, written by every CTA of the cluster
  __shared__ float wsh[kMaxSlots];
  cg::cluster_group cluster = cg::this_cluster();
  const int r = (int)cluster.block_rank();
  const int t = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();
  griddep_launch_dependents();
  const int per = p.H / kNormCluster;
  const int j0 = r * per;
  if (tid < p.k) wsh[tid] = ldcg_f32(p.w + (size_t)t * p.k + tid);
  if (tid == 0) wsh[kMaxSlots - 1] = p.y_shared ? ldcg_f32(p.sg + t) : 0.f;
  const float* yr = p.y_routed + (size_t)t * p.y_routed_tok_stride;
  const float* ysh = p.y_shared ? p.y_shared + (size_t)t * p.y_shared_tok_stride : nullptr;
  float* h = p.h + (size_t)t * p.H;
  float hv[kNormCPer], yv[kNormCPer][kMaxSlots];
#pragma unroll
  for (int u = 0; u < kNormCPer; ++u) {
    const int jj = tid + kNormCThreads * u;
    const bool in = jj < per;
    const int j = j0 + jj;
    hv[u] = in ? h[j] : 0.f;
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) yv[u][i] = (in && i < p.k) ? ldcg_f32(yr + (size_t)i * p.y_routed_slot_stride + j) : 0.f;
    yv[u][kMaxSlots - 1] = (in && ysh) ? ldcg_f32(ysh + j) : 0.f;
  }
  __syncthreads();
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kNormCPer; ++u) {
    float v = hv[u];
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i)
      if (i < p.k) v = fmaf(wsh[i], yv[u][i], v);
    if (ysh) v = fmaf(wsh[kMaxSlots - 1], yv[u][kMaxSlots - 1], v);
    hv[u] = v;
    if (tid + kNormCThreads * u < per) ss = fmaf(v, v, ss);
  }
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (tid < kNormCluster) {   // push this CTA's partial into slot r of every CTA of the cluster
    float s2 = 0.f;
    for (int w = 0; w < kNormCThreads / 32; ++w) s2 += red[w];
    *cluster.map_shared_rank(&parts[r], tid) = s2;
  }
  cluster.sync();   // after this, nobody touches another CTA's shared memory
  float tot = 0.f;
#pragma unroll
  for (int q = 0; q < kNormCluster; ++q) tot += parts[q];
  const float inv = 1.f / sqrtf(tot / (float)p.H + p.eps);
#pragma unroll
  for (int u = 0; u < kNormCPer; ++u) {
    const int jj = tid + kNormCThreads * u;
    if (jj < per) {
      const int j = j0 + jj;
      h[j] = hv[u];
      const float xo = hv[u] * inv * bf16_to_f32(p.gamma[j]);
      p.x_out[(size_t)t * p.H + j] = f32_to_bf16(xo);
      if (p.x_out_f32) p.x_out_f32[(size_t)t * p.H + j] = xo;
    }
  }
}

// ------------------------------------------------------------------ standalone dequant GEMV
struct GemvSmem { size_t btab, xg, ps, red, buf, total; };
__host__ __device__ inline GemvSmem gemv_smem(int K, int nspans, size_t slots) {
  GemvSmem L{};
  size_t o = 0;
  L.btab = o; o += sizeof(uint2) * (size_t)nspans * kBtabPerSpan;
  L.xg = o; o += sizeof(float) * (size_t)(K / kGroup);
  o = (o + 15) & ~(size_t)15;
  L.ps = o; o += sizeof(PartialSmem);
  L.red = o; o += sizeof(float) * 32;
  o = (o + 127) & ~(size_t)127;
  L.buf = o;
  const size_t xs = sizeof(float) * (size_t)K;
  o += slots > xs ? slots : xs;
  L.total = o;
  return L;
}

// grid nCTA, block 512. Units: (tile of 16 rows, span).
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GemvParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GemvSmem SL = gemv_smem(p.K, p.nspans, slots_bytes<BITS>());
  uint2* btab = (uint2*)(smem + SL.btab);
  float* Xg = (float*)(smem + SL.xg);
  PartialSmem& ps = *(PartialSmem*)(smem + SL.ps);
  float* red = (float*)(smem + SL.red);
  unsigned char* buf = smem + SL.buf;
  float* xs = (float*)buf;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Range cr = cta_range(p.U, blockIdx.x, p.nCTA);
  const size_t wpr = (size_t)p.K * BITS / 32, gpr = (size_t)p.K / kGroup;
  float amax = 0.f;
  for (int i = tid; i < p.K; i += kThreads) { const float v = p.x[i]; xs[i] = v; amax = fmaxf(amax, fabsf(v)); }
  amax = block_max(amax, red);
  const float sc = prescale_for(amax);
  for (int i = tid; i < p.K; i += kThreads) xs[i] *= sc;
  __syncthreads();
  for (int gi = warp; gi < p.K / kGroup; gi += kWarps) {
    float v = xs[gi * kGroup + lane] + xs[gi * kGroup + 32 + lane];
    v = warp_sum(v);
    if (lane == 0) Xg[gi] = v;
  }
  for (int i = tid; i < p.nspans * kBtabPerSpan; i += kThreads) btab[i] = btab_entry<BITS>(xs, i >> 6, (i >> 3) & 7, i & 7);
  __syncthreads();
  const Range wr = warp_range(cr, warp);
  auto row = [&](int tile, int r) {
    const size_t rr = (size_t)tile * 16 + r;
    return RowSrc{p.W.q + rr * wpr, p.W.scales + rr * gpr, p.W.biases + rr * gpr};
  };
  auto bt_of = [&](int) -> const uint2* { return btab; };
  auto xg_of = [&](int) -> const float* { return Xg; };
  run_units<BITS>(wr, p.nspans, buf + (size_t)warp * kUnitSlots * UnitSmem<BITS>::bytes, row, bt_of, xg_of, ps,
                  warp, lane);
  __syncthreads();
  const float inv = 1.f / sc;
  reduce_partials(cr, p.nspans, ps, [&](int tile, int r, float v) {
    atomicAdd(p.y + (size_t)tile * 16 + r, v * inv);
  });
}

// ------------------------------------------------------------------ grouping by expert
// One CTA: histogram, exclusive scan, then a stable scatter by one warp that
// walks the pairs in order 32 at a time (ranks of equal experts inside a chunk
// from __match_any_sync).
__global__ void __launch_bounds__(1024) group_kernel(GroupParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  int* cnt = (int*)smem;            // [E]
  int* fill = cnt + p.E;            // [E]
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int N = p.T * p.k;
  for (int e = tid; e < p.E; e += blockDim.x) { cnt[e] = 0; fill[e] = 0; }
  __syncthreads();
  for (int i = tid; i < N; i += blockDim.x) {
    const int e = p.idx[i];
    if (e >= 0 && e < p.E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // exclusive scan of cnt into fill (blockDim-wide chunks)
  int carry = 0;
  for (int base = 0; base < p.E; base += blockDim.x) {
    const int e = base + tid;
    const int v = e < p.E ? cnt[e] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int nw = blockDim.x >> 5;
      int wv = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, wv, o);
        if (lane >= o) wv += n;
      }
      if (lane < nw) warp_tot[lane] = wv;
    }
    __syncthreads();
    const int wbase = warp ? warp_tot[warp - 1] : 0;
    const int excl = carry + wbase + incl - v;
    if (e < p.E) {
      fill[e] = excl;
      p.counts[e] = v;
      p.offsets[e] = excl;
    }
    const int tot = warp_tot[(blockDim.x >> 5) - 1];
    __syncthreads();
    carry += tot;
  }
  if (tid == 0) p.offsets[p.E] = carry;
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
static cudaError_t launch_ex(const void* fn, dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, void** args) {
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

// Every kernel prefers the maximum shared-memory carveout, so an SM never has
// to be drained to change its L1/shared split between kernels of a chain
// (a dependent kernel can then start next to its predecessor).
static cudaError_t set_smem(const void* fn, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_route(const RouteParams& p, cudaStream_t s) {
  const int rows = p.E + (p.has_shared ? 1 : 0);
  dim3 grid((rows + kRouteWarps - 1) / kRouteWarps, p.T);
  RouteParams q = p;
  void* args[] = {&q};
  const size_t sm = sizeof(uint16_t) * (size_t)p.H;
  cudaError_t e = set_smem((const void*)route_logits_kernel, sm);
  if (e != cudaSuccess) return e;
  return launch_ex((const void*)route_logits_kernel, grid, dim3(kRouteWarps * 32), sm, s, false, args);
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s) {
  cudaError_t e = set_smem((const void*)topk_kernel, 0);
  if (e != cudaSuccess) return e;
  TopkParams q = p;
  void* args[] = {&q};
  return launch_ex((const void*)topk_kernel, dim3(p.T), dim3(kThreads), 0, s, false, args);
}

static int smem_optin() {
  static int v = 0;
  if (!v) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (v <= 0) v = 227 * 1024;
  }
  return v;
}

cudaError_t launch_gateup(const GateUpParams& p, int bits, int T, bool pdl, cudaStream_t s) {
  GateUpParams q = p;
  const size_t sm = gateup_smem(p.H, p.nspans, bits == 4 ? slots_bytes<4>() : slots_bytes<2>()).total;
  if (sm > (size_t)smem_optin()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)gateup_decode_kernel<4> : (const void*)gateup_decode_kernel<2>;
  cudaError_t e = set_smem(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  return launch_ex(fn, dim3(p.nCTA, T), dim3(kThreads), sm, s, pdl, args);
}

cudaError_t launch_down(const DownParams& p, int bits, int T, bool pdl, cudaStream_t s) {
  const long long per_slot = (long long)p.ntiles * p.nspans;
  const long long maxr = (p.U + p.nCTA - 1) / p.nCTA;
  int max_slots = (int)((maxr + per_slot - 1) / per_slot) + 1;
  if (max_slots > p.S) max_slots = p.S;
  DownParams q = p;
  const size_t sm = down_smem(p.I, p.nspans, max_slots, bits == 4 ? slots_bytes<4>() : slots_bytes<2>()).total;
  if (sm > (size_t)smem_optin()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)down_decode_kernel<4> : (const void*)down_decode_kernel<2>;
  cudaError_t e = set_smem(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q, &max_slots};
  return launch_ex(fn, dim3(p.nCTA, T), dim3(kThreads), sm, s, pdl, args);
}

cudaError_t launch_norm(const NormParams& p, bool pdl, cudaStream_t s) {
  cudaError_t e = set_smem((const void*)norm_cluster_kernel, 0);
  if (e != cudaSuccess) return e;
  NormParams q = p;
  void* args[] = {&q};
  return launch_ex((const void*)norm_cluster_kernel, dim3(kNormCluster, p.T), dim3(kNormCThreads), 0, s, pdl, args);
}

cudaError_t launch_gemv(const GemvParams& p, int bits, cudaStream_t s) {
  GemvParams q = p;
  const size_t sm = gemv_smem(p.K, p.nspans, bits == 4 ? slots_bytes<4>() : slots_bytes<2>()).total;
  if (sm > (size_t)smem_optin()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)gemv_kernel<4> : (const void*)gemv_kernel<2>;
  cudaError_t e = set_smem(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  return launch_ex(fn, dim3(p.nCTA), dim3(kThreads), sm, s, false, args);
}

cudaError_t launch_group(const GroupParams& p, cudaStream_t s) {
  const size_t sm = sizeof(int) * 2 * (size_t)p.E;
  cudaError_t e = set_smem((const void*)group_kernel, sm);
  if (e != cudaSuccess) return e;
  GroupParams q = p;
  void* args[] = {&q};
  return launch_ex((const void*)group_kernel, dim3(1), dim3(1024), sm, s, false, args);
}

}  // namespace qmoe
