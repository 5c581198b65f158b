// Top-k routing shared by the decode kernels and moe_route (sm_100a).
//
// Router ("router results" choose the experts, Hacker News thread on
// Flash-MoE, the comment on Table 3; softmax over all experts renormalised
// over the chosen k, Flash-MoE write-up summary, "Model architecture"): the k
// largest logits, descending, ties to the lower index; weights = exp(l_i -
// l_max) / sum over the chosen of exp(l_j - l_max); shared gate =
// sigmoid(logit of the shared-gate row).
//
// The logits that define the ranking are the plain fp64 ones: every bf16 x
// bf16 product is exact in fp64 and the products are summed in index order,
// then the bias is added. The decode router computes each logit faster (fp64
// over a summation tree instead of index order) together with a rigorous
// bound b_e on |fast - definition|. Selection runs on the fast values and is then
// certified with beta = max_e b_e: when consecutive selected logits, down to
// the (k+1)-th, are more than 2 beta apart, the definition's top k and their
// order are the same. Otherwise every expert whose fast logit is within
// 2 beta of the k-th (a set that contains the true top k) is recomputed
// exactly as the definition's index-order fp64 sum, and the selection runs
// again on those exact values.
#pragma once

#include "common.cuh"

namespace qmoe {

constexpr int kTopkPer = 8;   // logits per thread at most: E <= kTopkPer * blockDim

struct TopkSmem {
  unsigned long long ck[kWarps * (kMaxTopK + 1)];   // each warp's best keys, [warp][round]
  int ce[kWarps * (kMaxTopK + 1)];                  // their expert ids
  unsigned wb[kWarps];                              // each warp's largest bound (float bits)
  double thr;                                       // recheck threshold: k-th logit - 2 beta
  int sure;                                         // the fast selection is certified
  int idx[kMaxTopK + 1];                      // the selected, best first (one past k when certifying)
  float w[kMaxTopK];
  double lsel[kMaxTopK + 1];                  // their logits (the values ranked on)
  float sg;
  int rechecked;                              // the exact recheck ran
};

// What an exact recheck of a logit reads: the token's activations (global or
// shared memory), the router rows and the optional per-expert bias.
struct RouterRef {
  const uint16_t* x;       // bf16 [H]
  const uint16_t* w;       // bf16 [E][H]
  const float* bias;       // [E] or null
  int H;
};

// The definition's logit: sum over h in index order of the exact fp64
// products w[e][h] * x[h], then + bias[e].
static __device__ __noinline__ double exact_logit(const RouterRef& r, int e) {
  const uint4* wr = (const uint4*)(r.w + (size_t)e * r.H);
  const uint4* xr = (const uint4*)r.x;
  double acc = 0.0;
  for (int c = 0; c < r.H / 8; ++c) {
    const uint4 wv = __ldg(wr + c), xv = xr[c];
    const uint32_t wa[4] = {wv.x, wv.y, wv.z, wv.w}, xa[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = __dadd_rn(acc, __dmul_rn((double)bf16lo(wa[i]), (double)bf16lo(xa[i])));
      acc = __dadd_rn(acc, __dmul_rn((double)bf16hi(wa[i]), (double)bf16hi(xa[i])));
    }
  }
  if (r.bias) acc = __dadd_rn(acc, (double)r.bias[e]);
  return acc;
}

// Dot product of 8 bf16 pairs for the router: each bf16 x bf16 product is
// exact in fp32 (bf16 has 8 significant bits); it is converted to fp64
// (exactly) and added into one of two fp64 chains; sum |w x| goes to a (fp32).
__device__ __forceinline__ void dot8_bf16_f64(uint4 w, uint4 x, double (&acc)[2], float& a) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w}, xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float p0 = bf16lo(wv[i]) * bf16lo(xv[i]), p1 = bf16hi(wv[i]) * bf16hi(xv[i]);
    acc[0] += (double)p0;
    acc[1] += (double)p1;
    a += fabsf(p0) + fabsf(p1);
  }
}

// Bound on |fast logit - definition| for a logit of n products summed in
// fp64 in any order (a summation tree), given sa = the fp32 sum of |w x|
// over the n products, the fast logit acc (bias included) and the bias.
// With u = 2^-53 and S = sum |w x|:
//  - any summation tree of n exact terms is within (n-1) u / (1 - (n-1) u) S
//    of the exact sum (Higham, Accuracy and Stability of Numerical
//    Algorithms, sec. 4.2), and so is the definition's index-order sum;
//  - the roundings of "+ bias" on both sides are within u (|acc| + |bias|)
//    each (with room to spare);
//  - an fp32 product below 2^-126 in magnitude loses at most 2^-150 (the
//    definition forms the products in fp64);
//  - sa underestimates S by at most a factor 1 - n 2^-24 (n <= 8192).
// The margins 1.25 and 2^-50 cover the last point and the rounding of the
// bound itself; the result is rounded up to fp32.
__device__ __forceinline__ float logit_bound(int n, float sa, double acc, double bias) {
  const double nn = (double)n;
  const double b = 1.25 * 2.0 * (nn + 2.0) * 0x1p-53 * (double)sa + 0x1p-50 * (fabs(acc) + fabs(bias)) +
                   nn * 0x1p-148;
  return __double2float_ru(b);
}

// Order-preserving 64-bit key of a double (key 0 = NaN or not a candidate, ranks lowest).
__device__ __forceinline__ unsigned long long order_key(double v) {
  if (isnan(v)) return 0ull;
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(unsigned long long k) {
  const unsigned long long u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double((long long)u);
}

// Warp-wide best of (key desc, id asc) over the lanes' (key, id); returns the
// winning lane (uniform) and the winner's key and id in wk, wi.
__device__ __forceinline__ int warp_best(unsigned long long key, int id, unsigned long long& wk, int& wi) {
  const unsigned full = 0xffffffffu;
  const unsigned hi = (unsigned)(key >> 32), lo = (unsigned)key;
  const unsigned mh = __reduce_max_sync(full, hi);
  bool c = hi == mh;
  unsigned bal = __ballot_sync(full, c);
  if (bal & (bal - 1)) {   // several lanes share the high half
    const unsigned ml = __reduce_max_sync(full, c ? lo : 0u);
    c = c && lo == ml;
    bal = __ballot_sync(full, c);
    if (bal & (bal - 1)) {   // equal keys: lowest id
      const unsigned mi = __reduce_min_sync(full, c ? (unsigned)id : 0xffffffffu);
      c = c && (unsigned)id == mi;
      bal = __ballot_sync(full, c);
    }
  }
  const int wl = __ffs(bal) - 1;
  wk = ((unsigned long long)mh << 32) | __shfl_sync(full, lo, wl);
  wi = __shfl_sync(full, id, wl);
  return wl;
}

// Block-wide top-k of lg[0..E) (+ shared gate from lg[E] when has_shared),
// global memory written by an earlier kernel or CTA (read through L2).
// bnd: per-logit error bounds of fast logits, or null when lg already holds
// the definition's values. All threads of the block call it (blockDim =
// 32 * kWarps); results in ts (idx, w, sg), valid after the call, which ends
// with __syncthreads. Ids of missing entries (fewer than k logits that are
// not NaN) are -1. k <= 8, E <= kTopkPer * blockDim.
//
// Thread tid holds the order keys of e = tid + j * blockDim (j < PER); a key
// encodes its logit (key_value); 0 = not a candidate (NaN, or past E). Every
// warp selects its own best n = k + 1 (k without bounds) by rounds of a warp
// argmax of (key desc, id asc), with no block barrier; lane 0 stores them
// with the warp's largest bound. After one __syncthreads, warp 0 merges the
// warps' lists (each sorted best first) into the block's best n (exact:
// each of the block's best n is among its warp's best n) and certifies them
// against beta = the
// token's largest bound: the top k and their order are those of the
// definition when consecutive selected logits, down to the (k+1)-th, are more
// than 2 beta apart. Otherwise (rare) every expert within 2 beta of the k-th
// and the selected are recomputed exactly and the selection runs again.
template <int PER>
__device__ __forceinline__ void topk_warp_candidates(unsigned long long (&key)[PER], int n, int nt,
                                                     TopkSmem& ts, unsigned bmax_bits) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#pragma unroll 1
  for (int r = 0; r < n; ++r) {
    unsigned long long bk = 0ull;
    int bj = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (key[j] > bk) { bk = key[j]; bj = j; }
    unsigned long long wk;
    int wi;
    const int wl = warp_best(bk, tid + bj * nt, wk, wi);
    if (lane == wl && wk) {
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (j == bj) key[j] = 0ull;
    }
    if (lane == 0) { ts.ck[warp * (kMaxTopK + 1) + r] = wk; ts.ce[warp * (kMaxTopK + 1) + r] = wk ? wi : -1; }
  }
  if (lane == 0) ts.wb[warp] = bmax_bits;
}

template <int PER>
static __device__ __noinline__ void block_topk_per(const double* lg, const float* bnd, int E, int k, int has_shared,
                                                   const RouterRef& rr, TopkSmem& ts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nt = blockDim.x, nw = nt >> 5;
  const int n = bnd && k < E ? k + 1 : k;
  double l[PER];
  float b[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = tid + j * nt;
    l[j] = e < E ? __ldcg(lg + e) : 0.0;
    b[j] = (bnd && e < E) ? __ldcg(bnd + e) : 0.f;
  }
  const float gl = (tid == 0 && has_shared) ? (float)__ldcg(lg + E) : 0.f;
  unsigned long long key[PER];
  float bm = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    key[j] = tid + j * nt < E ? order_key(l[j]) : 0ull;
    bm = fmaxf(bm, b[j]);
  }
  // non-negative floats order as their bits
  topk_warp_candidates<PER>(key, n, nt, ts, __reduce_max_sync(0xffffffffu, __float_as_uint(bm)));
  __syncthreads();
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    if (warp == 0) {   // the best n of the warps' candidates: a merge of nw lists sorted best first
      int ptr = 0;
      const int base = lane * (kMaxTopK + 1);
      unsigned long long hk = lane < nw ? ts.ck[base] : 0ull;
      int hi = lane < nw ? ts.ce[base] : 0x7fffffff;
      for (int r = 0; r < n; ++r) {
        unsigned long long wk;
        int wi;
        const int wl = warp_best(hk, hi, wk, wi);
        if (lane == wl && wk) {   // the winning list moves to its next candidate
          ++ptr;
          hk = ptr < n ? ts.ck[base + ptr] : 0ull;
          hi = ptr < n ? ts.ce[base + ptr] : 0x7fffffff;
        }
        if (lane == 0) {
          ts.idx[r] = wk ? wi : -1;
          ts.lsel[r] = wk ? key_value(wk) : __longlong_as_double(0x7ff8000000000000ll);
        }
      }
      __syncwarp();
      // certification (lane 0): consecutive selected logits more than 2 beta apart
      if (lane == 0) {
        unsigned bb = 0;
        for (int w = 0; w < nw; ++w) bb = max(bb, ts.wb[w]);
        const double twob = 2.0 * (double)__uint_as_float(bb);
        bool sure = !bnd || pass == 1 || ts.idx[0] >= 0;
        if (bnd && pass == 0)
          for (int i = 0; i + 1 < n; ++i) sure = sure && ts.idx[i + 1] >= 0 && ts.lsel[i] - ts.lsel[i + 1] > twob;
        ts.sure = sure ? 1 : 0;
        ts.thr = ts.lsel[k - 1] - twob;
      }
    }
    __syncthreads();
    if (ts.sure) break;
    // ---- rare: the selected and every expert within 2 beta of the k-th, recomputed as the definition
    const double thr = ts.thr;
#pragma unroll 1
    for (int j = 0; j < PER; ++j) {
      const int e = tid + j * nt;
      double lj = 0.0;
#pragma unroll
      for (int q = 0; q < PER; ++q)
        if (q == j) lj = l[q];
      bool sel = false;
      for (int i = 0; i < n; ++i) sel |= ts.idx[i] == e;
      const bool cand = e < E && (sel || !(thr == thr) || lj >= thr);
      const unsigned long long nk = cand ? order_key(exact_logit(rr, e)) : 0ull;
#pragma unroll
      for (int q = 0; q < PER; ++q)
        if (q == j) key[q] = nk;
    }
    __syncthreads();   // every thread has read the first selection
    topk_warp_candidates<PER>(key, n, nt, ts, 0u);
    if (tid == 0) ts.rechecked = 1;
    __syncthreads();
  }
  if (warp == 0) {   // weights over the chosen k, shared gate
    const double first = ts.lsel[0];
    const float ex = (lane < k && ts.idx[lane] >= 0) ? expf((float)(ts.lsel[lane] - first)) : 0.f;
    const float z = warp_sum(ex);
    if (lane < k) ts.w[lane] = ex / z;
    if (lane == 0) ts.sg = has_shared ? 1.f / (1.f + expf(-gl)) : 0.f;
  }
  __syncthreads();
}
__device__ __forceinline__ void block_topk(const double* lg, const float* bnd, int E, int k, int has_shared,
                                           const RouterRef& rr, TopkSmem& ts) {
  if (threadIdx.x == 0) ts.rechecked = 0;
  if (E <= (int)blockDim.x) block_topk_per<1>(lg, bnd, E, k, has_shared, rr, ts);
  else block_topk_per<kTopkPer>(lg, bnd, E, k, has_shared, rr, ts);
}

// The chosen experts of a token (slots 0..k-1) into shared memory; an id
// outside [0, E) latches a device fault and uses expert 0.
__device__ __forceinline__ void load_slots(const TopkSmem& ts, int k, int E, const moe_expert* experts,
                                           moe_expert* slot_ex, uint32_t* status) {
  const int tid = threadIdx.x;
  if (tid < k) {
    int ex = ts.idx[tid];
    if (ex < 0 || ex >= E) { if (status) atomicExch(status, kStatusDeviceFault); ex = 0; }
    const unsigned long long* s8 = (const unsigned long long*)(experts + ex);
    unsigned long long v[sizeof(moe_expert) / 8];
#pragma unroll
    for (int q = 0; q < (int)(sizeof(moe_expert) / 8); ++q) v[q] = __ldg(s8 + q);
    unsigned long long* d8 = (unsigned long long*)(slot_ex + tid);
#pragma unroll
    for (int q = 0; q < (int)(sizeof(moe_expert) / 8); ++q) d8[q] = v[q];
  }
}

}  // namespace qmoe
