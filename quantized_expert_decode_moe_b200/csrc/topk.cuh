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
// then the bias is added. The decode router computes each logit faster
// (compensated fp32 over a summation tree) together with a rigorous bound
// b_e on |fast - definition|. Selection runs on the fast values and is then
// certified: with theta = min over the chosen of (l - b), the chosen set is
// certain when no other expert has l + b >= theta, and the order among the
// chosen is certain when adjacent chosen intervals [l - b, l + b] are
// disjoint. Otherwise every expert with l + b >= theta (a set that contains
// the true top k) is recomputed exactly as the definition's index-order fp64
// sum, and the selection runs again on those exact values.
#pragma once

#include "common.cuh"

namespace qmoe {

constexpr int kTopkPer = 8;   // logits per thread at most: E <= kTopkPer * blockDim

struct TopkSmem {
  unsigned long long ck[kWarps * kMaxTopK];   // candidate keys, [warp * k + round]
  int ce[kWarps * kMaxTopK];                  // candidate expert ids
  int idx[kMaxTopK];
  float w[kMaxTopK];
  double lsel[kMaxTopK];                      // logits of the chosen (the values ranked on)
  float bsel[kMaxTopK];                       // their error bounds
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
// product to about 2^-44 relative to sum |w x|, which goes to a.
__device__ __forceinline__ void dot8_bf16_comp(uint4 w, uint4 x, float (&s)[4], float (&c)[4], float& a) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w}, xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float p0 = bf16lo(wv[i]) * bf16lo(xv[i]), p1 = bf16hi(wv[i]) * bf16hi(xv[i]);
    two_sum_acc(s[i], c[i], p0);
    two_sum_acc(s[i], c[i], p1);
    a += fabsf(p0) + fabsf(p1);
  }
}

// Bound on |fast logit - definition| for a logit of n products computed as
// the compensated fp32 sum of the decode router (every addition of the main
// sum an error-free TwoSum, the rounding errors carried in a plain fp32 sum),
// given sa = the fp32 sum of |w x| over the n products, the fast fp64 logit
// acc (bias included) and the bias. With u = 2^-24 and S = sum |w x|:
//  - the TwoSum errors e_j satisfy sum |e_j| <= n u S, and carrying them in a
//    plain fp32 sum adds at most n u sum |e_j| <= n^2 u^2 S;
//  - the definition (index-order fp64 sum) is within n 2^-53 S of the exact
//    sum; three fp64 roundings of the results (s + c, + bias, the
//    definition's + bias) are within 2^-53 (|acc| + |bias|) each;
//  - an fp32 product below 2^-126 in magnitude loses at most 2^-150;
//  - sa underestimates S by at most a factor 1 - n u (n <= 8192).
// The margins 1.25 and 2^-50 cover the last point and the rounding of the
// bound itself; the result is rounded up to fp32.
__device__ __forceinline__ float logit_bound(int n, float sa, double acc, double bias) {
  const double nn = (double)n;
  const double b = 1.25 * (nn * nn * 0x1p-48 + nn * 0x1p-53) * (double)sa + 0x1p-50 * (fabs(acc) + fabs(bias)) +
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

// The k best of the block's keys (key desc, id asc). Thread tid holds the
// keys of e = tid + j * blockDim (j < kTopkPer; key 0 = not a candidate); the
// keys are consumed. Every warp takes its k best in k rounds, warp 0 merges
// the warps' candidates (exact: every global top-k entry is among its warp's
// top k). Results: ts.idx[i] (-1 when there are fewer than k candidates) and
// ts.lsel[i], valid after the call, which ends with __syncthreads.
// k <= 8 and k * warps <= 128.
template <int PER>
__device__ __forceinline__ void topk_select(unsigned long long (&key)[PER], int k, TopkSmem& ts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nt = blockDim.x;
  auto local_best = [&](unsigned long long& bk, int& bj) {   // lowest j among equal keys
    bk = 0ull; bj = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (key[j] > bk) { bk = key[j]; bj = j; }
  };
  unsigned long long bk;
  int bj;
  local_best(bk, bj);
  for (int r = 0; r < k; ++r) {
    unsigned long long wk;
    int wi;
    const int wl = warp_best(bk, tid + bj * nt, wk, wi);
    if (lane == 0) { ts.ck[warp * k + r] = wk; ts.ce[warp * k + r] = wk ? wi : -1; }
    if (lane == wl && wk) {
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (j == bj) key[j] = 0ull;
      local_best(bk, bj);
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int nc = (nt >> 5) * k;
    unsigned long long ck[4];   // each lane's candidates c = lane + 32q, sorted best first
    int ci[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = lane + 32 * q;
      ck[q] = c < nc ? ts.ck[c] : 0ull;
      ci[q] = c < nc ? ts.ce[c] : -1;
    }
    auto cx = [&](int a, int b) {   // compare-exchange: better one to a
      const bool sw = ck[b] > ck[a] || (ck[b] == ck[a] && ck[a] && (unsigned)ci[b] < (unsigned)ci[a]);
      if (sw) {
        const unsigned long long tk = ck[a]; ck[a] = ck[b]; ck[b] = tk;
        const int ti = ci[a]; ci[a] = ci[b]; ci[b] = ti;
      }
    };
    cx(0, 1); cx(2, 3); cx(0, 2); cx(1, 3); cx(1, 2);
    for (int r = 0; r < k; ++r) {
      unsigned long long wk;
      int wi;
      const int wl = warp_best(ck[0], ci[0], wk, wi);
      if (lane == wl) {
        ck[0] = ck[1]; ci[0] = ci[1]; ck[1] = ck[2]; ci[1] = ci[2]; ck[2] = ck[3]; ci[2] = ci[3];
        ck[3] = 0ull; ci[3] = -1;
      }
      if (lane == 0) {
        ts.idx[r] = wk ? wi : -1;
        ts.lsel[r] = wk ? key_value(wk) : __longlong_as_double(0x7ff8000000000000ll);
      }
    }
  }
  __syncthreads();
}

// Block-wide top-k of lg[0..E) (+ shared gate from lg[E] when has_shared),
// global memory written by an earlier kernel or CTA (read through L2).
// bnd: per-logit error bounds of fast logits (certified as described at the
// top of this file, with an exact recheck through rr when needed), or null
// when lg already holds the definition's values. All threads of the block
// call it (blockDim = 32 * kWarps); results in ts (idx, w, sg), valid after
// the call, which ends with __syncthreads. Ids of missing entries (fewer
// than k logits that are not NaN) are -1. k <= 8, E <= kTopkPer * blockDim.
template <int PER>
__device__ __forceinline__ void block_topk_per(const double* lg, const float* bnd, int E, int k, int has_shared,
                                               const RouterRef& rr, TopkSmem& ts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nt = blockDim.x;
  double l[PER];
  float b[PER];
  unsigned long long key[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = tid + j * nt;
    l[j] = e < E ? __ldcg(lg + e) : 0.0;
    b[j] = (bnd && e < E) ? __ldcg(bnd + e) : 0.f;
    key[j] = e < E ? order_key(l[j]) : 0ull;
  }
  const float gl = (tid == 0 && has_shared) ? (float)__ldcg(lg + E) : 0.f;
  topk_select(key, k, ts);
  if (tid == 0) ts.rechecked = 0;
  if (bnd) {
    int sel[kMaxTopK];
#pragma unroll
    for (int i = 0; i < kMaxTopK; ++i) sel[i] = i < k ? ts.idx[i] : -1;
    auto chosen = [&](int e) {
      bool c = false;
#pragma unroll
      for (int i = 0; i < kMaxTopK; ++i) c |= sel[i] == e;
      return c;
    };
#pragma unroll
    for (int j = 0; j < PER; ++j) {   // owners publish the bounds of the chosen
      const int e = tid + j * nt;
      if (e < E) {
#pragma unroll
        for (int i = 0; i < kMaxTopK; ++i)
          if (sel[i] == e) ts.bsel[i] = b[j];
      }
    }
    __syncthreads();
    double theta = ts.lsel[0] - (double)ts.bsel[0];
    bool unsure = !(theta == theta) || sel[0] < 0;
    for (int i = 1; i < k; ++i) {
      const double lo = ts.lsel[i] - (double)ts.bsel[i];
      unsure |= sel[i] < 0 || !(ts.lsel[i - 1] - (double)ts.bsel[i - 1] > ts.lsel[i] + (double)ts.bsel[i]);
      theta = lo < theta ? lo : theta;
    }
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      const int e = tid + j * nt;
      if (e < E && !chosen(e) && l[j] + (double)b[j] >= theta) unsure = true;
    }
    if (__syncthreads_or(unsure)) {   // rare: recompute the candidates exactly and select again
#pragma unroll
      for (int j = 0; j < PER; ++j) {
        const int e = tid + j * nt;
        key[j] = (e < E && (l[j] + (double)b[j] >= theta || chosen(e) || !(theta == theta)))
                     ? order_key(exact_logit(rr, e)) : 0ull;
      }
      topk_select(key, k, ts);
      if (tid == 0) ts.rechecked = 1;
    }
  }
  if (warp == 0) {   // weights over the chosen, shared gate
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
