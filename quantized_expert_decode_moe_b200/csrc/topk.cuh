// Top-k routing shared by the decode kernels and moe_route (sm_100a).
#pragma once

#include "common.cuh"

namespace qmoe {

// ------------------------------------------------------------------ top-k
// k largest logits, descending, ties to the lower index; weights = softmax over
// all E renormalised over the chosen k = exp(l_i - l_max) / sum_chosen exp(l_j - l_max);
// shared gate = sigmoid(logit E). Logits are compared through an
// order-preserving 64-bit integer key of their double bits (NaN ranks lowest).
// Every warp ranks its slice (one logit per lane per pass, in registers);
// warp 0 merges the warps' candidates. Exact: every global top-k entry is in
// its slice's top-k.
constexpr int kTopkPer = 8;   // logits per lane: E <= kTopkPer * 32 * warps

struct TopkSmem {
  unsigned long long ck[kWarps][kMaxTopK];   // candidate keys
  int ce[kWarps][kMaxTopK];                  // candidate expert ids
  int idx[kMaxTopK];
  float w[kMaxTopK];
  float sg;
};

__device__ __forceinline__ unsigned long long order_key(double v) {
  if (isnan(v)) return 0ull;
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double key_value(unsigned long long k) {
  const unsigned long long u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
  return __longlong_as_double((long long)u);
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

// Block-wide top-k of lg[0..E) (+ shared gate from lg[E] when has_shared),
// global memory written by an earlier kernel. All threads of the block call
// it; results in ts (valid after the call, which ends with __syncthreads).
__device__ __noinline__ static void block_topk(const double* lg, int E, int k, int has_shared, TopkSmem& ts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  constexpr int kNone = 0x7fffffff;
  unsigned long long key[kTopkPer];
#pragma unroll
  for (int j = 0; j < kTopkPer; ++j) {
    const int e = (j * nw + warp) * 32 + lane;
    key[j] = e < E ? order_key(__ldcg(lg + e)) : 0ull;
  }
  double gl = 0.0;
  if (warp == 0 && lane == 0 && has_shared) gl = __ldcg(lg + E);
  for (int r = 0; r < k; ++r) {
    unsigned long long bk = 0ull;
    int be = kNone, bj = -1;
#pragma unroll
    for (int j = 0; j < kTopkPer; ++j) {
      const int e = (j * nw + warp) * 32 + lane;
      if (e < E && key[j] > bk) { bk = key[j]; be = e; bj = j; }
    }
    unsigned long long wk = bk;
    int we = be;
    warp_argmax(wk, we);
    if (be == we && we != kNone) {
#pragma unroll
      for (int j = 0; j < kTopkPer; ++j)
        if (j == bj) key[j] = 0ull;
    }
    if (lane == 0) { ts.ck[warp][r] = wk; ts.ce[warp][r] = we; }
  }
  __syncthreads();
  if (warp == 0) {
    // candidates c = lane + 32 q (q < 4), c = warp' * kMaxTopK + r'
    unsigned long long ck[4];
    int ce[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = lane + 32 * q, w = c / kMaxTopK, r = c % kMaxTopK;
      const bool ok = w < nw && r < k;
      ck[q] = ok ? ts.ck[w][r] : 0ull;
      ce[q] = ok ? ts.ce[w][r] : kNone;
    }
    double lv0 = 0.0, z = 0.0;
    float ex[kMaxTopK];
    for (int r = 0; r < k; ++r) {
      unsigned long long bk = 0ull;
      int be = kNone, bq = -1;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (ce[q] != kNone && (ck[q] > bk || (ck[q] == bk && ce[q] < be))) { bk = ck[q]; be = ce[q]; bq = q; }
      unsigned long long wk = bk;
      int we = be;
      warp_argmax(wk, we);
      if (be == we && we != kNone) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q == bq) { ck[q] = 0ull; ce[q] = kNone; }
      }
      const double lv = key_value(wk);
      if (r == 0) lv0 = lv;
      ex[r] = expf((float)(lv - lv0));
      z += ex[r];
      if (lane == 0) ts.idx[r] = we == kNone ? -1 : we;
    }
    if (lane == 0) {
      const float iz = (float)(1.0 / z);
      for (int r = 0; r < k; ++r) ts.w[r] = ex[r] * iz;
      ts.sg = has_shared ? 1.f / (1.f + expf(-(float)gl)) : 0.f;
    }
  }
  __syncthreads();
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
