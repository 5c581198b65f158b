// Top-k routing shared by the decode kernels and moe_route (sm_100a).
#pragma once

#include "common.cuh"

namespace qmoe {

// ------------------------------------------------------------------ top-k
// k largest logits, descending, ties to the lower index; weights = softmax over
// all E renormalised over the chosen k = exp(l_i - l_max) / sum_chosen exp(l_j - l_max);
// shared gate = sigmoid(logit E). Logits are compared through an
// order-preserving 64-bit integer key of their double bits (key 0 = NaN or
// already taken, ranks lowest). Thread i holds logits i, i + blockDim, ...;
// every warp takes its k best in k rounds (one warp reduction of the key's
// high half per round; the low half and the index only on ties), warp 0 then
// takes the k best of the warps' candidates. Exact: every global top-k entry
// is among its warp's top-k.
constexpr int kTopkPer = 8;   // logits per thread: E <= kTopkPer * blockDim

struct TopkSmem {
  unsigned long long ck[kWarps * kMaxTopK];   // candidate keys, [warp * k + round]
  int ce[kWarps * kMaxTopK];                  // candidate expert ids
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

// Merge by warp 0 of the warps' candidates ts.ck/ce [nw][k], then the
// weights and the shared gate (lane 0 holds gl).
__device__ __forceinline__ void topk_merge(int k, int nw, int has_shared, float gl, TopkSmem& ts) {
  const int lane = threadIdx.x & 31, nc = nw * k;
  // each lane's candidates c = lane + 32q, sorted best first (keys desc, ids asc)
  unsigned long long ck[4];
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
  unsigned long long mine = 0ull, first = 0ull;
  int mid = -1;
  for (int r = 0; r < k; ++r) {
    unsigned long long wk;
    int wi;
    const int wl = warp_best(ck[0], ci[0], wk, wi);
    if (lane == wl) {
      ck[0] = ck[1]; ci[0] = ci[1]; ck[1] = ck[2]; ci[1] = ci[2]; ck[2] = ck[3]; ci[2] = ci[3];
      ck[3] = 0ull; ci[3] = -1;
    }
    if (r == 0) first = wk;
    if (lane == r) { mine = wk; mid = wk ? wi : -1; }
  }
  const float ex = (lane < k && mine) ? expf((float)(key_value(mine) - key_value(first))) : 0.f;
  const float z = warp_sum(ex);
  if (lane < k) { ts.idx[lane] = mid; ts.w[lane] = ex / z; }
  if (lane == 0) ts.sg = has_shared ? 1.f / (1.f + expf(-gl)) : 0.f;
}

// Block-wide top-k of lg[0..E) (+ shared gate from lg[E] when has_shared),
// global memory written by an earlier kernel. All threads of the block call
// it (blockDim = 32 * kWarps); results in ts, valid after the call, which ends
// with __syncthreads. Ids of missing entries (all logits NaN) are -1.
// k <= 8 and (candidates per warp) * warps <= 128.
__device__ __forceinline__ void block_topk(const double* lg, int E, int k, int has_shared, TopkSmem& ts) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = blockDim.x;
  float gl = 0.f;
  if (E <= nt) {   // one logit per thread
    unsigned long long key = tid < E ? order_key(__ldcg(lg + tid)) : 0ull;
    if (warp == 0 && lane == 0 && has_shared) gl = (float)__ldcg(lg + E);
    for (int r = 0; r < k; ++r) {
      unsigned long long wk;
      int wi;
      const int wl = warp_best(key, tid, wk, wi);
      if (lane == wl) key = 0ull;
      if (lane == 0) { ts.ck[warp * k + r] = wk; ts.ce[warp * k + r] = wk ? wi : -1; }
    }
  } else {
    unsigned long long key[kTopkPer];
#pragma unroll
    for (int j = 0; j < kTopkPer; ++j) {
      const int e = tid + j * nt;
      key[j] = e < E ? order_key(__ldcg(lg + e)) : 0ull;
    }
    if (warp == 0 && lane == 0 && has_shared) gl = (float)__ldcg(lg + E);
    // this thread's best (lowest index among equal keys: j ascending, strict >)
    auto local_best = [&](unsigned long long& bk, int& bj) {
      bk = 0ull; bj = 0;
#pragma unroll
      for (int j = 0; j < kTopkPer; ++j)
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
        for (int j = 0; j < kTopkPer; ++j)
          if (j == bj) key[j] = 0ull;
        local_best(bk, bj);
      }
    }
  }
  __syncthreads();
  if (warp == 0) topk_merge(k, nt >> 5, has_shared, gl, ts);
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
