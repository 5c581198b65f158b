// Host-resident routed experts with an HBM expert cache.
//
// The Flash-MoE engine keeps the experts outside the GPU (on SSD) and loads
// the ones the router picks for each token, leaving the caching to the
// operating system's page cache ("Key technologies > SSD expert streaming",
// "Trust the OS" of the Flash-MoE write-up). The B200 form of that idea: the
// routed experts stay in host memory, HBM holds `slots` of them, and a call
// routes on the GPU, reads the chosen ids back, copies the missing experts
// host -> HBM (least recently used slots are reused first) and then runs the
// layer's kernels with the expert table pointing at the slots.
//
// Everything is caller-owned: the host experts, a device buffer (the expert
// table the kernels read, then the slots) and a host buffer for the
// bookkeeping. The bookkeeping is plain host code (moe_cache_admit), so the
// policy can be exercised without a GPU.
#include <stdint.h>
#include <string.h>

#include "kernels.cuh"
#include "moe.h"

namespace qmoe {
namespace {

constexpr uint64_t kCacheMagic = 0x4d6f45436163686full;   // "MoECachh"
constexpr int kCacheMaxIds = 4096;                         // ids of one call: T * top_k
constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) & ~(kAlign - 1); }

// Byte sizes of the nine arrays of one expert: gate, up, down x (q, scales, biases).
void expert_arrays(const moe_layer* L, size_t (&sz)[9]) {
  const size_t H = (size_t)L->hidden, I = (size_t)L->inter, b = (size_t)L->bits, g = (size_t)L->group;
  const size_t qgu = I * H * b / 8, sgu = I * (H / g) * 2, qdn = H * I * b / 8, sdn = H * (I / g) * 2;
  const size_t v[9] = {qgu, sgu, sgu, qgu, sgu, sgu, qdn, sdn, sdn};
  for (int i = 0; i < 9; ++i) sz[i] = v[i];
}

struct CacheState {
  uint64_t magic;
  int32_t E, slots;
  size_t slot_bytes, off[9], sz[9];
  uint64_t clock, hits, misses, bytes;
  int32_t table_ready;       // every entry of the device table points at valid slot memory
  const moe_expert* host;    // caller's host experts [E]
  moe_expert* dev_table;     // device [E]
  char* dev_slots;           // device [slots][slot_bytes]
  // followed by: int32 slot_of[E], int32 owner[slots], uint64 last[slots],
  // int32 ids[kCacheMaxIds], moe_expert mirror[E] (host copy of the device
  // table), uint64 seen[E] (the call that last named each expert)
};

struct StateView {
  CacheState* st;
  int32_t* slot_of;
  int32_t* owner;
  uint64_t* last;
  int32_t* ids;
  moe_expert* mirror;
  uint64_t* seen;
};

size_t state_bytes_for(int E, int slots) {
  size_t o = (sizeof(CacheState) + 7) & ~(size_t)7;
  o += sizeof(int32_t) * (size_t)E;
  o = (o + 7) & ~(size_t)7;
  o += sizeof(int32_t) * (size_t)slots;
  o = (o + 7) & ~(size_t)7;
  o += sizeof(uint64_t) * (size_t)slots;
  o += sizeof(int32_t) * (size_t)kCacheMaxIds;
  o = (o + 7) & ~(size_t)7;
  o += sizeof(moe_expert) * (size_t)E;
  o = (o + 7) & ~(size_t)7;
  o += sizeof(uint64_t) * (size_t)E;
  return o;
}

StateView view_of(void* state) {
  StateView v;
  v.st = (CacheState*)state;
  char* p = (char*)state + ((sizeof(CacheState) + 7) & ~(size_t)7);
  const int E = v.st->E, S = v.st->slots;
  v.slot_of = (int32_t*)p; p += sizeof(int32_t) * (size_t)E;
  p = (char*)(((uintptr_t)p + 7) & ~(uintptr_t)7);
  v.owner = (int32_t*)p; p += sizeof(int32_t) * (size_t)S;
  p = (char*)(((uintptr_t)p + 7) & ~(uintptr_t)7);
  v.last = (uint64_t*)p; p += sizeof(uint64_t) * (size_t)S;
  v.ids = (int32_t*)p; p += sizeof(int32_t) * (size_t)kCacheMaxIds;
  p = (char*)(((uintptr_t)p + 7) & ~(uintptr_t)7);
  v.mirror = (moe_expert*)p; p += sizeof(moe_expert) * (size_t)E;
  p = (char*)(((uintptr_t)p + 7) & ~(uintptr_t)7);
  v.seen = (uint64_t*)p;
  return v;
}

bool valid_state(const void* state) {
  return state && ((uintptr_t)state & 7u) == 0 && ((const CacheState*)state)->magic == kCacheMagic;
}

}  // namespace
}  // namespace qmoe

using namespace qmoe;

extern "C" {

moe_status moe_cache_size(const moe_layer* layer, int32_t slots, size_t* dev_bytes, size_t* state_bytes) {
  if (!layer || !dev_bytes || !state_bytes || slots <= 0) return MOE_ERR_INVALID_ARGUMENT;
  if (layer->bits != 2 && layer->bits != 4) return MOE_ERR_UNSUPPORTED;
  if (layer->group != 64 || layer->hidden <= 0 || layer->inter <= 0 || layer->n_experts <= 0)
    return MOE_ERR_INVALID_ARGUMENT;
  size_t sz[9];
  expert_arrays(layer, sz);
  size_t slot = 0;
  for (int i = 0; i < 9; ++i) slot += align_up(sz[i]);
  *dev_bytes = align_up(sizeof(moe_expert) * (size_t)layer->n_experts) + slot * (size_t)slots;
  *state_bytes = state_bytes_for(layer->n_experts, slots);
  return MOE_OK;
}

moe_status moe_cache_init(const moe_layer* layer, const moe_expert* host_experts, int32_t slots, void* dev,
                          size_t dev_bytes, void* state, size_t state_bytes) {
  size_t need_dev = 0, need_state = 0;
  moe_status st = moe_cache_size(layer, slots, &need_dev, &need_state);
  if (st) return st;
  if (!host_experts || !dev || !state || ((uintptr_t)dev & (kAlign - 1)) || ((uintptr_t)state & 7u))
    return MOE_ERR_INVALID_ARGUMENT;
  if (dev_bytes < need_dev || state_bytes < need_state) return MOE_ERR_WORKSPACE;
  CacheState* c = (CacheState*)state;
  memset(state, 0, need_state);
  c->magic = kCacheMagic;
  c->E = layer->n_experts;
  c->slots = slots;
  expert_arrays(layer, c->sz);
  size_t o = 0;
  for (int i = 0; i < 9; ++i) {
    c->off[i] = o;
    o += align_up(c->sz[i]);
  }
  c->slot_bytes = o;
  c->host = host_experts;
  c->dev_table = (moe_expert*)dev;
  c->dev_slots = (char*)dev + align_up(sizeof(moe_expert) * (size_t)layer->n_experts);
  StateView v = view_of(state);
  for (int e = 0; e < c->E; ++e) v.slot_of[e] = -1;
  for (int s = 0; s < slots; ++s) v.owner[s] = -1;
  return MOE_OK;
}

moe_status moe_cache_admit(void* state, const int32_t* ids, int32_t n, int32_t* slot, int32_t* missed) {
  if (!valid_state(state) || n < 0 || (n > 0 && (!ids || !slot || !missed))) return MOE_ERR_INVALID_ARGUMENT;
  StateView v = view_of(state);
  CacheState* c = v.st;
  for (int i = 0; i < n; ++i)
    if (ids[i] < 0 || ids[i] >= c->E) return MOE_ERR_INVALID_ARGUMENT;
  // distinct ids of this call (seen[e] == now marks an expert named earlier in it)
  const uint64_t now = ++c->clock;   // every id of this call is stamped `now`: none of them is evicted by another
  int distinct = 0;
  for (int i = 0; i < n; ++i)
    if (v.seen[ids[i]] != now) {
      v.seen[ids[i]] = now;
      ++distinct;
    }
  if (distinct > c->slots) return MOE_ERR_UNSUPPORTED;
  // resident ids: hits
  for (int i = 0; i < n; ++i) {
    const int s = v.slot_of[ids[i]];
    missed[i] = 0;
    slot[i] = s;
    if (s >= 0) v.last[s] = now;
  }
  // missing ids: the least recently used slot (free slots first, lowest index on ties)
  for (int i = 0; i < n; ++i) {
    if (slot[i] >= 0) continue;
    const int e = ids[i];
    if (v.slot_of[e] >= 0) {   // a repeat of an id admitted earlier in this call
      slot[i] = v.slot_of[e];
      continue;
    }
    int best = -1;
    for (int s = 0; s < c->slots; ++s) {
      if (v.owner[s] >= 0 && v.last[s] == now) continue;   // in use by this call
      if (best < 0) {
        best = s;
        continue;
      }
      const bool fs = v.owner[s] < 0, fb = v.owner[best] < 0;
      if ((fs && !fb) || (!fs && !fb && v.last[s] < v.last[best])) best = s;
    }
    if (v.owner[best] >= 0) v.slot_of[v.owner[best]] = -1;   // evicted
    v.owner[best] = e;
    v.slot_of[e] = best;
    v.last[best] = now;
    slot[i] = best;
    missed[i] = 1;
  }
  // per distinct expert: a hit, or a miss (its first id carries the flag)
  for (int i = 0; i < n; ++i)
    if (v.seen[ids[i]] == now) {
      v.seen[ids[i]] = 0;   // counted
      if (missed[i]) ++c->misses;
      else ++c->hits;
    }
  return MOE_OK;
}

moe_status moe_cache_stats(const void* state, uint64_t* hits, uint64_t* misses, uint64_t* bytes_copied) {
  if (!valid_state(state)) return MOE_ERR_INVALID_ARGUMENT;
  const CacheState* c = (const CacheState*)state;
  if (hits) *hits = c->hits;
  if (misses) *misses = c->misses;
  if (bytes_copied) *bytes_copied = c->bytes;
  return MOE_OK;
}

moe_status moe_layer_forward_cached(const moe_layer* layer, void* state, const uint16_t* x_in, float* h, int32_t T,
                                    uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (!layer || !valid_state(state)) return MOE_ERR_INVALID_ARGUMENT;
  StateView v = view_of(state);
  CacheState* c = v.st;
  if (layer->n_experts != c->E || T <= 0) return MOE_ERR_INVALID_ARGUMENT;
  const int k = layer->top_k;
  if ((long long)T * k > kCacheMaxIds) return MOE_ERR_UNSUPPORTED;
  moe_layer L = *layer;
  L.experts = c->dev_table;   // the kernels read the cache's table
  cudaStream_t s = (cudaStream_t)stream;
  size_t need = 0;
  moe_status st = moe_workspace_size(&L, T, &need);
  if (st) return st;
  if (!ws || ws_bytes < need) return MOE_ERR_WORKSPACE;
  // 0. first use: every entry of the device table points at slot 0, so that no entry of the
  //    table is ever an invalid address (the kernels read only the chosen experts' entries)
  if (!c->table_ready) {
    moe_expert ex0;
    moe_qmat* dm[3] = {&ex0.gate, &ex0.up, &ex0.down};
    for (int m = 0; m < 3; ++m) {
      dm[m]->q = (const uint32_t*)(c->dev_slots + c->off[3 * m]);
      dm[m]->scales = (const uint16_t*)(c->dev_slots + c->off[3 * m + 1]);
      dm[m]->biases = (const uint16_t*)(c->dev_slots + c->off[3 * m + 2]);
    }
    for (int e = 0; e < c->E; ++e) v.mirror[e] = ex0;
    if (cudaMemcpyAsync(c->dev_table, v.mirror, sizeof(moe_expert) * (size_t)c->E, cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    c->table_ready = 1;
  }
  // 1. route (on the GPU) and read the chosen ids back
  int32_t* idx_dev = (int32_t*)((char*)ws + ws_layout(L.hidden, L.inter, L.n_experts, k,
                                                     k + (L.has_shared ? 1 : 0), T).pidx);
  float* w_dev = (float*)((char*)ws + ws_layout(L.hidden, L.inter, L.n_experts, k,
                                                k + (L.has_shared ? 1 : 0), T).pw);
  if ((st = moe_route(&L, x_in, T, idx_dev, w_dev, nullptr, ws, ws_bytes, stream))) return st;
  if (cudaMemcpyAsync(v.ids, idx_dev, sizeof(int32_t) * (size_t)T * k, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // 2. admit them; copy the missing experts into their slots and point the table at them
  int32_t slot[kCacheMaxIds], missed[kCacheMaxIds];
  if ((st = moe_cache_admit(state, v.ids, T * k, slot, missed))) return st;
  for (int i = 0; i < T * k; ++i) {
    if (!missed[i]) continue;
    const int e = v.ids[i];
    char* base = c->dev_slots + (size_t)slot[i] * c->slot_bytes;
    const moe_expert& hx = c->host[e];
    const moe_qmat* hm[3] = {&hx.gate, &hx.up, &hx.down};
    moe_qmat* dm[3] = {&v.mirror[e].gate, &v.mirror[e].up, &v.mirror[e].down};
    for (int m = 0; m < 3; ++m) {
      const void* src[3] = {hm[m]->q, hm[m]->scales, hm[m]->biases};
      void* dst[3] = {base + c->off[3 * m], base + c->off[3 * m + 1], base + c->off[3 * m + 2]};
      for (int a = 0; a < 3; ++a) {   // one copy per array
        if (!src[a]) return MOE_ERR_INVALID_ARGUMENT;
        if (cudaMemcpyAsync(dst[a], src[a], c->sz[3 * m + a], cudaMemcpyHostToDevice, s) != cudaSuccess)
          return MOE_ERR_CUDA;
        c->bytes += c->sz[3 * m + a];
      }
      dm[m]->q = (const uint32_t*)dst[0];
      dm[m]->scales = (const uint16_t*)dst[1];
      dm[m]->biases = (const uint16_t*)dst[2];
    }
    if (cudaMemcpyAsync(c->dev_table + e, &v.mirror[e], sizeof(moe_expert), cudaMemcpyHostToDevice, s) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // 3. the layer, with every chosen expert resident
  return moe_layer_forward(&L, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, ws_bytes, stream);
}

}  // extern "C"
