// Decode-path kernels of the quantized MoE expert forward (sm_100a):
// router logits, top-k, expert gate/up and down dequant GEMVs, combine +
// residual + RMSNorm, standalone dequant GEMV, and the grouping of routed
// (token, rank) pairs by expert.
#include <math.h>

#include <mutex>
#include <vector>

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"
#include "digits.cuh"
#include "topk.cuh"

namespace cg = cooperative_groups;

namespace qmoe {

static inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

WsLayout ws_layout(int H, int I, int E, int k, int S, int T) {
  WsLayout L{};
  size_t o = 0;
  L.status = o; o = align256(o + 256);
  L.logits = o; o = align256(o + sizeof(double) * (size_t)T * (E + 1));
  L.bound = o; o = align256(o + sizeof(float) * (size_t)T * (E + 1));
  L.gpart = o; o = align256(o + sizeof(float) * (size_t)kMaxCtas);
  L.a = o; o = align256(o + sizeof(float) * (size_t)T * S * I);
  L.hacc = o; o = align256(o + sizeof(float) * (size_t)T * H);
  L.mxx = o; o = align256(o + (size_t)T * (H / 32) * 112);
  L.mxa = o; o = align256(o + (size_t)T * S * (I / 32) * 112);
  L.counts = o; o = align256(o + sizeof(int32_t) * (size_t)E);
  L.offsets = o; o = align256(o + sizeof(int32_t) * (size_t)(E + 1));
  L.perm = o; o = align256(o + sizeof(int32_t) * (size_t)T * k);
  L.pidx = o; o = align256(o + sizeof(int32_t) * (size_t)T * k);
  L.pw = o; o = align256(o + sizeof(float) * (size_t)T * k);
  L.psg = o; o = align256(o + sizeof(float) * (size_t)T);
  const size_t prows = T > 8 ? (size_t)T * k + T : 0;   // the prefill buffers exist only for T > 8
  const size_t trows = T > 8 ? (size_t)T : 0;
  L.xd = o; o = align256(o + 2 * trows * H);
  L.xX = o; o = align256(o + sizeof(float) * trows * (H / kGroup));
  L.xrs = o; o = align256(o + sizeof(float) * trows * (H / kGroup));
  L.ad = o; o = align256(o + 2 * prows * I);
  L.aX = o; o = align256(o + sizeof(float) * prows * (I / kGroup));
  L.ars = o; o = align256(o + sizeof(float) * prows * (I / kGroup));
  L.chunks = o; o = align256(o + (T > 8 ? sizeof(int4) * pf_max_chunks(T, k, E, pf_chunk_tokens(H, I)) : 0));
  L.nchunks = o; o = align256(o + (T > 8 ? sizeof(int32_t) : 0));
  L.y = o; o = align256(o + sizeof(float) * prows * H);
  L.lpart = o; o = align256(o + (T > 8 ? sizeof(long long) * kRtSplitMax * (size_t)T * E : 0));
  const size_t rw = T > 8 ? route_tc_rows_w(E) : 0, rx = T > 8 ? route_tc_rows_x(T) : 0;
  L.wdig = o; o = align256(o + 3 * rw * (size_t)H);
  L.xdig = o; o = align256(o + 3 * rx * (size_t)H);
  L.wst = o; o = align256(o + sizeof(double) * 8 * rw);
  L.xst = o; o = align256(o + sizeof(double) * 8 * rx);
  const size_t tpad = T > 8 ? (size_t)((T + 15) & ~15) : 0;
  L.tcbx = o; o = align256(o + 2 * tpad * tc_cols(H));
  L.tcxs = o; o = align256(o + sizeof(float) * tpad);
  L.tcbah = o; o = align256(o + 2 * tpad * tc_cols(I));
  L.tcbal = o; o = align256(o + 2 * tpad * tc_cols(I));
  L.tcas = o; o = align256(o + sizeof(float) * tpad);
  size_t np = 0;
  if (T > 8) {
    const size_t gu = (size_t)tc_splits(2 * I, T, H) * 2 * I, dn = (size_t)tc_splits(H, T, I) * H;
    np = (gu > dn ? gu : dn) * (size_t)T;
  }
  L.tcpart = o; o = align256(o + sizeof(float) * np);
  L.tcrexp = o; o = align256(o + (T > 8 ? sizeof(int) * (size_t)(2 * I + H) : 0));
  L.tcaext = o;
  o = align256(o + (T > 8 ? (size_t)128 * (2 * (size_t)I * ((H + 1023) / 1024) + (size_t)H * ((I + 1023) / 1024)) : 0));
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

// cudaFuncSetAttribute once per kernel, device, attribute and value: a launch
// that repeats the last value set skips the driver call.
cudaError_t set_func_attr(const void* fn, cudaFuncAttribute attr, int value) {
  struct Entry {
    const void* fn;
    int dev, attr, value;
  };
  static std::mutex mu;
  static std::vector<Entry> seen;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& x : seen)
    if (x.fn == fn && x.dev == dev && x.attr == (int)attr) {
      if (x.value == value) return cudaSuccess;
      if ((e = cudaFuncSetAttribute(fn, attr, value)) == cudaSuccess) x.value = value;
      return e;
    }
  if ((e = cudaFuncSetAttribute(fn, attr, value)) == cudaSuccess) seen.push_back({fn, dev, (int)attr, value});
  return e;
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
// grid (ceil(rows / 2), T), block 256: four warps per router row (row E = the
// shared-expert gate), each over one quarter of H; every lane keeps its
// 16-byte chunks of the row in registers. Products exact in fp32, summed in
// fp64; each routed logit gets its certified bound (logit_bound).
constexpr int kRouteRows = 2;
constexpr int kRouteSplit = 4;
constexpr int kRouteThreads = kRouteRows * kRouteSplit * 32;
constexpr int kRouteChunks = 4;   // 16-byte weight chunks per lane per pass

// The router's weights do not depend on the previous kernel and are loaded
// before griddepcontrol.wait; x after it. Side jobs: optionally record the
// layer's inputs x and h (CTAs of token row 0), and write x's digit blocks
// for the digit-block layer kernels (a warp per 32-value block, from the x
// staged in shared memory).
__global__ void __launch_bounds__(kRouteThreads) route_logits_kernel(RouteParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint4* xs = (uint4*)smem;                                  // [H/8]
  __shared__ double part[kRouteRows][kRouteSplit];
  __shared__ float spart[kRouteRows][kRouteSplit];
  const int t = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = p.H / 8, half = nch / kRouteSplit;   // chunks per warp's part of the row
  const int nrows = p.E + (p.has_shared ? 1 : 0);
  const int rl = warp / kRouteSplit, hs = warp % kRouteSplit;
  const int e = blockIdx.x * kRouteRows + rl;
  const uint16_t* wrow = e < p.E ? p.router_w + (size_t)e * p.H : p.gate_w;
  const int cb = hs * half;   // first chunk of this warp's part
  double acc2[2] = {0.0, 0.0};
  float sa = 0.f;
  for (int c0 = 0; c0 < half; c0 += 32 * kRouteChunks) {
    uint4 wv[kRouteChunks];
#pragma unroll
    for (int i = 0; i < kRouteChunks; ++i) {
      const int c = c0 + lane + 32 * i;
      wv[i] = (e < nrows && c < half) ? ldg_stream_v4(wrow + (size_t)(cb + c) * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (c0 == 0) {
      griddep_wait();
      griddep_launch_dependents();
      const uint4* xr = (const uint4*)(p.x + (size_t)t * p.H);
      uint4 xv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = threadIdx.x + u * kRouteThreads;
        xv[u] = c < nch ? __ldcg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = threadIdx.x + u * kRouteThreads;
        if (c < nch) xs[c] = xv[u];
      }
      for (int c = threadIdx.x + 4 * kRouteThreads; c < nch; c += kRouteThreads) xs[c] = __ldcg(xr + c);
      if (t == 0 && (p.x_rec || p.h_rec)) {
        const size_t stride = (size_t)gridDim.x * kRouteThreads;
        const size_t i0 = (size_t)blockIdx.x * kRouteThreads + threadIdx.x;
        for (size_t i = i0; i < (size_t)p.T * p.H; i += stride) {
          if (p.h_rec) p.h_rec[i] = __ldcg(p.h + i);
          if (p.x_rec) p.x_rec[i] = __ldcg(p.x + i);
        }
      }
      __syncthreads();
      if (p.xblocks) {   // warp-uniform: every lane of a warp takes the same blocks
        const int nb = p.H / 32, nw = kRouteThreads / 32;
        for (int b = blockIdx.x * nw + warp; b < nb; b += gridDim.x * nw)
          mx_digit_lanes(bf16_to_f32(((const uint16_t*)xs)[b * 32 + lane]), lane,
                         p.xblocks + ((size_t)t * nb + b) * kMxDig, p.codec);
      }
    }
#pragma unroll
    for (int i = 0; i < kRouteChunks; ++i) {
      const int c = c0 + lane + 32 * i;
      if (c < half) dot8_bf16_f64(wv[i], xs[cb + c], acc2, sa);
    }
  }
  const double v = warp_sum_f64(acc2[0] + acc2[1]);
  sa = warp_sum(sa);
  if (lane == 0 && hs != 0) { part[rl][hs] = v; spart[rl][hs] = sa; }
  __syncthreads();
  if (lane == 0 && hs == 0 && e < nrows) {
    double acc = v;
#pragma unroll
    for (int q = 1; q < kRouteSplit; ++q) {
      acc += part[rl][q];
      sa += spart[rl][q];
    }
    const double bias = (e < p.E && p.router_bias) ? (double)p.router_bias[e] : 0.0;
    acc += bias;
    p.logits[(size_t)t * (p.E + 1) + e] = acc;
    if (p.bound && e < p.E) p.bound[(size_t)t * (p.E + 1) + e] = logit_bound(p.H, sa, acc, bias);
  }
}

// grid T, block 512: top-k of logits already in the workspace (moe_route).
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkParams p) {
  __shared__ TopkSmem ts;
  const int t = blockIdx.x, tid = threadIdx.x;
  griddep_wait();   // the logits' kernel has completed (no-op without a programmatic launch)
  griddep_launch_dependents();
  const RouterRef rr{p.x + (size_t)t * p.H, p.router_w, p.router_bias, p.H};
  block_topk(p.logits + (size_t)t * (p.E + 1), p.bound ? p.bound + (size_t)t * (p.E + 1) : nullptr, p.E, p.k,
             p.has_shared, rr, ts);
  if (tid < p.k) {
    p.idx[(size_t)t * p.k + tid] = ts.idx[tid];
    p.w[(size_t)t * p.k + tid] = ts.w[tid];
  }
  if (tid == 0 && p.sg) p.sg[t] = ts.sg;
  if (tid == 0 && p.rechecks && ts.rechecked) atomicAdd(p.rechecks, 1u);
}

// ------------------------------------------------------------------ RMSNorm of the accumulated h' (decode)
// grid T, block 1024: h' = hacc (residual + weighted expert outputs, complete
// after the wait); h <- h', x_out = h' / sqrt(mean(h'^2) + eps) * gamma.
constexpr int kNormThreads = 1024;
constexpr int kNormPer = 8;   // H <= 8192

__global__ void __launch_bounds__(kNormThreads) norm_decode_kernel(NormDecodeParams p) {
  __shared__ float red[kNormThreads / 32];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n4 = p.H / 4;
  float gv[kNormPer / 4][4];
#pragma unroll
  for (int u = 0; u < kNormPer / 4; ++u) {
    const int i = tid + u * kNormThreads;
    if (i < n4) {
      const uint2 g = *(const uint2*)(p.gamma + 4 * (size_t)i);
      gv[u][0] = bf16lo(g.x); gv[u][1] = bf16hi(g.x); gv[u][2] = bf16lo(g.y); gv[u][3] = bf16hi(g.y);
    }
  }
  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0 && p.sel_flag) p.sel_flag[t] = 0u;   // the down kernel has completed: no reader is left
  const float4* hr = (const float4*)(p.hacc + (size_t)t * p.H);
  float4 hv[kNormPer / 4];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kNormPer / 4; ++u) {
    const int i = tid + u * kNormThreads;
    hv[u] = i < n4 ? __ldcg(hr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < kNormPer / 4; ++u)
    ss += hv[u].x * hv[u].x + hv[u].y * hv[u].y + hv[u].z * hv[u].z + hv[u].w * hv[u].w;
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  float tot = warp_sum(red[lane]);
  const float inv = 1.f / sqrtf(tot / (float)p.H + p.eps);
  float4* ho = (float4*)(p.h + (size_t)t * p.H);
#pragma unroll
  for (int u = 0; u < kNormPer / 4; ++u) {
    const int i = tid + u * kNormThreads;
    if (i < n4) {
      ho[i] = hv[u];
      const float o0 = hv[u].x * inv * gv[u][0], o1 = hv[u].y * inv * gv[u][1];
      const float o2 = hv[u].z * inv * gv[u][2], o3 = hv[u].w * inv * gv[u][3];
      uint2 ob;
      ob.x = (uint32_t)f32_to_bf16(o0) | ((uint32_t)f32_to_bf16(o1) << 16);
      ob.y = (uint32_t)f32_to_bf16(o2) | ((uint32_t)f32_to_bf16(o3) << 16);
      *(uint2*)(p.x_out + (size_t)t * p.H + 4 * (size_t)i) = ob;
      if (p.x_out_f32) ((float4*)(p.x_out_f32 + (size_t)t * p.H))[i] = make_float4(o0, o1, o2, o3);
    }
  }
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
  const int nsp = p.y_shared_splits > 1 ? p.y_shared_splits : 1;
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
    float ys = 0.f;
    if (in && ysh)
      for (int q = 0; q < nsp; ++q) ys += ldcg_f32(ysh + (size_t)q * p.y_shared_split_stride + j);
    yv[u][kMaxSlots - 1] = ys;
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

// grid T, block 512 (many tokens: a token per CTA, float4 per thread). Same
// sums as norm_cluster_kernel, element by element: v = h; v = fma(w_i, y_i, v)
// for the routed slots in rank order; v = fma(sg, y_shared, v) with y_shared
// the sum of its splits in order.
constexpr int kNormRThreads = 512;
constexpr int kNormRPer = 4;   // float4 per thread: H <= 8192

__global__ void __launch_bounds__(kNormRThreads) norm_rows_kernel(NormParams p) {
  __shared__ float red[kNormRThreads / 32];
  __shared__ float wsh[kMaxSlots];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_wait();
  griddep_launch_dependents();
  if (tid < p.k) wsh[tid] = ldcg_f32(p.w + (size_t)t * p.k + tid);
  if (tid == 0) wsh[kMaxSlots - 1] = p.y_shared ? ldcg_f32(p.sg + t) : 0.f;
  __syncthreads();
  const int n4 = p.H / 4, nsp = p.y_shared_splits > 1 ? p.y_shared_splits : 1;
  const float4* hr = (const float4*)(p.h + (size_t)t * p.H);
  const float* yr = p.y_routed + (size_t)t * p.y_routed_tok_stride;
  const float* ysh = p.y_shared ? p.y_shared + (size_t)t * p.y_shared_tok_stride : nullptr;
  float4 hv[kNormRPer];
  float ss = 0.f;
#pragma unroll
  for (int u = 0; u < kNormRPer; ++u) {
    const int i = tid + kNormRThreads * u;
    if (i >= n4) continue;
    float4 v = hr[i];
    for (int r = 0; r < p.k; ++r) {
      const float4 y = __ldcg((const float4*)(yr + (size_t)r * p.y_routed_slot_stride) + i);
      const float w = wsh[r];
      v.x = fmaf(w, y.x, v.x); v.y = fmaf(w, y.y, v.y); v.z = fmaf(w, y.z, v.z); v.w = fmaf(w, y.w, v.w);
    }
    if (ysh) {
      float4 ys = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < nsp; ++q) {
        const float4 y = __ldcg((const float4*)(ysh + (size_t)q * p.y_shared_split_stride) + i);
        ys.x += y.x; ys.y += y.y; ys.z += y.z; ys.w += y.w;
      }
      const float w = wsh[kMaxSlots - 1];
      v.x = fmaf(w, ys.x, v.x); v.y = fmaf(w, ys.y, v.y); v.z = fmaf(w, ys.z, v.z); v.w = fmaf(w, ys.w, v.w);
    }
    hv[u] = v;
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = warp_sum(ss);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  const float tot = warp_sum(lane < kNormRThreads / 32 ? red[lane] : 0.f);
  const float inv = 1.f / sqrtf(tot / (float)p.H + p.eps);
#pragma unroll
  for (int u = 0; u < kNormRPer; ++u) {
    const int i = tid + kNormRThreads * u;
    if (i >= n4) continue;
    ((float4*)(p.h + (size_t)t * p.H))[i] = hv[u];
    const uint2 g = *(const uint2*)(p.gamma + 4 * (size_t)i);
    const float o0 = hv[u].x * inv * bf16lo(g.x), o1 = hv[u].y * inv * bf16hi(g.x);
    const float o2 = hv[u].z * inv * bf16lo(g.y), o3 = hv[u].w * inv * bf16hi(g.y);
    uint2 ob;
    ob.x = (uint32_t)f32_to_bf16(o0) | ((uint32_t)f32_to_bf16(o1) << 16);
    ob.y = (uint32_t)f32_to_bf16(o2) | ((uint32_t)f32_to_bf16(o3) << 16);
    *(uint2*)(p.x_out + (size_t)t * p.H + 4 * (size_t)i) = ob;
    if (p.x_out_f32) ((float4*)(p.x_out_f32 + (size_t)t * p.H))[i] = make_float4(o0, o1, o2, o3);
  }
}

// ------------------------------------------------------------------ standalone dequant GEMV
constexpr int kGemvSlots = 8;

template <int BITS, int NS>
__host__ __device__ inline size_t slots_bytes() { return (size_t)kWarps * NS * UnitSmem<BITS>::bytes; }

struct GemvSmem { size_t btab, xs, gsc, gs, ps, buf, total; };
__host__ __device__ inline GemvSmem gemv_smem(int K, int nspans, size_t slots) {
  GemvSmem L{};
  size_t o = 0;
  L.btab = o; o += sizeof(uint2) * (size_t)nspans * kBtPerSpan;
  L.xs = o; o += sizeof(float) * (size_t)K;
  L.gsc = o; o += sizeof(float) * (size_t)(K / kGroup);
  L.gs = o; o += sizeof(float) * 2 * (size_t)(K / kGroup);
  o = (o + 15) & ~(size_t)15;
  L.ps = o; o += sizeof(PartialSmem);
  o = (o + 127) & ~(size_t)127;
  L.buf = o; o += slots;
  L.total = o;
  return L;
}

// grid nCTA, block 512. Units: (tile of 16 rows, span); x (fp32) held per group in fixed point.
template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GemvParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const GemvSmem SL = gemv_smem(p.K, p.nspans, slots_bytes<BITS, kGemvSlots>());
  uint2* btab = (uint2*)(smem + SL.btab);
  float* xs = (float*)(smem + SL.xs);
  float* gsc = (float*)(smem + SL.gsc);
  float* gs = (float*)(smem + SL.gs);
  PartialSmem& ps = *(PartialSmem*)(smem + SL.ps);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ng = p.K / kGroup;
  unsigned char* wslots = smem + SL.buf + (size_t)warp * kGemvSlots * UnitSmem<BITS>::bytes;
  const Range cr = cta_range(p.U, blockIdx.x, p.nCTA);
  const Range wr = warp_range(cr, warp);
  const size_t wpr = (size_t)p.K * BITS / 32, gpr = (size_t)p.K / kGroup;
  auto row = [&](int tile, int r) {
    const size_t rr = (size_t)tile * 16 + r;
    return RowSrc{p.W.q + rr * wpr, p.W.scales + rr * gpr, p.W.biases + rr * gpr};
  };
  auto bt_of = [&](int) -> const uint2* { return btab; };
  auto gs_of = [&](int) -> const float* { return gs; };
  partials_clear(ps, warp, lane);
  WarpPipe<BITS> P;
  pipe_init<BITS>(P, wr, p.nspans, [](int) { return true; });
  pipe_issue<BITS, kGemvSlots>(P, wslots, row, lane);
  for (int i = tid; i < p.K; i += kThreads) xs[i] = p.x[i];
  __syncthreads();
  group_stats(xs, ng, gsc, gs, gs + ng, warp, lane, kWarps);
  __syncthreads();
  for (int i = tid; i < p.nspans * kBtPerSpan; i += kThreads) btab[i] = btab_at<BITS>(xs, gsc, i);
  __syncthreads();
  pipe_run<BITS, kGemvSlots>(P, wslots, row, bt_of, gs_of, ng, ps, warp, lane);
  __syncthreads();
  reduce_partials(cr, p.nspans, ps, [&](int tile, int r, float v) { atomicAdd(p.y + (size_t)tile * 16 + r, v); });
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
  cudaError_t e = set_func_attr(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  if (bytes <= 48 * 1024) return cudaSuccess;
  return set_func_attr(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_route(const RouteParams& p, cudaStream_t s, bool pdl) {
  const int rows = p.E + (p.has_shared ? 1 : 0);
  dim3 grid((rows + kRouteRows - 1) / kRouteRows, p.T);
  RouteParams q = p;
  void* args[] = {&q};
  const size_t sm = ((size_t)p.H * 2 + 15) & ~(size_t)15;
  cudaError_t e = set_smem((const void*)route_logits_kernel, sm);
  if (e != cudaSuccess) return e;
  return launch_ex((const void*)route_logits_kernel, grid, dim3(kRouteThreads), sm, s, pdl, args);
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s, bool pdl) {
  cudaError_t e = set_smem((const void*)topk_kernel, 0);
  if (e != cudaSuccess) return e;
  TopkParams q = p;
  void* args[] = {&q};
  return launch_ex((const void*)topk_kernel, dim3(p.T), dim3(kThreads), 0, s, pdl, args);
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

cudaError_t launch_norm_decode(const NormDecodeParams& p, bool pdl, cudaStream_t s) {
  cudaError_t e = set_smem((const void*)norm_decode_kernel, 0);
  if (e != cudaSuccess) return e;
  NormDecodeParams q = p;
  void* args[] = {&q};
  return launch_ex((const void*)norm_decode_kernel, dim3(p.T), dim3(kNormThreads), 0, s, pdl, args);
}

cudaError_t launch_norm(const NormParams& p, bool pdl, cudaStream_t s) {
  auto a16 = [](const void* q) { return ((uintptr_t)q & 15u) == 0; };
  const bool vec = a16(p.y_routed) && a16(p.y_shared) && a16(p.h) && a16(p.x_out) && a16(p.x_out_f32) &&
                   a16(p.gamma) && p.H % 4 == 0 && p.y_routed_slot_stride % 4 == 0 && p.y_shared_split_stride % 4 == 0;
  if (p.T >= 32 && vec) {   // enough tokens to fill the GPU with a CTA each (float4 rows)
    NormParams q = p;
    void* args[] = {&q};
    return launch_ex((const void*)norm_rows_kernel, dim3(p.T), dim3(kNormRThreads), 0, s, pdl, args);
  }
  cudaError_t e = set_smem((const void*)norm_cluster_kernel, 0);
  if (e != cudaSuccess) return e;
  NormParams q = p;
  void* args[] = {&q};
  return launch_ex((const void*)norm_cluster_kernel, dim3(kNormCluster, p.T), dim3(kNormCThreads), 0, s, pdl, args);
}

cudaError_t launch_gemv(const GemvParams& p, int bits, cudaStream_t s) {
  GemvParams q = p;
  const size_t sm = gemv_smem(p.K, p.nspans, bits == 4 ? slots_bytes<4, kGemvSlots>() : slots_bytes<2, kGemvSlots>()).total;
  if (sm > (size_t)smem_optin()) return cudaErrorInvalidConfiguration;
  const void* fn = bits == 4 ? (const void*)gemv_kernel<4> : (const void*)gemv_kernel<2>;
  cudaError_t e = set_smem(fn, sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  return launch_ex(fn, dim3(p.nCTA), dim3(kThreads), sm, s, false, args);
}

}  // namespace qmoe
