// Router logits of many tokens (prefill) in exact integer arithmetic on the
// tcgen05 tensor cores, with a rigorous bound on each logit's distance to the
// definition (the index-order fp64 sum of the exact bf16 products, bias added
// last), for the certified top-k of topk.cuh.
//
// Every router row and every token is written as 22-bit fixed point with its
// own power-of-two scale: V = rint(v 2^p) with max |v| 2^p < 2^22, split
// exactly into three balanced signed 8-bit digits, V = d2 2^16 + d1 2^8 + d0.
// The integer dot products of the digits (kind::i8 MMAs, s32 accumulators in
// tensor memory) are exact; pairs of equal weight 2^(8(i+j)) share one
// accumulator. The pair of the two low digits (weight 1) is left out and
// bounded instead, so four classes (i + j = 1..4, each below 2^28 in
// magnitude) fill the 512 columns of tensor memory for a 128 x 128 tile. A
// split's partial sum_s 2^(8s) acc_s is an exact int64 (below 2^61 in
// magnitude), so the splits add exactly in any order; the logit is that
// total times 2^-(p_t + q_e), in fp64, plus the bias.
//
// Bound. With x~ = X 2^-p, w~ = W 2^-q, dx = x - x~, dw = w - w~:
//   |sum x w - sum x~ w~| = |sum dx w + x~ dw| <= sum|dx| max|w| + sum|dw| max|x~|,
// max|x~| <= max|x| + 2^-p. The digits kernel sums the residuals |dv| of each
// row in fp64 (v and V 2^-p are exact there); most bf16 values are exact in
// 22-bit fixed point, so these terms are small. The pair left out is at most
// 2^-(p+q) min(sum|d0(w)| max|d0(x)|, sum|d0(x)| max|d0(w)|). The definition's
// index-order fp64 sum is within (H-1) 2^-53 max|x| sum|w| of the exact dot
// product (Higham, Accuracy and Stability of Numerical Algorithms, sec. 4.2);
// the conversion of the int64 total and the bias additions (ours and the
// definition's) cost at most 2^-52 (|l| + |b|). The sum, times 1.01, is
// rounded up to fp32.
//
// The shared-gate logit is not ranked: the digits kernel computes it as an
// fp64 sum of its exact products, in a fixed tree order.
//
// Kernels: route_digits_kernel (a CTA per row: scale, statistics, digit
// planes in the tensor cores' K-major tile layout, the gate logit),
// route_tc_kernel (one CTA per 128 router rows x 128 tokens x column split;
// one thread brings each stage with two bulk copies, one issues the MMAs,
// four warps read tensor memory and write the split's int64 partials),
// route_tc_combine_kernel (sum of the splits, scale, bias, bound).
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"
#include "tc.cuh"

namespace qmoe {

constexpr int kRtM = 128;          // router rows per CTA (one MMA tile)
constexpr int kRtN = 128;          // tokens per CTA
constexpr int kRtKS = 64;          // columns per stage
constexpr int kRtStages = 4;
constexpr int kRtClasses = 4;      // digit pairs grouped by i + j = 1..4
constexpr int kRtChunk = 128 * 16;                 // 16 columns of 128 rows: 2 KB
constexpr int kRtPlane = kRtKS / 16 * kRtChunk;    // one digit plane of a tile stage: 8 KB
constexpr int kRtTile = 3 * kRtPlane;              // three planes: 24 KB, contiguous in global memory
constexpr int kRtStageBytes = 2 * kRtTile;         // router rows, then tokens
constexpr int kRtStat = 8;                         // doubles per row of statistics
constexpr int kRdThreads = 256;                    // digits kernel: threads per row
constexpr int kRdMaxChunks = 2;                    // 16-element chunks per thread (H <= 8192)

static_assert(kRtM == 128 && kRtN == 128, "route_tc_rows_w / route_tc_rows_x pad to these tiles");
static_assert(kRdThreads * kRdMaxChunks * 16 >= 8192, "the digits kernel holds a row of up to 8192 values");

// Byte offset of 16-column chunk c of row r in a digit plane array of the
// tiled layout: tile r / 128, stage c / 4, plane q, chunk c % 4, row r % 128.
__device__ __forceinline__ size_t rt_dig_off(int r, int c, int q, int nstg) {
  return ((((size_t)(r >> 7) * nstg + (c >> 2)) * 3 + q) * 4 + (c & 3)) * kRtChunk + (size_t)(r & 127) * 16;
}

// ------------------------------------------------------------------ digits
// grid rows_w + rows_x, block kRdThreads: a CTA per row. Row b < rows_w is
// router row b (beyond E: zeros), then the tokens (beyond T: zeros; a token
// row also yields its shared-gate logit). Thread i handles the 16-element
// chunks c = i + kRdThreads j, held in registers between the two passes.
// Statistics per row: {2^-p, sum |v|, max |v|, sum |v - V 2^-p|, sum |d0|,
// max |d0|, 0, 0}.
__global__ void __launch_bounds__(kRdThreads) route_digits_kernel(RouteParams p) {
  __shared__ double red[4][kRdThreads / 32];
  __shared__ float redm[kRdThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rw = (int)route_tc_rows_w(p.E);
  const bool isw = (int)blockIdx.x < rw;
  const int r = isw ? (int)blockIdx.x : (int)blockIdx.x - rw;
  const uint16_t* src = isw ? (r < p.E ? p.router_w + (size_t)r * p.H : nullptr)
                            : (r < p.T ? p.x + (size_t)r * p.H : nullptr);
  const uint16_t* gw = (!isw && src && p.has_shared) ? p.gate_w : nullptr;
  const int nch = p.H / 16, nstg = p.H / kRtKS;
  int8_t* dig = isw ? p.wdig : p.xdig;
  uint4 v[kRdMaxChunks][2];
  float mx = 0.f;
  double sa = 0.0, g = 0.0;
#pragma unroll
  for (int j = 0; j < kRdMaxChunks; ++j) {
    const int c = tid + kRdThreads * j;
    v[j][0] = v[j][1] = make_uint4(0u, 0u, 0u, 0u);
    if (src && c < nch) {
      v[j][0] = __ldg((const uint4*)(src + 16 * c));
      v[j][1] = __ldg((const uint4*)(src + 16 * c) + 1);
      uint4 g0 = make_uint4(0u, 0u, 0u, 0u), g1 = g0;
      if (gw) {
        g0 = __ldg((const uint4*)(gw + 16 * c));
        g1 = __ldg((const uint4*)(gw + 16 * c) + 1);
      }
      const uint32_t w[8] = {v[j][0].x, v[j][0].y, v[j][0].z, v[j][0].w, v[j][1].x, v[j][1].y, v[j][1].z, v[j][1].w};
      const uint32_t gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a0 = bf16lo(w[i]), a1 = bf16hi(w[i]);
        mx = fmaxf(mx, fmaxf(fabsf(a0), fabsf(a1)));
        sa += (double)fabsf(a0) + (double)fabsf(a1);
        g += (double)a0 * (double)bf16lo(gg[i]) + (double)a1 * (double)bf16hi(gg[i]);   // exact products
      }
    }
  }
  mx = warp_max(mx);
  if (lane == 0) redm[warp] = mx;
  __syncthreads();
  mx = 0.f;
#pragma unroll
  for (int w = 0; w < kRdThreads / 32; ++w) mx = fmaxf(mx, redm[w]);
  int e = 0;
  if (mx > 0.f) {   // max |v| 2^e < 2^22
    int E2;
    frexpf(mx, &E2);
    e = 22 - E2;
  }
  const double inv = ldexp(1.0, -e);
  double res = 0.0, s0 = 0.0;   // sum |v - V 2^-e|, sum |d0|
  int m0 = 0;                   // max |d0|
#pragma unroll
  for (int j = 0; j < kRdMaxChunks; ++j) {
    const int c = tid + kRdThreads * j;
    if (c >= nch) continue;
    uint32_t d[3][4] = {};
    const uint32_t w[8] = {v[j][0].x, v[j][0].y, v[j][0].z, v[j][0].w, v[j][1].x, v[j][1].y, v[j][1].z, v[j][1].w};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float a = (i & 1) ? bf16hi(w[i >> 1]) : bf16lo(w[i >> 1]);
      const int V = (int)rintf(ldexpf(a, e));   // |V| <= 2^22
      res += fabs((double)a - (double)V * inv);
      const int d0 = ((V + 128) & 255) - 128;
      const int V1 = (V - d0) / 256;
      const int d1 = ((V1 + 128) & 255) - 128;
      const int d2 = (V1 - d1) / 256;
      s0 += (double)abs(d0);
      m0 = max(m0, abs(d0));
      d[0][i >> 2] |= (uint32_t)(d0 & 255) << (8 * (i & 3));
      d[1][i >> 2] |= (uint32_t)(d1 & 255) << (8 * (i & 3));
      d[2][i >> 2] |= (uint32_t)(d2 & 255) << (8 * (i & 3));
    }
#pragma unroll
    for (int q = 0; q < 3; ++q)
      *(uint4*)(dig + rt_dig_off(r, c, q, nstg)) = make_uint4(d[q][0], d[q][1], d[q][2], d[q][3]);
  }
  // block sums (fixed order: warp shuffles, then the warps in index order)
  double part[4] = {sa, res, s0, g};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    part[i] = warp_sum_f64(part[i]);
    if (lane == 0) red[i][warp] = part[i];
  }
  m0 = (int)__reduce_max_sync(0xffffffffu, (unsigned)m0);
  __syncthreads();
  if (lane == 0) redm[warp] = (float)m0;   // after the barrier: every thread has read the maxima
  __syncthreads();
  if (tid == 0) {
    double tot[4] = {0.0, 0.0, 0.0, 0.0};
    float mm = 0.f;
    for (int w = 0; w < kRdThreads / 32; ++w) {
#pragma unroll
      for (int i = 0; i < 4; ++i) tot[i] += red[i][w];
      mm = fmaxf(mm, redm[w]);
    }
    double* st = (isw ? p.wst : p.xst) + kRtStat * (size_t)r;
    st[0] = inv;
    st[1] = tot[0];
    st[2] = (double)mx;
    st[3] = tot[1];
    st[4] = tot[2];
    st[5] = (double)mm;
    st[6] = 0.0;
    st[7] = 0.0;
    if (gw) p.logits[(size_t)r * (p.E + 1) + p.E] = tot[3];
  }
}

// ------------------------------------------------------------------ integer GEMM
// grid (rows_w / 128, rows_x / 128, splits), block 128. Stage u holds, for
// kRtKS columns, the three digit planes of the CTA's 128 router rows (A) and
// of its 128 tokens (B), each a contiguous 24 KB block of the tiled layout
// (plane q, chunk c of 16 columns, row r at q 8 KB + c 2 KB + r 16). Thread 0
// brings them (two bulk copies), thread 32 issues per stage 8 digit pairs x
// 2 MMAs (K = 32) into the class accumulators (columns 128 s); all four warps
// then read tensor memory (thread = router row) and write the split's exact
// partial sum_s 2^(8(s+1)) acc_s as int64.
struct RtSmem {
  uint64_t full[kRtStages], empty[kRtStages], done;
  uint32_t tslot;
  int abort;
};

__global__ void __launch_bounds__(128, 1) route_tc_kernel(RouteParams p, int splits) {
  const unsigned long long wait_ns = p.wait_ns;
  uint32_t* status = p.status;
  extern __shared__ __align__(1024) unsigned char smem[];
  RtSmem& S = *(RtSmem*)(smem + kRtStages * kRtStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int mt = blockIdx.x, nt = blockIdx.y, split = blockIdx.z;
  const int nstg = p.H / kRtKS;
  const int i0 = (int)((long long)nstg * split / splits), i1 = (int)((long long)nstg * (split + 1) / splits);
  const int n = i1 - i0;
  if (tid == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.done, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) tc_alloc(&S.tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tslot;
  volatile int* abort_flag = &S.abort;

  if (tid == 0) {   // ---------------------------------------------------- digit tiles
    int last[kRtStages];
    for (int s = 0; s < kRtStages; ++s) last[s] = -1;
    const int8_t* wsrc = p.wdig + ((size_t)mt * nstg + i0) * kRtTile;
    const int8_t* xsrc = p.xdig + ((size_t)nt * nstg + i0) * kRtTile;
    for (int u = 0; u < n; ++u) {
      const int slot = u % kRtStages, use = u / kRtStages;
      if (use > 0 && !mbar_wait_bounded(&S.empty[slot], (use - 1) & 1, wait_ns, status)) *abort_flag = 1;
      if (*abort_flag) break;
      unsigned char* st = smem + (size_t)slot * kRtStageBytes;
      mbar_expect_tx(&S.full[slot], (unsigned)kRtStageBytes);
      bulk_g2s(st, wsrc + (size_t)u * kRtTile, kRtTile, &S.full[slot]);
      bulk_g2s(st + kRtTile, xsrc + (size_t)u * kRtTile, kRtTile, &S.full[slot]);
      last[slot] = use;
    }
    for (int s = 0; s < kRtStages; ++s)   // no copy may land after the CTA has left
      if (last[s] >= 0) mbar_wait_bounded(&S.full[s], last[s] & 1, wait_ns, status);
  } else if (tid == 32) {   // --------------------------------------------- MMA issue
    // s32 accumulators, A and B signed 8-bit, both K-major, M = 128, N = 128
    const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kRtN >> 3) << 17) |
                           ((uint32_t)(kRtM >> 4) << 24);
    bool started[kRtClasses] = {false, false, false, false};
    for (int u = 0; u < n; ++u) {
      const int slot = u % kRtStages, ph = (u / kRtStages) & 1;
      if (!mbar_wait_bounded(&S.full[slot], ph, wait_ns, status)) *abort_flag = 1;
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + (size_t)slot * kRtStageBytes), b0 = a0 + kRtTile;
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          if (i + j == 0) continue;   // the low pair: bounded, not computed
          const int cls = i + j - 1;
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const uint64_t ad = tc_smem_desc(a0 + i * kRtPlane + 2 * ks * kRtChunk, kRtChunk, 128);
            const uint64_t bd = tc_smem_desc(b0 + j * kRtPlane + 2 * ks * kRtChunk, kRtChunk, 128);
            const uint32_t acc = started[cls] ? 1u : 0u, z = 0u;
            asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                         " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n"
                         :: "r"(tbase + (uint32_t)(cls * kRtN)), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(z)
                         : "memory");
            started[cls] = true;
          }
        }
      tc_commit(&S.empty[slot]);
    }
    tc_commit(&S.done);
    mbar_wait_bounded(&S.done, 0, wait_ns, status);
  }
  // -------------------------------------------------------------------- epilogue (all warps)
  __syncwarp();
  bool ok = mbar_wait_bounded(&S.done, 0, wait_ns, status) && !*abort_flag;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();
  if (ok) {
    const int e = mt * kRtM + tid, t0 = nt * kRtN;
    const uint32_t lane_addr = tbase + ((uint32_t)(warp * 32) << 16);
    long long* out = p.lpart + (size_t)split * p.T * p.E + e;
    for (int c0 = 0; c0 < kRtN; c0 += 16) {
      uint32_t r[kRtClasses][16];
#pragma unroll
      for (int s = 0; s < kRtClasses; ++s) tc_ld16(lane_addr + s * kRtN + c0, r[s]);
      tc_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        long long v = 0;
#pragma unroll
        for (int s = 0; s < kRtClasses; ++s) v += (long long)(int)r[s][j] * (1LL << (8 * (s + 1)));
        const int t = t0 + c0 + j;
        if (t < p.T && e < p.E) out[(size_t)t * p.E] = v;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tc_dealloc(tbase, 512);
}

// ------------------------------------------------------------------ logits and bounds
// grid T, block kRdThreads: logit = (the splits' exact sum) 2^-(p_t + q_e) + bias, and its bound.
__global__ void __launch_bounds__(kRdThreads) route_tc_combine_kernel(RouteParams p, int splits) {
  const int t = blockIdx.x;
  const size_t ld = (size_t)p.E + 1;
  const double* xst = p.xst + kRtStat * (size_t)t;
  const double xs = xst[0], xmax = xst[2], xres = xst[3], xs0 = xst[4], xm0 = xst[5];
  const double H1 = (double)(p.H - 1);
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    long long tot = 0;
#pragma unroll
    for (int q = 0; q < kRtSplitMax; ++q)
      if (q < splits) tot += __ldcg(p.lpart + ((size_t)q * p.T + t) * p.E + e);
    const double* wst = p.wst + kRtStat * (size_t)e;
    const double ws = wst[0], wsum = wst[1], wmax = wst[2], wres = wst[3], ws0 = wst[4], wm0 = wst[5];
    const double sc = xs * ws;   // a power of two
    const double bias = p.router_bias ? (double)p.router_bias[e] : 0.0;
    const double l = (double)tot * sc + bias;
    p.logits[(size_t)t * ld + e] = l;
    if (p.bound) {
      const double b = xres * wmax + wres * (xmax + xs) + sc * fmin(ws0 * xm0, xs0 * wm0) +
                       H1 * 0x1p-53 * xmax * wsum + 0x1p-52 * (fabs(l) + fabs(bias));
      p.bound[(size_t)t * ld + e] = __double2float_ru(1.01 * b);
    }
  }
}

cudaError_t launch_route_gemm(const RouteParams& p, cudaStream_t s) {
  const int rw = (int)route_tc_rows_w(p.E), rx = (int)route_tc_rows_x(p.T);
  if (p.H % kRtKS || p.H > kRdThreads * kRdMaxChunks * 16) return cudaErrorInvalidConfiguration;
  RouteParams q = p;
  void* args1[] = {&q};
  cudaError_t e = cudaLaunchKernel((const void*)route_digits_kernel, dim3(rw + rx), dim3(kRdThreads), args1, 0, s);
  if (e != cudaSuccess) return e;
  const int tiles = (rw / kRtM) * (rx / kRtN), nstg = p.H / kRtKS;
  int splits = num_sms() / tiles;
  splits = splits < 1 ? 1 : (splits > kRtSplitMax ? kRtSplitMax : splits);
  splits = splits > nstg ? nstg : splits;
  const size_t sm = (size_t)kRtStages * kRtStageBytes + sizeof(RtSmem);
  e = set_func_attr((const void*)route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  void* args2[] = {&q, &splits};
  e = cudaLaunchKernel((const void*)route_tc_kernel, dim3(rw / kRtM, rx / kRtN, splits), dim3(128), args2, sm, s);
  if (e != cudaSuccess) return e;
  void* args3[] = {&q, &splits};
  return cudaLaunchKernel((const void*)route_tc_combine_kernel, dim3(p.T), dim3(kRdThreads), args3, 0, s);
}

}  // namespace qmoe
