// Router logits of many tokens (prefill) in exact integer arithmetic on the
// tcgen05 tensor cores, with a rigorous bound on each logit's distance to the
// definition (the index-order fp64 sum of the exact bf16 products, bias added
// last), for the certified top-k of topk.cuh.
//
// Every router row (and the shared-gate row) and every token is written as
// 22-bit fixed point with its own power-of-two scale: V = rint(v 2^p) with
// max |v| 2^p < 2^22, split exactly into three balanced signed 8-bit digits,
// V = d2 2^16 + d1 2^8 + d0. The integer dot products of the digits (9 pairs,
// kind::i8 MMAs, s32 accumulators in tensor memory) are exact; pairs of equal
// weight 2^(8(i+j)) share one accumulator (five classes, each below 2^28 in
// magnitude). The logit is then sum_s 2^(8s) acc_s 2^-(p_t + q_e), in fp64,
// plus the bias.
//
// Bound. With x~ = X 2^-p, w~ = W 2^-q, dx = x - x~, dw = w - w~:
//   |sum x w - sum x~ w~| = |sum dx w + x~ dw| <= sum|dx| max|w| + sum|dw| max|x~|,
// max|x~| <= max|x| + 2^-p; the digits kernel sums the residuals |dv| of each
// row (in fp64: v and V 2^-p are exact there), and most bf16 values are exact
// in 22-bit fixed point, so these terms are small;
// the definition's index-order fp64 sum is within (H+1) 2^-53 max|x| sum|w|
// of the exact dot product (Higham, Accuracy and Stability of Numerical
// Algorithms, sec. 4.2); our fp64 combination of the classes and splits adds
// at most 16 2^-53 max|x| sum|w| (every integer term converts exactly); the
// bias additions cost 2^-52 (|l| + |b|). The sum, times 1.01, is rounded up
// to fp32.
//
// Kernels: route_digits_kernel (a warp per row: scale, sums, digit planes in
// the tensor cores' K-major tile layout), route_tc_kernel (one CTA per 128
// router rows x 64 tokens x column split; one thread brings the digit tiles
// with bulk copies, one issues the MMAs, four warps read tensor memory and
// write the split's partial logit), route_tc_combine_kernel.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "sync.cuh"
#include "tc.cuh"

namespace qmoe {

constexpr int kRtM = 128;          // router rows per CTA (one MMA tile)
constexpr int kRtN = 64;           // tokens per CTA
constexpr int kRtKS = 64;          // columns per stage
constexpr int kRtStages = 4;
constexpr int kRtClasses = 5;      // digit pairs grouped by i + j
constexpr int kRtPlaneA = kRtKS / 16 * kRtM * 16;   // one digit plane of a weight tile: 8 KB
constexpr int kRtPlaneB = kRtKS / 16 * kRtN * 16;   // one digit plane of a token tile: 4 KB
constexpr int kRtStageBytes = 3 * (kRtPlaneA + kRtPlaneB);

static_assert(kRtM == 128 && kRtN == 64, "route_tc_rows_w / route_tc_rows_x pad to these tiles");

// ------------------------------------------------------------------ digits
// grid ceil((rows_w + rows_x) / 8), block 256: a warp per row. Row r < rows_w
// is router row r (r == E: the shared-gate row; beyond: zeros), then the
// tokens (beyond T: zeros). Lane l handles 16-element chunks c = l + 32 i.
__global__ void __launch_bounds__(256) route_digits_kernel(RouteParams p) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int rw = (int)route_tc_rows_w(p.E), rx = (int)route_tc_rows_x(p.T);
  if (row >= rw + rx) return;
  const bool isw = row < rw;
  const int r = isw ? row : row - rw;
  const int nrows = p.E + (p.has_shared ? 1 : 0);
  const uint16_t* src = isw ? (r < p.E ? p.router_w + (size_t)r * p.H : (r < nrows ? p.gate_w : nullptr))
                            : (r < p.T ? p.x + (size_t)r * p.H : nullptr);
  const int nch = p.H / 16, rows = isw ? rw : rx;
  int8_t* dig = isw ? p.wdig : p.xdig;
  double* st = (isw ? p.wst : p.xst) + 4 * (size_t)r;
  float mx = 0.f;
  double sa = 0.0;
  if (src)
    for (int c = lane; c < nch; c += 32) {
      const uint4 a = __ldg((const uint4*)(src + 16 * c)), b = __ldg((const uint4*)(src + 16 * c) + 1);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float v0 = fabsf(bf16lo(w[j])), v1 = fabsf(bf16hi(w[j]));
        mx = fmaxf(mx, fmaxf(v0, v1));
        sa += (double)v0 + (double)v1;
      }
    }
  mx = warp_max(mx);
  sa = warp_sum_f64(sa);
  int e = 0;
  if (mx > 0.f) {   // max |v| 2^e < 2^22
    int E2;
    frexpf(mx, &E2);
    e = 22 - E2;
  }
  const double inv = ldexp(1.0, -e);
  double res = 0.0;   // sum of |v - V 2^-e| over the row
  for (int c = lane; c < nch; c += 32) {
    uint32_t d[3][4] = {};
    if (src) {
      const uint4 a = __ldg((const uint4*)(src + 16 * c)), b = __ldg((const uint4*)(src + 16 * c) + 1);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float v = (j & 1) ? bf16hi(w[j >> 1]) : bf16lo(w[j >> 1]);
        const int V = (int)rintf(ldexpf(v, e));   // |V| <= 2^22
        res += fabs((double)v - (double)V * inv);
        const int d0 = ((V + 128) & 255) - 128;
        const int V1 = (V - d0) / 256;
        const int d1 = ((V1 + 128) & 255) - 128;
        const int d2 = (V1 - d1) / 256;
        d[0][j >> 2] |= (uint32_t)(d0 & 255) << (8 * (j & 3));
        d[1][j >> 2] |= (uint32_t)(d1 & 255) << (8 * (j & 3));
        d[2][j >> 2] |= (uint32_t)(d2 & 255) << (8 * (j & 3));
      }
    }
#pragma unroll
    for (int q = 0; q < 3; ++q)
      *(uint4*)(dig + (((size_t)q * nch + c) * rows + r) * 16) = make_uint4(d[q][0], d[q][1], d[q][2], d[q][3]);
  }
  res = warp_sum_f64(res);
  if (lane == 0) {   // {2^-e, sum |v|, max |v|, sum |v - V 2^-e|}
    st[0] = inv;
    st[1] = sa;
    st[2] = (double)mx;
    st[3] = res;
  }
}

// ------------------------------------------------------------------ integer GEMM
// grid (rows_w / 128, rows_x / 64, splits), block 128. Stage u holds, for
// kRtKS columns, the three digit planes of the CTA's 128 router rows (A) and
// of its 64 tokens (B), each plane as 4 chunks of 16 columns (chunk c of row
// r at c * rows * 16 + r * 16). Thread 0 brings them (bulk copies), thread 32
// issues per stage 9 digit pairs x 2 MMAs (K = 32) into the class
// accumulators (columns 64 s); all four warps then read tensor memory (thread
// = router row) and write the split's partial logit sum_s 2^(8s) acc_s.
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
  const int rw = (int)route_tc_rows_w(p.E), rx = (int)route_tc_rows_x(p.T);
  const int m0 = blockIdx.x * kRtM, t0 = blockIdx.y * kRtN, split = blockIdx.z;
  const int nch = p.H / 16, nstg = p.H / kRtKS;
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
    for (int u = 0; u < n; ++u) {
      const int slot = u % kRtStages, use = u / kRtStages, c0 = (i0 + u) * (kRtKS / 16);
      if (use > 0 && !mbar_wait_bounded(&S.empty[slot], (use - 1) & 1, wait_ns, status)) *abort_flag = 1;
      if (*abort_flag) break;
      unsigned char* st = smem + (size_t)slot * kRtStageBytes;
      mbar_expect_tx(&S.full[slot], (unsigned)kRtStageBytes);
      for (int q = 0; q < 3; ++q)
        for (int cc = 0; cc < kRtKS / 16; ++cc) {
          const size_t cq = (size_t)q * nch + c0 + cc;
          bulk_g2s(st + (q * 4 + cc) * (kRtM * 16), p.wdig + (cq * rw + m0) * 16, kRtM * 16, &S.full[slot]);
          bulk_g2s(st + 3 * kRtPlaneA + (q * 4 + cc) * (kRtN * 16), p.xdig + (cq * rx + t0) * 16, kRtN * 16,
                   &S.full[slot]);
        }
      last[slot] = use;
    }
    for (int s = 0; s < kRtStages; ++s)   // no copy may land after the CTA has left
      if (last[s] >= 0) mbar_wait_bounded(&S.full[s], last[s] & 1, wait_ns, status);
  } else if (tid == 32) {   // --------------------------------------------- MMA issue
    // s32 accumulators, A and B signed 8-bit, both K-major, M = 128, N = 64
    const uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kRtN >> 3) << 17) |
                           ((uint32_t)(kRtM >> 4) << 24);
    bool started[kRtClasses] = {false, false, false, false, false};
    for (int u = 0; u < n; ++u) {
      const int slot = u % kRtStages, ph = (u / kRtStages) & 1;
      if (!mbar_wait_bounded(&S.full[slot], ph, wait_ns, status)) *abort_flag = 1;
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(smem + (size_t)slot * kRtStageBytes), b0 = a0 + 3 * kRtPlaneA;
#pragma unroll
      for (int i = 0; i < 3; ++i)
#pragma unroll
        for (int j = 0; j < 3; ++j)
#pragma unroll
          for (int ks = 0; ks < 2; ++ks) {
            const int cls = i + j;
            const uint64_t ad = tc_smem_desc(a0 + (i * 4 + 2 * ks) * (kRtM * 16), kRtM * 16, 128);
            const uint64_t bd = tc_smem_desc(b0 + (j * 4 + 2 * ks) * (kRtN * 16), kRtN * 16, 128);
            const uint32_t acc = started[cls] ? 1u : 0u, z = 0u;
            asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                         " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n"
                         :: "r"(tbase + (uint32_t)(cls * kRtN)), "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(z)
                         : "memory");
            started[cls] = true;
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
    const int e = m0 + tid;
    const int nrows = p.E + (p.has_shared ? 1 : 0);
    const size_t ld = (size_t)p.E + 1;
    const uint32_t lane_addr = tbase + ((uint32_t)(warp * 32) << 16);
    for (int c0 = 0; c0 < kRtN; c0 += 16) {
      double v[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.0;
#pragma unroll
      for (int s = 0; s < kRtClasses; ++s) {
        uint32_t r[16];
        tc_ld16(lane_addr + s * kRtN + c0, r);
        tc_wait_ld();
        const double w = ldexp(1.0, 8 * s);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += (double)(int)r[j] * w;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = t0 + c0 + j;
        if (t < p.T && e < nrows) p.lpart[((size_t)split * p.T + t) * ld + e] = v[j];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tc_dealloc(tbase, 512);
}

// ------------------------------------------------------------------ logits and bounds
// grid T, block 512: logit = (sum of the splits) 2^-(p_t + q_e) + bias, and its bound.
// The shared-gate logit (column E) is the fp64 sum of its exact products instead (a block reduction).
__global__ void __launch_bounds__(kThreads) route_tc_combine_kernel(RouteParams p, int splits) {
  __shared__ double red[kThreads / 32];
  const int t = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const size_t ld = (size_t)p.E + 1;
  const double* xst = p.xst + 4 * (size_t)t;
  const double xs = xst[0], xmax = xst[2], xres = xst[3];
  if (p.has_shared) {
    double g = 0.0;
    const uint16_t* xr = p.x + (size_t)t * p.H;
    for (int k = threadIdx.x; k < p.H; k += blockDim.x)
      g += (double)bf16_to_f32(xr[k]) * (double)bf16_to_f32(p.gate_w[k]);
    g = warp_sum_f64(g);
    if (lane == 0) red[warp] = g;
    __syncthreads();
    if (threadIdx.x == 0) {
      double tot = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) tot += red[w];
      p.logits[(size_t)t * ld + p.E] = tot;
    }
  }
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) {
    double l = 0.0;
    for (int q = 0; q < splits; ++q) l += p.lpart[((size_t)q * p.T + t) * ld + e];
    const double* wst = p.wst + 4 * (size_t)e;
    const double ws = wst[0], wsum = wst[1], wmax = wst[2], wres = wst[3];
    l = l * xs * ws;   // powers of two: exact
    const double bias = p.router_bias ? (double)p.router_bias[e] : 0.0;
    l += bias;
    p.logits[(size_t)t * ld + e] = l;
    if (p.bound) {
      const double H = (double)p.H;
      const double b = xres * wmax + wres * (xmax + xs) + (H + 17.0) * 0x1p-53 * xmax * wsum +
                       0x1p-52 * (fabs(l) + fabs(bias));
      p.bound[(size_t)t * ld + e] = __double2float_ru(1.01 * b);
    }
  }
}

cudaError_t launch_route_gemm(const RouteParams& p, cudaStream_t s) {
  const int rw = (int)route_tc_rows_w(p.E), rx = (int)route_tc_rows_x(p.T);
  if (p.H % kRtKS) return cudaErrorInvalidConfiguration;
  RouteParams q = p;
  void* args1[] = {&q};
  cudaError_t e = cudaLaunchKernel((const void*)route_digits_kernel, dim3((rw + rx + 7) / 8), dim3(256), args1, 0, s);
  if (e != cudaSuccess) return e;
  const int blocks = (rw / kRtM) * (rx / kRtN), nstg = p.H / kRtKS;
  int splits = num_sms() / blocks;
  splits = splits < 1 ? 1 : (splits > kRgSplit ? kRgSplit : splits);
  splits = splits > nstg ? nstg : splits;
  const size_t sm = (size_t)kRtStages * kRtStageBytes + sizeof(RtSmem);
  e = cudaFuncSetAttribute((const void*)route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  void* args2[] = {&q, &splits};
  e = cudaLaunchKernel((const void*)route_tc_kernel, dim3(rw / kRtM, rx / kRtN, splits), dim3(128), args2, sm, s);
  if (e != cudaSuccess) return e;
  void* args3[] = {&q, &splits};
  return cudaLaunchKernel((const void*)route_tc_combine_kernel, dim3(p.T), dim3(kThreads), args3, 0, s);
}

}  // namespace qmoe
