// The shared expert of a prefill batch on the tcgen05 tensor cores.
//
// The shared expert sees every token of the batch, so for a few hundred
// tokens its gate/up and down projections are dense GEMMs (12.9 GFLOP at 512
// tokens of a hidden-4096 layer) rather than mat-vecs. They run here as
// tcgen05 MMAs (kind::f16, fp32 accumulators in tensor memory) on an exact
// fp16 form of the quantised weights; the routed experts, with a few tokens
// each, stay on the grouped integer kernels of prefill.cu.
//
// Exact operands. A weight of group g is w = q*s + b ("Key technologies >
// FMA-optimised dequant kernel" of the Flash-MoE write-up). With c = 8 for
// 4-bit codes and c = 2 for 2-bit codes,
//     w = s*(q - c) + beta_g,   beta_g = b + c*s,
// and s*(q - c) is exact in fp16: s is a bf16 (8 significant bits), q - c has
// at most 3, and a power-of-two scale 2^e per weight row keeps every value of
// the row inside fp16's normal range. The beta term enters the same MMA as
// extra columns: per group four columns (beta_hi, beta_lo, beta_hi, beta_lo)
// against the token's (S_hi, S_hi, S_lo, S_lo), S_g the sum of the token's
// activations over the group, so the products add up to (beta_hi + beta_lo)
// * (S_hi + S_lo), each split to about 22 bits. These columns follow the K
// data columns: Kx = K + 64*ceil(K/1024) columns in all (tc_cols).
//
// Activations: each token's vector is scaled by 2^p (max |v| 2^p < 2^9, so
// the group sums also stay below fp16's range) and stored as fp16. x (bf16)
// is exact in fp16; the SwiGLU outputs a (fp32) are stored as hi + lo fp16
// parts, two MMA accumulators whose sum carries about 22 bits of a.
//
// Order inside a 16-byte column chunk. The MMA sums over k in any order, as
// long as both operands use the same one. The weight chunks are written in
// the order the magic-number conversion produces them from a packed word
// (fp16 0x6400 | q = 1024 + q): 4-bit codes come out as pairs (q_t, q_t+4),
// 2-bit codes as (q_t, q_t+8), and the activation tables use the same order.
//
// Passes (one launch each):
//   tc_conv_kernel (x)   x -> fp16 tables + group-sum columns, 2^-p per token
//   tc_dense_kernel      part[s][t][m] over the gate and up rows of the shared expert
//   tc_conv_kernel (a)   sum the splits, SwiGLU, -> hi/lo tables + group sums
//   tc_dense_kernel      part[s][t][h] over the down rows
// and the prefill combine adds the down pass's splits in order.
//
// The dense kernel: one CTA per (128 weight rows, up to 256 tokens, column
// split). Warps 0-3 dequantise a 128 x 64 weight tile per stage (one thread
// per row) and run the epilogue (thread = tensor-memory lane = row); warp 4
// allocates tensor memory and one of its threads issues the MMAs; one thread
// of warp 5 brings the activation tiles with bulk copies. Stages are handed
// over on mbarriers (tiles full: producers' arrivals and the copies' bytes;
// tiles free: tcgen05.commit), every wait bounded.
#include <math.h>

#include "common.cuh"
#include "kernels.cuh"
#include "stage.cuh"
#include "sync.cuh"
#include "tc.cuh"

namespace qmoe {

constexpr int kTcM = 128;                    // weight rows per CTA (one MMA tile, one TMEM lane each)
constexpr int kTcKS = 64;                    // columns per stage
constexpr int kTcProducers = 128;            // warps 0-3
constexpr int kTcThreads = 192;              // + warp 4 (TMEM, MMA) + warp 5 (operand copies)
constexpr int kTcMaxStages = 6;
constexpr int kTcMaxSplits = 8;
constexpr int kTcMaxNt = 256;
constexpr int kTcABytes = kTcKS / 8 * kTcM * 16;   // one weight tile: 16 KB
constexpr int kTcConvThreads = 256;

static int tc_pad16(int T) { return (T + 15) & ~15; }
static int tc_nt(int T) { return tc_pad16(T) < kTcMaxNt ? tc_pad16(T) : kTcMaxNt; }

int tc_splits(int M, int T, int K) {
  const int nt = tc_nt(T);
  const int blocks = (M / kTcM) * ((tc_pad16(T) + nt - 1) / nt);
  const int nstg = tc_cols(K) / kTcKS;
  int s = num_sms() / (blocks > 0 ? blocks : 1);
  if (s > kTcMaxSplits) s = kTcMaxSplits;
  if (s > nstg) s = nstg;
  return s < 1 ? 1 : s;
}

__device__ __forceinline__ float tc_pow2(int e) { return ldexpf(1.f, e); }
// exponent e with v * 2^e < 2^lim (v > 0), clamped; 0 for v = 0
__device__ __forceinline__ int tc_exp_below(float v, int lim) {
  if (!(v > 0.f)) return 0;
  int E;
  frexpf(v, &E);   // v < 2^E
  int e = lim - E;
  return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// ------------------------------------------------------------------ operand tables
// Token CTAs: tw = min(256, max(32, pow2 >= K/16)) threads per token, 256/tw
// tokens per CTA; each thread holds 16-element spans of its token's values in
// registers (span sp = lane-in-token + tw q). Values v: the bf16 input x, or
// the SwiGLU of the gate/up pass's split sums (added in split order). Writes
// the token's fp16 columns (hi, and lo when b_lo is given) in chunk order, the
// group-sum columns, and 2^-p. Padding tokens (T <= t < Tpad) get zero
// columns. Row CTAs (after the token CTAs, one thread per weight row of the
// matrices in prep): the row exponent and the bias-column tiles.
constexpr int kTcConvSpans = 2;   // spans per thread: K <= 16 * 256 * 2

// element of a 16-element span held at position e of its chunk h (0 or 1)
template <int BITS>
__host__ __device__ constexpr int tc_span_elem(int h, int e) {
  return BITS == 4 ? 8 * h + (e >> 1) + 4 * (e & 1) : 4 * h + (e >> 1) + 8 * (e & 1);
}
__host__ __device__ inline int tc_token_threads(int K) {
  int tw = 32;
  while (tw < K / 16 && tw < kTcConvThreads) tw <<= 1;
  return tw;
}

// One weight row, one warp: e with max(c|s_g|, |beta_g|) 2^e < 2^14 over all
// its groups, then its bias columns (beta_hi, beta_lo, beta_hi, beta_lo per
// group, scaled by 2^e) in the dense kernel's tile layout. Lane l takes the
// column chunks j = l + 32 q, chunk j holding groups 2j and 2j+1.
constexpr int kTcPrepChunks = 2;   // chunks per lane: K <= 64 * 2 * 32 * kTcPrepChunks
template <int BITS>
__device__ void tc_prep_row(const TcRowPrep& P, int m) {
  constexpr float cq = BITS == 4 ? 8.f : 2.f;
  const int lane = threadIdx.x & 31;
  const int ng = P.K / kGroup, nxs = tc_cols(P.K) / 64 - ng;
  const bool second = m >= P.R0;
  const moe_qmat W = second ? P.w1 : P.w0;
  const int r = second ? m - P.R0 : m;
  const uint32_t* srow = (const uint32_t*)(W.scales + (size_t)r * ng);   // ng is even: bf16 pairs
  const uint32_t* brow = (const uint32_t*)(W.biases + (size_t)r * ng);
  float beta[kTcPrepChunks][2];
  float mx = 0.f;
#pragma unroll
  for (int q = 0; q < kTcPrepChunks; ++q) {
    const int j = lane + 32 * q;
    const bool in = j < ng / 2;
    const uint32_t sv = in ? __ldg(srow + j) : 0u, bv = in ? __ldg(brow + j) : 0u;
    const float s0 = bf16lo(sv), s1 = bf16hi(sv);
    beta[q][0] = fmaf(cq, s0, bf16lo(bv));
    beta[q][1] = fmaf(cq, s1, bf16hi(bv));
    mx = fmaxf(mx, fmaxf(cq * fmaxf(fabsf(s0), fabsf(s1)), fmaxf(fabsf(beta[q][0]), fabsf(beta[q][1]))));
  }
  mx = warp_max(mx);
  const int e = tc_exp_below(mx, 14);
  if (lane == 0) P.rexp[m] = e;
  const float rsc = tc_pow2(e);
  uint4* tile = (uint4*)P.aext + (size_t)(m / kTcM) * nxs * 8 * kTcM + (m % kTcM);
#pragma unroll
  for (int q = 0; q < kTcPrepChunks; ++q) {
    const int j = lane + 32 * q;   // chunk j = stage j / 8, chunk j % 8 of it
    if (j < nxs * 8) {
      uint32_t v[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float bt = j < ng / 2 ? beta[q][h] * rsc : 0.f;
        const uint32_t hl = pack_half2(half_hi(bt), half_lo(bt));
        v[2 * h] = hl;
        v[2 * h + 1] = hl;
      }
      tile[(size_t)j * kTcM] = make_uint4(v[0], v[1], v[2], v[3]);
    }
  }
}

template <int BITS>
__global__ void __launch_bounds__(kTcConvThreads) tc_conv_kernel(TcConvParams p) {
  __shared__ float red[kTcConvThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31;
  const int K = p.K, nsp = K / 16, ng = K / kGroup, nck = K / 8, nxk = tc_cols(K) / 8 - nck;
  const int tw = tc_token_threads(K), tpc = kTcConvThreads / tw;
  const int ntb = (p.Tpad + tpc - 1) / tpc;   // token CTAs
  if ((int)blockIdx.x >= ntb) {   // ---------------------------------------- weight rows, a warp each
    int m = (blockIdx.x - ntb) * (kTcConvThreads / 32) + (tid >> 5);
    for (int j = 0; j < p.nprep; ++j) {
      if (m < p.prep[j].M) {
        tc_prep_row<BITS>(p.prep[j], m);
        return;
      }
      m -= p.prep[j].M;
    }
    return;
  }
  const int sub = tid / tw, lt = tid % tw;
  const int t = blockIdx.x * tpc + sub;
  const bool real = t < p.T, live = t < p.Tpad;
  float v[kTcConvSpans][16];
  float m = 0.f;
#pragma unroll
  for (int q = 0; q < kTcConvSpans; ++q) {
    const int sp = lt + q * tw;
#pragma unroll
    for (int e = 0; e < 16; ++e) v[q][e] = 0.f;
    if (!real || sp >= nsp) continue;
    if (p.x) {
      const uint4* src = (const uint4*)(p.x + (size_t)t * K + 16 * sp);
      const uint4 a = __ldg(src), b = __ldg(src + 1);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[q][2 * j] = bf16lo(w[j]);
        v[q][2 * j + 1] = bf16hi(w[j]);
      }
    } else {   // SwiGLU of the gate/up split sums, splits added in order
      float g[16], u[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) g[e] = u[e] = 0.f;
      for (int s = 0; s < p.splits; ++s) {
        const float* row = p.part + ((size_t)s * p.T + t) * (2 * (size_t)p.I) + 16 * sp;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 gg = __ldcg((const float4*)row + j), uu = __ldcg((const float4*)(row + p.I) + j);
          g[4 * j] += gg.x; g[4 * j + 1] += gg.y; g[4 * j + 2] += gg.z; g[4 * j + 3] += gg.w;
          u[4 * j] += uu.x; u[4 * j + 1] += uu.y; u[4 * j + 2] += uu.z; u[4 * j + 3] += uu.w;
        }
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) v[q][e] = silu_f32(g[e]) * u[e];
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[q][e]));
  }
  // the token's max -> 2^p with max|v| 2^p < 2^9
  m = warp_max(m);
  if (lane == 0) red[tid >> 5] = m;
  __syncthreads();
  float mx = 0.f;
  for (int w = sub * (tw / 32); w < (sub + 1) * (tw / 32); ++w) mx = fmaxf(mx, red[w]);
  const int pe = tc_exp_below(mx, 9);
  const float sc = tc_pow2(pe);
  if (lt == 0 && live) p.tscale[t] = real ? tc_pow2(-pe) : 0.f;
#pragma unroll
  for (int q = 0; q < kTcConvSpans; ++q) {
    const int sp = lt + q * tw;
    float ssum = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      v[q][e] *= sc;
      ssum += v[q][e];
    }
    // a group is 4 spans = 4 consecutive lanes
    ssum += __shfl_xor_sync(0xffffffffu, ssum, 1);
    ssum += __shfl_xor_sync(0xffffffffu, ssum, 2);
    const float snext = __shfl_down_sync(0xffffffffu, ssum, 4);   // the next group's sum
    if (sp >= nsp || !live) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float v0 = v[q][tc_span_elem<BITS>(h, e)], v1 = v[q][tc_span_elem<BITS>(h, e + 1)];
        hi[e / 2] = pack_half2(half_hi(v0), half_hi(v1));
        lo[e / 2] = pack_half2(half_lo(v0), half_lo(v1));
      }
      const size_t o = ((size_t)(2 * sp + h) * p.Tpad + t) * 8;
      *(uint4*)(p.b_hi + o) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      if (p.b_lo) *(uint4*)(p.b_lo + o) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    // group-sum columns: chunk j holds groups 2j, 2j+1 as (S_hi, S_hi, S_lo, S_lo)
    if ((sp & 7) == 0) {
      uint32_t w[4];
      const float sg[2] = {ssum, snext};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const __half sh = half_hi(sg[h]), sl = half_lo(sg[h]);
        w[2 * h] = pack_half2(sh, sh);
        w[2 * h + 1] = pack_half2(sl, sl);
      }
      const size_t o = ((size_t)(nck + sp / 8) * p.Tpad + t) * 8;
      *(uint4*)(p.b_hi + o) = make_uint4(w[0], w[1], w[2], w[3]);
      if (p.b_lo) *(uint4*)(p.b_lo + o) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // padding group-sum columns (groups ng and above)
  if (live)
    for (int j = ng / 2 + lt; j < nxk; j += tw) {
      const size_t o = ((size_t)(nck + j) * p.Tpad + t) * 8;
      *(uint4*)(p.b_hi + o) = make_uint4(0u, 0u, 0u, 0u);
      if (p.b_lo) *(uint4*)(p.b_lo + o) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// ------------------------------------------------------------------ dense pass
// Shared-memory plan of the dense kernel: nst weight tiles (16 KB each), nst
// activation tiles (brows rows of 8 chunks: hi rows [0, nt), lo rows [nt, 2nt)),
// the mbarriers, the tensor-memory address, an abort flag, the token scales.
struct TcGeom {
  int brows;
  size_t stage_b, a_off, b_off, bar_off, tsc_off, total;
};
__host__ __device__ inline TcGeom tc_geom(int nt, int hilo, int nst) {
  TcGeom G;
  G.brows = nt * (hilo ? 2 : 1);
  G.stage_b = (size_t)G.brows * 16 * (kTcKS / 8);
  G.a_off = 0;
  G.b_off = (size_t)nst * kTcABytes;
  G.bar_off = G.b_off + (size_t)nst * G.stage_b;
  G.tsc_off = G.bar_off + ((size_t)(3 * nst + 1) * 8 + 8 + 15) / 16 * 16;
  G.total = G.tsc_off + (size_t)nt * 4;
  return G;
}
__host__ __device__ inline uint32_t tc_tmem_cols(int nt, int hilo) {
  uint32_t c = 32;
  while ((int)c < nt) c <<= 1;
  return hilo ? 2 * c : c;
}

// Raw data of one stage of one weight row: the codes of its group (32 bytes
// at 4 bits, 16 at 2) and the group's scale.
struct TcRaw {
  uint4 q0, q1;
  float s;
};

template <int BITS>
__device__ __forceinline__ void tc_load_raw(const uint32_t* qrow, const uint16_t* srow, int g, TcRaw& r) {
  constexpr int WPG = kGroup * BITS / 32;   // words per group: 8 or 4
  const uint4* q = (const uint4*)(qrow + (size_t)g * WPG);
  r.q0 = ldg_stream_v4(q);
  r.q1 = BITS == 4 ? ldg_stream_v4(q + 1) : make_uint4(0u, 0u, 0u, 0u);
  r.s = bf16_to_f32(__ldg(srow + g));
}

// 8 codes of one 4-bit word, or 8 of the 16 codes of a 2-bit word (half h),
// as fp16 s*(q - c) in chunk order
template <int BITS>
__device__ __forceinline__ uint4 tc_dequant_chunk(uint32_t w, int h, __half2 s2) {
  const uint32_t magic = 0x64006400u;
  const __half2 off = BITS == 4 ? __half2half2(__float2half_rn(1032.f)) : __half2half2(__float2half_rn(1026.f));
  uint32_t r[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int sh = BITS == 4 ? 4 * u : 2 * (u + 4 * h);
    const uint32_t m = BITS == 4 ? 0x000F000Fu : 0x00030003u;
    uint32_t v = ((w >> sh) & m) | magic;
    __half2 hv = *(__half2*)&v;
    hv = __hmul2(__hsub2(hv, off), s2);
    r[u] = *(uint32_t*)&hv;
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

template <int BITS>
__global__ void __launch_bounds__(kTcThreads, 1) tc_dense_kernel(TcParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int nst = p.nst;
  const TcGeom G = tc_geom(p.nt, p.hilo, nst);
  unsigned char* sA = smem + G.a_off;
  unsigned char* sB = smem + G.b_off;
  uint64_t* full_a = (uint64_t*)(smem + G.bar_off);
  uint64_t* full_b = full_a + nst;
  uint64_t* empty = full_b + nst;
  uint64_t* done = empty + nst;
  uint32_t* tslot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tslot + 1);
  float* tsc = (float*)(smem + G.tsc_off);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int m0 = blockIdx.x * kTcM, t0 = blockIdx.y * p.nt, split = blockIdx.z;
  const int ntok = min(p.nt, p.T - t0);          // tokens of this CTA
  const int npad = (ntok + 15) & ~15;            // MMA N
  const int ng = p.K / kGroup;                   // data stages = groups
  const int nstg = tc_cols(p.K) / kTcKS;
  const int i0 = (int)((long long)nstg * split / p.splits);
  const int i1 = (int)((long long)nstg * (split + 1) / p.splits);
  const int n = i1 - i0;
  // The row blocks of one split start at different stages (the sum order of a
  // row is still fixed), so that they do not all read the same activation tile
  // of L2 at the same time.
  const int rot = (int)(blockIdx.x % (unsigned)n);
  auto stage_of = [&](int u) { const int v = u + rot; return i0 + (v >= n ? v - n : v); };
  const uint32_t ncols = tc_tmem_cols(p.nt, p.hilo);
  const unsigned long long wns = p.wait_ns;

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full_a[s], kTcProducers + 1);   // + the copy thread (bias-column tiles)
      mbar_init(&full_b[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < p.nt; i += blockDim.x) tsc[i] = i < ntok ? p.tscale[t0 + i] : 0.f;
  if (warp == 4) tc_alloc(tslot, ncols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;

  if (tid < kTcProducers) {
    // ---------------------------------------------------------------- producers: weight tiles
    const int grow = m0 + tid;
    const bool second = grow >= p.R0;
    const moe_qmat W = second ? p.w1 : p.w0;
    const int r = second ? grow - p.R0 : grow;
    const uint32_t* qrow = W.q + (size_t)r * (p.K * BITS / 32);
    const uint16_t* srow = W.scales + (size_t)r * ng;
    const int d1 = i1 < ng ? i1 : ng;   // data stages of this CTA: [i0, d1); the rest are bias columns
    // codes of the next stages in a ring of four register sets, named (no moves between them)
    TcRaw r0{}, r1{}, r2{}, r3{};
    if (n > 0 && stage_of(0) < d1) tc_load_raw<BITS>(qrow, srow, stage_of(0), r0);
    if (n > 1 && stage_of(1) < d1) tc_load_raw<BITS>(qrow, srow, stage_of(1), r1);
    if (n > 2 && stage_of(2) < d1) tc_load_raw<BITS>(qrow, srow, stage_of(2), r2);
    const int e = __ldg(p.rexp + grow);
    const float rsc = tc_pow2(e);
    auto step = [&](int u, const TcRaw& cur, TcRaw& ahead) -> bool {
      const int i = stage_of(u), slot = u % nst, use = u / nst;
      if (u + 3 < n && stage_of(u + 3) < d1) tc_load_raw<BITS>(qrow, srow, stage_of(u + 3), ahead);
      if (use > 0 && !mbar_wait_bounded(&empty[slot], (use - 1) & 1, wns, p.status)) *abort_flag = 1;
      if (*abort_flag) return false;
      if (i < ng) {
        uint4* dst = (uint4*)(sA + (size_t)slot * kTcABytes) + tid;   // chunk c at + c*128 uint4
        const __half2 s2 = __half2half2(__float2half_rn(cur.s * rsc));
        const uint32_t w[8] = {cur.q0.x, cur.q0.y, cur.q0.z, cur.q0.w, cur.q1.x, cur.q1.y, cur.q1.z, cur.q1.w};
#pragma unroll
        for (int c = 0; c < 8; ++c)
          dst[c * kTcM] = BITS == 4 ? tc_dequant_chunk<4>(w[c], 0, s2) : tc_dequant_chunk<2>(w[c >> 1], c & 1, s2);
        fence_proxy_async();
      }
      mbar_arrive(&full_a[slot]);   // bias-column tiles arrive by bulk copy (warp 5)
      return true;
    };
    for (int u = 0; u < n; u += 4) {
      if (!step(u, r0, r3)) break;
      if (u + 1 >= n || !step(u + 1, r1, r0)) break;
      if (u + 2 >= n || !step(u + 2, r2, r1)) break;
      if (u + 3 >= n || !step(u + 3, r3, r2)) break;
    }
    // ---------------------------------------------------------------- epilogue
    bool ok = mbar_wait_bounded(done, 0, wns, p.status) && !*abort_flag;
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      const float rinv = tc_pow2(-e);
      const uint32_t lane_addr = tbase + ((uint32_t)(warp * 32) << 16);
      float* out = p.part + ((size_t)split * p.T + t0) * p.M + m0 + tid;
      for (int c0 = 0; c0 < npad; c0 += 16) {
        uint32_t hv[16], lv[16];
        tc_ld16(lane_addr + c0, hv);
        if (p.hilo) tc_ld16(lane_addr + ncols / 2 + c0, lv);
        tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = c0 + j;
          float v = __uint_as_float(hv[j]);
          if (p.hilo) v += __uint_as_float(lv[j]);
          if (t < ntok) out[(size_t)t * p.M] = v * rinv * tsc[t];
        }
      }
    }
  } else if (tid == 4 * 32) {
    // ---------------------------------------------------------------- MMA issue (one thread)
    const uint32_t idesc = tc_idesc_f16(kTcM, npad);
    const uint32_t bstride = (uint32_t)G.brows * 16;   // bytes between column chunks of a tile
    int u = 0;
    for (; u < n; ++u) {
      const int slot = u % nst, ph = (u / nst) & 1;
      if (!mbar_wait_bounded(&full_b[slot], ph, wns, p.status) || !mbar_wait_bounded(&full_a[slot], ph, wns, p.status))
        *abort_flag = 1;
      if (*abort_flag) break;
      tc_fence_after();
      const uint32_t a0 = smem_u32(sA + (size_t)slot * kTcABytes);
      const uint32_t b0 = smem_u32(sB + (size_t)slot * G.stage_b);
#pragma unroll
      for (int ks = 0; ks < kTcKS / 16; ++ks) {
        const uint64_t ad = tc_smem_desc(a0 + ks * 2 * (kTcM * 16), kTcM * 16, 128);
        const uint64_t bh = tc_smem_desc(b0 + ks * 2 * bstride, bstride, 128);
        tc_mma_f16(tbase, ad, bh, idesc, u > 0 || ks > 0);
        if (p.hilo) {
          const uint64_t bl = tc_smem_desc(b0 + ks * 2 * bstride + p.nt * 16, bstride, 128);
          tc_mma_f16(tbase + ncols / 2, ad, bl, idesc, u > 0 || ks > 0);
        }
      }
      tc_commit(&empty[slot]);
    }
    tc_commit(done);   // arrives once every MMA issued above has completed
    mbar_wait_bounded(done, 0, wns, p.status);
  } else if (tid == 5 * 32) {
    // ---------------------------------------------------------------- activation tiles (one thread)
    int last[kTcMaxStages], lastx[kTcMaxStages];   // last use of each slot with copies issued (B, bias tile)
    for (int s = 0; s < kTcMaxStages; ++s) last[s] = lastx[s] = -1;
    const unsigned rows_bytes = (unsigned)npad * 16;
    const unsigned bytes = rows_bytes * (kTcKS / 8) * (p.hilo ? 2u : 1u);
    for (int u = 0; u < n; ++u) {
      const int i = stage_of(u), slot = u % nst, use = u / nst;
      if (use > 0 && !mbar_wait_bounded(&empty[slot], (use - 1) & 1, wns, p.status)) *abort_flag = 1;
      if (*abort_flag) break;
      if (i >= ng) {   // bias columns: the prepared 128 x 64 tile of this row block
        mbar_expect_tx(&full_a[slot], (unsigned)kTcABytes);
        bulk_g2s(sA + (size_t)slot * kTcABytes, p.aext + ((size_t)blockIdx.x * (nstg - ng) + (i - ng)) * (kTcABytes / 2),
                 (unsigned)kTcABytes, &full_a[slot]);
      } else {
        mbar_arrive(&full_a[slot]);
      }
      mbar_expect_tx(&full_b[slot], bytes);
      unsigned char* dst = sB + (size_t)slot * G.stage_b;
#pragma unroll 1
      for (int c = 0; c < kTcKS / 8; ++c) {
        const size_t o = ((size_t)(i * (kTcKS / 8) + c) * p.Tpad + t0) * 8;
        bulk_g2s(dst + (size_t)c * G.brows * 16, p.b_hi + o, rows_bytes, &full_b[slot]);
        if (p.hilo) bulk_g2s(dst + (size_t)c * G.brows * 16 + (size_t)p.nt * 16, p.b_lo + o, rows_bytes, &full_b[slot]);
      }
      last[slot] = use;
      lastx[slot] = i >= ng ? use : -1;
    }
    // no copy may land after the CTA has left
    for (int s = 0; s < nst && s < kTcMaxStages; ++s)
      if (last[s] >= 0) {
        mbar_wait_bounded(&full_b[s], last[s] & 1, wns, p.status);
        if (lastx[s] >= 0) mbar_wait_bounded(&full_a[s], lastx[s] & 1, wns, p.status);
      }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) tc_dealloc(tbase, ncols);
}

// ------------------------------------------------------------------ launchers
static size_t tc_optin() {
  int optin = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  return optin > 0 ? (size_t)optin : (size_t)227 * 1024;
}
// deepest pipeline that fits one CTA's shared memory (0: none)
static int tc_stages(int nt, int hilo) {
  const size_t optin = tc_optin();
  for (int nst = kTcMaxStages; nst >= 2; --nst)
    if (tc_geom(nt, hilo, nst).total <= optin) return nst;
  return 0;
}

bool tc_supported(int H, int I, int bits) {
  if (bits != 2 && bits != 4) return false;
  if ((2 * I) % kTcM || H % kTcM || H % kGroup || I % kGroup) return false;
  return tc_stages(kTcMaxNt, 1) >= 2 && tc_stages(kTcMaxNt, 0) >= 2;
}

cudaError_t launch_tc_conv(const TcConvParams& p, cudaStream_t s) {
  if (p.K % kGroup || p.K > 16 * kTcConvThreads * kTcConvSpans) return cudaErrorInvalidConfiguration;
  for (int j = 0; j < p.nprep; ++j)
    if (p.prep[j].K > 64 * 2 * 32 * kTcPrepChunks || p.prep[j].M % kTcM) return cudaErrorInvalidConfiguration;
  const void* fn = p.bits == 4 ? (const void*)tc_conv_kernel<4> : (const void*)tc_conv_kernel<2>;
  const int tpc = kTcConvThreads / tc_token_threads(p.K);
  int rows = 0;
  for (int j = 0; j < p.nprep; ++j) rows += p.prep[j].M;
  const int nb = (p.Tpad + tpc - 1) / tpc + (rows + kTcConvThreads / 32 - 1) / (kTcConvThreads / 32);
  TcConvParams q = p;
  void* args[] = {&q};
  return cudaLaunchKernel(fn, dim3(nb), dim3(kTcConvThreads), args, 0, s);
}

// Sets nt, splits and nst from the shapes (callers read the split count with tc_splits).
cudaError_t launch_tc_dense(const TcParams& p, cudaStream_t s) {
  TcParams q = p;
  q.nt = tc_nt(p.T);
  q.splits = tc_splits(p.M, p.T, p.K);
  q.nst = tc_stages(q.nt, q.hilo);
  if (!q.nst || p.M % kTcM || p.K % kGroup || p.Tpad != tc_pad16(p.T)) return cudaErrorInvalidConfiguration;
  const size_t sm = tc_geom(q.nt, q.hilo, q.nst).total;
  const void* fn = p.bits == 4 ? (const void*)tc_dense_kernel<4> : (const void*)tc_dense_kernel<2>;
  cudaError_t e = set_func_attr(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  void* args[] = {&q};
  const dim3 grid(p.M / kTcM, (q.Tpad + q.nt - 1) / q.nt, q.splits);
  return cudaLaunchKernel(fn, grid, dim3(kTcThreads), args, sm, s);
}

}  // namespace qmoe
