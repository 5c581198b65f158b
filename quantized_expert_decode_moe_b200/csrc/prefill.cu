// Prefill path of the quantized MoE expert forward (T > 8 tokens, sm_100a):
// grouped dequantising GEMMs on the fp16 tensor cores.
//
// After routing, the (token, rank) pairs are grouped by expert (see
// group_kernel). For every expert e with n_e pairs, and for the shared expert
// with all T tokens, the products are dense GEMMs of the expert's weight rows
// with its tokens as the N dimension:
//   gate/up:  a[pair][j] = silu(G_e[j] . x_t) * (U_e[j] . x_t)
//   down:     y[pair][h] = D_e[h] . a[pair]
// A CTA owns one 16-row block of one expert's matrices (gate/up: 8 gate rows
// and the 8 up rows of the same intermediate indices, so SwiGLU is local) and
// runs all of that expert's tokens through it, 64 at a time. The block's
// packed codes, scales and biases arrive with bulk copies; the weights are
// dequantised in registers to fp16, w = q*s + b with one rounding (the codes
// 0..15 / 0..3 are exact in fp16), and each A fragment is reused for every
// 8-token tile of the pass (mma.sync m16n8k16, f16 x f16 -> f32). The warps
// split K and their partial sums are added in a fixed order.
#include <math.h>

#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace qmoe {

constexpr int kPfThreads = 256;
constexpr int kPfWarps = kPfThreads / 32;
constexpr int kPfTokens = 64;   // tokens per pass
constexpr int kPfTiles = kPfTokens / 8;

__device__ __forceinline__ void pf_mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(smem_u32(bar)) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void pf_expect(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void pf_bulk(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// Bounded wait for phase 0 of bar; on timeout latches MOE_ERR_TIMEOUT and returns false.
__device__ bool pf_wait(uint64_t* bar, unsigned long long bound_ns, uint32_t* status) {
  unsigned long long t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (;;) {
    uint32_t ok;
    asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n selp.u32 %0, 1, 0, p;\n}\n"
                 : "=r"(ok) : "r"(smem_u32(bar)) : "memory");
    if (ok) return true;
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    if (t - t0 > bound_ns) {
      if (status) atomicCAS(status, 0u, (uint32_t)MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two codes (lo, hi in 0..15) as an exact fp16 pair: 0x6400 is fp16 1024,
// (1024 + q) - 1024 = q exactly.
__device__ __forceinline__ uint32_t codes_h2(uint32_t lo, uint32_t hi) {
  const uint32_t v = 0x64006400u | lo | (hi << 16);
  const __half2 q = __hsub2(*(const __half2*)&v, __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400)));
  return *(const uint32_t*)&q;
}
// w = q*s + b for a pair of codes of one row and group (s, b bf16 -> fp16)
__device__ __forceinline__ uint32_t deq_pair(uint32_t q2, __half2 s2, __half2 b2) {
  const __half2 w = __hfma2(*(const __half2*)&q2, s2, b2);
  return *(const uint32_t*)&w;
}
__device__ __forceinline__ __half2 bf16_to_h2(uint16_t v) {
  const __half h = __float2half_rn(__uint_as_float((uint32_t)v << 16));
  return __halves2half2(h, h);
}

// Shared layout of both kernels: codes [16][RB], scales [16][K/64], biases
// [16][K/64] (bf16), token list, partial sums [warps][16 rows][kPfTokens].
struct PfLayout { size_t codes, scales, biases, tok, part, bar, total; };
__host__ __device__ inline PfLayout pf_layout(int K, int bits) {
  PfLayout L;
  size_t o = 0;
  L.codes = o; o += (size_t)16 * K * bits / 8;
  o = (o + 15) & ~(size_t)15;
  L.scales = o; o += (size_t)16 * (K / kGroup) * 2;
  o = (o + 15) & ~(size_t)15;
  L.biases = o; o += (size_t)16 * (K / kGroup) * 2;
  o = (o + 15) & ~(size_t)15;
  L.tok = o; o += sizeof(int) * 2 * kPfTokens;
  L.part = o; o += sizeof(float) * kPfWarps * 16 * kPfTokens;
  L.bar = o; o += 8;
  L.total = o;
  return L;
}

// Accumulates, for the rows of the block (rows 0-15 of `codes`) and up to 64
// tokens, the warp's K-slice [k0, k1) (multiples of 16) into acc[tile][4]; B
// operands come from `act` (fp16 [*][K], row of token i = act + row_of[i] * K).
// Codes are read once per 64 columns: lane t of a quad loads one quarter of
// its row's bytes for those columns and the quad shares them by shuffles.
template <int BITS>
__device__ __forceinline__ void pf_block_mma(const unsigned char* codes, const uint16_t* sc, const uint16_t* bi,
                                             int K, const __half* act, const int* row_of, int ntok, int k0, int k1,
                                             float (&acc)[kPfTiles][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3, qb = lane & ~3;
  const int RB = K * BITS / 8, ng = K / kGroup;
  const unsigned char* ra = codes + (size_t)g * RB;
  const unsigned char* rb = codes + (size_t)(g + 8) * RB;
  constexpr int CB = 64 * BITS / 8 / 4;   // bytes per lane per 64 columns: 8 (4-bit) or 4 (2-bit)
  uint2 ca = make_uint2(0u, 0u), cb = make_uint2(0u, 0u);
  __half2 sa, ba, sb, bb;
  for (int k = k0; k < k1; k += 16) {
    if (k == k0 || (k & 63) == 0) {
      const int grp = k / kGroup;
      sa = bf16_to_h2(sc[g * ng + grp]); ba = bf16_to_h2(bi[g * ng + grp]);
      sb = bf16_to_h2(sc[(g + 8) * ng + grp]); bb = bf16_to_h2(bi[(g + 8) * ng + grp]);
    }
    const int kc = k & ~63;   // first column of this 64-column chunk
    if (k == k0 || (k & 63) == 0) {
      const int off = kc * BITS / 8 + CB * t;
      if constexpr (BITS == 4) { ca = *(const uint2*)(ra + off); cb = *(const uint2*)(rb + off); }
      else { ca.x = *(const uint32_t*)(ra + off); cb.x = *(const uint32_t*)(rb + off); }
    }
    const int st = (k - kc) >> 4;   // step inside the chunk: its bytes are held by quad lane st
    uint32_t a0, a1, a2, a3;
    if constexpr (BITS == 4) {
      // step bytes [8 st, 8 st + 8): lo word -> columns k..k+7, hi word -> k+8..k+15; lane t takes byte t
      const uint32_t la = __shfl_sync(0xffffffffu, ca.x, qb + st) >> (8 * t);
      const uint32_t ha = __shfl_sync(0xffffffffu, ca.y, qb + st) >> (8 * t);
      const uint32_t lb = __shfl_sync(0xffffffffu, cb.x, qb + st) >> (8 * t);
      const uint32_t hb = __shfl_sync(0xffffffffu, cb.y, qb + st) >> (8 * t);
      a0 = deq_pair(codes_h2(la & 0xFu, (la >> 4) & 0xFu), sa, ba);
      a1 = deq_pair(codes_h2(lb & 0xFu, (lb >> 4) & 0xFu), sb, bb);
      a2 = deq_pair(codes_h2(ha & 0xFu, (ha >> 4) & 0xFu), sa, ba);
      a3 = deq_pair(codes_h2(hb & 0xFu, (hb >> 4) & 0xFu), sb, bb);
    } else {
      // step bytes [4 st, 4 st + 4): columns k + 4i .. k + 4i + 3 in byte i; lane t needs columns 2t, 2t+1
      // (byte t>>1, fields 2(t&1), +1) and 8+2t, 9+2t (byte 2 + (t>>1))
      const uint32_t wa = __shfl_sync(0xffffffffu, ca.x, qb + st), wb = __shfl_sync(0xffffffffu, cb.x, qb + st);
      const int s0 = 8 * (t >> 1) + 4 * (t & 1), s1 = s0 + 16;
      a0 = deq_pair(codes_h2((wa >> s0) & 3u, (wa >> (s0 + 2)) & 3u), sa, ba);
      a1 = deq_pair(codes_h2((wb >> s0) & 3u, (wb >> (s0 + 2)) & 3u), sb, bb);
      a2 = deq_pair(codes_h2((wa >> s1) & 3u, (wa >> (s1 + 2)) & 3u), sa, ba);
      a3 = deq_pair(codes_h2((wb >> s1) & 3u, (wb >> (s1 + 2)) & 3u), sb, bb);
    }
#pragma unroll
    for (int nt = 0; nt < kPfTiles; ++nt) {
      if (nt * 8 < ntok) {
        const int i = nt * 8 + g;
        uint32_t b0 = 0u, b1 = 0u;
        if (i < ntok) {
          const __half* xr = act + (size_t)row_of[i] * K + k + 2 * t;
          b0 = *(const uint32_t*)xr;
          b1 = *(const uint32_t*)(xr + 8);
        }
        mma_f16(acc[nt], a0, a1, a2, a3, b0, b1);
      }
    }
  }
}

// Writes the warp's partial sums: part[warp][row][token]
__device__ __forceinline__ void pf_store_part(float* part, const float (&acc)[kPfTiles][4], int ntok) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  float* pw = part + (size_t)warp * 16 * kPfTokens;
#pragma unroll
  for (int nt = 0; nt < kPfTiles; ++nt) {
    if (nt * 8 < ntok) {
      const int c = nt * 8 + 2 * t;
      pw[g * kPfTokens + c] = acc[nt][0];
      pw[g * kPfTokens + c + 1] = acc[nt][1];
      pw[(g + 8) * kPfTokens + c] = acc[nt][2];
      pw[(g + 8) * kPfTokens + c + 1] = acc[nt][3];
    }
  }
}

// tokens of expert e (e == E: the shared expert): n, and the i-th pair index /
// token through pair_of(i) (shared: the token itself)
struct PfGroup { int n, base; bool shared; };
__device__ __forceinline__ PfGroup pf_group(const PrefillParams& p, int e) {
  PfGroup G;
  G.shared = e == p.E;
  if (G.shared) { G.n = p.T; G.base = 0; }
  else { G.base = p.offsets[e]; G.n = p.offsets[e + 1] - G.base; }
  return G;
}

// grid (I/8, E + has_shared), block 256: a[row][j0..j0+8) for every pair of
// the expert (rows: pair index t*k + r; shared expert: T*k + t), fp16.
template <int BITS>
__global__ void __launch_bounds__(kPfThreads) prefill_gateup_kernel(PrefillParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = p.H, I = p.I;
  const PfLayout L = pf_layout(H, BITS);
  const int e = blockIdx.y;
  const PfGroup G = pf_group(p, e);
  if (G.n == 0) return;
  const moe_expert& ex = G.shared ? p.shared : p.experts[e];
  unsigned char* codes = smem + L.codes;
  uint16_t* sc = (uint16_t*)(smem + L.scales);
  uint16_t* bi = (uint16_t*)(smem + L.biases);
  int* rows = (int*)(smem + L.tok);          // act row (token) of pass token i
  int* outs = rows + kPfTokens;              // output row (pair) of pass token i
  float* part = (float*)(smem + L.part);
  uint64_t* bar = (uint64_t*)(smem + L.bar);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int j0 = blockIdx.x * 8;
  const int RB = H * BITS / 8, SRB = (H / kGroup) * 2;
  if (tid == 0) {
    pf_mbar_init(bar);
    pf_expect(bar, 2u * 8 * RB + 4u * 8 * SRB);
  }
  __syncthreads();
  if ((tid & 31) == 0 && warp < 6) {   // one copy per warp: gate/up codes, scales, biases (8-row blocks)
    const moe_qmat& m = (warp & 1) ? ex.up : ex.gate;
    const int half = warp & 1;
    if (warp < 2) pf_bulk(codes + (size_t)half * 8 * RB, (const char*)m.q + (size_t)j0 * RB, 8u * RB, bar);
    else if (warp < 4) pf_bulk((char*)sc + half * 8 * SRB, (const char*)m.scales + (size_t)j0 * SRB, 8u * SRB, bar);
    else pf_bulk((char*)bi + half * 8 * SRB, (const char*)m.biases + (size_t)j0 * SRB, 8u * SRB, bar);
  }
  pf_wait(bar, p.wait_ns, p.status);
  const int ks = H / kPfWarps;   // K-slice per warp (multiple of 16)
  for (int pass = 0; pass < G.n; pass += kPfTokens) {
    const int ntok = G.n - pass < kPfTokens ? G.n - pass : kPfTokens;
    if (tid < ntok) {
      const int i = pass + tid;
      const int pair = G.shared ? i : p.perm[G.base + i];
      rows[tid] = G.shared ? i : pair / p.k;
      outs[tid] = G.shared ? p.T * p.k + i : pair;
    }
    __syncthreads();
    float acc[kPfTiles][4];
#pragma unroll
    for (int nt = 0; nt < kPfTiles; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    pf_block_mma<BITS>(codes, sc, bi, H, p.xh, rows, ntok, warp * ks, (warp + 1) * ks, acc);
    pf_store_part(part, acc, ntok);
    __syncthreads();
    for (int q = tid; q < 8 * ntok; q += kPfThreads) {
      const int j = q / ntok, i = q - j * ntok;
      float gs = 0.f, us = 0.f;
      for (int w = 0; w < kPfWarps; ++w) {
        gs += part[((size_t)w * 16 + j) * kPfTokens + i];
        us += part[((size_t)w * 16 + 8 + j) * kPfTokens + i];
      }
      const float a = gs / (1.f + expf(-gs)) * us;
      p.a16[(size_t)outs[i] * I + j0 + j] = __float2half_rn(a);
    }
    __syncthreads();
  }
}

// grid (H/16, E + has_shared), block 256: y[row][h0..h0+16) for every pair of
// the expert (rows as above), fp32.
template <int BITS>
__global__ void __launch_bounds__(kPfThreads) prefill_down_kernel(PrefillParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int H = p.H, I = p.I;
  const PfLayout L = pf_layout(I, BITS);
  const int e = blockIdx.y;
  const PfGroup G = pf_group(p, e);
  if (G.n == 0) return;
  const moe_expert& ex = G.shared ? p.shared : p.experts[e];
  unsigned char* codes = smem + L.codes;
  uint16_t* sc = (uint16_t*)(smem + L.scales);
  uint16_t* bi = (uint16_t*)(smem + L.biases);
  int* rows = (int*)(smem + L.tok);
  float* part = (float*)(smem + L.part);
  uint64_t* bar = (uint64_t*)(smem + L.bar);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int h0 = blockIdx.x * 16;
  const int RB = I * BITS / 8, SRB = (I / kGroup) * 2;
  if (tid == 0) {
    pf_mbar_init(bar);
    pf_expect(bar, 16u * RB + 2u * 16 * SRB);
  }
  __syncthreads();
  if ((tid & 31) == 0 && warp < 3) {   // one copy per warp: codes, scales, biases (16-row blocks)
    if (warp == 0) pf_bulk(codes, (const char*)ex.down.q + (size_t)h0 * RB, 16u * RB, bar);
    else if (warp == 1) pf_bulk(sc, (const char*)ex.down.scales + (size_t)h0 * SRB, 16u * SRB, bar);
    else pf_bulk(bi, (const char*)ex.down.biases + (size_t)h0 * SRB, 16u * SRB, bar);
  }
  pf_wait(bar, p.wait_ns, p.status);
  const int ks = I / kPfWarps;
  for (int pass = 0; pass < G.n; pass += kPfTokens) {
    const int ntok = G.n - pass < kPfTokens ? G.n - pass : kPfTokens;
    if (tid < ntok) {
      const int i = pass + tid;
      rows[tid] = G.shared ? p.T * p.k + i : p.perm[G.base + i];   // a row = output row
    }
    __syncthreads();
    float acc[kPfTiles][4];
#pragma unroll
    for (int nt = 0; nt < kPfTiles; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    pf_block_mma<BITS>(codes, sc, bi, I, p.a16, rows, ntok, warp * ks, (warp + 1) * ks, acc);
    pf_store_part(part, acc, ntok);
    __syncthreads();
    for (int q = tid; q < 16 * ntok; q += kPfThreads) {
      const int r = q / ntok, i = q - r * ntok;
      float y = 0.f;
      for (int w = 0; w < kPfWarps; ++w) y += part[((size_t)w * 16 + r) * kPfTokens + i];
      p.y[(size_t)rows[i] * H + h0 + r] = y;
    }
    __syncthreads();
  }
}

// bf16 -> fp16 (exact for the magnitudes of normalised activations; fp16 keeps
// 11 significant bits, bf16 has 8)
__global__ void to_f16_kernel(const uint16_t* x, __half* xh, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    xh[i] = __float2half_rn(__uint_as_float((uint32_t)x[i] << 16));
}

static cudaError_t pf_prepare(const void* fn, size_t bytes) {
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t launch_prefill_gateup(const PrefillParams& p, int bits, cudaStream_t s) {
  PrefillParams q = p;
  void* args[] = {&q};
  const int groups = p.E + (p.has_shared ? 1 : 0);
  const size_t n = (size_t)p.T * p.H;
  to_f16_kernel<<<(unsigned)((n + 1023) / 1024 < 4096 ? (n + 1023) / 1024 : 4096), 1024, 0, s>>>(p.x, p.xh, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t sm = pf_layout(p.H, bits).total;
  const void* fn = bits == 4 ? (const void*)prefill_gateup_kernel<4> : (const void*)prefill_gateup_kernel<2>;
  if ((e = pf_prepare(fn, sm)) != cudaSuccess) return e;
  return cudaLaunchKernel(fn, dim3(p.I / 8, groups), dim3(kPfThreads), args, sm, s);
}

cudaError_t launch_prefill_down(const PrefillParams& p, int bits, cudaStream_t s) {
  PrefillParams q = p;
  void* args[] = {&q};
  const int groups = p.E + (p.has_shared ? 1 : 0);
  const size_t sm = pf_layout(p.I, bits).total;
  const void* fn = bits == 4 ? (const void*)prefill_down_kernel<4> : (const void*)prefill_down_kernel<2>;
  cudaError_t e = pf_prepare(fn, sm);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernel(fn, dim3(p.H / 16, groups), dim3(kPfThreads), args, sm, s);
}

}  // namespace qmoe
