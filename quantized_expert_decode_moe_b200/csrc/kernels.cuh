// Kernel parameter blocks and launchers of the quantized MoE expert forward.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace qmoe {

// Workspace carve-up for T tokens of one layer shape.
struct WsLayout {
  size_t status;      // uint32 status word (+ padding)
  size_t logits;      // double [T][E+1]; column E = shared-gate logit
  size_t a;           // float [T][S][I]  silu(gate) * up of each slot (slot S-1 = shared expert)
  size_t hacc;        // float [T][H]     h + weighted expert outputs
  // prefill
  size_t counts;      // int32 [E]
  size_t offsets;     // int32 [E+1]
  size_t perm;        // int32 [T*k]
  size_t pidx;        // int32 [T][k]   routed expert ids
  size_t pw;          // float [T][k]   routing weights
  size_t psg;         // float [T]      shared-expert gate
  size_t xd;          // u8 [T][2H]     digit tables of x (+ xX float [T][H/64], xrs float [T])
  size_t xX, xrs;
  size_t ad;          // u8 [T*k + T][2I]  digit tables of the SwiGLU outputs (+ aX, ars)
  size_t aX, ars;
  size_t chunks;      // int4 [max chunks] (expert, first position, tokens, 0)
  size_t nchunks;     // int32
  size_t y;           // float [T*k + T][H] expert outputs, same rows
  size_t total;
};
WsLayout ws_layout(int H, int I, int E, int k, int S, int T);

struct RouteParams {
  int H, E, T, has_shared;
  const uint16_t* x;            // [T][H]
  const uint16_t* router_w;     // [E][H]
  const float* router_bias;     // [E] or null
  const uint16_t* gate_w;       // [H] or null
  double* logits;               // [T][E+1]
  // side job of the decode chain (null when unused): copies of the layer's inputs x, h ([T][H])
  const float* h; uint16_t* x_rec; float* h_rec;
};

struct TopkParams {
  int E, k, T, has_shared;
  const double* logits;        // [T][E+1]
  int32_t* idx; float* w; float* sg;   // outputs (sg nullable)
};

struct GateUpParams {
  int H, I, E, k, S, has_shared, nCTA;
  const uint16_t* x;           // [T][H]
  const double* logits;        // [T][E+1]
  const moe_expert* experts;   // device [E]
  moe_expert shared;
  float* a;                    // [T][S][I]
  int32_t* idx_out; float* w_out;   // user copies of the routing, nullable
  uint32_t* status;
  unsigned long long wait_ns;  // bound of every device-side wait
};

struct DownParams {
  int H, I, E, k, S, has_shared, nCTA;
  const double* logits;        // [T][E+1]
  const float* a;              // [T][S][I]
  const float* h;              // [T][H] residual
  const moe_expert* experts;
  moe_expert shared;
  float* hacc;                 // [T][H]
  uint32_t* status;
  unsigned long long wait_ns;
};

struct NormDecodeParams {
  int H, T;
  const float* hacc; float* h; const uint16_t* gamma; float eps;
  uint16_t* x_out; float* x_out_f32;
};

struct NormParams {
  int H, k, T;
  const float* y_routed; long long y_routed_tok_stride, y_routed_slot_stride;
  const float* w; const float* y_shared; long long y_shared_tok_stride; const float* sg;
  float* h; const uint16_t* gamma; float eps;
  uint16_t* x_out; float* x_out_f32;
};

struct GemvParams {
  int R, K, nspans, ntiles, nCTA;
  long long U;
  moe_qmat W;
  const float* x;
  float* y;
  uint32_t* status;            // may be null (no workspace): timeouts are then not latched
  size_t stage_bytes;
  unsigned long long wait_ns;
};

struct PrefillParams {
  int H, I, E, k, T, has_shared;
  int nst, rt, rw;             // stages, tile groups and tiles per warp of the grouped kernels (set by their launcher)
  const uint16_t* x;           // [T][H] bf16
  unsigned char* xd;           // [T][2H]   digit tables of x
  float* xX;                   // [T][H/64] group sums of x
  float* xrs;                  // [T]       2^-p of each row of x
  float* a;                    // [T*k + T][I] silu(gate) * up per pair (t*k + r), then per token (shared)
  unsigned char* ad;           // [T*k + T][2I] digit tables of a
  float* aX;                   // [T*k + T][I/64]
  float* ars;                  // [T*k + T]
  float* y;                    // [T*k + T][H]
  const int4* chunks;          // {expert, first position (perm index, or token for the shared expert), tokens, 0}
  const int32_t* nchunks;      // [1]
  const int32_t* perm;         // [T*k]
  const moe_expert* experts;
  moe_expert shared;
  uint32_t* status;
  unsigned long long wait_ns;
};

struct GroupParams {
  int T, k, E, has_shared;
  int chunk;                   // tokens per chunk of the grouped GEMMs
  const int32_t* idx;
  int32_t* counts; int32_t* offsets; int32_t* perm;
  int4* chunks; int32_t* nchunks;
};

// launchers (return the launch's cudaError_t)
cudaError_t launch_route(const RouteParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_route_gemm(const RouteParams& p, cudaStream_t s);   // many tokens: tiled fp64
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);
cudaError_t launch_gateup(const GateUpParams& p, int bits, int T, bool pdl, cudaStream_t s);
cudaError_t launch_down(const DownParams& p, int bits, int T, bool pdl, cudaStream_t s);
cudaError_t launch_norm(const NormParams& p, bool pdl, cudaStream_t s);
cudaError_t launch_norm_decode(const NormDecodeParams& p, bool pdl, cudaStream_t s);
size_t gateup_smem_bytes(int H, int bits);
size_t down_smem_bytes(int I, int S, int bits);
int gateup_ctas(int I);
int down_ctas(int H);
cudaError_t launch_gemv(const GemvParams& p, int bits, cudaStream_t s);
cudaError_t launch_group(const GroupParams& p, cudaStream_t s);
cudaError_t launch_prefill_gateup(const PrefillParams& p, int bits, cudaStream_t s);   // digit tables of x + gate/up
cudaError_t launch_prefill_down(const PrefillParams& p, int bits, cudaStream_t s);     // digit tables of a + down
cudaError_t launch_selftest_wait(uint32_t* status, unsigned long long bound_ns, cudaStream_t s);
int num_sms();
int pf_chunk_tokens(int H, int I);   // tokens per chunk of the grouped GEMMs
size_t pf_max_chunks(int T, int k, int E, int chunk);
int choose_ncta(long long ntiles, int nspans);

}  // namespace qmoe
