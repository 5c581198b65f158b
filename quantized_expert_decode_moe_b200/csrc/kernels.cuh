// Kernel parameter blocks and launchers of the quantized MoE expert forward.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace qmoe {

// Workspace carve-up for T tokens of one layer shape.
struct WsLayout {
  size_t status;      // uint32 status word (+ padding)
  size_t logits;      // double [T][E+1]; column E = shared-gate logit
  size_t gu;          // float [T][S][2][I]  gate/up pre-activations
  size_t y;           // float [T][S][H]     expert outputs (unweighted)
  size_t w;           // float [T][k]        routing weights
  size_t sg;          // float [T]           shared gate
  size_t idx;         // int32 [T][k]        routed expert ids
  size_t slots;       // moe_expert [T][9]   chosen experts of each token
  // prefill
  size_t counts;      // int32 [E]
  size_t offsets;     // int32 [E+1]
  size_t perm;        // int32 [T*k]
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
  // side jobs of the decode chain (null when unused)
  float* zero_buf; size_t zero_n;   // accumulators cleared for the next kernels
  moe_expert shared; int I, bits; int prefetch_shared;
};

struct TopkParams {
  int E, k, T, has_shared;
  const double* logits;        // [T][E+1]
  int32_t* idx; float* w; float* sg;   // outputs (sg nullable)
};

struct GateUpParams {
  int H, I, E, k, S, has_shared, nspans, ntiles, nCTA;
  long long U;
  const uint16_t* x;           // [T][H]
  const double* logits;        // [T][E+1]
  const moe_expert* experts;   // device [E]
  moe_expert shared;
  float* gu;                   // [T][S][2][I]
  int32_t* idx_ws; float* w_ws; float* sg_ws;   // [T][k], [T][k], [T]
  moe_expert* slots_ws;                         // [T][kMaxSlots] chosen experts (routed, then shared)
  int32_t* idx_out; float* w_out;               // user copies, nullable
  uint32_t* status;
  int prefetch_down, prefetch_self;
  size_t stage_bytes;          // set by the launcher
  unsigned long long wait_ns;  // bound of every device-side wait
};

struct DownParams {
  int H, I, E, k, S, has_shared, nspans, ntiles, nCTA;
  long long U;
  const float* gu;             // [T][S][2][I]
  const int32_t* idx_ws;       // [T][k]
  const moe_expert* slots_ws;  // [T][kMaxSlots]
  const moe_expert* experts;
  moe_expert shared;
  float* y;                    // [T][S][H]
  uint32_t* status;
  size_t stage_bytes;
  unsigned long long wait_ns;
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

struct GroupParams {
  int T, k, E;
  const int32_t* idx;
  int32_t* counts; int32_t* offsets; int32_t* perm;
};

// launchers (return the launch's cudaError_t)
cudaError_t launch_route(const RouteParams& p, cudaStream_t s);
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);
cudaError_t launch_gateup(const GateUpParams& p, int bits, int T, bool pdl, cudaStream_t s);
cudaError_t launch_down(const DownParams& p, int bits, int T, bool pdl, cudaStream_t s);
cudaError_t launch_norm(const NormParams& p, bool pdl, cudaStream_t s);
cudaError_t launch_gemv(const GemvParams& p, int bits, cudaStream_t s);
cudaError_t launch_group(const GroupParams& p, cudaStream_t s);
int num_sms();
int choose_ncta(long long ntiles, int nspans);

}  // namespace qmoe
