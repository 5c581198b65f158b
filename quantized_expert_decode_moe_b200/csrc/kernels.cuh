// Kernel parameter blocks and launchers of the quantized MoE expert forward.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace qmoe {

constexpr int kMaxCtas = 1024;   // CTAs of the fused decode kernel at most
constexpr int kRtSplitMax = 12;  // column splits of the many-token router GEMM at most
constexpr size_t kSelFlagOffset = 80;   // byte offset of the decode chain's selection flags (8 words)

// Workspace carve-up for T tokens of one layer shape. The first 256 bytes are
// the header: the status word (word 0), the count of top-k selections that
// needed the exact recheck (word 4), the grid-barrier arrival counters
// (words 16..19), the decode chain's per-token selection flags (words
// 20..27) and the grid-barrier generations (words 32, 40, 48, 56).
struct WsLayout {
  size_t status;      // uint32 status word (+ padding)
  size_t logits;      // double [T][E+1]; column E = shared-gate logit
  size_t bound;       // float [T][E+1]  error bounds of fast logits
  size_t gpart;       // float [kMaxCtas] per-CTA partial sums (fused decode)
  size_t a;           // float [T][S][I]  silu(gate) * up of each slot (slot S-1 = shared expert)
  size_t hacc;        // float [T][H]     h + weighted expert outputs
  size_t mxx, mxa;    // MXFP4 layers: digit blocks of x [T][H/32][112 B] and of a [T][S][I/32][112 B]
  // prefill
  size_t counts;      // int32 [E]
  size_t offsets;     // int32 [E+1]
  size_t perm;        // int32 [T*k]
  size_t pidx;        // int32 [T][k]   routed expert ids
  size_t pw;          // float [T][k]   routing weights
  size_t psg;         // float [T]      shared-expert gate
  size_t xd;          // u8 [T][2H]     digit tables of x (+ xX float [T][H/64], xrs float [T][H/64])
  size_t xX, xrs;
  size_t ad;          // u8 [T*k + T][2I]  digit tables of the SwiGLU outputs (+ aX, ars)
  size_t aX, ars;
  size_t chunks;      // int4 [max chunks] (expert, first position, tokens, 0)
  size_t nchunks;     // int32
  size_t y;           // float [T*k + T][H] expert outputs, same rows
  size_t lpart;       // int64 [kRtSplitMax][T][E] exact partial router sums (T > 8)
  size_t wdig, xdig;  // int8 digit planes of the router rows and of x (T > 8)
  size_t wst, xst;    // double [rows][8] their scales, sums, maxima, rounding residuals, low digits (T > 8)
  // shared expert on the tensor cores (T > 8): fp16 operand tables of x and of its SwiGLU
  // outputs (hi, lo) [Kx/8][Tpad][8], per-token scales [Tpad], split partial sums
  size_t tcbx, tcxs, tcbah, tcbal, tcas, tcpart;
  size_t tcrexp, tcaext;   // row exponents [2I + H] int, bias-column tiles of gate/up then down
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
  float* bound;                 // [T][E+1]: bound on |logit - fp64 definition| (null: not written)
  // many tokens (route_tc.cu): per-split exact partial sums [kRtSplitMax][T][E]; the router
  // rows' and tokens' digit planes (int8, rows padded to 128, tiled: 128-row tile, 64-column
  // stage, plane, 16-column chunk, row) and per-row statistics {2^-p, sum |v|, max |v|,
  // sum |v - V 2^-p|, sum |d0|, max |d0|, 0, 0}
  long long* lpart;
  int8_t* wdig; int8_t* xdig; double* wst; double* xst;
  uint32_t* status; unsigned long long wait_ns;   // bound of the tcgen05 router's waits
  // side job of the decode chain (null when unused): copies of the layer's inputs x, h ([T][H])
  const float* h; uint16_t* x_rec; float* h_rec;
  // side job for the digit-block layer kernels (null when unused): x's digit blocks
  // [T][H/32][112 bytes] in the order of codec `codec`
  uint8_t* xblocks; int codec;
};

struct TopkParams {
  int E, k, T, has_shared, H;
  const double* logits;        // [T][E+1]
  const float* bound;          // [T][E+1] error bounds of fast logits, or null (logits exact)
  const uint16_t* x;           // [T][H]  } what an exact recheck of a logit reads
  const uint16_t* router_w;    // [E][H]  }
  const float* router_bias;    // [E] or null
  int32_t* idx; float* w; float* sg;   // outputs (sg nullable)
  uint32_t* rechecks;          // counter of selections that needed the exact recheck, or null
};

struct GateUpParams {
  int H, I, E, k, S, has_shared, nCTA;
  const uint16_t* x;           // [T][H]
  const double* logits;        // [T][E+1]
  const float* bound;          // [T][E+1] error bounds of the logits
  const uint16_t* router_w; const float* router_bias;   // for an exact recheck of near ties
  const moe_expert* experts;   // device [E]
  moe_expert shared;
  float* a;                    // [T][S][I]
  int32_t* idx_out; float* w_out;   // user copies of the routing, nullable
  uint32_t* rechecks;          // counter of selections that needed the exact recheck, or null
  // the first CTA of each token publishes its selection for the down kernel, then sets the flag
  int32_t* sel_idx; float* sel_w; float* sel_sg;   // [T][k], [T][k], [T]
  unsigned* sel_flag;          // [T]
  uint32_t* status;
  unsigned long long wait_ns;  // bound of every device-side wait
};

struct DownParams {
  int H, I, E, k, S, has_shared, nCTA;
  // the selection published by the gate/up kernel's first CTA of each token (behind sel_flag)
  const int32_t* sel_idx; const float* sel_w; const float* sel_sg;
  const unsigned* sel_flag;
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
  unsigned* sel_flag;          // [T] cleared (every reader has passed: the down kernel is complete)
};

struct NormParams {
  int H, k, T;
  const float* y_routed; long long y_routed_tok_stride, y_routed_slot_stride;
  const float* w; const float* y_shared; long long y_shared_tok_stride; const float* sg;
  int y_shared_splits; long long y_shared_split_stride;   // y_shared = sum of the splits (0 or 1: one)
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
  float* xrs;                  // [T][H/64] 2^-p of each group of x
  float* a;                    // [T*k + T][I] silu(gate) * up per pair (t*k + r), then per token (shared)
  unsigned char* ad;           // [T*k + T][2I] digit tables of a
  float* aX;                   // [T*k + T][I/64]
  float* ars;                  // [T*k + T][I/64]
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

// Dense pass of one expert over every token of a batch on the tcgen05 tensor
// cores (the shared expert in prefill, shared_tc.cu):
//   part[s][t][m] = sum over the columns of split s of W[m][k] * v_t[k]
// with W the dequantised (stacked) weight matrix, rows [0, R0) from w0 and
// [R0, M) from w1, and v_t the token's activations (hi + lo parts when hilo).
struct TcParams {
  int M, K, R0, bits;
  moe_qmat w0, w1;
  int T, Tpad;                 // tokens, and tokens padded to 16 (rows of the operand tables)
  int nt;                      // tokens per CTA (multiple of 16, <= 256)
  int hilo;                    // operand tables carry a lo part (b_lo) beside the hi part
  const __half* b_hi;          // [Kx/8][Tpad][8] fp16, Kx = K + 64*ceil(K/1024) (tc_cols)
  const __half* b_lo;          // same, or null
  const float* tscale;         // [T] 2^-p of each token's table
  const int* rexp;             // [M] exponent e of each weight row (row values scaled by 2^e)
  const __half* aext;          // bias-column tiles [M/128][Kx/64 - K/64][8][128][8] fp16
  int splits;                  // column splits (gridDim.z)
  int nst;                     // pipeline stages (set by the launcher)
  float* part;                 // [splits][T][M]
  uint32_t* status;
  unsigned long long wait_ns;
};
// Per-row preparation of a weight matrix for the dense pass: the row exponent
// and the bias-column tiles (shared_tc.cu).
struct TcRowPrep {
  int M, R0, K;
  moe_qmat w0, w1;
  int* rexp;                   // [M]
  __half* aext;                // [M/128][Kx/64 - K/64][8][128][8]
};
// Operand tables of a batch's activations for the dense pass (shared_tc.cu),
// and (row CTAs after the token CTAs) the weight rows' preparation.
struct TcConvParams {
  int K, T, Tpad, bits;
  const uint16_t* x;           // bf16 [T][K] (gate/up input) or null
  const float* part; int splits, I;   // gate/up partial sums [splits][T][2I] (down input) or null
  __half* b_hi; __half* b_lo;  // [Kx/8][Tpad][8]
  float* tscale;               // [Tpad]
  int nprep;                   // weight matrices to prepare (0..2)
  TcRowPrep prep[2];
};

// One layer of the fused decode kernel (device pointers).
struct FuLayer {
  const uint16_t* router_w;    // [E][H]
  const float* router_bias;    // [E] or null
  const moe_expert* experts;   // device [E]
  moe_expert shared;
  const uint16_t* gate_w;      // [H] or null
  const uint16_t* gamma;       // [H]
  float eps;
};
constexpr int kFuMaxLayers = 24;   // layers per launch of the fused kernel (kernel parameter space)

struct FusedParams {
  int H, I, E, k, S, has_shared, nCTA, L;
  const uint16_t* x_in;        // [H] bf16, the first layer's input
  float* h;                    // [H] residual in, h' of the last layer out
  uint16_t* x_out;             // [H] bf16, the last layer's output
  float* x_out_f32;            // [H] or null
  int32_t* idx_out; float* w_out;   // [L][k] routing of every layer, nullable
  uint16_t* x_rec; float* h_rec;    // [L][H] inputs x, h of every layer, nullable
  uint32_t* status;            // workspace status word
  unsigned* hdr;               // workspace header (grid barrier counters at words 16.., generations at 32..)
  double* logits; float* bound;     // [E+1]
  float* a;                    // [S][I]
  float* hacc;                 // [H]
  float* gpart;                // [nCTA] partial sums of squares
  unsigned long long wait_ns;
  FuLayer layer[kFuMaxLayers];
};

// launchers (return the launch's cudaError_t)
cudaError_t launch_route(const RouteParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_route_gemm(const RouteParams& p, cudaStream_t s);   // many tokens: exact integer tcgen05
// router rows and tokens, padded to the tcgen05 router's 128 x 128 tiles
__host__ __device__ inline size_t route_tc_rows_w(int E) { return (size_t)((E + 127) / 128) * 128; }
__host__ __device__ inline size_t route_tc_rows_x(int T) { return (size_t)((T + 127) / 128) * 128; }
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s, bool pdl = false);
// MXFP4 experts (mx.cu): mat-vec, and the many-token product on tcgen05 (kind::mxf4)
cudaError_t launch_mx_gemv(const uint32_t* q, const uint8_t* e, int R, int K, const float* x, float* y, cudaStream_t s);
cudaError_t launch_mx_gemm(const uint32_t* q, const uint8_t* e, int R, int K, const uint16_t* x, int T, float* y,
                           void* ws, unsigned long long wait_ns, cudaStream_t s);
size_t mx_gemm_ws_bytes(int R, int K, int T);
// Codecs of the digit-block layer kernels: MXFP4 (E2M1 codes, E8M0 scale per 32), affine 4-bit
// and 2-bit codes with a bf16 scale and bias per 64 (w = q s + b).
constexpr int kCodecMx = 0, kCodecQ4 = 4, kCodecQ2 = 2;
// a decode layer on digit blocks (MXFP4 or affine 4-/2-bit experts), after the router and the top-k
struct MxLayerParams {
  int H, I, k, S, T;
  int codec;                   // 0 MXFP4, 4 affine 4-bit, 2 affine 2-bit
  const uint16_t* x;           // [T][H] bf16
  const moe_expert* experts;   // device [E]: q codes; scales E8M0 bytes [R][K/32] (MXFP4) or bf16 scales
                               // and biases [R][K/64] (affine)
  moe_expert shared;           // slot k when S > k
  const int32_t* idx; const float* w; const float* sg;   // [T][k], [T][k], [T]
  float* h;                    // [T][H], in place: h + the weighted expert outputs
  const uint8_t* xdig;         // [T][H/32] digit blocks of x (launch_mx_digits, after the router)
  uint8_t* adig;               // [T][S][I/32] digit blocks of a (written by the gate/up kernel)
};
// digit blocks of rows of K bf16 values for the layer kernels of a codec: 112 bytes per 32
cudaError_t launch_mx_digits(const uint16_t* src, int rows, int K, uint8_t* dst, int codec, cudaStream_t s, bool pdl);
cudaError_t launch_mx_layer(const MxLayerParams& p, cudaStream_t s, bool pdl = false);
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
cudaError_t launch_selftest_grid(unsigned* hdr, unsigned long long bound_ns, cudaStream_t s);
int num_sms();
// cudaFuncSetAttribute, skipped when the kernel already has that value on the current device
cudaError_t set_func_attr(const void* fn, cudaFuncAttribute attr, int value);
bool fused_supported(int H, int I, int E, int k, int has_shared, int bits);
int fused_ctas(int H, int I);
size_t fused_smem_bytes(int H, int I, int S, int bits);
cudaError_t launch_fused(const FusedParams& p, int bits, cudaStream_t s);
bool chain_supported(int H, int I, int k, int has_shared, int bits);
bool prefill_supported(int H, int I, int bits);
int pf_chunk_tokens(int H, int I);   // tokens per chunk of the grouped GEMMs
size_t pf_max_chunks(int T, int k, int E, int chunk);
int choose_ncta(long long ntiles, int nspans);
// dense tensor-core pass of the shared expert (prefill)
// Kx: K data columns plus the bias-term columns (64 per 1024 data columns or part of them)
__host__ __device__ inline int tc_cols(int K) { return K + 64 * ((K + 1023) / 1024); }
int tc_splits(int M, int T, int K);                  // column splits of a pass
bool tc_supported(int H, int I, int bits);
cudaError_t launch_tc_conv(const TcConvParams& p, cudaStream_t s);
cudaError_t launch_tc_dense(const TcParams& p, cudaStream_t s);

}  // namespace qmoe
