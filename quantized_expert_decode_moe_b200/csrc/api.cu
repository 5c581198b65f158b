// C-ABI entry points of the quantized MoE expert forward: argument checks on
// the host, then asynchronous launches on the caller's stream.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "moe.h"

using namespace qmoe;

namespace {

constexpr int kMaxE = 4096;
constexpr int kMaxHI = 8192;
constexpr int kDecodeMaxT = 8;

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Bound of every device-side wait (a staged copy that never lands, a CTA
// that never reaches a grid barrier): 100 ms, or MOE_WAIT_TIMEOUT_NS from the
// environment (read once), clamped to [1 ms, 10 s] so that a normal wait on a
// busy or time-sliced GPU does not run out.
unsigned long long wait_bound_ns() {
  static unsigned long long v = 0;
  if (!v) {
    const char* e = getenv("MOE_WAIT_TIMEOUT_NS");
    unsigned long long x = e ? strtoull(e, nullptr, 10) : 0ull;
    if (!x) x = 100000000ull;
    if (x < 1000000ull) x = 1000000ull;
    if (x > 10000000000ull) x = 10000000000ull;
    v = x;
  }
  return v;
}

moe_status check_qmat(const moe_qmat& m) {
  if (!m.q || !m.scales || !m.biases) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(m.q) || !aligned16(m.scales) || !aligned16(m.biases)) return MOE_ERR_INVALID_ARGUMENT;
  return MOE_OK;
}

// group 32 selects the MXFP4 codec (E2M1 codes, E8M0 scale bytes in moe_qmat.scales, no biases)
bool is_mx(const moe_layer* L) { return L->group == 32; }

moe_status check_mxmat(const moe_qmat& m) {
  if (!m.q || !m.scales) return MOE_ERR_INVALID_ARGUMENT;
  return aligned16(m.q) ? MOE_OK : MOE_ERR_INVALID_ARGUMENT;
}

moe_status check_layer(const moe_layer* L) {
  if (!L) return MOE_ERR_INVALID_ARGUMENT;
  if (L->bits != 2 && L->bits != 4) return MOE_ERR_UNSUPPORTED;
  if (is_mx(L) ? L->bits != 4 : L->group != kGroup) return MOE_ERR_UNSUPPORTED;
  if (L->hidden <= 0 || L->inter <= 0 || L->hidden % kSpan || L->inter % kSpan) return MOE_ERR_INVALID_ARGUMENT;
  if (L->hidden > kMaxHI || L->inter > kMaxHI) return MOE_ERR_UNSUPPORTED;
  if (L->n_experts <= 0 || L->n_experts > kMaxE) return MOE_ERR_INVALID_ARGUMENT;
  if (L->top_k <= 0 || L->top_k > kMaxTopK || L->top_k > L->n_experts) return MOE_ERR_INVALID_ARGUMENT;
  if (L->has_shared != 0 && L->has_shared != 1) return MOE_ERR_INVALID_ARGUMENT;
  if (!(L->rms_eps > 0.f) || !isfinite(L->rms_eps)) return MOE_ERR_INVALID_ARGUMENT;
  if (!L->router_w || !L->experts || !L->rms_gamma) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(L->router_w) || !aligned16(L->experts) || !aligned16(L->rms_gamma)) return MOE_ERR_INVALID_ARGUMENT;
  if (L->router_bias && !aligned16(L->router_bias)) return MOE_ERR_INVALID_ARGUMENT;
  if (L->has_shared) {
    if (!L->shared_gate_w || !aligned16(L->shared_gate_w)) return MOE_ERR_INVALID_ARGUMENT;
    moe_status s;
    auto chk = is_mx(L) ? check_mxmat : check_qmat;
    if ((s = chk(L->shared.gate)) || (s = chk(L->shared.up)) || (s = chk(L->shared.down))) return s;
  }
  return MOE_OK;
}

int slots_of(const moe_layer* L) { return L->top_k + (L->has_shared ? 1 : 0); }

// The kernels that serve T tokens of a layer, chosen on the host before any
// launch: the fused single-kernel layer for one token, the four-kernel chain
// for up to 8 tokens, the grouped prefill path above that.
//
// Decode of affine layers defaults to the digit-block kernels (mx.cu, the
// kernels of the MXFP4 layers with the affine codecs): on B200 the four-kernel
// chain measured 24.4 us per 4-bit hidden-4096 layer-token and the fused
// kernel 44.6 us, whose phases run one after another inside each CTA.
// MOE_DECODE_KERNEL in the environment (read at every call) overrides it:
// "chain" selects the four-kernel chain, "fused" the fused kernel for
// single-token calls and stacks wherever it fits (the chain otherwise).
enum class Path { kNone, kFused, kChain, kPrefill, kMx, kDigit };
enum class DecodeKernel { kDefault, kFused, kChain };
DecodeKernel decode_kernel_env() {
  const char* e = getenv("MOE_DECODE_KERNEL");
  if (e && strcmp(e, "fused") == 0) return DecodeKernel::kFused;
  if (e && strcmp(e, "chain") == 0) return DecodeKernel::kChain;
  return DecodeKernel::kDefault;
}
// The digit-block layer kernels (MXFP4 layers at any number of tokens, affine
// ones up to 8): the down kernel holds the digit blocks of every slot's SwiGLU
// output in shared memory (112 bytes per 32 values).
bool digit_smem_fits(const moe_layer* L) { return (size_t)slots_of(L) * (L->inter / 32) * 112 <= 227 * 1024; }
bool mx_supported(const moe_layer* L, int T) {
  (void)T;
  return digit_smem_fits(L);
}
int codec_of(const moe_layer* L) { return is_mx(L) ? kCodecMx : L->bits; }

Path path_of(const moe_layer* L, int T) {
  if (is_mx(L)) return mx_supported(L, T) ? Path::kMx : Path::kNone;
  if (T > kDecodeMaxT)   // the grouped prefill, else the digit-block kernels token by token
    return prefill_supported(L->hidden, L->inter, L->bits) ? Path::kPrefill
                                                           : (digit_smem_fits(L) ? Path::kDigit : Path::kNone);
  const bool fused = fused_supported(L->hidden, L->inter, L->n_experts, L->top_k, L->has_shared, L->bits);
  const bool chain = chain_supported(L->hidden, L->inter, L->top_k, L->has_shared, L->bits);
  const bool digit = digit_smem_fits(L);
  const DecodeKernel env = decode_kernel_env();
  if (T == 1 && fused && (env == DecodeKernel::kFused || (!chain && !digit))) return Path::kFused;
  if (digit && env == DecodeKernel::kDefault) return Path::kDigit;
  if (chain) return Path::kChain;
  if (digit) return Path::kDigit;
  return Path::kNone;
}

// Prefill (T > 8): the shared expert runs as dense GEMMs on the tcgen05 tensor
// cores (shared_tc.cu) from 64 tokens up, on the grouped integer kernels below
// that. MOE_PREFILL_SHARED=tc or =mma in the environment (read at every call)
// forces one of them for every prefill call.
bool shared_on_tc(const moe_layer* L, int T) {
  if (!L->has_shared || T <= kDecodeMaxT || !tc_supported(L->hidden, L->inter, L->bits)) return false;
  const char* e = getenv("MOE_PREFILL_SHARED");
  if (e && strcmp(e, "tc") == 0) return true;
  if (e && strcmp(e, "mma") == 0) return false;
  return T >= 64;
}

WsLayout layout_of(const moe_layer* L, int T) {
  return ws_layout(L->hidden, L->inter, L->n_experts, L->top_k, slots_of(L), T);
}

moe_status ws_check(const moe_layer* L, int T, void* ws, size_t ws_bytes) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if (((uintptr_t)ws & 255u) != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (ws_bytes < layout_of(L, T).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <class T> T* at(void* ws, size_t off) { return (T*)((char*)ws + off); }

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// The four-kernel decode chain of one layer for T <= 8 tokens, linked by
// programmatic dependent launch. Every kernel lets its successor launch only
// after its own dependency wait, so a kernel's pre-wait part may read what the
// kernel two places before it wrote:
//   1. router logits (weights loaded before the wait, x after it);
//   2. gate/up + SwiGLU (B tables of x and the shared expert before the wait;
//      then top-k of the logits in every CTA and the routed experts);
//   3. down + combine (top-k, residual rows and the bulk copies of its rows of
//      every chosen expert before the wait; a -> B tables and
//      hacc = h + weighted expert outputs after it);
//   4. RMSNorm of hacc into x_out, h.
moe_status decode_chain(const moe_layer* L, const uint16_t* x_in, float* h, int T, uint16_t* x_out, float* x_out_f32,
                        int32_t* topk_idx, float* topk_w, void* ws, cudaStream_t s,
                        void* const* events = nullptr, uint16_t* x_rec = nullptr, float* h_rec = nullptr) {
  const bool pdl = events == nullptr;
  auto mark = [&](int i) { if (events) cudaEventRecord((cudaEvent_t)events[i], s); };
  mark(0);
  const int H = L->hidden, I = L->inter, E = L->n_experts, k = L->top_k, S = slots_of(L);
  const WsLayout W = layout_of(L, T);
  uint32_t* status = at<uint32_t>(ws, W.status);
  RouteParams rp{};
  rp.H = H; rp.E = E; rp.T = T; rp.has_shared = L->has_shared;
  rp.x = x_in; rp.router_w = L->router_w; rp.router_bias = L->router_bias; rp.gate_w = L->shared_gate_w;
  rp.logits = at<double>(ws, W.logits);
  rp.bound = at<float>(ws, W.bound);
  rp.h = h; rp.x_rec = x_rec; rp.h_rec = h_rec;
  cudaError_t e = launch_route(rp, s, pdl);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(1);

  GateUpParams gp{};
  gp.H = H; gp.I = I; gp.E = E; gp.k = k; gp.S = S; gp.has_shared = L->has_shared;
  gp.nCTA = gateup_ctas(I);
  gp.x = x_in; gp.logits = rp.logits; gp.bound = rp.bound; gp.experts = L->experts; gp.shared = L->shared;
  gp.router_w = L->router_w; gp.router_bias = L->router_bias;
  gp.a = at<float>(ws, W.a);
  gp.idx_out = topk_idx; gp.w_out = topk_w;
  gp.sel_idx = at<int32_t>(ws, W.pidx); gp.sel_w = at<float>(ws, W.pw); gp.sel_sg = at<float>(ws, W.psg);
  gp.sel_flag = at<unsigned>(ws, kSelFlagOffset);
  gp.status = status; gp.wait_ns = wait_bound_ns();
  gp.rechecks = at<uint32_t>(ws, 16);
  if ((e = launch_gateup(gp, L->bits, T, pdl, s)) != cudaSuccess)
    return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  mark(2);

  DownParams dp{};
  dp.H = H; dp.I = I; dp.E = E; dp.k = k; dp.S = S; dp.has_shared = L->has_shared;
  dp.nCTA = down_ctas(H);
  dp.sel_idx = gp.sel_idx; dp.sel_w = gp.sel_w; dp.sel_sg = gp.sel_sg; dp.sel_flag = gp.sel_flag;
  dp.a = gp.a; dp.h = h; dp.experts = L->experts; dp.shared = L->shared;
  dp.hacc = at<float>(ws, W.hacc);
  dp.status = status; dp.wait_ns = gp.wait_ns;
  if ((e = launch_down(dp, L->bits, T, pdl, s)) != cudaSuccess)
    return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  mark(3);

  NormDecodeParams np{};
  np.H = H; np.T = T;
  np.hacc = dp.hacc; np.h = h; np.gamma = L->rms_gamma; np.eps = L->rms_eps; np.x_out = x_out; np.x_out_f32 = x_out_f32;
  np.sel_flag = gp.sel_flag;
  if ((e = launch_norm_decode(np, pdl, s)) != cudaSuccess) return MOE_ERR_CUDA;
  mark(4);
  return MOE_OK;
}

// A layer on the digit-block kernels (MXFP4 experts at any number of tokens; affine ones in decode,
// and above 8 tokens where the grouped prefill cannot take the shape): router, certified top-k,
// gate/up with SwiGLU, down with the weighted combine and the residual (mx.cu), RMSNorm.
moe_status mx_chain(const moe_layer* L, const uint16_t* x_in, float* h, int T, uint16_t* x_out, float* x_out_f32,
                    int32_t* topk_idx, float* topk_w, void* ws, cudaStream_t s, void* const* events = nullptr,
                    uint16_t* x_rec = nullptr, float* h_rec = nullptr) {
  // programmatic launches between the kernels (decode: the router of up to 8 tokens supports them)
  const bool pdl = events == nullptr && !topk_idx && !topk_w && T <= kDecodeMaxT;
  auto mark = [&](int i) { if (events) cudaEventRecord((cudaEvent_t)events[i], s); };
  mark(0);
  const int H = L->hidden, I = L->inter, E = L->n_experts, k = L->top_k, S = slots_of(L);
  const WsLayout W = layout_of(L, T);
  RouteParams rp{};
  rp.H = H; rp.E = E; rp.T = T; rp.has_shared = L->has_shared;
  rp.x = x_in; rp.router_w = L->router_w; rp.router_bias = L->router_bias; rp.gate_w = L->shared_gate_w;
  rp.logits = at<double>(ws, W.logits);
  rp.bound = at<float>(ws, W.bound);
  rp.h = h; rp.x_rec = x_rec; rp.h_rec = h_rec;
  const int codec = codec_of(L);
  if (T > kDecodeMaxT) {   // many tokens: the exact integer router on tcgen05
    rp.lpart = at<long long>(ws, W.lpart);
    rp.wdig = at<int8_t>(ws, W.wdig); rp.xdig = at<int8_t>(ws, W.xdig);
    rp.wst = at<double>(ws, W.wst); rp.xst = at<double>(ws, W.xst);
    rp.status = at<uint32_t>(ws, W.status); rp.wait_ns = wait_bound_ns();
    if (launch_route_gemm(rp, s) != cudaSuccess) return MOE_ERR_CUDA;
    // the digit blocks of x after the router
    if (launch_mx_digits(x_in, T, H, at<uint8_t>(ws, W.mxx), codec, s, false) != cudaSuccess) return MOE_ERR_CUDA;
  } else {   // decode: the router writes the digit blocks of x (the gate/up kernel reads them before its own wait)
    rp.xblocks = at<uint8_t>(ws, W.mxx);
    rp.codec = codec;
    if (launch_route(rp, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
  }
  mark(1);
  TopkParams tp{};
  tp.E = E; tp.k = k; tp.T = T; tp.has_shared = L->has_shared; tp.H = H;
  tp.logits = rp.logits; tp.bound = rp.bound;
  tp.x = x_in; tp.router_w = L->router_w; tp.router_bias = L->router_bias;
  tp.idx = at<int32_t>(ws, W.pidx); tp.w = at<float>(ws, W.pw); tp.sg = L->has_shared ? at<float>(ws, W.psg) : nullptr;
  tp.rechecks = at<uint32_t>(ws, 16);
  if (launch_topk(tp, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t sel = sizeof(int32_t) * (size_t)T * k;
  if (topk_idx && cudaMemcpyAsync(topk_idx, tp.idx, sel, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (topk_w && cudaMemcpyAsync(topk_w, tp.w, sel, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return MOE_ERR_CUDA;
  mark(2);
  MxLayerParams mp{};
  mp.H = H; mp.I = I; mp.k = k; mp.S = S; mp.T = T; mp.codec = codec;
  mp.x = x_in; mp.experts = L->experts; mp.shared = L->shared;
  mp.idx = tp.idx; mp.w = tp.w; mp.sg = tp.sg;
  mp.h = h;
  mp.xdig = at<uint8_t>(ws, W.mxx); mp.adig = at<uint8_t>(ws, W.mxa);
  if (launch_mx_layer(mp, s, pdl) != cudaSuccess) return MOE_ERR_CUDA;
  mark(3);
  NormParams np{};
  np.H = H; np.k = 0; np.T = T;
  np.h = h; np.gamma = L->rms_gamma; np.eps = L->rms_eps; np.x_out = x_out; np.x_out_f32 = x_out_f32;
  if (launch_norm(np, pdl, s) != cudaSuccess) return MOE_ERR_CUDA;
  mark(4);
  return MOE_OK;
}

// The fused decode kernel over layers [0, n) of `layers` (one token, n <= kFuMaxLayers).
moe_status fused_forward(const moe_layer* layers, int n, const uint16_t* x_in, float* h, uint16_t* x_out,
                         float* x_out_f32, int32_t* idx_out, float* w_out, uint16_t* x_rec, float* h_rec, void* ws,
                         cudaStream_t s) {
  const moe_layer& L0 = layers[0];
  const WsLayout W = layout_of(&L0, 1);
  FusedParams p{};
  p.H = L0.hidden; p.I = L0.inter; p.E = L0.n_experts; p.k = L0.top_k; p.S = slots_of(&L0);
  p.has_shared = L0.has_shared; p.nCTA = fused_ctas(L0.hidden, L0.inter); p.L = n;
  p.x_in = x_in; p.h = h; p.x_out = x_out; p.x_out_f32 = x_out_f32;
  p.idx_out = idx_out; p.w_out = w_out; p.x_rec = x_rec; p.h_rec = h_rec;
  p.status = at<uint32_t>(ws, W.status); p.hdr = at<unsigned>(ws, 0);
  p.logits = at<double>(ws, W.logits); p.bound = at<float>(ws, W.bound);
  p.a = at<float>(ws, W.a); p.hacc = at<float>(ws, W.hacc); p.gpart = at<float>(ws, W.gpart);
  p.wait_ns = wait_bound_ns();
  for (int l = 0; l < n; ++l) {
    const moe_layer& Ly = layers[l];
    FuLayer& f = p.layer[l];
    f.router_w = Ly.router_w; f.router_bias = Ly.router_bias; f.experts = Ly.experts; f.shared = Ly.shared;
    f.gate_w = Ly.shared_gate_w; f.gamma = Ly.rms_gamma; f.eps = Ly.rms_eps;
  }
  return cuda_status(launch_fused(p, L0.bits, s));
}

// Prefill (T > 8): router logits for all tokens, top-k, grouping of the
// (token, rank) pairs by expert into chunks, grouped GEMMs (gate/up + SwiGLU,
// then down) of the packed codes against fixed-point activation digits on the
// integer tensor cores, combine + residual + RMSNorm.
moe_status prefill_chain(const moe_layer* L, const uint16_t* x_in, float* h, int T, uint16_t* x_out,
                         float* x_out_f32, int32_t* topk_idx, float* topk_w, void* ws, cudaStream_t s,
                         void* const* events = nullptr) {
  auto mark = [&](int i) { if (events) cudaEventRecord((cudaEvent_t)events[i], s); };
  mark(0);
  const int H = L->hidden, I = L->inter, E = L->n_experts, k = L->top_k;
  const WsLayout W = layout_of(L, T);
  uint32_t* status = at<uint32_t>(ws, W.status);
  RouteParams rp{};
  rp.H = H; rp.E = E; rp.T = T; rp.has_shared = L->has_shared;
  rp.x = x_in; rp.router_w = L->router_w; rp.router_bias = L->router_bias; rp.gate_w = L->shared_gate_w;
  rp.logits = at<double>(ws, W.logits);
  rp.bound = at<float>(ws, W.bound);
  rp.lpart = at<long long>(ws, W.lpart);
  rp.wdig = at<int8_t>(ws, W.wdig); rp.xdig = at<int8_t>(ws, W.xdig);
  rp.wst = at<double>(ws, W.wst); rp.xst = at<double>(ws, W.xst);
  rp.status = at<uint32_t>(ws, W.status); rp.wait_ns = wait_bound_ns();
  cudaError_t e = launch_route_gemm(rp, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  mark(1);
  TopkParams tp{};
  tp.E = E; tp.k = k; tp.T = T; tp.has_shared = L->has_shared; tp.H = H;
  tp.logits = rp.logits; tp.bound = rp.bound;
  tp.x = x_in; tp.router_w = L->router_w; tp.router_bias = L->router_bias;
  tp.rechecks = at<uint32_t>(ws, 16);
  tp.idx = at<int32_t>(ws, W.pidx); tp.w = at<float>(ws, W.pw); tp.sg = at<float>(ws, W.psg);
  if ((e = launch_topk(tp, s)) != cudaSuccess) return MOE_ERR_CUDA;
  if (topk_idx && cudaMemcpyAsync(topk_idx, tp.idx, sizeof(int32_t) * (size_t)T * k, cudaMemcpyDeviceToDevice, s))
    return MOE_ERR_CUDA;
  if (topk_w && cudaMemcpyAsync(topk_w, tp.w, sizeof(float) * (size_t)T * k, cudaMemcpyDeviceToDevice, s))
    return MOE_ERR_CUDA;
  const bool tc = shared_on_tc(L, T);
  GroupParams gp{};
  gp.T = T; gp.k = k; gp.E = E; gp.has_shared = L->has_shared && !tc; gp.chunk = pf_chunk_tokens(H, I); gp.idx = tp.idx;
  gp.counts = at<int32_t>(ws, W.counts); gp.offsets = at<int32_t>(ws, W.offsets); gp.perm = at<int32_t>(ws, W.perm);
  gp.chunks = at<int4>(ws, W.chunks); gp.nchunks = at<int32_t>(ws, W.nchunks);
  if ((e = launch_group(gp, s)) != cudaSuccess) return MOE_ERR_CUDA;
  mark(2);
  PrefillParams pp{};
  pp.H = H; pp.I = I; pp.E = E; pp.k = k; pp.T = T; pp.has_shared = L->has_shared && !tc;
  pp.x = x_in;
  pp.xd = at<unsigned char>(ws, W.xd); pp.xX = at<float>(ws, W.xX); pp.xrs = at<float>(ws, W.xrs);
  pp.a = at<float>(ws, W.a);
  pp.ad = at<unsigned char>(ws, W.ad); pp.aX = at<float>(ws, W.aX); pp.ars = at<float>(ws, W.ars);
  pp.y = at<float>(ws, W.y);
  pp.chunks = gp.chunks; pp.nchunks = gp.nchunks; pp.perm = gp.perm;
  pp.experts = L->experts; pp.shared = L->shared;
  pp.status = status; pp.wait_ns = wait_bound_ns();
  // shared expert on the tensor cores: operand tables of x, gate/up partial sums
  const int Tpad = (T + 15) & ~15;
  TcConvParams cx{};
  TcParams tg{};
  if (tc) {
    cx.K = H; cx.T = T; cx.Tpad = Tpad; cx.bits = L->bits; cx.x = x_in;
    cx.b_hi = at<__half>(ws, W.tcbx); cx.tscale = at<float>(ws, W.tcxs);
    // the same launch prepares the shared expert's gate/up and down rows
    cx.nprep = 2;
    cx.prep[0] = TcRowPrep{2 * I, I, H, L->shared.gate, L->shared.up, at<int>(ws, W.tcrexp), at<__half>(ws, W.tcaext)};
    cx.prep[1] = TcRowPrep{H, H, I, L->shared.down, L->shared.down, at<int>(ws, W.tcrexp) + 2 * I,
                           at<__half>(ws, W.tcaext) + (size_t)2 * I * ((H + 1023) / 1024) * 64};
    if ((e = launch_tc_conv(cx, s)) != cudaSuccess) return MOE_ERR_CUDA;
    tg.M = 2 * I; tg.K = H; tg.R0 = I; tg.bits = L->bits; tg.w0 = L->shared.gate; tg.w1 = L->shared.up;
    tg.T = T; tg.Tpad = Tpad; tg.hilo = 0; tg.b_hi = cx.b_hi; tg.tscale = cx.tscale;
    tg.rexp = cx.prep[0].rexp; tg.aext = cx.prep[0].aext;
    tg.part = at<float>(ws, W.tcpart); tg.status = status; tg.wait_ns = pp.wait_ns;
    if ((e = launch_tc_dense(tg, s)) != cudaSuccess)
      return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  }
  if ((e = launch_prefill_gateup(pp, L->bits, s)) != cudaSuccess)
    return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  mark(3);
  if (tc) {   // SwiGLU of the split sums -> hi/lo tables of a, down partial sums
    TcConvParams ca{};
    ca.K = I; ca.T = T; ca.Tpad = Tpad; ca.bits = L->bits;
    ca.part = tg.part; ca.splits = tc_splits(2 * I, T, H); ca.I = I;
    ca.b_hi = at<__half>(ws, W.tcbah); ca.b_lo = at<__half>(ws, W.tcbal); ca.tscale = at<float>(ws, W.tcas);
    if ((e = launch_tc_conv(ca, s)) != cudaSuccess) return MOE_ERR_CUDA;
    TcParams td = tg;
    td.M = H; td.K = I; td.R0 = H; td.w0 = L->shared.down; td.w1 = L->shared.down;
    td.hilo = 1; td.b_hi = ca.b_hi; td.b_lo = ca.b_lo; td.tscale = ca.tscale;
    td.rexp = cx.prep[1].rexp; td.aext = cx.prep[1].aext;
    if ((e = launch_tc_dense(td, s)) != cudaSuccess)
      return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  }
  if ((e = launch_prefill_down(pp, L->bits, s)) != cudaSuccess)
    return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : MOE_ERR_CUDA;
  mark(4);
  NormParams np{};
  np.H = H; np.k = k; np.T = T;
  np.y_routed = pp.y; np.y_routed_tok_stride = (long long)k * H; np.y_routed_slot_stride = H;
  np.w = tp.w;
  np.y_shared = L->has_shared ? pp.y + (size_t)T * k * H : nullptr; np.y_shared_tok_stride = H;
  if (tc) {
    np.y_shared = at<float>(ws, W.tcpart);
    np.y_shared_splits = tc_splits(H, T, I);
    np.y_shared_split_stride = (long long)T * H;
  }
  np.sg = tp.sg;
  np.h = h; np.gamma = L->rms_gamma; np.eps = L->rms_eps; np.x_out = x_out; np.x_out_f32 = x_out_f32;
  if ((e = launch_norm(np, false, s)) != cudaSuccess) return MOE_ERR_CUDA;
  mark(5);
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return 1; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_FAULT: return "device-side fault (expert id out of range)";
  }
  return "unknown status";
}

moe_status moe_workspace_size(const moe_layer* layer, int32_t max_tokens, size_t* bytes) {
  moe_status st = check_layer(layer);
  if (st) return st;
  if (!bytes || max_tokens <= 0) return MOE_ERR_INVALID_ARGUMENT;
  if (path_of(layer, max_tokens) == Path::kNone) return MOE_ERR_UNSUPPORTED;
  *bytes = layout_of(layer, max_tokens).total;
  return MOE_OK;
}

moe_status moe_layer_path(const moe_layer* layer, int32_t T, int32_t* path, int32_t* n_events) {
  moe_status st = check_layer(layer);
  if (st) return st;
  if (T <= 0) return MOE_ERR_INVALID_ARGUMENT;
  const Path pa = path_of(layer, T);
  int32_t code = 0, ev = 0;
  switch (pa) {
    case Path::kFused: code = MOE_PATH_FUSED; ev = 2; break;
    case Path::kChain: code = MOE_PATH_CHAIN; ev = 5; break;
    case Path::kPrefill: code = MOE_PATH_PREFILL; ev = 6; break;
    case Path::kMx: code = MOE_PATH_MXFP4; ev = 5; break;
    case Path::kDigit: code = MOE_PATH_DIGIT; ev = 5; break;
    default: return MOE_ERR_UNSUPPORTED;
  }
  if (path) *path = code;
  if (n_events) *n_events = ev;
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream));
}

moe_status moe_route(const moe_layer* layer, const uint16_t* x, int32_t T, int32_t* topk_idx, float* topk_w,
                     float* shared_gate, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_layer(layer);
  if (st) return st;
  if (T <= 0 || !x || !topk_idx || !topk_w || !aligned16(x)) return MOE_ERR_INVALID_ARGUMENT;
  if ((st = ws_check(layer, T, ws, ws_bytes))) return st;
  const WsLayout W = layout_of(layer, T);
  cudaStream_t s = (cudaStream_t)stream;
  RouteParams rp{};
  rp.H = layer->hidden; rp.E = layer->n_experts; rp.T = T; rp.has_shared = layer->has_shared;
  rp.x = x; rp.router_w = layer->router_w; rp.router_bias = layer->router_bias; rp.gate_w = layer->shared_gate_w;
  rp.logits = at<double>(ws, W.logits);
  rp.bound = at<float>(ws, W.bound);
  rp.lpart = at<long long>(ws, W.lpart);
  rp.wdig = at<int8_t>(ws, W.wdig); rp.xdig = at<int8_t>(ws, W.xdig);
  rp.wst = at<double>(ws, W.wst); rp.xst = at<double>(ws, W.xst);
  rp.status = at<uint32_t>(ws, W.status); rp.wait_ns = wait_bound_ns();
  if ((T > kDecodeMaxT ? launch_route_gemm(rp, s) : launch_route(rp, s, false)) != cudaSuccess) return MOE_ERR_CUDA;
  TopkParams tp{};
  tp.E = layer->n_experts; tp.k = layer->top_k; tp.T = T; tp.has_shared = layer->has_shared; tp.H = layer->hidden;
  tp.logits = rp.logits; tp.bound = rp.bound;
  tp.x = x; tp.router_w = layer->router_w; tp.router_bias = layer->router_bias;
  tp.idx = topk_idx; tp.w = topk_w; tp.sg = shared_gate;
  tp.rechecks = at<uint32_t>(ws, 16);
  return cuda_status(launch_topk(tp, s));
}

static moe_status gemv_common(const moe_qmat* W, int32_t R, int32_t K, int32_t group, const float* x, float* y,
                              int bits, void* stream) {
  if (!W || !x || !y) return MOE_ERR_INVALID_ARGUMENT;
  if (group != kGroup) return MOE_ERR_UNSUPPORTED;
  if (R <= 0 || R % 16 || K <= 0 || K % kSpan || K > 65536) return MOE_ERR_INVALID_ARGUMENT;
  moe_status st = check_qmat(*W);
  if (st) return st;
  if (!aligned16(x) || !aligned16(y)) return MOE_ERR_INVALID_ARGUMENT;
  cudaStream_t s = (cudaStream_t)stream;
  GemvParams p{};
  p.R = R; p.K = K; p.nspans = K / kSpan; p.ntiles = (R + 15) / 16;
  p.U = (long long)p.ntiles * p.nspans; p.nCTA = choose_ncta(p.ntiles, p.nspans);
  p.W = *W; p.x = x; p.y = y; p.status = nullptr; p.wait_ns = wait_bound_ns();
  if (cudaMemsetAsync(y, 0, sizeof(float) * (size_t)R, s) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t e = launch_gemv(p, bits, s);
  return e == cudaErrorInvalidConfiguration ? MOE_ERR_UNSUPPORTED : cuda_status(e);
}

moe_status moe_expert_gemv_q4(const moe_qmat* W, int32_t R, int32_t K, int32_t group, const float* x, float* y,
                              void* stream) {
  return gemv_common(W, R, K, group, x, y, 4, stream);
}

moe_status moe_expert_gemv_q2(const moe_qmat* W, int32_t R, int32_t K, int32_t group, const float* x, float* y,
                              void* stream) {
  return gemv_common(W, R, K, group, x, y, 2, stream);
}

moe_status moe_expert_gemv_mxfp4(const moe_mxmat* W, int32_t R, int32_t K, const float* x, float* y, void* stream) {
  if (!W || !W->q || !W->scales || !x || !y || R <= 0 || K <= 0 || K % 32) return MOE_ERR_INVALID_ARGUMENT;
  if (K > kMaxHI) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(W->q) || !aligned16(x)) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_mx_gemv(W->q, W->scales, R, K, x, y, (cudaStream_t)stream));
}

moe_status moe_mxfp4_workspace_size(int32_t R, int32_t K, int32_t T, size_t* bytes) {
  if (!bytes || R <= 0 || K <= 0 || T <= 0) return MOE_ERR_INVALID_ARGUMENT;
  if (R % 128 || K % 128 || K > kMaxHI) return MOE_ERR_UNSUPPORTED;
  *bytes = mx_gemm_ws_bytes(R, K, T);
  return MOE_OK;
}

moe_status moe_expert_gemm_mxfp4(const moe_mxmat* W, int32_t R, int32_t K, const uint16_t* x, int32_t T, float* y,
                                 void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  moe_status st = moe_mxfp4_workspace_size(R, K, T, &need);
  if (st) return st;
  if (!W || !W->q || !W->scales || !x || !y || !ws) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(W->q) || ((uintptr_t)W->scales & 3) || !aligned16(x) || ((uintptr_t)ws & 255))
    return MOE_ERR_INVALID_ARGUMENT;
  if (ws_bytes < need) return MOE_ERR_WORKSPACE;
  return cuda_status(launch_mx_gemm(W->q, W->scales, R, K, x, T, y, ws, wait_bound_ns(), (cudaStream_t)stream));
}

moe_status moe_combine_residual_norm(int32_t T, int32_t H, int32_t k, const float* y_routed, const float* topk_w,
                                     const float* y_shared, const float* shared_gate, float* h,
                                     const uint16_t* gamma, float eps, uint16_t* x_out, float* x_out_f32,
                                     void* stream) {
  if (T <= 0 || H <= 0 || k < 0 || k > kMaxTopK) return MOE_ERR_INVALID_ARGUMENT;
  if (H % 8 || H > kMaxHI) return MOE_ERR_UNSUPPORTED;   // eight equal row slices per token, H <= 8192
  if ((k > 0 && (!y_routed || !topk_w)) || !h || !gamma || !x_out) return MOE_ERR_INVALID_ARGUMENT;
  if (y_shared && !shared_gate) return MOE_ERR_INVALID_ARGUMENT;
  if (!(eps > 0.f) || !isfinite(eps)) return MOE_ERR_INVALID_ARGUMENT;
  NormParams np{};
  np.H = H; np.k = k; np.T = T;
  np.y_routed = y_routed; np.y_routed_tok_stride = (long long)k * H; np.y_routed_slot_stride = H;
  np.w = topk_w; np.y_shared = y_shared; np.y_shared_tok_stride = H; np.sg = shared_gate;
  np.h = h; np.gamma = gamma; np.eps = eps; np.x_out = x_out; np.x_out_f32 = x_out_f32;
  return cuda_status(launch_norm(np, false, (cudaStream_t)stream));
}

moe_status moe_group_tokens(int32_t T, int32_t k, int32_t E, const int32_t* topk_idx, int32_t* counts,
                            int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  (void)ws; (void)ws_bytes;
  if (T <= 0 || k <= 0 || k > kMaxTopK || E <= 0 || E > kMaxE) return MOE_ERR_INVALID_ARGUMENT;
  if (!topk_idx || !counts || !offsets || !perm) return MOE_ERR_INVALID_ARGUMENT;
  GroupParams p{};
  p.T = T; p.k = k; p.E = E; p.idx = topk_idx; p.counts = counts; p.offsets = offsets; p.perm = perm;
  return cuda_status(launch_group(p, (cudaStream_t)stream));
}

moe_status moe_layer_forward(const moe_layer* layer, const uint16_t* x_in, float* h, int32_t T, uint16_t* x_out,
                             float* x_out_f32, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                             void* stream) {
  moe_status st = check_layer(layer);
  if (st) return st;
  if (T <= 0 || !x_in || !h || !x_out) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(h) || !aligned16(x_out)) return MOE_ERR_INVALID_ARGUMENT;
  if ((st = ws_check(layer, T, ws, ws_bytes))) return st;
  const Path path = path_of(layer, T);
  cudaStream_t s = (cudaStream_t)stream;
  switch (path) {
    case Path::kPrefill: return prefill_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s);
    case Path::kFused:
      return fused_forward(layer, 1, x_in, h, x_out, x_out_f32, topk_idx, topk_w, nullptr, nullptr, ws, s);
    case Path::kChain: return decode_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s);
    case Path::kMx:
    case Path::kDigit: return mx_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s);
    default: return MOE_ERR_UNSUPPORTED;
  }
}

moe_status moe_layer_forward_timed(const moe_layer* layer, const uint16_t* x_in, float* h, int32_t T,
                                   uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w, void* ws,
                                   size_t ws_bytes, void* const* events, int32_t n_events, void* stream) {
  moe_status st = check_layer(layer);
  if (st) return st;
  if (T <= 0 || !x_in || !h || !x_out) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(h) || !aligned16(x_out)) return MOE_ERR_INVALID_ARGUMENT;
  if ((st = ws_check(layer, T, ws, ws_bytes))) return st;
  const Path path = path_of(layer, T);
  if (path == Path::kNone) return MOE_ERR_UNSUPPORTED;
  // kernels (or kernel groups) of the path + 1
  const int need = path == Path::kPrefill ? 6 : (path == Path::kFused ? 2 : 5);
  if (!events || n_events < need) return MOE_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < need; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARGUMENT;
  cudaStream_t s = (cudaStream_t)stream;
  if (path == Path::kPrefill)
    return prefill_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s, events);
  if (path == Path::kMx || path == Path::kDigit)
    return mx_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s, events);
  if (path == Path::kFused) {
    if (cudaEventRecord((cudaEvent_t)events[0], s) != cudaSuccess) return MOE_ERR_CUDA;
    if ((st = fused_forward(layer, 1, x_in, h, x_out, x_out_f32, topk_idx, topk_w, nullptr, nullptr, ws, s)))
      return st;
    return cuda_status(cudaEventRecord((cudaEvent_t)events[1], s));
  }
  return decode_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s, events);
}

moe_status moe_stack_forward(const moe_layer* layers, int32_t L, const uint16_t* x_in, float* h, uint16_t* x_out,
                             int32_t* topk_idx_all, uint16_t* layer_inputs, float* layer_h, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!layers || L <= 0 || !x_in || !h || !x_out) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(h) || !aligned16(x_out)) return MOE_ERR_INVALID_ARGUMENT;
  moe_status st;
  for (int l = 0; l < L; ++l) {
    if ((st = check_layer(&layers[l]))) return st;
    const moe_layer& a = layers[l], &b = layers[0];
    if (a.hidden != b.hidden || a.inter != b.inter || a.n_experts != b.n_experts || a.top_k != b.top_k ||
        a.bits != b.bits || a.group != b.group || a.has_shared != b.has_shared)
      return MOE_ERR_INVALID_ARGUMENT;
  }
  if ((st = ws_check(&layers[0], 1, ws, ws_bytes))) return st;
  const Path path = path_of(&layers[0], 1);   // every layer has the first one's shape
  if (path == Path::kNone) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  const int H = layers[0].hidden, k = layers[0].top_k;
  if (path == Path::kFused) {   // up to kFuMaxLayers layers per launch, x and h stay on chip in between
    for (int l0 = 0; l0 < L; l0 += kFuMaxLayers) {
      const int n = L - l0 < kFuMaxLayers ? L - l0 : kFuMaxLayers;
      if ((st = fused_forward(layers + l0, n, l0 == 0 ? x_in : x_out, h, x_out, nullptr,
                              topk_idx_all ? topk_idx_all + (size_t)l0 * k : nullptr, nullptr,
                              layer_inputs ? layer_inputs + (size_t)l0 * H : nullptr,
                              layer_h ? layer_h + (size_t)l0 * H : nullptr, ws, s)))
        return st;
    }
    return MOE_OK;
  }
  for (int l = 0; l < L; ++l) {
    const uint16_t* xin = l == 0 ? x_in : x_out;
    if (path == Path::kMx || path == Path::kDigit) {
      if ((st = mx_chain(&layers[l], xin, h, 1, x_out, nullptr, topk_idx_all ? topk_idx_all + (size_t)l * k : nullptr,
                         nullptr, ws, s, nullptr, layer_inputs ? layer_inputs + (size_t)l * H : nullptr,
                         layer_h ? layer_h + (size_t)l * H : nullptr)))
        return st;
      continue;
    }
    if ((st = decode_chain(&layers[l], xin, h, 1, x_out, nullptr, topk_idx_all ? topk_idx_all + (size_t)l * k : nullptr,
                           nullptr, ws, s, nullptr, layer_inputs ? layer_inputs + (size_t)l * H : nullptr,
                           layer_h ? layer_h + (size_t)l * H : nullptr)))
      return st;
  }
  return MOE_OK;
}

}  // extern "C"

// Scratch of moe_layer_forward_noalloc: one file-scope device array, so that
// callers that cannot allocate still get a workspace. Host code only sees a
// host-side stand-in under this name; the device address is looked up once
// per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on failure).
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" {

moe_status moe_layer_forward_noalloc(const moe_layer* layer, const uint16_t* x_in, float* h, int32_t T,
                                     uint16_t* x_out, float* x_out_f32, int32_t* topk_idx, float* topk_w,
                                     void* stream) {
  moe_status st = check_layer(layer);
  if (st) return st;
  if (T <= 0 || !x_in || !h || !x_out) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned16(x_in) || !aligned16(h) || !aligned16(x_out)) return MOE_ERR_INVALID_ARGUMENT;
  if (T > kDecodeMaxT) return MOE_ERR_UNSUPPORTED;
  const Path path = path_of(layer, T);
  if (path == Path::kNone) return MOE_ERR_UNSUPPORTED;
  if (layout_of(layer, T).total > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  void* ws = noalloc_scratch();
  if (!ws) return MOE_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // The scratch starts zeroed (a static device array), so its status word and
  // grid-barrier counters start clear; a latched error stays until
  // moe_noalloc_poll_status reads it. The kernels clear their own accumulators.
  if (path == Path::kFused)
    return fused_forward(layer, 1, x_in, h, x_out, x_out_f32, topk_idx, topk_w, nullptr, nullptr, ws, s);
  if (path == Path::kMx || path == Path::kDigit) return mx_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s);
  return decode_chain(layer, x_in, h, T, x_out, x_out_f32, topk_idx, topk_w, ws, s);
}

moe_status moe_noalloc_poll_status(void* stream) {
  void* ws = noalloc_scratch();
  if (!ws) return MOE_ERR_CUDA;
  return moe_poll_status(ws, stream);
}

moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t bound_ns, void* stream) {
  if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  if (((uintptr_t)ws & 255u) != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (bound_ns == 0 || bound_ns > 10000000000ull) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_selftest_wait((uint32_t*)ws, (unsigned long long)bound_ns, (cudaStream_t)stream));
}

moe_status moe_selftest_grid_timeout(void* ws, size_t ws_bytes, uint64_t bound_ns, void* stream) {
  if (!ws || ws_bytes < 256) return MOE_ERR_WORKSPACE;
  if (((uintptr_t)ws & 255u) != 0) return MOE_ERR_INVALID_ARGUMENT;
  if (bound_ns == 0 || bound_ns > 10000000000ull) return MOE_ERR_INVALID_ARGUMENT;
  return cuda_status(launch_selftest_grid((unsigned*)ws, (unsigned long long)bound_ns, (cudaStream_t)stream));
}

moe_status moe_poll_status(void* ws, void* stream) {
  if (!ws) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v) {   // clear the status word and the grid-barrier counters a failed call may have left mid-round
    if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  return (moe_status)v;
}

}  // extern "C"
