/*
 * CPU oracle for the quantized MoE expert forward (Flash-MoE engine).
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and
 * the bench's CPU-baseline leg may load this library. The product path never
 * calls it, links it or falls back to it.
 *
 * Plain, slow, obviously correct: every value is carried in IEEE double,
 * every dot product is a naive loop accumulated in index order, and nothing
 * is blocked, fused or reordered. It shares no code with the CUDA library.
 *
 * What it computes (Flash-MoE write-up as summarised on the pages):
 *   - "Model architecture": each layer has 512 experts and K=4 active per
 *     token, one of them a shared expert; hidden size 4096.
 *   - "Key technologies > FMA-optimised dequant kernel": a weight is the code
 *     (nibble) times a group scale plus a group bias, w = q*s + b, applied to
 *     the activation as (q*s + b)*x.
 *   - "Key technologies > Metal compute shaders": 4-bit/2-bit dequant
 *     matrix-vector products, SwiGLU, RMS normalisation, and the MoE combine
 *     with residual and gate.
 *   - "Key technologies > Deferred GPU expert compute": combine +
 *     normalisation + residual run on the device and feed the next layer.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - Packed layout: uint32 words, row-major [R][K*bits/32]; element k of a
 *     row is in word k/(32/bits), bits [bits*(k%(32/bits)), +bits), LSB first.
 *     Scales and biases are bf16 [R][K/G], group = G consecutive k of a row.
 *   - Router: logits l = W_r x (+ optional per-expert bias); p = softmax(l)
 *     over all experts; the k largest logits are chosen (ties: lower index
 *     first), output in descending-logit order; weights are p renormalised
 *     over the chosen k.
 *   - Shared expert: gate sigma(g_s . x), applied to its output.
 *   - SwiGLU: silu(gate) * up, silu(z) = z / (1 + e^-z).
 *   - Combine: h' = h + sum_i w_i y_i + sigma(g_s.x) y_s.
 *   - RMSNorm: x_out = h' / sqrt(mean(h'^2) + eps) * gamma.
 *   - Prefill grouping: histogram of chosen experts, exclusive scan, stable
 *     scatter of the flattened (token, rank) pairs.
 *
 * Parity pins: see the oracle tests (closed forms, exact rational arithmetic,
 * library routines on tiny shapes, the pages' byte counts).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1

int oracle_abi_version(void) { return 1; }

int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bf16 (ties to even), directly (no float step). */
uint16_t oracle_double_to_bf16(double v) {
  if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
  int e;
  double m = frexp(v, &e);                /* v = m * 2^e, 0.5 <= |m| < 1 */
  double r = nearbyint(ldexp(m, 8));      /* 8 significant bits, ties to even */
  double q = ldexp(r, e - 8);             /* exactly representable in float */
  float f = (float)q;
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/* code of element (r, k) in the packed canonical layout */
static unsigned code_at(const uint32_t* q, int K, int bits, int r, int k) {
  int per_word = 32 / bits;
  size_t words_per_row = (size_t)K / per_word;
  uint32_t w = q[(size_t)r * words_per_row + (size_t)(k / per_word)];
  unsigned shift = (unsigned)(bits * (k % per_word));
  return (w >> shift) & ((1u << bits) - 1u);
}

/* Dequantised weight w[r][k] = q * s + b (exact in double). */
double oracle_weight(const uint32_t* q, const uint16_t* s, const uint16_t* b,
                     int K, int G, int bits, int r, int k) {
  size_t gi = (size_t)r * (size_t)(K / G) + (size_t)(k / G);
  return (double)code_at(q, K, bits, r, k) * oracle_bf16_to_double(s[gi]) + oracle_bf16_to_double(b[gi]);
}

/* Dense dequantisation of a whole matrix into double [R][K]. */
int oracle_dequant(int R, int K, int G, int bits, const uint32_t* q, const uint16_t* s,
                   const uint16_t* b, double* w) {
  if (R < 0 || K <= 0 || G <= 0 || K % G || (bits != 2 && bits != 4)) return ORC_EINVAL;
  for (int r = 0; r < R; ++r)
    for (int k = 0; k < K; ++k) w[(size_t)r * K + k] = oracle_weight(q, s, b, K, G, bits, r, k);
  return ORC_OK;
}

/* y[r] = sum_k (q[r][k] * s + b) * x[k], naive, index order, in double. */
int oracle_qgemv(int R, int K, int G, int bits, const uint32_t* q, const uint16_t* s,
                 const uint16_t* b, const double* x, double* y) {
  if (R < 0 || K <= 0 || G <= 0 || K % G || (bits != 2 && bits != 4) || K % (32 / bits)) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    double acc = 0.0;
    for (int k = 0; k < K; ++k) acc += oracle_weight(q, s, b, K, G, bits, r, k) * x[k];
    y[r] = acc;
  }
  return ORC_OK;
}

double oracle_silu(double z) { return z / (1.0 + exp(-z)); }
double oracle_sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* a = silu(g) * u */
void oracle_swiglu(int n, const double* g, const double* u, double* a) {
  for (int i = 0; i < n; ++i) a[i] = oracle_silu(g[i]) * u[i];
}

/* One expert: y = D (silu(G x) * (U x)). gate/up are [I][H], down is [H][I]. */
int oracle_expert(int H, int I, int G, int bits,
                  const uint32_t* gq, const uint16_t* gs, const uint16_t* gb,
                  const uint32_t* uq, const uint16_t* us, const uint16_t* ub,
                  const uint32_t* dq, const uint16_t* ds, const uint16_t* db,
                  const double* x, double* y, double* a_out /* [I], nullable */) {
  double* g = (double*)malloc(sizeof(double) * (size_t)I);
  double* u = (double*)malloc(sizeof(double) * (size_t)I);
  double* a = (double*)malloc(sizeof(double) * (size_t)I);
  int rc = ORC_EINVAL;
  if (!g || !u || !a) goto done;
  if ((rc = oracle_qgemv(I, H, G, bits, gq, gs, gb, x, g))) goto done;
  if ((rc = oracle_qgemv(I, H, G, bits, uq, us, ub, x, u))) goto done;
  oracle_swiglu(I, g, u, a);
  if (a_out) memcpy(a_out, a, sizeof(double) * (size_t)I);
  rc = oracle_qgemv(H, I, G, bits, dq, ds, db, a, y);
done:
  free(g); free(u); free(a);
  return rc;
}

/*
 * Router for T tokens. x bf16 [T][H], Wr bf16 [E][H], bias fp32 [E] (nullable),
 * gs bf16 [H] (nullable). Outputs: logits [T][E] (nullable), idx [T][k],
 * w [T][k], shared_gate [T] (nullable; sigma(gs . x)).
 */
int oracle_route(int T, int H, int E, int k, const uint16_t* x, const uint16_t* Wr,
                 const float* bias, const uint16_t* gs, double* logits_out,
                 int32_t* idx, double* w, double* shared_gate) {
  if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return ORC_EINVAL;
  double* l = (double*)malloc(sizeof(double) * (size_t)E);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  char* taken = (char*)malloc((size_t)E);
  if (!l || !p || !taken) { free(l); free(p); free(taken); return ORC_EINVAL; }
  for (int t = 0; t < T; ++t) {
    const uint16_t* xt = x + (size_t)t * H;
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += oracle_bf16_to_double(Wr[(size_t)e * H + h]) * oracle_bf16_to_double(xt[h]);
      if (bias) acc += (double)bias[e];
      l[e] = acc;
      if (logits_out) logits_out[(size_t)t * E + e] = acc;
    }
    /* full softmax over all experts */
    double lmax = l[0];
    for (int e = 1; e < E; ++e) if (l[e] > lmax) lmax = l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) { p[e] = exp(l[e] - lmax); z += p[e]; }
    for (int e = 0; e < E; ++e) p[e] /= z;
    /* top-k by logit, ties to the lower index, descending order */
    memset(taken, 0, (size_t)E);
    double psum = 0.0;
    for (int i = 0; i < k; ++i) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;
      }
      taken[best] = 1;
      idx[(size_t)t * k + i] = best;
      psum += p[best];
    }
    /* renormalise the chosen probabilities */
    for (int i = 0; i < k; ++i) w[(size_t)t * k + i] = p[idx[(size_t)t * k + i]] / psum;
    if (shared_gate) {
      if (gs) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h) acc += oracle_bf16_to_double(gs[h]) * oracle_bf16_to_double(xt[h]);
        shared_gate[t] = oracle_sigmoid(acc);
      } else {
        shared_gate[t] = 0.0;
      }
    }
  }
  free(l); free(p); free(taken);
  return ORC_OK;
}

/*
 * Combine + residual + RMSNorm for one token.
 * y_routed [k][H], w [k], y_shared [H] (nullable), sg = shared gate value,
 * h_in [H]. Outputs h_out [H], x_out [H] (double) and x_out_bf16 [H] (nullable).
 */
int oracle_combine_norm(int H, int k, const double* y_routed, const double* w,
                        const double* y_shared, double sg, const double* h_in,
                        const uint16_t* gamma, double eps, double* h_out,
                        double* x_out, uint16_t* x_out_bf16) {
  if (H <= 0 || k < 0) return ORC_EINVAL;
  double ss = 0.0;
  for (int j = 0; j < H; ++j) {
    double v = h_in[j];
    for (int i = 0; i < k; ++i) v += w[i] * y_routed[(size_t)i * H + j];
    if (y_shared) v += sg * y_shared[j];
    h_out[j] = v;
    ss += v * v;
  }
  double inv = 1.0 / sqrt(ss / (double)H + eps);
  for (int j = 0; j < H; ++j) {
    double v = h_out[j] * inv * oracle_bf16_to_double(gamma[j]);
    x_out[j] = v;
    if (x_out_bf16) x_out_bf16[j] = oracle_double_to_bf16(v);
  }
  return ORC_OK;
}

/*
 * Prefill grouping of routed (token, rank) pairs by expert.
 * idx [T][k] -> counts [E], offsets [E+1] (exclusive scan), perm [T*k]:
 * perm[offsets[e] + n] is the n-th pair (in flattened t*k + r order) routed to e.
 */
int oracle_group_by_expert(int T, int k, int E, const int32_t* idx, int32_t* counts,
                           int32_t* offsets, int32_t* perm) {
  if (T < 0 || k <= 0 || E <= 0) return ORC_EINVAL;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int p = 0; p < T * k; ++p) {
    int e = idx[p];
    if (e < 0 || e >= E) return ORC_EINVAL;
    counts[e]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  if (!fill) return ORC_EINVAL;
  for (int p = 0; p < T * k; ++p) {
    int e = idx[p];
    perm[offsets[e] + fill[e]++] = p;
  }
  free(fill);
  return ORC_OK;
}

/* One packed matrix: codes, scales, biases (host pointers). */
typedef struct {
  const uint32_t* q;
  const uint16_t* s;
  const uint16_t* b;
} orc_mat;

typedef struct {
  orc_mat gate, up, down;
} orc_expert;

/*
 * Whole MoE layer for T tokens with every expert resident in host memory.
 * experts: host array [E] (nullable entries are not allowed for chosen ones);
 * shared: nullable. x bf16 [T][H]; h_in [T][H] double; outputs h_out, x_out
 * [T][H] double, x_out_bf16 [T][H], idx [T][k], w [T][k], shared_gate [T].
 * Per token, the routed outputs are summed in rank order, then the shared one.
 */
int oracle_layer(int T, int H, int I, int E, int k, int G, int bits, double eps,
                 const uint16_t* Wr, const float* router_bias, const uint16_t* gs,
                 const uint16_t* gamma, const orc_expert* experts, const orc_expert* shared,
                 const uint16_t* x, const double* h_in, double* h_out, double* x_out,
                 uint16_t* x_out_bf16, int32_t* idx, double* w, double* shared_gate) {
  int rc;
  double* sgate = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  double* xd = (double*)malloc(sizeof(double) * (size_t)H);
  double* yr = (double*)malloc(sizeof(double) * (size_t)k * H);
  double* ys = (double*)malloc(sizeof(double) * (size_t)H);
  if (!sgate || !xd || !yr || !ys) { rc = ORC_EINVAL; goto done; }
  if ((rc = oracle_route(T, H, E, k, x, Wr, router_bias, shared ? gs : NULL, NULL, idx, w, sgate))) goto done;
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < H; ++j) xd[j] = oracle_bf16_to_double(x[(size_t)t * H + j]);
    for (int i = 0; i < k; ++i) {
      const orc_expert* ex = &experts[idx[(size_t)t * k + i]];
      if ((rc = oracle_expert(H, I, G, bits, ex->gate.q, ex->gate.s, ex->gate.b, ex->up.q, ex->up.s,
                              ex->up.b, ex->down.q, ex->down.s, ex->down.b, xd, yr + (size_t)i * H, NULL)))
        goto done;
    }
    if (shared) {
      if ((rc = oracle_expert(H, I, G, bits, shared->gate.q, shared->gate.s, shared->gate.b, shared->up.q,
                              shared->up.s, shared->up.b, shared->down.q, shared->down.s, shared->down.b,
                              xd, ys, NULL)))
        goto done;
    }
    if ((rc = oracle_combine_norm(H, k, yr, w + (size_t)t * k, shared ? ys : NULL, sgate[t],
                                  h_in + (size_t)t * H, gamma, eps, h_out + (size_t)t * H,
                                  x_out + (size_t)t * H, x_out_bf16 ? x_out_bf16 + (size_t)t * H : NULL)))
      goto done;
    if (shared_gate) shared_gate[t] = shared ? sgate[t] : 0.0;
  }
done:
  free(sgate); free(xd); free(yr); free(ys);
  return rc;
}

/*
 * MXFP4 expert matrices (page 4, "300b on 32gb MoE-streaming findings +
 * optimisations": the streamed experts are MXFP4). The pages name the format
 * only; the reading is the OCP Microscaling Formats (MX) v1.0 definition:
 *   - a block of 32 consecutive k of a row shares one scale, E8M0: an 8-bit
 *     biased exponent, value 2^(byte - 127), byte 0xFF = NaN;
 *   - each element is FP4 E2M1: bit 3 sign, bits 2..1 exponent (bias 1),
 *     bit 0 mantissa; exponent field 0 is subnormal (0.5 * mantissa),
 *     otherwise 2^(exponent - 1) * (1 + mantissa / 2); no infinities or NaN;
 *   - weight = scale * element.
 * Layout (same packing as the 4-bit codes): codes uint32 [R][K/8], element k
 * of a row in word k/8 at bits 4*(k%8), LSB first; scales uint8 [R][K/32].
 */
double oracle_e2m1(unsigned code) {
  const unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  const double mag = e == 0 ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
  return s ? -mag : mag;
}

double oracle_e8m0(unsigned byte) {
  if ((byte & 0xFFu) == 0xFFu) return NAN;
  return ldexp(1.0, (int)(byte & 0xFFu) - 127);
}

/* Weight (r, k) of an MXFP4 matrix, exact in double. */
double oracle_mx_weight(const uint32_t* q, const uint8_t* e, int K, int r, int k) {
  const unsigned code = code_at(q, K, 4, r, k);
  return oracle_e2m1(code) * oracle_e8m0(e[(size_t)r * (size_t)(K / 32) + (size_t)(k / 32)]);
}

/* Dense dequantisation of an MXFP4 matrix into double [R][K]. */
int oracle_mx_dequant(int R, int K, const uint32_t* q, const uint8_t* e, double* w) {
  if (R < 0 || K <= 0 || K % 32) return ORC_EINVAL;
  for (int r = 0; r < R; ++r)
    for (int k = 0; k < K; ++k) w[(size_t)r * K + k] = oracle_mx_weight(q, e, K, r, k);
  return ORC_OK;
}

/* y[r] = sum_k w[r][k] x[k] for an MXFP4 matrix, naive, index order, in double. */
int oracle_mx_gemv(int R, int K, const uint32_t* q, const uint8_t* e, const double* x, double* y) {
  if (R < 0 || K <= 0 || K % 32) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    double acc = 0.0;
    for (int k = 0; k < K; ++k) acc += oracle_mx_weight(q, e, K, r, k) * x[k];
    y[r] = acc;
  }
  return ORC_OK;
}
