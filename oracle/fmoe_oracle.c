/*
 * fmoe_oracle.c -- plain, slow, fp64 CPU oracle of the routed-MoE decode block
 * and of the Gated DeltaNet state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code with the CUDA path.
 *
 * What it computes follows the Flash-MoE pages:
 *   - "What is Flash-MoE" (a2a-mcp.org), MoE section: a router picks 4 of
 *     512 routed experts per layer and one shared expert always runs;
 *   - same page, section 2 (FMA-optimised dequantisation kernel): the naive
 *     dequantisation form  w = code * scale + bias  (the oracle uses this form,
 *     element by element, never the rearranged fma form);
 *   - same page, section 3 (hand-tuned Metal shaders): two-pass RMSNorm (sum of
 *     squares, then apply), fused SwiGLU, and one combine pass of the weighted
 *     expert outputs, the residual and the sigmoid-gated shared expert;
 *   - "Flash-MoE" wiki summary (jeongsk), per-layer pipeline: routing
 *     projection, then softmax and top-K selection;
 *   - same page section 4 and the wiki summary's key technique 4: the Gated
 *     DeltaNet state update of the linear-attention layers (or_gdn_step, at
 *     the end of this file).
 * Readings where the pages are silent (code order LSB-first, unsigned codes,
 * groups of 64 along the input dimension, router [E][H] in bf16, softmax over
 * all E then top-K then renormalisation, ties to the lower index, eps 1e-6)
 * are the ones listed in the design notes of this repository.
 *
 * Arithmetic is fp64 throughout; bf16 and fp32 inputs widen exactly.
 * OpenMP parallelises only independent output rows (no reordering of any sum).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One packed matrix [rows][cols]: words uint32[rows][cols*bits/32],
 * scale/bias bf16[rows][cols/group]. */
typedef struct {
  int bits, group, rows, cols;
  const uint32_t* qw;
  const uint16_t* scale;
  const uint16_t* bias;
} or_matrix;

/* A bank of expert records: record e at base + e*stride, or at records[e]
 * when the pointer table `records` is not NULL (lets a test hold only the
 * records a token selects); off[] holds the byte offsets of gate{qw,scale,bias},
 * up{...}, down{...} inside a record. */
typedef struct {
  int bits, group, hidden, inter, num_experts;
  const uint8_t* base;
  int64_t stride;
  int64_t off[9];
  const uint8_t* const* records;
} or_bank;

typedef struct {
  or_bank routed, shared;
  const uint16_t* w_router;      /* bf16 [E][H] */
  const float* router_bias;      /* fp32 [E] or NULL */
  const uint16_t* w_shared_gate; /* bf16 [H] */
  const float* gamma;            /* fp32 [H]; NULL: no normalisation, x = h */
  double eps;
  int top_k;
} or_layer;

static int g_threads = 1;

void or_set_threads(int n) { g_threads = n > 0 ? n : 1; }

int or_get_threads(void) { return g_threads; }

int or_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

double or_bf16(uint16_t v) {
  uint32_t u = (uint32_t)v << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Code of column c in one row of packed words: word c / (32/bits), field
 * c % (32/bits) counted from the least significant bit. */
unsigned or_code(const uint32_t* row_words, int bits, int c) {
  const int per_word = 32 / bits;
  const uint32_t w = row_words[c / per_word];
  return (w >> (bits * (c % per_word))) & ((1u << bits) - 1u);
}

/* Dequantised weight (r, c): code * scale + bias of the row's group c/group. */
double or_weight(const or_matrix* m, int r, int c) {
  const int wpr = m->cols * m->bits / 32, gpr = m->cols / m->group;
  const unsigned q = or_code(m->qw + (int64_t)r * wpr, m->bits, c);
  const int g = c / m->group;
  return (double)q * or_bf16(m->scale[(int64_t)r * gpr + g]) + or_bf16(m->bias[(int64_t)r * gpr + g]);
}

/* y[r] = sum_c W(r, c) * x[c], one weight at a time. */
void or_matvec(const or_matrix* m, const double* x, double* y) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
  for (int r = 0; r < m->rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < m->cols; ++c) acc += or_weight(m, r, c) * x[c];
    y[r] = acc;
  }
}

/* Two-pass RMSNorm: pass 1 sum of squares, pass 2 x_i = h_i / sqrt(ss/H + eps) * gamma_i.
 * gamma == NULL means unit weights. */
void or_rmsnorm(const float* h, const float* gamma, double eps, int H, double* x) {
  double ss = 0.0;
  for (int i = 0; i < H; ++i) ss += (double)h[i] * (double)h[i];
  const double denom = sqrt(ss / (double)H + eps);
  for (int i = 0; i < H; ++i) x[i] = (double)h[i] / denom * (gamma ? (double)gamma[i] : 1.0);
}

/* Router logits l_e = sum_i Wr[e,i] x_i (+ bias_e). */
void or_router_logits(const uint16_t* wr, const float* bias, const double* x, int E, int H, double* logits) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int i = 0; i < H; ++i) acc += or_bf16(wr[(int64_t)e * H + i]) * x[i];
    logits[e] = acc + (bias ? (double)bias[e] : 0.0);
  }
}

/* p = exp(l - max) / sum exp(l - max). */
void or_softmax(const double* l, int n, double* p) {
  double mx = l[0];
  for (int i = 1; i < n; ++i) mx = l[i] > mx ? l[i] : mx;
  double s = 0.0;
  for (int i = 0; i < n; ++i) {
    p[i] = exp(l[i] - mx);
    s += p[i];
  }
  for (int i = 0; i < n; ++i) p[i] /= s;
}

typedef struct {
  double v;
  int i;
} or_pair;

static int or_pair_cmp(const void* a, const void* b) {
  const or_pair* x = (const or_pair*)a;
  const or_pair* y = (const or_pair*)b;
  if (x->v > y->v) return -1;
  if (x->v < y->v) return 1;
  return (x->i > y->i) - (x->i < y->i);
}

/* The k largest values of p by a full sort: descending value, ties to the lower index. */
void or_topk(const double* p, int n, int k, int* idx) {
  or_pair* a = (or_pair*)malloc(sizeof(or_pair) * (size_t)n);
  for (int i = 0; i < n; ++i) {
    a[i].v = p[i];
    a[i].i = i;
  }
  qsort(a, (size_t)n, sizeof(or_pair), or_pair_cmp);
  for (int j = 0; j < k; ++j) idx[j] = a[j].i;
  free(a);
}

static or_matrix or_bank_matrix(const or_bank* b, int e, int which) {
  or_matrix m;
  const uint8_t* rec = b->records ? b->records[e] : b->base + (int64_t)e * b->stride;
  m.bits = b->bits;
  m.group = b->group;
  m.rows = which == 2 ? b->hidden : b->inter;
  m.cols = which == 2 ? b->inter : b->hidden;
  m.qw = (const uint32_t*)(rec + b->off[3 * which]);
  m.scale = (const uint16_t*)(rec + b->off[3 * which + 1]);
  m.bias = (const uint16_t*)(rec + b->off[3 * which + 2]);
  return m;
}

/* Expert FFN: g = Wg x, u = Wu x, a = silu(g) * u with silu(z) = z / (1 + e^-z), y = Wd a.
 * `a_out` (length inter) may be NULL. */
void or_expert_ffn(const or_bank* b, int e, const double* x, double* y, double* a_out) {
  const int I = b->inter;
  double* g = (double*)malloc(sizeof(double) * (size_t)I);
  double* u = (double*)malloc(sizeof(double) * (size_t)I);
  or_matrix mg = or_bank_matrix(b, e, 0), mu = or_bank_matrix(b, e, 1), md = or_bank_matrix(b, e, 2);
  or_matvec(&mg, x, g);
  or_matvec(&mu, x, u);
  for (int r = 0; r < I; ++r) g[r] = g[r] / (1.0 + exp(-g[r])) * u[r];
  if (a_out) memcpy(a_out, g, sizeof(double) * (size_t)I);
  or_matvec(&md, g, y);
  free(g);
  free(u);
}

/* The whole block for T tokens h[T][H]:
 *   x = RMSNorm(h); l = Wr x (+bias); p = softmax(l); top-K of p;
 *   w_k = p_k / sum_topK p; sigma = sigmoid(wsg . x);
 *   out = h + sum_k w_k FFN_{e_k}(x) + sigma FFN_shared(x).
 * force_idx (nullable, [T][K]) replaces the top-K selection; the weights are
 * then p of the forced experts renormalised.  Optional outputs (nullable):
 * idx_out [T][K], w_out [T][K], probs_out [T][E], logits_out [T][E],
 * sigma_out [T]. */
void or_moe_layer(const or_layer* L, const float* h, int T, const int* force_idx, double* out, int* idx_out,
                  double* w_out, double* probs_out, double* logits_out, double* sigma_out) {
  const int H = L->routed.hidden, E = L->routed.num_experts, K = L->top_k;
  double* x = (double*)malloc(sizeof(double) * (size_t)H);
  double* y = (double*)malloc(sizeof(double) * (size_t)H);
  double* l = (double*)malloc(sizeof(double) * (size_t)E);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  int* idx = (int*)malloc(sizeof(int) * (size_t)K);
  for (int t = 0; t < T; ++t) {
    const float* ht = h + (int64_t)t * H;
    double* ot = out + (int64_t)t * H;
    if (L->gamma)
      or_rmsnorm(ht, L->gamma, L->eps, H, x);
    else
      for (int i = 0; i < H; ++i) x[i] = (double)ht[i];
    or_router_logits(L->w_router, L->router_bias, x, E, H, l);
    or_softmax(l, E, p);
    if (force_idx)
      memcpy(idx, force_idx + (int64_t)t * K, sizeof(int) * (size_t)K);
    else
      or_topk(p, E, K, idx);
    double psum = 0.0;
    for (int k = 0; k < K; ++k) psum += p[idx[k]];
    double zs = 0.0;
    for (int i = 0; i < H; ++i) zs += or_bf16(L->w_shared_gate[i]) * x[i];
    const double sigma = 1.0 / (1.0 + exp(-zs));
    for (int i = 0; i < H; ++i) ot[i] = (double)ht[i];
    for (int k = 0; k < K; ++k) {
      const double wk = p[idx[k]] / psum;
      or_expert_ffn(&L->routed, idx[k], x, y, NULL);
      for (int i = 0; i < H; ++i) ot[i] += wk * y[i];
      if (w_out) w_out[(int64_t)t * K + k] = wk;
      if (idx_out) idx_out[(int64_t)t * K + k] = idx[k];
    }
    or_expert_ffn(&L->shared, 0, x, y, NULL);
    for (int i = 0; i < H; ++i) ot[i] += sigma * y[i];
    if (probs_out) memcpy(probs_out + (int64_t)t * E, p, sizeof(double) * (size_t)E);
    if (logits_out) memcpy(logits_out + (int64_t)t * E, l, sizeof(double) * (size_t)E);
    if (sigma_out) sigma_out[t] = sigma;
  }
  free(x);
  free(y);
  free(l);
  free(p);
  free(idx);
}

/* ------------------------------------------------------------------------------------
 * Gated DeltaNet state update, one decode step.
 *
 * "What is Flash-MoE" (a2a-mcp.org), section 4 (Accelerate BLAS for the Gated DeltaNet
 * layers), and the "Flash-MoE" wiki summary (jeongsk), key technique 4: each of the 45
 * linear-attention layers keeps a 128 x 128 state matrix per head, 64 heads, and updates
 * it with three single-precision BLAS calls: a scaling (sscal), a matrix-vector product
 * (sgemv) and a rank-1 update (sger).  Read as the gated delta rule, per head and in
 * that order:
 *   S <- alpha S                    scaling: the gate decays the whole memory
 *   u  = S k                        matrix-vector: what the memory returns for key k
 *   S <- S + beta (v - u) k^T       rank-1 update: move the answer for k toward v
 *   o  = S q                        matrix-vector: the read-out for query q
 * S: [n][dv][dk] (row i of a head is value coordinate i, column j key coordinate j),
 * updated in place; q, k: [n][dk]; v, o: [n][dv]; alpha, beta: [n].  Each step is its
 * own loop, in the order above; OpenMP runs heads (independent) in parallel.
 * ------------------------------------------------------------------------------------ */
void or_gdn_step(int n, int dk, int dv, double* S, const double* q, const double* k, const double* v,
                 const double* alpha, const double* beta, double* o) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(g_threads)
  for (int h = 0; h < n; ++h) {
    double* Sh = S + (int64_t)h * dv * dk;
    const double* qh = q + (int64_t)h * dk;
    const double* kh = k + (int64_t)h * dk;
    const double* vh = v + (int64_t)h * dv;
    const double a = alpha[h], b = beta[h];
    double* u = (double*)malloc(sizeof(double) * (size_t)dv);
    for (int i = 0; i < dv; ++i)
      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] *= a;
    for (int i = 0; i < dv; ++i) {
      double acc = 0.0;
      for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * kh[j];
      u[i] = acc;
    }
    for (int i = 0; i < dv; ++i)
      for (int j = 0; j < dk; ++j) Sh[(int64_t)i * dk + j] += b * (vh[i] - u[i]) * kh[j];
    for (int i = 0; i < dv; ++i) {
      double acc = 0.0;
      for (int j = 0; j < dk; ++j) acc += Sh[(int64_t)i * dk + j] * qh[j];
      o[(int64_t)h * dv + i] = acc;
    }
    free(u);
  }
}
