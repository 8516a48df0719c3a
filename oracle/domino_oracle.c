/*
 * domino_oracle.c -- fp64 CPU oracle of the Domino head.  TEST INFRASTRUCTURE ONLY.
 *
 * This file is test infrastructure, not the product.  Only the tests, the package's smoke() and
 * bench.py's CPU-baseline leg may load it.  It shares no code, header, table or helper with
 * the CUDA library; the two meet only through the seeded input arrays.
 *
 * What it computes (Domino review page, paper.oopus.info, section 二 "Domino Head", the
 * head equation  L_final = L_base + W2 . sigma(W1 . [H_i ; S_{i-1}])  and the two bullets above
 * it: a GRU causal encoder with hidden size 1024 reads the embeddings of the tokens already
 * drafted and yields the causal state S_{i-1}; a rank-256 low-rank head with a SiLU activation
 * adds its output to the backbone logits over the whole vocabulary; the LM head is not
 * recomputed).
 *
 * Readings taken where the pages are silent (each one also listed in the design notes):
 *   - GRU cell: the PyTorch nn.GRUCell form, gate rows ordered (r, z, n), two bias vectors, the
 *     reset gate multiplying (W_hn h + b_hn).
 *   - Position i uses S_{i-1}; S_{-1} = S0 is supplied by the caller; the state after the last
 *     position is never consumed, so a block of L positions performs L-1 GRU updates.
 *   - "sigma" in the head equation is the SiLU named in the text: silu(a) = a / (1 + exp(-a)).
 *   - W1 and W2 carry no bias (none in the head equation).
 *   - The GRU input is the raw embedding row (dimension d) of the drafted token.
 *   - Greedy drafting (the "greedy decoding" setting of the news.sig.ai article) takes the
 *     argmax of L_final; ties go to the lowest vocabulary index.
 *   - Accept length = number of leading positions j whose draft token equals the argmax
 *     (lowest index on ties) of the target logits at j; no bonus token.
 *   - Sampled (temperature > 0) verification, which the pages call lossless without restating
 *     it, follows the published speculative-sampling rule (see oracle_accept_sample); the random
 *     draws it needs are inputs.
 *
 * Precision: every stored input (fp32, or bf16 bit patterns) is widened exactly to double;
 * all arithmetic is double; exp and tanh come from libm.  No blocking, fusion or reordering
 * beyond the equations: each dot product is a plain ascending loop.
 *
 * Parallelism: OpenMP over independent output elements only (vocabulary rows of W2, GRU
 * units, rank rows of W1).  Each output's own summation order is fixed, so results do not
 * depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1

typedef struct {
  int32_t B, L, d, Hs, r, V, dtype;
} oracle_shape_t;

/* Exact widening of one stored element to double. */
static double elem(const void* p, size_t i, int dtype) {
  if (dtype == ORACLE_F32) return (double)((const float*)p)[i];
  uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
static double silu(double x) { return x / (1.0 + exp(-x)); }

static int nthreads_or_default(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

int oracle_max_threads(void) { return nthreads_or_default(0); }

/*
 * One GRU step, PyTorch nn.GRUCell form (reading above):
 *   r = sigmoid(W_ir x + b_ir + W_hr h + b_hr)
 *   z = sigmoid(W_iz x + b_iz + W_hz h + b_hz)
 *   n = tanh(W_in x + b_in + r * (W_hn h + b_hn))
 *   h' = (1 - z) * n + z * h
 * W_ih is [3Hs, d] and W_hh is [3Hs, Hs], rows grouped (r | z | n).  x is given in double.
 */
static void gru_step(int d, int Hs, int dtype, const void* W_ih, const void* W_hh, const void* b_ih,
                     const void* b_hh, const double* x, const double* h, double* h_out, int nt) {
  int j;
#pragma omp parallel for num_threads(nt) schedule(static)
  for (j = 0; j < Hs; ++j) {
    double gi[3], gh[3];
    for (int g = 0; g < 3; ++g) {
      size_t row = (size_t)g * Hs + j;
      double si = elem(b_ih, row, dtype);
      for (int c = 0; c < d; ++c) si += elem(W_ih, row * d + c, dtype) * x[c];
      double sh = elem(b_hh, row, dtype);
      for (int k = 0; k < Hs; ++k) sh += elem(W_hh, row * Hs + k, dtype) * h[k];
      gi[g] = si;
      gh[g] = sh;
    }
    double r = sigmoid(gi[0] + gh[0]);
    double z = sigmoid(gi[1] + gh[1]);
    double n = tanh(gi[2] + r * gh[2]);
    h_out[j] = (1.0 - z) * n + z * h[j];
  }
}

/* Public single GRU step on double inputs (used by the library-routine pin). */
void oracle_gru_step(int d, int Hs, int dtype, const void* W_ih, const void* W_hh, const void* b_ih,
                     const void* b_hh, const double* x, const double* h, double* h_out) {
  gru_step(d, Hs, dtype, W_ih, W_hh, b_ih, b_hh, x, h, h_out, 1);
}

/*
 * The head over one block, for every batch row.
 *   tokens_in == NULL : greedy drafting, t_i = argmax_v z_i[v] (lowest index on ties)
 *   tokens_in != NULL : teacher forcing, t_i = tokens_in[b, i]
 * Outputs (each may be NULL):
 *   tokens_out [B, L] int32     the token chosen (or given) at each position
 *   logits_out [B, L, V] double L_final at each position
 *   states_out [B, L, Hs] double the state each position consumed: states_out[b,0] = S0[b]
 *   margin_out [B, L] double    top-1 minus top-2 of L_final (0 on a tie)
 * Returns 0, or -1 on a bad shape, -2 on a teacher-forcing token outside [0, V).
 */
int oracle_head(const oracle_shape_t* s, const void* embed, const void* W_ih, const void* W_hh,
                const void* b_ih, const void* b_hh, const void* W1, const void* W2,
                const void* base_logits, const void* hidden, const float* S0,
                const int32_t* tokens_in, int32_t* tokens_out, double* logits_out,
                double* states_out, double* margin_out, int nthreads) {
  const int B = s->B, L = s->L, d = s->d, Hs = s->Hs, r = s->r, V = s->V, dt = s->dtype;
  if (B < 1 || L < 1 || d < 1 || Hs < 1 || r < 1 || V < 1 || (dt != ORACLE_F32 && dt != ORACLE_BF16))
    return -1;
  const int nt = nthreads_or_default(nthreads);
  const int W1cols = d + Hs;
  double* S = (double*)malloc(sizeof(double) * Hs);
  double* Snext = (double*)malloc(sizeof(double) * Hs);
  double* x = (double*)malloc(sizeof(double) * d);
  double* u = (double*)malloc(sizeof(double) * r);
  double* z = (double*)malloc(sizeof(double) * V);
  int rc = 0;
  if (!S || !Snext || !x || !u || !z) { rc = -1; goto done; }

  for (int b = 0; b < B && rc == 0; ++b) {
    for (int j = 0; j < Hs; ++j) S[j] = (double)S0[(size_t)b * Hs + j];  /* S_{-1} = S0 */
    for (int i = 0; i < L; ++i) {
      const size_t pos = (size_t)b * L + i;
      /* a = W1 . [H_i ; S_{i-1}]  (H block first, then S block);  u = silu(a) */
      int k;
#pragma omp parallel for num_threads(nt) schedule(static)
      for (k = 0; k < r; ++k) {
        double a = 0.0;
        for (int c = 0; c < d; ++c) a += elem(W1, (size_t)k * W1cols + c, dt) * elem(hidden, pos * d + c, dt);
        for (int j = 0; j < Hs; ++j) a += elem(W1, (size_t)k * W1cols + d + j, dt) * S[j];
        u[k] = silu(a);
      }
      /* L_final = L_base + W2 . u  over the whole vocabulary */
      int v;
#pragma omp parallel for num_threads(nt) schedule(static)
      for (v = 0; v < V; ++v) {
        double acc = 0.0;
        for (int q = 0; q < r; ++q) acc += elem(W2, (size_t)v * r + q, dt) * u[q];
        z[v] = elem(base_logits, pos * V + v, dt) + acc;
      }
      /* argmax (lowest index on ties) and the top-2 margin */
      int best = 0;
      for (int w = 1; w < V; ++w)
        if (z[w] > z[best]) best = w;
      double second = -INFINITY;
      for (int w = 0; w < V; ++w)
        if (w != best && z[w] > second) second = z[w];
      int t;
      if (tokens_in) {
        t = tokens_in[pos];
        if (t < 0 || t >= V) { rc = -2; break; }
      } else {
        t = best;
      }
      if (tokens_out) tokens_out[pos] = t;
      if (margin_out) margin_out[pos] = (V > 1) ? z[best] - second : 0.0;
      if (logits_out) memcpy(logits_out + pos * (size_t)V, z, sizeof(double) * V);
      if (states_out) memcpy(states_out + pos * (size_t)Hs, S, sizeof(double) * Hs);
      /* S_i = GRU(embed[t_i], S_{i-1}); the state after the last position is never used */
      if (i < L - 1) {
        for (int c = 0; c < d; ++c) x[c] = elem(embed, (size_t)t * d + c, dt);
        gru_step(d, Hs, dt, W_ih, W_hh, b_ih, b_hh, x, S, Snext, nt);
        memcpy(S, Snext, sizeof(double) * Hs);
      }
    }
  }
done:
  free(S); free(Snext); free(x); free(u); free(z);
  return rc;
}

/*
 * Greedy accept length: for each row b, the number of leading positions j (0 <= j < L) with
 * draft_tokens[b, j] equal to the argmax (lowest index on ties) of target_logits[b, j, :].
 * Both sides compare the same fp32 values, so the result is exact.
 */
int oracle_accept_len(int B, int L, int V, const int32_t* draft_tokens, const float* target_logits,
                      int32_t* accept_out) {
  if (B < 1 || L < 1 || V < 1) return -1;
  for (int b = 0; b < B; ++b) {
    int k = 0;
    for (int j = 0; j < L; ++j) {
      const float* row = target_logits + ((size_t)b * L + j) * (size_t)V;
      int best = 0;
      for (int v = 1; v < V; ++v)
        if ((double)row[v] > (double)row[best]) best = v;
      if (draft_tokens[(size_t)b * L + j] != best) break;
      k = j + 1;
    }
    accept_out[b] = k;
  }
  return 0;
}

/*
 * Stochastic (temperature > 0) verification of a draft block: the acceptance rule of speculative
 * sampling (Leviathan, Kalman and Matias, "Fast Inference from Transformers via Speculative
 * Decoding", ICML 2023; Chen et al., "Accelerating Large Language Model Decoding with Speculative
 * Sampling", 2023).  The pages call Domino's verification lossless (review page, section 一: the
 * target model checks the whole block in one parallel pass; researchpapers.dev summary) and spell
 * out only the greedy setting; this is the published rule that makes sampled verification
 * lossless, which they do not restate.
 *
 * Row b, positions j = 0, 1, ... in order:
 *   p_j = softmax(target_logits[b, j, :] / T)
 *   q_j = softmax(draft_logits[b, j, :] / T), or, when draft_logits is NULL (a greedy draft), the
 *         one-hot distribution on the draft token
 *   x = draft_tokens[b, j] is accepted when uniforms[b, j] < p_j(x) / q_j(x); the first rejected
 *   position k ends the row.  Its replacement token is drawn from the residual
 *   res(v) = max(0, p_k(v) - q_k(v)) by inverse transform with u = uniforms[b, L]: the smallest v
 *   (ascending) whose running sum of res exceeds u * Z, Z = sum_v res(v) (the last v with
 *   res(v) > 0 if the running sum never does).
 * accept_out[b] = k (L when every position is accepted); next_out[b] = the replacement token, or
 * -1 when all L were accepted (no bonus token: there are no target logits past the block).
 * ratio_out (optional, [B, L]) receives p_j(x) / q_j(x) for j <= k and -1 after.
 * uniforms is [B, L + 1] in [0, 1).  Returns 0, or -1 on a bad argument.
 */
static void softmax_row(const float* t, int V, double T, double* out) {
  double m = (double)t[0];
  for (int v = 1; v < V; ++v)
    if ((double)t[v] > m) m = (double)t[v];
  double s = 0.0;
  for (int v = 0; v < V; ++v) {
    out[v] = exp(((double)t[v] - m) / T);
    s += out[v];
  }
  for (int v = 0; v < V; ++v) out[v] /= s;
}

/* Residual of position (p, q) for draft token x: res[v] = max(0, p[v] - q[v]) with q one-hot on x
 * when q is NULL.  Returns Z = sum_v res[v] (ascending). */
static double residual(const double* p, const double* q, int x, int V, double* res) {
  double z = 0.0;
  for (int v = 0; v < V; ++v) {
    const double qv = q ? q[v] : (v == x ? 1.0 : 0.0);
    const double r = p[v] - qv;
    res[v] = r > 0.0 ? r : 0.0;
    z += res[v];
  }
  return z;
}

int oracle_accept_sample(int B, int L, int V, const int32_t* draft_tokens, const float* draft_logits,
                         const float* target_logits, float temperature, const float* uniforms, int32_t* accept_out,
                         int32_t* next_out, double* ratio_out) {
  if (B < 1 || L < 1 || V < 1 || !(temperature > 0.0f)) return -1;
  const double T = (double)temperature;
  double* p = (double*)malloc(sizeof(double) * (size_t)V);
  double* q = draft_logits ? (double*)malloc(sizeof(double) * (size_t)V) : NULL;
  double* res = (double*)malloc(sizeof(double) * (size_t)V);
  if (!p || !res || (draft_logits && !q)) {
    free(p); free(q); free(res);
    return -1;
  }
  for (int b = 0; b < B; ++b) {
    int k = L, next = -1;
    for (int j = 0; j < L; ++j) {
      const size_t row = (size_t)b * L + j;
      const int x = draft_tokens[row];
      if (x < 0 || x >= V) { free(p); free(q); free(res); return -1; }
      softmax_row(target_logits + row * (size_t)V, V, T, p);
      if (q) softmax_row(draft_logits + row * (size_t)V, V, T, q);
      const double ratio = p[x] / (q ? q[x] : 1.0);
      if (ratio_out) ratio_out[row] = ratio;
      if ((double)uniforms[(size_t)b * (L + 1) + j] < ratio) continue;
      k = j;
      const double z = residual(p, q, x, V, res);
      const double target = (double)uniforms[(size_t)b * (L + 1) + L] * z;
      double run = 0.0;
      int last = -1;
      for (int v = 0; v < V; ++v) {
        if (res[v] > 0.0) last = v;
        run += res[v];
        if (run > target && res[v] > 0.0) { next = v; break; }
      }
      if (next < 0) next = last;
      break;
    }
    if (ratio_out)
      for (int j = k + 1; j < L; ++j) ratio_out[(size_t)b * L + j] = -1.0;
    accept_out[b] = k;
    next_out[b] = next;
  }
  free(p); free(q); free(res);
  return 0;
}

/* The running sums of the residual used by oracle_accept_sample at one position:
 * cdf[v] = sum_{w <= v} res(w) (ascending), for the target row t, the draft row dq (NULL: one-hot
 * on x) and temperature T.  Returns Z = cdf[V - 1]. */
double oracle_residual_cdf(int V, const float* t, const float* dq, int x, float temperature, double* cdf) {
  const double T = (double)temperature;
  double* p = (double*)malloc(sizeof(double) * (size_t)V);
  double* q = dq ? (double*)malloc(sizeof(double) * (size_t)V) : NULL;
  if (!p || (dq && !q)) { free(p); free(q); return -1.0; }
  softmax_row(t, V, T, p);
  if (q) softmax_row(dq, V, T, q);
  double z = residual(p, q, x, V, cdf);
  double run = 0.0;
  for (int v = 0; v < V; ++v) {
    run += cdf[v];
    cdf[v] = run;
  }
  free(p); free(q);
  return z;
}
