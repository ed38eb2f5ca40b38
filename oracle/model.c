/*
 * CPU oracle for looped-Transformer decoding: plain fp64 arithmetic of one
 * token row of one Transformer layer, and of the readout logits.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and
 * bench.py's CPU-baseline leg may load this library.  It shares no code with
 * the CUDA library.
 *
 * What it follows ("LoopSpec: Pipelined Self-Speculative Decoding for Looped
 * Transformers", liuzhao09.github.io/papers/loopspec.html):
 *   - section 2.1, Eq. 1: H^(0) = P(X), H^(r) = B(H^(r-1)), p_r = C(H^(r));
 *     the shared block B is applied R times with the same weights;
 *   - section 2.1 / Fig. 2: the state of a prefix differs per loop depth and
 *     the KV caches of different depths are never mixed -- the caller hands
 *     each call the cache plane of one (layer, depth);
 *   - section 2.4: a branch reuses its parent's prefix cache through a list
 *     of cache indices ("slots"), which is the `slots` argument here.
 * The pages do not spell out the layer; the reading used is a Llama-style
 * pre-norm layer: RMSNorm -> QKV -> RoPE (rotate-half, absolute position) ->
 * causal softmax attention -> O projection added to the residual with scale s,
 * RMSNorm -> SwiGLU MLP added with scale s.  No biases, no GQA.
 *
 * Weights are fp32 arrays (bf16 models pass their bf16-rounded values); all
 * activations and accumulations are double.  Loops run in the plain textbook
 * order; OpenMP only splits independent output rows.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* y[n_out] = W[n_out x n_in] . x[n_in] */
void orc_matvec(int n_out, int n_in, const float* W, const double* x, double* y) {
#pragma omp parallel for schedule(static)
  for (int i = 0; i < n_out; ++i) {
    const float* w = W + (size_t)i * n_in;
    double acc = 0.0;
    for (int k = 0; k < n_in; ++k) acc += (double)w[k] * x[k];
    y[i] = acc;
  }
}

/* out = h / sqrt(mean(h^2) + eps) * g */
void orc_rmsnorm(int d, const double* h, const float* g, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < d; ++i) ss += h[i] * h[i];
  double inv = 1.0 / sqrt(ss / d + eps);
  for (int i = 0; i < d; ++i) out[i] = h[i] * inv * (double)g[i];
}

/* Rotary embedding, rotate-half pairing (i, i + hd/2), angle pos * theta^(-2i/hd). */
void orc_rope(int n_heads, int hd, int pos, double theta, double* v) {
  int half = hd / 2;
  for (int h = 0; h < n_heads; ++h) {
    double* x = v + (size_t)h * hd;
    for (int i = 0; i < half; ++i) {
      double inv_freq = pow(theta, -2.0 * i / hd);
      double ang = pos * inv_freq;
      double c = cos(ang), s = sin(ang);
      double x1 = x[i], x2 = x[i + half];
      x[i] = x1 * c - x2 * s;
      x[i + half] = x2 * c + x1 * s;
    }
  }
}

/* Softmax attention of one query row over n_pos cached rows K[slots[j]],
 * V[slots[j]] (planes of width d), scale 1/sqrt(hd), per head. */
void orc_attend(int n_heads, int hd, int d, int n_pos, const double* q, const double* K,
                const double* V, const int* slots, double* out) {
  double* sc = (double*)malloc(sizeof(double) * (n_pos > 0 ? n_pos : 1));
  double scale = 1.0 / sqrt((double)hd);
  for (int h = 0; h < n_heads; ++h) {
    double m = -INFINITY;
    for (int j = 0; j < n_pos; ++j) {
      const double* k = K + (size_t)slots[j] * d + (size_t)h * hd;
      double dot = 0.0;
      for (int e = 0; e < hd; ++e) dot += q[h * hd + e] * k[e];
      sc[j] = dot * scale;
      if (sc[j] > m) m = sc[j];
    }
    double den = 0.0;
    for (int j = 0; j < n_pos; ++j) {
      sc[j] = exp(sc[j] - m);
      den += sc[j];
    }
    for (int e = 0; e < hd; ++e) out[h * hd + e] = 0.0;
    for (int j = 0; j < n_pos; ++j) {
      const double* v = V + (size_t)slots[j] * d + (size_t)h * hd;
      double w = sc[j] / den;
      for (int e = 0; e < hd; ++e) out[h * hd + e] += w * v[e];
    }
  }
  free(sc);
}

/*
 * One layer applied to the hidden row h (in place) of the token at position
 * `pos`.  Its key/value rows are written to K/V[own_slot] (planes [n_slots][d])
 * and attention reads slots[0..pos] (the prefix's rows, own row last).
 */
void orc_layer(int d, int n_heads, int hd, int f, double eps, double theta, double s,
               const float* g1, const float* wqkv, const float* wo, const float* g2,
               const float* wgu, const float* wd, double* h, int pos, double* K, double* V,
               const int* slots, int own_slot) {
  double* a = (double*)malloc(sizeof(double) * d);
  double* qkv = (double*)malloc(sizeof(double) * 3 * d);
  double* o = (double*)malloc(sizeof(double) * d);
  double* y = (double*)malloc(sizeof(double) * d);
  double* gu = (double*)malloc(sizeof(double) * 2 * f);
  double* act = (double*)malloc(sizeof(double) * f);

  orc_rmsnorm(d, h, g1, eps, a);
  orc_matvec(3 * d, d, wqkv, a, qkv);
  double* q = qkv;
  double* k = qkv + d;
  double* v = qkv + 2 * d;
  orc_rope(n_heads, hd, pos, theta, q);
  orc_rope(n_heads, hd, pos, theta, k);
  memcpy(K + (size_t)own_slot * d, k, sizeof(double) * d);
  memcpy(V + (size_t)own_slot * d, v, sizeof(double) * d);
  orc_attend(n_heads, hd, d, pos + 1, q, K, V, slots, o);
  orc_matvec(d, d, wo, o, y);
  for (int i = 0; i < d; ++i) h[i] += s * y[i];

  orc_rmsnorm(d, h, g2, eps, a);
  orc_matvec(2 * f, d, wgu, a, gu);
  for (int i = 0; i < f; ++i) {
    double g = gu[i];
    act[i] = g / (1.0 + exp(-g)) * gu[f + i];
  }
  orc_matvec(d, f, wd, act, y);
  for (int i = 0; i < d; ++i) h[i] += s * y[i];

  free(a); free(qkv); free(o); free(y); free(gu); free(act);
}

/* Readout logits z = W_head . (RMSNorm(h) * g_final). */
void orc_logits(int d, int vocab, const double* h, const float* g_final, double eps,
                const float* head, double* z) {
  double* a = (double*)malloc(sizeof(double) * d);
  orc_rmsnorm(d, h, g_final, eps, a);
  orc_matvec(vocab, d, head, a, z);
  free(a);
}
