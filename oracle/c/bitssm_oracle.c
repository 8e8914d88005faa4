/*
 * Host oracle of the BitSSM forward pass, plain C (see bitssm_oracle.h).
 * TEST INFRASTRUCTURE ONLY.  Straight loops, float64 arithmetic, float32
 * only where a value decides an integer code.  Built with
 * -ffp-contract=off so that every a * b + c is two rounded operations, as
 * written.  Independent units (token rows, scan channels) are spread over
 * OpenMP threads; each output is computed by one thread in a fixed order.
 */
#include "bitssm_oracle.h"

#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

#define EPS_NORM 1e-5
#define EPS_W 1e-5f
#define Q_ACT 127

/* ------------------------------------------------------------ weights */

int oracle_absmean_ternary(const float* W, int n_out, int k_in, int group, int8_t* Wq, float* s) {
  if (!W || !Wq || !s || n_out <= 0 || k_in <= 0 || group < 0) return -1;
  if (group == 0) {
    double sum = 0.0;
    for (long i = 0; i < (long)n_out * k_in; ++i) sum += fabs((double)W[i]);
    const float sv = (float)(sum / ((double)n_out * k_in));
    const float denom = sv + EPS_W;
    s[0] = sv;
    for (long i = 0; i < (long)n_out * k_in; ++i) {
      float c = rintf(W[i] / denom);
      Wq[i] = (int8_t)(c > 1.f ? 1 : (c < -1.f ? -1 : (int)c));
    }
    return 0;
  }
  const int ng = (k_in + group - 1) / group;
  for (int n = 0; n < n_out; ++n) {
    for (int j = 0; j < ng; ++j) {
      const int k0 = j * group, k1 = (j + 1) * group < k_in ? (j + 1) * group : k_in;
      double sum = 0.0;
      for (int k = k0; k < k1; ++k) sum += fabs((double)W[(long)n * k_in + k]);
      const float sv = (float)(sum / (double)(k1 - k0));
      const float denom = sv + EPS_W;
      s[(long)n * ng + j] = sv;
      for (int k = k0; k < k1; ++k) {
        float c = rintf(W[(long)n * k_in + k] / denom);
        Wq[(long)n * k_in + k] = (int8_t)(c > 1.f ? 1 : (c < -1.f ? -1 : (int)c));
      }
    }
  }
  return 0;
}

int oracle_pack_ternary(const int8_t* Wq, int n_out, int k_in, uint8_t* packed) {
  if (!Wq || !packed || n_out <= 0 || k_in <= 0) return -1;
  const int kb = (k_in + 3) / 4;
  for (int n = 0; n < n_out; ++n)
    for (int b = 0; b < kb; ++b) {
      unsigned byte = 0;
      for (int i = 0; i < 4; ++i) {
        const int k = 4 * b + i;
        const unsigned code = k < k_in ? (unsigned)(Wq[(long)n * k_in + k] + 1) : 1u;
        byte |= code << (2 * i);
      }
      packed[(long)n * kb + b] = (uint8_t)byte;
    }
  return 0;
}

/* ------------------------------------------------------------ activations */

/* codes of one float32 row; returns m = max|v| */
static float codes_row(const float* v, int K, int32_t* q) {
  float m = 0.f;
  for (int k = 0; k < K; ++k) {
    const float a = fabsf(v[k]);
    if (a > m) m = a;
  }
  if (m == 0.f) {
    for (int k = 0; k < K; ++k) q[k] = 0;
    return m;
  }
  const float sigma = (float)Q_ACT / m;
  for (int k = 0; k < K; ++k) {
    const float prod = v[k] * sigma;
    float c = rintf(prod);
    if (c > 127.f) c = 127.f;
    if (c < -128.f) c = -128.f;
    q[k] = (int32_t)c;
  }
  return m;
}

int oracle_absmax_codes(const float* v, long rows, int K, int32_t* q, float* m) {
  if (!v || !q || !m || rows < 0 || K <= 0) return -1;
#pragma omp parallel for schedule(static)
  for (long r = 0; r < rows; ++r) m[r] = codes_row(v + r * K, K, q + r * K);
  return 0;
}

/* 1 / sqrt(mean v^2 + eps) of a float64 row */
static double rms_factor(const double* v, int K) {
  double ss = 0.0;
  for (int k = 0; k < K; ++k) ss += v[k] * v[k];
  return 1.0 / sqrt(ss / K + EPS_NORM);
}

/* acc = q . Wq[j] over K, exact in int64 */
static int64_t int_dot(const int32_t* q, const int8_t* w, int K) {
  int64_t acc = 0;
  for (int k = 0; k < K; ++k) acc += (int64_t)q[k] * (int64_t)w[k];
  return acc;
}

/* A8 BitLinear of one row given as float32 values */
static void bl_a8_row(const float* x, int K, const int8_t* Wq, float s, int n_out, int32_t* q,
                      double* xd, double* y) {
  const float m = codes_row(x, K, q);
  for (int k = 0; k < K; ++k) xd[k] = (double)x[k];
  const double deq = (double)m * rms_factor(xd, K) / Q_ACT;
  for (int j = 0; j < n_out; ++j)
    y[j] = (double)int_dot(q, Wq + (long)j * K, K) * (double)s * deq;
}

/* A16 BitLinear of one float64 row, scales per group (group 0: s[0]) */
static void bl_a16_row(const double* v, int K, const int8_t* Wq, const float* s, int n_out,
                       int group, double* y) {
  const double r = rms_factor(v, K);
  const int g = group > 0 ? group : K;
  const int ng = (K + g - 1) / g;
  for (int n = 0; n < n_out; ++n) {
    double total = 0.0;
    for (int j = 0; j < ng; ++j) {
      const int k0 = j * g, k1 = (j + 1) * g < K ? (j + 1) * g : K;
      double part = 0.0;
      for (int k = k0; k < k1; ++k) part += v[k] * (double)Wq[(long)n * K + k];
      total += part * (double)(group > 0 ? s[(long)n * ng + j] : s[0]);
    }
    y[n] = total * r;
  }
}

int oracle_bitlinear_forward(const float* x, int M, int K, const int8_t* Wq, const float* s,
                             int n_out, int group, int act_mode, double* y) {
  if (!x || !Wq || !s || !y || M < 0 || K <= 0 || n_out <= 0) return -1;
  if (act_mode != 0 && act_mode != 1) return -1;
  if (act_mode == 0 && group != 0) return -1;
  int bad = 0;
#pragma omp parallel
  {
    int32_t* q = (int32_t*)malloc(sizeof(int32_t) * K);
    double* xd = (double*)malloc(sizeof(double) * K);
    if (!q || !xd) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(static)
      for (int m = 0; m < M; ++m) {
        if (act_mode == 0) {
          bl_a8_row(x + (long)m * K, K, Wq, s[0], n_out, q, xd, y + (long)m * n_out);
        } else {
          for (int k = 0; k < K; ++k) xd[k] = (double)x[(long)m * K + k];
          bl_a16_row(xd, K, Wq, s, n_out, group, y + (long)m * n_out);
        }
      }
    }
    free(q);
    free(xd);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------ scan */

static double softplus(double z) { return (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z))); }

int oracle_selective_scan_forward(const double* u, const double* delta, const double* A,
                                  const double* Bm, const double* Cm, const double* D,
                                  const double* h0, double* y, double* h_last, int B, int L,
                                  int E, int N) {
  if (B < 0 || L < 0 || E <= 0 || N <= 0 || !A || !D) return -1;
  if (L > 0 && (!u || !delta || !Bm || !Cm || !y)) return -1;
  int bad = 0;
#pragma omp parallel
  {
    double* h = (double*)malloc(sizeof(double) * N);
    if (!h) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for collapse(2) schedule(static)
      for (int b = 0; b < B; ++b)
        for (int e = 0; e < E; ++e) {
          for (int n = 0; n < N; ++n) h[n] = h0 ? h0[((long)b * E + e) * N + n] : 0.0;
          for (int t = 0; t < L; ++t) {
            const long te = ((long)b * L + t) * E + e;
            const long tn = ((long)b * L + t) * N;
            const double dt = delta[te];
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
              const double a = exp(dt * A[(long)e * N + n]);
              const double bb = dt * Bm[tn + n] * u[te];
              h[n] = a * h[n] + bb;
              acc += h[n] * Cm[tn + n];
            }
            y[te] = acc + D[e] * u[te];
          }
          if (h_last)
            for (int n = 0; n < N; ++n) h_last[((long)b * E + e) * N + n] = h[n];
        }
    }
    free(h);
  }
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------ the mixer */

/* Codes of an integer row (as float32, exact below 2^24) and the
 * dequantisation factor of the real row c * acc. */
static double int_row_codes(const int64_t* acc, int K, double c, int32_t* q, float* tmp,
                            double* tmpd) {
  for (int k = 0; k < K; ++k) tmp[k] = (float)acc[k];
  const float m_int = codes_row(tmp, K, q);
  for (int k = 0; k < K; ++k) tmpd[k] = c * (double)acc[k];
  const double m = c * (double)m_int;
  return m * rms_factor(tmpd, K) / Q_ACT;
}

static double silu(double v) {
  const double e = exp(-fabs(v));
  return v >= 0.0 ? v / (1.0 + e) : v * e / (1.0 + e);
}

int oracle_bitssm_forward(const oracle_layer* p, const float* x, double* out, int B, int L,
                          int act_mode, const double* h0, double* h_last) {
  if (!p || !x || !out || B < 0 || L < 0 || (act_mode != 0 && act_mode != 1)) return -1;
  const int d = p->d_model, E = p->d_inner, N = p->d_state, R = p->dt_rank;
  if (d <= 0 || E <= 0 || N <= 0 || R <= 0) return -1;
  if (act_mode == 0 && p->group != 0) return -1;
  const int block = p->d_conv != 0;
  if (block && (act_mode != 0 || p->d_conv < 1 || !p->Wq_z || !p->s_z || !p->conv_w || h0))
    return -1;
  const long T = (long)B * L;
  const int Kmax = (d > E ? d : E);
  double* u = (double*)calloc((size_t)T * E, sizeof(double));
  double* delta = (double*)calloc((size_t)T * E, sizeof(double));
  double* Bm = (double*)calloc((size_t)T * N, sizeof(double));
  double* Cm = (double*)calloc((size_t)T * N, sizeof(double));
  double* y = (double*)calloc((size_t)T * E, sizeof(double));
  int64_t* acc_in = (int64_t*)calloc((size_t)T * E, sizeof(int64_t));
  double* deq_x = (double*)calloc((size_t)T, sizeof(double));
  double* z = block ? (double*)calloc((size_t)T * E, sizeof(double)) : NULL;
  double* u_pre = block ? (double*)calloc((size_t)T * E, sizeof(double)) : NULL;
  double* A = (double*)malloc(sizeof(double) * E * N);
  double* D = (double*)malloc(sizeof(double) * E);
  int bad = !u || !delta || !Bm || !Cm || !y || !acc_in || !deq_x || !A || !D ||
            (block && (!z || !u_pre));
  if (!bad) {
    for (long i = 0; i < (long)E * N; ++i) A[i] = (double)p->A[i];
    for (int e = 0; e < E; ++e) D[e] = (double)p->D[e];
  }
  /* phase 1, per token: in_proj (and the gate branch z) */
  if (!bad) {
#pragma omp parallel
    {
      int32_t* q = (int32_t*)malloc(sizeof(int32_t) * Kmax);
      double* td = (double*)malloc(sizeof(double) * Kmax);
      if (!q || !td) {
#pragma omp atomic write
        bad = 1;
      } else {
#pragma omp for schedule(static)
        for (long t = 0; t < T; ++t) {
          const float* xt = x + t * d;
          for (int k = 0; k < d; ++k) td[k] = (double)xt[k];
          if (act_mode == 0) {
            const float m = codes_row(xt, d, q);
            deq_x[t] = (double)m * rms_factor(td, d) / Q_ACT;
            double* dst = block ? u_pre : u;
            for (int e = 0; e < E; ++e) {
              acc_in[t * E + e] = int_dot(q, p->Wq_in + (long)e * d, d);
              dst[t * E + e] = (double)acc_in[t * E + e] * (double)p->s_in[0] * deq_x[t];
              if (block)
                z[t * E + e] = (double)int_dot(q, p->Wq_z + (long)e * d, d) * (double)p->s_z[0] *
                               deq_x[t];
            }
          } else {
            bl_a16_row(td, d, p->Wq_in, p->s_in, E, p->group, u + t * E);
          }
        }
      }
      free(q);
      free(td);
    }
  }
  /* phase 2, block form: u = SiLU(causal depthwise conv of u_pre) */
  if (!bad && block) {
    const int K = p->d_conv;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
      for (int e = 0; e < E; ++e)
        for (int t = 0; t < L; ++t) {
          double acc = p->conv_b ? (double)p->conv_b[e] : 0.0;
          for (int k = 0; k < K; ++k) {
            const int src = t - (K - 1) + k;  /* tap K-1 is the current step */
            if (src >= 0) acc += (double)p->conv_w[(long)e * K + k] * u_pre[((long)b * L + src) * E + e];
          }
          u[((long)b * L + t) * E + e] = silu(acc);
        }
  }
  /* phase 3, per token: x_proj (Delta-down | B | C), Delta-up, softplus */
  if (!bad) {
#pragma omp parallel
    {
      int32_t* q = (int32_t*)malloc(sizeof(int32_t) * Kmax);
      float* tf = (float*)malloc(sizeof(float) * Kmax);
      double* td = (double*)malloc(sizeof(double) * Kmax);
      int64_t* acc_x = (int64_t*)malloc(sizeof(int64_t) * (R + 2 * N));
      double* dt_low = (double*)malloc(sizeof(double) * R);
      double* draw = (double*)malloc(sizeof(double) * E);
      if (!q || !tf || !td || !acc_x || !dt_low || !draw) {
#pragma omp atomic write
        bad = 1;
      } else {
#pragma omp for schedule(static)
        for (long t = 0; t < T; ++t) {
          if (act_mode == 0) {
            double deq_u;
            if (block) {
              /* codes of the float32 value of u */
              for (int e = 0; e < E; ++e) tf[e] = (float)u[t * E + e];
              const float m = codes_row(tf, E, q);
              deq_u = (double)m * rms_factor(u + t * E, E) / Q_ACT;
            } else {
              /* codes of the integer row acc_in */
              const double c_u = (double)p->s_in[0] * deq_x[t];
              deq_u = int_row_codes(acc_in + t * E, E, c_u, q, tf, td);
            }
            for (int j = 0; j < R; ++j) acc_x[j] = int_dot(q, p->Wq_dt_down + (long)j * E, E);
            for (int n = 0; n < N; ++n) {
              acc_x[R + n] = int_dot(q, p->Wq_b + (long)n * E, E);
              acc_x[R + N + n] = int_dot(q, p->Wq_c + (long)n * E, E);
              Bm[t * N + n] = (double)acc_x[R + n] * (double)p->s_b[0] * deq_u;
              Cm[t * N + n] = (double)acc_x[R + N + n] * (double)p->s_c[0] * deq_u;
            }
            /* Delta-up on the codes of the integer row acc_x[:R] */
            const double c_dt = (double)p->s_dt_down[0] * deq_u;
            const double deq_dt = int_row_codes(acc_x, R, c_dt, q, tf, td);
            for (int e = 0; e < E; ++e) {
              const double dr = (double)int_dot(q, p->Wq_dt_up + (long)e * R, R) *
                                (double)p->s_dt_up[0] * deq_dt;
              delta[t * E + e] = softplus(dr + (double)p->dt_bias[e]);
            }
          } else {
            bl_a16_row(u + t * E, E, p->Wq_dt_down, p->s_dt_down, R, p->group, dt_low);
            bl_a16_row(u + t * E, E, p->Wq_b, p->s_b, N, p->group, Bm + t * N);
            bl_a16_row(u + t * E, E, p->Wq_c, p->s_c, N, p->group, Cm + t * N);
            bl_a16_row(dt_low, R, p->Wq_dt_up, p->s_dt_up, E, p->group, draw);
            for (int e = 0; e < E; ++e)
              delta[t * E + e] = softplus(draw[e] + (double)p->dt_bias[e]);
          }
        }
      }
      free(q); free(tf); free(td); free(acc_x); free(dt_low); free(draw);
    }
  }
  /* phase 4: the scan */
  if (!bad)
    bad = oracle_selective_scan_forward(u, delta, A, Bm, Cm, D, h0, y, h_last, B, L, E, N) != 0;
  /* phase 5, per token: (gate and) out_proj */
  if (!bad) {
#pragma omp parallel
    {
      int32_t* q = (int32_t*)malloc(sizeof(int32_t) * E);
      float* tf = (float*)malloc(sizeof(float) * E);
      double* yg = (double*)malloc(sizeof(double) * E);
      if (!q || !tf || !yg) {
#pragma omp atomic write
        bad = 1;
      } else {
#pragma omp for schedule(static)
        for (long t = 0; t < T; ++t) {
          const double* yt = y + t * E;
          if (block) {
            for (int e = 0; e < E; ++e) yg[e] = yt[e] * silu(z[t * E + e]);
            yt = yg;
          }
          if (act_mode == 0) {
            /* out_proj on the codes of the float32 value of y (or y_g) */
            for (int e = 0; e < E; ++e) tf[e] = (float)yt[e];
            const float m = codes_row(tf, E, q);
            const double deq_y = (double)m * rms_factor(yt, E) / Q_ACT;
            for (int j = 0; j < d; ++j)
              out[t * d + j] = (double)int_dot(q, p->Wq_out + (long)j * E, E) *
                               (double)p->s_out[0] * deq_y;
          } else {
            bl_a16_row(yt, E, p->Wq_out, p->s_out, d, p->group, out + t * d);
          }
        }
      }
      free(q); free(tf); free(yg);
    }
  }
  free(u); free(delta); free(Bm); free(Cm); free(y); free(acc_in); free(deq_x); free(z);
  free(u_pre); free(A); free(D);
  return bad ? -1 : 0;
}

/* ------------------------------------------------------------ SSD scan */

int oracle_ssd_scan_forward(const double* x, const double* dt, const double* A, const double* Bm,
                            const double* Cm, const double* D, const double* S0, double* y,
                            double* S_last, int B, int L, int H, int P, int G, int N) {
  if (B < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || H % G != 0 || !A) return -1;
  if (L > 0 && (!x || !dt || !Bm || !Cm || !y)) return -1;
  const int per = H / G;
  int bad = 0;
#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * N);
    if (!S) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for collapse(3) schedule(static)
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
          for (int pp = 0; pp < P; ++pp) {
            const int g = h / per;
            const long srow = (((long)b * H + h) * P + pp) * N;
            for (int n = 0; n < N; ++n) S[n] = S0 ? S0[srow + n] : 0.0;
            for (int t = 0; t < L; ++t) {
              const double dtv = dt[((long)b * L + t) * H + h];
              const double a = exp(dtv * A[h]);
              const double xv = x[(((long)b * L + t) * H + h) * P + pp];
              const long bc = (((long)b * L + t) * G + g) * N;
              double acc = 0.0;
              for (int n = 0; n < N; ++n) {
                S[n] = a * S[n] + dtv * xv * Bm[bc + n];
                acc += S[n] * Cm[bc + n];
              }
              y[(((long)b * L + t) * H + h) * P + pp] = acc + (D ? D[h] : 0.0) * xv;
            }
            if (S_last)
              for (int n = 0; n < N; ++n) S_last[srow + n] = S[n];
          }
    }
    free(S);
  }
  return bad ? -1 : 0;
}

int oracle_set_threads(int n) {
  const int prev = omp_get_max_threads();
  if (n >= 1) omp_set_num_threads(n);
  return prev;
}
