/*
 * bitssm_oracle.h - host oracle of the BitSSM forward pass, plain C.
 *
 * TEST INFRASTRUCTURE ONLY: called by tests/, __graft_entry__ and the CPU
 * baseline of bench.py, never by the product path.  It shares no code or
 * header with the CUDA library; its entry points carry the library's names
 * with an `oracle_` prefix and take HOST pointers.
 *
 * Arithmetic: float64, except where a floating-point value decides an
 * integer (an int8 activation code, a ternary weight code): those decisions
 * are taken in IEEE float32 with round-to-nearest-even, as the definitions
 * state.  Sources (page title and part): "Associative Recall Under Ternary
 * Quantization" (TriSSM README: opening paragraph, the caption "The BitSSM
 * sequence mixer", the Overview table); "Ternary Mamba" (abstract:
 * W1.58A16 with grouped scales).  Readings of open points are the ones the
 * numpy oracle (oracle/bitssm_oracle.py) states, and the two are held to
 * each other by tests/test_oracle_c.py.
 *
 * Every function returns 0, or -1 for an invalid argument.
 */
#ifndef BITSSM_ORACLE_H
#define BITSSM_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Absmean ternarisation of W [n_out, k_in] (float32): s = mean|W| (summed in
 * float64, stored float32), Wq = clip(rint(fl32(W / fl32(s + 1e-5))), -1, 1).
 * group 0: one scale (s[0]); group g > 0: s [n_out, ceil(k_in/g)], one per
 * run of g consecutive K-elements of a row. */
int oracle_absmean_ternary(const float* W, int n_out, int k_in, int group, int8_t* Wq, float* s);

/* 2-bit encoding: code w + 1 at bits 2*(k mod 4) of byte k/4 of its row,
 * padding code 1.  packed [n_out, ceil(k_in/4)]. */
int oracle_pack_ternary(const int8_t* Wq, int n_out, int k_in, uint8_t* packed);

/* Per-row absmax int8 codes of float32 rows v [rows, K]: m = max|v|,
 * sigma = fl32(127/m), q = clamp(rint(fl32(v * sigma)), -128, 127); a zero
 * row gets zero codes.  q int32 [rows, K], m float [rows]. */
int oracle_absmax_codes(const float* v, long rows, int K, int32_t* q, float* m);

/* One BitLinear on rows x [M, K] (float32 values), ternary Wq [n_out, K]
 * with scales s (group 0: s[0]; group 128: s [n_out, ceil(K/128)]).
 * act_mode 0 (A8): unit-gain RMSNorm folded into the absmax codes,
 *   y = acc * s * m * r / 127, r = 1 / sqrt(mean x^2 + 1e-5);
 * act_mode 1 (A16): no codes, y_n = r * sum_g s[n, g] sum_{k in g} Wq[n, k] x_k.
 * y double [M, n_out]. */
int oracle_bitlinear_forward(const float* x, int M, int K, const int8_t* Wq, const float* s,
                             int n_out, int group, int act_mode, double* y);

/* Sequential selective scan in float64: u, delta [B, L, E]; A [E, N];
 * Bm, Cm [B, L, N]; D [E]; h0 [B, E, N] or NULL (zero); y [B, L, E];
 * h_last [B, E, N] or NULL.
 *   h_t = exp(delta_t[e] A[e, n]) h_{t-1} + delta_t[e] B_t[n] u_t[e]
 *   y_t[e] = sum_n C_t[n] h_t[e, n] + D[e] u_t[e] */
int oracle_selective_scan_forward(const double* u, const double* delta, const double* A,
                                  const double* Bm, const double* Cm, const double* D,
                                  const double* h0, double* y, double* h_last, int B, int L,
                                  int E, int N);

/* Ternary weights of one mixer (codes and scales as oracle_absmean_ternary
 * returns them, all with the same group), shapes:
 *   in [E, d], dt_down [R, E], b [N, E], c [N, E], dt_up [E, R], out [d, E];
 * A [E, N] (negative), D [E], dt_bias [E] (float32). */
typedef struct oracle_layer {
  const int8_t *Wq_in, *Wq_dt_down, *Wq_b, *Wq_c, *Wq_dt_up, *Wq_out;
  const float *s_in, *s_dt_down, *s_b, *s_c, *s_dt_up, *s_out;
  const float *A, *D, *dt_bias;
  int d_model, d_inner, d_state, dt_rank, group;
  /* Mamba-1 block form (d_conv != 0, A8, zero start state only): the gate
   * branch z_proj [E, d] and the depthwise causal conv taps [E, d_conv]
   * (tap d_conv-1 on the current step) and bias [E] (may be NULL). */
  const int8_t* Wq_z;
  const float* s_z;
  const float *conv_w, *conv_b;
  int d_conv;
} oracle_layer;

/* The mixer on x [B, L, d_model] (float32 values) -> out double [B, L, d].
 * A8: the codes fed to x_proj and to Delta-up are decided on the integer
 * accumulator rows of the projection before; out_proj quantises the float32
 * value of y.  A16: every projection is the A16 BitLinear of its input row.
 * h0 / h_last as in oracle_selective_scan_forward (nullable). */
int oracle_bitssm_forward(const oracle_layer* p, const float* x, double* out, int B, int L,
                          int act_mode, const double* h0, double* h_last);

/* SSD scan of Mamba-2 in float64, step by step: x, y [B, L, H, P];
 * dt [B, L, H] (after the softplus); A [H]; Bm, Cm [B, L, G, N]; D [H] or
 * NULL; S0, S_last [B, H, P, N] or NULL; head h reads group h / (H / G).
 *   S_t = exp(dt_t[h] A[h]) S_{t-1} + dt_t[h] x_t[h] (outer) B_t[g]
 *   y_t[h] = S_t C_t[g] + D[h] x_t[h] */
int oracle_ssd_scan_forward(const double* x, const double* dt, const double* A, const double* Bm,
                            const double* Cm, const double* D, const double* S0, double* y,
                            double* S_last, int B, int L, int H, int P, int G, int N);

/* Threads the oracle's parallel loops use from now on (n >= 1), for timing
 * it on one core; returns the previous count. */
int oracle_set_threads(int n);

#ifdef __cplusplus
}
#endif

#endif /* BITSSM_ORACLE_H */
