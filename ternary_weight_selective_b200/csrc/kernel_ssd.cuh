// The SSD scan of Mamba-2: the selective recurrence with one decay per head
// ("Ternary Mamba" abstract: the W1.58A16 model is Mamba-2 1.3B; "SSDi8"
// abstract: SSD, the state space duality of Mamba-2).  Per sequence b, head h
// (head dimension P) and B/C group g = h / (H / G):
//   S_t = exp(dt_t[h] A[h]) S_{t-1} + dt_t[h] x_t[h] (outer) B_t[g]   (S: [P, N])
//   y_t[h] = S_t C_t[g] + D[h] x_t[h]
//
// First form: the recurrence on the ordinary FMA pipes.  One CTA per (head,
// sequence); thread (p, j) owns kSsdNS consecutive states of row p of S, so
// a row is spread over N / kSsdNS lanes of one warp and y_t[h][p] is a
// shuffle sum over them.  The decay is one exp2 per step and thread.  Time
// runs in chunks of kSsdChunk steps whose x, dt, B and C are staged in
// shared memory by the whole CTA (coalesced loads), then consumed step by
// step from there.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace bitssm {

constexpr int kSsdNS = 16;     // states per thread
constexpr float kLog2eSsd = 1.4426950408889634f;
constexpr int kSsdChunk = 16;  // time steps staged per chunk

struct SsdParams {
  const float* x;      // [B, L, H, P]
  const float* dt;     // [B, L, H], after the softplus
  const float* A;      // [H], < 0
  const float* Bm;     // [B, L, G, N]
  const float* Cm;     // [B, L, G, N]
  const float* D;      // [H] or null (zero)
  const float* S0;     // [B, H, P, N] or null (zero)
  float* y;            // [B, L, H, P]
  float* S_last;       // [B, H, P, N] or null
  int B, L, H, P, G, N;
};

// Shared memory of one CTA: x [chunk][P], dt [chunk], B and C [chunk][N].
inline size_t ssd_smem_bytes(int P, int N) {
  return sizeof(float) * ((size_t)kSsdChunk * P + kSsdChunk + 2 * (size_t)kSsdChunk * N);
}

__global__ void __launch_bounds__(1024) ssd_scan_kernel(SsdParams Q) {
  extern __shared__ float ssd_sm[];
  const int h = blockIdx.x;
  const int b = blockIdx.y;
  const int P = Q.P, N = Q.N, H = Q.H, L = Q.L;
  const int tpp = N / kSsdNS;  // lanes per row of S (a power of two <= 32)
  const int p = threadIdx.x / tpp;
  const int j0 = (threadIdx.x % tpp) * kSsdNS;
  const int g = h / (H / Q.G);
  float* sx = ssd_sm;                 // [chunk][P]
  float* sdt = sx + kSsdChunk * P;    // [chunk]
  float* sB = sdt + kSsdChunk;        // [chunk][N]
  float* sC = sB + kSsdChunk * N;     // [chunk][N]

  float s[kSsdNS];
  const long srow = (((long)b * H + h) * P + p) * N + j0;
#pragma unroll
  for (int j = 0; j < kSsdNS; ++j) s[j] = Q.S0 != nullptr ? Q.S0[srow + j] : 0.f;
  const float a_l2 = Q.A[h] * kLog2eSsd;
  const float d_h = Q.D != nullptr ? Q.D[h] : 0.f;

  for (int t0 = 0; t0 < L; t0 += kSsdChunk) {
    const int nt = min(kSsdChunk, L - t0);
    __syncthreads();  // the previous chunk has been consumed
    for (int i = threadIdx.x; i < nt * P; i += blockDim.x) {
      const int tt = i / P, pp = i - tt * P;
      sx[i] = __ldg(Q.x + (((long)b * L + t0 + tt) * H + h) * P + pp);
    }
    for (int i = threadIdx.x; i < nt; i += blockDim.x)
      sdt[i] = __ldg(Q.dt + ((long)b * L + t0 + i) * H + h);
    for (int i = threadIdx.x; i < nt * N; i += blockDim.x) {
      const int tt = i / N, n = i - tt * N;
      const long src = (((long)b * L + t0 + tt) * Q.G + g) * N + n;
      sB[i] = __ldg(Q.Bm + src);
      sC[i] = __ldg(Q.Cm + src);
    }
    __syncthreads();
    for (int tt = 0; tt < nt; ++tt) {
      const float dtv = sdt[tt];
      const float a = ex2_approx(dtv * a_l2);
      const float xv = sx[tt * P + p];
      const float bx = dtv * xv;
      const float4* Bt = reinterpret_cast<const float4*>(sB + tt * N + j0);
      const float4* Ct = reinterpret_cast<const float4*>(sC + tt * N + j0);
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < kSsdNS / 4; ++q) {
        const float4 bq = Bt[q], cq = Ct[q];
        s[4 * q + 0] = fmaf(a, s[4 * q + 0], bx * bq.x);
        s[4 * q + 1] = fmaf(a, s[4 * q + 1], bx * bq.y);
        s[4 * q + 2] = fmaf(a, s[4 * q + 2], bx * bq.z);
        s[4 * q + 3] = fmaf(a, s[4 * q + 3], bx * bq.w);
        acc = fmaf(s[4 * q + 0], cq.x, acc);
        acc = fmaf(s[4 * q + 1], cq.y, acc);
        acc = fmaf(s[4 * q + 2], cq.z, acc);
        acc = fmaf(s[4 * q + 3], cq.w, acc);
      }
      for (int o = tpp >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (j0 == 0) Q.y[(((long)b * L + t0 + tt) * H + h) * P + p] = acc + d_h * xv;
    }
  }
  if (Q.S_last != nullptr) {
#pragma unroll
    for (int j = 0; j < kSsdNS; ++j) Q.S_last[srow + j] = s[j];
  }
}

}  // namespace bitssm
