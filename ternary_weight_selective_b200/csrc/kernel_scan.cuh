// Selective scan of the BitSSM mixer (TriSSM README, caption "The BitSSM
// sequence mixer": the recurrence is evaluated with a parallel associative
// scan; "Ternary State-Space Models" abstract: SSM parallel scan):
//
//   delta = softplus(delta_raw + bias[e])
//   h[e,n] <- exp(delta * A[e,n]) * h[e,n] + delta * B_t[n] * u_t[e]
//   y_t[e]  = sum_n C_t[n] * h[e,n] + D[e] * u_t[e]
//
// Parallel structure: the recurrence is an associative composition of affine
// maps h -> a h + b per (batch, channel, state); the B*E*16 state lanes are
// independent, and a step of one lane depends on the previous step only
// through one FMA (a and b are computed off the chain).  This kernel gives
// every (batch, channel) 16/NPT threads, each owning NPT states in
// registers, walks the time axis in chunks of TC steps staged in shared
// memory, and reduces y over the channel's threads with warp shuffles.
//
// FUSED_DT: delta_raw is not read from memory but formed here from the int8
// codes of the low-rank Delta projection (the Delta-up BitLinear):
//   delta_raw[t,e] = s_up * deq_dt[t] * sum_r W_up[e,r] * q_dt[t,r]
// as an exact int32 dot product (dp4a), so the [T, E] delta tensor never
// exists in memory.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels_rows.cuh"
#include "ptx.cuh"

namespace bitssm {

constexpr int kScanN = 16;   // d_state
constexpr int kScanTC = 32;  // time steps per staged chunk
constexpr float kLog2e = 1.4426950408889634f;

struct ScanParams {
  const void* u;          // [B, L, E]
  const void* delta_raw;  // [B, L, E] (unfused)
  const int8_t* q_dt;     // [B*L, ld_qdt] (fused)
  long ld_qdt;
  const float* deq_dt;    // [B*L] (fused)
  const int8_t* W_up;     // [E, ld_w] int8 {-1,0,1} (fused)
  long ld_w;
  const float* s_up;      // device scalar (fused)
  int R;                  // padded to a multiple of 4 (zero codes beyond dt_rank)
  const float* bias;      // [E]
  const float* A;         // [E, 16]
  const float* Bm;        // [B, L, 16]
  const float* Cm;        // [B, L, 16]
  const float* D;         // [E]
  const float* h0;        // [B, E, 16] nullable
  void* y;                // [B, L, E]
  float* h_last;          // [B, E, 16] nullable
  int B, L, E;
};

template <typename T>
__device__ __forceinline__ void store_as(T* p, float v);
template <>
__device__ __forceinline__ void store_as<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_as<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float softplus_f(float z) {
  return fmaxf(z, 0.f) + log1pf(expf(-fabsf(z)));
}

// Shared-memory footprint of one CTA (bytes), for CE channels per CTA.
__host__ __device__ constexpr int scan_smem_bytes(int CE, int Rmax) {
  return kScanTC * CE * 4 * 3        // u_s, dt_s, y_s
         + kScanTC * kScanN * 4 * 2  // B_s, C_s
         + kScanTC * Rmax            // qdt_s
         + kScanTC * 4               // deq_s
         + CE * Rmax;                // W_s
}

template <int NPT, bool FUSED, typename Tu, typename Td, typename Ty>
__global__ void __launch_bounds__(128) selective_scan_kernel(ScanParams P) {
  constexpr int TPC = kScanN / NPT;  // threads per channel
  constexpr int CE = 128 / TPC;      // channels per CTA
  extern __shared__ __align__(16) uint8_t smem[];
  float* u_s = reinterpret_cast<float*>(smem);
  float* dt_s = u_s + kScanTC * CE;
  float* y_s = dt_s + kScanTC * CE;
  float* B_s = y_s + kScanTC * CE;
  float* C_s = B_s + kScanTC * kScanN;
  float* deq_s = C_s + kScanTC * kScanN;
  int8_t* qdt_s = reinterpret_cast<int8_t*>(deq_s + kScanTC);
  int8_t* W_s = qdt_s + kScanTC * (FUSED ? P.R : 0);

  const int tid = threadIdx.x;
  const int b = blockIdx.y;
  const int e0 = blockIdx.x * CE;
  const int c = tid / TPC;        // channel within the CTA
  const int g = tid % TPC;        // state group
  const int e = e0 + c;
  const bool ch_ok = e < P.E;
  const int E = P.E, L = P.L;
  const long tok0 = (long)b * L;

  if constexpr (FUSED) {
    // Delta-up weights of this CTA's channels, [CE][R]
    for (int i = tid; i < CE * P.R; i += 128) {
      const int cc = i / P.R, r = i - cc * P.R;
      W_s[i] = (e0 + cc < E) ? P.W_up[(long)(e0 + cc) * P.ld_w + r] : (int8_t)0;
    }
  }

  float A2[NPT], h[NPT];
#pragma unroll
  for (int j = 0; j < NPT; ++j) {
    const int n = g * NPT + j;
    A2[j] = ch_ok ? P.A[(long)e * kScanN + n] * kLog2e : 0.f;
    h[j] = (ch_ok && P.h0 != nullptr) ? P.h0[((long)b * E + e) * kScanN + n] : 0.f;
  }
  const float Dv = ch_ok ? P.D[e] : 0.f;
  float s_up = 0.f;
  if constexpr (FUSED) s_up = *P.s_up;

  for (int t0 = 0; t0 < L; t0 += kScanTC) {
    const int tc = min(kScanTC, L - t0);
    __syncthreads();  // previous chunk's y_s consumed, W_s written
    // ---- stage the chunk
    for (int i = tid; i < kScanTC * CE; i += 128) {
      const int t = i / CE, cc = i - t * CE;
      float uv = 0.f, dv = 0.f;
      if (t < tc && e0 + cc < E) {
        const long idx = (tok0 + t0 + t) * E + e0 + cc;
        uv = load_as_float(reinterpret_cast<const Tu*>(P.u) + idx);
        if constexpr (!FUSED) dv = load_as_float(reinterpret_cast<const Td*>(P.delta_raw) + idx);
      }
      u_s[i] = uv;
      dt_s[i] = dv;
    }
    for (int i = tid; i < kScanTC * kScanN; i += 128) {
      const int t = i / kScanN;
      const long idx = (tok0 + t0) * kScanN + i;
      B_s[i] = t < tc ? P.Bm[idx] : 0.f;
      C_s[i] = t < tc ? P.Cm[idx] : 0.f;
    }
    if constexpr (FUSED) {
      for (int i = tid; i < kScanTC * P.R; i += 128) {
        const int t = i / P.R, r = i - t * P.R;
        qdt_s[i] = t < tc ? P.q_dt[(tok0 + t0 + t) * P.ld_qdt + r] : (int8_t)0;
      }
      for (int t = tid; t < kScanTC; t += 128) deq_s[t] = t < tc ? P.deq_dt[tok0 + t0 + t] : 0.f;
    }
    __syncthreads();
    // ---- phase A: delta for every (t, channel) of the chunk, once
    for (int i = tid; i < kScanTC * CE; i += 128) {
      const int t = i / CE, cc = i - t * CE;
      float z;
      if constexpr (FUSED) {
        int acc = 0;
        const int* wq = reinterpret_cast<const int*>(W_s + cc * P.R);
        const int* qq = reinterpret_cast<const int*>(qdt_s + t * P.R);
        for (int r4 = 0; r4 < P.R / 4; ++r4) acc = __dp4a(wq[r4], qq[r4], acc);
        z = (float)acc * s_up * deq_s[t];
      } else {
        z = dt_s[i];
      }
      const float bias = (e0 + cc < E) ? P.bias[e0 + cc] : 0.f;
      dt_s[i] = softplus_f(z + bias);
    }
    __syncthreads();
    // ---- phase B: the recurrence, TC steps
    for (int t = 0; t < tc; ++t) {
      const float dlt = dt_s[t * CE + c];
      const float uv = u_s[t * CE + c];
      const float du = dlt * uv;
      float yp = 0.f;
#pragma unroll
      for (int j = 0; j < NPT; ++j) {
        const int n = g * NPT + j;
        const float a = ex2_approx(dlt * A2[j]);
        h[j] = fmaf(a, h[j], du * B_s[t * kScanN + n]);
        yp = fmaf(C_s[t * kScanN + n], h[j], yp);
      }
#pragma unroll
      for (int o = TPC / 2; o > 0; o >>= 1) yp += __shfl_xor_sync(0xffffffffu, yp, o);
      if (g == 0) y_s[t * CE + c] = fmaf(Dv, uv, yp);
    }
    __syncthreads();
    // ---- phase C: write the chunk's outputs
    for (int i = tid; i < kScanTC * CE; i += 128) {
      const int t = i / CE, cc = i - t * CE;
      if (t < tc && e0 + cc < E)
        store_as(reinterpret_cast<Ty*>(P.y) + (tok0 + t0 + t) * E + e0 + cc, y_s[i]);
    }
  }
  if (P.h_last != nullptr && ch_ok) {
#pragma unroll
    for (int j = 0; j < NPT; ++j) P.h_last[((long)b * E + e) * kScanN + g * NPT + j] = h[j];
  }
}

}  // namespace bitssm
