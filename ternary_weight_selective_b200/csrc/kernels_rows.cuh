// Row-wise kernels: absmax int8 quantisation with the RMSNorm folded in,
// the RMSNorm factor alone, absmean ternary packing, and the expansion of
// packed ternary weights to tensor-core operand form.
//
// Quantiser (BitNet b1.58 BitLinear activations, TriSSM README opening
// paragraph; an RMSNorm precedes each ternary projection, TriSSM README
// caption "The BitSSM sequence mixer"):
//   m = max|v|, sigma = fl32(127 / m), q = clamp(rint(fl32(v * sigma)), -128, 127)
//   r = 1 / sqrt(mean(v^2) + eps),  deq = m * r / 127
// Unit-gain RMSNorm scales a row by r > 0 and max|v r| = m r, so the codes of
// the normalised row are the codes of v, and the dequantisation factor of
// the normalised row's codes, expressed against v, is m r / 127.
// The code decision uses IEEE round-to-nearest float32 division and
// multiplication (__fdiv_rn, __fmul_rn) and round-half-to-even conversion,
// never a contracted or approximate form.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace bitssm {

constexpr float kEpsNorm = 1e-5f;
constexpr float kEpsW = 1e-5f;

template <typename T>
__device__ __forceinline__ float load_as_float(const T* p);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_as_float<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int quant_code(float v, float sigma) {
  int q = __float2int_rn(__fmul_rn(v, sigma));
  return max(-128, min(127, q));
}

// Exact conversions on the FMA/ALU pipes for |x| < 2^22, through the float
// 1.5 * 2^23 (bit pattern 0x4B400000), whose ulp is 1: adding an integer-
// valued or real x lands in [2^23, 2^24), where the IEEE round-to-nearest-
// even addition performs rint(x) and the low mantissa bits hold rint(x) in
// two's complement.
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

// softplus(z) = max(z, 0) + log1p(t), t = exp(-|z|) in (0, 1], with log1p(t)
// = t * p(t) and p a degree-8 least-squares fit of log1p(t)/t on [0, 1]
// (coefficients from gen_softplus_poly.py; relative error ~3e-8 before
// float32 rounding).  One exp2 and nine FMAs.
__device__ __forceinline__ float softplus_fast(float z) {
  const float t = ex2_approx(-fabsf(z) * kLog2e);
  float p = 5.253457797e-03f;
  p = fmaf(p, t, -2.958850739e-02f);
  p = fmaf(p, t, 7.836166802e-02f);
  p = fmaf(p, t, -1.367476971e-01f);
  p = fmaf(p, t, 1.911143108e-01f);
  p = fmaf(p, t, -2.484436989e-01f);
  p = fmaf(p, t, 3.331927134e-01f);
  p = fmaf(p, t, -4.999950152e-01f);
  p = fmaf(p, t, 9.999999705e-01f);
  return fmaxf(z, 0.f) + t * p;
}

__device__ __forceinline__ float i2f_exact(int a) { return __int_as_float(a + kMagicBits) - kMagic; }
// Bit pattern whose low byte is the int8 code rint(v * sigma).  With
// sigma = 127 / max|v| the product never exceeds 127 in magnitude (so the
// clamp to [-128, 127] of the definition never binds).  Both steps are
// IEEE round-to-nearest (no contraction into an FMA).
__device__ __forceinline__ uint32_t code_bits(float v, float sigma) {
  return __float_as_uint(__fadd_rn(__fmul_rn(v, sigma), kMagic));
}
// Four codes (low bytes of four code_bits words) packed into one word.
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// One warp per row.  x [M, K] (row pitch ldx elements) -> q int8 [M, ldq]
// (columns K..ldq-1 written as 0), deq [M].  The row is read twice (the
// second time from L1/L2): once for max|v| and sum(v^2), once for the codes.
template <typename T>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T* __restrict__ x, int M, int K,
                                                         long ldx, int8_t* __restrict__ q,
                                                         long ldq, float* __restrict__ deq) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    const T* xr = x + row * ldx;
    float mx = 0.f, ss = 0.f;
    for (int k = lane; k < K; k += 32) {
      float v = load_as_float(xr + k);
      mx = fmaxf(mx, fabsf(v));
      ss = fmaf(v, v, ss);
    }
    mx = warp_max(mx);
    ss = warp_sum(ss);
    const float sigma = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;
    int8_t* qr = q + row * ldq;
    // 4 codes per lane per step, written as one 32-bit word
    for (int k0 = lane * 4; k0 < ldq; k0 += 128) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int k = k0 + j;
        int c = 0;
        if (k < K) c = quant_code(load_as_float(xr + k), sigma);
        word |= (uint32_t)(c & 0xff) << (8 * j);
      }
      *reinterpret_cast<uint32_t*>(qr + k0) = word;
    }
    if (lane == 0) {
      const float r = 1.0f / sqrtf(ss / (float)K + kEpsNorm);
      deq[row] = mx * r / 127.f;
    }
  }
}

// Vector form of quant_rows_kernel for rows of at most VPL*32 16-byte
// vectors: every lane loads its vectors once into registers (16-byte loads,
// coalesced across the warp), and writes its codes as one 4- or 8-byte store
// per vector.  Requires K and ldx multiples of the vector width and a
// 16-byte aligned x.
template <typename T, int VPL>
__global__ void __launch_bounds__(256) quant_rows_vec_kernel(const T* __restrict__ x, int M, int K,
                                                             long ldx, int8_t* __restrict__ q,
                                                             long ldq, float* __restrict__ deq) {
  constexpr int EPV = 16 / (int)sizeof(T);  // elements per vector
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    const T* xr = x + row * ldx;
    float v[VPL][EPV];
    float mx = 0.f, ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int k0 = (i * 32 + lane) * EPV;
      if (k0 < K) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(xr + k0));
        if constexpr (sizeof(T) == 4) {
          v[i][0] = __uint_as_float(raw.x);
          v[i][1] = __uint_as_float(raw.y);
          v[i][2] = __uint_as_float(raw.z);
          v[i][3] = __uint_as_float(raw.w);
        } else {
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            v[i][2 * j] = __uint_as_float(w[j] << 16);
            v[i][2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < EPV; ++j) v[i][j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < EPV; ++j) {
        mx = fmaxf(mx, fabsf(v[i][j]));
        ss = fmaf(v[i][j], v[i][j], ss);
      }
    }
    mx = warp_max(mx);
    ss = warp_sum(ss);
    const float sigma = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;
    int8_t* qr = q + row * ldq;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int k0 = (i * 32 + lane) * EPV;
      if (k0 < K) {
        uint32_t w[EPV / 4];
#pragma unroll
        for (int j4 = 0; j4 < EPV / 4; ++j4)
          w[j4] = pack4(code_bits(v[i][4 * j4], sigma), code_bits(v[i][4 * j4 + 1], sigma),
                        code_bits(v[i][4 * j4 + 2], sigma), code_bits(v[i][4 * j4 + 3], sigma));
        if constexpr (EPV == 4) *reinterpret_cast<uint32_t*>(qr + k0) = w[0];
        else *reinterpret_cast<uint2*>(qr + k0) = make_uint2(w[0], w[1]);
      }
    }
    for (int k = K + lane; k < ldq; k += 32) qr[k] = 0;
    if (lane == 0) {
      const float r = 1.0f / sqrtf(ss / (float)K + kEpsNorm);
      deq[row] = mx * r / 127.f;
    }
  }
}

// ------------------------------------------------------ Mamba-1 block pieces
// SiLU(v) = v / (1 + e^-v) in float32 with every step IEEE round-to-nearest
// (no contraction), so that evaluating it twice gives the same bits.  For
// v -> -inf, e^-v overflows to inf and the quotient is -0; for v -> +inf it
// is v.
__device__ __forceinline__ float silu_rn(float v) {
  return __fdiv_rn(v, __fadd_rn(1.f, expf(-v)));
}

// Depthwise causal conv + SiLU on the in_proj branch, then the absmax int8
// codes of the result (the quantiser above).  One warp per token row
// t = b * L + l of u_pre [M, E] (M = B * L):
//   u[t, e] = SiLU(cb[e] + sum_k w[e, k] * u_pre[t - (K-1) + k, e]),
// a tap that reaches before the start of its sequence (l - (K-1) + k < 0)
// contributes nothing.  w float [E, K], cb float [E] or null (zero).
// Writes u float [M, E], q int8 [M, ldq] (columns E..ldq-1 zero), deq [M].
__global__ void __launch_bounds__(256) conv_silu_quant_kernel(
    const float* __restrict__ u_pre, int M, int L, int E, const float* __restrict__ w,
    const float* __restrict__ cb, int K, float* __restrict__ u, int8_t* __restrict__ q, long ldq,
    float* __restrict__ deq) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    const int l = (int)(row % L);
    const int taps = K < l + 1 ? K : l + 1;  // taps inside the sequence
    float mx = 0.f, ss = 0.f;
    for (int e = lane; e < E; e += 32) {
      float acc = cb != nullptr ? __ldg(cb + e) : 0.f;
      for (int back = 0; back < taps; ++back)  // back = steps into the past
        acc = fmaf(__ldg(w + (long)e * K + (K - 1 - back)), __ldg(u_pre + (row - back) * E + e), acc);
      const float v = silu_rn(acc);
      u[row * E + e] = v;
      mx = fmaxf(mx, fabsf(v));
      ss = fmaf(v, v, ss);
    }
    mx = warp_max(mx);
    ss = warp_sum(ss);
    const float sigma = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;
    int8_t* qr = q + row * ldq;
    // each lane reads back only the elements it wrote itself
    for (int e = lane; e < ldq; e += 32)
      qr[e] = e < E ? (int8_t)quant_code(u[row * E + e], sigma) : (int8_t)0;
    if (lane == 0) {
      const float r = 1.0f / sqrtf(ss / (float)E + kEpsNorm);
      deq[row] = mx * r / 127.f;
    }
  }
}

// The gate of the Mamba-1 block and the absmax codes of the gated row: one
// warp per row, y_g = y * SiLU(z) (y, z float [M, E]), then q int8 [M, ldq]
// and deq [M] of y_g as quant_rows_kernel.  y_g is formed twice (for the row
// statistics, then for the codes), bit-identically.  With keep != 0, y is
// overwritten with y_g (for stage checks).
__global__ void __launch_bounds__(256) gate_quant_kernel(float* __restrict__ y,
                                                         const float* __restrict__ z, int M, int E,
                                                         int8_t* __restrict__ q, long ldq,
                                                         float* __restrict__ deq, int keep) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    float* yr = y + row * E;
    const float* zr = z + row * E;
    float mx = 0.f, ss = 0.f;
    for (int e = lane; e < E; e += 32) {
      const float g = __fmul_rn(yr[e], silu_rn(__ldg(zr + e)));
      mx = fmaxf(mx, fabsf(g));
      ss = fmaf(g, g, ss);
    }
    mx = warp_max(mx);
    ss = warp_sum(ss);
    const float sigma = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;
    int8_t* qr = q + row * ldq;
    for (int e = lane; e < ldq; e += 32) {
      int c = 0;
      if (e < E) {
        const float g = __fmul_rn(yr[e], silu_rn(__ldg(zr + e)));
        c = quant_code(g, sigma);
        if (keep) yr[e] = g;
      }
      qr[e] = (int8_t)c;
    }
    if (lane == 0) {
      const float r = 1.0f / sqrtf(ss / (float)E + kEpsNorm);
      deq[row] = mx * r / 127.f;
    }
  }
}

// SiLU on the special-function unit: v * 1 / (1 + 2^(-v log2 e)), with the
// IEEE-rounded reciprocal.  Relative error about |v| * 6e-8 + 3e-7 (the
// exp2 approximation and the rounding of its argument); -0 for v -> -inf.
__device__ __forceinline__ float silu_fast(float v) {
  return v * __frcp_rn(1.f + ex2_approx(-v * kLog2e));
}

__device__ __forceinline__ float4 silu4(float4 a) {
  return make_float4(silu_fast(a.x), silu_fast(a.y), silu_fast(a.z), silu_fast(a.w));
}

// Row statistics and codes of VPL float4 vectors per lane (the quantiser
// above); every lane of the warp calls it for one row.
template <int VPL>
__device__ __forceinline__ void quant_row_regs(const float4 (&v)[VPL], int lane, int E,
                                               int8_t* qr, long ldq, float* deq_row) {
  float mx = 0.f, ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
    ss = fmaf(v[i].x, v[i].x, ss);
    ss = fmaf(v[i].y, v[i].y, ss);
    ss = fmaf(v[i].z, v[i].z, ss);
    ss = fmaf(v[i].w, v[i].w, ss);
  }
  mx = warp_max(mx);
  ss = warp_sum(ss);
  const float sigma = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    *reinterpret_cast<uint32_t*>(qr + (i * 32 + lane) * 4) =
        pack4(code_bits(v[i].x, sigma), code_bits(v[i].y, sigma), code_bits(v[i].z, sigma),
              code_bits(v[i].w, sigma));
  for (long k = (long)VPL * 128 + lane; k < ldq; k += 32) qr[k] = 0;
  if (lane == 0) {
    const float r = 1.0f / sqrtf(ss / (float)E + kEpsNorm);
    *deq_row = mx * r / 127.f;
  }
}

// Vector form of conv_silu_quant_kernel for E = 128 * VPL: each lane holds
// 4 * VPL channels of its row in registers (16-byte loads of all the taps'
// rows at once, coalesced across the warp), the taps are staged transposed
// ([tap][channel]) in shared memory, and the codes are written as one word
// per 4 channels.  u_pre and u 16-byte aligned.
template <int VPL>
__global__ void __launch_bounds__(256) conv_silu_quant_vec_kernel(
    const float* __restrict__ u_pre, int M, int L, int E, const float* __restrict__ w,
    const float* __restrict__ cb, int K, float* __restrict__ u, int8_t* __restrict__ q, long ldq,
    float* __restrict__ deq) {
  __shared__ float4 s_w[4][VPL * 32];
  __shared__ float4 s_b[VPL * 32];
  for (int i = threadIdx.x; i < VPL * 32; i += blockDim.x) {
    const int c = 4 * i;
#pragma unroll
    for (int k = 0; k < 4; ++k)
      s_w[k][i] = k < K ? make_float4(__ldg(w + (long)c * K + k), __ldg(w + (long)(c + 1) * K + k),
                                      __ldg(w + (long)(c + 2) * K + k), __ldg(w + (long)(c + 3) * K + k))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    s_b[i] = cb != nullptr ? make_float4(__ldg(cb + c), __ldg(cb + c + 1), __ldg(cb + c + 2), __ldg(cb + c + 3))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    const int l = (int)(row % L);
    float4 tap[4][VPL];
#pragma unroll
    for (int back = 0; back < 4; ++back)  // back = steps into the past
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        tap[back][i] = (back < K && back <= l)
                           ? __ldg(reinterpret_cast<const float4*>(u_pre + (row - back) * E) + i * 32 + lane)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      float4 a = s_b[i * 32 + lane];
#pragma unroll
      for (int back = 0; back < 4; ++back) {
        if (back < K) {
          const float4 t = s_w[K - 1 - back][i * 32 + lane];
          a.x = fmaf(t.x, tap[back][i].x, a.x);
          a.y = fmaf(t.y, tap[back][i].y, a.y);
          a.z = fmaf(t.z, tap[back][i].z, a.z);
          a.w = fmaf(t.w, tap[back][i].w, a.w);
        }
      }
      v[i] = silu4(a);
      reinterpret_cast<float4*>(u + row * E)[i * 32 + lane] = v[i];
    }
    quant_row_regs<VPL>(v, lane, E, q + row * ldq, ldq, deq + row);
  }
}

// Vector form of gate_quant_kernel for E = 128 * VPL: y_g = y * SiLU(z)
// formed once in registers; y and z 16-byte aligned.
template <int VPL>
__global__ void __launch_bounds__(256) gate_quant_vec_kernel(float* __restrict__ y,
                                                             const float* __restrict__ z, int M,
                                                             int E, int8_t* __restrict__ q,
                                                             long ldq, float* __restrict__ deq,
                                                             int keep) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    float4* yr = reinterpret_cast<float4*>(y + row * E);
    const float4* zr = reinterpret_cast<const float4*>(z + row * E);
    float4 yv[VPL], zv[VPL], g[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      yv[i] = yr[i * 32 + lane];
      zv[i] = __ldg(zr + i * 32 + lane);
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const float4 sz = silu4(zv[i]);
      g[i] = make_float4(yv[i].x * sz.x, yv[i].y * sz.y, yv[i].z * sz.z, yv[i].w * sz.w);
      if (keep) yr[i * 32 + lane] = g[i];
    }
    quant_row_regs<VPL>(g, lane, E, q + row * ldq, ldq, deq + row);
  }
}

// r[m] = 1 / sqrt(mean(x[m]^2) + eps), one warp per row.
template <typename T>
__global__ void __launch_bounds__(256) row_rms_kernel(const T* __restrict__ x, int M, int K,
                                                      long ldx, float* __restrict__ r) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    const T* xr = x + row * ldx;
    float ss = 0.f;
    for (int k = lane; k < K; k += 32) {
      float v = load_as_float(xr + k);
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) r[row] = 1.0f / sqrtf(ss / (float)K + kEpsNorm);
  }
}

// Sum of squares of the floats held in one 16-byte vector of T.
template <typename T>
__device__ __forceinline__ float vec_sumsq(const uint4 q, float acc);
template <>
__device__ __forceinline__ float vec_sumsq<float>(const uint4 q, float acc) {
  acc = fmaf(__uint_as_float(q.x), __uint_as_float(q.x), acc);
  acc = fmaf(__uint_as_float(q.y), __uint_as_float(q.y), acc);
  acc = fmaf(__uint_as_float(q.z), __uint_as_float(q.z), acc);
  return fmaf(__uint_as_float(q.w), __uint_as_float(q.w), acc);
}
template <>
__device__ __forceinline__ float vec_sumsq<__nv_bfloat16>(const uint4 q, float acc) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xffff0000u);
    acc = fmaf(a, a, acc);
    acc = fmaf(b, b, acc);
  }
  return acc;
}

// row_rms_kernel with 16-byte loads: a warp per row, four vectors in flight
// per lane into four partial sums (rows of K * sizeof(T) bytes, a multiple
// of 16, at 16-byte aligned starts).
template <typename T>
__global__ void __launch_bounds__(256) row_rms_vec_kernel(const T* __restrict__ x, int M, int K,
                                                          long ldx, float* __restrict__ r) {
  constexpr int kEpv = 16 / (int)sizeof(T);
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nvec = K / kEpv;
  for (long row = (long)blockIdx.x * warps + (threadIdx.x >> 5); row < M;
       row += (long)gridDim.x * warps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int v = lane;
    for (; v + 96 < nvec; v += 128) {
      const uint4 q0 = __ldg(xr + v), q1 = __ldg(xr + v + 32), q2 = __ldg(xr + v + 64),
                  q3 = __ldg(xr + v + 96);
      s0 = vec_sumsq<T>(q0, s0);
      s1 = vec_sumsq<T>(q1, s1);
      s2 = vec_sumsq<T>(q2, s2);
      s3 = vec_sumsq<T>(q3, s3);
    }
    for (; v < nvec; v += 32) s0 = vec_sumsq<T>(__ldg(xr + v), s0);
    const float ss = warp_sum((s0 + s1) + (s2 + s3));
    if (lane == 0) r[row] = 1.0f / sqrtf(ss / (float)K + kEpsNorm);
  }
}

// ---------------------------------------------------------------------------
// Absmean ternary packing (BitNet b1.58 weights; grouped scales: Ternary
// Mamba abstract).  s = mean|W| summed in float64 and rounded to float;
// W_q = clip(rint(W / fl32(s + 1e-5)), -1, 1); code c = W_q + 1 at bits
// 2*(k mod 4) of byte k/4, padding c = 1.
// ---------------------------------------------------------------------------

// Per-tensor scale, pass 1: `nparts` fixed partial sums of |W| in float64
// (grid-stride over a fixed partition, so the summation order is fixed).
__global__ void __launch_bounds__(256) absmean_partial_kernel(const float* __restrict__ W,
                                                              long count,
                                                              double* __restrict__ parts) {
  __shared__ double red[8];
  double acc = 0.0;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (long)gridDim.x * blockDim.x)
    acc += fabs((double)W[i]);
  acc = warp_sum_d(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    parts[blockIdx.x] = t;
  }
}

__device__ __forceinline__ uint32_t ternary_code2(float w, float denom) {
  int c = __float2int_rn(__fdiv_rn(w, denom));
  c = max(-1, min(1, c));
  return (uint32_t)(c + 1);
}

// Per-tensor scale, pass 2: every block sums the partials in the same order,
// then packs one byte (4 codes) per thread.
__global__ void __launch_bounds__(256) pack_tensor_kernel(const float* __restrict__ W, int n_out,
                                                          int k_in, const double* __restrict__ parts,
                                                          int nparts, uint8_t* __restrict__ packed,
                                                          float* __restrict__ scales) {
  __shared__ float s_sh;
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < nparts; ++i) t += parts[i];
    s_sh = (float)(t / ((double)n_out * (double)k_in));
    if (blockIdx.x == 0) scales[0] = s_sh;
  }
  __syncthreads();
  const float denom = __fadd_rn(s_sh, kEpsW);
  const int kb = (k_in + 3) / 4;
  const long nbytes = (long)n_out * kb;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < nbytes;
       i += (long)gridDim.x * blockDim.x) {
    const long n = i / kb;
    const int b = (int)(i - n * kb);
    uint32_t byte = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = 4 * b + j;
      uint32_t c = 1;
      if (k < k_in) c = ternary_code2(W[n * k_in + k], denom);
      byte |= c << (2 * j);
    }
    packed[i] = (uint8_t)byte;
  }
}

// Grouped scales: one warp per (row, group); the group's float64 sum of |W|
// is reduced across the warp, then the warp packs the group's codes.
__global__ void __launch_bounds__(256) pack_group_kernel(const float* __restrict__ W, int n_out,
                                                         int k_in, int group,
                                                         uint8_t* __restrict__ packed,
                                                         float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int ng = (k_in + group - 1) / group;
  const int kb = (k_in + 3) / 4;
  const long total = (long)n_out * ng;
  const int warps = blockDim.x >> 5;
  for (long gi = (long)blockIdx.x * warps + (threadIdx.x >> 5); gi < total;
       gi += (long)gridDim.x * warps) {
    const long n = gi / ng;
    const int j = (int)(gi - n * ng);
    const int k0 = j * group;
    const int k1 = min(k_in, k0 + group);
    double acc = 0.0;
    for (int k = k0 + lane; k < k1; k += 32) acc += fabs((double)W[n * k_in + k]);
    acc = warp_sum_d(acc);
    const float s = (float)(acc / (double)(k1 - k0));
    if (lane == 0) scales[gi] = s;
    const float denom = __fadd_rn(s, kEpsW);
    // group is a multiple of 4, so bytes never straddle groups
    for (int b = k0 / 4 + lane; b < (k1 + 3) / 4; b += 32) {
      uint32_t byte = 0;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int k = 4 * b + jj;
        uint32_t c = 1;
        if (k < k1) c = ternary_code2(W[n * k_in + k], denom);
        byte |= c << (2 * jj);
      }
      packed[n * kb + b] = (uint8_t)byte;
    }
  }
}

// ---------------------------------------------------------------------------
// Expansion of packed ternary weights to tensor-core operand rows.
// ---------------------------------------------------------------------------

// One expansion job: rows [row0, row0 + n_out) of a destination matrix with
// row pitch ld elements; columns k_in..ld-1 are written as zero.
struct ExpandJob {
  const uint8_t* packed;
  const float* scales;
  int n_out, k_in, group;
  int row0;
  void* dst;
  int ld;
  float* s_t;   // bf16 expansion: transposed group scales [G][ld_s] (rows row0..)
  long ld_s;
};
struct ExpandJobs {
  ExpandJob job[8];
  int count;
};

// 16 codes (one 32-bit word of packed bytes) -> 16 int8 in a uint4.
__device__ __forceinline__ uint4 expand16_i8(uint32_t p) {
  // t_j holds, in byte b, the code of element 4b + j
  const uint32_t t0 = p & 0x03030303u;
  const uint32_t t1 = (p >> 2) & 0x03030303u;
  const uint32_t t2 = (p >> 4) & 0x03030303u;
  const uint32_t t3 = (p >> 6) & 0x03030303u;
  const uint32_t a01 = __byte_perm(t0, t1, 0x5140);  // t0.b0 t1.b0 t0.b1 t1.b1
  const uint32_t a23 = __byte_perm(t2, t3, 0x5140);
  const uint32_t b01 = __byte_perm(t0, t1, 0x7362);  // t0.b2 t1.b2 t0.b3 t1.b3
  const uint32_t b23 = __byte_perm(t2, t3, 0x7362);
  uint4 o;
  o.x = __byte_perm(a01, a23, 0x5410);  // elements 0..3
  o.y = __byte_perm(a01, a23, 0x7632);  // elements 4..7
  o.z = __byte_perm(b01, b23, 0x5410);  // elements 8..11
  o.w = __byte_perm(b01, b23, 0x7632);  // elements 12..15
  // c in {0,1,2} per byte -> c - 1 as int8: (c + 0x7f) ^ 0x80, no carries
  o.x = (o.x + 0x7f7f7f7fu) ^ 0x80808080u;
  o.y = (o.y + 0x7f7f7f7fu) ^ 0x80808080u;
  o.z = (o.z + 0x7f7f7f7fu) ^ 0x80808080u;
  o.w = (o.w + 0x7f7f7f7fu) ^ 0x80808080u;
  return o;
}

// int8 expansion over one flat index space covering every job: each thread
// writes 16 consecutive elements (one 32-bit word of packed codes) of one
// row.  `first[j]` is the first flat index of job j (first[count] = total).
__global__ void __launch_bounds__(256) expand_i8_kernel(ExpandJobs jobs, int4 first_lo,
                                                        int4 first_hi) {
  const int first[8] = {first_lo.x, first_lo.y, first_lo.z, first_lo.w,
                        first_hi.x, first_hi.y, first_hi.z, first_hi.w};
  const int total = first[jobs.count];
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    int ji = 0;
#pragma unroll
    for (int k = 1; k < 7; ++k)
      if (k < jobs.count && i >= first[k]) ji = k;
    const ExpandJob& J = jobs.job[ji];
    const int chunks = J.ld / 16;
    const int li = i - first[ji];
    const int n = li / chunks;
    const int ch = li - n * chunks;
    const int kb = (J.k_in + 3) / 4;
    const uint8_t* src = J.packed + (long)n * kb;
    uint32_t p;
    if ((kb & 3) == 0 && ch * 4 + 4 <= kb) {
      p = __ldg(reinterpret_cast<const uint32_t*>(src) + ch);
    } else {
      p = 0x55555555u;  // code 1 (w = 0) in every slot
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int byte = ch * 4 + b;
        if (byte < kb) p = (p & ~(0xffu << (8 * b))) | ((uint32_t)src[byte] << (8 * b));
      }
    }
    *reinterpret_cast<uint4*>(reinterpret_cast<int8_t*>(J.dst) + (long)(J.row0 + n) * J.ld + ch * 16) =
        expand16_i8(p);
  }
}

// bf16 expansion: exact ternary values {-1, 0, 1} (the group scales are
// applied in fp32 by the GEMM epilogue), 8 elements per thread, plus the
// transposed fp32 group scales s_t[g][row0 + n] = s[n, g] (s[0] for group 0).
__global__ void __launch_bounds__(256) expand_bf16_kernel(ExpandJobs jobs) {
  for (int ji = 0; ji < jobs.count; ++ji) {
    const ExpandJob J = jobs.job[ji];
    const int kb = (J.k_in + 3) / 4;
    const int chunks = J.ld / 8;
    const long total = (long)J.n_out * chunks;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long)gridDim.x * blockDim.x) {
      const long n = i / chunks;
      const int ch = (int)(i - n * chunks);
      const uint8_t* src = J.packed + n * kb;
      uint32_t out[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        uint32_t pair = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int k = ch * 8 + e2 * 2 + h;
          uint32_t bits = 0;
          if (k < J.k_in) {
            const int c = (src[k >> 2] >> (2 * (k & 3))) & 3;
            // bf16 bit patterns of -1, 0, +1
            bits = c == 0 ? 0xBF80u : (c == 2 ? 0x3F80u : 0u);
          }
          pair |= bits << (16 * h);
        }
        out[e2] = pair;
      }
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(J.dst) + (long)(J.row0 + n) * J.ld + ch * 8;
      *reinterpret_cast<uint4*>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (J.s_t != nullptr) {
      const int G = (J.k_in + 127) / 128;
      const int ng = J.group > 0 ? (J.k_in + J.group - 1) / J.group : 1;
      const long nsc = (long)G * J.n_out;
      for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < nsc;
           i += (long)gridDim.x * blockDim.x) {
        const int g = (int)(i / J.n_out);
        const int n = (int)(i - (long)g * J.n_out);
        J.s_t[(long)g * J.ld_s + J.row0 + n] = J.group > 0 ? J.scales[(long)n * ng + g] : J.scales[0];
      }
    }
  }
}

}  // namespace bitssm
