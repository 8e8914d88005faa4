// Ternary-weight GEMM on the 5th-generation tensor cores (tcgen05), fed by
// TMA, accumulating in tensor memory, with the BitLinear rescale and the
// next stage's quantisation fused into the epilogue.
//
//   D[m, n] = sum_k A[m, k] * W[n, k]       (A: activations, W: weights)
//
// A8: A = int8 activation codes, W = int8 {-1, 0, 1}, D int32 (kind::i8);
//     the multiply-free ternary product of "Ternary State-Space Models"
//     (abstract) is carried out exactly by the int8 datapath.
// A16: A = bf16 activations, W = bf16 w * bf16(s_group), D fp32 (kind::f16).
//
// Tile: 128 rows (tokens) x BN columns (output features, BN <= 512; above 256
// the tile is issued as two N = 256 halves), K in panels of 128 bytes.
// Operands are K-major in the 128-byte-swizzled layout that TMA writes.
//
// Warp roles (192 threads): warp 0 lane 0 issues TMA loads into a ring of
// STAGES stage buffers; warp 1 owns the TMEM allocation and lane 0 issues the
// MMAs and commits; warps 2..5 run the epilogue, each on the 32 TMEM lanes
// (rows) of quadrant warp % 4.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "kernels_rows.cuh"
#include "ptx.cuh"

namespace bitssm {

enum EpiKind : int {
  EPI_STORE = 0,      // y = acc * alpha * row_scale[m] (+ residual) -> f32 / bf16 / raw i32
  EPI_QUANT_ROW = 1,  // A8 in_proj: u (f32) + codes of the int32 row + deq_u
  EPI_XPROJ_A8 = 2,   // A8 x_proj: dt codes + deq_dt from the int32 row, B and C (f32)
  EPI_ROWSS = 3,      // A16 in_proj: u (bf16) = acc * r_x + partial sum(u^2) per tile
  EPI_XPROJ_A16 = 4,  // A16 x_proj: dt_low (bf16) + r_dt, B and C (f32)
};

struct GemmParams {
  int M, N, K;                 // K in elements
  int out_dtype;               // EPI_STORE: 0 f32, 1 bf16, 2 raw i32
  const float* alpha;          // device scalar: per-matrix scale s_w (null = 1)
  const float* row_scale;      // [M] per-row factor (A8: deq; A16: r); may be null (= 1)
  void* out;                   // EPI_STORE / QUANT_ROW u / ROWSS u / XPROJ_A16 dt_low
  long ld_out;                 // elements
  const void* residual;        // EPI_STORE, same dtype/pitch as out, nullable
  // EPI_QUANT_ROW / EPI_XPROJ_A8
  int8_t* q_out;               // codes [M, ld_q]
  long ld_q;
  float* deq_out;              // [M]
  // EPI_XPROJ_*: column split [0,R) dt | [R,R+Ns) B | [R+Ns, R+2Ns) C
  int R, Ns;
  const float* alpha_dt;       // device scalars (per-matrix scales of the three slices)
  const float* alpha_B;
  const float* alpha_C;
  float* Bm;                   // [M, Ns]
  float* Cm;                   // [M, Ns]
  // EPI_ROWSS: partial sums [M, gridDim.y];  EPI_XPROJ_A16: reads them (nparts)
  float* ss_part;
  const float* ss_in;
  int ss_nparts;
  int ss_count;                // number of columns the partial sums cover
  float* r_out;                // EPI_XPROJ_A16: r_dt [M]
};

template <bool kBF16>
struct GemmTraits {
  static constexpr int kElemBytes = kBF16 ? 2 : 1;
  static constexpr int kPanelElems = 128 / kElemBytes;  // K elements per 128-byte panel
  static constexpr int kKPerMma = 32 / kElemBytes;      // K elements per MMA (32 bytes)
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
}

template <bool kBF16>
__device__ __forceinline__ float acc_to_float(uint32_t bits) {
  if constexpr (kBF16) return __uint_as_float(bits);
  else return (float)(int)bits;  // exact: |acc| < 2^24
}

// Store 16 consecutive outputs of one row.
__device__ __forceinline__ void store16(void* base, long idx, int dtype, const float (&v)[16],
                                        int valid) {
  if (dtype == 0) {
    float* p = reinterpret_cast<float*>(base) + idx;
    if (valid == 16 && (idx & 3) == 0) {
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4*>(p + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    } else {
      for (int j = 0; j < valid; ++j) p[j] = v[j];
    }
  } else {
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(base) + idx;
    if (valid == 16 && (idx & 7) == 0) {
#pragma unroll
      for (int j = 0; j < 16; j += 8) {
        uint4 w = make_uint4(pack_bf16x2(v[j], v[j + 1]), pack_bf16x2(v[j + 2], v[j + 3]),
                             pack_bf16x2(v[j + 4], v[j + 5]), pack_bf16x2(v[j + 6], v[j + 7]));
        *reinterpret_cast<uint4*>(p + j) = w;
      }
    } else {
      for (int j = 0; j < valid; ++j) p[j] = __float2bfloat16_rn(v[j]);
    }
  }
}

__device__ __forceinline__ void load16_residual(const void* base, long idx, int dtype,
                                                float (&v)[16], int valid) {
  if (dtype == 0) {
    const float* p = reinterpret_cast<const float*>(base) + idx;
    for (int j = 0; j < valid; ++j) v[j] += p[j];
  } else {
    const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(base) + idx;
    for (int j = 0; j < valid; ++j) v[j] += __bfloat162float(p[j]);
  }
}

template <bool kBF16, int BN, int STAGES, int EPI>
struct GemmConfig {
  using Tr = GemmTraits<kBF16>;
  static constexpr int kABytes = 128 * 128;           // 128 rows x 128 B
  static constexpr int kBBytes = BN * 128;            // BN rows x 128 B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kBarOffset + 256;
  static constexpr int kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : BN <= 256 ? 256 : 512;
  static constexpr int kNHalf = BN > 256 ? 2 : 1;
  static constexpr int kMmaN = BN > 256 ? 256 : BN;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 512, "BN");
  static_assert(BN <= 256 || BN == 512, "BN above 256 must be 512");
};

template <bool kBF16, int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1)
    ternary_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapW, GemmParams P) {
  using Cfg = GemmConfig<kBF16, BN, STAGES, EPI>;
  using Tr = GemmTraits<kBF16>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_base = sbase + Cfg::kBarOffset;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t done_bar = bar_base + 8u * (2 * STAGES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kBarOffset + 8 * (2 * STAGES + 1));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int num_panels = (P.K + Tr::kPanelElems - 1) / Tr::kPanelElems;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(done_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    constexpr int kWBox = BN > 256 ? 256 : BN;
    constexpr uint32_t kTx = Cfg::kABytes + Cfg::kBBytes;
    for (int p = 0; p < num_panels; ++p) {
      const int s = p % STAGES;
      const uint32_t ph = (uint32_t)(p / STAGES) & 1u;
      if (p >= STAGES && !mbar_wait(empty_bar(s), ph ^ 1u, DEVFLAG_TIMEOUT_TMA)) break;
      const uint32_t sa = sbase + s * Cfg::kStageBytes;
      mbar_arrive_expect_tx(full_bar(s), kTx);
      const int kc = p * Tr::kPanelElems;
      tma_load_2d(sa, &mapA, kc, m0, full_bar(s));
#pragma unroll
      for (int h = 0; h < BN / kWBox; ++h)
        tma_load_2d(sa + Cfg::kABytes + h * kWBox * 128, &mapW, kc, n0 + h * kWBox, full_bar(s));
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t kIdesc =
        kBF16 ? umma_idesc(1u, 1u, 128u, (uint32_t)Cfg::kMmaN) : umma_idesc(2u, 1u, 128u, (uint32_t)Cfg::kMmaN);
    bool ok = true;
    for (int p = 0; p < num_panels && ok; ++p) {
      const int s = p % STAGES;
      const uint32_t ph = (uint32_t)(p / STAGES) & 1u;
      ok = mbar_wait(full_bar(s), ph, DEVFLAG_TIMEOUT_MMA);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = sbase + s * Cfg::kStageBytes;
      const uint32_t sb = sa + Cfg::kABytes;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t adesc = sw128_kmajor_desc(sa + kk * 32);
#pragma unroll
        for (int h = 0; h < Cfg::kNHalf; ++h) {
          const uint64_t bdesc = sw128_kmajor_desc(sb + h * 256 * 128 + kk * 32);
          const uint32_t acc = (p > 0 || kk > 0) ? 1u : 0u;
          if constexpr (kBF16) umma_bf16(tmem + h * 256, adesc, bdesc, kIdesc, acc);
          else umma_i8(tmem + h * 256, adesc, bdesc, kIdesc, acc);
        }
      }
      umma_commit(empty_bar(s));
    }
    umma_commit(done_bar);
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int m = m0 + row;
    const bool live = m < P.M;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const bool ok = mbar_wait(done_bar, 0u, DEVFLAG_TIMEOUT_EPI);
    tc_fence_after();
    if (ok) {
      const float rs = (P.row_scale != nullptr && live) ? P.row_scale[m] : 1.0f;

      if constexpr (EPI == EPI_STORE) {
        const float f = (P.alpha != nullptr ? *P.alpha : 1.f) * rs;
        const int ncols = min(BN, P.N - n0);
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
          if (!live || c0 >= ncols) continue;
          const int valid = min(16, ncols - c0);
          const long idx = (long)m * P.ld_out + n0 + c0;
          if (P.out_dtype == 2) {
            int* o = reinterpret_cast<int*>(P.out) + idx;
            for (int j = 0; j < valid; ++j) o[j] = (int)r[j];
            continue;
          }
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = acc_to_float<kBF16>(r[j]) * f;
          if (P.residual != nullptr) load16_residual(P.residual, idx, P.out_dtype, v, valid);
          store16(P.out, idx, P.out_dtype, v, valid);
        }
      } else if constexpr (EPI == EPI_QUANT_ROW) {
        // whole row in this tile (n0 == 0, N <= BN)
        const int N = P.N;
        int maxabs = 0;
        float ss = 0.f;
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (c0 + j < N) {
              const int a = (int)r[j];
              maxabs = max(maxabs, abs(a));
              const float fa = (float)a;
              ss = fmaf(fa, fa, ss);
            }
          }
        }
        const float c = (P.alpha != nullptr ? *P.alpha : 1.f) * rs;  // u = acc * c
        const float sigma = maxabs > 0 ? __fdiv_rn(127.f, (float)maxabs) : 0.f;
        if (live) {
          const float mu = (float)maxabs * c;
          const float r_u = 1.0f / sqrtf(c * c * (ss / (float)N) + kEpsNorm);
          P.deq_out[m] = mu * r_u / 127.f;
        }
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
          if (!live) continue;
          const int valid = min(16, N - c0);
          if (valid > 0) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = (float)(int)r[j] * c;
            store16(P.out, (long)m * P.ld_out + c0, 0, v, valid);
          }
          if (c0 < P.ld_q) {
            uint32_t w[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint32_t word = 0;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int col = c0 + g * 4 + j;
                const int code = col < N ? quant_code((float)(int)r[g * 4 + j], sigma) : 0;
                word |= (uint32_t)(code & 0xff) << (8 * j);
              }
              w[g] = word;
            }
            *reinterpret_cast<uint4*>(P.q_out + (long)m * P.ld_q + c0) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      } else if constexpr (EPI == EPI_XPROJ_A8) {
        // columns: [0,R) dt | [R,R+Ns) B | [R+Ns,R+2Ns) C ; whole row in this tile
        const int R = P.R, Ns = P.Ns;
        int maxabs = 0;
        float ss = 0.f;
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            if (col < R) {
              const int a = (int)r[j];
              maxabs = max(maxabs, abs(a));
              const float fa = (float)a;
              ss = fmaf(fa, fa, ss);
            }
          }
        }
        const float cdt = *P.alpha_dt * rs;  // dt_low = acc * cdt
        const float sigma = maxabs > 0 ? __fdiv_rn(127.f, (float)maxabs) : 0.f;
        if (live) {
          const float mdt = (float)maxabs * cdt;
          const float r_dt = 1.0f / sqrtf(cdt * cdt * (ss / (float)R) + kEpsNorm);
          P.deq_out[m] = mdt * r_dt / 127.f;
        }
        const float cB = *P.alpha_B * rs, cC = *P.alpha_C * rs;
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
          if (!live) continue;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            const int a = (int)r[j];
            if (col < R) {
              P.q_out[(long)m * P.ld_q + col] = (int8_t)quant_code((float)a, sigma);
            } else if (col < R + Ns) {
              P.Bm[(long)m * Ns + (col - R)] = (float)a * cB;
            } else if (col < R + 2 * Ns) {
              P.Cm[(long)m * Ns + (col - R - Ns)] = (float)a * cC;
            }
          }
        }
        if (live)
          for (int col = R; col < P.ld_q; ++col) P.q_out[(long)m * P.ld_q + col] = 0;
      } else if constexpr (EPI == EPI_ROWSS) {
        const int ncols = min(BN, P.N - n0);
        float ss = 0.f;
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
          if (!live || c0 >= ncols) continue;
          const int valid = min(16, ncols - c0);
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            v[j] = __uint_as_float(r[j]) * rs;
            if (j < valid) ss = fmaf(v[j], v[j], ss);
          }
          store16(P.out, (long)m * P.ld_out + n0 + c0, 1, v, valid);
        }
        if (live) P.ss_part[(long)m * gridDim.y + blockIdx.y] = ss;
      } else if constexpr (EPI == EPI_XPROJ_A16) {
        const int R = P.R, Ns = P.Ns;
        float r_u = 1.f;
        if (live) {
          float t = 0.f;
          for (int j = 0; j < P.ss_nparts; ++j) t += P.ss_in[(long)m * P.ss_nparts + j];
          r_u = 1.0f / sqrtf(t / (float)P.ss_count + kEpsNorm);
        }
        float ss = 0.f;
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          tmem_ld16(trow + c0, r);
          if (!live) continue;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            const float v = __uint_as_float(r[j]) * r_u;
            if (col < R) {
              const __nv_bfloat16 b = __float2bfloat16_rn(v);
              reinterpret_cast<__nv_bfloat16*>(P.out)[(long)m * P.ld_out + col] = b;
              const float vb = __bfloat162float(b);
              ss = fmaf(vb, vb, ss);
            } else if (col < R + Ns) {
              P.Bm[(long)m * Ns + (col - R)] = v;
            } else if (col < R + 2 * Ns) {
              P.Cm[(long)m * Ns + (col - R - Ns)] = v;
            }
          }
        }
        if (live) P.r_out[m] = 1.0f / sqrtf(ss / (float)R + kEpsNorm);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace bitssm
