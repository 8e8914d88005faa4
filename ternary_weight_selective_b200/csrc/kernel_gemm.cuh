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
  EPI_DELTA = 5,      // dt_proj: delta = softplus(acc * alpha * row_scale[m] + bias[n]) -> f32
                      // (A16: the group-scaled kernel, alpha = 1; A8: the int8 kernel)
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
  const float* bias;           // EPI_DELTA: [N]
  // group-scaled (W1.58A16) kernel: fp32 scales transposed, s_t[g * ld_s + n]
  const float* s_t;
  long ld_s;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(a)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(b)) << 16);
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

template <int BN, int STAGES, int CSPLIT>
struct GemmConfig {
  static constexpr int kABytes = 128 * 128;           // 128 rows x 128 B
  static constexpr int kBBytes = BN * 128;            // BN rows x 128 B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kRedOffset = kBarOffset + 256;  // row partials [2][CSPLIT][128]
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kRedOffset + 2 * CSPLIT * 128 * 4;
  static constexpr int kTmemCols = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : BN <= 256 ? 256 : 512;
  static constexpr int kNHalf = BN > 256 ? 2 : 1;
  static constexpr int kMmaN = BN > 256 ? 256 : BN;
  static constexpr int kSlice = BN / CSPLIT;           // columns per epilogue warp
  static constexpr int kThreads = 64 + 128 * CSPLIT;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 512, "BN");
  static_assert(BN <= 256 || BN == 512, "BN above 256 must be 512");
  static_assert(kSlice % 32 == 0, "slice");
};

// Each thread of the warp reads 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// 16 outputs of one row: v[j] += residual[idx + j] (vector loads when aligned).
__device__ __forceinline__ void add_residual16(const void* base, long idx, int dtype, float (&v)[16],
                                               int valid) {
  if (dtype == 0) {
    const float* p = reinterpret_cast<const float*>(base) + idx;
    if (valid == 16 && (idx & 3) == 0) {
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        const float4 r = *reinterpret_cast<const float4*>(p + j);
        v[j] += r.x; v[j + 1] += r.y; v[j + 2] += r.z; v[j + 3] += r.w;
      }
    } else {
      for (int j = 0; j < valid; ++j) v[j] += p[j];
    }
  } else {
    const __nv_bfloat16* p = reinterpret_cast<const __nv_bfloat16*>(base) + idx;
    if (valid == 16 && (idx & 7) == 0) {
#pragma unroll
      for (int j = 0; j < 16; j += 8) {
        const uint4 r = *reinterpret_cast<const uint4*>(p + j);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          v[j + 2 * k] += __uint_as_float(w[k] << 16);
          v[j + 2 * k + 1] += __uint_as_float(w[k] & 0xffff0000u);
        }
      }
    } else {
      for (int j = 0; j < valid; ++j) v[j] += __bfloat162float(p[j]);
    }
  }
}

constexpr int kStageFloats = 32 * 36;  // one warp's 32 x 32 fp32 transpose buffer (padded rows)

// One warp stores a 32-row x 32-column fp32 block, row i held by lane i in
// v[0..31], through its shared buffer: the lanes first write their rows,
// then each store instruction covers 4 (fp32) or 8 (bf16) rows of 128 / 64
// contiguous bytes.  out row r of the block is out + (row0 + r) * ld + col0;
// rows >= M and columns >= ncols are skipped; residual (nullable) is added.
template <int OUT_BF16>
__device__ __forceinline__ void warp_store_block(float* sbuf, const float (&v)[32], int lane,
                                                 void* out, const void* residual, long ld,
                                                 long row0, int col0, long M, int ncols) {
  float4* srow = reinterpret_cast<float4*>(sbuf + lane * 36);
#pragma unroll
  for (int k = 0; k < 8; ++k) srow[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  __syncwarp();
  if constexpr (!OUT_BF16) {
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int r = it * 4 + (lane >> 3);
      const int cc = (lane & 7) * 4;
      const long m = row0 + r;
      if (m < M && col0 + cc < ncols) {
        float4 val = *reinterpret_cast<const float4*>(sbuf + r * 36 + cc);
        float* dst = reinterpret_cast<float*>(out) + m * ld + col0 + cc;
        if (col0 + cc + 4 <= ncols) {
          if (residual != nullptr) {
            const float4 rr = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(residual) + m * ld + col0 + cc);
            val.x += rr.x; val.y += rr.y; val.z += rr.z; val.w += rr.w;
          }
          *reinterpret_cast<float4*>(dst) = val;
        } else {
          const float vv[4] = {val.x, val.y, val.z, val.w};
          for (int j = 0; col0 + cc + j < ncols; ++j)
            dst[j] = vv[j] + (residual ? reinterpret_cast<const float*>(residual)[m * ld + col0 + cc + j] : 0.f);
        }
      }
    }
  } else {
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int r = it * 8 + (lane >> 2);
      const int cc = (lane & 3) * 8;
      const long m = row0 + r;
      if (m < M && col0 + cc < ncols) {
        const float4 a = *reinterpret_cast<const float4*>(sbuf + r * 36 + cc);
        const float4 b = *reinterpret_cast<const float4*>(sbuf + r * 36 + cc + 4);
        float vv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out) + m * ld + col0 + cc;
        if (col0 + cc + 8 <= ncols) {
          if (residual != nullptr) {
            const uint4 rr = *reinterpret_cast<const uint4*>(
                reinterpret_cast<const __nv_bfloat16*>(residual) + m * ld + col0 + cc);
            const uint32_t w[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              vv[2 * k] += __uint_as_float(w[k] << 16);
              vv[2 * k + 1] += __uint_as_float(w[k] & 0xffff0000u);
            }
          }
          *reinterpret_cast<uint4*>(dst) =
              make_uint4(pack_bf16x2(vv[0], vv[1]), pack_bf16x2(vv[2], vv[3]),
                         pack_bf16x2(vv[4], vv[5]), pack_bf16x2(vv[6], vv[7]));
        } else {
          for (int j = 0; col0 + cc + j < ncols; ++j) {
            const float rres = residual ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(residual)[m * ld + col0 + cc + j]) : 0.f;
            dst[j] = __float2bfloat16_rn(vv[j] + rres);
          }
        }
      }
    }
  }
  __syncwarp();
}


// int8 x ternary GEMM (A8).  Warp 0 lane 0: TMA producer; warp 1: TMEM
// owner and MMA issuer (lane 0); warps 2 .. 2+4*CSPLIT-1: epilogue, warp w
// on the 32 TMEM lanes (rows) of quadrant w % 4 and on column slice
// (w - 2) / 4 of width BN / CSPLIT.  Row-wide reductions of the
// whole-row epilogues are combined through shared memory.
template <int BN, int STAGES, int EPI, int CSPLIT>
__global__ void __launch_bounds__(GemmConfig<BN, STAGES, CSPLIT>::kThreads, 1)
    ternary_gemm_kernel(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapW, GemmParams P) {
  using Cfg = GemmConfig<BN, STAGES, CSPLIT>;
  constexpr int kPanelElems = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_base = sbase + Cfg::kBarOffset;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t done_bar = bar_base + 8u * (2 * STAGES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kBarOffset + 8 * (2 * STAGES + 1));
  float* red_a = reinterpret_cast<float*>(smem + Cfg::kRedOffset);  // [CSPLIT][128]
  float* red_b = red_a + CSPLIT * 128;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int num_panels = (P.K + kPanelElems - 1) / kPanelElems;

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
      const int kc = p * kPanelElems;
      tma_load_2d(sa, &mapA, kc, m0, full_bar(s));
#pragma unroll
      for (int h = 0; h < BN / kWBox; ++h)
        tma_load_2d(sa + Cfg::kABytes + h * kWBox * 128, &mapW, kc, n0 + h * kWBox, full_bar(s));
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t kIdesc = umma_idesc(2u, 1u, 128u, (uint32_t)Cfg::kMmaN);
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
          umma_i8(tmem + h * 256, adesc, bdesc, kIdesc, (p > 0 || kk > 0) ? 1u : 0u);
        }
      }
      umma_commit(empty_bar(s));
    }
    umma_commit(done_bar);
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int q = warp & 3;
    const int slice = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const int m = m0 + row;
    const bool live = m < P.M;
    const int cs = slice * Cfg::kSlice;  // first column of this warp's slice
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + cs;
    const bool ok = mbar_wait(done_bar, 0u, DEVFLAG_TIMEOUT_EPI);
    tc_fence_after();
    const float rs = (P.row_scale != nullptr && live) ? P.row_scale[m] : 1.0f;

    if constexpr (EPI == EPI_STORE) {
      const float f = (P.alpha != nullptr ? *P.alpha : 1.f) * rs;
      if (P.out_dtype == 2) {
        // raw int32 accumulators (bit-exact checks): straight from each lane's row
        const int ncols = min(BN, P.N - n0);
#pragma unroll 1
        for (int c0 = 0; c0 < Cfg::kSlice; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(trow + c0, r);
          if (!ok || !live) continue;
          const int col = cs + c0;
          const int valid = min(32, ncols - col);
          int* o = reinterpret_cast<int*>(P.out) + (long)m * P.ld_out + n0 + col;
          for (int j = 0; j < valid; ++j) o[j] = (int)r[j];
        }
      } else {
        // f32 / bf16: 32 x 32 blocks transposed through per-warp buffers in
        // the idle pipeline stages, so that every store is a coalesced row
        // segment (rows >= M and columns >= N are skipped inside)
        static_assert(4 * CSPLIT * kStageFloats * 4 <= STAGES * Cfg::kStageBytes, "output staging");
        float* stg = reinterpret_cast<float*>(smem) + (warp - 2) * kStageFloats;
#pragma unroll 1
        for (int c0 = 0; c0 < Cfg::kSlice; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(trow + c0, r);
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = i2f_exact((int)r[j]) * f;
          if (!ok) continue;
          if (P.out_dtype == 1)
            warp_store_block<1>(stg, v, lane, P.out, P.residual, P.ld_out, m0 + q * 32, n0 + cs + c0, P.M, P.N);
          else
            warp_store_block<0>(stg, v, lane, P.out, P.residual, P.ld_out, m0 + q * 32, n0 + cs + c0, P.M, P.N);
        }
      }
    } else if constexpr (EPI == EPI_DELTA) {
      // delta = softplus(acc * alpha * row_scale + bias) in fp32, stored
      // through the per-warp transpose buffers in the idle pipeline stages
      // (every lane takes part; rows >= M are skipped inside the store)
      static_assert(4 * CSPLIT * kStageFloats * 4 <= STAGES * Cfg::kStageBytes, "output staging");
      const float f = (P.alpha != nullptr ? *P.alpha : 1.f) * rs;
      float* stg = reinterpret_cast<float*>(smem) + (warp - 2) * kStageFloats;
#pragma unroll 1
      for (int c0 = 0; c0 < Cfg::kSlice; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + c0, r);
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = n0 + cs + c0 + j;
          v[j] = softplus_fast(fmaf(i2f_exact((int)r[j]), f, col < P.N ? __ldg(P.bias + col) : 0.f));
        }
        if (ok) warp_store_block<0>(stg, v, lane, P.out, nullptr, P.ld_out, m0 + q * 32, n0 + cs + c0, P.M, P.N);
      }
    } else if constexpr (EPI == EPI_QUANT_ROW) {
      // whole row in this tile (n0 == 0, N <= BN).  Pass 1: max|acc| in
      // integers; pass 2: u = acc * c, the codes of the int32 row and
      // sum(acc^2); the slices of a row combine both through shared memory.
      const int N = P.N;
      const bool full = N == BN;
      int maxabs = 0;
#pragma unroll 1
      for (int c0 = 0; c0 < Cfg::kSlice; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + c0, r);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (full || cs + c0 + j < N) maxabs = max(maxabs, abs((int)r[j]));
      }
      if constexpr (CSPLIT > 1) {
        red_a[slice * 128 + row] = __int_as_float(maxabs);
        named_bar_sync(1, 128 * CSPLIT);
#pragma unroll
        for (int k = 0; k < CSPLIT; ++k) maxabs = max(maxabs, __float_as_int(red_a[k * 128 + row]));
      }
      const float c = (P.alpha != nullptr ? *P.alpha : 1.f) * rs;  // u = acc * c
      const float sigma = maxabs > 0 ? __fdiv_rn(127.f, (float)maxabs) : 0.f;
      float ss = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < Cfg::kSlice; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + c0, r);
        const int col0 = cs + c0;
        float a[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          a[j] = i2f_exact((int)r[j]);
          if (full || col0 + j < N) ss = fmaf(a[j], a[j], ss);
        }
        if (!ok || !live) continue;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int col = col0 + hh * 16;
          const int valid = full ? 16 : min(16, N - col);
          if (valid > 0) {
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = a[hh * 16 + j] * c;
            store16(P.out, (long)m * P.ld_out + col, 0, v, valid);
          }
          if (col < P.ld_q) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t cb[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int jj = hh * 16 + 4 * k + j;
                cb[j] = (full || col0 + jj < N) ? code_bits(a[jj], sigma) : 0u;
              }
              w[k] = pack4(cb[0], cb[1], cb[2], cb[3]);
            }
            *reinterpret_cast<uint4*>(P.q_out + (long)m * P.ld_q + col) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if constexpr (CSPLIT > 1) {
        red_b[slice * 128 + row] = ss;
        named_bar_sync(1, 128 * CSPLIT);
        ss = 0.f;
#pragma unroll
        for (int k = 0; k < CSPLIT; ++k) ss += red_b[k * 128 + row];
      }
      if (live && slice == 0) {
        const float mu = (float)maxabs * c;
        const float r_u = 1.0f / sqrtf(c * c * (ss / (float)N) + kEpsNorm);
        P.deq_out[m] = mu * r_u / 127.f;
      }
    } else if constexpr (EPI == EPI_XPROJ_A8) {
      // columns: [0,R) dt | [R,R+Ns) B | [R+Ns,R+2Ns) C ; one slice holds the whole row
      static_assert(CSPLIT == 1, "x_proj epilogue keeps the whole row in one warp");
      const int R = P.R, Ns = P.Ns;
      int maxabs = 0;
      float ss = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < BN && c0 < R; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + c0, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (c0 + j < R) {
            const int a = (int)r[j];
            maxabs = max(maxabs, abs(a));
            const float fa = i2f_exact(a);
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
      const bool fast = (R % 16 == 0) && (Ns == 16) && (P.ld_q == R);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + c0, r);
        if (!ok || !live) continue;
        if (fast) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col = c0 + hh * 16;
            const uint32_t* rr = r + hh * 16;
            if (col < R) {
              uint32_t w[4];
#pragma unroll
              for (int k = 0; k < 4; ++k)
                w[k] = pack4(code_bits(i2f_exact((int)rr[4 * k]), sigma),
                             code_bits(i2f_exact((int)rr[4 * k + 1]), sigma),
                             code_bits(i2f_exact((int)rr[4 * k + 2]), sigma),
                             code_bits(i2f_exact((int)rr[4 * k + 3]), sigma));
              *reinterpret_cast<uint4*>(P.q_out + (long)m * P.ld_q + col) = make_uint4(w[0], w[1], w[2], w[3]);
            } else if (col < R + 2 * Ns) {
              const bool isB = col < R + Ns;
              const float cf = isB ? cB : cC;
              float4* dst = reinterpret_cast<float4*>((isB ? P.Bm : P.Cm) + (long)m * Ns);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_float4(i2f_exact((int)rr[4 * v]) * cf, i2f_exact((int)rr[4 * v + 1]) * cf,
                                     i2f_exact((int)rr[4 * v + 2]) * cf, i2f_exact((int)rr[4 * v + 3]) * cf);
            }
          }
        } else {
          for (int j = 0; j < 32; ++j) {
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
      }
      if (live && !fast)
        for (int col = R; col < P.ld_q; ++col) P.q_out[(long)m * P.ld_q + col] = 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// W1.58A16 GEMM with exact per-group weight scales ("Ternary Mamba: Grouped
// Quantization-Aware Training of W1.58A16 State Space Models", abstract):
//
//   D[m, n] = sum_g s[n, g] * sum_{k in group g} x[m, k] * w[n, k]
//
// The tensor core multiplies bf16 activations by exact ternary weights
// {-1, 0, 1} and accumulates one 128-wide K group at a time into one of two
// TMEM buffers (cols 0..BN-1 and 256..256+BN-1).  Eight epilogue warps (two
// per TMEM lane quadrant, each owning BN/2 columns) read the finished group
// from TMEM, multiply it by the fp32 group scales and add it to fp32
// register accumulators, while the MMA warp fills the other buffer with the
// next group.  The scale is thus applied in fp32 exactly as defined, not
// rounded into the bf16 operand.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int BN, int STAGES, int NEPI = 8>
struct GsConfig {
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // Ring of per-group scale rows (BN floats each), filled by the producer
  // with the group's first panel.  The producer runs at most STAGES panels
  // (STAGES/2 groups) ahead of the MMAs, which run at most two groups ahead
  // of the epilogue, so this many slots are never overwritten while read.
  static constexpr int kScaleSlots = 8;
  static_assert(kScaleSlots >= STAGES / 2 + 3, "scale ring");
  static constexpr int kScaleOffset = STAGES * kStageBytes;
  static constexpr int kBarOffset = kScaleOffset + kScaleSlots * BN * 4;
  static constexpr int kSmemBytes = 1024 + kBarOffset + 256;
  // NEPI epilogue warps: NEPI/4 per TMEM lane quadrant, each owning a
  // column slice of kHalf columns
  static constexpr int kSlices = NEPI / 4;
  static constexpr int kHalf = BN / kSlices;  // columns per epilogue warp
  static constexpr int kThreads = 64 + 32 * NEPI;
  static_assert(NEPI == 8 || NEPI == 16, "NEPI");
  // slices of whole 16-column TMEM loads (the transposed-store epilogues also
  // need whole 32-column blocks, checked where they are used)
  static_assert(BN % (16 * kSlices) == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert(NEPI * kStageFloats * 4 <= STAGES * kStageBytes, "output staging");
};

template <int BN, int STAGES, int EPI, int NEPI>
__global__ void __launch_bounds__(GsConfig<BN, STAGES, NEPI>::kThreads, 1)
    ternary_gemm_gs_kernel(const __grid_constant__ CUtensorMap mapA,
                           const __grid_constant__ CUtensorMap mapW, GemmParams P) {
  using Cfg = GsConfig<BN, STAGES, NEPI>;
  constexpr int kPanel = 64;             // bf16 elements per 128-byte panel
  constexpr int kPanelsPerGroup = 2;     // 128-element weight groups
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_base = sbase + Cfg::kBarOffset;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto pfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto pempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kBarOffset + 8 * (2 * STAGES + 4));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int n0 = blockIdx.y * BN;
  const int num_panels = (P.K + kPanel - 1) / kPanel;
  const int num_groups = (num_panels + kPanelsPerGroup - 1) / kPanelsPerGroup;
  // one 256-column accumulator buffer per group in flight: a single group
  // needs one, leaving the other half of TMEM to a second CTA on the SM
  const uint32_t tmem_cols = num_groups > 1 ? 512u : 256u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(pfull_bar(b), 1);
      mbar_init(pempty_bar(b), NEPI);
    }
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    constexpr uint32_t kTx = Cfg::kABytes + Cfg::kBBytes;
    constexpr uint32_t kScaleRow = BN * 4;
    for (int p = 0; p < num_panels; ++p) {
      const int s = p % STAGES;
      const uint32_t ph = (uint32_t)(p / STAGES) & 1u;
      if (p >= STAGES && !mbar_wait(empty_bar(s), ph ^ 1u, DEVFLAG_TIMEOUT_TMA)) break;
      const uint32_t sa = sbase + s * Cfg::kStageBytes;
      const bool first = (p % kPanelsPerGroup) == 0;
      mbar_arrive_expect_tx(full_bar(s), kTx + (first ? kScaleRow : 0u));
      const int kc = p * kPanel;
      tma_load_2d(sa, &mapA, kc, m0, full_bar(s));
      tma_load_2d(sa + Cfg::kABytes, &mapW, kc, n0, full_bar(s));
      if (first) {
        // this group's scales for the tile's columns: s_t[g][n0 .. n0+BN)
        const int grp = p / kPanelsPerGroup;
        bulk_load_1d(sbase + Cfg::kScaleOffset + (grp % Cfg::kScaleSlots) * kScaleRow,
                     P.s_t + (long)grp * P.ld_s + n0, kScaleRow, full_bar(s));
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t kIdesc = umma_idesc(1u, 1u, 128u, (uint32_t)BN);
    bool ok = true;
    int p = 0;
    for (int g = 0; g < num_groups && ok; ++g) {
      const int buf = g & 1;
      if (g >= 2) ok = mbar_wait(pempty_bar(buf), (uint32_t)((g >> 1) - 1) & 1u, DEVFLAG_TIMEOUT_MMA);
      if (!ok) break;
      tc_fence_after();
      const int p_end = min(num_panels, p + kPanelsPerGroup);
      for (int pi = 0; p < p_end; ++p, ++pi) {
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
          const uint64_t bdesc = sw128_kmajor_desc(sb + kk * 32);
          umma_bf16(tmem + buf * 256, adesc, bdesc, kIdesc, (pi > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(empty_bar(s));
      }
      umma_commit(pfull_bar(buf));
    }
  } else if (warp >= 2) {
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // column slice
    const int row = q * 32 + lane;
    const int m = m0 + row;
    const bool live = m < P.M;
    const int c_base = half * Cfg::kHalf;  // first column of this warp (tile-relative)
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + c_base;
    float acc[Cfg::kHalf];
#pragma unroll
    for (int j = 0; j < Cfg::kHalf; ++j) acc[j] = 0.f;
    bool ok = true;
    for (int g = 0; g < num_groups; ++g) {
      const int buf = g & 1;
      ok = mbar_wait(pfull_bar(buf), (uint32_t)(g >> 1) & 1u, DEVFLAG_TIMEOUT_EPI);
      if (!ok) break;
      tc_fence_after();
      // the group's scale row landed with its first panel, before the MMAs
      const float4* s4 = reinterpret_cast<const float4*>(
          smem + Cfg::kScaleOffset + (g % Cfg::kScaleSlots) * (BN * 4) + c_base * 4);
      // columns per TMEM round trip: 16, or 32 for a 32-column slice
      // (register budget of the accumulators)
      constexpr int kLd = Cfg::kHalf == 32 ? 32 : 16;
#pragma unroll
      for (int c0 = 0; c0 < Cfg::kHalf; c0 += kLd) {
        uint32_t r[kLd];
        if constexpr (kLd == 16)
          tmem_ld16(trow + buf * 256 + c0, r);
        else
          tmem_ld32(trow + buf * 256 + c0, r);
#pragma unroll
        for (int v = 0; v < kLd / 4; ++v) {
          const float4 sv = s4[c0 / 4 + v];
          acc[c0 + 4 * v + 0] = fmaf(sv.x, __uint_as_float(r[4 * v + 0]), acc[c0 + 4 * v + 0]);
          acc[c0 + 4 * v + 1] = fmaf(sv.y, __uint_as_float(r[4 * v + 1]), acc[c0 + 4 * v + 1]);
          acc[c0 + 4 * v + 2] = fmaf(sv.z, __uint_as_float(r[4 * v + 2]), acc[c0 + 4 * v + 2]);
          acc[c0 + 4 * v + 3] = fmaf(sv.w, __uint_as_float(r[4 * v + 3]), acc[c0 + 4 * v + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pempty_bar(buf));
    }
    // STORE / ROWSS with a float or bf16 output: coalesced stores through a
    // per-warp transpose buffer in the (now idle) pipeline stages.  Every
    // lane takes part (rows >= M are skipped inside the store).
    if constexpr (EPI == EPI_STORE || EPI == EPI_ROWSS || EPI == EPI_DELTA) {
      static_assert(Cfg::kHalf % 32 == 0, "transposed stores take 32-column blocks");
      const int odt = EPI == EPI_ROWSS ? 1 : EPI == EPI_DELTA ? 0 : P.out_dtype;
      if (ok && odt != 2) {
        const float rs = (live && P.row_scale != nullptr) ? P.row_scale[m] : 1.0f;
        float* stg = reinterpret_cast<float*>(smem) + (warp - 2) * kStageFloats;
        const void* res = EPI == EPI_STORE ? P.residual : nullptr;
        const int ncols = min(BN, P.N - n0);
        float ss = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < Cfg::kHalf; c0 += 32) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            v[j] = acc[c0 + j] * rs;
            if (EPI == EPI_ROWSS && c_base + c0 + j < ncols) ss = fmaf(v[j], v[j], ss);
          }
          if constexpr (EPI == EPI_DELTA) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int col = c_base + c0 + j;
              v[j] = softplus_fast(v[j] + (col < ncols ? __ldg(P.bias + n0 + col) : 0.f));
            }
          }
          if (odt == 1)
            warp_store_block<1>(stg, v, lane, P.out, res, P.ld_out, m0 + q * 32, n0 + c_base + c0, P.M, P.N);
          else
            warp_store_block<0>(stg, v, lane, P.out, res, P.ld_out, m0 + q * 32, n0 + c_base + c0, P.M, P.N);
        }
        if (EPI == EPI_ROWSS && live) P.ss_part[(long)m * (Cfg::kSlices * gridDim.y) + Cfg::kSlices * blockIdx.y + half] = ss;
      }
    }
    float ss_dt = 0.f;  // EPI_XPROJ_A16: this slice's sum of dt^2
    if (ok && live) {
      const float rs = P.row_scale != nullptr ? P.row_scale[m] : 1.0f;
      (void)rs;
      if constexpr (EPI == EPI_STORE) {
        if (P.out_dtype == 2) {
          const int ncols = min(BN, P.N - n0);
#pragma unroll
          for (int c0 = 0; c0 < Cfg::kHalf; c0 += 16) {
            const int col = c_base + c0;
            if (col >= ncols) break;
            const int valid = min(16, ncols - col);
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] = acc[c0 + j] * rs;
            const long idx = (long)m * P.ld_out + n0 + col;
            if (P.residual != nullptr) add_residual16(P.residual, idx, P.out_dtype, v, valid);
            store16(P.out, idx, P.out_dtype, v, valid);
          }
        }
      } else if constexpr (EPI == EPI_XPROJ_A16) {
        // columns [0,R) dt | [R,R+Ns) B | [R+Ns,R+2Ns) C; each column slice
        // sums the squares of the dt values it holds
        const int R = P.R, Ns = P.Ns;
        float t = 0.f;
        for (int j = 0; j < P.ss_nparts; ++j) t += P.ss_in[(long)m * P.ss_nparts + j];
        const float r_u = 1.0f / sqrtf(t / (float)P.ss_count + kEpsNorm);
#pragma unroll
        for (int j = 0; j < Cfg::kHalf; ++j) {
          const int col = c_base + j;
          const float v = acc[j] * r_u;
          if (col < R) {
            const __nv_bfloat16 b = __float2bfloat16_rn(v);
            reinterpret_cast<__nv_bfloat16*>(P.out)[(long)m * P.ld_out + col] = b;
            const float vb = __bfloat162float(b);
            ss_dt = fmaf(vb, vb, ss_dt);
          } else if (col < R + Ns) {
            P.Bm[(long)m * Ns + (col - R)] = v;
          } else if (col < R + 2 * Ns) {
            P.Cm[(long)m * Ns + (col - R - Ns)] = v;
          }
        }
      }
    }
    if constexpr (EPI == EPI_XPROJ_A16) {
      // r_dt from the slices' partial sums (the pipeline stages are idle now)
      float* red = reinterpret_cast<float*>(smem);
      red[half * 128 + row] = ss_dt;
      named_bar_sync(1, 32 * NEPI);
      if (half == 0 && ok && live) {
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < Cfg::kSlices; ++k) s += red[k * 128 + row];
        P.r_out[m] = 1.0f / sqrtf(s / (float)P.R + kEpsNorm);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace bitssm
