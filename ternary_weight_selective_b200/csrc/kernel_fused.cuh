// Fused A8 kernels around the selective scan (TriSSM README: BitSSM block,
// "an RMSNorm precedes each ternary projection"; BitNet b1.58 BitLinear):
//
//   bitssm_pre_kernel : RMSNorm + absmax int8 codes of x -> in_proj (tcgen05,
//                       int32 in TMEM) -> u = acc * s_in * deq_x and the codes
//                       of the int32 row -> x_proj (tcgen05) -> B, C, the dt
//                       codes and their factor.
//   bitssm_post_kernel: RMSNorm + absmax int8 codes of y -> out_proj
//                       (tcgen05) -> out = acc * s_out * deq_y (+ residual).
//
// One CTA owns a tile of 128 tokens.  The activation codes never leave the
// SM: worker warps write them straight into shared memory in the 128-byte-
// swizzled K-major layout the tensor core reads; only the weights arrive by
// TMA.  Outputs are written through a per-warp shared-memory transpose so
// that every global store instruction covers whole 32-byte sectors.
//
// Warp roles: warp 0 lane 0 issues the weight TMA loads; warp 1 owns TMEM
// and lane 0 issues the MMAs; warps 2..17 (16 workers) quantise the input
// rows (8 rows each) and run the epilogues, worker w on TMEM lane quadrant
// w % 4 and column slice (w - 2) / 4.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "kernel_gemm.cuh"
#include "kernels_rows.cuh"
#include "ptx.cuh"

namespace bitssm {

constexpr int kFusedWorkers = 16;
constexpr int kFusedThreads = 64 + 32 * kFusedWorkers;

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Byte offset of (row, k) in a 128-row K-major operand stored as 128-byte
// panels with the 128-byte swizzle (16-byte chunk c of row r sits at chunk
// c ^ (r % 8)): the layout a SWIZZLE_128B TMA box of 128 B x 128 rows writes.
__device__ __forceinline__ uint32_t sw128_off(int row, int kbyte) {
  const int kb = kbyte & 127;
  return (uint32_t)((kbyte >> 7) * (128 * 128) + row * 128 + ((((kb >> 4) ^ (row & 7)) << 4) | (kb & 15)));
}

// One warp stores a 32-row x 32-column block of int16 values, row i held
// by lane i as 16 words of two int16 each, through its shared buffer: rows
// of 64 bytes whose four 16-byte chunks are permuted by (row / 2) % 4 so
// that neither the row writes nor the read-back hit a bank twice; each
// store instruction covers 8 rows of 64 contiguous bytes.  Rows >= M are
// skipped.
__device__ __forceinline__ void warp_store_block_i16(uint32_t* sbuf, const uint32_t (&w)[16], int lane,
                                                     int16_t* out, long ld, long row0, int col0,
                                                     long M) {
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    *reinterpret_cast<uint4*>(sbuf + lane * 16 + ((k ^ sw) << 2)) =
        make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  __syncwarp();
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = it * 8 + (lane >> 2);
    const int k = lane & 3;  // 16-byte chunk of the row
    const long m = row0 + r;
    if (m < M)
      *reinterpret_cast<uint4*>(out + m * ld + col0 + 8 * k) =
          *reinterpret_cast<const uint4*>(sbuf + r * 16 + ((k ^ ((r >> 1) & 3)) << 2));
  }
  __syncwarp();
}

// Load EPL consecutive elements (EPL * sizeof(T) a multiple of 8 bytes, the
// address aligned to it) as floats.
template <typename T, int EPL>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[EPL]) {
  if constexpr (sizeof(T) == 4) {
#pragma unroll
    for (int k = 0; k < EPL / 4; ++k) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(p) + k);
      v[4 * k] = f.x; v[4 * k + 1] = f.y; v[4 * k + 2] = f.z; v[4 * k + 3] = f.w;
    }
  } else if constexpr (EPL % 8 == 0) {
#pragma unroll
    for (int k = 0; k < EPL / 8; ++k) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + k);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * k + 2 * j] = __uint_as_float(w[j] << 16);
        v[8 * k + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
      }
    }
  } else {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
  }
}

// Quantise the 8 rows 8*wi .. 8*wi+7 of the tile (K = 32*EPL columns, one
// warp, EPL consecutive elements per lane, RB rows loaded per batch) into
// the swizzled codes operand `a_s` (row pitch: 128-byte panels), deq into
// deq_s[row] (and deq_g when not null), and the codes also into q_g (when
// not null, row pitch ldq).
template <typename T, int EPL, int RB>
__device__ __forceinline__ void quantize_rows_to_smem(const T* __restrict__ x, long ldx, long m0,
                                                      long M, int wi, int lane, uint8_t* a_s,
                                                      float* deq_s, float* deq_g, int8_t* q_g,
                                                      long ldq) {
  constexpr int K = 32 * EPL;
  static_assert(EPL % 4 == 0, "EPL");
#pragma unroll 1
  for (int r0 = 0; r0 < 8; r0 += RB) {
    float v[RB][EPL];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      const long m = m0 + wi * 8 + r0 + b;
      if (m < M) {
        load_vec<T, EPL>(x + m * ldx + lane * EPL, v[b]);
      } else {
#pragma unroll
        for (int j = 0; j < EPL; ++j) v[b][j] = 0.f;
      }
    }
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      const int row = wi * 8 + r0 + b;
      const long m = m0 + row;
      float mx = 0.f, ss = 0.f;
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        mx = fmaxf(mx, fabsf(v[b][j]));
        ss = fmaf(v[b][j], v[b][j], ss);
      }
      mx = warp_max(mx);
      ss = warp_sum(ss);
      const float sigma = mx > 0.f ? __fdiv_rn(127.f, mx) : 0.f;
      // this lane's EPL codes are contiguous in one 16-byte chunk of the row
      uint32_t w[EPL / 4];
#pragma unroll
      for (int j0 = 0; j0 < EPL; j0 += 4)
        w[j0 / 4] = pack4(code_bits(v[b][j0], sigma), code_bits(v[b][j0 + 1], sigma),
                          code_bits(v[b][j0 + 2], sigma), code_bits(v[b][j0 + 3], sigma));
#pragma unroll
      for (int c0 = 0; c0 < EPL; c0 += 16) {
        const int k = lane * EPL + c0;
        uint8_t* dst = a_s + sw128_off(row, k);
        int8_t* gdst = (q_g != nullptr && m < M) ? q_g + m * ldq + k : nullptr;
        if constexpr (EPL >= 16) {
          const uint4 q4 = make_uint4(w[c0 / 4], w[c0 / 4 + 1], w[c0 / 4 + 2], w[c0 / 4 + 3]);
          *reinterpret_cast<uint4*>(dst) = q4;
          if (gdst) *reinterpret_cast<uint4*>(gdst) = q4;
        } else if constexpr (EPL == 8) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
          if (gdst) *reinterpret_cast<uint2*>(gdst) = make_uint2(w[0], w[1]);
        } else {
          *reinterpret_cast<uint32_t*>(dst) = w[0];
          if (gdst) *reinterpret_cast<uint32_t*>(gdst) = w[0];
        }
      }
      if (lane == 0) {
        const float r = 1.0f / sqrtf(ss / (float)K + kEpsNorm);
        const float dq = mx * r / 127.f;
        deq_s[row] = dq;
        if (deq_g != nullptr && m < M) deq_g[m] = dq;
      }
    }
  }
}

struct PreParams {
  const void* x;        // [M, d] f32 / bf16
  int M, d, E;
  int xrows;            // R + 2N
  int R, Ns;
  const float* s_in;    // device scalars
  const float* s_dt;
  const float* s_B;
  const float* s_C;
  int16_t* u;           // [M, E] int16: the exact in_proj accumulators (|acc| <= 127 d)
  float* u_scale;       // [M]: u = u * u_scale (s_in * deq_x)
  float* deq_x;         // [M] (inspection)
  float* deq_u;         // [M] (inspection)
  int8_t* q_dt;         // [M, ld_qdt]
  int ld_qdt;
  float* deq_dt;        // [M]
  float* Bm;            // [M, Ns]
  float* Cm;            // [M, Ns]
  int8_t* q_x;          // nullable: also store the codes of x [M, ld_qx]
  int ld_qx;
  int8_t* q_u;          // nullable: also store the codes of u [M, ld_qu]
  int ld_qu;
};

// Shared-memory plan of the pre kernel (bytes, 1024-aligned regions):
//   phase 1: A1 codes of x [K1P panels x 16 KB] | W_in [K1P panels x BN1*128]
//   phase 2: A2 codes of u [E/128 panels x 16 KB] | u transpose buffers
//            (reusing phase 1's space once the in_proj MMAs are done)
//   always:  W_x [E/128 panels x BN2*128] after phase 1, loaded at start
template <int BN1, int K1P, int BN2>
struct PreCfg {
  static constexpr int kA1 = K1P * 16384;
  static constexpr int kW1 = K1P * BN1 * 128;
  static constexpr int kPhase1 = kA1 + kW1;
  static constexpr int kE1P = BN1 / 128;  // x_proj K panels (E <= BN1)
  static constexpr int kA2 = kE1P * 16384;
  static constexpr int kStg = kFusedWorkers * kStageFloats * 4;
  static constexpr int kPhase2 = kA2 + kStg;
  static constexpr int kW2Off = ((kPhase1 > kPhase2 ? kPhase1 : kPhase2) + 1023) / 1024 * 1024;
  static constexpr int kW2 = kE1P * BN2 * 128;
  static constexpr int kMain = kW2Off + kW2;
  static constexpr int kAux = kMain;  // barriers, slots, row arrays
  static constexpr int kAuxBytes = 256 + 128 * 4 * 2 + 2 * 4 * 128 * 4;
  static constexpr int kSmemBytes = 1024 + kMain + kAuxBytes;
  static constexpr int kTmemCols = BN1 <= 128 ? 128 : BN1 <= 256 ? 256 : 512;
  static_assert(kSmemBytes <= 227 * 1024, "pre kernel shared memory");
};

template <typename Tx, int BN1, int K1P, int BN2>
__global__ void __launch_bounds__(kFusedThreads, 1)
    bitssm_pre_kernel(const __grid_constant__ CUtensorMap mapWin,
                      const __grid_constant__ CUtensorMap mapWx, PreParams P) {
  using Cfg = PreCfg<BN1, K1P, BN2>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* aux = smem + Cfg::kAux;
  const uint32_t bw1 = smem_u32(aux + 0);     // W_in landed (tx)
  const uint32_t ba1 = smem_u32(aux + 8);     // A1 written (16 worker arrivals)
  const uint32_t bd1 = smem_u32(aux + 16);    // in_proj MMAs done (commit)
  const uint32_t bw2 = smem_u32(aux + 24);    // W_x landed (tx)
  const uint32_t ba2 = smem_u32(aux + 32);    // A2 written (16 worker arrivals)
  const uint32_t bd2 = smem_u32(aux + 40);    // x_proj MMAs done (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux + 48);
  float* deqx_s = reinterpret_cast<float*>(aux + 256);
  float* dequ_s = deqx_s + 128;
  float* red_a = dequ_s + 128;   // [4][128]
  float* red_b = red_a + 512;    // [4][128]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long m0 = (long)blockIdx.x * 128;
  const int d = P.d, E = P.E;
  (void)d;

  if (threadIdx.x == 0) {
    mbar_init(bw1, 1);
    mbar_init(ba1, kFusedWorkers);
    mbar_init(bd1, 1);
    mbar_init(bw2, 1);
    mbar_init(ba2, kFusedWorkers);
    mbar_init(bd2, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapWin);
    tma_prefetch_desc(&mapWx);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // W_in: K1P panels of BN1 rows (boxes of <= 256 rows)
      constexpr int kBox = BN1 > 256 ? 256 : BN1;
      mbar_arrive_expect_tx(bw1, (uint32_t)Cfg::kW1);
      for (int p = 0; p < K1P; ++p)
        for (int h = 0; h < BN1 / kBox; ++h)
          tma_load_2d(sbase + Cfg::kA1 + p * BN1 * 128 + h * kBox * 128, &mapWin, p * 128, h * kBox, bw1);
      mbar_arrive_expect_tx(bw2, (uint32_t)Cfg::kW2);
      for (int p = 0; p < Cfg::kE1P; ++p)
        tma_load_2d(sbase + Cfg::kW2Off + p * BN2 * 128, &mapWx, p * 128, 0, bw2);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(bw1, 0u, DEVFLAG_TIMEOUT_MMA) && mbar_wait(ba1, 0u, DEVFLAG_TIMEOUT_MMA);
      tc_fence_after();
      if (ok) {
        constexpr int kN1 = BN1 > 256 ? 256 : BN1;
        constexpr uint32_t kId1 = umma_idesc(2u, 1u, 128u, (uint32_t)kN1);
        for (int ks = 0; ks < 4 * K1P; ++ks) {
          const int p = ks >> 2, kk = ks & 3;
          const uint64_t adesc = sw128_kmajor_desc(sbase + p * 16384 + kk * 32);
#pragma unroll
          for (int h = 0; h < BN1 / kN1; ++h) {
            const uint64_t bdesc = sw128_kmajor_desc(sbase + Cfg::kA1 + p * BN1 * 128 + h * kN1 * 128 + kk * 32);
            umma_i8(tmem + h * kN1, adesc, bdesc, kId1, ks > 0 ? 1u : 0u);
          }
        }
      }
      umma_commit(bd1);
      ok = mbar_wait(bw2, 0u, DEVFLAG_TIMEOUT_MMA) && mbar_wait(ba2, 0u, DEVFLAG_TIMEOUT_MMA);
      tc_fence_after();
      if (ok) {
        constexpr uint32_t kId2 = umma_idesc(2u, 1u, 128u, (uint32_t)BN2);
        for (int ks = 0; ks < 4 * Cfg::kE1P; ++ks) {
          const int p = ks >> 2, kk = ks & 3;
          const uint64_t adesc = sw128_kmajor_desc(sbase + p * 16384 + kk * 32);
          const uint64_t bdesc = sw128_kmajor_desc(sbase + Cfg::kW2Off + p * BN2 * 128 + kk * 32);
          umma_i8(tmem, adesc, bdesc, kId2, ks > 0 ? 1u : 0u);
        }
      }
      umma_commit(bd2);
    }
  } else {
    // ---------------- workers
    const int wi = warp - 2;          // 0..15
    const int q = warp & 3;           // TMEM lane quadrant
    const int slice = wi >> 2;        // 0..3
    const int row = q * 32 + lane;
    const long m = m0 + row;
    const bool live = m < P.M;
    // 1) codes of x into A1, deq_x into shared memory
    quantize_rows_to_smem<Tx, 4 * K1P, 4>(reinterpret_cast<const Tx*>(P.x), d, m0, P.M, wi, lane,
                                          smem, deqx_s, P.deq_x, P.q_x, P.ld_qx);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(ba1);
    // 2) in_proj epilogue: u, codes of the int32 row into A2, deq_u
    const bool ok1 = mbar_wait(bd1, 0u, DEVFLAG_TIMEOUT_EPI);
    tc_fence_after();
    named_bar_sync(1, 32 * kFusedWorkers);  // deq_x of every row visible
    constexpr int kSl = BN1 / 4;           // columns per worker
    const int cs = slice * kSl;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + cs;
    constexpr bool full = true;  // the fused path runs with E == BN1
    int maxabs = 0;
#pragma unroll 1
    for (int c0 = 0; c0 < kSl; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(trow + c0, r);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (full || cs + c0 + j < E) maxabs = max(maxabs, abs((int)r[j]));
    }
    red_a[slice * 128 + row] = __int_as_float(maxabs);
    named_bar_sync(1, 32 * kFusedWorkers);
#pragma unroll
    for (int k = 0; k < 4; ++k) maxabs = max(maxabs, __float_as_int(red_a[k * 128 + row]));
    const float c = *P.s_in * deqx_s[row];  // u = acc * c
    const float sigma = maxabs > 0 ? __fdiv_rn(127.f, (float)maxabs) : 0.f;
    float ss = 0.f;
    float* stg = reinterpret_cast<float*>(smem + Cfg::kA2) + wi * kStageFloats;
#pragma unroll 1
    for (int c0 = 0; c0 < kSl; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(trow + c0, r);
      const int col0 = cs + c0;
      float a[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        a[j] = i2f_exact((int)r[j]);
        if (full || col0 + j < E) ss = fmaf(a[j], a[j], ss);
      }
      // codes of the row into A2 (two 16-byte chunks)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t cb[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int jj = hh * 16 + 4 * k + j;
            cb[j] = (full || col0 + jj < E) ? code_bits(a[jj], sigma) : 0u;
          }
          w[k] = pack4(cb[0], cb[1], cb[2], cb[3]);
        }
        *reinterpret_cast<uint4*>(smem + sw128_off(row, col0 + hh * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
        if (P.q_u != nullptr && live)
          *reinterpret_cast<uint4*>(P.q_u + m * P.ld_qu + col0 + hh * 16) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      uint32_t uw[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) uw[j] = __byte_perm(r[2 * j], r[2 * j + 1], 0x5410);
      if (ok1) warp_store_block_i16(reinterpret_cast<uint32_t*>(stg), uw, lane, P.u, E, m0 + q * 32, col0, P.M);
    }
    red_b[slice * 128 + row] = ss;
    fence_proxy_async_smem();
    named_bar_sync(1, 32 * kFusedWorkers);
    if (lane == 0) mbar_arrive(ba2);
    ss = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) ss += red_b[k * 128 + row];
    const float deq_u = (float)maxabs * c * (1.0f / sqrtf(c * c * (ss / (float)E) + kEpsNorm)) / 127.f;
    if (slice == 0) {
      dequ_s[row] = deq_u;
      if (live) {
        P.deq_u[m] = deq_u;
        P.u_scale[m] = c;
      }
    }
    // 3) x_proj epilogue (slice-0 workers hold whole rows): dt codes, B, C
    const bool ok2 = mbar_wait(bd2, 0u, DEVFLAG_TIMEOUT_EPI);
    tc_fence_after();
    if (slice == 0) {
      const int R = P.R, Ns = P.Ns;
      const uint32_t trow2 = tmem + ((uint32_t)(q * 32) << 16);
      int mx = 0;
      float ssd = 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < BN2 && c0 < R; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow2 + c0, r);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (c0 + j < R) {
            const int av = (int)r[j];
            mx = max(mx, abs(av));
            const float fa = i2f_exact(av);
            ssd = fmaf(fa, fa, ssd);
          }
        }
      }
      const float cdt = *P.s_dt * deq_u;
      const float sg = mx > 0 ? __fdiv_rn(127.f, (float)mx) : 0.f;
      if (live && ok2) {
        const float r_dt = 1.0f / sqrtf(cdt * cdt * (ssd / (float)R) + kEpsNorm);
        P.deq_dt[m] = (float)mx * cdt * r_dt / 127.f;
      }
      const float cB = *P.s_B * deq_u, cC = *P.s_C * deq_u;
      const bool fast = (R % 16 == 0) && (Ns == 16) && (P.ld_qdt == R);
#pragma unroll 1
      for (int c0 = 0; c0 < BN2; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow2 + c0, r);
        if (!live || !ok2) continue;
        if (fast) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col = c0 + hh * 16;
            const uint32_t* rr = r + hh * 16;
            if (col < R) {
              uint32_t w[4];
#pragma unroll
              for (int k = 0; k < 4; ++k)
                w[k] = pack4(code_bits(i2f_exact((int)rr[4 * k]), sg), code_bits(i2f_exact((int)rr[4 * k + 1]), sg),
                             code_bits(i2f_exact((int)rr[4 * k + 2]), sg), code_bits(i2f_exact((int)rr[4 * k + 3]), sg));
              *reinterpret_cast<uint4*>(P.q_dt + m * P.ld_qdt + col) = make_uint4(w[0], w[1], w[2], w[3]);
            } else if (col < R + 2 * Ns) {
              const bool isB = col < R + Ns;
              const float cf = isB ? cB : cC;
              float4* dst = reinterpret_cast<float4*>((isB ? P.Bm : P.Cm) + m * Ns);
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4)
                dst[v4] = make_float4(i2f_exact((int)rr[4 * v4]) * cf, i2f_exact((int)rr[4 * v4 + 1]) * cf,
                                      i2f_exact((int)rr[4 * v4 + 2]) * cf, i2f_exact((int)rr[4 * v4 + 3]) * cf);
            }
          }
        } else {
          for (int j = 0; j < 32; ++j) {
            const int col = c0 + j;
            const int av = (int)r[j];
            if (col < R) {
              P.q_dt[m * P.ld_qdt + col] = (int8_t)(code_bits(i2f_exact(av), sg) & 0xff);
            } else if (col < R + Ns) {
              P.Bm[m * Ns + (col - R)] = i2f_exact(av) * cB;
            } else if (col < R + 2 * Ns) {
              P.Cm[m * Ns + (col - R - Ns)] = i2f_exact(av) * cC;
            }
          }
        }
      }
      if (live && !fast)
        for (int col = R; col < P.ld_qdt; ++col) P.q_dt[m * P.ld_qdt + col] = 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

struct PostParams {
  const float* y;       // [M, E] f32
  int M, E, d;
  const float* s_out;   // device scalar
  void* out;            // [M, d] f32 / bf16
  const void* residual; // nullable, like out
  float* deq_y;         // [M] (inspection)
  int8_t* q_y;          // nullable: also store the codes of y [M, ld_qy]
  int ld_qy;
};

// Shared memory of the post kernel: A codes of y [E/128 panels x 16 KB] |
// W_out [E/128 panels x BN*128]; after the MMAs the same space holds the
// output transpose buffers.
template <int BN, int KP>
struct PostCfg {
  static constexpr int kA = KP * 16384;
  static constexpr int kW = KP * BN * 128;
  static constexpr int kMain = kA + kW > kFusedWorkers * kStageFloats * 4 ? kA + kW : kFusedWorkers * kStageFloats * 4;
  static constexpr int kAuxBytes = 256 + 128 * 4;
  static constexpr int kSmemBytes = 1024 + kMain + kAuxBytes;
  static constexpr int kTmemCols = BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
  static_assert(kSmemBytes <= 227 * 1024, "post kernel shared memory");
};

template <int OUT_BF16, int BN, int KP>
__global__ void __launch_bounds__(kFusedThreads, 1)
    bitssm_post_kernel(const __grid_constant__ CUtensorMap mapW, PostParams P) {
  using Cfg = PostCfg<BN, KP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint8_t* aux = smem + Cfg::kMain;
  const uint32_t bw = smem_u32(aux + 0);
  const uint32_t ba = smem_u32(aux + 8);
  const uint32_t bd = smem_u32(aux + 16);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(aux + 24);
  float* deq_s = reinterpret_cast<float*>(aux + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long m0 = (long)blockIdx.x * 128;
  const int E = P.E, d = P.d;
  (void)E;

  if (threadIdx.x == 0) {
    mbar_init(bw, 1);
    mbar_init(ba, kFusedWorkers);
    mbar_init(bd, 1);
    fence_mbar_init();
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

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bw, (uint32_t)Cfg::kW);
      for (int p = 0; p < KP; ++p)
        tma_load_2d(sbase + Cfg::kA + p * BN * 128, &mapW, p * 128, 0, bw);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool ok = mbar_wait(bw, 0u, DEVFLAG_TIMEOUT_MMA) && mbar_wait(ba, 0u, DEVFLAG_TIMEOUT_MMA);
      tc_fence_after();
      if (ok) {
        constexpr uint32_t kId = umma_idesc(2u, 1u, 128u, (uint32_t)BN);
        for (int ks = 0; ks < 4 * KP; ++ks) {
          const int p = ks >> 2, kk = ks & 3;
          umma_i8(tmem, sw128_kmajor_desc(sbase + p * 16384 + kk * 32),
                  sw128_kmajor_desc(sbase + Cfg::kA + p * BN * 128 + kk * 32), kId, ks > 0 ? 1u : 0u);
        }
      }
      umma_commit(bd);
    }
  } else {
    const int wi = warp - 2;
    const int q = warp & 3;
    const int slice = wi >> 2;
    const int row = q * 32 + lane;
    // 1) codes of y into A
    quantize_rows_to_smem<float, 4 * KP, 4>(P.y, E, m0, P.M, wi, lane, smem, deq_s, P.deq_y, P.q_y,
                                            P.ld_qy);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(ba);
    // 2) epilogue: out = acc * s_out * deq_y (+ residual), BN/4 columns per worker
    const bool ok = mbar_wait(bd, 0u, DEVFLAG_TIMEOUT_EPI);
    tc_fence_after();
    named_bar_sync(1, 32 * kFusedWorkers);  // every worker past the MMA: A/W space reusable
    constexpr int kSl = BN / 4;
    const int cs = slice * kSl;
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16) + cs;
    const float f = *P.s_out * deq_s[row];
    float* stg = reinterpret_cast<float*>(smem) + wi * kStageFloats;
    if constexpr (kSl >= 32) {
#pragma unroll 1
      for (int c0 = 0; c0 < kSl; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(trow + c0, r);
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = i2f_exact((int)r[j]) * f;
        if (ok) warp_store_block<OUT_BF16>(stg, v, lane, P.out, P.residual, d, m0 + q * 32, cs + c0, P.M, d);
      }
    } else {
      // BN = 64: 16 columns per worker
      uint32_t r[16];
      tmem_ld16(trow, r);
      float v[32];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = i2f_exact((int)r[j]) * f;
#pragma unroll
      for (int j = 16; j < 32; ++j) v[j] = 0.f;
      if (ok) warp_store_block<OUT_BF16>(stg, v, lane, P.out, P.residual, d, m0 + q * 32, cs, P.M, min(d, cs + 16));
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
