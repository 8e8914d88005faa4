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
// through one FMA (a and b are computed off the chain), so the B*E*16 lanes
// are scanned side by side, each walking the time axis once.
//
// DFIN: the delta_raw input already holds delta (bias added and softplus
// applied by the producer), read as is.
//
// FUSED_DT: delta_raw is not read from memory but formed here from the int8
// codes of the low-rank Delta projection (the Delta-up BitLinear):
//   delta_raw[t,e] = s_up * deq_dt[t] * sum_r W_up[e,r] * q_dt[t,r]
// as an exact int32 dot product (dp4a), so the [T, E] delta tensor never
// exists in memory.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "kernels_rows.cuh"
#include "ptx.cuh"

namespace bitssm {

constexpr int kScanN = 16;   // d_state

struct ScanParams {
  const void* u;          // [B, L, E]  (int16 when u_scale is set: u = u_i16 * u_scale[token])
  const float* u_scale;   // [B*L] nullable
  const void* delta_raw;  // [B, L, E] (unfused)
  const int8_t* q_dt;     // [B*L, ld_qdt] (fused)
  long ld_qdt;
  const float* deq_dt;    // [B*L] (fused)
  const int8_t* W_up;     // [E, ld_w] int8 {-1,0,1} (fused)
  long ld_w;
  const float* s_up;      // device scalar (fused)
  int R;                  // padded to a multiple of 16 (zero codes beyond dt_rank)
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

// Sum over the TPC threads of a channel of yp[s] (one partial per step s of
// the block), scattered so that thread g of the channel returns the total
// for step g: log2(TPC) rounds of pairwise exchange, halving the kept steps.
template <int TPC>
__device__ __forceinline__ float reduce_scatter(const float (&yp)[TPC], int g);
template <>
__device__ __forceinline__ float reduce_scatter<1>(const float (&yp)[1], int) { return yp[0]; }
template <>
__device__ __forceinline__ float reduce_scatter<2>(const float (&yp)[2], int g) {
  const bool b0 = g & 1;
  float keep = b0 ? yp[1] : yp[0];
  const float send = b0 ? yp[0] : yp[1];
  return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}
template <>
__device__ __forceinline__ float reduce_scatter<4>(const float (&yp)[4], int g) {
  const bool b1 = (g >> 1) & 1;
  float k0 = b1 ? yp[2] : yp[0];
  float k1 = b1 ? yp[3] : yp[1];
  const float s0 = b1 ? yp[0] : yp[2];
  const float s1 = b1 ? yp[1] : yp[3];
  k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
  const bool b0 = g & 1;
  float keep = b0 ? k1 : k0;
  const float send = b0 ? k0 : k1;
  return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

constexpr int kScanChunk = 16;  // time steps per staged chunk

// Shared-memory layout of one stage (one chunk of kScanChunk steps).
template <int CE, bool FUSED, typename Tu, typename Td>
struct ScanStage {
  static constexpr int kU = kScanChunk * CE * (int)sizeof(Tu);
  static constexpr int kD = FUSED ? 0 : kScanChunk * CE * (int)sizeof(Td);
  static constexpr int kBC = kScanChunk * kScanN * 4;
  static constexpr int kQ = FUSED ? kScanChunk * 128 : 0;  // dt codes, row pitch 128 B
  static constexpr int kDeq = FUSED ? kScanChunk * 4 : 0;
  // int16 u (exact in_proj accumulators) comes with a per-token scale
  static constexpr bool kI16 = std::is_same<Tu, int16_t>::value;
  static constexpr int kUs = kI16 ? kScanChunk * 4 : 0;
  static constexpr int oU = 0, oD = oU + kU, oB = oD + kD, oC = oB + kBC, oQ = oC + kBC,
                       oDeq = oQ + kQ, oUs = oDeq + kDeq;
  static constexpr int kBytes = oUs + kUs;
};

// Selective scan.  A CTA of 128 threads owns CE = 128*NPT/16 channels of one
// batch; each channel has TPC = 16/NPT consecutive lanes, lane g owning
// states g*NPT .. g*NPT+NPT-1 in registers.  Inputs are staged in chunks of
// 16 steps through a double-buffered shared-memory ring filled with cp.async
// (the copy of chunk c+1 runs while chunk c is computed; one barrier per
// chunk).  Per chunk, lane g first forms delta, delta*u and D*u for its
// 16/TPC steps (t = g, g+TPC, ...; the Delta-up dot product and the softplus
// are computed once per (token, channel), and the independent steps give
// the scheduler room to overlap them); then the 16 steps are advanced, fully
// unrolled, with the channel's lanes exchanging delta and delta*u by
// shuffles, and the per-step partial outputs are reduce-scattered so that
// lane g stores y for its own steps.  RV = number of 16-code vectors of the
// Delta-up row (dt_rank padded to 16*RV).
template <int NPT, bool FUSED, int RV, typename Tu, typename Td, typename Ty, bool DFIN = false>
__global__ void __launch_bounds__(128) selective_scan_kernel(ScanParams P) {
  constexpr int TPC = kScanN / NPT;
  constexpr int CE = 128 / TPC;
  constexpr int SPL = kScanChunk / TPC;  // steps per lane per chunk
  using St = ScanStage<CE, FUSED, Tu, Td>;
  extern __shared__ __align__(16) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int b = blockIdx.y;
  const int e0 = blockIdx.x * CE;
  const int c = tid / TPC;
  const int g = tid % TPC;
  const int e = e0 + c;
  const bool ch_ok = e < P.E;
  const int E = P.E, L = P.L;
  const long tok0 = (long)b * L;
  const int src0 = lane & ~(TPC - 1);

  // issue the copies of chunk `ch` into stage `stg`
  auto issue = [&](int ch, int stg) {
    const int t0 = ch * kScanChunk;
    const uint32_t sb = sbase + stg * St::kBytes;
    constexpr int kVecRow = CE * (int)sizeof(Tu) / 16;  // 16-byte vectors per step row
    for (int i = tid; i < kScanChunk * kVecRow; i += 128) {
      const int t = i / kVecRow, v = i - t * kVecRow;
      const int ee = e0 + v * (16 / (int)sizeof(Tu));
      const int avail = (t0 + t < L) ? max(0, min(16, (E - ee) * (int)sizeof(Tu))) : 0;
      const Tu* src = reinterpret_cast<const Tu*>(P.u) + (tok0 + min(t0 + t, L - 1)) * E + min(ee, E - 1);
      cp_async16(sb + St::oU + i * 16, src, avail);
    }
    if constexpr (!FUSED) {
      constexpr int kVecRowD = CE * (int)sizeof(Td) / 16;
      for (int i = tid; i < kScanChunk * kVecRowD; i += 128) {
        const int t = i / kVecRowD, v = i - t * kVecRowD;
        const int ee = e0 + v * (16 / (int)sizeof(Td));
        const int avail = (t0 + t < L) ? max(0, min(16, (E - ee) * (int)sizeof(Td))) : 0;
        const Td* src = reinterpret_cast<const Td*>(P.delta_raw) + (tok0 + min(t0 + t, L - 1)) * E + min(ee, E - 1);
        cp_async16(sb + St::oD + i * 16, src, avail);
      }
    }
    // B and C: kScanChunk rows of 64 bytes each, contiguous
    for (int i = tid; i < kScanChunk * 4 * 2; i += 128) {
      const int which = i / (kScanChunk * 4), j = i - which * (kScanChunk * 4);
      const int t = j / 4;
      const float* base = which ? P.Cm : P.Bm;
      const int avail = (t0 + t < L) ? 16 : 0;
      cp_async16(sb + (which ? St::oC : St::oB) + j * 16,
                 base + (tok0 + min(t0 + t, L - 1)) * kScanN + (j & 3) * 4, avail);
    }
    if constexpr (FUSED) {
      for (int i = tid; i < kScanChunk * RV; i += 128) {
        const int t = i / RV, v = i - t * RV;
        const int avail = (t0 + t < L) ? 16 : 0;
        cp_async16(sb + St::oQ + t * 128 + v * 16,
                   P.q_dt + (tok0 + min(t0 + t, L - 1)) * P.ld_qdt + v * 16, avail);
      }
      for (int t = tid; t < kScanChunk; t += 128)
        cp_async4(sb + St::oDeq + t * 4, P.deq_dt + tok0 + min(t0 + t, L - 1), (t0 + t < L) ? 4 : 0);
    }
    if constexpr (St::kUs > 0) {
      for (int t = tid; t < kScanChunk; t += 128)
        cp_async4(sb + St::oUs + t * 4, P.u_scale + tok0 + min(t0 + t, L - 1), (t0 + t < L) ? 4 : 0);
    }
  };

  // states and decay rates as pairs: the recurrence runs on the paired
  // fp32 pipe (fma.rn.f32x2 / mul.rn.f32x2), two states per instruction
  float2 A2[NPT / 2], h[NPT / 2];
#pragma unroll
  for (int j = 0; j < NPT / 2; ++j) {
    const int n = g * NPT + 2 * j;
    A2[j] = ch_ok ? make_float2(P.A[(long)e * kScanN + n] * kLog2e, P.A[(long)e * kScanN + n + 1] * kLog2e)
                  : make_float2(0.f, 0.f);
    h[j] = (ch_ok && P.h0 != nullptr)
               ? make_float2(P.h0[((long)b * E + e) * kScanN + n], P.h0[((long)b * E + e) * kScanN + n + 1])
               : make_float2(0.f, 0.f);
  }
  const float Dv = ch_ok ? P.D[e] : 0.f;
  const float bias = ch_ok ? P.bias[e] : 0.f;
  float s_up = 0.f;
  int4 wq[FUSED ? RV : 1];
  if constexpr (FUSED) {
    s_up = *P.s_up;
#pragma unroll
    for (int r = 0; r < RV; ++r)
      wq[r] = ch_ok ? __ldg(reinterpret_cast<const int4*>(P.W_up + (long)e * P.ld_w) + r)
                    : make_int4(0, 0, 0, 0);
  }
  Ty* yrow = reinterpret_cast<Ty*>(P.y) + tok0 * E + e;

  const int nchunks = (L + kScanChunk - 1) / kScanChunk;
  issue(0, 0);
  cp_async_commit();
  for (int ch = 0; ch < nchunks; ++ch) {
    cp_async_wait_all();
    __syncthreads();  // chunk ch is visible; chunk ch-1's stage is free
    if (ch + 1 < nchunks) issue(ch + 1, (ch + 1) & 1);
    cp_async_commit();
    const uint8_t* sp = smem + (ch & 1) * St::kBytes;
    const Tu* u_s = reinterpret_cast<const Tu*>(sp + St::oU);
    const float* B_s = reinterpret_cast<const float*>(sp + St::oB);
    const float* C_s = reinterpret_cast<const float*>(sp + St::oC);
    const int t0 = ch * kScanChunk;
    const int steps = min(kScanChunk, L - t0);

    // ---- delta, delta*u and D*u of this lane's steps tl = i*TPC + g
    float dl[SPL], du[SPL], Du[SPL];
#pragma unroll
    for (int i = 0; i < SPL; ++i) {
      const int tl = i * TPC + g;
      float uv;
      if constexpr (St::kUs > 0)
        uv = i2f_exact((int)u_s[tl * CE + c]) * reinterpret_cast<const float*>(sp + St::oUs)[tl];
      else
        uv = load_as_float(u_s + tl * CE + c);
      float z;
      if constexpr (FUSED) {
        const int4* qv = reinterpret_cast<const int4*>(sp + St::oQ + tl * 128);
        int acc = 0;
#pragma unroll
        for (int r = 0; r < RV; ++r) {
          const int4 q4 = qv[r];
          acc = __dp4a(wq[r].x, q4.x, acc);
          acc = __dp4a(wq[r].y, q4.y, acc);
          acc = __dp4a(wq[r].z, q4.z, acc);
          acc = __dp4a(wq[r].w, q4.w, acc);
        }
        z = fmaf(i2f_exact(acc) * s_up, reinterpret_cast<const float*>(sp + St::oDeq)[tl], bias);
      } else {
        z = load_as_float(reinterpret_cast<const Td*>(sp + St::oD) + tl * CE + c);
        if constexpr (!DFIN) z += bias;
      }
      // delta = 0 past the end: h unchanged
      if constexpr (DFIN)
        dl[i] = tl < steps ? z : 0.f;
      else
        dl[i] = tl < steps ? softplus_fast(z) : 0.f;
      du[i] = dl[i] * uv;
      Du[i] = Dv * uv;
    }
    // ---- delta and delta*u of all 16 steps of the chunk, in every lane
    float dls[kScanChunk], dus[kScanChunk];
#pragma unroll
    for (int tl = 0; tl < kScanChunk; ++tl) {
      const int i = tl / TPC, s2 = tl % TPC;
      dls[tl] = TPC > 1 ? __shfl_sync(0xffffffffu, dl[i], src0 + s2) : dl[i];
      dus[tl] = TPC > 1 ? __shfl_sync(0xffffffffu, du[i], src0 + s2) : du[i];
    }
    // ---- advance the states through the chunk.  The decay factors of step
    // tl+1 are issued before the state updates of step tl, so each exp2 has
    // a full step of independent work between it and its use.
    float ys[SPL];
    float2 a_cur[NPT / 2];
    {
      const float2 d2 = make_float2(dls[0], dls[0]);
#pragma unroll
      for (int j = 0; j < NPT / 2; ++j) {
        const float2 x = __fmul2_rn(d2, A2[j]);
        a_cur[j] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      }
    }
    float yp[TPC];
#pragma unroll
    for (int tl = 0; tl < kScanChunk; ++tl) {
      float2 a_nxt[NPT / 2];
      const float2 dn2 = make_float2(dls[tl + 1 < kScanChunk ? tl + 1 : tl], dls[tl + 1 < kScanChunk ? tl + 1 : tl]);
      const float4* Bp = reinterpret_cast<const float4*>(B_s + tl * kScanN + g * NPT);
      const float4* Cp = reinterpret_cast<const float4*>(C_s + tl * kScanN + g * NPT);
      const float2 du2 = make_float2(dus[tl], dus[tl]);
      if constexpr (NPT >= 16) {
        // 16 states: stage by stage, each stage independent across the 8
        // state pairs (delta*u*B, the state updates, the next step's decay
        // factors, then the output as four short sums) -- 1% faster here,
        // slower with 4 states per thread, where the interleaved order wins.
        float2 bu[NPT / 2];
#pragma unroll
        for (int v = 0; v < NPT / 4; ++v) {
          const float4 b4 = Bp[v];
          bu[2 * v] = __fmul2_rn(du2, make_float2(b4.x, b4.y));
          bu[2 * v + 1] = __fmul2_rn(du2, make_float2(b4.z, b4.w));
        }
#pragma unroll
        for (int j = 0; j < NPT / 2; ++j) h[j] = __ffma2_rn(a_cur[j], h[j], bu[j]);
        if (tl + 1 < kScanChunk) {
#pragma unroll
          for (int j = 0; j < NPT / 2; ++j) {
            const float2 x = __fmul2_rn(dn2, A2[j]);
            a_nxt[j] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          }
        }
        constexpr int kAcc = NPT / 2 >= 4 ? 4 : NPT / 2;
        float2 acc[kAcc];
#pragma unroll
        for (int v = 0; v < NPT / 4; ++v) {
          const float4 c4 = Cp[v];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int j = 2 * v + k;
            const float2 cc = k ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
            if (j < kAcc)
              acc[j] = __fmul2_rn(cc, h[j]);
            else
              acc[j % kAcc] = __ffma2_rn(cc, h[j], acc[j % kAcc]);
          }
        }
#pragma unroll
        for (int k = 1; k < kAcc; ++k) acc[0] = __fadd2_rn(acc[0], acc[k]);
        yp[tl % TPC] = acc[0].x + acc[0].y;
      } else {
        // Per group of four states: first the exp2s of the next step's decay
        // factors (issued a step ahead of use), then this step's state
        // updates, so the special-function and FMA pipes are fed side by side.
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int v = 0; v < NPT / 4; ++v) {
          if (tl + 1 < kScanChunk) {
            const float2 x0 = __fmul2_rn(dn2, A2[2 * v]);
            const float2 x1 = __fmul2_rn(dn2, A2[2 * v + 1]);
            a_nxt[2 * v] = make_float2(ex2_approx(x0.x), ex2_approx(x0.y));
            a_nxt[2 * v + 1] = make_float2(ex2_approx(x1.x), ex2_approx(x1.y));
          }
          const float4 b4 = Bp[v];
          const float4 c4 = Cp[v];
          h[2 * v] = __ffma2_rn(a_cur[2 * v], h[2 * v], __fmul2_rn(du2, make_float2(b4.x, b4.y)));
          h[2 * v + 1] = __ffma2_rn(a_cur[2 * v + 1], h[2 * v + 1], __fmul2_rn(du2, make_float2(b4.z, b4.w)));
          acc0 = __ffma2_rn(make_float2(c4.x, c4.y), h[2 * v], acc0);
          acc1 = __ffma2_rn(make_float2(c4.z, c4.w), h[2 * v + 1], acc1);
        }
        acc0 = __fadd2_rn(acc0, acc1);
        yp[tl % TPC] = acc0.x + acc0.y;
      }
      if (tl % TPC == TPC - 1) ys[tl / TPC] = reduce_scatter<TPC>(yp, g) + Du[tl / TPC];
      if (tl + 1 < kScanChunk) {
#pragma unroll
        for (int j = 0; j < NPT / 2; ++j) a_cur[j] = a_nxt[j];
      }
    }
    if (ch_ok) {
#pragma unroll
      for (int i = 0; i < SPL; ++i) {
        const int tl = i * TPC + g;
        if (tl < steps) store_as(yrow + (long)(t0 + tl) * E, ys[i]);
      }
    }
  }
  if (P.h_last != nullptr && ch_ok) {
#pragma unroll
    for (int j = 0; j < NPT / 2; ++j) {
      P.h_last[((long)b * E + e) * kScanN + g * NPT + 2 * j] = h[j].x;
      P.h_last[((long)b * E + e) * kScanN + g * NPT + 2 * j + 1] = h[j].y;
    }
  }
}

}  // namespace bitssm
