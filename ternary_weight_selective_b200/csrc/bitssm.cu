// C ABI of the BitSSM forward library (declarations and contracts in
// include/bitssm.h): argument checks, the workspace plan, TMA descriptor
// encoding, and the launch sequence of each entry point.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bitssm.h"
#include "kernel_fused.cuh"
#include "kernel_gemm.cuh"
#include "kernel_scan.cuh"
#include "kernel_ssd.cuh"
#include "kernels_rows.cuh"
#include "ptx.cuh"

namespace bitssm {
namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }
inline int round_up(int v, int m) { return (v + m - 1) / m * m; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// Name of the last CUDA error this library saw on this thread.
thread_local char g_last_error[256] = "no error";
void note_cuda_error(cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
}
// Status of the launches enqueued since the previous check.
int launch_status() {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return BITSSM_OK;
  note_cuda_error(e);
  return BITSSM_ERR_CUDA;
}

// Opt `kern` into `bytes` of dynamic shared memory on the current device.  The
// attribute is per device, so it is set once per kernel and device (bit d of
// `done` marks device d; concurrent first calls may both set it, harmlessly).
template <typename Kern>
int set_smem_attr_once(Kern kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return launch_status();
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return BITSSM_OK;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return launch_status();
  done.fetch_or(bit, std::memory_order_release);
  return BITSSM_OK;
}

// SM count of the current device (looked up once per device).
std::atomic<int> g_num_sms[64];
int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = g_num_sms[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D K-major operand [rows, k] with row pitch `ld` elements; box = one
// 128-byte K panel x box_rows rows, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* map, const void* ptr, bool bf16, long k, long rows, long ld,
              int box_rows) {
  if (!get_encode()) return false;
  const int esz = bf16 ? 2 : 1;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) != 0 || (ld * esz) % 16 != 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * esz)};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                        2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------ GEMM launch
// kStagesWant = 0: as many pipeline stages (up to 4) as 200 KB holds.  The
// delta GEMM (K <= 128: one panel) takes two (room for the output transpose
// buffers of its 16 epilogue warps), so two CTAs share an SM and one's
// epilogue stores overlap another's loads.
template <int BN, int EPI, int kStagesWant = 0>
int launch_gemm_bn(const void* A, long lda, const void* W, long ldw, long w_rows,
                   const GemmParams& P, cudaStream_t st) {
  constexpr int kStage = 128 * 128 + BN * 128;
  constexpr int kStages =
      kStagesWant > 0 ? kStagesWant : ((200 * 1024 / kStage) >= 4 ? 4 : (200 * 1024 / kStage));
  // epilogue warps per TMEM quadrant: 128-column slices (x_proj keeps whole
  // rows); the delta GEMM, bound by its softplus epilogue, 64-column slices
  constexpr int kSplit = EPI == EPI_XPROJ_A8 ? 1
                         : EPI == EPI_DELTA  ? BN / 64
                                             : (BN >= 256 ? BN / 128 : 1);
  using Cfg = GemmConfig<BN, kStages, kSplit>;
  auto kern = ternary_gemm_kernel<BN, kStages, EPI, kSplit>;
  static std::atomic<uint64_t> attr_done{0};
  if (int rc = set_smem_attr_once(kern, Cfg::kSmemBytes, attr_done)) return rc;
  CUtensorMap mA, mW;
  if (!make_map(&mA, A, false, P.K, P.M, lda, 128)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (!make_map(&mW, W, false, P.K, w_rows, ldw, BN > 256 ? 256 : BN))
    return BITSSM_ERR_UNSUPPORTED_SHAPE;
  dim3 grid((P.M + 127) / 128, (P.N + BN - 1) / BN);
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mA, mW, P);
  return launch_status();
}

// int8 GEMM N tile: the smallest instantiated BN covering the columns the
// epilogue needs in one tile (whole-row epilogues), else 256 with N tiling.
template <int EPI>
int launch_gemm(const void* A, long lda, const void* W, long ldw, long w_rows, const GemmParams& P,
                cudaStream_t st) {
  if constexpr (EPI == EPI_DELTA) {
    if (P.K > 128) return BITSSM_ERR_UNSUPPORTED_SHAPE;
    if (P.N <= 128) return launch_gemm_bn<128, EPI, 2>(A, lda, W, ldw, w_rows, P, st);
    return launch_gemm_bn<256, EPI, 2>(A, lda, W, ldw, w_rows, P, st);
  }
  const int need = EPI == EPI_STORE ? (P.N < 256 ? P.N : 256) : P.N;
  if constexpr (EPI == EPI_STORE) {
    // at most two K panels: two stages, so that two CTAs share an SM and one
    // CTA's epilogue stores overlap the other's loads
    if (P.K <= 256) {
      if (need <= 64) return launch_gemm_bn<64, EPI, 2>(A, lda, W, ldw, w_rows, P, st);
      if (need <= 128) return launch_gemm_bn<128, EPI, 2>(A, lda, W, ldw, w_rows, P, st);
      return launch_gemm_bn<256, EPI, 2>(A, lda, W, ldw, w_rows, P, st);
    }
  }
  if (need <= 64) return launch_gemm_bn<64, EPI>(A, lda, W, ldw, w_rows, P, st);
  if (need <= 128) return launch_gemm_bn<128, EPI>(A, lda, W, ldw, w_rows, P, st);
  if (need <= 256) return launch_gemm_bn<256, EPI>(A, lda, W, ldw, w_rows, P, st);
  if constexpr (EPI == EPI_QUANT_ROW) {
    if (need <= 512) return launch_gemm_bn<512, EPI>(A, lda, W, ldw, w_rows, P, st);
  }
  return BITSSM_ERR_UNSUPPORTED_SHAPE;
}

// W1.58A16 GEMM with exact fp32 group scales (transposed scales in P.s_t).
// Epilogue warps of the group-scaled GEMM: 8 (two column slices), or 16
// (four slices of at least 32 columns) for a single 128-wide K group (STORE /
// DELTA with two stages), where the epilogue is the whole cost, when the
// stages can hold sixteen output transpose buffers (16 warps measured slower
// for the 32-group x_proj: fewer registers per thread).  The u^2 partial
// sums of ROWSS are laid out for 8.
constexpr int gs_nepi(int epi, int bn, int stages) {
  return (epi == EPI_STORE || epi == EPI_DELTA) && stages == 2 && bn >= 128 &&
                 16 * kStageFloats * 4 <= stages * (128 * 128 + bn * 128)
             ? 16
             : 8;
}

template <int BN, int EPI, int kStages>
int launch_gemm_gs_st(const void* A, long lda, const void* W, long ldw, long w_rows,
                      const GemmParams& P, cudaStream_t st) {
  constexpr int kNepi = gs_nepi(EPI, BN, kStages);
  using Cfg = GsConfig<BN, kStages, kNepi>;
  auto kern = ternary_gemm_gs_kernel<BN, kStages, EPI, kNepi>;
  static std::atomic<uint64_t> attr_done{0};
  if (int rc = set_smem_attr_once(kern, Cfg::kSmemBytes, attr_done)) return rc;
  CUtensorMap mA, mW;
  if (!make_map(&mA, A, true, P.K, P.M, lda, 128)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (!make_map(&mW, W, true, P.K, w_rows, ldw, BN)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  dim3 grid((P.M + 127) / 128, (P.N + BN - 1) / BN);
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, st>>>(mA, mW, P);
  return launch_status();
}

// Four pipeline stages; a single 128-wide K group (dt_proj) takes two, so
// that two CTAs (each with half of TMEM) share an SM.
template <int BN, int EPI>
int launch_gemm_gs_bn(const void* A, long lda, const void* W, long ldw, long w_rows,
                      const GemmParams& P, cudaStream_t st) {
  if (P.K <= 128) return launch_gemm_gs_st<BN, EPI, 2>(A, lda, W, ldw, w_rows, P, st);
  return launch_gemm_gs_st<BN, EPI, 4>(A, lda, W, ldw, w_rows, P, st);
}

// N tile of the group-scaled GEMM: whole-row epilogues need every column in
// one tile (and the dt columns within the first half).
inline int gs_bn(int N, bool whole_row) {
  const int need = whole_row ? N : (N < 256 ? N : 256);
  // a whole-row tile of up to 160 columns (x_proj at dt_rank 128, d_state 16)
  // keeps the MMA and the per-group promotion to the columns that exist
  if (whole_row && need > 128 && need <= 160) return 160;
  return need <= 64 ? 64 : need <= 128 ? 128 : 256;
}

template <int EPI>
int launch_gemm_gs(const void* A, long lda, const void* W, long ldw, long w_rows,
                   const GemmParams& P, cudaStream_t st) {
  const bool whole = EPI == EPI_XPROJ_A16;
  if (whole && P.N > 256) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  const int bn = gs_bn(P.N, whole);
  if (bn == 64) return launch_gemm_gs_bn<64, EPI>(A, lda, W, ldw, w_rows, P, st);
  if (bn == 128) return launch_gemm_gs_bn<128, EPI>(A, lda, W, ldw, w_rows, P, st);
  if constexpr (EPI == EPI_XPROJ_A16) {
    if (bn == 160) return launch_gemm_gs_bn<160, EPI>(A, lda, W, ldw, w_rows, P, st);
  }
  return launch_gemm_gs_bn<256, EPI>(A, lda, W, ldw, w_rows, P, st);
}

// Partial sums of u^2 per A16 in_proj row: one per N tile and epilogue
// column slice.
inline int rowss_parts(int E) {
  const int bn = gs_bn(E, false);
  return (gs_nepi(EPI_ROWSS, bn, 4) / 4) * ((E + bn - 1) / bn);
}

// Transposed fp32 group scales of an expanded bf16 matrix: [G][ld_s]
inline int scale_groups(int k_in) { return (k_in + 127) / 128; }
inline long scale_ld(int rows) { return (long)round_up(rows, 256); }

// ------------------------------------------------------------ row kernels
inline int rows_grid(long M) {
  long g = (M + 7) / 8;
  long cap = (long)num_sms() * 16;
  return (int)(g < cap ? (g < 1 ? 1 : g) : cap);
}

template <typename T>
bool launch_quant_rows_vec(const void* x, int M, int K, long ldx, int8_t* q, long ldq, float* deq,
                           cudaStream_t st) {
  constexpr int EPV = 16 / (int)sizeof(T);
  if (K % EPV || ldx % EPV || (reinterpret_cast<uintptr_t>(x) & 15) || (ldq % 8)) return false;
  const int vpl = (K + 32 * EPV - 1) / (32 * EPV);
  const T* xp = reinterpret_cast<const T*>(x);
  if (vpl == 1) quant_rows_vec_kernel<T, 1><<<rows_grid(M), 256, 0, st>>>(xp, M, K, ldx, q, ldq, deq);
  else if (vpl == 2) quant_rows_vec_kernel<T, 2><<<rows_grid(M), 256, 0, st>>>(xp, M, K, ldx, q, ldq, deq);
  else if (vpl <= 4) quant_rows_vec_kernel<T, 4><<<rows_grid(M), 256, 0, st>>>(xp, M, K, ldx, q, ldq, deq);
  else return false;
  return true;
}

int launch_quant_rows(const void* x, int dtype, int M, int K, long ldx, int8_t* q, long ldq,
                      float* deq, cudaStream_t st) {
  if (M == 0) return BITSSM_OK;
  const bool vec = dtype == BITSSM_F32
                       ? launch_quant_rows_vec<float>(x, M, K, ldx, q, ldq, deq, st)
                       : launch_quant_rows_vec<__nv_bfloat16>(x, M, K, ldx, q, ldq, deq, st);
  if (vec) return launch_status();
  if (dtype == BITSSM_F32)
    quant_rows_kernel<float><<<rows_grid(M), 256, 0, st>>>(reinterpret_cast<const float*>(x), M, K,
                                                           ldx, q, ldq, deq);
  else
    quant_rows_kernel<__nv_bfloat16><<<rows_grid(M), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), M, K, ldx, q, ldq, deq);
  return launch_status();
}

// Block-form row kernels: the vector forms for d_inner a multiple of 128 up
// to 512 (rows of whole 16-byte vectors, one to four per lane), else the
// scalar forms.
bool vec_rows_ok(int E, const void* a, const void* b) {
  return E % 128 == 0 && E <= 512 && (reinterpret_cast<uintptr_t>(a) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(b) & 15) == 0;
}

// Grid of the vector row kernels: about as many 256-thread blocks as fit on
// the SMs at once, each warp looping over rows (the conv kernel stages its
// taps in shared memory once per block, so short-lived blocks would repeat
// that for every eight rows).
inline int vec_rows_grid(long M, int blocks_per_sm) {
  const long g = (M + 7) / 8;
  const long cap = (long)num_sms() * blocks_per_sm;
  return (int)(g < cap ? (g < 1 ? 1 : g) : cap);
}

int launch_conv_silu_quant(const float* u_pre, int M, int L, int E, const float* w, const float* cb,
                           int K, float* u, int8_t* q, long ldq, float* deq, cudaStream_t st) {
  if (M == 0) return BITSSM_OK;
  if (vec_rows_ok(E, u_pre, u)) {
    const int g = vec_rows_grid(M, 3);
    switch (E / 128) {
      case 1: conv_silu_quant_vec_kernel<1><<<g, 256, 0, st>>>(u_pre, M, L, E, w, cb, K, u, q, ldq, deq); break;
      case 2: conv_silu_quant_vec_kernel<2><<<g, 256, 0, st>>>(u_pre, M, L, E, w, cb, K, u, q, ldq, deq); break;
      case 3: conv_silu_quant_vec_kernel<3><<<g, 256, 0, st>>>(u_pre, M, L, E, w, cb, K, u, q, ldq, deq); break;
      default: conv_silu_quant_vec_kernel<4><<<g, 256, 0, st>>>(u_pre, M, L, E, w, cb, K, u, q, ldq, deq); break;
    }
  } else {
    conv_silu_quant_kernel<<<rows_grid(M), 256, 0, st>>>(u_pre, M, L, E, w, cb, K, u, q, ldq, deq);
  }
  return launch_status();
}

int launch_gate_quant(float* y, const float* z, int M, int E, int8_t* q, long ldq, float* deq,
                      int keep, cudaStream_t st) {
  if (M == 0) return BITSSM_OK;
  if (vec_rows_ok(E, y, z)) {
    const int g = vec_rows_grid(M, 4);
    switch (E / 128) {
      case 1: gate_quant_vec_kernel<1><<<g, 256, 0, st>>>(y, z, M, E, q, ldq, deq, keep); break;
      case 2: gate_quant_vec_kernel<2><<<g, 256, 0, st>>>(y, z, M, E, q, ldq, deq, keep); break;
      case 3: gate_quant_vec_kernel<3><<<g, 256, 0, st>>>(y, z, M, E, q, ldq, deq, keep); break;
      default: gate_quant_vec_kernel<4><<<g, 256, 0, st>>>(y, z, M, E, q, ldq, deq, keep); break;
    }
  } else {
    gate_quant_kernel<<<rows_grid(M), 256, 0, st>>>(y, z, M, E, q, ldq, deq, keep);
  }
  return launch_status();
}

int launch_row_rms(const void* x, int dtype, int M, int K, long ldx, float* r, cudaStream_t st) {
  if (M == 0) return BITSSM_OK;
  const int es = dtype == BITSSM_F32 ? 4 : 2;
  if ((K * es) % 16 == 0 && (ldx * es) % 16 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0) {
    if (dtype == BITSSM_F32)
      row_rms_vec_kernel<float><<<rows_grid(M), 256, 0, st>>>(reinterpret_cast<const float*>(x), M,
                                                              K, ldx, r);
    else
      row_rms_vec_kernel<__nv_bfloat16><<<rows_grid(M), 256, 0, st>>>(
          reinterpret_cast<const __nv_bfloat16*>(x), M, K, ldx, r);
    return launch_status();
  }
  if (dtype == BITSSM_F32)
    row_rms_kernel<float><<<rows_grid(M), 256, 0, st>>>(reinterpret_cast<const float*>(x), M, K,
                                                        ldx, r);
  else
    row_rms_kernel<__nv_bfloat16><<<rows_grid(M), 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16*>(x), M, K, ldx, r);
  return launch_status();
}

int launch_expand(const ExpandJobs& jobs, bool bf16, cudaStream_t st) {
  long total = 0;
  int first[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int i = 0; i < jobs.count; ++i) {
    first[i] = (int)total;
    total += (long)jobs.job[i].n_out * (jobs.job[i].ld / (bf16 ? 8 : 16));
  }
  if (jobs.count < 8) first[jobs.count] = (int)total;
  long g = (total + 255) / 256;
  long cap = (long)num_sms() * 8;
  int grid = (int)(g < 1 ? 1 : (g < cap ? g : cap));
  if (bf16) expand_bf16_kernel<<<grid, 256, 0, st>>>(jobs);
  else
    expand_i8_kernel<<<grid, 256, 0, st>>>(jobs, make_int4(first[0], first[1], first[2], first[3]),
                                           make_int4(first[4], first[5], first[6], first[7]));
  return launch_status();
}

// ------------------------------------------------------------ scan launch
template <int NPT, bool FUSED, int RV, typename Tu, typename Td, typename Ty, bool DFIN>
int launch_scan_t(const ScanParams& P, cudaStream_t st) {
  constexpr int TPC = kScanN / NPT;
  constexpr int CE = 128 / TPC;
  constexpr int smem = 2 * ScanStage<CE, FUSED, Tu, Td>::kBytes;
  auto kern = selective_scan_kernel<NPT, FUSED, RV, Tu, Td, Ty, DFIN>;
  static std::atomic<uint64_t> attr_done{0};
  if (smem > 48 * 1024)
    if (int rc = set_smem_attr_once(kern, smem, attr_done)) return rc;
  dim3 grid((unsigned)((P.E + CE - 1) / CE), (unsigned)P.B);
  kern<<<grid, 128, smem, st>>>(P);
  return launch_status();
}

// States per thread: 16 (one thread per channel, no exchange) when there are
// enough channels to give every SM sub-partition ~1.5 warps, else 8 or 4.
// Tuning override of the states-per-thread choice (4, 8 or 16), read once
// from the environment variable BITSSM_SCAN_NPT; 0 = automatic.
int scan_npt_override() {
  static const int v = [] {
    const char* e = std::getenv("BITSSM_SCAN_NPT");
    const int n = e ? std::atoi(e) : 0;
    return (n == 4 || n == 8 || n == 16) ? n : 0;
  }();
  return v;
}

template <bool FUSED, int RV, typename Tu, typename Td, typename Ty, bool DFIN>
int launch_scan_rv(const ScanParams& P, cudaStream_t st) {
  const long channels = (long)P.B * P.E;
  const long want = (long)num_sms() * 4 * 48;
  int npt = channels >= want ? 16 : (channels * 2 >= want ? 8 : 4);
  if (DFIN) {
    // with delta read ready-made, the per-step work is the recurrence alone:
    // take the most states per thread that still gives ~3 warps per SM
    // sub-partition (measured: 4 states per thread at B*E = 16384)
    const long threads_min = (long)num_sms() * 4 * 3 * 32;
    npt = channels >= threads_min ? 16 : (channels * 2 >= threads_min ? 8 : 4);
  }
  if (DFIN) {
    // with delta read ready-made, the per-step work is the recurrence alone:
    // take the most states per thread that still gives ~3 warps per SM
    // sub-partition (measured: 4 states per thread at B*E = 16384)
    const long threads_min = (long)num_sms() * 4 * 3 * 32;
    npt = channels * 2 >= threads_min ? 8 : 4;
    if (channels >= threads_min) npt = 16;
  }
  if (scan_npt_override() != 0) npt = scan_npt_override();
  if (npt == 16) return launch_scan_t<16, FUSED, RV, Tu, Td, Ty, DFIN>(P, st);
  if (npt == 8) return launch_scan_t<8, FUSED, RV, Tu, Td, Ty, DFIN>(P, st);
  return launch_scan_t<4, FUSED, RV, Tu, Td, Ty, DFIN>(P, st);
}

template <bool FUSED, typename Tu, typename Td, typename Ty, bool DFIN = false>
int launch_scan(const ScanParams& P, cudaStream_t st) {
  if (std::is_same<Tu, int16_t>::value != (P.u_scale != nullptr)) return BITSSM_ERR_INVALID_ARG;
  if constexpr (FUSED) {
    switch (P.R / 16) {  // Delta-up width (dt_rank padded to 16)
      case 1: return launch_scan_rv<true, 1, Tu, Td, Ty, false>(P, st);
      case 2: return launch_scan_rv<true, 2, Tu, Td, Ty, false>(P, st);
      case 3: case 4: return launch_scan_rv<true, 4, Tu, Td, Ty, false>(P, st);
      default: return launch_scan_rv<true, 8, Tu, Td, Ty, false>(P, st);
    }
  }
  return launch_scan_rv<false, 1, Tu, Td, Ty, DFIN>(P, st);
}

// ------------------------------------------------------------ validation
bool tw_ok(const bitssm_tw* w) {
  return w != nullptr && w->packed != nullptr && w->scales != nullptr && w->n_out > 0 &&
         w->k_in > 0 && (w->group == 0 || w->group == 128);
}

// ------------------------------------------------------------ layer plan
struct LayerPlan {
  int T, d, E, N, R;
  int ld_d, ld_E, ld_R;    // padded K pitches (elements)
  int xrows;               // R + 2N
  bool a16;
  bool block;              // Mamba-1 block form (conv + SiLU on u, SiLU(z) gate)
  // expanded weights (offsets relative to the expanded block)
  size_t w_in, w_x, w_up, w_out, w_z, w_bytes;
  // A16: transposed fp32 group scales inside the expanded block
  size_t s_in, s_x, s_up, s_out;
  // workspace offsets (absolute; expanded block at 0 when not prepared)
  size_t base;
  bitssm_ws_view v;
  size_t ss_u;             // A16 partial sums
  int ss_parts;
  bool predelta;           // A8 fused: delta formed by a GEMM before the scan
  size_t total;
};

bool layer_shape_ok(const bitssm_layer* p, int act_mode) {
  if (p == nullptr) return false;
  const bitssm_tw* ws[6] = {&p->in_proj, &p->dt_down, &p->b_proj, &p->c_proj, &p->dt_up, &p->out_proj};
  for (auto w : ws)
    if (!tw_ok(w)) return false;
  if (p->A == nullptr || p->D == nullptr || p->dt_bias == nullptr) return false;
  const int d = p->d_model, E = p->d_inner, N = p->d_state, R = p->dt_rank;
  if (d <= 0 || E <= 0 || N <= 0 || R <= 0) return false;
  if (p->in_proj.n_out != E || p->in_proj.k_in != d) return false;
  if (p->dt_down.n_out != R || p->dt_down.k_in != E) return false;
  if (p->b_proj.n_out != N || p->b_proj.k_in != E) return false;
  if (p->c_proj.n_out != N || p->c_proj.k_in != E) return false;
  if (p->dt_up.n_out != E || p->dt_up.k_in != R) return false;
  if (p->out_proj.n_out != d || p->out_proj.k_in != E) return false;
  const int want_group = act_mode == BITSSM_A16 ? -1 : 0;
  for (auto w : ws)
    if (want_group == 0 && w->group != 0) return false;
  if (p->d_conv != 0) {  // Mamba-1 block form
    if (p->d_conv < 1 || p->d_conv > 4 || p->conv_w == nullptr || !tw_ok(&p->z_proj)) return false;
    if (p->z_proj.n_out != E || p->z_proj.k_in != d) return false;
    if (want_group == 0 && p->z_proj.group != 0) return false;
  }
  return true;
}

int layer_supported(const bitssm_layer* p, int act_mode) {
  if (p->d_state != kScanN) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (p->d_conv != 0 && act_mode != BITSSM_A8) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (p->d_model % 16 != 0 || p->d_inner % 16 != 0) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (act_mode == BITSSM_A8) {
    if (p->d_inner > 512) return BITSSM_ERR_UNSUPPORTED_SHAPE;   // whole u row in one tile
    if (p->dt_rank + 2 * p->d_state > 256) return BITSSM_ERR_UNSUPPORTED_SHAPE;
    if (round_up(p->dt_rank, 16) > 128) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  } else {
    if (p->dt_rank % 8 != 0) return BITSSM_ERR_UNSUPPORTED_SHAPE;  // bf16 TMA pitch
    if (p->dt_rank + 2 * p->d_state > 256) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  }
  return BITSSM_OK;
}

// The A8 layer runs as the fused three-kernel path for these shapes.
bool a8_fused(const LayerPlan& P) {
  return !P.block && (P.d == 128 || P.d == 256) && (P.E == 256 || P.E == 512) && P.xrows <= 64 && P.R <= 64;
}

// Fused A8 with few channels (B * E below ~96 per SM sub-partition, where the
// fused scan would take 4 states per thread): the Delta-up projection and the
// softplus run first as an int8 GEMM writing delta, and the scan reads it
// ready-made (the scan then spends its issue slots on the recurrence alone).
bool a8_predelta(const LayerPlan& P, int B) {
  const long want = (long)num_sms() * 4 * 48;
  return !P.a16 && a8_fused(P) && 2L * B * P.E < want;
}

LayerPlan plan_layer(const bitssm_layer* p, int B, int L, int act_mode, bool prepared) {
  LayerPlan P;
  std::memset(&P, 0, sizeof(P));
  P.T = B * L;
  P.d = p->d_model;
  P.E = p->d_inner;
  P.N = p->d_state;
  P.R = p->dt_rank;
  P.a16 = act_mode == BITSSM_A16;
  P.block = p->d_conv != 0;
  P.ld_d = round_up(P.d, 16);
  P.ld_E = round_up(P.E, 16);
  P.ld_R = round_up(P.R, 16);
  P.xrows = P.R + 2 * P.N;
  const size_t es = P.a16 ? 2 : 1;
  size_t o = 0;
  P.w_in = o; o = align_up(o + (size_t)P.E * P.ld_d * es);
  P.w_x = o; o = align_up(o + (size_t)P.xrows * P.ld_E * es);
  P.w_up = o; o = align_up(o + (size_t)P.E * P.ld_R * es);
  P.w_out = o; o = align_up(o + (size_t)P.d * P.ld_E * es);
  if (P.block) { P.w_z = o; o = align_up(o + (size_t)P.E * P.ld_d * es); }
  if (P.a16) {
    P.s_in = o; o = align_up(o + (size_t)scale_groups(P.d) * scale_ld(P.E) * 4);
    P.s_x = o; o = align_up(o + (size_t)scale_groups(P.E) * scale_ld(P.xrows) * 4);
    P.s_up = o; o = align_up(o + (size_t)scale_groups(P.R) * scale_ld(P.E) * 4);
    P.s_out = o; o = align_up(o + (size_t)scale_groups(P.E) * scale_ld(P.d) * 4);
  }
  P.w_bytes = o;
  size_t a = prepared ? 0 : P.w_bytes;
  const size_t T = (size_t)P.T;
  const size_t none = (size_t)-1;
  bitssm_ws_view& v = P.v;
  v.q_x = v.deq_x = v.u = v.q_u = v.deq_u = v.Bm = v.Cm = v.q_dt = v.deq_dt = v.y = v.q_y = v.deq_y = none;
  v.r_x = v.dt_low = v.r_dt = v.delta_raw = v.r_y = none;
  v.u_scale = v.delta = none;
  v.u_pre = v.z = none;
  v.u_dtype = P.a16 ? BITSSM_BF16 : BITSSM_F32;
  P.ss_u = none;
  auto take = [&](size_t bytes) {
    size_t r = a;
    a = align_up(a + bytes);
    return r;
  };
  v.ld_qx = P.ld_d;
  v.ld_qu = P.ld_E;
  v.ld_qdt = P.ld_R;
  if (!P.a16) {
    v.q_x = take(T * P.ld_d);
    v.deq_x = take(T * 4);
    v.u = take(T * P.E * 4);
    v.u_scale = take(T * 4);
    v.q_u = take(T * P.ld_E);
    v.deq_u = take(T * 4);
    v.Bm = take(T * P.N * 4);
    v.Cm = take(T * P.N * 4);
    v.q_dt = take(T * P.ld_R);
    v.deq_dt = take(T * 4);
    v.y = take(T * P.E * 4);
    v.q_y = take(T * P.ld_E);
    v.deq_y = take(T * 4);
    if (P.block) {
      v.u_pre = take(T * P.E * 4);
      v.z = take(T * P.E * 4);
    }
  } else {
    P.ss_parts = rowss_parts(P.E);
    v.r_x = take(T * 4);
    v.u = take(T * P.E * 2);
    P.ss_u = take(T * P.ss_parts * 4);
    v.dt_low = take(T * P.ld_R * 2);
    v.r_dt = take(T * 4);
    v.Bm = take(T * P.N * 4);
    v.Cm = take(T * P.N * 4);
    v.delta = take(T * P.E * 4);
    v.y = take(T * P.E * 2);
    v.r_y = take(T * 4);
  }
  P.predelta = a8_predelta(P, B);
  if (P.predelta) v.delta = take(T * P.E * 4);
  P.total = a;
  return P;
}

void fill_expand_jobs(const bitssm_layer* p, const LayerPlan& P, uint8_t* wbase, ExpandJobs& J) {
  auto job = [&](int i, const bitssm_tw& w, int row0, size_t off, int ld, size_t soff, long ld_s) {
    J.job[i].packed = w.packed;
    J.job[i].scales = w.scales;
    J.job[i].n_out = w.n_out;
    J.job[i].k_in = w.k_in;
    J.job[i].group = w.group;
    J.job[i].row0 = row0;
    J.job[i].dst = wbase + off;
    J.job[i].ld = ld;
    J.job[i].s_t = P.a16 ? reinterpret_cast<float*>(wbase + soff) : nullptr;
    J.job[i].ld_s = ld_s;
  };
  job(0, p->in_proj, 0, P.w_in, P.ld_d, P.s_in, scale_ld(P.E));
  job(1, p->dt_down, 0, P.w_x, P.ld_E, P.s_x, scale_ld(P.xrows));
  job(2, p->b_proj, P.R, P.w_x, P.ld_E, P.s_x, scale_ld(P.xrows));
  job(3, p->c_proj, P.R + P.N, P.w_x, P.ld_E, P.s_x, scale_ld(P.xrows));
  job(4, p->dt_up, 0, P.w_up, P.ld_R, P.s_up, scale_ld(P.E));
  job(5, p->out_proj, 0, P.w_out, P.ld_E, P.s_out, scale_ld(P.d));
  J.count = 6;
  if (P.block) {
    job(6, p->z_proj, 0, P.w_z, P.ld_d, 0, 0);
    J.count = 7;
  }
}

// Expansion of a layer's weights into `wbase` (A16: the padding rows of the
// transposed scales are zeroed first).
int expand_layer(const bitssm_layer* p, const LayerPlan& P, uint8_t* wbase, cudaStream_t st) {
  if (P.a16) {
    if (cudaMemsetAsync(wbase + P.s_in, 0, P.w_bytes - P.s_in, st) != cudaSuccess)
      return launch_status();
  }
  ExpandJobs J;
  std::memset(&J, 0, sizeof(J));
  fill_expand_jobs(p, P, wbase, J);
  return launch_expand(J, P.a16, st);
}

// Optional per-launch events: events[i] is recorded before the i-th kernel
// of a forward and events[count] after the last one.
struct Marks {
  void* const* ev = nullptr;
  int n = 0;
  int i = 0;
  cudaStream_t st = nullptr;
  bool failed = false;
  void mark() {
    if (ev != nullptr && i < n) {
      // Under stream capture the record must be an external event-record
      // node of the graph (so graph replays can be timed); outside capture
      // it is a plain record.
      cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
      cudaError_t e = cudaStreamIsCapturing(st, &cs);
      if (e == cudaSuccess) {
        cudaEvent_t evt = reinterpret_cast<cudaEvent_t>(ev[i]);
        e = cs == cudaStreamCaptureStatusActive
                ? cudaEventRecordWithFlags(evt, st, cudaEventRecordExternal)
                : cudaEventRecord(evt, st);
      }
      if (e != cudaSuccess) {
        note_cuda_error(e);
        failed = true;
      }
    }
    ++i;
  }
};

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(base) + off);
}

// Whether the A8 layer runs as the fused pre kernel + scan + post kernel:
// d_model of 128 or 256, d_inner of 256 or 512, dt_rank + 2 d_state <= 64.

template <typename Tx, int BN1, int K1P>
int launch_pre_t(const PreParams& Q, const void* w_in, long ld_in, const void* w_x, long ld_x,
                 int xrows, cudaStream_t st) {
  using Cfg = PreCfg<BN1, K1P, 64>;
  auto kern = bitssm_pre_kernel<Tx, BN1, K1P, 64>;
  static std::atomic<uint64_t> attr_done{0};
  if (int rc = set_smem_attr_once(kern, Cfg::kSmemBytes, attr_done)) return rc;
  CUtensorMap mWin, mWx;
  if (!make_map(&mWin, w_in, false, Q.d, Q.E, ld_in, BN1 > 256 ? 256 : BN1)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (!make_map(&mWx, w_x, false, Q.E, xrows, ld_x, 64)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  kern<<<(Q.M + 127) / 128, kFusedThreads, Cfg::kSmemBytes, st>>>(mWin, mWx, Q);
  return launch_status();
}

template <typename Tx>
int launch_pre(const PreParams& Q, const void* w_in, long ld_in, const void* w_x, long ld_x,
               int xrows, cudaStream_t st) {
  if (Q.E == 512) {
    if (Q.d == 256) return launch_pre_t<Tx, 512, 2>(Q, w_in, ld_in, w_x, ld_x, xrows, st);
    return launch_pre_t<Tx, 512, 1>(Q, w_in, ld_in, w_x, ld_x, xrows, st);
  }
  if (Q.d == 256) return launch_pre_t<Tx, 256, 2>(Q, w_in, ld_in, w_x, ld_x, xrows, st);
  return launch_pre_t<Tx, 256, 1>(Q, w_in, ld_in, w_x, ld_x, xrows, st);
}

template <int OUT_BF16, int BN, int KP>
int launch_post_t(const PostParams& Q, const void* w, long ldw, cudaStream_t st) {
  using Cfg = PostCfg<BN, KP>;
  auto kern = bitssm_post_kernel<OUT_BF16, BN, KP>;
  static std::atomic<uint64_t> attr_done{0};
  if (int rc = set_smem_attr_once(kern, Cfg::kSmemBytes, attr_done)) return rc;
  CUtensorMap mW;
  if (!make_map(&mW, w, false, Q.E, Q.d, ldw, BN)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  kern<<<(Q.M + 127) / 128, kFusedThreads, Cfg::kSmemBytes, st>>>(mW, Q);
  return launch_status();
}

template <int OUT_BF16>
int launch_post(const PostParams& Q, const void* w, long ldw, cudaStream_t st) {
  if (Q.E == 512) {
    if (Q.d == 256) return launch_post_t<OUT_BF16, 256, 4>(Q, w, ldw, st);
    return launch_post_t<OUT_BF16, 128, 4>(Q, w, ldw, st);
  }
  if (Q.d == 256) return launch_post_t<OUT_BF16, 256, 2>(Q, w, ldw, st);
  return launch_post_t<OUT_BF16, 128, 2>(Q, w, ldw, st);
}

int forward_a8_fused(const bitssm_layer* p, const LayerPlan& P, const uint8_t* wexp,
                     const void* x, void* out, const void* residual, int B, int L, int dtype,
                     void* ws, cudaStream_t st, Marks& mk, float* h) {
  const bitssm_ws_view& v = P.v;
  const bool keep = (p->flags & BITSSM_KEEP_CODES) != 0;
  int rc;
  mk.mark();
  {
    PreParams Q;
    std::memset(&Q, 0, sizeof(Q));
    Q.x = x; Q.M = P.T; Q.d = P.d; Q.E = P.E; Q.xrows = P.xrows; Q.R = P.R; Q.Ns = P.N;
    Q.s_in = p->in_proj.scales; Q.s_dt = p->dt_down.scales; Q.s_B = p->b_proj.scales;
    Q.s_C = p->c_proj.scales;
    Q.u = at<int16_t>(ws, v.u); Q.u_scale = at<float>(ws, v.u_scale);
    Q.deq_x = at<float>(ws, v.deq_x); Q.deq_u = at<float>(ws, v.deq_u);
    Q.q_dt = at<int8_t>(ws, v.q_dt); Q.ld_qdt = P.ld_R; Q.deq_dt = at<float>(ws, v.deq_dt);
    Q.Bm = at<float>(ws, v.Bm); Q.Cm = at<float>(ws, v.Cm);
    if (keep) {
      Q.q_x = at<int8_t>(ws, v.q_x); Q.ld_qx = P.ld_d;
      Q.q_u = at<int8_t>(ws, v.q_u); Q.ld_qu = P.ld_E;
    }
    rc = dtype == BITSSM_F32
             ? launch_pre<float>(Q, wexp + P.w_in, P.ld_d, wexp + P.w_x, P.ld_E, P.xrows, st)
             : launch_pre<__nv_bfloat16>(Q, wexp + P.w_in, P.ld_d, wexp + P.w_x, P.ld_E, P.xrows, st);
    if (rc) return rc;
  }
  if (P.predelta) {  // delta = softplus(s_up * deq_dt * (W_up . q_dt) + bias), int8 GEMM
    mk.mark();
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = P.T; G.N = P.E; G.K = P.ld_R;
    G.out_dtype = BITSSM_F32;
    G.alpha = p->dt_up.scales;
    G.row_scale = at<float>(ws, v.deq_dt);
    G.bias = p->dt_bias;
    G.out = at<float>(ws, v.delta); G.ld_out = P.E;
    rc = launch_gemm<EPI_DELTA>(at<int8_t>(ws, v.q_dt), P.ld_R, wexp + P.w_up, P.ld_R, P.E, G, st);
    if (rc) return rc;
  }
  mk.mark();
  {
    ScanParams S;
    std::memset(&S, 0, sizeof(S));
    S.u = at<int16_t>(ws, v.u); S.u_scale = at<float>(ws, v.u_scale);
    S.q_dt = at<int8_t>(ws, v.q_dt); S.ld_qdt = P.ld_R;
    S.deq_dt = at<float>(ws, v.deq_dt);
    S.W_up = reinterpret_cast<const int8_t*>(wexp + P.w_up); S.ld_w = P.ld_R;
    S.s_up = p->dt_up.scales;
    S.R = P.ld_R;
    S.bias = p->dt_bias; S.A = p->A; S.D = p->D;
    S.Bm = at<float>(ws, v.Bm); S.Cm = at<float>(ws, v.Cm);
    S.y = at<float>(ws, v.y);
    S.B = B; S.L = L; S.E = P.E;
    S.h0 = h; S.h_last = h;  // carried state (nullable): read, then overwritten
    if (P.predelta) {
      S.delta_raw = at<float>(ws, v.delta);  // already delta
      rc = launch_scan<false, int16_t, float, float, true>(S, st);
    } else {
      rc = launch_scan<true, int16_t, float, float>(S, st);
    }
    if (rc) return rc;
  }
  mk.mark();
  {
    PostParams Q;
    std::memset(&Q, 0, sizeof(Q));
    Q.y = at<float>(ws, v.y); Q.M = P.T; Q.E = P.E; Q.d = P.d;
    Q.s_out = p->out_proj.scales;
    Q.out = out; Q.residual = residual;
    Q.deq_y = at<float>(ws, v.deq_y);
    if (keep) { Q.q_y = at<int8_t>(ws, v.q_y); Q.ld_qy = P.ld_E; }
    rc = dtype == BITSSM_F32 ? launch_post<0>(Q, wexp + P.w_out, P.ld_E, st)
                             : launch_post<1>(Q, wexp + P.w_out, P.ld_E, st);
    if (rc) return rc;
  }
  mk.mark();
  return BITSSM_OK;
}

int forward_a8(const bitssm_layer* p, const LayerPlan& P, const uint8_t* wexp, const void* x,
               void* out, const void* residual, int B, int L, int dtype, void* ws,
               cudaStream_t st, Marks& mk, float* h) {
  const bitssm_ws_view& v = P.v;
  const int T = P.T;
  int rc;
  // a1: RMSNorm + absmax int8 codes of x
  mk.mark();
  rc = launch_quant_rows(x, dtype, T, P.d, P.d, at<int8_t>(ws, v.q_x), P.ld_d, at<float>(ws, v.deq_x), st);
  if (rc) return rc;
  if (P.block) {
    // Mamba-1 block form: the two in_proj branches on the same codes of x,
    // then u = SiLU(causal conv(u_pre)) and its codes
    for (int branch = 0; branch < 2; ++branch) {
      mk.mark();
      GemmParams G;
      std::memset(&G, 0, sizeof(G));
      G.M = T; G.N = P.E; G.K = P.d;
      G.out_dtype = BITSSM_F32;
      G.alpha = branch == 0 ? p->in_proj.scales : p->z_proj.scales;
      G.row_scale = at<float>(ws, v.deq_x);
      G.out = at<float>(ws, branch == 0 ? v.u_pre : v.z); G.ld_out = P.E;
      rc = launch_gemm<EPI_STORE>(at<int8_t>(ws, v.q_x), P.ld_d, wexp + (branch == 0 ? P.w_in : P.w_z),
                                  P.ld_d, P.E, G, st);
      if (rc) return rc;
    }
    mk.mark();
    rc = launch_conv_silu_quant(at<float>(ws, v.u_pre), T, L, P.E, p->conv_w, p->conv_b, p->d_conv,
                                at<float>(ws, v.u), at<int8_t>(ws, v.q_u), P.ld_E,
                                at<float>(ws, v.deq_u), st);
    if (rc) return rc;
  } else {
  // a2 + a3: in_proj, u = acc * s_in * deq_x, codes of u from the int32 row
  mk.mark();
  {
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.E; G.K = P.d;
    G.alpha = p->in_proj.scales;
    G.row_scale = at<float>(ws, v.deq_x);
    G.out = at<float>(ws, v.u); G.ld_out = P.E;
    G.q_out = at<int8_t>(ws, v.q_u); G.ld_q = P.ld_E;
    G.deq_out = at<float>(ws, v.deq_u);
    rc = launch_gemm<EPI_QUANT_ROW>(at<int8_t>(ws, v.q_x), P.ld_d, wexp + P.w_in, P.ld_d, P.E, G, st);
    if (rc) return rc;
  }
  }
  // a4: x_proj (Delta-down | B | C), dt codes from the int32 row
  mk.mark();
  {
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.xrows; G.K = P.E;
    G.row_scale = at<float>(ws, v.deq_u);
    G.q_out = at<int8_t>(ws, v.q_dt); G.ld_q = P.ld_R;
    G.deq_out = at<float>(ws, v.deq_dt);
    G.R = P.R; G.Ns = P.N;
    G.alpha_dt = p->dt_down.scales; G.alpha_B = p->b_proj.scales; G.alpha_C = p->c_proj.scales;
    G.Bm = at<float>(ws, v.Bm); G.Cm = at<float>(ws, v.Cm);
    rc = launch_gemm<EPI_XPROJ_A8>(at<int8_t>(ws, v.q_u), P.ld_E, wexp + P.w_x, P.ld_E, P.xrows, G, st);
    if (rc) return rc;
  }
  // a5 + a6: Delta-up + softplus fused into the selective scan
  mk.mark();
  {
    ScanParams S;
    std::memset(&S, 0, sizeof(S));
    S.u = at<float>(ws, v.u);
    S.q_dt = at<int8_t>(ws, v.q_dt); S.ld_qdt = P.ld_R;
    S.deq_dt = at<float>(ws, v.deq_dt);
    S.W_up = reinterpret_cast<const int8_t*>(wexp + P.w_up); S.ld_w = P.ld_R;
    S.s_up = p->dt_up.scales;
    S.R = P.ld_R;
    S.bias = p->dt_bias; S.A = p->A; S.D = p->D;
    S.Bm = at<float>(ws, v.Bm); S.Cm = at<float>(ws, v.Cm);
    S.y = at<float>(ws, v.y);
    S.B = B; S.L = L; S.E = P.E;
    S.h0 = h; S.h_last = h;  // carried state (nullable): read, then overwritten
    rc = launch_scan<true, float, float, float>(S, st);
    if (rc) return rc;
  }
  // a7: codes of y (block form: of the gated y * SiLU(z))
  mk.mark();
  if (P.block) {
    rc = launch_gate_quant(at<float>(ws, v.y), at<float>(ws, v.z), T, P.E, at<int8_t>(ws, v.q_y),
                           P.ld_E, at<float>(ws, v.deq_y), (p->flags & BITSSM_KEEP_CODES) ? 1 : 0, st);
  } else {
    rc = launch_quant_rows(at<float>(ws, v.y), BITSSM_F32, T, P.E, P.E, at<int8_t>(ws, v.q_y), P.ld_E,
                           at<float>(ws, v.deq_y), st);
  }
  if (rc) return rc;
  // a8: out_proj (+ residual)
  mk.mark();
  {
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.d; G.K = P.E;
    G.out_dtype = dtype;
    G.alpha = p->out_proj.scales;
    G.row_scale = at<float>(ws, v.deq_y);
    G.out = out; G.ld_out = P.d;
    G.residual = residual;
    rc = launch_gemm<EPI_STORE>(at<int8_t>(ws, v.q_y), P.ld_E, wexp + P.w_out, P.ld_E, P.d, G, st);
    if (rc) return rc;
  }
  mk.mark();
  return BITSSM_OK;
}

int forward_a16(const bitssm_layer* p, const LayerPlan& P, const uint8_t* wexp, const void* x,
                void* out, const void* residual, int B, int L, void* ws, cudaStream_t st,
                Marks& mk, float* h) {
  const bitssm_ws_view& v = P.v;
  const int T = P.T;
  int rc;
  mk.mark();
  rc = launch_row_rms(x, BITSSM_BF16, T, P.d, P.d, at<float>(ws, v.r_x), st);
  if (rc) return rc;
  mk.mark();
  {  // in_proj: u = r_x * acc (bf16) + partial sum(u^2) per N tile
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.E; G.K = P.d;
    G.row_scale = at<float>(ws, v.r_x);
    G.out = at<__nv_bfloat16>(ws, v.u); G.ld_out = P.E;
    G.ss_part = at<float>(ws, P.ss_u);
    G.s_t = reinterpret_cast<const float*>(wexp + P.s_in); G.ld_s = scale_ld(P.E);
    rc = launch_gemm_gs<EPI_ROWSS>(x, P.d, wexp + P.w_in, P.ld_d, P.E, G, st);
    if (rc) return rc;
  }
  mk.mark();
  {  // x_proj: dt_low (bf16) + r_dt, B, C
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.xrows; G.K = P.E;
    G.out = at<__nv_bfloat16>(ws, v.dt_low); G.ld_out = P.ld_R;
    G.R = P.R; G.Ns = P.N;
    G.Bm = at<float>(ws, v.Bm); G.Cm = at<float>(ws, v.Cm);
    G.ss_in = at<float>(ws, P.ss_u); G.ss_nparts = P.ss_parts; G.ss_count = P.E;
    G.r_out = at<float>(ws, v.r_dt);
    G.s_t = reinterpret_cast<const float*>(wexp + P.s_x); G.ld_s = scale_ld(P.xrows);
    rc = launch_gemm_gs<EPI_XPROJ_A16>(at<__nv_bfloat16>(ws, v.u), P.E, wexp + P.w_x, P.ld_E,
                                       P.xrows, G, st);
    if (rc) return rc;
  }
  mk.mark();
  {  // dt_proj: delta = softplus(r_dt * acc + dt_bias) (f32)
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.E; G.K = P.R;
    G.out_dtype = BITSSM_F32;
    G.row_scale = at<float>(ws, v.r_dt);
    G.bias = p->dt_bias;
    G.out = at<float>(ws, v.delta); G.ld_out = P.E;
    G.s_t = reinterpret_cast<const float*>(wexp + P.s_up); G.ld_s = scale_ld(P.E);
    rc = launch_gemm_gs<EPI_DELTA>(at<__nv_bfloat16>(ws, v.dt_low), P.ld_R, wexp + P.w_up, P.ld_R,
                                   P.E, G, st);
    if (rc) return rc;
  }
  mk.mark();
  {
    ScanParams S;
    std::memset(&S, 0, sizeof(S));
    S.u = at<__nv_bfloat16>(ws, v.u);
    S.delta_raw = at<float>(ws, v.delta);  // already delta (bias and softplus applied)
    S.bias = p->dt_bias; S.A = p->A; S.D = p->D;
    S.Bm = at<float>(ws, v.Bm); S.Cm = at<float>(ws, v.Cm);
    S.y = at<__nv_bfloat16>(ws, v.y);
    S.B = B; S.L = L; S.E = P.E;
    S.h0 = h; S.h_last = h;  // carried state (nullable): read, then overwritten
    rc = launch_scan<false, __nv_bfloat16, float, __nv_bfloat16, true>(S, st);
    if (rc) return rc;
  }
  mk.mark();
  rc = launch_row_rms(at<__nv_bfloat16>(ws, v.y), BITSSM_BF16, T, P.E, P.E, at<float>(ws, v.r_y), st);
  if (rc) return rc;
  mk.mark();
  {
    GemmParams G;
    std::memset(&G, 0, sizeof(G));
    G.M = T; G.N = P.d; G.K = P.E;
    G.out_dtype = BITSSM_BF16;
    G.row_scale = at<float>(ws, v.r_y);
    G.out = out; G.ld_out = P.d;
    G.residual = residual;
    G.s_t = reinterpret_cast<const float*>(wexp + P.s_out); G.ld_s = scale_ld(P.d);
    rc = launch_gemm_gs<EPI_STORE>(at<__nv_bfloat16>(ws, v.y), P.E, wexp + P.w_out, P.ld_E, P.d,
                                   G, st);
    if (rc) return rc;
  }
  mk.mark();
  return BITSSM_OK;
}

int check_layer_args(const bitssm_layer* p, int B, int L, int dtype, int act_mode) {
  if (act_mode != BITSSM_A8 && act_mode != BITSSM_A16) return BITSSM_ERR_INVALID_ARG;
  if (dtype != BITSSM_F32 && dtype != BITSSM_BF16) return BITSSM_ERR_INVALID_ARG;
  if (B < 0 || L < 0) return BITSSM_ERR_INVALID_ARG;
  if (!layer_shape_ok(p, act_mode)) return BITSSM_ERR_INVALID_ARG;
  if (act_mode == BITSSM_A16 && dtype != BITSSM_BF16) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if ((long)B * L > (1L << 30)) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  return layer_supported(p, act_mode);
}

}  // namespace

// Lets other translation units of this library set the message returned by
// bitssm_last_error() for a status they return.
void set_last_error_message(const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
}
}  // namespace bitssm

using namespace bitssm;

namespace bitssm {
// Self-test of the bounded-wait path: one thread waits on an mbarrier that
// nothing arrives on, with the given limit; the wait gives up and raises
// DEVFLAG_TIMEOUT_SELFTEST in the device error word, and the kernel returns.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x == 0) {
    const uint32_t b = smem_u32(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    (void)mbar_wait_for(b, 0u, DEVFLAG_TIMEOUT_SELFTEST, limit_ns);
  }
}
}  // namespace bitssm

extern "C" {

int bitssm_version(void) { return BITSSM_ABI_VERSION; }

const char* bitssm_last_error(void) { return g_last_error; }

const char* bitssm_status_string(int status) {
  switch (status) {
    case BITSSM_OK: return "ok";
    case BITSSM_ERR_INVALID_ARG: return "invalid argument";
    case BITSSM_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case BITSSM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case BITSSM_ERR_CUDA: return "CUDA error";
    case BITSSM_ERR_TIMEOUT: return "bounded device wait ran out";
    case BITSSM_ERR_DEVICE_FLAG: return "device-side check failed";
    default: return "unknown status";
  }
}

int bitssm_selftest_wait(unsigned int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return BITSSM_ERR_INVALID_ARG;
  bitssm::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(1000ull * limit_us);
  return launch_status();
}

int bitssm_device_error(unsigned int* flags, int clear) {
  if (flags == nullptr) return BITSSM_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return BITSSM_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return BITSSM_ERR_CUDA;
  *flags = v;
  if (clear) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_error_word, &z, sizeof(z)) != cudaSuccess) return BITSSM_ERR_CUDA;
  }
  return v ? BITSSM_ERR_TIMEOUT : BITSSM_OK;
}

// ---------------------------------------------------------------- packing
int bitssm_pack_workspace_size(int n_out, int k_in, int group, size_t* bytes) {
  if (bytes == nullptr || n_out <= 0 || k_in <= 0 || (group != 0 && group != 128))
    return BITSSM_ERR_INVALID_ARG;
  *bytes = group == 0 ? align_up(sizeof(double) * 1024) : 0;
  return BITSSM_OK;
}

int bitssm_pack_ternary(const float* W, int n_out, int k_in, int group, uint8_t* packed,
                        float* scales, void* ws, size_t ws_bytes, void* stream) {
  if (W == nullptr || packed == nullptr || scales == nullptr || n_out <= 0 || k_in <= 0 ||
      (group != 0 && group != 128))
    return BITSSM_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if (group == 0) {
    size_t need = 0;
    bitssm_pack_workspace_size(n_out, k_in, group, &need);
    if (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255))
      return BITSSM_ERR_WORKSPACE;
    const int nparts = 1024;
    double* parts = reinterpret_cast<double*>(ws);
    absmean_partial_kernel<<<nparts, 256, 0, st>>>(W, (long)n_out * k_in, parts);
    const long nbytes = (long)n_out * ((k_in + 3) / 4);
    long g = (nbytes + 255) / 256;
    long cap = (long)num_sms() * 8;
    pack_tensor_kernel<<<(int)(g < cap ? g : cap), 256, 0, st>>>(W, n_out, k_in, parts, nparts,
                                                                packed, scales);
  } else {
    const long groups = (long)n_out * ((k_in + group - 1) / group);
    long g = (groups + 7) / 8;
    long cap = (long)num_sms() * 16;
    pack_group_kernel<<<(int)(g < cap ? g : cap), 256, 0, st>>>(W, n_out, k_in, group, packed,
                                                               scales);
  }
  return launch_status();
}

int bitssm_check_packed(const uint8_t* packed_host, int n_out, int k_in, long* bad) {
  if (packed_host == nullptr || bad == nullptr || n_out <= 0 || k_in <= 0)
    return BITSSM_ERR_INVALID_ARG;
  const int kb = (k_in + 3) / 4;
  long count = 0;
  for (long n = 0; n < n_out; ++n)
    for (int b = 0; b < kb; ++b) {
      const unsigned byte = packed_host[n * kb + b];
      for (int i = 0; i < 4; ++i) {
        const unsigned code = (byte >> (2 * i)) & 3u;
        const bool pad = 4 * b + i >= k_in;
        if (code == 3u || (pad && code != 1u)) ++count;
      }
    }
  *bad = count;
  return count == 0 ? BITSSM_OK : BITSSM_ERR_INVALID_ARG;
}

// ---------------------------------------------------------------- BitLinear
int bitlinear_workspace_size(const bitssm_tw* w, int M, int act_mode, size_t* bytes) {
  if (bytes == nullptr || !tw_ok(w) || M < 0) return BITSSM_ERR_INVALID_ARG;
  const int ld = round_up(w->k_in, 16);
  if (act_mode == BITSSM_A8) {
    *bytes = align_up((size_t)w->n_out * ld) + align_up((size_t)M * ld) + align_up((size_t)M * 4);
  } else if (act_mode == BITSSM_A16) {
    *bytes = align_up((size_t)w->n_out * ld * 2) +
             align_up((size_t)scale_groups(w->k_in) * scale_ld(w->n_out) * 4) +
             align_up((size_t)M * 4);
  } else {
    return BITSSM_ERR_INVALID_ARG;
  }
  return BITSSM_OK;
}

int bitlinear_forward(const bitssm_tw* w, const void* x, int M, int x_dtype, void* y, int y_dtype,
                      int act_mode, void* ws, size_t ws_bytes, void* stream) {
  if (!tw_ok(w) || M < 0 || (M > 0 && (x == nullptr || y == nullptr)))
    return BITSSM_ERR_INVALID_ARG;
  if (x_dtype != BITSSM_F32 && x_dtype != BITSSM_BF16) return BITSSM_ERR_INVALID_ARG;
  if (y_dtype != BITSSM_F32 && y_dtype != BITSSM_BF16 && y_dtype != BITSSM_I32)
    return BITSSM_ERR_INVALID_ARG;
  if (act_mode != BITSSM_A8 && act_mode != BITSSM_A16) return BITSSM_ERR_INVALID_ARG;
  if (act_mode == BITSSM_A8 && w->group != 0) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (act_mode == BITSSM_A16 && (x_dtype != BITSSM_BF16 || y_dtype == BITSSM_I32 || w->k_in % 8))
    return BITSSM_ERR_UNSUPPORTED_SHAPE;
  size_t need = 0;
  bitlinear_workspace_size(w, M, act_mode, &need);
  if (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255))
    return BITSSM_ERR_WORKSPACE;
  if (M == 0) return BITSSM_OK;
  cudaStream_t st = as_stream(stream);
  const int ld = round_up(w->k_in, 16);
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  const bool a16 = act_mode == BITSSM_A16;
  const size_t w_bytes = align_up((size_t)w->n_out * ld * (a16 ? 2 : 1));
  const size_t s_bytes = a16 ? align_up((size_t)scale_groups(w->k_in) * scale_ld(w->n_out) * 4) : 0;
  ExpandJobs J;
  std::memset(&J, 0, sizeof(J));
  J.count = 1;
  J.job[0].packed = w->packed;
  J.job[0].scales = w->scales;
  J.job[0].n_out = w->n_out;
  J.job[0].k_in = w->k_in;
  J.job[0].group = w->group;
  J.job[0].row0 = 0;
  J.job[0].dst = base;
  J.job[0].ld = ld;
  if (a16) {
    J.job[0].s_t = reinterpret_cast<float*>(base + w_bytes);
    J.job[0].ld_s = scale_ld(w->n_out);
    if (cudaMemsetAsync(base + w_bytes, 0, s_bytes, st) != cudaSuccess) return launch_status();
  }
  int rc = launch_expand(J, a16, st);
  if (rc) return rc;
  GemmParams G;
  std::memset(&G, 0, sizeof(G));
  G.M = M; G.N = w->n_out; G.K = w->k_in;
  G.out = y; G.ld_out = w->n_out;
  G.out_dtype = y_dtype;
  if (!a16) {
    int8_t* q = reinterpret_cast<int8_t*>(base + w_bytes);
    float* deq = reinterpret_cast<float*>(base + w_bytes + align_up((size_t)M * ld));
    rc = launch_quant_rows(x, x_dtype, M, w->k_in, w->k_in, q, ld, deq, st);
    if (rc) return rc;
    G.alpha = w->scales;
    G.row_scale = deq;
    return launch_gemm<EPI_STORE>(q, ld, base, ld, w->n_out, G, st);
  }
  float* r = reinterpret_cast<float*>(base + w_bytes + s_bytes);
  rc = launch_row_rms(x, BITSSM_BF16, M, w->k_in, w->k_in, r, st);
  if (rc) return rc;
  G.row_scale = r;
  G.s_t = reinterpret_cast<const float*>(base + w_bytes);
  G.ld_s = scale_ld(w->n_out);
  return launch_gemm_gs<EPI_STORE>(x, w->k_in, base, ld, w->n_out, G, st);
}

// ---------------------------------------------------------------- scan
int selective_scan_forward(const void* u, const void* delta_raw, const float* delta_bias,
                           const float* A, const float* Bm, const float* Cm, const float* D,
                           const float* h0, void* y, float* h_last, int B, int L, int E, int N,
                           int dtype, void* stream) {
  if (B < 0 || L < 0 || E <= 0 || N <= 0) return BITSSM_ERR_INVALID_ARG;
  if (dtype != BITSSM_F32 && dtype != BITSSM_BF16) return BITSSM_ERR_INVALID_ARG;
  if (N != kScanN || E % 8 != 0) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0 || L == 0) {
    if (h_last != nullptr && B > 0) {
      cudaStream_t st = as_stream(stream);
      const size_t bytes = (size_t)B * E * N * sizeof(float);
      cudaError_t e = h0 != nullptr ? cudaMemcpyAsync(h_last, h0, bytes, cudaMemcpyDeviceToDevice, st)
                                    : cudaMemsetAsync(h_last, 0, bytes, st);
      return e == cudaSuccess ? BITSSM_OK : BITSSM_ERR_CUDA;
    }
    return BITSSM_OK;
  }
  if (u == nullptr || delta_raw == nullptr || delta_bias == nullptr || A == nullptr ||
      Bm == nullptr || Cm == nullptr || D == nullptr || y == nullptr)
    return BITSSM_ERR_INVALID_ARG;
  if (B > 65535) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  ScanParams S;
  std::memset(&S, 0, sizeof(S));
  S.u = u; S.delta_raw = delta_raw; S.bias = delta_bias; S.A = A; S.Bm = Bm; S.Cm = Cm; S.D = D;
  S.h0 = h0; S.y = y; S.h_last = h_last; S.B = B; S.L = L; S.E = E;
  cudaStream_t st = as_stream(stream);
  if (dtype == BITSSM_F32) return launch_scan<false, float, float, float>(S, st);
  return launch_scan<false, __nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(S, st);
}

// ---------------------------------------------------------------- SSD scan
int ssd_scan_forward(const float* x, const float* dt, const float* A, const float* Bm,
                     const float* Cm, const float* D, const float* S0, float* y, float* S_last,
                     int B, int L, int H, int P, int G, int N, void* stream) {
  if (B < 0 || L < 0 || H <= 0 || P <= 0 || G <= 0 || N <= 0 || H % G != 0)
    return BITSSM_ERR_INVALID_ARG;
  const int tpp = N / kSsdNS;
  if (N % kSsdNS != 0 || tpp > 32 || (tpp & (tpp - 1)) != 0) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  const long threads = (long)P * tpp;
  if (threads % 32 != 0 || threads > 1024 || B > 65535) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return BITSSM_OK;  // nothing to do
  if (A == nullptr) return BITSSM_ERR_INVALID_ARG;
  if (L > 0 && (x == nullptr || dt == nullptr || Bm == nullptr || Cm == nullptr || y == nullptr))
    return BITSSM_ERR_INVALID_ARG;
  const size_t smem = ssd_smem_bytes(P, N);
  if (smem > 200 * 1024) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  if (smem > 48 * 1024) {
    static std::atomic<uint64_t> attr_done{0};
    if (int rc = set_smem_attr_once(ssd_scan_kernel, (int)smem, attr_done)) return rc;
  }
  SsdParams Q;
  Q.x = x; Q.dt = dt; Q.A = A; Q.Bm = Bm; Q.Cm = Cm; Q.D = D; Q.S0 = S0; Q.y = y; Q.S_last = S_last;
  Q.B = B; Q.L = L; Q.H = H; Q.P = P; Q.G = G; Q.N = N;
  ssd_scan_kernel<<<dim3((unsigned)H, (unsigned)B), (unsigned)threads, smem, as_stream(stream)>>>(Q);
  return launch_status();
}

// ---------------------------------------------------------------- layer
int bitssm_prepared_size(const bitssm_layer* p, int act_mode, size_t* bytes) {
  if (bytes == nullptr || (act_mode != BITSSM_A8 && act_mode != BITSSM_A16) ||
      !layer_shape_ok(p, act_mode))
    return BITSSM_ERR_INVALID_ARG;
  *bytes = plan_layer(p, 1, 1, act_mode, false).w_bytes;
  return BITSSM_OK;
}

int bitssm_prepare_weights(const bitssm_layer* p, int act_mode, void* dst, size_t dst_bytes,
                           void* stream) {
  size_t need = 0;
  int rc = bitssm_prepared_size(p, act_mode, &need);
  if (rc) return rc;
  if (dst == nullptr || dst_bytes < need || (reinterpret_cast<uintptr_t>(dst) & 255))
    return BITSSM_ERR_WORKSPACE;
  LayerPlan P = plan_layer(p, 1, 1, act_mode, false);
  return expand_layer(p, P, reinterpret_cast<uint8_t*>(dst), as_stream(stream));
}

int bitssm_workspace_size(const bitssm_layer* p, int B, int L, int dtype, int act_mode,
                          size_t* bytes) {
  if (bytes == nullptr) return BITSSM_ERR_INVALID_ARG;
  int rc = check_layer_args(p, B, L, dtype, act_mode);
  if (rc) return rc;
  *bytes = plan_layer(p, B, L, act_mode, p->prepared != nullptr).total;
  return BITSSM_OK;
}

int bitssm_workspace_layout(const bitssm_layer* p, int B, int L, int dtype, int act_mode,
                            bitssm_ws_view* view) {
  if (view == nullptr) return BITSSM_ERR_INVALID_ARG;
  int rc = check_layer_args(p, B, L, dtype, act_mode);
  if (rc) return rc;
  const LayerPlan P = plan_layer(p, B, L, act_mode, p->prepared != nullptr);
  *view = P.v;
  if (act_mode == BITSSM_A8 && a8_fused(P)) {
    view->u_dtype = BITSSM_I16;
    if (!(p->flags & BITSSM_KEEP_CODES)) view->q_x = view->q_u = view->q_y = (size_t)-1;
  } else {
    view->u_scale = (size_t)-1;
  }
  return BITSSM_OK;
}

}  // extern "C"

namespace bitssm {
namespace {
int forward_impl(const bitssm_layer* p, const void* x, void* out, const void* residual, int B,
                 int L, int dtype, int act_mode, void* ws, size_t ws_bytes, void* stream,
                 Marks& mk, float* h = nullptr) {
  int rc = check_layer_args(p, B, L, dtype, act_mode);
  if (rc) return rc;
  if (h != nullptr && p->d_conv != 0) return BITSSM_ERR_UNSUPPORTED_SHAPE;
  const long T = (long)B * L;
  if (T > 0 && (x == nullptr || out == nullptr)) return BITSSM_ERR_INVALID_ARG;
  const bool prepared = p->prepared != nullptr;
  LayerPlan P = plan_layer(p, B, L, act_mode, prepared);
  if (ws == nullptr || ws_bytes < P.total || (reinterpret_cast<uintptr_t>(ws) & 255))
    return BITSSM_ERR_WORKSPACE;
  if (prepared && (reinterpret_cast<uintptr_t>(p->prepared) & 255)) return BITSSM_ERR_WORKSPACE;
  if (T == 0) return BITSSM_OK;
  cudaStream_t st = as_stream(stream);
  mk.st = st;
  const uint8_t* wexp;
  if (prepared) {
    wexp = reinterpret_cast<const uint8_t*>(p->prepared);
  } else {
    mk.mark();
    rc = expand_layer(p, P, reinterpret_cast<uint8_t*>(ws), st);
    if (rc) return rc;
    wexp = reinterpret_cast<const uint8_t*>(ws);
  }
  if (act_mode == BITSSM_A8)
    rc = a8_fused(P) ? forward_a8_fused(p, P, wexp, x, out, residual, B, L, dtype, ws, st, mk, h)
                     : forward_a8(p, P, wexp, x, out, residual, B, L, dtype, ws, st, mk, h);
  else
    rc = forward_a16(p, P, wexp, x, out, residual, B, L, ws, st, mk, h);
  if (rc == BITSSM_OK && mk.failed) rc = BITSSM_ERR_CUDA;
  return rc;
}
}  // namespace
}  // namespace bitssm

extern "C" {

int bitssm_forward(const bitssm_layer* p, const void* x, void* out, const void* residual, int B,
                   int L, int dtype, int act_mode, void* ws, size_t ws_bytes, void* stream) {
  Marks mk;
  return forward_impl(p, x, out, residual, B, L, dtype, act_mode, ws, ws_bytes, stream, mk);
}

int bitssm_forward_state(const bitssm_layer* p, const void* x, void* out, const void* residual,
                         float* h, int B, int L, int dtype, int act_mode, void* ws, size_t ws_bytes,
                         void* stream) {
  if (h == nullptr) return BITSSM_ERR_INVALID_ARG;
  Marks mk;
  return forward_impl(p, x, out, residual, B, L, dtype, act_mode, ws, ws_bytes, stream, mk, h);
}

int bitssm_step(const bitssm_layer* p, const void* x, void* out, const void* residual, float* h,
                int B, int dtype, int act_mode, void* ws, size_t ws_bytes, void* stream) {
  return bitssm_forward_state(p, x, out, residual, h, B, 1, dtype, act_mode, ws, ws_bytes, stream);
}

int bitssm_forward_launches(const bitssm_layer* p, int B, int L, int act_mode) {
  if (p == nullptr || B < 0 || L < 0 || (act_mode != BITSSM_A8 && act_mode != BITSSM_A16))
    return -1;
  const int expand = p->prepared != nullptr ? 0 : 1;
  if (act_mode == BITSSM_A16) return expand + 7;
  const LayerPlan P = plan_layer(p, B, L, act_mode, p->prepared != nullptr);
  if (P.block) return expand + 8;
  return expand + (a8_fused(P) ? (P.predelta ? 4 : 3) : 6);
}

int bitssm_forward_timed(const bitssm_layer* p, const void* x, void* out, const void* residual,
                         int B, int L, int dtype, int act_mode, void* ws, size_t ws_bytes,
                         void* const* events, int n_events, void* stream) {
  const int nl = bitssm_forward_launches(p, B, L, act_mode);
  if (nl < 0 || events == nullptr || n_events < nl + 1) return BITSSM_ERR_INVALID_ARG;
  for (int i = 0; i <= nl; ++i)
    if (events[i] == nullptr) return BITSSM_ERR_INVALID_ARG;
  Marks mk;
  mk.ev = events;
  mk.n = n_events;
  return forward_impl(p, x, out, residual, B, L, dtype, act_mode, ws, ws_bytes, stream, mk);
}

int bitssm_stack_forward(const bitssm_layer* layers, int n_layers, const void* x, void* out,
                         int B, int L, int dtype, int act_mode, void* ws, size_t ws_bytes,
                         void* stream) {
  if (layers == nullptr || n_layers <= 0) return BITSSM_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l) {
    int rc = check_layer_args(&layers[l], B, L, dtype, act_mode);
    if (rc) return rc;
    if (layers[l].d_model != layers[0].d_model || layers[l].d_inner != layers[0].d_inner ||
        layers[l].dt_rank != layers[0].dt_rank || (layers[l].d_conv != 0) != (layers[0].d_conv != 0))
      return BITSSM_ERR_INVALID_ARG;
  }
  for (int l = 0; l < n_layers; ++l) {
    const void* in = l == 0 ? x : out;
    int rc = bitssm_forward(&layers[l], in, out, in, B, L, dtype, act_mode, ws, ws_bytes, stream);
    if (rc) return rc;
  }
  return BITSSM_OK;
}

}  // extern "C"
