// bitssm_forward_host: the mixer (or a residual stack) on host input and
// output buffers, with the host<->device copies overlapped with the forward.
// The contract is in include/bitssm.h.
//
// The batch is cut into chunks of whole sequences (sequences are independent:
// every stage but the scan is token-local, and the scan runs per sequence).
// Chunk i's host-to-device copy runs on one helper stream, its forward on the
// caller's stream once that copy has landed, and its device-to-host copy on a
// second helper stream once the forward is done, so the copies of chunks i+1
// and i-1 proceed while chunk i computes (PCIe moves data both ways at once).
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "bitssm.h"

namespace bitssm {
void set_last_error_message(const char* msg);
}

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxChunks = 16;

// Two helper streams and a pool of events per device, created on first use
// (with that device current) and kept for the life of the process.
struct Helpers {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, done = nullptr;
  cudaEvent_t copied[kMaxChunks] = {}, computed[kMaxChunks] = {};
  bool ready = false;
};

std::mutex g_mutex;
Helpers g_helpers[kMaxDevices];

int fail(cudaError_t e, const char* what) {
  char msg[256];
  std::snprintf(msg, sizeof(msg), "bitssm_forward_host: %s: %s", what, cudaGetErrorString(e));
  bitssm::set_last_error_message(msg);
  return BITSSM_ERR_CUDA;
}

// Called with g_mutex held.
int helpers_for_current_device(Helpers** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return BITSSM_ERR_INVALID_ARG;
  Helpers& h = g_helpers[dev];
  if (!h.ready) {
    const unsigned ef = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&h.in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&h.out, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&h.start, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&h.done, ef)) != cudaSuccess)
      return fail(e, "helper stream / event creation");
    for (int i = 0; i < kMaxChunks; ++i)
      if ((e = cudaEventCreateWithFlags(&h.copied[i], ef)) != cudaSuccess ||
          (e = cudaEventCreateWithFlags(&h.computed[i], ef)) != cudaSuccess)
        return fail(e, "helper event creation");
    h.ready = true;
  }
  *out = &h;
  return BITSSM_OK;
}

}  // namespace

extern "C" int bitssm_forward_host(const bitssm_layer* layers, int n_layers, const void* x_host,
                                   void* out_host, int B, int L, int dtype, int act_mode,
                                   void* x_dev, void* out_dev, void* ws, size_t ws_bytes,
                                   int n_chunks, void* stream) {
  if (layers == nullptr || n_layers <= 0 || B < 0 || L < 0 || n_chunks < 1 ||
      n_chunks > kMaxChunks || (dtype != BITSSM_F32 && dtype != BITSSM_BF16))
    return BITSSM_ERR_INVALID_ARG;
  if ((long)B * L == 0) return BITSSM_OK;
  if (x_host == nullptr || out_host == nullptr || x_dev == nullptr || out_dev == nullptr)
    return BITSSM_ERR_INVALID_ARG;
  const int chunks = n_chunks < B ? n_chunks : B;
  const size_t seq_bytes = (size_t)L * layers[0].d_model * (dtype == BITSSM_BF16 ? 2 : 4);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the workspace of the largest chunk, checked before anything is queued
  {
    size_t need = 0;
    int rc = bitssm_workspace_size(&layers[0], (B + chunks - 1) / chunks, L, dtype, act_mode, &need);
    if (rc != BITSSM_OK) return rc;
    if (ws == nullptr || ws_bytes < need) return BITSSM_ERR_WORKSPACE;
  }

  std::lock_guard<std::mutex> lock(g_mutex);
  Helpers* h = nullptr;
  int rc = helpers_for_current_device(&h);
  if (rc != BITSSM_OK) return rc;
  cudaError_t e;
  // everything already queued on the caller's stream comes first
  if ((e = cudaEventRecord(h->start, st)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(h->in, h->start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(h->out, h->start, 0)) != cudaSuccess)
    return fail(e, "ordering after the caller's stream");
  // chunk c holds sequences [b0(c), b0(c+1)): sizes differ by at most one
  auto b0 = [&](int c) { return (int)((long)B * c / chunks); };
  for (int c = 0; c < chunks; ++c) {
    const size_t off = (size_t)b0(c) * seq_bytes, bytes = (size_t)(b0(c + 1) - b0(c)) * seq_bytes;
    if ((e = cudaMemcpyAsync(static_cast<char*>(x_dev) + off, static_cast<const char*>(x_host) + off,
                             bytes, cudaMemcpyHostToDevice, h->in)) != cudaSuccess ||
        (e = cudaEventRecord(h->copied[c], h->in)) != cudaSuccess)
      return fail(e, "host-to-device copy");
  }
  for (int c = 0; c < chunks; ++c) {
    const int Bc = b0(c + 1) - b0(c);
    const size_t off = (size_t)b0(c) * seq_bytes, bytes = (size_t)Bc * seq_bytes;
    if ((e = cudaStreamWaitEvent(st, h->copied[c], 0)) != cudaSuccess)
      return fail(e, "wait for a chunk's input");
    const void* xc = static_cast<const char*>(x_dev) + off;
    void* oc = static_cast<char*>(out_dev) + off;
    rc = n_layers == 1
             ? bitssm_forward(&layers[0], xc, oc, nullptr, Bc, L, dtype, act_mode, ws, ws_bytes, st)
             : bitssm_stack_forward(layers, n_layers, xc, oc, Bc, L, dtype, act_mode, ws, ws_bytes, st);
    if (rc != BITSSM_OK) {
      // keep the copies already queued ordered before the caller's later work
      if (cudaEventRecord(h->done, h->in) == cudaSuccess) cudaStreamWaitEvent(st, h->done, 0);
      if (cudaEventRecord(h->done, h->out) == cudaSuccess) cudaStreamWaitEvent(st, h->done, 0);
      return rc;
    }
    if ((e = cudaEventRecord(h->computed[c], st)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(h->out, h->computed[c], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(static_cast<char*>(out_host) + off, oc, bytes, cudaMemcpyDeviceToHost,
                             h->out)) != cudaSuccess)
      return fail(e, "device-to-host copy");
  }
  // the caller's stream completes after the last copy back
  if ((e = cudaEventRecord(h->done, h->out)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(st, h->done, 0)) != cudaSuccess)
    return fail(e, "joining the caller's stream");
  return BITSSM_OK;
}
