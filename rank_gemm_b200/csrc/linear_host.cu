// linear_host.cu -- svdq_linear_host: the whole layer from host X to host Y,
// with the host<->device copies overlapped with the layer.
//
// M is cut into row slabs.  Three streams carry a slab each step: the
// library's copy-in stream moves slab i's X to the device, the caller's
// stream runs the layer (kernels 1 and 2 through svdq_linear) on slab i - 1,
// and the library's copy-out stream moves slab i - 2's Y to the host; the two
// copy directions use separate copy engines and overlap with each other and
// with the kernels.  Two device slab buffers of X and of Y alternate; events
// order each buffer's reuse.  The call is ordered on the caller's stream: its
// work starts after everything issued on `stream` before it, and everything
// issued on `stream` after it starts once the last Y slab is on the host.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "svdq.h"

namespace {

constexpr int MAX_DEVICES = 64;

struct CopyState {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t x_ready[2], x_free[2], y_ready[2], y_free[2];
};
std::mutex g_mu;
CopyState g_copy[MAX_DEVICES];

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Rows per slab: about an eighth of M, a multiple of 128 (whole row blocks of
// kernel 2), at least 128.
int slab_rows(int M) {
  const int eighth = (M + 7) / 8;
  return std::max(128, (eighth + 127) / 128 * 128);
}

bool make_state(CopyState& c) {
  if (cudaStreamCreateWithFlags(&c.in, cudaStreamNonBlocking) != cudaSuccess ||
      cudaStreamCreateWithFlags(&c.out, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&c.start, cudaEventDisableTiming) != cudaSuccess)
    return false;
  for (int b = 0; b < 2; ++b)
    if (cudaEventCreateWithFlags(&c.x_ready[b], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.x_free[b], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.y_ready[b], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c.y_free[b], cudaEventDisableTiming) != cudaSuccess)
      return false;
  c.ready = true;
  return true;
}

svdq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SVDQ_OK;
  cudaGetLastError();
  return SVDQ_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t svdq_linear_host_workspace_bytes(const svdq_weights* w, int M) {
  if (!w || M < 0) return 0;
  svdq_weights_info i;
  if (svdq_weights_view(w, &i) != SVDQ_OK) return 0;
  const size_t S = (size_t)std::min(slab_rows(M), std::max(M, 1));
  return 2 * align256(S * i.K * 2) + 2 * align256(S * i.N * 2) + align256(svdq_linear_workspace_bytes(w, (int)S));
}

svdq_status svdq_linear_host(const svdq_weights* w, int M, const void* X_host, svdq_epilogue epi, void* Y_host,
                             void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!w || (M > 0 && (!X_host || !Y_host))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  svdq_status s = svdq::handle_device_status(w);
  if (s != SVDQ_OK) return s;
  if (M == 0) return SVDQ_OK;
  if (!workspace || ws_bytes < svdq_linear_host_workspace_bytes(w, M)) return SVDQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SVDQ_ERR_ALIGNMENT;
  svdq_weights_info info;
  if ((s = svdq_weights_view(w, &info)) != SVDQ_OK) return s;
  const size_t K = (size_t)info.K, N = (size_t)info.N;
  const int S = std::min(slab_rows(M), M);
  const int n_slabs = (M + S - 1) / S;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return cuda_status(cudaErrorInvalidDevice);
  std::lock_guard<std::mutex> lk(g_mu);   // one call at a time uses a device's copy streams and events
  CopyState& c = g_copy[dev];
  if (!c.ready && !make_state(c)) return cuda_status(cudaErrorUnknown);

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* dX[2] = {ws, ws + align256((size_t)S * K * 2)};
  uint8_t* dY[2] = {dX[1] + align256((size_t)S * K * 2), dX[1] + align256((size_t)S * K * 2) + align256((size_t)S * N * 2)};
  uint8_t* lin = dY[1] + align256((size_t)S * N * 2);
  const size_t lin_bytes = ws_bytes - (size_t)(lin - ws);
  const uint8_t* xh = static_cast<const uint8_t*>(X_host);
  uint8_t* yh = static_cast<uint8_t*>(Y_host);

  cudaError_t e = cudaEventRecord(c.start, stream);   // everything earlier on `stream` comes first
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c.in, c.start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c.out, c.start, 0);
  for (int i = 0; e == cudaSuccess && i < n_slabs; ++i) {
    const int b = i & 1, rows = std::min(S, M - i * S);
    const size_t r0 = (size_t)i * S;
    // X slab i in: buffer b is free once slab i - 2's layer has read it
    if (i >= 2) e = cudaStreamWaitEvent(c.in, c.x_free[b], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(dX[b], xh + r0 * K * 2, (size_t)rows * K * 2, cudaMemcpyHostToDevice, c.in);
    if (e == cudaSuccess) e = cudaEventRecord(c.x_ready[b], c.in);
    // the layer on slab i, on the caller's stream; its Y buffer is free once
    // slab i - 2's Y has reached the host
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, c.x_ready[b], 0);
    if (e == cudaSuccess && i >= 2) e = cudaStreamWaitEvent(stream, c.y_free[b], 0);
    if (e != cudaSuccess) break;
    s = svdq_linear(w, rows, dX[b], epi, dY[b], lin, lin_bytes, stream);
    if (s != SVDQ_OK) return s;
    e = cudaEventRecord(c.x_free[b], stream);
    if (e == cudaSuccess) e = cudaEventRecord(c.y_ready[b], stream);
    // Y slab i out
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c.out, c.y_ready[b], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(yh + r0 * N * 2, dY[b], (size_t)rows * N * 2, cudaMemcpyDeviceToHost, c.out);
    if (e == cudaSuccess) e = cudaEventRecord(c.y_free[b], c.out);
  }
  // the caller's stream continues after the last copy out
  if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, c.y_free[(n_slabs - 1) & 1], 0);
  return cuda_status(e);
}

}  // extern "C"
