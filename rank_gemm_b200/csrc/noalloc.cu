// noalloc.cu -- svdq_linear_noalloc: the whole layer with its intermediates
// (qX, sX, LR) kept in a scratch array compiled into the library, for callers
// that cannot allocate device memory when they run the layer (cudaMalloc can
// synchronize the device and take milliseconds; an application that owns
// all device memory may give a plug-in no allocator).  See include/svdq.h.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "svdq.h"

namespace {

// The scratch array: one copy per GPU that loads the library, alive until the
// process exits.  Host code must not pass its name to a kernel (on the host
// the name only stands in for the symbol); the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_linear_scratch[SVDQ_NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void* g_scratch_addr[MAX_DEVICES];   // device address of g_linear_scratch, per device

}  // namespace

extern "C" svdq_status svdq_linear_noalloc(const svdq_weights* w, int M, const void* X, svdq_epilogue epi,
                                           void* Y, cudaStream_t stream) {
  // the checks of svdq_linear, in its order, before the size test
  if (!w || (M > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  svdq_status s = svdq::handle_device_status(w);   // compute capability 10.0 and the handle's device
  if (s != SVDQ_OK) return s;
  if (svdq_linear_workspace_bytes(w, M) > SVDQ_NOALLOC_SCRATCH_BYTES) return SVDQ_ERR_WORKSPACE;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  void* scratch = nullptr;
  {
    // Set-up, once per device, with that device current: look up where the
    // scratch array lives on it.  No memory is allocated here.
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_linear_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return SVDQ_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return svdq_linear(w, M, X, epi, Y, scratch, SVDQ_NOALLOC_SCRATCH_BYTES, stream);
}
