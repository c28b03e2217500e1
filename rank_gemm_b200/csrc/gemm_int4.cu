// gemm_int4.cu -- kernel 2 for INT4 (placeholder until the int8 tensor-core path lands).
#include "common.cuh"
#include "kernels.h"

namespace svdq {

cudaError_t launch_gemm_int4(const uint8_t*, const uint8_t*, const CUtensorMap&, const CUtensorMap&, K2I8Params,
                             int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace svdq
