// act_amax.cu -- amax(|X^|) of one call's activation, X^ = X diag(lambda)^-1,
// for the per-call NVFP4 activation tensor scale (the FP32 tensor scale of
// the "SVDQuant" paper's NVFP4 setting, taken from the batch itself).
//
// One streaming pass over X: every CTA folds its share into one float32
// (kept as its bit pattern) and writes it to its own slot of `parts` (every
// slot, every call); no atomics, so nothing needs clearing between calls and
// the result does not depend on scheduling.  Kernels 1 and 2 reduce the
// slots themselves after their grid-dependency wait.  HBM-bound: 2 bytes of
// X per element.  (A NaN in X is skipped by the bf16 max, not propagated.)
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int THREADS = 512;
constexpr int UNROLL = 12;   // independent 16-byte loads in flight per thread

__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

}  // namespace

// Thread i owns column vector c = i % kv (8 columns) and rows r0 = i / kv,
// r0 + R, r0 + 2R, ...: it keeps the running max of |x| per column in bf16
// and multiplies once at the end.  That is exact: float32 rounding is
// monotone and symmetric, so max_m |fl32(x_mk * il_k)| = fl32(max_m |x_mk| *
// |il_k|) for il_k = fl32(1 / lambda_k).
__global__ void __launch_bounds__(THREADS, 2)
    act_amax_partials_kernel(const __nv_bfloat16* __restrict__ X, int M, uint32_t kv, uint32_t R,
                             const float* __restrict__ inv_lambda, uint32_t* __restrict__ parts) {
  __shared__ uint32_t red[THREADS / 32];
  grid_launch_dependents();
  grid_dependency_wait();   // X comes from the previous kernel on the stream
  const uint32_t i = blockIdx.x * THREADS + threadIdx.x;
  uint32_t m = 0;
  if (i < kv * R) {
    const uint32_t c = i % kv, r0 = i / kv;
    const uint4* xv = reinterpret_cast<const uint4*>(X) + c;
    uint4 mx = make_uint4(0u, 0u, 0u, 0u);   // bit patterns of non-negative bf16 pairs
    for (uint32_t r = r0; r < (uint32_t)M; r += UNROLL * R) {
      uint4 x[UNROLL];
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        const uint32_t rr = r + u * R;
        x[u] = rr < (uint32_t)M ? __ldg(xv + (size_t)rr * kv) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < UNROLL; ++u) {
        mx.x = max_bf16x2(mx.x, x[u].x & 0x7FFF7FFFu);
        mx.y = max_bf16x2(mx.y, x[u].y & 0x7FFF7FFFu);
        mx.z = max_bf16x2(mx.z, x[u].z & 0x7FFF7FFFu);
        mx.w = max_bf16x2(mx.w, x[u].w & 0x7FFF7FFFu);
      }
    }
    const float4 a = __ldg(reinterpret_cast<const float4*>(inv_lambda + 8 * c));
    const float4 b = __ldg(reinterpret_cast<const float4*>(inv_lambda + 8 * c) + 1);
    const float v[8] = {__fmul_rn(__uint_as_float(mx.x << 16), a.x), __fmul_rn(__uint_as_float(mx.x & 0xFFFF0000u), a.y),
                        __fmul_rn(__uint_as_float(mx.y << 16), a.z), __fmul_rn(__uint_as_float(mx.y & 0xFFFF0000u), a.w),
                        __fmul_rn(__uint_as_float(mx.z << 16), b.x), __fmul_rn(__uint_as_float(mx.z & 0xFFFF0000u), b.y),
                        __fmul_rn(__uint_as_float(mx.w << 16), b.z), __fmul_rn(__uint_as_float(mx.w & 0xFFFF0000u), b.w)};
#pragma unroll
    for (int k = 0; k < 8; ++k) m = max(m, __float_as_uint(v[k]) & 0x7FFFFFFFu);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < THREADS / 32 ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) parts[blockIdx.x] = m;
  }
}

namespace {
// rows per thread stride: about two CTAs of 512 threads per SM in total
uint32_t amax_row_stride(int K, int num_sms) {
  const uint32_t kv = (uint32_t)(K / 8), target = 2u * (uint32_t)num_sms * THREADS;
  return target / kv > 0 ? target / kv : 1u;
}
}  // namespace

int act_amax_num_parts(int K, int num_sms) {
  const uint32_t kv = (uint32_t)(K / 8), R = amax_row_stride(K, num_sms);
  const uint64_t grid = ((uint64_t)kv * R + THREADS - 1) / THREADS;
  return grid <= (uint64_t)AMAX_MAX_PARTS ? (int)grid : 0;
}

cudaError_t launch_act_amax(const __nv_bfloat16* X, int M, int K, const float* inv_lambda, uint32_t* parts,
                            int num_sms, cudaStream_t stream) {
  const int n_parts = act_amax_num_parts(K, num_sms);
  if (n_parts <= 0) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)n_parts);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, act_amax_partials_kernel, X, M, (uint32_t)(K / 8), amax_row_stride(K, num_sms),
                            inv_lambda, parts);
}

}  // namespace svdq
