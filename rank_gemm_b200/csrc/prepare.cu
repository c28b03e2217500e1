// prepare.cu -- offline kernels: calibration of the smoothing factors and
// preparation of the quantized residual (SVDQuant overview figure, Stages 2
// and 3, "svdq-int4-flux.1-dev" model card).
//
//   calibrate : lambda_k = max|X[:,k]|^a / max|W[k,:]|^(1-a)   (float64, one
//               rounding), then the static NVFP4 activation tensor scale
//               max|fl32(x / lambda)| / 2688.
//   residual  : R = lambda o W - lambda o (L1f L2) in float64, i ascending,
//               separate multiply and add (the __d*_rn intrinsics are never
//               contracted into FMA), one rounding to float32; running amax.
//   quantize  : R per output column in 16- (NVFP4) or 64- (INT4) groups along
//               K with the same quantizer as the activations (common.cuh),
//               written in the layouts kernel 2 consumes; plus the transposed
//               low-rank factors (L2 divided by alpha), bias in float32 and
//               1/lambda.
// Maxima use atomicMax on the bit pattern of non-negative floats, which is
// order-independent, so every output is deterministic.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

__device__ __forceinline__ float bf(const __nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ unsigned warp_max_u32(unsigned v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Column maxima of |A| for a row-major [rows][K] bf16 matrix.
__global__ void colmax_kernel(const __nv_bfloat16* A, int rows, int K, int rows_per_block,
                              unsigned* out_bits) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const int r0 = blockIdx.y * rows_per_block;
  const int r1 = min(rows, r0 + rows_per_block);
  float m = 0.f;
  for (int r = r0; r < r1; ++r) m = fmaxf(m, fabsf(bf(A[(size_t)r * K + k])));
  atomicMax(out_bits + k, __float_as_uint(m));
}

__global__ void lambda_kernel(const unsigned* ax_bits, const unsigned* aw_bits, int K, float alpha,
                              float* lambda) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const double ax = (double)__uint_as_float(ax_bits[k]);
  const double aw = (double)__uint_as_float(aw_bits[k]);
  float lam = 1.f;
  if (ax != 0.0 && aw != 0.0) {
    double num, den;
    if (alpha == 0.5f) {
      num = __dsqrt_rn(ax);
      den = __dsqrt_rn(aw);
    } else {
      num = pow(ax, (double)alpha);
      den = pow(aw, 1.0 - (double)alpha);
    }
    lam = __double2float_rn(__ddiv_rn(num, den));
  }
  lambda[k] = lam;
}

__global__ void act_amax_kernel(const __nv_bfloat16* X, int M, int K, const float* lambda,
                                unsigned* amax_bits) {
  const size_t total = (size_t)M * K;
  unsigned m = 0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(i % K);
    const float v = __fmul_rn(bf(X[i]), __frcp_rn(lambda[k]));
    m = max(m, __float_as_uint(fabsf(v)));
  }
  m = warp_max_u32(m);
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, m);
}

__global__ void act_scale_kernel(const unsigned* amax_bits, float* act_scale) {
  const float a = __uint_as_float(*amax_bits);
  *act_scale = (a == 0.f) ? 1.f : __fdiv_rn(a, 2688.0f);
}

// R^T[n][k] for a 32 (k) x 32 (n) tile per block of 32 x 8 threads.
__global__ void residual_kernel(PrepParams p) {
  __shared__ double l1s[32][33];   // [k][i]
  __shared__ double l2s[32][33];   // [i][n]
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int k0 = blockIdx.x * 32, n0 = blockIdx.y * 32;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int i0 = 0; i0 < p.rank; i0 += 32) {
    for (int j = ty; j < 32; j += 8) {
      const int k = k0 + j, i = i0 + tx;
      l1s[j][tx] = (k < p.K && i < p.rank) ? (double)bf(p.L1f[(size_t)k * p.rank + i]) : 0.0;
      const int ii = i0 + j, n = n0 + tx;
      l2s[j][tx] = (ii < p.rank && n < p.N) ? (double)bf(p.L2[(size_t)ii * p.N + n]) : 0.0;
    }
    __syncthreads();
    const int iend = min(32, p.rank - i0);
    for (int i = 0; i < iend; ++i) {
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = __dadd_rn(acc[q], __dmul_rn(l1s[ty + 8 * q][i], l2s[i][tx]));
    }
    __syncthreads();
  }
  unsigned amax = 0;
  const int n = n0 + tx;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int k = k0 + ty + 8 * q;
    if (k < p.K && n < p.N) {
      const double lam = (double)p.lambda[k];
      const double t1 = __dmul_rn(lam, (double)bf(p.Wt[(size_t)n * p.K + k]));
      const double t2 = __dmul_rn(lam, acc[q]);
      const float r = __double2float_rn(__dsub_rn(t1, t2));
      p.R[(size_t)n * p.K + k] = r;
      amax = max(amax, __float_as_uint(fabsf(r)));
    }
  }
  amax = warp_max_u32(amax);
  if ((threadIdx.x & 31) == 0) atomicMax(p.amax_bits, amax);
}

// One thread per 16-element group of one row of R^T (rows = output features).
__global__ void quantize_weights_kernel(PrepParams p, float s_tR, float six_st) {
  const int groups_per_row = p.K_pad / 16;
  const size_t total = (size_t)p.N_pad * groups_per_row;
  const size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (idx >= total) return;   // total is a multiple of 32: whole warps exit together
  const int n = (int)(idx / groups_per_row), g = (int)(idx % groups_per_row);
  const int k0 = g * 16;
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = 0.f;
  if (n < p.N && k0 < p.K) {
    const float4* src = reinterpret_cast<const float4*>(p.R + (size_t)n * p.K + k0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = src[q];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  }
  uint2 codes;
  if (p.fmt == 0) {
    uint32_t sc;
    quant_nvfp4_16(v, s_tR, six_st, codes, sc);
    p.sR[sf_atom_offset(n, g, p.K_pad)] = (uint8_t)sc;
  } else {
    __half sc;
    quant_int4_16of64(v, codes, sc);
    if ((g & 3) == 0) reinterpret_cast<float*>(p.sR)[int4_scale_offset(n, g / 4, p.K_pad)] = __half2float(sc);
  }
  *reinterpret_cast<uint2*>(p.qR + (size_t)n * (p.K_pad / 2) + k0 / 2) = codes;
  if (p.qR8) *reinterpret_cast<uint4*>(p.qR8 + (size_t)n * p.K_pad + k0) = int4x16_to_e4m3(codes);
}

__global__ void factors_kernel(PrepParams p, float alpha) {
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  const int stride = gridDim.x * blockDim.x;
  // L1t = ([L1f | A])^T in kernel 1's staged layout: per 64-wide k stage one
  // [r_tot x 64] bf16 box, each row's eight 16-byte chunks placed with the
  // 128-byte swizzle (chunk c of row r at c ^ (r % 8)), zeros for k >= K.
  for (int i = tid; i < p.r_tot * p.K_pad; i += stride) {
    const int r = i / p.K_pad, k = i % p.K_pad;
    __nv_bfloat16 v = __float2bfloat16(0.f);
    if (k < p.K)
      v = (r < p.rank) ? p.L1f[(size_t)k * p.rank + r] : p.loraA[(size_t)k * p.lora_rank + (r - p.rank)];
    const int kb = k >> 6, c = k & 63;
    const size_t off = (size_t)kb * p.r_tot * 64 + (size_t)r * 64 + ((((c >> 3) ^ (r & 7)) << 3) | (c & 7));
    p.L1t[off] = v;
  }
  // L2a [N_pad][r_pad] = ([L2 ; B] / alpha)^T, zero padded
  for (int i = tid; i < p.N_pad * p.r_pad; i += stride) {
    const int n = i / p.r_pad, r = i % p.r_pad;
    float v = 0.f;
    if (n < p.N && r < p.r_tot) {
      const float src = (r < p.rank) ? bf(p.L2[(size_t)r * p.N + n])
                                     : bf(p.loraB[(size_t)(r - p.rank) * p.N + n]);
      v = __fdiv_rn(src, alpha);
    }
    p.L2a[i] = __float2bfloat16_rn(v);
  }
  for (int n = tid; n < p.N_pad; n += stride)
    p.bias_f[n] = (n < p.N && p.bias) ? bf(p.bias[n]) : 0.f;
  for (int k = tid; k < p.K; k += stride) p.lambda_inv[k] = __frcp_rn(p.lambda[k]);
  // kernel 1's copy of 1/lambda, permuted inside every 64-wide stage so that
  // its quantizer threads (one per 16-column group g, four adjacent lanes per
  // row) read 16-byte chunk q of their group from position 4 q + g:
  // conflict-free shared-memory reads
  for (int k = tid; k < p.K_pad; k += stride) {
    const int kb = k >> 6, g = (k >> 4) & 3, q = (k >> 2) & 3, e = k & 3;
    p.lambda_inv_k1[(size_t)kb * 64 + (q * 4 + g) * 4 + e] = (k < p.K) ? __frcp_rn(p.lambda[k]) : 0.f;
  }
}

// Kernel 2's copy of the NVFP4 weight scales: every (row, 64-k block) word
// of the atom layout written to its four replicas (see sfw_rep_offset).
__global__ void replicate_weight_scales_kernel(PrepParams p) {
  const int kbs = p.K_pad / 64;
  const size_t total = (size_t)p.N_pad * kbs;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(i / kbs), kb = (int)(i % kbs);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p.sR + sf_atom_offset(n, kb * 4, p.K_pad));
#pragma unroll
    for (int q = 0; q < 4; ++q) *reinterpret_cast<uint32_t*>(p.sR_rep + sfw_rep_offset(n, kb, q, p.K_pad)) = w;
  }
}

__global__ void selftest_timeout_kernel(DeviceErr err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must give up by itself.
  mbar_wait(smem_u32(&bar), 0, &abort_flag, err);
}

}  // namespace

cudaError_t launch_calibrate(int M, int K, int N, const __nv_bfloat16* X, const __nv_bfloat16* Wt,
                             float alpha, float* lambda_out, float* act_scale_out, unsigned* ws,
                             cudaStream_t stream) {
  unsigned* ax = ws;
  unsigned* aw = ws + K;
  unsigned* amax = ws + 2 * K;
  cudaError_t e = cudaMemsetAsync(ws, 0, (2 * (size_t)K + 1) * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  const int rpb = 256;
  dim3 gx((K + 255) / 256, (M + rpb - 1) / rpb), gw((K + 255) / 256, (N + rpb - 1) / rpb);
  if (M > 0) colmax_kernel<<<gx, 256, 0, stream>>>(X, M, K, rpb, ax);
  colmax_kernel<<<gw, 256, 0, stream>>>(Wt, N, K, rpb, aw);
  lambda_kernel<<<(K + 255) / 256, 256, 0, stream>>>(ax, aw, K, alpha, lambda_out);
  if (M > 0) act_amax_kernel<<<1184, 256, 0, stream>>>(X, M, K, lambda_out, amax);
  act_scale_kernel<<<1, 1, 0, stream>>>(amax, act_scale_out);
  return cudaGetLastError();
}

cudaError_t launch_prepare_residual(const PrepParams& p, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(p.amax_bits, 0, sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  dim3 grid((p.K + 31) / 32, (p.N + 31) / 32), block(32, 8);
  residual_kernel<<<grid, block, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prepare_quantize(const PrepParams& p, float s_tR, float alpha, cudaStream_t stream) {
  const size_t total = (size_t)p.N_pad * (p.K_pad / 16);
  const float six_st = 6.0f * s_tR;   // one IEEE float32 multiply on the host
  quantize_weights_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(p, s_tR, six_st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  factors_kernel<<<592, 256, 0, stream>>>(p, alpha);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.fmt != 0) return e;
  replicate_weight_scales_kernel<<<592, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_selftest_timeout(DeviceErr err, cudaStream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(err);
  return cudaGetLastError();
}

}  // namespace svdq
