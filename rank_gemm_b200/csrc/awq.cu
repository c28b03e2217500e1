// awq.cu -- the AWQ W4A16 linear layer: 4-bit weights (zero-point code per
// group of 64 along K, binary16 scale), 16-bit activations.  The Diffusers
// blog "Integrating Nunchaku 4-bit diffusion inference into Diffusers"
// ("Introducing Nunchaku Lite": the awq_w4a16 kernel family for the adaptive
// normalization and modulation projections, memory-bound and sensitive to
// precision; "Native loading in Diffusers": precision int4, group_size 64).
//
//   prepare (offline):  W' = fl32(w * s_k) (AWQ's per-input-channel scale),
//     per (group g, output n): lo/hi = min/max W', d = binary16(max(hi - lo,
//     1e-5) / 15) (saturating), zero = clamp(rint(-lo / d), 0, 15),
//     code = clamp(rint(w' / d) + zero, 0, 15).
//   layer:  y[m,n] = sum_g d[g,n] sum_{k in g} (code[k,n] - zero[g,n]) x'[m,k] + b[n],
//     x' = fl32(x * fl32(1/s_k)), fp32 accumulation, Y = bf16(y).
//
// The layer is a weight stream: at the batch sizes of a modulation
// projection (a few rows) every weight byte is used M times, so the kernel
// runs on the CUDA cores and is sized for HBM: lanes of a warp take 32
// consecutive output features and read the k-chunk-major code layout
// (512 contiguous bytes per warp and chunk); the 8 warps of a CTA split K;
// x' sits in shared memory and every lane reads the same word (broadcast).
// A code becomes a float with one logic operation: its nibble, kept at bit
// 4j of a 16-bit half-word, is OR-ed into the mantissa of 2^23, giving
// 2^23 + 16^j q exactly; subtracting 2^23 + 16^j zero leaves 16^j (q - zero),
// and x' is staged pre-multiplied by 16^-j (exact), so one packed fp32 FMA
// takes two codes.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int GROUP = 64;
constexpr int CHUNK = 32;                        // codes per 16-byte chunk of one output feature
constexpr int WARPS = AWQ_WARPS;
constexpr int THREADS = 32 * WARPS;
constexpr float MAGIC = 8388608.0f;              // 2^23

__device__ __forceinline__ uint64_t f2(float lo, float hi) {
  return ((uint64_t)__float_as_uint(hi) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
// nibbles at bits 4i and 4j of h, each OR-ed into the mantissa of 2^23
__device__ __forceinline__ uint64_t nib2(uint32_t h, uint32_t mi, uint32_t mj) {
  return ((uint64_t)((h & mj) | 0x4B000000u) << 32) | ((h & mi) | 0x4B000000u);
}

}  // namespace

// ---------------------------------------------------------------- prepare
// One thread per (group, output feature); reads the group's 64 weights of
// row n (128 contiguous bytes of W_t).
__global__ void awq_quantize_kernel(AwqPrepParams p) {
  const int G = p.K / GROUP;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= G * p.N_pad) return;
  const int g = i / p.N_pad, n = i - g * p.N_pad;
  uint8_t* code = p.code;                       // [K/32][N_pad][16]
  if (n >= p.N) {                               // pad features: code 0, zero 0, scale 0
    for (int h = 0; h < 2; ++h)
      *reinterpret_cast<uint4*>(code + ((size_t)(2 * g + h) * p.N_pad + n) * 16) = make_uint4(0u, 0u, 0u, 0u);
    p.scale[(size_t)g * p.N_pad + n] = __float2half_rn(0.f);
    p.zero[(size_t)g * p.N_pad + n] = 0;
    return;
  }
  const __nv_bfloat16* w = p.Wt + (size_t)n * p.K + (size_t)g * GROUP;
  float v[GROUP];
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll 8
  for (int j = 0; j < GROUP; ++j) {
    const float s = p.s ? p.s[g * GROUP + j] : 1.0f;
    v[j] = __fmul_rn(__bfloat162float(w[j]), s);
    lo = fminf(lo, v[j]);
    hi = fmaxf(hi, v[j]);
  }
  const float rng = fmaxf(__fsub_rn(hi, lo), 1e-5f);
  // binary16, round to nearest even, saturating at 65504
  const float dr = fminf(fmaxf(__fdiv_rn(rng, 15.0f), -65504.0f), 65504.0f);
  const __half dh = __float2half_rn(dr);
  const float d = __half2float(dh);
  const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, d)), 0.f), 15.f);
  uint32_t words[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) words[t] = 0u;
#pragma unroll
  for (int j = 0; j < GROUP; ++j) {
    const float q = fminf(fmaxf(rintf(__fdiv_rn(v[j], d)) + zf, 0.f), 15.f);
    words[j >> 3] |= (uint32_t)q << (4 * (j & 7));
  }
  for (int h = 0; h < 2; ++h)
    *reinterpret_cast<uint4*>(code + ((size_t)(2 * g + h) * p.N_pad + n) * 16) =
        make_uint4(words[4 * h], words[4 * h + 1], words[4 * h + 2], words[4 * h + 3]);
  p.scale[(size_t)g * p.N_pad + n] = dh;
  p.zero[(size_t)g * p.N_pad + n] = (uint8_t)zf;
}

// ---------------------------------------------------------------- layer
__global__ void __launch_bounds__(THREADS)
    awq_gemv_kernel(AwqParams p) {
  extern __shared__ __align__(16) float xs[];   // [mb][K] x' / 16^(k mod 4), then [WARPS][mb][32] partials
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * 32 + lane;          // < N_pad
  const int G = p.K / GROUP;
  const int gper = (G + WARPS - 1) / WARPS, g0 = warp * gper, g1 = min(G, g0 + gper);
  float* red = xs + (size_t)p.mb * p.K;
  const uint32_t xs_base = smem_u32(xs);

  for (int m0 = 0; m0 < p.M; m0 += p.mb) {
    const int mc = min(p.mb, p.M - m0);
    __syncthreads();                              // the previous block's reads of xs are done
    for (int i = threadIdx.x; i < mc * p.K; i += THREADS) {
      const int m = i / p.K, k = i - m * p.K;
      const float x = __fmul_rn(__bfloat162float(p.X[(size_t)(m0 + m) * p.K + k]), __ldg(p.inv_s + k));
      xs[i] = x * __uint_as_float((uint32_t)(127 - 4 * (k & 3)) << 23);   // times 16^-(k mod 4): exact
    }
    __syncthreads();

    float acc[AWQ_MB_MAX];
#pragma unroll
    for (int m = 0; m < AWQ_MB_MAX; ++m) acc[m] = 0.f;
#pragma unroll 2
    for (int g = g0; g < g1; ++g) {
      const float d = __half2float(p.scale[(size_t)g * p.N_pad + n]);
      const float z = (float)p.zero[(size_t)g * p.N_pad + n];
      const uint64_t c01 = f2(MAGIC + z, MAGIC + 16.f * z), c23 = f2(MAGIC + 256.f * z, MAGIC + 4096.f * z);
      uint4 wv[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        wv[h] = __ldg(reinterpret_cast<const uint4*>(p.code + ((size_t)(2 * g + h) * p.N_pad + n) * 16));
      uint64_t gacc[AWQ_MB_MAX];
#pragma unroll
      for (int m = 0; m < AWQ_MB_MAX; ++m) gacc[m] = 0ull;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t words[4] = {wv[h].x, wv[h].y, wv[h].z, wv[h].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t lo = words[q], hi = words[q] >> 16;
          // 16^j (code - zero) for the word's 8 codes, in pairs
          const uint64_t v01 = f2_sub(nib2(lo, 0x000Fu, 0x00F0u), c01);
          const uint64_t v23 = f2_sub(nib2(lo, 0x0F00u, 0xF000u), c23);
          const uint64_t v45 = f2_sub(nib2(hi, 0x000Fu, 0x00F0u), c01);
          const uint64_t v67 = f2_sub(nib2(hi, 0x0F00u, 0xF000u), c23);
          const uint32_t xa = xs_base + (uint32_t)(((2 * g + h) * CHUNK + q * 8) * 4);
#pragma unroll
          for (int m = 0; m < AWQ_MB_MAX; ++m) {
            if (m < mc) {
              const uint4 x0 = lds128(xa + (uint32_t)(m * p.K * 4));
              const uint4 x1 = lds128(xa + (uint32_t)(m * p.K * 4) + 16);
              gacc[m] = f2_fma(v01, ((uint64_t)x0.y << 32) | x0.x, gacc[m]);
              gacc[m] = f2_fma(v23, ((uint64_t)x0.w << 32) | x0.z, gacc[m]);
              gacc[m] = f2_fma(v45, ((uint64_t)x1.y << 32) | x1.x, gacc[m]);
              gacc[m] = f2_fma(v67, ((uint64_t)x1.w << 32) | x1.z, gacc[m]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < AWQ_MB_MAX; ++m)
        acc[m] = fmaf(d, __uint_as_float((uint32_t)gacc[m]) + __uint_as_float((uint32_t)(gacc[m] >> 32)), acc[m]);
    }
    // the 8 warps' partial sums, added in a fixed order (the same result on every run)
#pragma unroll
    for (int m = 0; m < AWQ_MB_MAX; ++m)
      if (m < mc) red[(warp * p.mb + m) * 32 + lane] = acc[m];
    __syncthreads();
    if (warp < mc && n < p.N) {
      float y = p.bias[n];
      for (int w = 0; w < WARPS; ++w) y += red[(w * p.mb + warp) * 32 + lane];
      p.Y[(size_t)(m0 + warp) * p.N + n] = __float2bfloat16_rn(y);
    }
  }
}

size_t awq_smem_bytes(int K, int mb) { return ((size_t)mb * K + (size_t)WARPS * mb * 32) * 4; }

int awq_rows_per_block(int K, int M) {
  // as many activation rows as fit in 48 KB of staged x' (at least one)
  int mb = (int)((48 * 1024) / ((size_t)K * 4));
  mb = mb < 1 ? 1 : (mb > AWQ_MB_MAX ? AWQ_MB_MAX : mb);
  return M < mb ? (M < 1 ? 1 : M) : mb;
}

// 1/s (correctly rounded) and the bias widened to fp32 over N_pad
__global__ void awq_vectors_kernel(AwqPrepParams p) {
  const int stride = gridDim.x * blockDim.x;
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < p.K; k += stride)
    p.inv_s[k] = p.s ? __frcp_rn(p.s[k]) : 1.0f;
  for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < p.N_pad; n += stride)
    p.bias_f[n] = (n < p.N && p.bias) ? __bfloat162float(p.bias[n]) : 0.f;
}

cudaError_t launch_awq_quantize(const AwqPrepParams& p, cudaStream_t stream) {
  const int total = (p.K / GROUP) * p.N_pad;
  awq_quantize_kernel<<<(total + 127) / 128, 128, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  awq_vectors_kernel<<<64, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_awq_gemv(AwqParams p, cudaStream_t stream) {
  const size_t smem = awq_smem_bytes(p.K, p.mb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(awq_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  awq_gemv_kernel<<<p.N_pad / 32, THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace svdq
