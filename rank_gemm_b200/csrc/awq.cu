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
// 4j of a 16-bit half-word (the codes of 8 consecutive k sit in a 32-bit word
// in the order of awq_nibble_pos), is OR-ed into the mantissa of 2^23, giving
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
constexpr int CODE_BYTES = 2 * WARPS * 32 * 16;  // a stage: 16 chunks x 32 features x 16 B
constexpr int SCALE_BYTES = WARPS * 32 * 2;      // 8 groups x 32 binary16 scales
constexpr int ZERO_BYTES = WARPS * 32;           // 8 groups x 32 zero points
constexpr int STAGE_BYTES = CODE_BYTES + SCALE_BYTES + ZERO_BYTES;

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
    words[j >> 3] |= (uint32_t)q << (4 * awq_nibble_pos(j & 7));
  }
  for (int h = 0; h < 2; ++h)
    *reinterpret_cast<uint4*>(code + ((size_t)(2 * g + h) * p.N_pad + n) * 16) =
        make_uint4(words[4 * h], words[4 * h + 1], words[4 * h + 2], words[4 * h + 3]);
  p.scale[(size_t)g * p.N_pad + n] = dh;
  p.zero[(size_t)g * p.N_pad + n] = (uint8_t)zf;
}

// ---------------------------------------------------------------- layer
// A CTA takes blocks of 32 output features (one per lane) in turn.  Warp 8
// is the TMA producer: per stage it loads 8 groups of codes for the block's
// 32 features ([16 chunks][32][16 B], 8 KB) with their binary16 scales and
// zero points into a 4-stage ring, so about 35 KB per CTA are in flight
// without costing registers.  Consumer warp w takes group 8 t + w of stage
// t: two 16-byte code chunks and its scale and zero point from shared
// memory, x' from the staged rows (the same word in every lane).  MB:
// activation rows per pass (the template keeps unused rows' accumulators out
// of the registers).
template <int MB>
__global__ void __launch_bounds__(THREADS + 32, 3)
    awq_gemv_kernel(const __grid_constant__ CUtensorMap tmCode, const __grid_constant__ CUtensorMap tmScale,
                    const __grid_constant__ CUtensorMap tmZero, AwqParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;                                         // AWQ_STAGES x STAGE_BYTES
  float* xs = reinterpret_cast<float*>(ring + AWQ_STAGES * STAGE_BYTES);   // [mb][K] x' / 16^(k mod 4)
  float* red = xs + (size_t)p.mb * p.K;                         // [WARPS][mb][32]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + WARPS * p.mb * 32);
  uint64_t* empty = full + AWQ_STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + AWQ_STAGES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = p.N_pad / 32;                               // 32-feature blocks, taken in turn by the CTAs
  const int G = p.K / GROUP, T = (G + WARPS - 1) / WARPS;      // stages per block and pass
  const int passes = (p.M + p.mb - 1) / p.mb;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmCode);
    tma_prefetch_desc(&tmScale);
    tma_prefetch_desc(&tmZero);
    for (int i = 0; i < AWQ_STAGES; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), WARPS);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == WARPS) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      for (int ps = 0; ps < passes; ++ps) {
        for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
          const int n0 = blk * 32;
          for (int t = 0; t < T; ++t, ++it) {
            const int st = it % AWQ_STAGES;
            if (!mbar_wait(smem_u32(&empty[st]), ((it / AWQ_STAGES) & 1) ^ 1, abort_flag, p.err)) return;
            const uint32_t dst = smem_u32(ring + st * STAGE_BYTES), bar = smem_u32(&full[st]);
            mbar_arrive_expect_tx(bar, STAGE_BYTES);
            tma_load_3d(dst, &tmCode, 0, n0, t * 2 * WARPS, bar);
            tma_load_2d(dst + CODE_BYTES, &tmScale, n0, t * WARPS, bar);
            tma_load_2d(dst + CODE_BYTES + SCALE_BYTES, &tmZero, n0, t * WARPS, bar);
          }
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const uint32_t xs_base = smem_u32(xs);
  int it = 0;
  bool ok = true;
  for (int ps = 0; ps < passes; ++ps) {
    const int m0 = ps * p.mb, mc = min(p.mb, p.M - m0);
    named_bar_sync(1, THREADS);                  // the previous pass's reads of xs are done
    // x' staged 8 columns per thread and step: 16 bytes of X and 32 of 1/s,
    // all of a thread's loads issued before the first is used
    {
      const int kv = p.K / 8, nv = mc * kv;
      for (int i0 = threadIdx.x; i0 < nv; i0 += 2 * THREADS) {
        uint4 xv[2];
        float4 ia[2], ib[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u * THREADS;
          if (i < nv) {
            const int m = i / kv, k = (i - m * kv) * 8;
            xv[u] = __ldg(reinterpret_cast<const uint4*>(p.X + (size_t)(m0 + m) * p.K + k));
            ia[u] = __ldg(reinterpret_cast<const float4*>(p.inv_s + k));
            ib[u] = __ldg(reinterpret_cast<const float4*>(p.inv_s + k) + 1);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u * THREADS;
          if (i < nv) {
            const float il[8] = {ia[u].x, ia[u].y, ia[u].z, ia[u].w, ib[u].x, ib[u].y, ib[u].z, ib[u].w};
            const uint32_t xw[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
            float o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float x = __uint_as_float((j & 1) ? (xw[j >> 1] & 0xFFFF0000u) : (xw[j >> 1] << 16));
              // fl32(x / s) times 16^-(p mod 4), p = awq_nibble_pos(j) (the code's
              // position in its half-word): exact
              o[j] = __fmul_rn(x, il[j]) * __uint_as_float((uint32_t)(127 - 4 * (awq_nibble_pos(j) & 3)) << 23);
            }
            // staged in nibble order: position p of the 8 holds column k with awq_nibble_pos(k) = p
            float4* dst = reinterpret_cast<float4*>(xs + (size_t)i * 8);
            dst[0] = make_float4(o[0], o[2], o[4], o[6]);
            dst[1] = make_float4(o[1], o[3], o[5], o[7]);
          }
        }
      }
    }
    named_bar_sync(1, THREADS);

    for (int blk = blockIdx.x; blk < nblk; blk += gridDim.x) {
      const int n = blk * 32 + lane;
      float acc[MB];
#pragma unroll
      for (int m = 0; m < MB; ++m) acc[m] = 0.f;
      for (int t = 0; t < T; ++t, ++it) {
        const int st = it % AWQ_STAGES;
        if (ok && !mbar_wait(smem_u32(&full[st]), (it / AWQ_STAGES) & 1, abort_flag, p.err)) ok = false;
        const int g = t * WARPS + warp;
        if (ok && g < G) {
          const uint8_t* sb = ring + st * STAGE_BYTES;
          const uint4 w0 = lds128(smem_u32(sb + ((2 * warp) * 32 + lane) * 16));
          const uint4 w1 = lds128(smem_u32(sb + ((2 * warp + 1) * 32 + lane) * 16));
          const float d = __half2float(reinterpret_cast<const __half*>(sb + CODE_BYTES)[warp * 32 + lane]);
          const float z = (float)sb[CODE_BYTES + SCALE_BYTES + warp * 32 + lane];
          const uint64_t c01 = f2(MAGIC + z, MAGIC + 16.f * z), c23 = f2(MAGIC + 256.f * z, MAGIC + 4096.f * z);
          uint64_t gacc[MB];
#pragma unroll
          for (int m = 0; m < MB; ++m) gacc[m] = 0ull;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 wv = h ? w1 : w0;
            const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
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
              for (int m = 0; m < MB; ++m) {
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
          for (int m = 0; m < MB; ++m)
            acc[m] = fmaf(d, __uint_as_float((uint32_t)gacc[m]) + __uint_as_float((uint32_t)(gacc[m] >> 32)), acc[m]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[st]));   // the warp's reads of stage st are consumed
      }
      // the 8 warps' partial sums, added in a fixed order (the same result on every run)
#pragma unroll
      for (int m = 0; m < MB; ++m)
        if (m < mc) red[(warp * p.mb + m) * 32 + lane] = acc[m];
      named_bar_sync(1, THREADS);
      if (warp < mc && n < p.N) {
        float y = p.bias[n];
        for (int w = 0; w < WARPS; ++w) y += red[(w * p.mb + warp) * 32 + lane];
        p.Y[(size_t)(m0 + warp) * p.N + n] = __float2bfloat16_rn(y);
      }
      named_bar_sync(1, THREADS);                // red is free for the next block
    }
  }
}

size_t awq_smem_bytes(int K, int mb) {
  return 1024 /*alignment*/ + (size_t)AWQ_STAGES * STAGE_BYTES + ((size_t)mb * K + (size_t)WARPS * mb * 32) * 4 +
         2 * AWQ_STAGES * 8 + 16;
}

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

cudaError_t launch_awq_gemv(const CUtensorMap& tmCode, const CUtensorMap& tmScale, const CUtensorMap& tmZero,
                           AwqParams p, int num_sms, cudaStream_t stream) {
  const size_t smem = awq_smem_bytes(p.K, p.mb);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  // the smallest instantiation that holds mb rows
  void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, AwqParams) =
      p.mb <= 1 ? awq_gemv_kernel<1> : p.mb <= 2 ? awq_gemv_kernel<2> : awq_gemv_kernel<4>;
  static_assert(AWQ_MB_MAX == 4, "instantiations cover 1, 2 and 4 rows");
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  // CTAs take the 32-feature blocks in turn, the same number each (about
  // three resident per SM)
  const int nblk = p.N_pad / 32, slots = 3 * num_sms;
  const int per = (nblk + slots - 1) / slots, grid = (nblk + per - 1) / per;
  kern<<<grid, THREADS + 32, smem, stream>>>(tmCode, tmScale, tmZero, p);
  return cudaGetLastError();
}

}  // namespace svdq
