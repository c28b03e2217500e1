// lowrank_up.cu -- the stand-alone up projection of the unfused baseline
// ("Nunchaku engine design" figure (a), "svdq-int4-flux.1-dev" model card:
// run naively, the low-rank branch writes the 16-bit output a second time).
//
//   Y[m][n] = bf16(epi(Y[m][n] + alpha * sum_i LR[m][i] L2a[n][i]))
//
// Read-modify-write of Y with a bf16 mma.sync tile of 128 x 128 outputs per
// CTA; it exists only to measure the overhead the fused kernel 2 removes.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int TM = 128, TN = 128, THREADS = 256;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(THREADS) lowrank_up_kernel(UpParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int ld = p.r_tot + 8;                       // padded row (bf16 elements)
  __nv_bfloat16* sA = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sB = sA + TM * ld;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cpr = p.r_tot / 8;                      // 16-byte chunks per row
  for (int i = tid; i < TM * cpr; i += THREADS) {
    const int r = i / cpr, c = i % cpr;
    uint4 va = make_uint4(0, 0, 0, 0), vb = make_uint4(0, 0, 0, 0);
    if (m0 + r < p.M) va = *reinterpret_cast<const uint4*>(p.LR + (size_t)(m0 + r) * p.r_pad + 8 * c);
    vb = *reinterpret_cast<const uint4*>(p.L2a + (size_t)(n0 + r) * p.r_pad + 8 * c);
    *reinterpret_cast<uint4*>(sA + r * ld + 8 * c) = va;
    *reinterpret_cast<uint4*>(sB + r * ld + 8 * c) = vb;
  }
  __syncthreads();
  const int wm = (warp & 3) * 32, wn = (warp >> 2) * 64;
  float acc[2][8][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b][0] = acc[a][b][1] = acc[a][b][2] = acc[a][b][3] = 0.f;
  const uint32_t baseA = smem_u32(sA), baseB = smem_u32(sB);
  for (int k = 0; k < p.r_tot; k += 16) {
    uint32_t af[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      const int row = wm + a * 16 + (lane & 15), col = k + (lane >> 4) * 8;
      ldsm_x4(baseA + (row * ld + col) * 2, af[a][0], af[a][1], af[a][2], af[a][3]);
    }
#pragma unroll
    for (int b = 0; b < 8; b += 2) {
      // two n8 tiles per ldmatrix.x4: (n 0-7, k 0-7), (n 0-7, k 8-15), (n 8-15, k 0-7), (n 8-15, k 8-15)
      const int nrow = wn + b * 8 + ((lane >> 4) << 3) + (lane & 7), col = k + ((lane >> 3) & 1) * 8;
      uint32_t b0, b1, b2, b3;
      ldsm_x4(baseB + (nrow * ld + col) * 2, b0, b1, b2, b3);
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        mma16816(acc[a][b], af[a], b0, b1);
        mma16816(acc[a][b + 1], af[a], b2, b3);
      }
    }
  }
  const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = m0 + wm + a * 16 + g + 8 * h, n = n0 + wn + b * 8 + 2 * t4;
        if (m < p.M && n < p.N) {
          __nv_bfloat162* y = reinterpret_cast<__nv_bfloat162*>(p.Y + (size_t)m * p.N + n);
          const float2 old = __bfloat1622float2(*y);
          float v0 = old.x + p.alpha * acc[a][b][2 * h], v1 = old.y + p.alpha * acc[a][b][2 * h + 1];
          if (p.epi == 1) {
            v0 = gelu_tanh(v0);
            v1 = gelu_tanh(v1);
          }
          *y = __floats2bfloat162_rn(v0, v1);
        }
      }
}

}  // namespace

cudaError_t launch_lowrank_up(UpParams p, cudaStream_t stream) {
  const size_t smem = (size_t)2 * TM * (p.r_tot + 8) * 2;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(lowrank_up_kernel), (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + TN - 1) / TN, (p.M + TM - 1) / TM);
  lowrank_up_kernel<<<grid, THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace svdq
