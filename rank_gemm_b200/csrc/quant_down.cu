// quant_down.cu -- kernel 1: activation quantization fused with the low-rank
// down projection ("Nunchaku engine design" figure (b), "svdq-int4-flux.1-dev"
// model card: the Quantize and Down Projection kernels read the same input,
// so they are fused and X is read from HBM once).
//
// One CTA owns 32 rows of X and walks all of K in 128-column stages.  TMA
// stages each [32 x 128] bf16 tile of X (and the matching [r_tot x 128] tile
// of L1f^T) into shared memory through a multi-stage mbarrier ring.  From the
// same staged tile:
//   * every thread quantizes one 16-element group of one row (x^ = x / lambda,
//     amax, block scale, 4-bit codes) and writes packed codes and scales in
//     the layout kernel 2's tensor-core MMA consumes;
//   * every warp runs bf16 mma.sync tiles of LR = X L1f with fp32 accumulators
//     that stay in registers across the whole K loop (no atomics, no second
//     pass), then writes LR in bf16 once at the end.
// The kernel is HBM-bound: per row it reads 2K bytes of X and writes about
// K/2 + K/16 bytes of codes and scales plus 2 r_pad bytes of LR.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int BM = 32;         // rows per CTA
constexpr int BK = 128;        // K columns per stage (two 64-column TMA boxes)
constexpr int THREADS = 256;

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Address of the 16-byte chunk holding columns [8c, 8c+8) of row `row` in a
// [rows x 64] bf16 box written by TMA with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t box_base, int row, int c) {
  return box_base + row * 128 + ((c ^ (row & 7)) << 4);
}

constexpr int MAX_PAIRS_PER_WARP = 8;   // r_tot <= 256 -> 2 * 32 (m, n) tiles over 8 warps

}  // namespace

__global__ void __launch_bounds__(THREADS, 1)
    quant_down_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmL1,
                      K1Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * BM;

  // CTAs past the last activation row only clear the scale rows that pad the
  // last 128-row scale-factor block.
  if (m0 >= p.M) {
    if (!p.do_quant) return;
    const int ngroups = p.K_pad / 16;
    for (int i = tid; i < BM * ngroups; i += THREADS) {
      const int r = m0 + i / ngroups, g = i % ngroups;
      if (p.fmt == 0)
        p.sX[sf_atom_offset(r, g, p.K_pad)] = 0;
      else if ((g & 3) == 0)
        reinterpret_cast<__half*>(p.sX)[int4_scale_offset(r, g / 4, p.K_pad)] = __float2half(0.f);
    }
    return;
  }

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int x_bytes = BM * BK * 2;                        // 8 KB
  const int l_bytes = p.do_lr ? p.r_tot * BK * 2 : 0;    // r_tot x 128 bf16
  const int stage_bytes = x_bytes + l_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + p.stages * stage_bytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + p.stages);

  const int nk = p.K_pad / BK;
  if (tid == 0) {
    tma_prefetch_desc(&tmX);
    if (p.do_lr) tma_prefetch_desc(&tmL1);
    for (int s = 0; s < p.stages; ++s) mbar_init(smem_u32(&full[s]), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int kt) {
    const int s = kt % p.stages;
    const uint32_t st = smem_u32(base + s * stage_bytes);
    const uint32_t bar = smem_u32(&full[s]);
    mbar_arrive_expect_tx(bar, stage_bytes);
    tma_load_2d(st, &tmX, kt * BK, m0, bar);
    tma_load_2d(st + x_bytes / 2, &tmX, kt * BK + 64, m0, bar);
    if (p.do_lr) {
      tma_load_2d(st + x_bytes, &tmL1, kt * BK, 0, bar);
      tma_load_2d(st + x_bytes + l_bytes / 2, &tmL1, kt * BK + 64, 0, bar);
    }
  };
  if (tid == 0)
    for (int kt = 0; kt < min(nk, p.stages); ++kt) issue(kt);

  // LR accumulators: warp w owns (m-tile w & 1) x (n-tiles (w >> 1) + 4 i).
  const int mt = warp & 1;
  const int n_tiles = p.r_tot / 8;
  float acc[MAX_PAIRS_PER_WARP][4];
#pragma unroll
  for (int i = 0; i < MAX_PAIRS_PER_WARP; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  // quantization role: row qr, 16-column group qg of the stage
  const int qr = tid >> 3, qg = tid & 7;
  const int m = m0 + qr;
  const size_t qx_row_bytes = (size_t)(p.K_pad / 2);

  bool ok = true;
  for (int kt = 0; kt < nk; ++kt) {
    const int s = kt % p.stages;
    if (!mbar_wait(smem_u32(&full[s]), (kt / p.stages) & 1, abort_flag, p.err)) {
      ok = false;
      break;
    }
    const uint32_t st = smem_u32(base + s * stage_bytes);

    if (p.do_quant) {
      const int k0 = kt * BK + qg * 16;
      const uint32_t box = st + (qg >> 2) * (x_bytes / 2);
      const int c0 = (qg & 3) * 2;
      uint4 u0, u1;
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(u0.x), "=r"(u0.y), "=r"(u0.z), "=r"(u0.w)
                   : "r"(sw128_chunk(box, qr, c0)));
      asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(u1.x), "=r"(u1.y), "=r"(u1.z), "=r"(u1.w)
                   : "r"(sw128_chunk(box, qr, c0 + 1)));
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      float v[16];
      if (k0 < p.K) {
        const float4* il = reinterpret_cast<const float4*>(p.inv_lambda + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 f = __ldg(il + q);
          const float fl[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * q + e;
            const uint32_t bits = (j & 1) ? (w[j >> 1] & 0xFFFF0000u) : (w[j >> 1] << 16);
            v[j] = __fmul_rn(__uint_as_float(bits), fl[e]);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
      }
      uint2 codes;
      if (p.fmt == 0) {
        uint32_t sc;
        quant_nvfp4_16(v, p.s_t, p.six_st, codes, sc);
        // four consecutive groups (one 64-k block) of a row -> one 32-bit store
        const uint32_t s1 = __shfl_down_sync(0xffffffffu, sc, 1);
        const uint32_t s2 = __shfl_down_sync(0xffffffffu, sc, 2);
        const uint32_t s3 = __shfl_down_sync(0xffffffffu, sc, 3);
        if ((qg & 3) == 0) {
          const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
          *reinterpret_cast<uint32_t*>(p.sX + sf_atom_offset(m, k0 / 16, p.K_pad)) = word;
        }
      } else {
        __half sc;
        quant_int4_16of64(v, codes, sc);
        if ((qg & 3) == 0) reinterpret_cast<__half*>(p.sX)[int4_scale_offset(m, k0 / 64, p.K_pad)] = sc;
      }
      if (m < p.M) *reinterpret_cast<uint2*>(p.qX + (size_t)m * qx_row_bytes + k0 / 2) = codes;
    }

    if (p.do_lr) {
      const int kvalid = min(BK, p.K - kt * BK);   // multiple of 64 (may be <= 0 in the pad)
      const uint32_t lbase = st + x_bytes;
#pragma unroll 2
      for (int j = 0; j < BK / 16; ++j) {
        if (j * 16 >= kvalid) break;
        const int half = j >> 2;                       // which 64-column box
        const int cj = (j & 3) * 2;                    // 16-byte chunk index of this k16 step
        uint32_t a0, a1, a2, a3;
        {
          const int row = mt * 16 + (lane & 15);
          ldmatrix_x4(sw128_chunk(st + half * (x_bytes / 2), row, cj + (lane >> 4)), a0, a1, a2, a3);
        }
#pragma unroll
        for (int i = 0; i < MAX_PAIRS_PER_WARP; ++i) {
          const int nt = (warp >> 1) + 4 * i;
          if (nt < n_tiles) {
            const int n = nt * 8 + (lane & 7);
            uint32_t b0, b1;
            ldmatrix_x2(sw128_chunk(lbase + half * (l_bytes / 2), n, cj + ((lane >> 3) & 1)), b0, b1);
            mma_16816(acc[i], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }

    __syncthreads();                                   // stage s fully consumed
    if (tid == 0 && kt + p.stages < nk) issue(kt + p.stages);
  }

  if (!ok) return;

  if (p.do_lr) {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int i = 0; i < MAX_PAIRS_PER_WARP; ++i) {
      const int nt = (warp >> 1) + 4 * i;
      if (nt < n_tiles) {
        const int col = nt * 8 + 2 * t4;
        const int r0 = m0 + mt * 16 + g, r1 = r0 + 8;
        if (r0 < p.M)
          *reinterpret_cast<__nv_bfloat162*>(p.LR + (size_t)r0 * p.r_pad + col) =
              __floats2bfloat162_rn(acc[i][0], acc[i][1]);
        if (r1 < p.M)
          *reinterpret_cast<__nv_bfloat162*>(p.LR + (size_t)r1 * p.r_pad + col) =
              __floats2bfloat162_rn(acc[i][2], acc[i][3]);
      }
    }
    // zero padding columns [r_tot, r_pad)
    const int padc = p.r_pad - p.r_tot;
    for (int i = tid; i < BM * padc; i += THREADS) {
      const int r = m0 + i / padc, c = p.r_tot + i % padc;
      if (r < p.M) p.LR[(size_t)r * p.r_pad + c] = __float2bfloat16(0.f);
    }
  }
}

size_t quant_down_smem_bytes(int r_tot, bool do_lr, int* stages_out, int nk) {
  const int stage_bytes = BM * BK * 2 + (do_lr ? r_tot * BK * 2 : 0);
  int stages = (196 * 1024) / stage_bytes;
  stages = stages < 2 ? 2 : (stages > 8 ? 8 : stages);
  if (stages > nk) stages = nk < 1 ? 1 : nk;
  *stages_out = stages;
  return (size_t)stages * stage_bytes + 1024 /*alignment slack*/ + 8 * stages + 64;
}

cudaError_t launch_quant_down(const CUtensorMap& tmX, const CUtensorMap& tmL1, K1Params p,
                              cudaStream_t stream) {
  const int nk = p.K_pad / BK;
  const size_t smem = quant_down_smem_bytes(p.r_tot, p.do_lr != 0, &p.stages, nk);
  cudaError_t e = cudaFuncSetAttribute(quant_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = round_up(p.M, 128) / BM;
  quant_down_kernel<<<grid, THREADS, smem, stream>>>(tmX, tmL1, p);
  return cudaGetLastError();
}

}  // namespace svdq
