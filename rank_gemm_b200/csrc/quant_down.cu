// quant_down.cu -- kernel 1: activation quantization fused with the low-rank
// down projection ("Nunchaku engine design" figure (b), "svdq-int4-flux.1-dev"
// model card: the Quantize and Down Projection kernels read the same input,
// so they are fused and X is read from HBM once).
//
// One CTA owns 32 rows of X and walks all of K in 256-column stages.  A
// producer warp keeps a TMA ring of stages in flight; a stage holds the
// [32 x 256] bf16 tile of X (four 128-byte-swizzled boxes), the matching
// [r_tot x 256] tile of L1f^T (stored pre-swizzled, one contiguous bulk copy)
// and the 256 values of 1/lambda.  Each CTA walks
// the stages starting at its own offset, so the CTAs of a wave read different
// L1f^T tiles and different X columns at any moment.  From the same staged
// tile:
//   * 16 quantizer warps: every thread one 16-element group of one row
//     (x^ = x / lambda, amax, block scale, 4-bit codes), written packed with
//     scales in the layout kernel 2's tensor-core MMA consumes;
//   * one thread issues the down projection on the 5th-generation tensor core
//     as the transposed product LR^T = L1f^T X^T: A = the L1f^T tile (128 rows
//     per MMA, rows past r_tot are ignored), B = the staged X tile itself
//     (N = 32 rows), fp32 accumulation in a 32-column TMEM tile across all of
//     K; four warps read it out at the end and store LR in bf16.
// Stages are released through an mbarrier (the 16 quantizer warps plus the
// MMA commit) instead of a CTA-wide sync, so warps drift apart and overlap
// their load, math and store phases.  The kernel is HBM-bound: per row it
// reads 2K bytes of X and writes about K/2 + K/16 bytes of codes and scales
// plus 2 r_pad bytes of LR.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int BM = 32;                       // rows per CTA (= MMA N)
constexpr int BK = 256;                      // K columns per stage (four 64-column TMA boxes)
constexpr int QWARPS = 16;                   // quantizer warps
constexpr int THREADS = 32 * (QWARPS + 2);   // + producer warp + MMA warp
constexpr int X_BOX = BM * 128;              // one [32 x 64] bf16 box
constexpr int X_BYTES = 4 * X_BOX;           // 16 KB
constexpr int IL_BYTES = BK * 4;             // 1/lambda for the stage
constexpr int W_PROD = 0, W_MMA = 1, W_Q0 = 2;
constexpr int CHAINS = 1;                     // LR accumulators (interleaved k16 steps)

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 u;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
  return u;
}

// Address of the 16-byte chunk holding columns [8c, 8c+8) of row `row` in a
// [rows x 64] bf16 box written by TMA with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t box_base, int row, int c) {
  return box_base + row * 128 + ((c ^ (row & 7)) << 4);
}

struct Layout {
  int stages, l_box, x_ring, il_ring, l_ring, bar_off;
};

// Shared memory: X ring | 1/lambda ring | L1f^T boxes (compact) + a tail so
// an M = 128 MMA reading past the last box stays inside the allocation |
// barriers.
__host__ __device__ inline Layout make_layout(int stages, int r_tot, bool do_lr) {
  Layout L;
  L.stages = stages;
  L.l_box = do_lr ? r_tot * 128 : 0;
  L.x_ring = 0;
  L.il_ring = stages * X_BYTES;
  L.l_ring = L.il_ring + stages * IL_BYTES;
  const int tail = do_lr ? (r_tot > 128 ? 32768 : 16384) : 0;
  L.bar_off = L.l_ring + stages * 4 * L.l_box + tail;
  return L;
}

}  // namespace

__global__ void __launch_bounds__(THREADS, 1)
    quant_down_kernel(const __grid_constant__ CUtensorMap tmX, K1Params p) {
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
  const Layout L = make_layout(p.stages, p.r_tot, p.do_lr != 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* dfull = empty + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* inv_tab = reinterpret_cast<float*>(tmem_slot + 4);        // 128 entries, NVFP4 only
  // LR accumulates in CHAINS independent TMEM tiles (k16 step j goes to chain
  // j % CHAINS) so consecutive MMAs do not wait on each other's result; per
  // 128-row half of L1f^T: CHAINS x 32 columns
  const int halves = p.r_tot > 128 ? 2 : 1;
  const uint32_t tmem_cols = (uint32_t)(halves * CHAINS * BM);

  const int nk = p.K_pad / BK;
  const int k_first = blockIdx.x % nk;                   // this CTA's first stage
  if (tid == 0) {
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), (p.do_quant ? QWARPS : 0) + (p.do_lr ? 1 : 0));
    }
    mbar_init(smem_u32(dfull), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (p.fmt == 0 && tid < 128) inv_tab[tid] = nvfp4_inv_entry((uint32_t)tid, p.s_t);
  if (p.do_lr && warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = p.do_lr ? *tmem_slot : 0u;

  if (warp == W_PROD) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      for (int it = 0; it < nk; ++it) {
        const int s = it % p.stages;
        if (!mbar_wait(smem_u32(&empty[s]), ((it / p.stages) & 1) ^ 1, abort_flag, p.err)) break;
        const int kt = (k_first + it) % nk;
        const uint32_t bar = smem_u32(&full[s]);
        mbar_arrive_expect_tx(bar, X_BYTES + 4 * L.l_box + IL_BYTES);
        const uint32_t xs = smem_u32(base + L.x_ring + s * X_BYTES);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(xs + b * X_BOX, &tmX, kt * BK + 64 * b, m0, bar);
        if (p.do_lr)   // the stage's L1f^T tile is stored contiguous and pre-swizzled: one bulk copy
          bulk_load(smem_u32(base + L.l_ring + s * 4 * L.l_box), p.L1t + (size_t)kt * p.r_tot * BK, 4 * L.l_box, bar);
        bulk_load(smem_u32(base + L.il_ring + s * IL_BYTES), p.inv_lambda + kt * BK, IL_BYTES, bar);
      }
    }
  } else if (warp == W_MMA) {
    // ---------------------------------------------------------------- tensor-core down projection
    if (p.do_lr && lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, BM);
      uint32_t started = 0;                          // bit c: chain c has its first product
      bool ok = true;
      for (int it = 0; it < nk; ++it) {
        const int s = it % p.stages;
        if (!mbar_wait(smem_u32(&full[s]), (it / p.stages) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kt = (k_first + it) % nk;
        const int kvalid = p.K - kt * BK;              // multiple of 64 (may be <= 0 in the pad)
        const uint32_t xs = smem_u32(base + L.x_ring + s * X_BYTES);
        const uint32_t ls = smem_u32(base + L.l_ring + s * 4 * L.l_box);
        for (int j = 0; j < BK / 16; ++j) {
          if (j * 16 >= kvalid) break;
          const int box = j >> 2, koff = (j & 3) * 32, c = j % CHAINS;
          const uint64_t bdesc = desc_k_sw128(xs + box * X_BOX + koff);
          for (int h = 0; h < halves; ++h)
            mma_bf16(tmem + (h * CHAINS + c) * BM, desc_k_sw128(ls + box * L.l_box + h * 16384 + koff), bdesc,
                     idesc, (started >> c) & 1u);
          started |= 1u << c;
        }
        tc_commit(smem_u32(&empty[s]));
      }
      if (ok) tc_commit(smem_u32(dfull));
    }
  } else if (p.do_quant) {
    // ---------------------------------------------------------------- quantizers
    // row qr, 16-column group qg of the stage
    const int ct = tid - 32 * W_Q0;
    const int qr = ct >> 4, qg = ct & 15;
    const int m = m0 + qr;
    const size_t qx_row_bytes = (size_t)(p.K_pad / 2);
    for (int it = 0; it < nk; ++it) {
      const int s = it % p.stages;
      if (!mbar_wait(smem_u32(&full[s]), (it / p.stages) & 1, abort_flag, p.err)) break;
      const int kt = (k_first + it) % nk;
      const int k0 = kt * BK + qg * 16;
      const uint32_t box = smem_u32(base + L.x_ring + s * X_BYTES) + (qg >> 2) * X_BOX;
      const int c0 = (qg & 3) * 2;
      const uint4 u0 = lds128(sw128_chunk(box, qr, c0));
      const uint4 u1 = lds128(sw128_chunk(box, qr, c0 + 1));
      const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      // 1/lambda of this group: chunk q at position 16 q + qg of the permuted
      // stage copy (zeros past K, where TMA also filled x with zeros)
      const uint32_t ila = smem_u32(base + L.il_ring + s * IL_BYTES) + qg * 16;
      float il[16];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 f = lds128(ila + 256 * q);
        il[4 * q] = __uint_as_float(f.x);
        il[4 * q + 1] = __uint_as_float(f.y);
        il[4 * q + 2] = __uint_as_float(f.z);
        il[4 * q + 3] = __uint_as_float(f.w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&empty[s]));   // shared-memory reads of stage s are done
      float v[16];
#pragma unroll
      for (int j = 0; j < 16; j += 2)   // bf16 pair -> two floats, times 1/lambda
        mul2_rn(__uint_as_float(w[j >> 1] << 16), __uint_as_float(w[j >> 1] & 0xFFFF0000u), il[j], il[j + 1],
                v[j], v[j + 1]);
      uint2 codes;
      if (p.fmt == 0) {
        uint32_t sc;
        quant_nvfp4_16_tab(v, p.six_st, inv_tab, codes, sc);
        p.sX[sf_atom_offset(m, k0 / 16, p.K_pad)] = (uint8_t)sc;
      } else {
        __half sc;
        quant_int4_16of64(v, codes, sc);
        if ((qg & 3) == 0) reinterpret_cast<__half*>(p.sX)[int4_scale_offset(m, k0 / 64, p.K_pad)] = sc;
      }
      if (m < p.M) *reinterpret_cast<uint2*>(p.qX + (size_t)m * qx_row_bytes + k0 / 2) = codes;
    }
  }

  if (p.do_lr && warp >= W_Q0 && warp < W_Q0 + 4) {
    // ---------------------------------------------------------------- LR read-out
    // TMEM lane = rank index r (row of LR^T), column = row n of this CTA's X tile
    if (mbar_wait(smem_u32(dfull), 0, abort_flag, p.err)) {
      tc_fence_after();
      const int sub = warp & 3;
      for (int h = 0; h < halves; ++h) {
        float acc[BM];
#pragma unroll
        for (int n = 0; n < BM; ++n) acc[n] = 0.f;
        for (int c = 0; c < CHAINS; ++c) {               // fixed order: chain 0, 1, 2, 3
          uint32_t d[32];
          tmem_ld32(tmem + ((uint32_t)(sub * 32) << 16) + (h * CHAINS + c) * BM, d);
          tmem_wait_ld();
#pragma unroll
          for (int n = 0; n < BM; ++n) acc[n] += __uint_as_float(d[n]);
        }
        const int r = 128 * h + 32 * sub + lane;
        if (r < p.r_tot) {
#pragma unroll
          for (int n = 0; n < BM; ++n)
            if (m0 + n < p.M) p.LR[(size_t)(m0 + n) * p.r_pad + r] = __float2bfloat16_rn(acc[n]);
        }
      }
    }
  }
  if (p.do_lr) {
    // zero padding columns [r_tot, r_pad)
    const int padc = p.r_pad - p.r_tot;
    for (int i = tid; i < BM * padc; i += THREADS) {
      const int r = m0 + i / padc, c = p.r_tot + i % padc;
      if (r < p.M) p.LR[(size_t)r * p.r_pad + c] = __float2bfloat16(0.f);
    }
  }

  // Every thread reaches this point, also after a timeout (the loops above
  // leave early when the abort flag is set); TMEM is freed on every path.
  tc_fence_before();
  __syncthreads();
  if (p.do_lr && warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

size_t quant_down_smem_bytes(int r_tot, bool do_lr, int* stages_out, int nk) {
  const int stage_bytes = X_BYTES + IL_BYTES + (do_lr ? 4 * r_tot * 128 : 0);
  const int tail = do_lr ? (r_tot > 128 ? 32768 : 16384) : 0;
  int stages = (200 * 1024 - tail) / stage_bytes;
  stages = stages < 2 ? 2 : (stages > 6 ? 6 : stages);
  if (stages > nk) stages = nk < 1 ? 1 : nk;
  *stages_out = stages;
  const Layout L = make_layout(stages, r_tot, do_lr);
  return (size_t)L.bar_off + 1024 /*alignment slack*/ + 8 * (2 * stages + 1) + 16 + 128 * 4 + 64;
}

cudaError_t launch_quant_down(const CUtensorMap& tmX, K1Params p, cudaStream_t stream) {
  const int nk = p.K_pad / BK;
  const size_t smem = quant_down_smem_bytes(p.r_tot, p.do_lr != 0, &p.stages, nk);
  cudaError_t e = cudaFuncSetAttribute(quant_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = round_up(p.M, 128) / BM;
  quant_down_kernel<<<grid, THREADS, smem, stream>>>(tmX, p);
  return cudaGetLastError();
}

}  // namespace svdq
