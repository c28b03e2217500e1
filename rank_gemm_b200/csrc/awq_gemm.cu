// awq_gemm.cu -- the AWQ W4A16 layer on the 5th-generation tensor core, for
// batches large enough that the layer is a dense contraction (the W4A16
// side of the "SVDQuant" abstract's comparison: 4-bit weights, 16-bit
// activations, the product at 16-bit tensor-core rate).  The weight format
// is the awq_w4a16 family's of the Diffusers blog ("Introducing Nunchaku
// Lite"; "Native loading in Diffusers": int4, group_size 64), the same
// handle and code layout as the GEMV in awq.cu.
//
//   Y = bf16( X'16 W^16 + b ),  w^16 = bf16((code - zero) d) (one rounding
//   of the exact product), X'16 = bf16(fl32(x fl32(1/s))) (X itself when the
//   handle has no AWQ scale), float32 accumulation in TMEM.
//
// Persistent, one CTA per SM, 128 x 256 output tiles, 64-wide k-tiles:
//   warp 0      TMA producer: the [128 x 64] bf16 X tile (128-byte swizzle),
//               the tile's codes ([2 chunks][256 features][16 B]), binary16
//               scales and zero points (and 1/s) into a 4-stage ring.
//   warp 1      TMEM owner and single-thread MMA issuer: four
//               tcgen05.mma.kind::f16 (bf16, K = 16) per k-tile into one of two
//               128 x 256 float32 accumulators (the epilogue of one tile runs
//               under the MMAs of the next).
//   warps 2-17  dequantizers, two threads per output feature of the tile
//               (one per 32-k chunk): per k-tile the feature's 64 codes become
//               64 bf16 weights written as one 128-byte row of the K-major,
//               128-byte-swizzled B tile (a 3-stage ring of its own), with the
//               exact pair arithmetic below; with an AWQ scale they also
//               rewrite the X tile as bf16(x / s) in place.
//   warps 18-21 epilogue, one per TMEM sub-partition: accumulator + bias ->
//               bf16, 32-byte stores.
// Dequantization, two weights per instruction: the codes of k and k + 1 sit
// at bits 4j and 16 + 4j of their word (awq_nibble_pos), so one shift and one
// AND/OR put 128 + q into each bf16 half; subtracting 128 + zero leaves
// q - zero exactly; with d = dh + dl (dh = bf16(d); dl, at most 3 significant
// bits, exact in bf16) the product (q - zero) dl is exact and
// fma((q - zero), dh, (q - zero) dl) rounds (q - zero) d once.
// All waits are bounded (mbar_wait); TMEM is freed on every exit path.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int DQ_WARPS = 16;                                 // BN features x two 32-k chunks, one per thread
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (2 + DQ_WARPS + EPI_WARPS);     // 704
constexpr int W_PROD = 0, W_MMA = 1, W_DQ0 = 2, W_EPI0 = 2 + DQ_WARPS;
constexpr int NS_A = 4, NS_B = 3;
constexpr int X_BYTES = BM * BK * 2;                         // 16 KB
constexpr int CODE_BYTES = 2 * BN * 16;                      // 8 KB
constexpr int SCALE_BYTES = BN * 2;
constexpr int ZERO_BYTES = BN;
constexpr int INVS_BYTES = BK * 4;
constexpr int OFF_CODE = X_BYTES, OFF_SCALE = OFF_CODE + CODE_BYTES, OFF_ZERO = OFF_SCALE + SCALE_BYTES,
              OFF_INVS = OFF_ZERO + ZERO_BYTES;
constexpr int A_STAGE = OFF_INVS + INVS_BYTES;               // 25,600 bytes
static_assert(A_STAGE % 1024 == 0, "X tiles must stay 1024-byte aligned for the 128-byte swizzle");
constexpr int B_BYTES = BN * BK * 2;                         // 32 KB
constexpr uint32_t TMEM_COLS = 512;                          // two 256-column accumulators
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

struct Ctl {
  uint64_t a_full[NS_A], a_empty[NS_A], b_full[NS_B], b_empty[NS_B], t_full[2], t_empty[2];
  uint32_t tmem_base;
  int abort;
};
constexpr size_t SMEM_BYTES = 1024 + (size_t)NS_A * A_STAGE + (size_t)NS_B * B_BYTES + sizeof(Ctl);

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint32_t bf2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t bf16_bits(__nv_bfloat16 h) { return (uint32_t)__bfloat16_as_ushort(h); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&o)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(o[0]), "r"(o[1]), "r"(o[2]),
               "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
               : "memory");
}

// The four bf16 pairs (k, k + 1), k = 8w + 0, 2, 4, 6, of one code word
// (awq_nibble_pos order), each (q - zero) d rounded once.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t zz, uint32_t dh, uint32_t dl) {
  uint32_t r[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t t = ((w >> (4 * j)) & 0x000F000Fu) | 0x43004300u;   // bf16 pair (128 + q_k, 128 + q_k+1)
    const uint32_t qz = bf2_sub(t, zz);                                 // q - zero, exact
    r[j] = bf2_fma(qz, dh, bf2_mul(qz, dl));                            // (q - zero) d, one rounding
  }
  return make_uint4(r[0], r[1], r[2], r[3]);
}

}  // namespace

template <bool HAS_S>
__global__ void __launch_bounds__(THREADS, 1)
    awq_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmCode,
                    const __grid_constant__ CUtensorMap tmScale, const __grid_constant__ CUtensorMap tmZero,
                    AwqGemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ringA = base;
  uint8_t* ringB = base + NS_A * A_STAGE;
  Ctl* ctl = reinterpret_cast<Ctl*>(ringB + NS_B * B_BYTES);
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmCode);
    tma_prefetch_desc(&tmScale);
    tma_prefetch_desc(&tmZero);
    for (int s = 0; s < NS_A; ++s) {
      mbar_init(smem_u32(&ctl->a_full[s]), 1);
      mbar_init(smem_u32(&ctl->a_empty[s]), DQ_WARPS + 1);   // the dequantizers + the MMA commit
    }
    for (int s = 0; s < NS_B; ++s) {
      mbar_init(smem_u32(&ctl->b_full[s]), DQ_WARPS);
      mbar_init(smem_u32(&ctl->b_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&ctl->t_full[s]), 1);
      mbar_init(smem_u32(&ctl->t_empty[s]), EPI_WARPS);
    }
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == W_MMA) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int nk = p.K / BK;
  constexpr uint32_t TX = X_BYTES + CODE_BYTES + SCALE_BYTES + ZERO_BYTES + (HAS_S ? INVS_BYTES : 0);

  if (warp == W_PROD) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const uint32_t sa = it % NS_A, pa = (it / NS_A) & 1;
          if (!mbar_wait(smem_u32(&ctl->a_empty[sa]), pa ^ 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t st = smem_u32(ringA + sa * A_STAGE), bar = smem_u32(&ctl->a_full[sa]);
          mbar_arrive_expect_tx(bar, TX);
          tma_load_2d(st, &tmX, kt * BK, mb * BM, bar);
          tma_load_3d(st + OFF_CODE, &tmCode, 0, nb * BN, 2 * kt, bar);
          tma_load_2d(st + OFF_SCALE, &tmScale, nb * BN, kt, bar);
          tma_load_2d(st + OFF_ZERO, &tmZero, nb * BN, kt, bar);
          if (HAS_S) bulk_load(st + OFF_INVS, p.inv_s + kt * BK, INVS_BYTES, bar);
        }
      }
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++tl) {
        const uint32_t ab = tl & 1, pt = (tl >> 1) & 1;
        if (!mbar_wait(smem_u32(&ctl->t_empty[ab]), pt ^ 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + ab * BN;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const uint32_t sa = it % NS_A, pa = (it / NS_A) & 1, sb = it % NS_B, pb = (it / NS_B) & 1;
          if (!mbar_wait(smem_u32(&ctl->a_full[sa]), pa, abort_flag, p.err) ||
              !mbar_wait(smem_u32(&ctl->b_full[sb]), pb, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(ringA + sa * A_STAGE), b = smem_u32(ringB + sb * B_BYTES);
#pragma unroll
          for (int j = 0; j < BK / 16; ++j)
            mma_bf16(acc, desc_k_sw128(a + 32 * j), desc_k_sw128(b + 32 * j), IDESC, (kt | j) != 0);
          tc_commit(smem_u32(&ctl->a_empty[sa]));
          tc_commit(smem_u32(&ctl->b_empty[sb]));
        }
        if (!ok) break;
        tc_commit(smem_u32(&ctl->t_full[ab]));
      }
    }
  } else if (warp < W_EPI0) {
    // ------------------------------------------------------------ dequantizers
    const int t = threadIdx.x - 32 * W_DQ0;   // 0..511
    const int n = t & 255, h = t >> 8;         // feature of the tile, 32-k chunk
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      for (int kt = 0; kt < nk; ++kt, ++it) {
        const uint32_t sa = it % NS_A, pa = (it / NS_A) & 1, sb = it % NS_B, pb = (it / NS_B) & 1;
        if (!mbar_wait(smem_u32(&ctl->a_full[sa]), pa, abort_flag, p.err) ||
            !mbar_wait(smem_u32(&ctl->b_empty[sb]), pb ^ 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        const uint8_t* sg = ringA + sa * A_STAGE;
        const float d = __half2float(reinterpret_cast<const __half*>(sg + OFF_SCALE)[n]);
        const __nv_bfloat16 dh = __float2bfloat16_rn(d);
        const __nv_bfloat16 dl = __float2bfloat16_rn(d - __bfloat162float(dh));   // exact: d has 11 bits
        const uint32_t DH = bf16_bits(dh) * 0x10001u, DL = bf16_bits(dl) * 0x10001u;
        const uint32_t z = sg[OFF_ZERO + n];
        const uint32_t ZZ = 0x43004300u | (z << 16) | z;                       // (128 + zero, 128 + zero)
        const uint4 c0 = lds128(smem_u32(sg + OFF_CODE + h * 4096 + n * 16));   // k 32h .. 32h + 31
        const uint32_t row = smem_u32(ringB + sb * B_BYTES) + (uint32_t)n * 128;
        const uint32_t sw = (uint32_t)(n & 7);
        const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // 16-byte chunk c = 4h + q = k 8c .. 8c + 7
          const uint32_t c = 4 * h + q;
          const uint4 v = dequant_word(words[q], ZZ, DH, DL);
          sts128(row + ((c ^ sw) << 4), v.x, v.y, v.z, v.w);
        }
        if (HAS_S) {
          // X tile in place: x' = bf16(fl32(x * fl32(1/s))); thread t takes
          // row t / 2, chunks 4 (t % 2) .. + 3
          const int r = t >> 2;
          const uint32_t xrow = smem_u32(ringA + sa * A_STAGE) + (uint32_t)r * 128;
          const float* invs = reinterpret_cast<const float*>(sg + OFF_INVS);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * (t & 3) + cc;
            const uint32_t addr = xrow + ((uint32_t)(c ^ (r & 7)) << 4);
            const uint4 x = lds128(addr);
            const float4 i0 = *reinterpret_cast<const float4*>(invs + 8 * c);
            const float4 i1 = *reinterpret_cast<const float4*>(invs + 8 * c + 4);
            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
            const float il[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q)
              o[q] = pack_bf16x2(__fmul_rn(__uint_as_float(xw[q] << 16), il[2 * q]),
                                 __fmul_rn(__uint_as_float(xw[q] & 0xFFFF0000u), il[2 * q + 1]));
            sts128(addr, o[0], o[1], o[2], o[3]);
          }
        }
        fence_proxy_async_smem();   // the B tile (and X tile) writes, before the tensor core reads them
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&ctl->b_full[sb]));
          mbar_arrive(smem_u32(&ctl->a_empty[sa]));
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3, row = sub * 32 + lane;
    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++tl) {
      const int mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
      const uint32_t ab = tl & 1, pt = (tl >> 1) & 1;
      if (!mbar_wait(smem_u32(&ctl->t_full[ab]), pt, abort_flag, p.err)) break;
      tc_fence_after();
      const int m = mb * BM + row;
      const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + ab * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + 32 * c, r);
        tmem_wait_ld();
        if (c == BN / 32 - 1) {   // the whole accumulator is in registers: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&ctl->t_empty[ab]));
        }
        if (m < p.M) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int n0 = nb * BN + 32 * c + 16 * q;
            if (n0 < p.N) {
              const float4* bv = reinterpret_cast<const float4*>(p.bias + n0);
              uint32_t o[8];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float4 b4 = __ldg(bv + j);
                o[2 * j] = pack_bf16x2(__uint_as_float(r[16 * q + 4 * j]) + b4.x,
                                       __uint_as_float(r[16 * q + 4 * j + 1]) + b4.y);
                o[2 * j + 1] = pack_bf16x2(__uint_as_float(r[16 * q + 4 * j + 2]) + b4.z,
                                           __uint_as_float(r[16 * q + 4 * j + 3]) + b4.w);
              }
              st_global_v8(p.Y + (size_t)m * p.N + n0, o);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_awq_gemm(const CUtensorMap& tmX, const CUtensorMap& tmCode, const CUtensorMap& tmScale,
                            const CUtensorMap& tmZero, AwqGemmParams p, bool has_s, int num_sms,
                            cudaStream_t stream) {
  void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, AwqGemmParams) =
      has_s ? awq_gemm_kernel<true> : awq_gemm_kernel<false>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  kern<<<tiles < num_sms ? tiles : num_sms, THREADS, SMEM_BYTES, stream>>>(tmX, tmCode, tmScale, tmZero, p);
  return cudaGetLastError();
}

}  // namespace svdq
