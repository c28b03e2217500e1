// gemm_int4.cu -- kernel 2 for INT4: the 4-bit GEMM fused with the low-rank up
// projection ("Nunchaku engine design" figure (b), "svdq-int4-flux.1-dev" model
// card), on the FP8 tensor-core path.
//
// INT4 block scales are binary16 per 64 elements, which no block-scaled MMA
// kind can take, so each 64-group is its own product:
//     y[m,n] = sum_g sX[m,g] sR[n,g] (sum_{k in g} qX[m,k] qR[n,k]) + LR[m,:] L2[n,:] + b[n]
// The codes (-8..7) reach this kernel as FP8 E4M3 bytes, which hold them
// exactly (kernel 1 writes the activations that way; the weights handle keeps
// an E4M3 copy next to the packed codes), so TMA stages them straight into
// the operand tiles.  Every group runs as two tcgen05.mma.kind::f8f6f4
// (K = 32) into a fresh fp32 TMEM tile, whose sums (|.| <= 64 * 64) are exact;
// CUDA cores apply sX sR and accumulate in fp32 registers: a packed f32x2
// multiply forms two scale products, one scalar FMA per output element per
// group adds the rescaled sum (scalar FMAs read the TMEM-load registers as
// they are; packed FMAs needed a register-pair copy per pair).  That
// arithmetic is the bound of this kernel.  (A first version unpacked packed
// int4 tiles in shared memory for every output tile; that byte shuffling set
// its pace.)
//
// One 128 x 128 output tile per CTA at a time, persistent over tiles:
//   warp 0       TMA producer: per 128-wide k-tile the [128 x 128 B] E4M3
//                tiles of qX and qR (128-byte swizzle) into the operand ring
//                and the k-tile's scale chunks of both (1 KB each) into a
//                scale ring; then the low-rank chunks (LR and L2, 64 columns).
//   warp 1       TMEM owner and MMA issuer (per 128-wide k-tile, its two
//                groups into the two halves of one of two TMEM buffers; the
//                low-rank chunks as kind::f16 into one more buffer use).
//   warps 2-17   rescale + epilogue: 4 warps per TMEM sub-partition, 32 columns
//                each, one barrier round trip per k-tile (two groups), read
//                from TMEM in 16-column chunks with each chunk's load issued
//                before the previous chunk's arithmetic; fp32 accumulators in
//                registers; bias, GELU, bf16 store.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int BM = K2_I4_ROWS, BN = K2_I4_ROWS;
constexpr int MS = 6;                    // operand ring: E4M3 k-tiles / bf16 low-rank chunks
constexpr int SC = 8;                    // scale ring (one k-tile's scales of qX and qR)
constexpr int OP_BYTES = 16384;          // E4M3 [128 x 128 B] or bf16 [128 x 64]
constexpr int STAGE_BYTES = 2 * OP_BYTES;
constexpr int SC_HALF = 1024;            // float32 [2 groups][128 rows]
constexpr int SC_BYTES = 2 * SC_HALF;
constexpr int W_MMA = 1, W_RESCALE = 2;
constexpr int RS_WARPS = 16;             // four per TMEM sub-partition, 32 columns each
constexpr int RS_COLS = BN / (RS_WARPS / 4);
constexpr int THREADS = (W_RESCALE + RS_WARPS) * 32;
constexpr int NKB = 2;                   // TMEM k-tile buffers, each the two groups' BN columns side by side
constexpr uint32_t KB_COLS = 2 * BN;
constexpr uint32_t TMEM_COLS = NKB * KB_COLS;
// kind::f8f6f4: fp32 D, E4M3 A and B (format code 0), K-major
constexpr uint32_t IDESC_F8 = (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t IDESC_BF = idesc_bf16_f32(BM, BN);

struct Ctl {
  uint64_t full[MS], empty[MS], cfull[SC], cempty[SC], dfull[NKB], dempty[NKB];
  uint32_t tmem_base;
  int abort;
};
constexpr size_t SMEM_BYTES = (size_t)MS * STAGE_BYTES + (size_t)SC * SC_BYTES + 1024 + sizeof(Ctl);

__device__ __forceinline__ void mma_f8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Packed float32 pairs kept in 64-bit registers (element 0 in the low half).
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t u2(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }
__device__ __forceinline__ void lds2x64(uint32_t addr, uint64_t& a, uint64_t& b) {
  asm volatile("ld.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(addr));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
// 32 lanes x 16 consecutive 32-bit columns -> 16 registers per thread.
__device__ __forceinline__ void tmem_ld16_i4(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// Waits for this thread's TMEM loads; r is passed through, so no use of the
// loaded registers can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}
// acc[off .. off + 7] += (sx sr) d for 16 columns: d = the group's exact
// fp32 sums, sx sr the product of two binary16 scales (exact in fp32)
__device__ __forceinline__ void rescale16(float (&acc)[32], int off, const uint32_t (&r)[16], uint64_t sx2,
                                          uint32_t sra) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint64_t sr01, sr23;
    lds2x64(sra + q * 16, sr01, sr23);
    const uint64_t c01 = f2_mul(sx2, sr01), c23 = f2_mul(sx2, sr23);
    float* a = acc + 2 * off + 4 * q;
    a[0] = fmaf(__uint_as_float((uint32_t)c01), __uint_as_float(r[4 * q]), a[0]);
    a[1] = fmaf(__uint_as_float((uint32_t)(c01 >> 32)), __uint_as_float(r[4 * q + 1]), a[1]);
    a[2] = fmaf(__uint_as_float((uint32_t)c23), __uint_as_float(r[4 * q + 2]), a[2]);
    a[3] = fmaf(__uint_as_float((uint32_t)(c23 >> 32)), __uint_as_float(r[4 * q + 3]), a[3]);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

__global__ void __launch_bounds__(THREADS, 1)
    gemm_int4_kernel(const __grid_constant__ CUtensorMap tmX8, const __grid_constant__ CUtensorMap tmR8,
                     const __grid_constant__ CUtensorMap tmLR, const __grid_constant__ CUtensorMap tmL2,
                     K2I8Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;                             // MS x 32 KB
  uint8_t* sring = ring + MS * STAGE_BYTES;         // SC x 2 KB
  Ctl* ctl = reinterpret_cast<Ctl*>(sring + SC * SC_BYTES);
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmX8);
    tma_prefetch_desc(&tmR8);
    if (p.nl) {
      tma_prefetch_desc(&tmLR);
      tma_prefetch_desc(&tmL2);
    }
    for (int s = 0; s < MS; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    for (int c = 0; c < SC; ++c) {
      mbar_init(smem_u32(&ctl->cfull[c]), 1);
      mbar_init(smem_u32(&ctl->cempty[c]), RS_WARPS);
    }
    for (int b = 0; b < NKB; ++b) {
      mbar_init(smem_u32(&ctl->dfull[b]), 1);
      mbar_init(smem_u32(&ctl->dempty[b]), RS_WARPS);
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
  const int nk = p.nk, nl = p.nl;

  if (warp == 0) {
    if (lane == 0) {
      // -------------------------------------------------------------- producer
      int s = 0, c = 0;
      uint32_t ph = 0, cph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
        for (int it = 0; it < nk + nl; ++it) {
          if (!mbar_wait(smem_u32(&ctl->empty[s]), ph ^ 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t dst = smem_u32(ring + s * STAGE_BYTES), bar = smem_u32(&ctl->full[s]);
          mbar_arrive_expect_tx(bar, STAGE_BYTES);
          if (it < nk) {
            tma_load_2d(dst, &tmX8, it * 128, mb * BM, bar);
            tma_load_2d(dst + OP_BYTES, &tmR8, it * 128, nb * BN, bar);
            // the k-tile's scale chunks: 128 rows x 2 groups of float32 each
            if (!mbar_wait(smem_u32(&ctl->cempty[c]), cph ^ 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            const uint32_t cdst = smem_u32(sring + c * SC_BYTES), cbar = smem_u32(&ctl->cfull[c]);
            mbar_arrive_expect_tx(cbar, SC_BYTES);
            bulk_load(cdst, p.sX + ((size_t)mb * nk + it) * 256, SC_HALF, cbar);
            bulk_load(cdst + SC_HALF, p.sR + ((size_t)nb * nk + it) * 256, SC_HALF, cbar);
            if (++c == SC) {
              c = 0;
              cph ^= 1;
            }
          } else {
            tma_load_2d(dst, &tmLR, (it - nk) * 64, mb * BM, bar);
            tma_load_2d(dst + OP_BYTES, &tmL2, (it - nk) * 64, nb * BN, bar);
          }
          if (++s == MS) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == W_MMA) {
    if (lane == 0) {
      // -------------------------------------------------------------- MMA issuer
      int s = 0;
      uint32_t ph = 0, uses = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        for (int it = 0; ok && it < nk; ++it) {
          if (!mbar_wait(smem_u32(&ctl->full[s]), ph, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(ring + s * STAGE_BYTES), b = a + OP_BYTES;
          const uint32_t buf = uses % NKB, dph = (uses / NKB) & 1;
          if (!mbar_wait(smem_u32(&ctl->dempty[buf]), dph ^ 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int j = 0; j < 2; ++j) {   // group j of the k-tile into columns j BN of the buffer
            const uint32_t d = tmem + buf * KB_COLS + j * BN;
            mma_f8(d, desc_k_sw128(a + 64 * j), desc_k_sw128(b + 64 * j), IDESC_F8, 0);
            mma_f8(d, desc_k_sw128(a + 64 * j + 32), desc_k_sw128(b + 64 * j + 32), IDESC_F8, 1);
          }
          tc_commit(smem_u32(&ctl->dfull[buf]));
          ++uses;
          tc_commit(smem_u32(&ctl->empty[s]));
          if (++s == MS) {
            s = 0;
            ph ^= 1;
          }
        }
        if (!ok) break;
        if (nl) {
          const uint32_t buf = uses % NKB, dph = (uses / NKB) & 1;
          if (!mbar_wait(smem_u32(&ctl->dempty[buf]), dph ^ 1, abort_flag, p.err)) break;
          for (int c = 0; c < nl; ++c) {
            if (!mbar_wait(smem_u32(&ctl->full[s]), ph, abort_flag, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a = smem_u32(ring + s * STAGE_BYTES), b = a + OP_BYTES;
            const int steps = min(4, (p.r_tot - 64 * c) / 16);
            for (int j = 0; j < steps; ++j)
              mma_bf16(tmem + buf * KB_COLS, desc_k_sw128(a + 32 * j), desc_k_sw128(b + 32 * j), IDESC_BF,
                       (c | j) != 0);
            tc_commit(smem_u32(&ctl->empty[s]));
            if (++s == MS) {
              s = 0;
              ph ^= 1;
            }
          }
          if (!ok) break;
          tc_commit(smem_u32(&ctl->dfull[buf]));
          ++uses;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- rescale + epilogue
    const int rw = warp - W_RESCALE;                 // 0..15
    const int sub = warp & 3, quarter = rw >> 2;     // TMEM sub-partition, 32-column quarter
    const int row = sub * 32 + lane;
    uint32_t uses = 0;
    int c = 0;
    uint32_t cph = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mb = tile % p.num_m_blocks, nb = tile / p.num_m_blocks;
      const int m = mb * BM + row, n0 = nb * BN + quarter * RS_COLS;
      float acc[RS_COLS];
#pragma unroll
      for (int i = 0; i < RS_COLS; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int kt = 0; ok && kt < nk; ++kt) {
        if (!mbar_wait(smem_u32(&ctl->cfull[c]), cph, abort_flag, p.err)) {
          ok = false;
          break;
        }
        const float* sc = reinterpret_cast<const float*>(sring + c * SC_BYTES);
        const uint32_t buf = uses % NKB, dph = (uses / NKB) & 1;
        ++uses;
        if (!mbar_wait(smem_u32(&ctl->dfull[buf]), dph, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the two groups' sums of this warp's 32 columns in four 16-column
        // chunks, each chunk's TMEM load issued before the previous chunk's
        // arithmetic; after the last load the buffer goes back to the MMA warp
        const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + buf * KB_COLS + quarter * RS_COLS;
        const uint32_t scb = smem_u32(sc);
        const uint32_t sx0 = lds_u32(scb + 4u * row), sx1 = lds_u32(scb + 4u * (128 + row));
        const uint32_t sra = scb + 4u * (256 + quarter * RS_COLS);
        uint32_t ra[16], rb[16];
        tmem_ld16_i4(taddr, ra);
        tmem_wait_ld16(ra);
        tmem_ld16_i4(taddr + 16, rb);
        rescale16(acc, 0, ra, u2(sx0, sx0), sra);
        tmem_wait_ld16(rb);
        tmem_ld16_i4(taddr + BN, ra);
        rescale16(acc, 8, rb, u2(sx0, sx0), sra + 64);
        tmem_wait_ld16(ra);
        tmem_ld16_i4(taddr + BN + 16, rb);
        rescale16(acc, 0, ra, u2(sx1, sx1), sra + 512);
        tmem_wait_ld16(rb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->dempty[buf]));
        rescale16(acc, 8, rb, u2(sx1, sx1), sra + 512 + 64);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->cempty[c]));   // this warp is done with the k-tile's scales
        if (++c == SC) {
          c = 0;
          cph ^= 1;
        }
      }
      if (ok && nl) {
        // the low-rank branch: LR (L2) accumulated in fp32 by the tensor core
        const uint32_t buf = uses % NKB, dph = (uses / NKB) & 1;
        ++uses;
        if (!mbar_wait(smem_u32(&ctl->dfull[buf]), dph, abort_flag, p.err)) {
          ok = false;
        } else {
          tc_fence_after();
          uint32_t r[32];
          tmem_ld32(tmem + ((uint32_t)(sub * 32) << 16) + buf * KB_COLS + quarter * RS_COLS, r);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&ctl->dempty[buf]));
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] += __uint_as_float(r[i]);
        }
      }
      if (!ok) break;
      if (m < p.M) {
        // 16 columns (32 bytes, one full sector) per store
#pragma unroll
        for (int c16 = 0; c16 < RS_COLS; c16 += 16) {
          const int n = n0 + c16;
          if (n < p.N) {
            float y[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 bq = __ldg(reinterpret_cast<const float4*>(p.bias + n) + q);
              const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                y[4 * q + e] = acc[c16 + 4 * q + e] + bb[e];
                if (p.epi == 1) y[4 * q + e] = gelu_tanh(y[4 * q + e]);
              }
            }
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) o[j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
            asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p.Y + (size_t)m * p.N + n),
                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
                         : "memory");
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

cudaError_t launch_gemm_int4(const CUtensorMap& tmX8, const CUtensorMap& tmR8, const CUtensorMap& tmLR,
                             const CUtensorMap& tmL2, K2I8Params p, int num_sms, cudaStream_t stream) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(gemm_int4_kernel), SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int grid = tiles < num_sms ? tiles : num_sms;
  gemm_int4_kernel<<<grid, THREADS, SMEM_BYTES, stream>>>(tmX8, tmR8, tmLR, tmL2, p);
  return cudaGetLastError();
}

}  // namespace svdq
