// gemm_nvfp4.cu -- kernel 2 for NVFP4: the 4-bit GEMM fused with the low-rank
// up projection ("Nunchaku engine design" figure (b), "svdq-int4-flux.1-dev"
// model card: Up Projection and 4-Bit Compute share their output, so the
// 16-bit branch is accumulated into the same output tile and Y is written
// once).
//
// Persistent, warp-specialized, one 128 x 256 output tile per CTA at a time:
//   warp 0      TMA producer: per 256-wide k-tile, the [128 x 128 B] tile of qX,
//               the [256 x 128 B] tile of qR (both 128-byte swizzled) and the
//               8 + 16 KB of E4M3 scales in their replicated layout (plain
//               bulk copies); then, per
//               64-wide chunk of the low-rank dimension, the [128 x 64] bf16 tile
//               of LR and the [256 x 64] bf16 tile of L2/alpha, into the same
//               ring slots (a bf16 tile of 64 columns has the byte shape of an
//               FP4 tile of 256 columns).
//   warp 1      TMEM owner and single-thread MMA issuer: six
//               tcgen05.cp.128x256b move a k-tile's scales to TMEM (the copies
//               cost per instruction, so the scales are stored pre-replicated
//               for the four TMEM sub-partitions and moved 8 columns at a
//               time), tcgen05.mma.kind::mxf4nvf4 (block16,
//               E4M3 scales) accumulates Q(X^) Q(R) in a 128 x 256 fp32 TMEM
//               tile, then tcgen05.mma.kind::f16 adds LR (L2/alpha) into the
//               same tile; tcgen05.commit releases ring slots and hands the
//               finished tile to the epilogue.
//   warps 2-9   epilogue: two warps per TMEM sub-partition, 128 columns each
//               (two 64-column blocks, interleaved with the other warp's);
//               the whole 128 x 256 tile is loaded to registers and the TMEM
//               accumulator released before y = alpha acc + b, optional GELU,
//               bf16 and the 32-byte stores, which overlap the next tile's MMAs.
//               In emit mode (cross-layer fusion) the epilogue instead writes
//               the next layer's kernel-1 outputs: its NVFP4 codes and
//               replicated scales from bf16 pairs parked in free TMEM
//               columns, and the float32 partial of its low-rank down
//               projection, which the MMA warp computes on the tensor core
//               with those parked pairs as the A operand (A in TMEM) and the
//               next layer's L1 slice as B, loaded as one extra ring stage a
//               few k-tiles into the following tile.
// All waits are bounded (see mbar_wait); TMEM is freed on every exit path.
#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int BLOCK_M = K2_NV_ROWS_A, BLOCK_N = K2_NV_ROWS_B, STAGES = 3;
constexpr int A_BYTES = BLOCK_M * 128;          // 16 KB
constexpr int B_BYTES = BLOCK_N * 128;          // 32 KB
constexpr int SF_BLOCK = 4096;                  // one replicated scale block (8 TMEM columns)
constexpr int SFA_BYTES = 2 * SF_BLOCK;         // 4 k-blocks x 128 rows
constexpr int SFB_BYTES = 4 * SF_BLOCK;         // 4 k-blocks x 2 row halves
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;   // 72 KB
constexpr int THREADS = 320;              // producer, MMA, 8 epilogue warps
constexpr int EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0, SFA_COL = 256, SFB_COL = 272;
constexpr uint32_t STASH_COL = 320;   // emit mode: bf16 pairs of the row slices, 64 columns per half
constexpr uint32_t DPART_COL = 448;   // emit mode: the next layer's LR partial, up to 64 float32 columns
constexpr int EMIT_AT = 6;            // emit mode: the partial's stage follows this FP4 k-tile of the next tile
constexpr uint32_t IDESC_F4 = idesc_nvf4(BLOCK_M, BLOCK_N);
constexpr uint32_t IDESC_BF = idesc_bf16_f32(BLOCK_M, BLOCK_N);

struct Ctl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull, tempty;
  uint64_t stash_full, part_full, part_empty;   // emit mode
  uint32_t tmem_base;
  int abort;
};

constexpr int BIAS_BYTES = EPI_WARPS * 128 * 4;   // warp-private bias slices
constexpr int TAB_BYTES = 128 * 4;                // emit mode: the next layer's 1/scale table
constexpr int INVL_BYTES = EPI_WARPS * 128 * 4;   // emit mode: warp-private slices of the next layer's 1/lambda
constexpr size_t SMEM_BYTES =
    (size_t)STAGES * STAGE_BYTES + BIAS_BYTES + TAB_BYTES + INVL_BYTES + 1024 + sizeof(Ctl);

// Tile order: groups of 8 row blocks, column blocks within a group, so the
// CTAs running at the same time share each activation tile among ~8 and each
// weight tile among ~18 readers instead of reading one weight tile all at once.
__device__ __forceinline__ void tile_coords(int tile, int nmb, int nnb, int& mb, int& nb) {
  constexpr int GM = 8;
  const int grp = tile / (GM * nnb), rr = tile % (GM * nnb);
  const int gs = min(GM, nmb - grp * GM);
  mb = grp * GM + rr % gs;
  nb = rr / gs;
}

// 32 bytes in one store (16-byte stores would leave every 32-byte sector
// half written by each of two instructions).  p must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&o)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(o[0]), "r"(o[1]), "r"(o[2]),
               "r"(o[3]), "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7])
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// D (TMEM) += A (TMEM: 128 lanes x 16 bf16, two per 32-bit column) B (smem descriptor), kind::f16.
__device__ __forceinline__ void mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns -> 16 registers per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// The k-iterations of one tile: the FP4 k-tiles, then the low-rank chunks;
// in emit mode with a previous tile, that tile's LR-partial stage comes after
// FP4 k-tile EMIT_AT (or the last one), by when its epilogue has parked its
// output.  kind 0: FP4 k-tile idx; 1: low-rank chunk idx; 2: the partial.
struct Iter {
  int kind, idx;
};
__device__ __forceinline__ Iter iter_of(int it, int nk, bool with_part) {
  if (!with_part) return it < nk ? Iter{0, it} : Iter{1, it - nk};
  const int at = min(EMIT_AT, nk - 1) + 1;
  if (it < at) return Iter{0, it};
  if (it == at) return Iter{2, 0};
  return it - 1 < nk ? Iter{0, it - 1} : Iter{1, it - 1 - nk};
}

// Emit mode: the stash holds the tile's 256 bf16 columns in the order the
// epilogue warps park them (warp column set ch, then the 128-column half),
// i.e. stash position p holds tile column p with bits 6 and 7 swapped: the
// 64-wide block q of the stash is column block (q & 1) * 2 + (q >> 1).
__device__ __forceinline__ uint32_t stash_block(uint32_t q) { return ((q & 1u) << 1) | (q >> 1); }

}  // namespace

// MODE 0: the layer.  MODE 1 (emit): instead of Y, write the next layer's
// kernel-1 outputs from this layer's bf16 output (see K2Params::Next).
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmLR, const __grid_constant__ CUtensorMap tmL2,
                      K2Params p) {
  constexpr bool EMIT = MODE == 1;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(base + STAGES * STAGE_BYTES);
  float* inv_tab2 = reinterpret_cast<float*>(base + STAGES * STAGE_BYTES + BIAS_BYTES);
  float* invl_s = reinterpret_cast<float*>(base + STAGES * STAGE_BYTES + BIAS_BYTES + TAB_BYTES);
  Ctl* ctl = reinterpret_cast<Ctl*>(base + STAGES * STAGE_BYTES + BIAS_BYTES + TAB_BYTES + INVL_BYTES);
  volatile int* abort_flag = &ctl->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p.nl) {
      tma_prefetch_desc(&tmLR);
      tma_prefetch_desc(&tmL2);
    }
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
    }
    mbar_init(smem_u32(&ctl->tfull), 1);
    mbar_init(smem_u32(&ctl->tempty), EPI_WARPS);
    mbar_init(smem_u32(&ctl->stash_full), EPI_WARPS);
    mbar_init(smem_u32(&ctl->part_full), 1);
    mbar_init(smem_u32(&ctl->part_empty), EPI_WARPS);
    ctl->abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  if (EMIT && threadIdx.x >= 64 && threadIdx.x < 192)
    inv_tab2[threadIdx.x - 64] = nvfp4_inv_entry((uint32_t)(threadIdx.x - 64), p.next.s_t);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  grid_launch_dependents();
  grid_dependency_wait();   // qX, sX and LR from kernel 1 are visible from here

  const int num_tiles = p.num_m_blocks * p.num_n_blocks;
  const int kiters = p.nk + p.nl;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int prev_nb = -1;   // emit mode: the previous tile's column block
      // the weight tiles (codes and scales) stay in L2 ahead of the streamed
      // activations and outputs: every row block's CTA reads them again
      const uint64_t keep = l2_policy_evict_last();
      // one more pass of the loop in emit mode: the last tile's partial stage
      for (int tile = blockIdx.x; ok && (tile < num_tiles || (EMIT && prev_nb >= 0)); tile += gridDim.x) {
        const bool last = tile >= num_tiles;
        int mb = 0, nb = 0;
        if (!last) tile_coords(tile, p.num_m_blocks, p.num_n_blocks, mb, nb);
        const bool with_part = EMIT && prev_nb >= 0;
        const int n_it = last ? 1 : kiters + (with_part ? 1 : 0);
        for (int it = 0; it < n_it; ++it) {
          if (!mbar_wait(smem_u32(&ctl->empty[stage]), phase ^ 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t st = smem_u32(base + stage * STAGE_BYTES);
          const uint32_t bar = smem_u32(&ctl->full[stage]);
          const Iter I = last ? Iter{2, 0} : iter_of(it, p.nk, with_part);
          if (I.kind == 0) {
            const int kt = I.idx;
            mbar_arrive_expect_tx(bar, STAGE_BYTES);
            tma_load_2d(st, &tmA, kt * 128, mb * BLOCK_M, bar);
            tma_load_2d_hint(st + A_BYTES, &tmB, kt * 128, nb * BLOCK_N, bar, keep);
            bulk_load(st + A_BYTES + B_BYTES, p.sX + ((size_t)mb * p.nk + kt) * SFA_BYTES, SFA_BYTES, bar);
            bulk_load_hint(st + A_BYTES + B_BYTES + SFA_BYTES, p.sR + ((size_t)nb * p.nk + kt) * SFB_BYTES,
                           SFB_BYTES, bar, keep);
          } else if (I.kind == 1) {
            mbar_arrive_expect_tx(bar, A_BYTES + B_BYTES);
            tma_load_2d(st, &tmLR, I.idx * 64, mb * BLOCK_M, bar);
            tma_load_2d(st + A_BYTES, &tmL2, I.idx * 64, nb * BLOCK_N, bar);
          } else {
            // the next layer's L1 rows of the previous tile's 256 columns:
            // four staged [r_tot x 64] boxes, contiguous
            const uint32_t bytes = 4u * (uint32_t)p.next.r_tot * 128u;
            mbar_arrive_expect_tx(bar, bytes);
            bulk_load(st, p.next.L1t + (size_t)prev_nb * 4 * p.next.r_tot * 64, bytes, bar);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        prev_nb = last ? -1 : nb;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      bool prev = false;            // emit mode: a previous tile's partial is still to come
      uint32_t part_phase = 0;      // emit mode: stash_full / part_full / part_empty uses
      const uint32_t idesc_p = EMIT ? idesc_bf16_f32(BLOCK_M, p.next.r_tot) : 0u;
      // the next layer's LR partial of the previous tile: A = the parked bf16
      // output (TMEM), B = its L1 rows (the stage), D = DPART_COL
      auto partial = [&](uint32_t a) -> bool {
        if (!mbar_wait(smem_u32(&ctl->stash_full), part_phase, abort_flag, p.err) ||
            !mbar_wait(smem_u32(&ctl->part_empty), part_phase ^ 1, abort_flag, p.err))
          return false;
        tc_fence_after();
        const uint32_t box = (uint32_t)p.next.r_tot * 128u;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          mma_bf16_ta(tmem + DPART_COL, tmem + STASH_COL + 8 * j,
                      desc_k_sw128(a + stash_block((uint32_t)j >> 2) * box + 32 * (j & 3)), idesc_p, j != 0);
        return true;
      };
      for (int tile = blockIdx.x; ok && (tile < num_tiles || (EMIT && prev)); tile += gridDim.x) {
        const bool last = tile >= num_tiles;
        const bool with_part = EMIT && prev;
        if (!last) {
          if (!mbar_wait(smem_u32(&ctl->tempty), acc_phase ^ 1, abort_flag, p.err)) break;
          tc_fence_after();
        }
        const int n_it = last ? 1 : kiters + (with_part ? 1 : 0);
        for (int it = 0; it < n_it; ++it) {
          if (!mbar_wait(smem_u32(&ctl->full[stage]), phase, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(base + stage * STAGE_BYTES);
          const uint32_t b = a + A_BYTES;
          const Iter I = last ? Iter{2, 0} : iter_of(it, p.nk, with_part);
          if (I.kind == 0) {
            const uint32_t sfa = b + B_BYTES, sfb = sfa + SFA_BYTES;
            // six copies of 8 columns: SFA k-blocks (0,1), (2,3); SFB k-block kb, both row halves
#pragma unroll
            for (int j = 0; j < 2; ++j) tmem_cp_sf_block(tmem + SFA_COL + 8 * j, sfa + j * SF_BLOCK);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) tmem_cp_sf_block(tmem + SFB_COL + 8 * kb, sfb + kb * SF_BLOCK);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb)
              mma_nvf4(tmem + ACC_COL, desc_k_sw128(a + 32 * kb), desc_k_sw128(b + 32 * kb), IDESC_F4,
                       tmem + SFA_COL + 4 * kb, tmem + SFB_COL + 8 * kb, (I.idx | kb) != 0);
          } else if (I.kind == 1) {
            const int steps = min(4, (p.r_tot - 64 * I.idx) / 16);
            for (int j = 0; j < steps; ++j)
              mma_bf16(tmem + ACC_COL, desc_k_sw128(a + 32 * j), desc_k_sw128(b + 32 * j), IDESC_BF, 1);
          } else {
            if (!partial(a)) {
              ok = false;
              break;
            }
          }
          tc_commit(smem_u32(&ctl->empty[stage]));
          if (I.kind == 2) {
            tc_commit(smem_u32(&ctl->part_full));
            part_phase ^= 1;
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok || last) break;
        tc_commit(smem_u32(&ctl->tfull));
        acc_phase ^= 1;
        prev = true;
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Warp e = warp - 2 drains TMEM lanes 32 (warp % 4) .. +31 (its sub-partition),
    // the 64-column blocks 2 k + e / 4, k = 0, 1, as four 32-column chunks
    // c (block c / 2, half c % 2; the two warps of a sub-partition interleave
    // by 64 columns, so in emit mode each owns whole scale blocks): all four
    // loads are issued before one wait, the accumulator is released at once,
    // and the bias / GELU / bf16 / store work then overlaps the MMAs of the
    // next tile.
    const int e = warp - 2, sub = warp & 3, ch = e >> 2;
    const int row = sub * 32 + lane;
    float* bslice = bias_s + e * 128;
    float* ilslice = invl_s + e * 128;
    // per-call activation tensor scale: alpha = s_tX s_tR = 2^j from the amax
    // partials (kernel 1 scaled LR to match)
    const float alpha =
        p.amax_parts ? exp2i_f32(dyn_scale_exponent(warp_amax_bits(p.amax_parts, p.n_parts, lane), p.s_tR))
                     : p.alpha;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.num_m_blocks, p.num_n_blocks, mb, nb);
      const int n0 = nb * BLOCK_N + ch * 64;   // chunk c covers n0 + 128 (c / 2) + 32 (c % 2) .. +31
      // this warp's 128 bias values, staged before the accumulator is ready
      const int nl = n0 + 128 * (lane >> 4) + 32 * ((lane >> 3) & 1) + 4 * (lane & 7);   // value 4 lane of the slice
      const float4 bv = __ldg(reinterpret_cast<const float4*>(p.bias + nl));
      // emit mode: the next layer's 1/lambda for the same columns (zeros past its K)
      float4 ilv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (EMIT && nl < p.N) ilv = __ldg(reinterpret_cast<const float4*>(p.next.inv_lambda + nl));
      __syncwarp();
      reinterpret_cast<float4*>(bslice)[lane] = bv;
      if (EMIT) reinterpret_cast<float4*>(ilslice)[lane] = ilv;
      __syncwarp();
      if (!mbar_wait(smem_u32(&ctl->tfull), acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      uint32_t r[4][32];
      const uint32_t taddr = tmem + ((uint32_t)(sub * 32) << 16) + ACC_COL + ch * 64;
      tmem_ld32(taddr, r[0]);
      tmem_ld32(taddr + 32, r[1]);
      tmem_ld32(taddr + 128, r[2]);
      tmem_ld32(taddr + 160, r[3]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ctl->tempty));
      acc_phase ^= 1;
      const int m = mb * BLOCK_M + row;
      if (!EMIT) {
        if (m < p.M) {
          __nv_bfloat16* yrow = p.Y + (size_t)m * p.N;
          // 16 columns (32 bytes, one full sector) per store
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int col = c * 32 + q * 16;   // in bslice
              const int n = n0 + 128 * (c >> 1) + 32 * (c & 1) + q * 16;
              if (n < p.N) {
                float y[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                  y[j] = fmaf(alpha, __uint_as_float(r[c][q * 16 + j]), bslice[col + j]);
                  if (p.epi == 1) y[j] = gelu_tanh(y[j]);
                }
                uint32_t o[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
                st_global_v8(yrow + n, o);
              }
            }
          }
        }
      } else {
        // ------------------------------------------------ the next layer's kernel 1 on this tile
        // x2 = bf16(y) is the next layer's activation: its 16-column groups
        // here are its NVFP4 groups (codes and replicated scales exactly as
        // kernel 1 writes them), and sum_n x2[m,n] L1f2[n,:] over this
        // warp's 128 columns is a partial of its LR
        const K2Params::Next& nx = p.next;
        const size_t qrow = (size_t)p.N_pad / 2;
        // phase A: the row slice to bf16 pairs, parked in free TMEM columns of
        // this warp's lanes (the fp32 accumulator registers are free after it)
        const uint32_t stash = tmem + ((uint32_t)(sub * 32) << 16) + STASH_COL + ch * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            float y0 = fmaf(alpha, __uint_as_float(r[c][j]), bslice[c * 32 + j]);
            float y1 = fmaf(alpha, __uint_as_float(r[c][j + 1]), bslice[c * 32 + j + 1]);
            if (p.epi == 1) {
              y0 = gelu_tanh(y0);
              y1 = gelu_tanh(y1);
            }
            pk[j / 2] = pack_bf16x2(y0, y1);
          }
          tmem_st16(stash + c * 16, pk);
        }
        tmem_wait_st();
        // the MMA warp may now run the LR partial over the whole tile with the
        // parked pairs as its A operand
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->stash_full));
        // phase B2: codes and scales, the whole stash in two loads and one wait
        {
          uint32_t pa[32], pb[32];
          tmem_ld32(stash, pa);
          tmem_ld32(stash + 32, pb);
          tmem_wait_ld();
          uint32_t sword = 0u, cw[8];
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const int n = n0 + 128 * (g >> 2) + 16 * (g & 3);
            float xb[16];
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const uint32_t b2 = g < 4 ? pa[g * 8 + j / 2] : pb[(g - 4) * 8 + j / 2];
              xb[j] = __uint_as_float(b2 << 16);
              xb[j + 1] = __uint_as_float(b2 & 0xFFFF0000u);
            }
            // quantize x^2 = fl32(x2 / lambda2) (zero 1/lambda2 past the next layer's K)
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              const float4 il = *reinterpret_cast<const float4*>(ilslice + g * 16 + j);
              v[j] = __fmul_rn(xb[j], il.x);
              v[j + 1] = __fmul_rn(xb[j + 1], il.y);
              v[j + 2] = __fmul_rn(xb[j + 2], il.z);
              v[j + 3] = __fmul_rn(xb[j + 3], il.w);
            }
            uint2 codes;
            uint32_t sc;
            quant_nvfp4_16_tab(v, nx.six_st, inv_tab2, codes, sc);
            sword |= sc << (8 * (g & 3));
            cw[2 * (g & 3)] = codes.x;
            cw[2 * (g & 3) + 1] = codes.y;
            if ((g & 3) == 3) {   // one 64-column block: 32 bytes of codes, one scale word in four replicas
              const int kb = (n - 48) / 64;
              if (m < p.M) st_global_v8(nx.qX + (size_t)m * qrow + kb * 32, cw);
              const uint32_t wv = m < p.M ? sword : 0u;
#pragma unroll
              for (int rep = 0; rep < 4; ++rep)
                *reinterpret_cast<uint32_t*>(nx.sX + sfx_rep_offset(m, kb, rep, p.N_pad)) = wv;
              sword = 0u;
            }
          }
        }
        // the LR partial of this tile (sum over its 256 columns), once the MMA
        // warp has computed it: the two warps of a sub-partition take half of
        // the r_tot columns each, then hand the TMEM columns back
        if (!mbar_wait(smem_u32(&ctl->part_full), acc_phase ^ 1, abort_flag, p.err)) break;
        tc_fence_after();
        {
          const int half = nx.r_tot / 2, c0 = ch * half;   // a multiple of 8
          float* prow = nx.part + ((size_t)nb * (p.num_m_blocks * BLOCK_M) + m) * LR_PART_STRIDE + c0;
          const uint32_t dsrc = tmem + ((uint32_t)(sub * 32) << 16) + DPART_COL + (uint32_t)c0;
          for (int c8 = 0; c8 < half; c8 += 8) {
            uint32_t d[8];
            tmem_ld8(dsrc + (uint32_t)c8, d);
            tmem_wait_ld();
            reinterpret_cast<uint4*>(prow + c8)[0] = make_uint4(d[0], d[1], d[2], d[3]);
            reinterpret_cast<uint4*>(prow + c8)[1] = make_uint4(d[4], d[5], d[6], d[7]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ctl->part_empty));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

cudaError_t launch_gemm_nvfp4(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmLR,
                              const CUtensorMap& tmL2, K2Params p, int num_sms, cudaStream_t stream, bool emit_next) {
  void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const CUtensorMap, K2Params) =
      emit_next ? gemm_nvfp4_kernel<1> : gemm_nvfp4_kernel<0>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = p.num_m_blocks * p.num_n_blocks;
  const int grid = tiles < num_sms ? tiles : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, tmLR, tmL2, p);
}

__global__ void next_lr_reduce_kernel(const float* __restrict__ part, int parts, int M, int M_128, int r_tot, int r_pad,
                                      __nv_bfloat16* LR) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * r_pad) return;
  const int m = i / r_pad, c = i - m * r_pad;
  float acc = 0.f;
  if (c < r_tot)
    for (int q = 0; q < parts; ++q) acc += part[((size_t)q * M_128 + m) * LR_PART_STRIDE + c];   // fixed order
  LR[i] = __float2bfloat16_rn(acc);
}

cudaError_t launch_next_lr_reduce(const float* part, int parts, int M, int M_128, int r_tot, int r_pad,
                                  __nv_bfloat16* LR, cudaStream_t stream) {
  const int n = M * r_pad;
  next_lr_reduce_kernel<<<(n + 255) / 256, 256, 0, stream>>>(part, parts, M, M_128, r_tot, r_pad, LR);
  return cudaGetLastError();
}

}  // namespace svdq
