// quant_down.cu -- kernel 1: activation quantization fused with the low-rank
// down projection ("Nunchaku engine design" figure (b), "svdq-int4-flux.1-dev"
// model card: the Quantize and Down Projection kernels read the same input,
// so they are fused and X is read from HBM once).
//
// A cluster of S CTAs (S = 2 at large batches, up to 8 at small ones, so that
// the grid still fills the SMs; 1 when a split grid would need two waves)
// owns 64 rows of X; CTA c of the cluster walks
// the c-th of S slices of K in 256-column stages.  A producer warp keeps a TMA ring of
// stages in flight; a stage holds the [64 x 256] bf16 tile of X (four
// 128-byte-swizzled [64 x 64] boxes: 512 contiguous bytes of every row, which
// HBM streams faster than 256), the matching [r_tot x 256] tile of L1f^T
// (stored pre-swizzled, one contiguous bulk copy) and the 256 values of
// 1/lambda.
// From the same staged tile:
//   * 16 quantizer warps: every thread two 16-element groups of one row
//     (x^ = x / lambda, amax, block scale, 4-bit codes), written packed with
//     scales in the layout kernel 2's tensor-core MMA consumes;
//   * two threads (of two warps) issue the down projection on the
//     5th-generation tensor core: A = the staged X tile (M = 64 rows), B = the
//     L1f^T tile (N = r_tot), the lower and the upper 128 columns of every
//     stage into two fp32 TMEM accumulators across the CTA's slice of K.
// At the end four warps move the partial [64 x r_tot] tile (the sum of the two
// accumulators) from TMEM to shared memory; after a cluster barrier CTA c
// adds the S partials of rows
// [64c/S, 64(c+1)/S) through distributed shared memory, always in the order
// CTA 0, 1, .., S-1 (so LR is the same on every run), and stores LR in bf16.
// Why 64 rows: the four-way split of a 128-row tile needs clusters of four,
// and at one CTA per SM only 33 of those are resident at once on 148 SMs;
// 64-row clusters of two fill every SM at the FLUX batch sizes, and small
// batches split K further instead of leaving SMs idle.
// Stages are released through an mbarrier (the 16 quantizer warps plus the
// two MMA commits) instead of a CTA-wide sync, so warps drift apart and overlap
// their load, math and store phases.  The kernel is HBM-bound: per row it
// reads 2K bytes of X and writes about K/2 + K/16 bytes of codes and scales
// plus 2 r_pad bytes of LR.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace svdq {

namespace {

constexpr int BM = K1_BOX_ROWS;              // rows per cluster (= MMA M = TMA box rows)
constexpr int BK = 256;                      // K columns per stage (four 64-column swizzled boxes)
constexpr int QWARPS = 16;                   // quantizer warps: 64 rows x 8 groups
constexpr int THREADS = 32 * (QWARPS + 4);   // + producer warp, two MMA warps, one idle warp
constexpr int X_BOX = BM * 128;              // one [64 x 64] bf16 box, 8 KB
constexpr int X_BYTES = 4 * X_BOX;           // 32 KB
constexpr int IL_BYTES = BK * 4;             // 1/lambda for the stage
// Warp roles.  Warp w runs on SM sub-partition w % 4: the first MMA warp (2)
// and the producer (3) share theirs with three quantizer warps each, so an
// MMA-issuing thread competes with fewer busy warps (kernel 1 alone on QKV
// 14.0 -> 13.3 us); quantizers are warps 0, 1 and 4..17.  A second MMA warp
// (19, sub-partition 3) issues the upper half of every stage's K16 steps into
// an accumulator of its own, which halves the issue work per thread (the
// down projection alone 9.8 -> 8.6 us on QKV); warp 18 has no role.
constexpr int W_PROD = 3, W_MMA = 2, W_Q0 = 4, W_IDLE = 18, W_MMA2 = 19;
constexpr int MAX_STAGES = 8;

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ float4 dsmem_ld_f32x4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

// Address of the 16-byte chunk holding columns [8c, 8c+8) of row `row` in a
// [rows x 64] bf16 box written by TMA with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_chunk(uint32_t box_base, int row, int c) {
  return box_base + row * 128 + ((c ^ (row & 7)) << 4);
}

// Row stride (floats) of the partial LR tile in shared memory: a multiple of
// 4 (16-byte rows) that is 4 or 20 mod 32, so the 16-byte writes of 8
// consecutive rows hit 8 different bank quads.
__host__ __device__ constexpr int part_stride(int r_tot) { return r_tot + 4; }

struct Layout {
  int stages, l_bytes, x_ring, l_ring, il_ring, bar_off;
};

// Shared memory: X ring | L1f^T ring | 1/lambda ring | barriers.  The partial
// LR tile reuses the start of the ring once every stage has been consumed.
__host__ __device__ inline Layout make_layout(int stages, int r_tot, bool do_lr) {
  Layout L;
  L.stages = stages;
  L.l_bytes = do_lr ? 4 * r_tot * 128 : 0;  // r_tot % 16 == 0: 2 KB multiples keep the 1 KB swizzle atoms aligned
  L.x_ring = 0;
  L.l_ring = stages * X_BYTES;
  L.il_ring = L.l_ring + stages * L.l_bytes;
  int end = L.il_ring + stages * IL_BYTES;
  const int part = do_lr ? BM * part_stride(r_tot) * 4 : 0;
  if (part > end) end = part;
  L.bar_off = round_up(end, 16);
  return L;
}

__host__ __device__ constexpr uint32_t tmem_cols_for(int r_tot) {
  return r_tot <= 32 ? 32u : r_tot <= 64 ? 64u : r_tot <= 128 ? 128u : 256u;
}

}  // namespace

// FMT: 0 NVFP4, 1 INT4 (one instantiation per format, so the stage loop has no
// format branches)
template <int FMT>
__global__ void __launch_bounds__(THREADS, 1)
    quant_down_kernel(const __grid_constant__ CUtensorMap tmX, K1Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // slice of K; with the low-rank branch the S CTAs of a row block form a
  // cluster, and the cluster rank equals this index
  const int S = p.ksplit;
  const int split = blockIdx.x % S;
  const int m0 = (blockIdx.x / S) * BM;
  // stages of 256 columns: nk / S each, the first nk % S CTAs one more
  // (possibly none: then the partial LR is zero)
  const int nk = p.K_pad / BK, nq = nk / S, nr = nk % S;
  const int ns = nq + (split < nr ? 1 : 0);
  const int kb0 = split * nq + min(split, nr);           // first 256-column block of this CTA

  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Layout L = make_layout(p.stages, p.r_tot, p.do_lr != 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* dfull = empty + p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* inv_tab = reinterpret_cast<float*>(tmem_slot + 4);        // 128 entries, NVFP4 only
  const uint32_t tmem_cols = tmem_cols_for(p.r_tot);

  if (tid == 0) {
    tma_prefetch_desc(&tmX);
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), (p.do_quant ? QWARPS : 0) + (p.do_lr ? 2 : 0));
    }
    mbar_init(smem_u32(dfull), 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  float* lr_scale_s = inv_tab + 128;                                 // per-call scale only
  if ((FMT == 0) && !p.amax_parts && tid < 128) inv_tab[tid] = nvfp4_inv_entry((uint32_t)tid, p.s_t);
  if (p.do_lr && warp == W_MMA) {
    tmem_alloc(smem_u32(tmem_slot), 2 * tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = p.do_lr ? *tmem_slot : 0u;
  grid_launch_dependents();
  grid_dependency_wait();   // X, the weights and the output buffers are safe to touch from here

  if (warp == W_PROD) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      for (int it = 0, s = 0, ph = 0; it < ns; ++it, s = (s + 1 == p.stages) ? 0 : s + 1, ph ^= (s == 0) ? 1 : 0) {
        if (!mbar_wait(smem_u32(&empty[s]), (uint32_t)ph ^ 1u, abort_flag, p.err)) break;
        const int kb = kb0 + it;
        const uint32_t bar = smem_u32(&full[s]);
        mbar_arrive_expect_tx(bar, X_BYTES + L.l_bytes + IL_BYTES);
#pragma unroll
        for (int b = 0; b < 4; ++b) tma_load_2d(smem_u32(base + L.x_ring + s * X_BYTES + b * X_BOX), &tmX, kb * BK + 64 * b, m0, bar);
        if (p.do_lr)   // the stage's L1f^T tile is stored contiguous and pre-swizzled: one bulk copy
          bulk_load(smem_u32(base + L.l_ring + s * L.l_bytes), p.L1t + (size_t)kb * p.r_tot * BK, L.l_bytes, bar);
        bulk_load(smem_u32(base + L.il_ring + s * IL_BYTES), p.inv_lambda + kb * BK, IL_BYTES, bar);
      }
    }
  } else if (warp == W_MMA || warp == W_MMA2) {
    // ---------------------------------------------------------------- tensor-core down projection
    if (p.do_lr && lane == 0) {
      const int half = warp == W_MMA2 ? 1 : 0;   // K16 steps 8 half .. 8 half + 7 of every stage
      const uint32_t acc = tmem + (uint32_t)half * tmem_cols;
      const uint32_t idesc = idesc_bf16_f32(BM, p.r_tot);
      uint32_t started = 0;
      bool ok = true;
      for (int it = 0, s = 0, ph = 0; it < ns; ++it, s = (s + 1 == p.stages) ? 0 : s + 1, ph ^= (s == 0) ? 1 : 0) {
        if (!mbar_wait(smem_u32(&full[s]), (uint32_t)ph, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kvalid = p.K - (kb0 + it) * BK;      // multiple of 64 (may be <= 0 in the pad)
        // descriptors of the stage's first 16 columns; a K16 step adds its byte
        // offset / 16 to the start-address field (no carry: the shared window
        // is below 256 KB)
        const uint64_t dx = desc_k_sw128(smem_u32(base + L.x_ring + s * X_BYTES));
        const uint64_t dl = desc_k_sw128(smem_u32(base + L.l_ring + s * L.l_bytes));
        const uint32_t lstep = (uint32_t)p.r_tot * 8;   // (r_tot * 128) >> 4
        if (kvalid >= BK) {
#pragma unroll
          for (int jj = 0; jj < BK / 32; ++jj) {
            const int j = 8 * half + jj;
            const uint32_t b = j >> 2, ko = (j & 3) * 2;
            mma_bf16(acc, dx + (b * (X_BOX >> 4) + ko), dl + (b * lstep + ko), idesc, (jj == 0) ? started : 1u);
          }
          started = 1u;
        } else {
          for (int jj = 0; jj < BK / 32; ++jj) {
            const int j = 8 * half + jj;
            if (j * 16 >= kvalid) break;
            const uint32_t b = j >> 2, ko = (j & 3) * 2;
            mma_bf16(acc, dx + (b * (X_BOX >> 4) + ko), dl + (b * lstep + ko), idesc, started);
            started = 1u;
          }
        }
        tc_commit(smem_u32(&empty[s]));
      }
      if (ok) tc_commit(smem_u32(dfull));
    }
  } else if (p.do_quant && warp != W_IDLE) {
    // ---------------------------------------------------------------- quantizers
    // box qb, rows qr and qr + 32, 16-column group qg of the stage: both of a
    // thread's groups use the same 16 values of 1/lambda (read once); a warp
    // covers 8 rows of one box (conflict-free swizzled reads), the four groups
    // of a row sit in one quad of lanes
    const int qw = warp < 2 ? warp : warp - 2;   // quantizer index 0..15
    const int qb = qw & 3, qr = (qw >> 2) * 8 + (lane >> 2), qg = lane & 3;
    float six_st = p.six_st;
    if (p.amax_parts) {
      // per-call tensor scale: every quantizer warp reduces the amax partials
      // (written by the amax pass, visible after the dependency wait), the
      // first four build the 1/scale table, then the 16 warps meet
      const int j = dyn_scale_exponent(warp_amax_bits(p.amax_parts, p.n_parts, lane), p.s_tR);
      const float s_t = __fdiv_rn(exp2i_f32(j), p.s_tR);
      six_st = __fmul_rn(6.f, s_t);
      const int qt = qw * 32 + lane;
      if (qt < 128) inv_tab[qt] = nvfp4_inv_entry((uint32_t)qt, s_t);
      if (qt == 0) {
        *lr_scale_s = exp2i_f32(p.k_alpha - j);
        if (blockIdx.x == 0 && p.dyn_record) {
          p.dyn_record[0] = s_t;
          p.dyn_record[1] = __int_as_float(j);
          p.dyn_record[2] = exp2i_f32(j);
        }
      }
      named_bar_sync(1, 32 * QWARPS);
    }
    // NVFP4: packed codes (K_pad / 2 bytes a row); INT4: one E4M3 byte per code
    const size_t qx_row_bytes = (FMT == 0) ? (size_t)(p.K_pad / 2) : (size_t)p.K_pad;
    // this thread's store addresses at its first stage; each further stage
    // moves them by one 256-column k-tile: codes by 128 (NVFP4) or 256 (INT4)
    // bytes, replicated NVFP4 scales by two 4 KB blocks, INT4 scales by 512 floats
    uint8_t* qxp[2];
    uint8_t* sxp[2];
    bool in_rows[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + qr + 32 * h, kb = 4 * kb0 + qb;
      in_rows[h] = m < p.M;
      qxp[h] = p.qX + (size_t)m * qx_row_bytes + (size_t)kb * ((FMT == 0) ? 32 : 64) + qg * ((FMT == 0) ? 8 : 16);
      sxp[h] = (FMT == 0) ? p.sX + sfx_rep_offset(m, kb, qg, p.K_pad)
                          : p.sX + 4 * int4_scale_offset(m, kb, p.K_pad);
    }
    const size_t qx_step = (FMT == 0) ? 128 : 256, sx_step = (FMT == 0) ? 8192 : 2048;
    for (int it = 0, s = 0, ph = 0; it < ns; ++it, s = (s + 1 == p.stages) ? 0 : s + 1, ph ^= (s == 0) ? 1 : 0) {
      if (!mbar_wait(smem_u32(&full[s]), (uint32_t)ph, abort_flag, p.err)) break;
      // this thread's two groups of the stage: rows qr and qr + 32 of box qb;
      // read both and form x^ = x * (1/lambda) in registers, release the
      // stage, then quantize and store
      float v[2][16];
      const uint32_t box = smem_u32(base + L.x_ring + s * X_BYTES + qb * X_BOX);
      uint32_t w[2][8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 u0 = lds128(sw128_chunk(box, qr + 32 * h, 2 * qg));
        const uint4 u1 = lds128(sw128_chunk(box, qr + 32 * h, 2 * qg + 1));
        w[h][0] = u0.x; w[h][1] = u0.y; w[h][2] = u0.z; w[h][3] = u0.w;
        w[h][4] = u1.x; w[h][5] = u1.y; w[h][6] = u1.z; w[h][7] = u1.w;
      }
      // 1/lambda of this group: chunk q at position 4 q + qg of the 64-column
      // block's permuted copy (zeros past K, where TMA also filled x with zeros)
      const uint32_t ila = smem_u32(base + L.il_ring + s * IL_BYTES) + qb * 256 + qg * 16;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 f = lds128(ila + 64 * q);
#pragma unroll
        for (int h = 0; h < 2; ++h) {   // bf16 pair -> two floats, times 1/lambda
          mul2_rn(__uint_as_float(w[h][2 * q] << 16), __uint_as_float(w[h][2 * q] & 0xFFFF0000u),
                  __uint_as_float(f.x), __uint_as_float(f.y), v[h][4 * q], v[h][4 * q + 1]);
          mul2_rn(__uint_as_float(w[h][2 * q + 1] << 16), __uint_as_float(w[h][2 * q + 1] & 0xFFFF0000u),
                  __uint_as_float(f.z), __uint_as_float(f.w), v[h][4 * q + 2], v[h][4 * q + 3]);
        }
      }
      // every lane has consumed its shared-memory loads of stage s (the products
      // above used them): the slot may be refilled.  A relaxed arrival, so that
      // it does not wait for the previous stage's global stores.
      __syncwarp();
      if (lane == 0) mbar_arrive_relaxed(smem_u32(&empty[s]));
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint2 codes;
        if ((FMT == 0)) {
          uint32_t sc;
          quant_nvfp4_16_tab(v[h], six_st, inv_tab, codes, sc);
          // the row's four scale bytes form one word; kernel 2 wants it in four
          // replicas (one per TMEM sub-partition): lane qg of the quad writes replica qg
          uint32_t sw = sc << (8 * qg);
          sw |= __shfl_xor_sync(0xffffffffu, sw, 1);
          sw |= __shfl_xor_sync(0xffffffffu, sw, 2);
          *reinterpret_cast<uint32_t*>(sxp[h]) = sw;
        } else {
          __half sc;
          quant_int4_16of64(v[h], codes, sc);
          // stored widened to float32 (exact): kernel 2 multiplies in float32
          if (qg == 0) *reinterpret_cast<float*>(sxp[h]) = __half2float(sc);
        }
        if (in_rows[h]) {
          if ((FMT == 0))
            *reinterpret_cast<uint2*>(qxp[h]) = codes;
          else
            *reinterpret_cast<uint4*>(qxp[h]) = int4x16_to_e4m3(codes);
        }
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        qxp[h] += qx_step;
        sxp[h] += sx_step;
      }
    }
  }

  // All stages are consumed (or a wait gave up): the ring can hold the partial tile.
  tc_fence_before();
  __syncthreads();
  if (p.do_lr) {
    const int ps = part_stride(p.r_tot);
    const uint32_t part = smem_u32(base);
    if (warp >= W_Q0 && warp < W_Q0 + 4) {
      // ---------------------------------------------------------------- TMEM -> shared partial
      // M = 64 accumulator: row i in TMEM lane 32 (i / 16) + i % 16, column =
      // rank index; lanes 16-31 of each sub-partition are unused
      const int sub = warp & 3, row = 16 * sub + lane;
      const bool has_mma = ns > 0 && kb0 * BK < p.K;     // else this slice is empty or in the K pad: zeros
      const bool has_mma2 = ns > 0 && p.K - kb0 * BK > BK / 2;   // the second accumulator got at least one step
      if (mbar_wait(smem_u32(dfull), 0, abort_flag, p.err)) {
        tc_fence_after();
        for (int c0 = 0; c0 < p.r_tot; c0 += 32) {
          uint32_t d[32];
          if (has_mma) {
            tmem_ld32(tmem + ((uint32_t)(sub * 32) << 16) + (uint32_t)c0, d);
            if (has_mma2) {
              uint32_t e[32];
              tmem_ld32(tmem + ((uint32_t)(sub * 32) << 16) + tmem_cols + (uint32_t)c0, e);
              tmem_wait_ld();
#pragma unroll
              for (int n = 0; n < 32; ++n) d[n] = __float_as_uint(__uint_as_float(d[n]) + __uint_as_float(e[n]));
            } else {
              tmem_wait_ld();
            }
          } else {
#pragma unroll
            for (int n = 0; n < 32; ++n) d[n] = 0u;
          }
#pragma unroll
          for (int n = 0; n < 32; n += 4)
            if (lane < 16 && c0 + n < p.r_tot) sts128(part + (uint32_t)(row * ps + c0 + n) * 4, d[n], d[n + 1], d[n + 2], d[n + 3]);
        }
      }
    }
    cluster_sync_all();
    // ---------------------------------------------------------------- cluster reduction
    // this CTA's 64 / S rows; four consecutive columns per task; pad columns -> 0
    const int rows_per = BM / S, quads = p.r_pad / 4;
    // per-call scale: LR carries 2^(k_alpha - j) so that kernel 2's single
    // factor 2^j restores it (a power of two: exact before the bf16 rounding)
    const float lrs = p.amax_parts ? *lr_scale_s : 1.f;
    for (int i = tid; i < rows_per * quads; i += THREADS) {
      const int rr = split * rows_per + i / quads, c = (i % quads) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c < p.r_tot) {
        const uint32_t a = part + (uint32_t)(rr * ps + c) * 4;
        for (int q = 0; q < S; ++q) {   // fixed order: CTA 0, 1, .., S-1
          const float4 v = dsmem_ld_f32x4(dsmem_map(a, (uint32_t)q));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        if (p.amax_parts) {
          acc.x *= lrs;
          acc.y *= lrs;
          acc.z *= lrs;
          acc.w *= lrs;
        }
      }
      const int m = m0 + rr;
      if (m < p.M) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(p.LR + (size_t)m * p.r_pad + c) = pk;
      }
    }
    cluster_sync_all();   // no CTA leaves while another still reads its partial
  }

  // Every thread reaches this point, also after a timeout (the loops above
  // leave early when the abort flag is set); TMEM is freed on every path.
  tc_fence_before();
  __syncthreads();
  if (p.do_lr && warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * tmem_cols);
  }
}

size_t quant_down_smem_bytes(int r_tot, bool do_lr, int* stages_out, int ns) {
  // as many stages as fit in 216 KB (large ranks get a single stage)
  const int stage_bytes = X_BYTES + IL_BYTES + (do_lr ? 4 * r_tot * 128 : 0);
  int stages = (216 * 1024) / stage_bytes;
  stages = stages < 1 ? 1 : (stages > MAX_STAGES ? MAX_STAGES : stages);
  if (stages > ns) stages = ns < 1 ? 1 : ns;
  *stages_out = stages;
  const Layout L = make_layout(stages, r_tot, do_lr);
  return (size_t)L.bar_off + 1024 /*alignment slack*/ + 8 * (2 * stages + 1) + 16 + 128 * 4 + 64;
}

namespace {

// Clusters of s CTAs (with `smem` bytes each) that the current device runs at
// once, from the occupancy query, remembered per (device, s, smem).
int resident_clusters(int s, size_t smem, const cudaLaunchConfig_t& base_cfg) {
  struct Entry {
    int dev, s;
    size_t smem;
    int n;
  };
  static std::mutex mu;
  static Entry table[64];
  static int used = 0;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
      if (table[i].dev == dev && table[i].s == s && table[i].smem == smem) return table[i].n;
  }
  cudaLaunchConfig_t cfg = base_cfg;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = s;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)s);
  int n = 0;
  // both instantiations take the same threads and shared memory
  if (cudaOccupancyMaxActiveClusters(&n, quant_down_kernel<0>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (used < 64) table[used++] = Entry{dev, s, smem, n};
  return n;
}

}  // namespace

cudaError_t launch_quant_down(const CUtensorMap& tmX, K1Params p, int num_sms, cudaStream_t stream) {
  // row blocks up to the next multiple of 128, so that every row of the last
  // 128-row scale block gets its (zero) scales
  const int row_blocks = round_up(p.M, 128) / BM, nk = p.K_pad / BK;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(THREADS);
  cfg.stream = stream;
  // K split: 2 (the whole grid in one wave at the FLUX batch sizes); 4 or 8
  // when that still fits in one wave with every cluster resident, so that a
  // small batch spreads over more SMs (each CTA then walks fewer stages);
  // none when even S = 2 would need more than one wave: each CTA then walks
  // all of K and skips the cluster reduction, whose tail every wave would pay
  // (LoRA-sweep layer at M = 16384: 136.0 -> 126.1 us)
  int S = 2 * row_blocks > num_sms ? 1 : 2;
  size_t smem = 0;
  for (int cand = 8; cand >= 2; cand /= 2) {
    if (cand > nk || cand * row_blocks > num_sms) continue;
    smem = quant_down_smem_bytes(p.r_tot, p.do_lr != 0, &p.stages, (nk + cand - 1) / cand);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(quant_down_kernel<0>), smem);
    if (e == cudaSuccess) e = ensure_dynamic_smem(reinterpret_cast<const void*>(quant_down_kernel<1>), smem);
    if (e != cudaSuccess) return e;
    cfg.dynamicSmemBytes = smem;
    if (!p.do_lr || resident_clusters(cand, smem, cfg) >= row_blocks) {
      S = cand;
      break;
    }
  }
  p.ksplit = S;
  smem = quant_down_smem_bytes(p.r_tot, p.do_lr != 0, &p.stages, (nk + S - 1) / S);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;   // never launch past the shared-memory limit
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(quant_down_kernel<0>), smem);
  if (e == cudaSuccess) e = ensure_dynamic_smem(reinterpret_cast<const void*>(quant_down_kernel<1>), smem);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((unsigned)(S * row_blocks));
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.do_lr ? 2 : 1;   // only the LR reduction needs the cluster
  return p.fmt == 0 ? cudaLaunchKernelEx(&cfg, quant_down_kernel<0>, tmX, p)
                    : cudaLaunchKernelEx(&cfg, quant_down_kernel<1>, tmX, p);
}

}  // namespace svdq
