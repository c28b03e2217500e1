// common.cuh -- device building blocks for the SVDQuant W4A4 kernels (sm_100a).
//
// Inline-PTX wrappers for mbarriers, TMA (cp.async.bulk[.tensor]) and the
// 5th-generation tensor core (tcgen05: TMEM allocation, MMA, smem->TMEM copy,
// TMEM loads), bounded waits that report a timeout instead of hanging, and
// the 4-bit group quantizer shared by the activation kernel and the weight
// preparation (so activations and the residual follow one rounding rule).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace svdq {

// ----------------------------------------------------------------- error word
// Bits OR-ed into the per-device error word (see api.cu).
constexpr unsigned ERR_TIMEOUT = 1u;
constexpr unsigned ERR_BOUNDS = 2u;

struct DeviceErr {
  unsigned* word;          // device error word
  unsigned long long limit_ns;  // wait limit for every bounded wait
};

__device__ __forceinline__ void raise_error(const DeviceErr& e, unsigned bits) {
  atomicOr(e.word, bits);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- addresses
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 u;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr));
  return u;
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Arrive without release semantics: does not wait for this thread's earlier
// memory operations (for instance global stores of a previous stage) to be
// performed.  Use only where the data the arrival hands over has already been
// consumed into registers.
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// The suspend-time hint lets a waiting warp sleep until the phase completes
// (or up to 1 ms) instead of polling, so waiting warps leave the issue slots
// to the warps that work.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(1000000u)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Gives up after
// err.limit_ns (or as soon as another thread of the CTA has given up, seen
// through *abort), records ERR_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          const DeviceErr& err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > err.limit_ns) {
      *abort = 1;
      __threadfence_block();
      raise_error(err, ERR_TIMEOUT);
      return false;
    }
  }
}

// ----------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 2-D tiled load of the box at (x = inner coordinate, y = row) into smem.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 3-D tiled load of the box at (x, y, z) into smem.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// An L2 policy for loads whose data should stay in L2 (evict it last): the
// weight tiles of a GEMM, read again by every row block's CTA.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// tma_load_2d with an L2 cache policy (l2_policy_evict_last).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const void* tmap, int x, int y, uint32_t bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// Contiguous bulk copy global -> smem (both 16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// bulk_load with an L2 cache policy.
__device__ __forceinline__ void bulk_load_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                               uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued
// before has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// ----------------------------------------------------------------- programmatic dependent launch
// Kernels 1 and 2 are launched with programmatic stream serialization: a
// kernel may start (set up barriers and TMEM) while the previous kernel on
// the stream is still running, and waits here before its first global
// memory access; the previous kernel's writes are visible after the wait.
// Without that launch attribute both instructions do nothing.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Lets the next kernel on the stream be scheduled onto SMs this grid frees.
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier `id` (1..15; 0 is __syncthreads) over `threads` threads of
// the CTA (a multiple of 32; whole warps).
__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ----------------------------------------------------------------- thread-block clusters
// Every thread of every CTA in the cluster arrives, then waits for all.
// Release/acquire order the shared-memory writes before it against the
// distributed-shared-memory reads after it.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t dsmem_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}


// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"):
//   bits  0-13 start address >> 4, 16-29 leading byte offset >> 4,
//   32-45 stride byte offset >> 4, 46-47 version (1 on sm_100),
//   49-51 base offset, 52 leading-offset mode, 61-63 swizzle mode
//   (0 none, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | ((uint64_t)swizzle << 61);
}

// K-major operand tile with 128-byte rows in the 128-byte swizzle layout
// written by TMA (8-row groups 1024 bytes apart).
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t addr) {
  return smem_desc(addr, 16, 1024, 2);
}

// Instruction descriptor, kind::f16 with bf16 A/B, fp32 accumulate, K-major A and B.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor, kind::mxf4nvf4 block-scaled: E2M1 A/B, UE4M3 scales
// (16-element blocks), K-major A and B, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (0u << 23) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// One 4 KB replicated scale block (see sfx_rep_offset) -> 8 TMEM columns of all 128 lanes.
__device__ __forceinline__ void tmem_cp_sf_block(uint32_t taddr, uint32_t smem_addr) {
  const uint64_t d = smem_desc(smem_addr, 128, 256, 0);
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 8 consecutive 32-bit columns -> 8 registers per thread.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes <- 16 registers per thread.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}


// ----------------------------------------------------------------- conversions
// Eight floats -> eight E2M1 codes in one word (element j in bits 4j..4j+3),
// round to nearest even, saturate to +-6, sign kept.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float x0, float x1, float x2, float x3, float x4,
                                               float x5, float x6, float x7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
  return r;
}

// Non-negative float -> E4M3 byte, round to nearest even, saturate to 448.
__device__ __forceinline__ uint32_t cvt_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  // E4M3 -> f32 exactly: bias 7, 3 mantissa bits, subnormals at 2^-9 steps.
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  float v = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
  return (code & 0x80u) ? -v : v;
}

// ----------------------------------------------------------------- packed float32 helpers
// Two IEEE float32 multiplies (round to nearest even) in one instruction.
__device__ __forceinline__ void mul2_rn(float a0, float a1, float b0, float b1, float& r0, float& r1) {
  uint64_t a, b, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}



__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max |v_j| over 16 values
__device__ __forceinline__ float absmax16(const float (&v)[16]) {
  float a = max3f(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
  a = max3f(a, fabsf(v[3]), fabsf(v[4]));
  a = max3f(a, fabsf(v[5]), fabsf(v[6]));
  a = max3f(a, fabsf(v[7]), fabsf(v[8]));
  a = max3f(a, fabsf(v[9]), fabsf(v[10]));
  a = max3f(a, fabsf(v[11]), fabsf(v[12]));
  a = max3f(a, fabsf(v[13]), fabsf(v[14]));
  return fmaxf(a, fabsf(v[15]));
}

// GELU, tanh form: 0.5 y (1 + tanh(u)) with u = sqrt(2/pi) (y + 0.044715 y^3),
// evaluated as the equal y / (1 + e^(-2u)), e^(-2u) = 2^(-2u log2 e), with
// the hardware base-2 exponential and reciprocal approximations (relative
// error near 1e-6, far inside the layer's bf16 output): two special-function
// instructions instead of a full-precision tanh.  Large negative y: the
// exponential overflows to +inf and the result is -0.
__device__ __forceinline__ float gelu_tanh(float y) {
  constexpr float kTwoULog2e = 2.302208198144325f;   // 2 sqrt(2/pi) log2(e)
  const float z = y * fmaf(0.044715f * y, y, 1.0f);   // y + 0.044715 y^3
  float t, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(-kTwoULog2e * z));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + t));
  return y * r;
}

// ----------------------------------------------------------------- 4-bit group quantizers
// NVFP4, one 16-element group: a = max|v|; sb = E4M3(a / six_st) with six_st
// = fl32(6 s_t); d = fl32(f32(sb) s_t); inv = fl32(1/d) (0 if d == 0);
// code_j = E2M1(fl32(v_j inv)), sign kept.  Returns the 16 codes packed in 8
// bytes (element 2j in the low nibble of byte j) and the scale byte.
__device__ __forceinline__ void quant_nvfp4_16(const float (&v)[16], float s_t, float six_st,
                                               uint2& codes, uint32_t& scale) {
  const float a = absmax16(v);
  const uint32_t sb = cvt_e4m3(__fdiv_rn(a, six_st));
  const float d = __fmul_rn(e4m3_to_f32(sb), s_t);
  const float inv = (d == 0.f) ? 0.f : __frcp_rn(d);
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float x[8];
#pragma unroll
    for (int j = 0; j < 8; j += 2) mul2_rn(v[8 * h + j], v[8 * h + j + 1], inv, inv, x[j], x[j + 1]);
    // the converter keeps the sign of a negative value that rounds to zero
    // (code 0x8), the same rule as the definition; the exhaustive bf16 sweep
    // in the GPU tests checks it
    w[h] = cvt_e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
  }
  codes = make_uint2(w[0], w[1]);
  scale = sb;
}

// The same NVFP4 group quantizer with the per-code reciprocal taken from a
// table: inv_tab[c] = fl32(1 / fl32(f32(E4M3 c) s_t)) (0 where that product
// is 0), built once with exactly the operations above, so the codes are
// bit-identical to quant_nvfp4_16.
__device__ __forceinline__ float nvfp4_inv_entry(uint32_t code, float s_t) {
  const float d = __fmul_rn(e4m3_to_f32(code), s_t);
  return (d == 0.f) ? 0.f : __frcp_rn(d);
}

__device__ __forceinline__ void quant_nvfp4_16_tab(const float (&v)[16], float six_st, const float* inv_tab,
                                                   uint2& codes, uint32_t& scale) {
  const float a = absmax16(v);
  const uint32_t sb = cvt_e4m3(__fdiv_rn(a, six_st));
  const float inv = inv_tab[sb];
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float x[8];
#pragma unroll
    for (int j = 0; j < 8; j += 2) mul2_rn(v[8 * h + j], v[8 * h + j + 1], inv, inv, x[j], x[j + 1]);
    w[h] = cvt_e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
  }
  codes = make_uint2(w[0], w[1]);
  scale = sb;
}

// INT4, one 64-element group held as 4 x 16 values by 4 cooperating lanes
// (lanes l, l^1, l^2, l^3 of one quad): sb = fp16(fl32(a / 7)),
// d = f32(sb), inv = fl32(1/d) (0 if d == 0), code = clamp(rint(fl32(v inv)), -8, 7).
// Each lane returns its 16 codes as 8 bytes (two's-complement nibbles).
__device__ __forceinline__ void quant_int4_16of64(const float (&v)[16], uint2& codes,
                                                  __half& scale) {
  float a = absmax16(v);
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  const __half sb = __float2half_rn(__fdiv_rn(a, 7.0f));
  const float d = __half2float(sb);
  const float inv = (d == 0.f) ? 0.f : __frcp_rn(d);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    int q = __float2int_rn(__fmul_rn(v[j], inv));
    q = max(-8, min(7, q));
    w[j >> 3] |= ((uint32_t)q & 0xFu) << ((j & 7) * 4);
  }
  codes = make_uint2(w[0], w[1]);
  scale = sb;
}

// INT4 codes in FP8 E4M3 containers (E4M3 holds -8..7 exactly), the operand
// form of the INT4 tensor-core product.  Table: E4M3 bytes of the two's
// complement codes 0..7 (values 0..7) and 8..15 (values -8..-1), code c at
// byte c % 4 of its word.
constexpr uint32_t E4M3_POS_LO = 0x44403800u, E4M3_POS_HI = 0x4E4C4A48u;   // 0, 1, 2, 3 | 4, 5, 6, 7
constexpr uint32_t E4M3_NEG_LO = 0xCACCCED0u, E4M3_NEG_HI = 0xB8C0C4C8u;   // -8, -7, -6, -5 | -4, -3, -2, -1
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}
// The four codes in the low 16 bits of sel (k order, low nibble first) ->
// four E4M3 bytes (k order): look up code & 7 in both halves of the table,
// then pick per byte by bit 3 of the code.
__device__ __forceinline__ uint32_t int4x4_to_e4m3(uint32_t sel) {
  const uint32_t s7 = sel & 0x7777u;
  const uint32_t pos = prmt_b32(E4M3_POS_LO, E4M3_POS_HI, s7), neg = prmt_b32(E4M3_NEG_LO, E4M3_NEG_HI, s7);
  return prmt_b32(pos, neg, ((sel >> 1) & 0x4444u) | 0x3210u);
}
// 16 packed codes (8 bytes, element 2j in the low nibble of byte j) -> 16 E4M3 bytes.
__device__ __forceinline__ uint4 int4x16_to_e4m3(uint2 c) {
  return make_uint4(int4x4_to_e4m3(c.x), int4x4_to_e4m3(c.x >> 16), int4x4_to_e4m3(c.y), int4x4_to_e4m3(c.y >> 16));
}

// Byte offset of (row, 16-group) inside the tcgen05 scale-factor layout:
// 512-byte atoms of 128 rows x 4 groups, ordered (row block, 64-k block).
__host__ __device__ __forceinline__ size_t sf_atom_offset(int row, int g16, int kpad) {
  const int rb = row >> 7, kb = g16 >> 2;
  return ((size_t)rb * (kpad >> 6) + kb) * 512 + (size_t)(row & 31) * 16 + ((row & 127) >> 5) * 4 +
         (g16 & 3);
}

// NVFP4 scales as kernel 2 moves them into TMEM: 4 KB blocks, each the
// source of one tcgen05.cp.128x256b (128 lanes x 32 bytes, canonical
// no-swizzle K-major form: 8-lane groups 256 bytes apart, the two 16-byte
// halves of a lane 128 bytes apart).  Lane L carries row L % 32 of two scale
// atoms (each the 16 bytes of rows r, r+32, r+64, r+96 x 4 groups), so all
// four TMEM sub-partitions receive every atom, as the block-scaled MMA reads
// them.  One copy per 8 TMEM columns instead of one per 4: the scale copies
// cost per instruction.
//   activations: per (128-row block, 256-wide k-tile) two blocks; block j
//     holds 64-k blocks 2j (first half) and 2j+1 (second half);
//   weights: per (256-row block, 256-wide k-tile) four blocks; block kb holds
//     64-k block kb of rows 0-127 (first half) and of rows 128-255 (second).
// These return the byte offset of the word with the four scales of (row, 64-k
// block kb) in replica q (0..3).
__host__ __device__ __forceinline__ size_t sfx_rep_offset(int row, int kb, int q, int kpad) {
  const int rb = row >> 7, r = row & 127, kt = kb >> 2, kin = kb & 3, lane = (r & 31) + 32 * q;
  return (((size_t)rb * (kpad >> 8) + kt) * 2 + (kin >> 1)) * 4096 + (size_t)(lane >> 3) * 256 + (kin & 1) * 128 +
         (lane & 7) * 16 + (r >> 5) * 4;
}
__host__ __device__ __forceinline__ size_t sfw_rep_offset(int row, int kb, int q, int kpad) {
  const int nb = row >> 8, h = (row >> 7) & 1, r = row & 127, kt = kb >> 2, kin = kb & 3, lane = (r & 31) + 32 * q;
  return (((size_t)nb * (kpad >> 8) + kt) * 4 + kin) * 4096 + (size_t)(lane >> 3) * 256 + h * 128 + (lane & 7) * 16 +
         (r >> 5) * 4;
}

// Element offset of (row, 64-group) in the INT4 scale layout (binary16
// values stored widened to float32):
// 512-byte chunks of 128 rows x 2 groups (one 128-wide k-tile), ordered
// (row block, k-tile), group-major inside a chunk.
__host__ __device__ __forceinline__ size_t int4_scale_offset(int row, int g64, int kpad) {
  return (((size_t)(row >> 7) * (kpad >> 7) + (g64 >> 1)) * 2 + (g64 & 1)) * 128 + (row & 127);
}

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

// ----------------------------------------------------------------- per-call NVFP4 activation tensor scale
// (the FP32 tensor scale of the "SVDQuant" paper's NVFP4 setting, chosen from
// the call's own amax(|X^|) instead of the calibrated value)
//
// Largest of n <= 1024 non-negative float32 values kept as their bit
// patterns (for those the integer order is the float order), reduced by one
// warp.  The values were written by an earlier kernel: read through L2, all
// loads issued before the first is used (one L2 round trip, not n / 32).
__device__ __forceinline__ uint32_t warp_amax_bits(const uint32_t* parts, int n, int lane) {
  uint32_t v[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) v[t] = (lane + 32 * t < n) ? __ldcg(parts + lane + 32 * t) : 0u;
  uint32_t m = 0;
#pragma unroll
  for (int t = 0; t < 32; ++t) m = max(m, v[t]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// j = the smallest integer with 2^j >= s_tR a / 2688 (a = 0 counts as 2688),
// evaluated in float64, where a s_tR is exact and the division is IEEE
// round-to-nearest; then s_tX = fl32(2^j / s_tR) and s_tX s_tR is 2^j up to
// one float32 rounding, so no activation block scale exceeds 448.
__device__ __forceinline__ int dyn_scale_exponent(uint32_t amax_bits, float s_tR) {
  const float a = __uint_as_float(amax_bits);
  const double x = (a > 0.f ? (double)a : 2688.0) * (double)s_tR / 2688.0;
  const unsigned long long b = (unsigned long long)__double_as_longlong(x);
  const int e = (int)((b >> 52) & 0x7FF) - 1023;   // x is a normal float64: x >= 2^-298
  return (b & 0xFFFFFFFFFFFFFull) ? e + 1 : e;     // x = 2^e exactly, else round up
}

// fl32(2^j): exact for -149 <= j <= 127, infinity above, zero below.
__device__ __forceinline__ float exp2i_f32(int j) {
  if (j > 127) return __uint_as_float(0x7F800000u);
  if (j >= -126) return __uint_as_float((uint32_t)(j + 127) << 23);
  if (j >= -149) return __uint_as_float(1u << (j + 149));
  return 0.f;
}

}  // namespace svdq
