// kernels.h -- launch interfaces between the host API (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "svdq.h"

namespace svdq {

// Raises `kernel`'s dynamic shared-memory limit on the current device to at
// least `bytes`, calling the runtime only the first time a larger limit is
// needed (the call costs microseconds of host time, more than a small
// kernel's launch).
cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes);

// SVDQ_OK when the current device is supported (compute capability 10.0)
// and holds the handle `w`; the status any entry point would return otherwise.
svdq_status handle_device_status(const svdq_weights* w);

// ---------------------------------------------------------------- kernel 1
struct K1Params {
  int M, K, K_pad, r_tot, r_pad;
  int fmt;                 // 0 NVFP4, 1 INT4
  int do_quant, do_lr;     // fused: both; unfused baseline: one of them
  int stages;              // set by the launcher
  int ksplit;              // CTAs per row block (the cluster with the low-rank branch), set by the launcher
  const float* inv_lambda; // [K_pad], permuted per 64-wide stage (see prepare.cu)
  const __nv_bfloat16* L1t; // L1f^T in the staged layout (one contiguous tile per stage)
  float s_t, six_st;       // NVFP4 activation tensor scale and fl32(6 s_t)
  // per-call NVFP4 tensor scale (null: s_t above): the amax partials of X^,
  // reduced after the grid-dependency wait; s_t = fl32(2^j / s_tR) and LR
  // leaves scaled by 2^(k_alpha - j), where 2^k_alpha is the prepared alpha
  const uint32_t* amax_parts;
  int n_parts, k_alpha;
  float s_tR;
  float* dyn_record;       // if set, CTA 0 writes {s_t, j as int32 bits, 2^j}
  uint8_t* qX;             // [M][K_pad/2]
  uint8_t* sX;             // scale layout (see svdq.h)
  __nv_bfloat16* LR;       // [M][r_pad]
  DeviceErr err;
};
// Kernel 1 stages X in [K1_BOX_ROWS x 64] bf16 TMA boxes (128-byte swizzle);
// the host encodes tmX with exactly this box.
constexpr int K1_BOX_ROWS = 64;
cudaError_t launch_quant_down(const CUtensorMap& tmX, K1Params p, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- kernel 2
struct K2Params {
  int M, N, K_pad, r_tot, r_pad, N_pad;
  int num_m_blocks, num_n_blocks;
  int nk;                  // K_pad / 256 4-bit k-tiles
  int nl;                  // r_pad / 64 low-rank k-tiles (0: plain W4A4 GEMM)
  const uint8_t* sX;       // activation scales, replicated layout (sfx_rep_offset)
  const uint8_t* sR;       // weight scales, replicated layout (sfw_rep_offset)
  const float* bias;       // [N_pad]
  float alpha;             // s_tX * s_tR
  const uint32_t* amax_parts;  // per-call tensor scale: alpha = 2^j from these (null: alpha above)
  int n_parts;
  float s_tR;
  int epi;                 // 0 none, 1 GELU (tanh form)
  __nv_bfloat16* Y;        // [M][N]
  DeviceErr err;
  // Emit mode (the next layer's kernel-1 outputs instead of Y): this
  // layer's bf16 output Y is the next layer's activation X2 (its K = N)
  struct Next {
    const float* inv_lambda;   // [N] the next layer's 1/lambda
    const __nv_bfloat16* L1t;  // its first factor (with any LoRA A) in kernel 1's staged layout: per 64 rows
                               // of K one [r_tot x 64] bf16 box, 128-byte swizzled (a K-major MMA B operand)
    float s_t, six_st;         // its static NVFP4 activation tensor scale and fl32(6 s_t)
    int r_tot;                 // <= 64
    uint8_t* qX;               // [M][N_pad / 2]
    uint8_t* sX;               // replicated layout over N_pad (sfx_rep_offset)
    float* part;               // [num_n_blocks][M_128][LR_PART_STRIDE] partial LR, one per column block
  } next;
};
constexpr int LR_PART_STRIDE = 64;   // floats per row of an emit-mode LR partial
// TMA box heights the host encodes for kernel 2's operands (rows of a tile):
// NVFP4 stages 128 rows of qX / LR and 256 rows of qR / L2a per k-tile; INT4
// stages 128 of each.
constexpr int K2_NV_ROWS_A = 128, K2_NV_ROWS_B = 256;
constexpr int K2_I4_ROWS = 128;
cudaError_t launch_gemm_nvfp4(const CUtensorMap& tmA, const CUtensorMap& tmB,
                              const CUtensorMap& tmLR, const CUtensorMap& tmL2, K2Params p,
                              int num_sms, cudaStream_t stream, bool emit_next = false);
// LR of the next layer from the emit mode's partials: bf16 of their sum in
// partial order, zeros for r_tot <= i < r_pad.
cudaError_t launch_next_lr_reduce(const float* part, int parts, int M, int M_128, int r_tot, int r_pad,
                                  __nv_bfloat16* LR, cudaStream_t stream);

struct K2I8Params {
  int M, N, K_pad, r_tot, r_pad, N_pad;
  int num_m_blocks, num_n_blocks;
  int nk;                  // K_pad / 128 k-tiles (two 64-groups each)
  int nl;                  // r_pad / 64 low-rank chunks (0: plain W4A4 GEMM)
  const float* sX;         // binary16 values widened to float32, chunked (int4_scale_offset)
  const float* sR;
  const float* bias;
  int epi;
  __nv_bfloat16* Y;
  DeviceErr err;
};
cudaError_t launch_gemm_int4(const CUtensorMap& tmX8, const CUtensorMap& tmR8, const CUtensorMap& tmLR,
                             const CUtensorMap& tmL2, K2I8Params p, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- per-call activation amax
// One uint32 slot per CTA (the bits of that CTA's amax(|X^|)); at most
// AMAX_MAX_PARTS slots.
constexpr int AMAX_MAX_PARTS = 1024;
static_assert(AMAX_MAX_PARTS <= 1024, "warp_amax_bits reads at most 32 slots a lane");
int act_amax_num_parts(int K, int num_sms);   // slots the pass writes (0: K too large)
cudaError_t launch_act_amax(const __nv_bfloat16* X, int M, int K, const float* inv_lambda, uint32_t* parts,
                            int num_sms, cudaStream_t stream);

// ---------------------------------------------------------------- unfused up projection
struct UpParams {
  int M, N, r_tot, r_pad;
  const __nv_bfloat16* LR;   // [M][r_pad]
  const __nv_bfloat16* L2a;  // [N_pad][r_pad]
  float alpha;
  int epi;
  __nv_bfloat16* Y;          // [M][N], read-modify-write
};
cudaError_t launch_lowrank_up(UpParams p, cudaStream_t stream);

// ---------------------------------------------------------------- preparation / calibration
cudaError_t launch_calibrate(int M, int K, int N, const __nv_bfloat16* X, const __nv_bfloat16* Wt,
                             float alpha, float* lambda_out, float* act_scale_out, unsigned* ws,
                             cudaStream_t stream);

struct PrepParams {
  int fmt, K, N, K_pad, N_pad, rank, lora_rank, r_tot, r_pad;
  const __nv_bfloat16* Wt;     // [N][K]
  const float* lambda;         // [K]
  const __nv_bfloat16* L1f;    // [K][rank]
  const __nv_bfloat16* L2;     // [rank][N]
  const __nv_bfloat16* bias;   // [N] or null
  const __nv_bfloat16* loraA;  // [K][lora_rank] or null
  const __nv_bfloat16* loraB;  // [lora_rank][N] or null
  float* R;                    // scratch [N][K]
  unsigned* amax_bits;         // scratch, 1 word
  uint8_t* qR;                 // [N_pad][K_pad/2]
  uint8_t* sR;                 // scales
  uint8_t* sR_rep;             // NVFP4: kernel 2's replicated copy (sfw_rep_offset)
  uint8_t* qR8;                // INT4: kernel 2's copy of the codes as E4M3 bytes [N_pad][K_pad]
  __nv_bfloat16* L1t;          // [K_pad/64][r_tot][64], 128-byte swizzled
  __nv_bfloat16* L2a;          // [N_pad][r_pad]
  float* bias_f;               // [N_pad]
  float* lambda_inv;           // [K]
  float* lambda_inv_k1;        // [K_pad], permuted per 64-wide stage for kernel 1
};
cudaError_t launch_prepare_residual(const PrepParams& p, cudaStream_t stream);
cudaError_t launch_prepare_quantize(const PrepParams& p, float s_tR, float alpha,
                                    cudaStream_t stream);

cudaError_t launch_selftest_timeout(DeviceErr err, cudaStream_t stream);

// Randomized truncated SVD of W^ = diag(lambda) W (see rsvd.cu); synchronous.
// L1f bf16 [K][r], L2 bf16 [r][N] on the device; sigma_out (host, may be
// null) receives the min(r + 8, K, N) estimated singular values.
cudaError_t lowrank_factors(int K, int N, int r, const __nv_bfloat16* Wt, const float* lam, uint64_t seed,
                            __nv_bfloat16* L1f, __nv_bfloat16* L2, double* sigma_out, cudaStream_t s);

// ---------------------------------------------------------------- AWQ W4A16 layer
// Codes: uint8 [K/32][N_pad][16] (chunk c holds k in [32c, 32c+32) of feature
// n, 4 bits each; 32-bit word w of a chunk holds k = 32c + 8w + i at bit
// 4 awq_nibble_pos(i): the even k in the low half-word, the odd in the high,
// so one shift and mask give the bf16 pair (k, k + 1) and the float32
// pairs (k, k + 2)); scale binary16 and zero uint8 [K/64][N_pad]; N_pad = N
// rounded up to 32.
__host__ __device__ constexpr int awq_nibble_pos(int i) { return (i >> 1) + 4 * (i & 1); }
constexpr int AWQ_WARPS = 8;      // warps of a CTA, splitting K
constexpr int AWQ_MB_MAX = 4;     // activation rows per pass over the weights
constexpr int AWQ_STAGES = 4;     // TMA ring depth (stages of 8 groups x 32 features)
static_assert(AWQ_MB_MAX <= AWQ_WARPS, "one warp per row writes the outputs");
struct AwqPrepParams {
  int K, N, N_pad;
  const __nv_bfloat16* Wt;        // [N][K]
  const float* s;                 // [K] AWQ input-channel scales, or null (all 1)
  const __nv_bfloat16* bias;      // [N] or null
  uint8_t* code;
  __half* scale;
  uint8_t* zero;
  float* inv_s;                   // [K] fl32(1/s)
  float* bias_f;                  // [N_pad]
};
struct AwqParams {
  int M, K, N, N_pad, mb;         // mb: activation rows staged per pass
  const __nv_bfloat16* X;         // [M][K]
  const uint8_t* code;
  const __half* scale;
  const uint8_t* zero;
  const float* inv_s;             // [K] fl32(1/s)
  const float* bias;              // [N_pad]
  __nv_bfloat16* Y;               // [M][N]
  DeviceErr err;
};
// The tensor-core form (awq_gemm.cu): 128 x 256 tiles over 64-wide k-tiles.
struct AwqGemmParams {
  int M, K, N, N_pad;
  int num_m_blocks, num_n_blocks;  // ceil(M / 128), ceil(N / 256)
  const float* inv_s;              // [K] fl32(1/s) (read only when the handle has an AWQ scale)
  const float* bias;               // [N_pad]
  __nv_bfloat16* Y;                // [M][N], N % 16 == 0, 32-byte aligned
  DeviceErr err;
};
// tmX: X bf16 [M][K], box {64, 128}, 128-byte swizzle; tmCode: the codes as a
// 3-D uint8 tensor [K/32][N_pad][16], box {16, 256, 2}; tmScale / tmZero:
// [K/64][N_pad] binary16 / uint8, box {256, 1}.
cudaError_t launch_awq_gemm(const CUtensorMap& tmX, const CUtensorMap& tmCode, const CUtensorMap& tmScale,
                            const CUtensorMap& tmZero, AwqGemmParams p, bool has_s, int num_sms,
                            cudaStream_t stream);
cudaError_t launch_awq_quantize(const AwqPrepParams& p, cudaStream_t stream);
// tmCode: codes as a 3-D uint8 tensor [K/32][N_pad][16], box {16, 32, 16};
// tmScale / tmZero: [K/64][N_pad] binary16 / uint8, box {32, 8}.
cudaError_t launch_awq_gemv(const CUtensorMap& tmCode, const CUtensorMap& tmScale, const CUtensorMap& tmZero,
                           AwqParams p, int num_sms, cudaStream_t stream);
int awq_rows_per_block(int K, int M);
size_t awq_smem_bytes(int K, int mb);

}  // namespace svdq
