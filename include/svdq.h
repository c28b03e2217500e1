/*
 * svdq.h -- C ABI of the SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (SVDQuant overview figure, Stages 2 and 3, "svdq-int4-flux.1-dev"
 * model card; abstract of "SVDQuant: Absorbing Outliers by Low-Rank Components
 * for 4-Bit Diffusion Models"):
 *
 *     Y = X^ L1 L2  +  Q(X^) Q(R)  +  b,      X^ = X diag(lambda)^-1,
 *     W^ = diag(lambda) W ~= L1 L2 + R   (rank-r SVD split, R quantized to 4 bits)
 *
 * computed as two fused kernels ("Nunchaku engine design" figure (b) of the
 * same model card: the down projection shares its input with the quantize
 * kernel, the up projection shares its output with the 4-bit GEMM):
 *
 *     kernel 1  svdq_quantize_act_lowrank_down : X -> (qX, sX, LR = X L1f)
 *     kernel 2  svdq_w4a4_gemm_lowrank_up      : (qX, sX, LR) -> Y
 *
 * Conventions shared by every call
 *   - Shapes: M tokens (rows of X and Y), K input features, N output features.
 *     The math weight is W (K x N); the API takes it in nn.Linear order
 *     W_t[N][K] (row n = output feature n), because the layer replaces an
 *     nn.Linear (Diffusers blog, "Introducing Nunchaku Lite").
 *   - Requirements: K % 64 == 0, N % 16 == 0, M >= 0 (M == 0 is a no-op),
 *     rank + lora_rank a multiple of 16 in [16, 256].
 *   - "dev" pointers are device memory of the current CUDA device; "host"
 *     pointers are host memory.  Every device pointer must be 16-byte aligned;
 *     the output Y of the W4A4 layer calls (svdq_linear, svdq_linear_noalloc,
 *     svdq_linear_dynamic, svdq_linear_unfused, svdq_mlp,
 *     svdq_w4a4_gemm_lowrank_up, svdq_w4a4_gemm) 32-byte aligned, because
 *     their GEMM writes Y in 32-byte row segments.
 *   - The caller owns X, Y, qX, sX, LR and any workspace; their sizes come from
 *     the query calls.  The library owns the buffers behind an svdq_weights
 *     handle and frees them in svdq_free_weights.
 *   - Launches are asynchronous on `stream` (0 = legacy default stream).
 *     Argument, shape and alignment errors are returned before anything is
 *     launched.  A kernel that detects a problem while running (a wait that
 *     exceeded its time limit, a failed bounds check) records it in a device
 *     error word; svdq_poll_device_error() reports it.
 *   - Every call returns SVDQ_ERR_UNSUPPORTED_DEVICE unless the current
 *     device has compute capability 10.0, instead of producing wrong output
 *     (Diffusers blog, "Hardware support": unsupported GPUs are rejected at
 *     load time with a clear error).  There is no CPU fallback.
 *   - No call aborts the process or throws across the ABI.
 *
 * Library-defined layouts (svdq_weights_view reports them):
 *   K_pad = K rounded up to a multiple of 256, r_tot = rank + lora_rank,
 *   r_pad = r_tot rounded up to a multiple of 64.
 *   qX    NVFP4: uint8 [M][K_pad/2]: two 4-bit codes per byte, even k in the
 *         low nibble.  INT4: uint8 [M][K_pad]: every code (-8..7) as its FP8
 *         E4M3 byte (the operand form of kernel 2's tensor-core product).
 *         Columns k >= K hold code 0.
 *   sX    NVFP4: E4M3 block scales (one per 16 k), each stored four times
 *         (once per tensor-memory sub-partition, the form kernel 2 copies
 *         into tensor memory): the scale of row r and 16-group g (0..3) of
 *         the 64-column block kb sits at byte
 *           ((((r / 128) * (K_pad/256) + kb / 4) * 2 + (kb % 4) / 2) * 4096
 *           + (L / 8) * 256 + (kb % 2) * 128 + (L % 8) * 16
 *           + ((r % 128) / 32) * 4 + g
 *         for each replica L = r % 32 + 32 q, q = 0..3.  4 * M_128 * K_pad/16
 *         bytes (M_128 = M rounded up to 128); rows >= M hold 0.
 *         INT4: block scales (one per 64 k) rounded to binary16 and stored
 *         widened to float32 (exactly), in 1 KB chunks of 128 rows x 2
 *         groups: the scale of row r and 64-group g sits at float32 element
 *         (((r / 128) * (K_pad/128) + g / 2) * 2 + g % 2) * 128 + r % 128;
 *         rows >= M and groups >= K/64 hold 0.
 *   LR    bf16 [M][r_pad]: X L1f for the r_tot low-rank columns, zeros after.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, unknown enum, bad scalar */
  SVDQ_ERR_SHAPE = 2,              /* dimension outside the requirements above */
  SVDQ_ERR_ALIGNMENT = 3,          /* a device pointer below its alignment (16 bytes; 32 for a layer's Y) */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute capability 10.0 */
  SVDQ_ERR_WORKSPACE = 5,          /* workspace missing or smaller than required */
  SVDQ_ERR_CUDA = 6,               /* a CUDA runtime or driver call failed */
  SVDQ_ERR_TIMEOUT = 7,            /* a device-side wait exceeded its time limit */
  SVDQ_ERR_DEVICE_FAULT = 8,       /* a device-side bounds or consistency check failed */
  SVDQ_ERR_NO_MEMORY = 9           /* device allocation for a weight handle failed */
} svdq_status;

typedef enum { SVDQ_NVFP4 = 0, SVDQ_INT4 = 1 } svdq_format;

typedef enum { SVDQ_EPI_NONE = 0, SVDQ_EPI_GELU_TANH = 1 } svdq_epilogue;

/* Opaque, library-owned prepared weights of one layer. */
typedef struct svdq_weights svdq_weights;

/* Read-only view of a handle (device pointers stay owned by the handle). */
typedef struct {
  int fmt;                 /* svdq_format */
  int K, N, rank, lora_rank, r_tot;
  int K_pad, N_pad, r_pad; /* N_pad = N rounded up to a multiple of 256 */
  const void* qR;          /* dev uint8 [N_pad][K_pad/2]: two 4-bit codes per byte, even k in the
                              low nibble (rows = output features; INT4 kernel 2 reads an E4M3
                              copy the handle also holds) */
  const void* sR;          /* dev: scales of R, one copy each (NVFP4: 512-byte atoms
                              of 128 rows x 64 k at ((n/128) * (K_pad/64) + k/64) * 512,
                              byte (n % 32) * 16 + ((n % 128) / 32) * 4 + (k % 64) / 16;
                              INT4: laid out like sX), over N_pad rows */
  const void* L1t;         /* dev bf16 (lambda^-1-folded L1 | LoRA A)^T in kernel 1's staged layout:
                              one [r_tot x 64] box per 64-wide k block, in k order; chunk c of row r at c ^ (r % 8) */
  const void* L2a;         /* dev bf16 [N_pad][r_pad]: (L2 ; LoRA B) transposed, divided by alpha */
  const void* bias;        /* dev float32 [N_pad] (zeros if no bias was given) */
  const float* lambda_inv; /* dev float32 [K]: correctly rounded 1/lambda */
  float s_tR;              /* NVFP4 weight tensor scale (1 for INT4) */
  float s_tX;              /* NVFP4 static activation tensor scale (1 for INT4) */
  float alpha;             /* 2^k = s_tX * s_tR up to one float32 rounding (1 for INT4) */
} svdq_weights_info;

/* ------------------------------------------------------------------------
 * Offline calibration (SVDQuant overview figure, Stage 2: outliers migrate
 * from the activation to the weight).
 *
 * lambda_k = max_m|X[m,k]|^alpha / max_n|W[k,n]|^(1-alpha), in float64,
 * rounded once to float32 (1 where either maximum is 0); then
 * act_scale = max|fl32(X[m,k] * fl32(1/lambda_k))| / 2688 (the static NVFP4
 * activation tensor scale; 1 if that maximum is 0).
 *   X          dev bf16 [M][K]    calibration activation
 *   W_t        dev bf16 [N][K]    weight in nn.Linear order
 *   alpha      migration strength in [0, 1]
 *   lambda_out dev float32 [K]    written
 *   act_scale_out dev float32 [1] written
 *   workspace  dev, at least svdq_calibrate_workspace_bytes(K) bytes, 16-aligned
 * Errors: INVALID_ARG (null, alpha outside [0,1]), SHAPE, ALIGNMENT,
 *         WORKSPACE, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------ */
size_t svdq_calibrate_workspace_bytes(int K);
svdq_status svdq_calibrate(int M, int K, int N, const void* X, const void* W_t, float alpha,
                           float* lambda_out, float* act_scale_out, void* workspace,
                           size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The low-rank split on the device (Stage 3 of the overview figure: the
 * truncated SVD of W^ = diag(lambda) W), for callers without factors.
 * Randomized range finder with subspace iteration (Halko, Martinsson, Tropp,
 * "Finding structure with randomness", SIAM Review 2011, Algorithms 4.4 and
 * 5.1), float64 throughout: a Rademacher sketch of l = min(rank + 8, K, N)
 * columns drawn from Philox4x32-10 (Salmon et al., SC 2011; entry (n, j) is
 * the top bit of word n l + j, block at counter (index lo, index hi, 0, 0),
 * key (seed lo, seed hi)), three subspace iterations with CholeskyQR2
 * orthonormalization, then the small SVD through the eigenproblem of the
 * projected Gram matrix.  Returns the factors folded as svdq_prepare_weights
 * takes them, each right singular vector signed so its largest-magnitude
 * entry is positive.  It approximates the exact truncated SVD; for a matrix
 * of rank <= l it is exact to float64 rounding.
 *   W_t     dev bf16 [N][K];  lambda dev float32 [K]
 *   seed    the sketch's Philox key
 *   L1f     dev bf16 [K][rank]  = bf16(diag(lambda)^-1 U_r S_r)
 *   L2      dev bf16 [rank][N]  = bf16(V_r^T)
 *   sigma   host double [min(rank + 8, K, N)] or NULL: the estimated
 *           singular values, descending
 * Synchronous (returns when done); allocates and frees its own device
 * scratch (8 K N bytes for W^ plus a few tall-skinny blocks).
 * Errors: INVALID_ARG, SHAPE (rank < 1 or > min(K, N)), ALIGNMENT,
 *         UNSUPPORTED_DEVICE, NO_MEMORY, CUDA.
 * ------------------------------------------------------------------------ */
#define SVDQ_SPLIT_SEED 0x5EEDull
svdq_status svdq_lowrank_factors(int K, int N, int rank, const void* W_t, const float* lambda,
                                 unsigned long long seed, void* L1f, void* L2, double* sigma,
                                 cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Offline weight preparation (Stage 3 of the overview figure: W^ splits into
 * a 16-bit rank-r branch and a 4-bit residual; abstract: LoRAs join the
 * low-rank branch without re-quantizing the residual).
 *
 * Given the folded low-rank factors L1f = bf16(diag(lambda)^-1 U_r S_r)
 * (K x rank) and L2 = bf16(V_r^T) (rank x N) from a truncated SVD of
 * W^ = diag(lambda) W, computes on the device
 *     R[k,n] = fp32(lambda_k W[k,n] - lambda_k sum_{i<rank} L1f[k,i] L2[i,n])
 * (float64, i ascending, no fused multiply-add), the NVFP4 tensor scale
 * s_tR = fl32(2^k / act_scale) with k the smallest integer such that
 * 2^k >= act_scale max|R| / 2688 (so s_tR >= max|R| / 2688 and the product
 * alpha = act_scale s_tR is the power of two 2^k, which lets L2 / alpha be
 * stored exactly in bf16), the 4-bit codes and block scales of R per output
 * column (groups of 16 along K for NVFP4, 64 for INT4), and the layouts the
 * kernels consume.  A LoRA (A: K x lora_rank, B: lora_rank x N) is appended
 * to the factors: L1' = [L1f | A], L2' = [L2 ; B]; R does not change.
 *   fmt        SVDQ_NVFP4 or SVDQ_INT4
 *   W_t        dev bf16 [N][K]
 *   lambda     dev float32 [K]    smoothing factors (see svdq_calibrate)
 *   L1f        dev bf16 [K][rank] row-major, or NULL together with L2: the
 *              factors then come from svdq_lowrank_factors (seed
 *              SVDQ_SPLIT_SEED) on the device; rank <= min(K, N)
 *   L2         dev bf16 [rank][N] row-major, or NULL (see L1f)
 *   bias       dev bf16 [N] or NULL (no bias)
 *   lora_A     dev bf16 [K][lora_rank] or NULL (then lora_rank must be 0)
 *   lora_B     dev bf16 [lora_rank][N] or NULL
 *   act_scale  NVFP4 static activation tensor scale s_tX (> 0, finite);
 *              ignored for INT4
 *   out        host: receives the new handle (NULL on error)
 * The call synchronizes `stream` before returning.  Errors: INVALID_ARG
 * (including exactly one of L1f, L2 NULL), SHAPE, ALIGNMENT,
 * UNSUPPORTED_DEVICE, NO_MEMORY, CUDA; nothing is leaked.
 * ------------------------------------------------------------------------ */
svdq_status svdq_prepare_weights(svdq_format fmt, int K, int N, int rank, const void* W_t,
                                 const float* lambda, const void* L1f, const void* L2,
                                 const void* bias, const void* lora_A, const void* lora_B,
                                 int lora_rank, float act_scale, cudaStream_t stream,
                                 svdq_weights** out);

/* Frees the handle and its device buffers (synchronizes the device first).
 * NULL is accepted and ignored. */
svdq_status svdq_free_weights(svdq_weights* w);

/* Fills *info with the handle's layout and device pointers. */
svdq_status svdq_weights_view(const svdq_weights* w, svdq_weights_info* info);

/* Sizes in bytes of the caller-owned intermediates for M rows (any pointer
 * may be NULL to skip it). */
svdq_status svdq_act_buffer_sizes(const svdq_weights* w, int M, size_t* qx_bytes,
                                  size_t* sx_bytes, size_t* lr_bytes);

/* ------------------------------------------------------------------------
 * Kernel 1 -- quantize + low-rank down projection, fused ("Nunchaku engine
 * design" figure (b): both read the same input, so X is read from HBM once).
 *   x^ = fl32(x * lambda_inv_k); per row and 16- (NVFP4) or 64- (INT4)
 *   group: amax -> block scale -> 4-bit codes, exactly as svdq_prepare_weights
 *   quantizes R, with the handle's s_tX as the NVFP4 tensor scale;
 *   LR = bf16(X L1') with float32 accumulation.
 *   X   dev bf16 [M][K]
 *   qX, sX, LR  dev, sizes from svdq_act_buffer_sizes, layouts above
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------ */
svdq_status svdq_quantize_act_lowrank_down(const svdq_weights* w, int M, const void* X,
                                           void* qX, void* sX, void* LR, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Kernel 2 -- 4-bit GEMM + low-rank up projection, fused (figure (b): both
 * write the same output, so the 16-bit branch adds no HBM round trip).
 *   y[m,n] = alpha * ( sum_k dq(qX)[m,k] dq(qR)[n,k] + sum_i LR[m,i] L2a[n,i] ) + b[n]
 *   (NVFP4: block-scaled tensor-core MMA with E4M3 scales per 16; INT4:
 *   an exact tensor-core product per 64-group on the codes held as E4M3,
 *   rescaled by sX[m,g] sR[n,g]); optional GELU (tanh form, evaluated as
 *   y / (1 + e^(-2u)) with the hardware exp2 and reciprocal approximations,
 *   relative error near 1e-6); Y = bf16(y).
 *   qX, sX, LR  dev, as written by kernel 1 (or by an equivalent producer)
 *   Y   dev bf16 [M][N] row-major
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------ */
svdq_status svdq_w4a4_gemm_lowrank_up(const svdq_weights* w, int M, const void* qX,
                                      const void* sX, const void* LR, svdq_epilogue epi,
                                      void* Y, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The whole layer: kernel 1 then kernel 2 on `stream`, with qX, sX and LR
 * placed in the caller's workspace.
 *   X  dev bf16 [M][K];  Y  dev bf16 [M][N]
 *   workspace  dev, at least svdq_linear_workspace_bytes(w, M) bytes
 * Errors: as kernels 1 and 2, plus WORKSPACE.
 * ------------------------------------------------------------------------ */
size_t svdq_linear_workspace_bytes(const svdq_weights* w, int M);
svdq_status svdq_linear(const svdq_weights* w, int M, const void* X, svdq_epilogue epi, void* Y,
                        void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The whole layer with a per-call NVFP4 activation tensor scale.
 * The "SVDQuant" paper's NVFP4 setting gives the activation an FP32 tensor
 * scale on top of the E4M3 scales per 16 elements, but does not say how it
 * is chosen.  svdq_linear uses the one fixed at preparation (act_scale);
 * this entry point takes it from the call's own X^ = X diag(lambda)^-1:
 *   a    = amax |X^| over all M x K elements (X^ rounded to float32 as in
 *          kernel 1; a = 0 counts as 2688),
 *   j    = the smallest integer with 2^j >= s_tR a / 2688 (float64),
 *   s_tX = fl32(2^j / s_tR),
 * so s_tX s_tR is the power of two 2^j, as alpha is at preparation, and no
 * activation block scale exceeds 448 however X is distributed.  Kernel 2
 * multiplies by 2^j; kernel 1 stores LR times 2^(k - j), where 2^k is the
 * prepared alpha (svdq_weights_view), so LR L2a keeps its weight.
 * Launches: one streaming pass over X (amax per CTA into the workspace, no
 * atomics), then kernels 1 and 2, which read the partial maxima after their
 * grid-dependency wait (no host round trip; stream capture works).
 * INT4 has no tensor scale: for INT4 weights this is svdq_linear.
 *   X  dev bf16 [M][K];  Y  dev bf16 [M][N]
 *   workspace  dev, at least svdq_linear_dynamic_workspace_bytes(w, M):
 *     bytes [0, svdq_linear_workspace_bytes(w, M)) hold qX, sX and LR as
 *     svdq_linear places them (each at a 256-byte aligned offset, in that
 *     order, sizes svdq_act_buffer_sizes); then 16 bytes written by the call
 *     (NVFP4 only): float s_tX, int32 j, float 2^j, unused; then the amax
 *     slots.  Every byte read is written first by the same call.
 * Errors: as svdq_linear.
 * ------------------------------------------------------------------------ */
size_t svdq_linear_dynamic_workspace_bytes(const svdq_weights* w, int M);
svdq_status svdq_linear_dynamic(const svdq_weights* w, int M, const void* X, svdq_epilogue epi, void* Y,
                                void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * One layer straight into the next (the cross-layer fusion of the Diffusers
 * blog's "fused GELU/MLP" in "Introducing Nunchaku Lite": the first layer's
 * epilogue produces the second layer's kernel-1 outputs, so its output
 * never goes to memory in 16 bits and the second layer's kernel 1, which
 * would read it back, does not run).
 *
 * svdq_linear_emit_next: layer w1 on X (kernel 1, then kernel 2 with the
 *   epilogue `epi`) computes its bf16 output Y1 = bf16(epi(y)) tile by tile
 *   and writes, instead of Y1, what svdq_quantize_act_lowrank_down(w2, M,
 *   Y1, ...) would write: qX2 and sX2 (the NVFP4 codes and replicated scales
 *   of Y1 diag(lambda2)^-1 with w2's static activation tensor scale),
 *   identical to kernel 1's given the same Y1; and LR2 = bf16(Y1 L1f2) from
 *   float32 partials, one per 256-column tile of Y1 (computed on the tensor
 *   core from the tile's bf16 values held in tensor memory), added in a
 *   fixed order (the same on every run; float32 summation order differs from
 *   kernel 1's, within the LR bound).
 *   Requires both handles NVFP4, w2's K == w1's N and r_tot of w2 <= 64.
 *   qX2, sX2, LR2  dev, sizes from svdq_act_buffer_sizes(w2, M); qX2 32-byte
 *                  aligned (each row's codes of a 64-column block go out as
 *                  one 32-byte store)
 *   workspace      dev, svdq_linear_emit_next_workspace_bytes(w1, w2, M)
 * svdq_mlp: the pair: Y = layer w2 (epilogue epi2) of layer w1 (epi1) of X,
 *   through svdq_linear_emit_next and kernel 2 of w2; Y dev bf16 [M][N2];
 *   workspace svdq_mlp_workspace_bytes(w1, w2, M).
 * Errors: as svdq_linear; SHAPE when the pair does not chain as above;
 *         INVALID_ARG for an INT4 handle or handles on different devices.
 * ------------------------------------------------------------------------ */
size_t svdq_linear_emit_next_workspace_bytes(const svdq_weights* w1, const svdq_weights* w2, int M);
svdq_status svdq_linear_emit_next(const svdq_weights* w1, const svdq_weights* w2, int M, const void* X,
                                  svdq_epilogue epi, void* qX2, void* sX2, void* LR2, void* workspace,
                                  size_t ws_bytes, cudaStream_t stream);
size_t svdq_mlp_workspace_bytes(const svdq_weights* w1, const svdq_weights* w2, int M);
svdq_status svdq_mlp(const svdq_weights* w1, const svdq_weights* w2, int M, const void* X, svdq_epilogue epi1,
                     svdq_epilogue epi2, void* Y, void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The whole layer from host memory to host memory, with the copies
 * overlapped with the kernels (no counterpart in the paper: an integration
 * convenience for callers whose activations live on the host).  M is cut
 * into slabs of about M / 8 rows (a multiple of 128, at least 128); while the
 * layer runs on slab i on `stream`, the library's own copy-in stream moves
 * slab i + 1's X to the device and its copy-out stream moves slab i - 1's Y
 * to the host (the two directions use separate copy engines).  Each slab is
 * one cudaMemcpyAsync per direction.  Row m of Y depends on row m of X only,
 * so the result is bit-identical to svdq_linear on the whole batch.
 *   X_host  host bf16 [M][K], Y_host host bf16 [M][N]; page-locked memory
 *           (cudaHostAlloc / cudaHostRegister) is needed for the copies to
 *           run asynchronously and overlap
 *   workspace  dev, 256-byte aligned, at least
 *           svdq_linear_host_workspace_bytes(w, M) bytes (two X slabs, two
 *           Y slabs and one slab's svdq_linear workspace)
 * Ordering: the call's work starts after the work already on `stream`; work
 * issued on `stream` afterwards starts after the last Y slab is on the host.
 * The two copy streams and their events are created at a device's first call
 * (no device memory is allocated) and are shared by every call on that device:
 * calls from several host threads are serialised by a lock while they are
 * issued.
 * Errors: as svdq_linear.
 * ------------------------------------------------------------------------ */
size_t svdq_linear_host_workspace_bytes(const svdq_weights* w, int M);
svdq_status svdq_linear_host(const svdq_weights* w, int M, const void* X_host, svdq_epilogue epi, void* Y_host,
                             void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * svdq_linear without a workspace argument (no counterpart in the paper: it
 * is an integration convenience, not part of the method).
 *
 * Some callers cannot allocate device memory at the point where they run
 * the layer: cudaMalloc may synchronize the whole device and take
 * milliseconds, which a latency-critical serving loop cannot afford, and a
 * plug-in hosted by an application that owns all device memory through its
 * own allocator is often given no allocator at all.  This entry point keeps
 * the intermediates qX, sX and LR in a scratch array that is part of the
 * library image (SVDQ_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that
 * loads the library until the process exits).  It calls no cudaMalloc,
 * cudaFree or allocating library routine; the caller still passes X and Y.
 *   - Sizes: svdq_linear_workspace_bytes(w, M) must not exceed
 *     SVDQ_NOALLOC_SCRATCH_BYTES (32 MiB).  Per row that is about
 *     3 K_pad / 4 + 2 r_pad bytes for NVFP4 (codes K_pad / 2, scales in four
 *     replicas K_pad / 4, LR 2 r_pad; r_pad = rank + LoRA rank rounded up to
 *     64) and K_pad + K_pad / 16 + 2 r_pad bytes for INT4, with the scales
 *     over M rounded up to 128 rows.  Largest M at r_pad = 64: NVFP4 13,784
 *     rows at K = 3072 and 3,584 at K = 12288; INT4 9,886 at K = 3072 and
 *     2,544 at K = 12288.  A larger request returns SVDQ_ERR_WORKSPACE
 *     before anything is launched (after the argument and device checks,
 *     in the order of svdq_linear).
 *   - The first call on each device looks up the scratch array's device
 *     address for that device (a runtime query, no allocation) and keeps it
 *     for the life of the process, so that first call should come before
 *     any stream capture.  A device reset (cudaDeviceReset, or anything that
 *     destroys the primary context) invalidates this and every other piece
 *     of per-device state the library keeps: do not call the library on a
 *     device after resetting it.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents; nothing in it needs clearing, because kernel 1
 *     rewrites every byte kernel 2 reads.  Calls whose kernels overlap on
 *     the GPU (different streams, no ordering between them) race on the
 *     array: order them, e.g. issue them on one stream.
 * Errors: as svdq_linear, plus WORKSPACE when M is too large.
 * ------------------------------------------------------------------------ */
#define SVDQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
svdq_status svdq_linear_noalloc(const svdq_weights* w, int M, const void* X, svdq_epilogue epi, void* Y,
                                cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Unfused baseline ("Nunchaku engine design" figure (a): run naively, the
 * rank-32 branch costs an extra 16-bit read of X in the down projection and
 * an extra 16-bit write of Y in the up projection, 57% latency overhead).
 * These exist to measure that overhead against the fused path; they compute
 * the same codes, scales and LR as kernel 1.
 *   svdq_quantize_act     X -> qX, sX           (no low-rank work)
 *   svdq_lowrank_down     X -> LR               (reads X again)
 *   svdq_w4a4_gemm        qX, sX -> Y = bf16(alpha acc + b)   (no low-rank, no GELU)
 *   svdq_lowrank_up       Y <- bf16(epi(Y + alpha LR L2a))    (read-modify-write of Y)
 *   svdq_linear_unfused   the four above in order; same workspace as svdq_linear
 * ------------------------------------------------------------------------ */
svdq_status svdq_quantize_act(const svdq_weights* w, int M, const void* X, void* qX, void* sX,
                              cudaStream_t stream);
svdq_status svdq_lowrank_down(const svdq_weights* w, int M, const void* X, void* LR,
                              cudaStream_t stream);
svdq_status svdq_w4a4_gemm(const svdq_weights* w, int M, const void* qX, const void* sX,
                           void* Y, cudaStream_t stream);
svdq_status svdq_lowrank_up(const svdq_weights* w, int M, const void* LR, svdq_epilogue epi,
                            void* Y, cudaStream_t stream);
svdq_status svdq_linear_unfused(const svdq_weights* w, int M, const void* X, svdq_epilogue epi,
                                void* Y, void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * AWQ W4A16 linear layer: 4-bit weights, 16-bit activations.
 * The second kernel family of the Diffusers blog "Integrating Nunchaku 4-bit
 * diffusion inference into Diffusers" ("Introducing Nunchaku Lite":
 * awq_w4a16, for the adaptive-normalization and modulation projections,
 * which are memory-bound and sensitive to precision; "Native loading in
 * Diffusers": precision int4, group_size 64).
 *
 *   prepare:  W' = fl32(w * s_k) with AWQ's per-input-channel scale s (all
 *             ones if NULL); per group g of 64 input features and output
 *             feature n: lo, hi = min, max of W'; d = binary16 of
 *             fl32(max(hi - lo, 1e-5) / 15), round to nearest even,
 *             saturating at 65504; zero = clamp(rint(-lo / d), 0, 15);
 *             code = clamp(rint(w' / d) + zero, 0, 15) (IEEE float32
 *             divisions, rint = round half to even).
 *   layer:    y[m,n] = sum_g d[g,n] sum_{k in g} (code[k,n] - zero[g,n]) x'[m,k]
 *             + b[n], x' = fl32(x * fl32(1/s_k)); float32 accumulation;
 *             Y = bf16(y).
 * The layer reads every weight byte once per call and is sized for small M
 * (the rows of a modulation projection: a few per image); it stages up to
 * 4 activation rows at a time (fewer when K > 3072) and streams the weights
 * once per group of rows.
 *
 * svdq_awq_prepare: W_t dev bf16 [N][K] (nn.Linear order); s dev float32 [K]
 *   or NULL; bias dev bf16 [N] or NULL.  K % 64 == 0, N >= 1.  Synchronous
 *   on `stream` (returns when the handle is ready).  The handle owns its
 *   buffers until svdq_awq_free.
 *   Errors: INVALID_ARG, SHAPE, ALIGNMENT, UNSUPPORTED_DEVICE, NO_MEMORY, CUDA.
 * svdq_awq_linear: X dev bf16 [M][K], Y dev bf16 [M][N], M >= 0 (0: no-op).
 *   Errors: INVALID_ARG (null, or the handle belongs to another device),
 *   SHAPE, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * svdq_awq_view layouts (N_pad = N rounded up to 32; pad features hold
 *   code 0, zero 0, scale 0):
 *   code   uint8 [K/32][N_pad][16]: 16 bytes per (32-feature chunk c, n), the
 *          codes of k = 32c .. 32c + 31, 4 bits each; the 32-bit word w
 *          (little-endian) holds k = 32c + 8w + i at bits 4p .. 4p + 3 with
 *          p = i / 2 + 4 (i % 2) (even k in the low half-word, odd k in the
 *          high half-word, each in increasing order)
 *   scale  binary16 [K/64][N_pad];  zero  uint8 [K/64][N_pad]
 *   inv_s  float32 [K] = fl32(1/s);  bias  float32 [N_pad]
 * ------------------------------------------------------------------------ */
typedef struct svdq_awq_weights svdq_awq_weights;
typedef struct {
  int K, N, N_pad;
  const void* code;
  const void* scale;
  const void* zero;
  const float* inv_s;
  const float* bias;
} svdq_awq_info;
svdq_status svdq_awq_prepare(int K, int N, const void* W_t, const float* s, const void* bias,
                             cudaStream_t stream, svdq_awq_weights** out);
svdq_status svdq_awq_free(svdq_awq_weights* w);
svdq_status svdq_awq_view(const svdq_awq_weights* w, svdq_awq_info* info);
svdq_status svdq_awq_linear(const svdq_awq_weights* w, int M, const void* X, void* Y, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * The same W4A16 layer on the tensor core, for batches where it is a dense
 * contraction (the W4A16 side of the "SVDQuant" abstract's speed comparison,
 * 3.0x / 3.1x for W4A4 over W4A16 on the pages' GPUs).  The product runs on
 * 16-bit operands as W4A16 GEMMs do: each dequantized weight is rounded once
 * to bf16, w^16 = bf16((code - zero) d), and the activation is
 * X'16 = bf16(fl32(x fl32(1/s))) (X itself when the handle has no AWQ
 * scale); Y = bf16(X'16 W^16 + b) with float32 accumulation.  Because of the
 * weight rounding this differs from svdq_awq_linear (float32 weights) by up
 * to sum_k |x'_k| |w^16 - w^| per output; use svdq_awq_linear for the
 * precision-sensitive few-row modulation projections and this call for
 * batches of hundreds of rows and more.
 *   X dev bf16 [M][K] (16-byte aligned), Y dev bf16 [M][N] (32-byte aligned),
 *   N % 16 == 0, M >= 0 (0: no-op).  Asynchronous on `stream`.
 *   Errors: INVALID_ARG (null, or the handle belongs to another device),
 *   SHAPE, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA.
 * ------------------------------------------------------------------------ */
svdq_status svdq_awq_gemm(const svdq_awq_weights* w, int M, const void* X, void* Y, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Diagnostics.
 * svdq_poll_device_error: synchronizes `stream`, then reads and clears the
 *   current device's error word.  Returns SVDQ_OK, SVDQ_ERR_TIMEOUT (a wait
 *   ran out; the kernel that hit it skipped the rest of its work and
 *   returned), SVDQ_ERR_DEVICE_FAULT, or SVDQ_ERR_CUDA (the stream itself
 *   reported an error).
 * svdq_selftest_wait_timeout: launches one CTA that waits on a barrier
 *   nothing will complete, with a wait limit of `limit_us` microseconds;
 *   the bounded wait must give up, set the error word and return, leaving
 *   the context usable.  Used to test the timeout path without a fault.
 * svdq_status_string: static English text for a status (never NULL).
 * ------------------------------------------------------------------------ */
svdq_status svdq_poll_device_error(cudaStream_t stream);
svdq_status svdq_selftest_wait_timeout(unsigned limit_us, cudaStream_t stream);
const char* svdq_status_string(svdq_status s);

/* Test hook: pretend the device has compute capability major.minor for the
 * capability check (major < 0 restores the real value). */
void svdq_debug_override_cc(int major, int minor);

#ifdef __cplusplus
}
#endif
#endif /* SVDQ_H_ */
