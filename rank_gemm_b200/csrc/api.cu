// api.cu -- host side of the C ABI declared in include/svdq.h.
//
// Validates every argument before touching the device, keeps per-device
// state (capability check, SM count, device error word), encodes the TMA
// tensor maps, owns the prepared-weight handles and launches the kernels.
// No entry point aborts or throws; every failure is a status code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "svdq.h"
#include "common.cuh"
#include "kernels.h"

using namespace svdq;

namespace svdq {

// (kernel, device) -> the dynamic shared-memory limit already set
cudaError_t ensure_dynamic_smem(const void* kernel, size_t bytes) {
  struct Entry {
    const void* fn;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static Entry table[256];
  static int used = 0;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  int i = 0;
  for (; i < used; ++i)
    if (table[i].fn == kernel && table[i].dev == dev) break;
  if (i < used && table[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (i == used) {
    if (used == 256) return cudaSuccess;   // table full: correct, only slower (set on every call)
    table[used++] = Entry{kernel, dev, bytes};
  } else {
    table[i].bytes = bytes;
  }
  return cudaSuccess;
}

}  // namespace svdq

// Device error word: kernels OR ERR_* bits into it (one copy per device).
__device__ unsigned g_svdq_error_word;

struct svdq_weights {
  int dev;
  svdq_format fmt;
  int K, N, rank, lora_rank, r_tot, K_pad, N_pad, r_pad;
  uint8_t* qR;
  uint8_t* sR;
  uint8_t* sR_rep;   // NVFP4: kernel 2's replicated copy of sR
  uint8_t* qR8;      // INT4: kernel 2's copy of qR, one E4M3 byte per code [N_pad][K_pad]
  __nv_bfloat16* L1t;
  __nv_bfloat16* L2a;
  float* bias_f;
  float* lambda_inv;
  float* lambda_inv_k1;
  float s_tR, s_tX, alpha;
  CUtensorMap tm_qR, tm_L2a;
  CUtensorMap tm_qR8, tm_L2a_i4;      // INT4 kernel: E4M3 codes and L2a in 128-row boxes
};

namespace {

constexpr int MAX_DEVICES = 64;

struct DevState {
  bool ready;
  int cc_major, cc_minor, num_sms;
  unsigned* err_word;
};

std::mutex g_mu;
DevState g_dev[MAX_DEVICES];
int g_cc_override_major = -1, g_cc_override_minor = 0;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

unsigned long long wait_limit_ns() {
  static unsigned long long v = [] {
    const char* s = std::getenv("SVDQ_WAIT_LIMIT_MS");
    const long ms = s ? std::atol(s) : 2000;
    return (unsigned long long)(ms > 0 ? ms : 2000) * 1000000ull;
  }();
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// kernel 2 writes Y in 32-byte row segments (one st.global.v8 each)
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

svdq_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SVDQ_OK;
  cudaGetLastError();   // clear a non-sticky error so the next call starts clean
  return SVDQ_ERR_CUDA;
}

// Current device's state; SVDQ_ERR_UNSUPPORTED_DEVICE unless compute capability 10.0.
svdq_status current_device(DevState** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return SVDQ_ERR_UNSUPPORTED_DEVICE;
    }
    const bool sm100 = d.cc_major == 10 && d.cc_minor == 0;
    if (sm100) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_svdq_error_word) != cudaSuccess) return from_cuda(cudaErrorUnknown);
      if (cudaMemset(p, 0, sizeof(unsigned)) != cudaSuccess) return from_cuda(cudaErrorUnknown);
      d.err_word = static_cast<unsigned*>(p);
      if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
          return from_cuda(cudaErrorUnknown);
        g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
    }
    d.ready = true;
  }
  const int maj = g_cc_override_major >= 0 ? g_cc_override_major : d.cc_major;
  const int min = g_cc_override_major >= 0 ? g_cc_override_minor : d.cc_minor;
  if (!(maj == 10 && min == 0) || !d.err_word) return SVDQ_ERR_UNSUPPORTED_DEVICE;
  *out = &d;
  return SVDQ_OK;
}

DeviceErr dev_err(const DevState* d) { return DeviceErr{d->err_word, wait_limit_ns()}; }

// 2-D tensor map, row-major [rows][inner]; boxes land in shared memory with
// the given swizzle (128-byte by default).
bool tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t rows,
             uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
             CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D uint8 tensor [d2][d1][d0] with byte strides s1 (between d1 rows) and
// s2 (between d2 planes), no swizzle.
bool tmap_3d_u8(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
                uint32_t b0, uint32_t b1, uint32_t b2) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// NVFP4: packed codes; INT4: one E4M3 byte per code
size_t qx_bytes(const svdq_weights* w, int M) {
  return (size_t)M * (w->fmt == SVDQ_NVFP4 ? w->K_pad / 2 : w->K_pad);
}
size_t sx_bytes(const svdq_weights* w, int M) {
  const size_t rows = (size_t)round_up(M, 128);
  // NVFP4: four replicas of every scale word (see sfx_rep_offset)
  return w->fmt == SVDQ_NVFP4 ? rows * (w->K_pad / 16) * 4 : rows * (w->K_pad / 64) * 4;
}
size_t lr_bytes(const svdq_weights* w, int M) { return (size_t)M * w->r_pad * 2; }

svdq_status check_handle_device(const svdq_weights* w, DevState** d) {
  svdq_status s = current_device(d);
  if (s != SVDQ_OK) return s;
  int dev = -1;
  cudaGetDevice(&dev);
  return dev == w->dev ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
}

}  // namespace

// For entry points compiled in other files: the current device's check
// (compute capability 10.0, or the debug override) and that the handle lives
// on it.
svdq_status svdq::handle_device_status(const svdq_weights* w) {
  DevState* d = nullptr;
  return check_handle_device(w, &d);
}

namespace {

// Per-call NVFP4 activation tensor scale: where the amax slots are and where
// kernel 1 reports the scale it chose.
struct DynScale {
  const uint32_t* parts;
  int n_parts;
  float* record;
};

K1Params k1_params(const svdq_weights* w, const DevState* d, int M, void* qX, void* sX, void* LR,
                   int do_quant, int do_lr, const DynScale* dyn) {
  K1Params p;
  p.M = M;
  p.K = w->K;
  p.K_pad = w->K_pad;
  p.r_tot = w->r_tot;
  p.r_pad = w->r_pad;
  p.fmt = (int)w->fmt;
  p.do_quant = do_quant;
  p.do_lr = do_lr;
  p.stages = 0;
  p.ksplit = 2;
  p.inv_lambda = w->lambda_inv_k1;
  p.L1t = w->L1t;
  p.s_t = w->s_tX;
  p.six_st = 6.0f * w->s_tX;   // one IEEE float32 multiply on the host
  p.amax_parts = dyn ? dyn->parts : nullptr;
  p.n_parts = dyn ? dyn->n_parts : 0;
  p.k_alpha = std::ilogb(w->alpha);   // the prepared alpha is a power of two
  p.s_tR = w->s_tR;
  p.dyn_record = dyn ? dyn->record : nullptr;
  p.qX = static_cast<uint8_t*>(qX);
  p.sX = static_cast<uint8_t*>(sX);
  p.LR = static_cast<__nv_bfloat16*>(LR);
  p.err = dev_err(d);
  return p;
}

svdq_status run_k1(const svdq_weights* w, int M, const void* X, void* qX, void* sX, void* LR,
                   int do_quant, int do_lr, cudaStream_t stream, const DynScale* dyn = nullptr) {
  DevState* d = nullptr;
  svdq_status s = check_handle_device(w, &d);
  if (s != SVDQ_OK) return s;
  CUtensorMap tmX;
  if (!tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, w->K, M, (uint64_t)w->K * 2, 64, K1_BOX_ROWS))
    return SVDQ_ERR_CUDA;
  return from_cuda(launch_quant_down(tmX, k1_params(w, d, M, qX, sX, LR, do_quant, do_lr, dyn), d->num_sms, stream));
}

svdq_status run_k2(const svdq_weights* w, int M, const void* qX, const void* sX, const void* LR,
                   svdq_epilogue epi, void* Y, bool lowrank, cudaStream_t stream,
                   const DynScale* dyn = nullptr, const K2Params::Next* next = nullptr) {
  DevState* d = nullptr;
  svdq_status s = check_handle_device(w, &d);
  if (s != SVDQ_OK) return s;
  CUtensorMap tmLR;
  std::memset(&tmLR, 0, sizeof(tmLR));
  const bool nv = w->fmt == SVDQ_NVFP4;
  if (lowrank && !tmap_2d(&tmLR, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, LR, w->r_pad, M, (uint64_t)w->r_pad * 2,
                          64, nv ? K2_NV_ROWS_A : K2_I4_ROWS))
    return SVDQ_ERR_CUDA;
  if (nv) {
    CUtensorMap tmA;
    if (!tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, qX, w->K_pad / 2, M, w->K_pad / 2, 128, K2_NV_ROWS_A))
      return SVDQ_ERR_CUDA;
    K2Params p;
    p.M = M;
    p.N = w->N;
    p.K_pad = w->K_pad;
    p.r_tot = w->r_tot;
    p.r_pad = w->r_pad;
    p.N_pad = w->N_pad;
    p.num_m_blocks = (M + 127) / 128;
    p.num_n_blocks = w->N_pad / 256;
    p.nk = w->K_pad / 256;
    p.nl = lowrank ? w->r_pad / 64 : 0;
    p.sX = static_cast<const uint8_t*>(sX);
    p.sR = w->sR_rep;
    p.bias = w->bias_f;
    p.alpha = w->alpha;
    p.amax_parts = dyn ? dyn->parts : nullptr;
    p.n_parts = dyn ? dyn->n_parts : 0;
    p.s_tR = w->s_tR;
    p.epi = (int)epi;
    p.Y = static_cast<__nv_bfloat16*>(Y);
    p.err = dev_err(d);
    std::memset(&p.next, 0, sizeof(p.next));
    if (next) p.next = *next;
    return from_cuda(launch_gemm_nvfp4(tmA, w->tm_qR, tmLR, w->tm_L2a, p, d->num_sms, stream, next != nullptr));
  }
  CUtensorMap tmX8;
  if (!tmap_2d(&tmX8, CU_TENSOR_MAP_DATA_TYPE_UINT8, qX, w->K_pad, M, w->K_pad, 128, K2_I4_ROWS))
    return SVDQ_ERR_CUDA;
  K2I8Params p;
  p.M = M;
  p.N = w->N;
  p.K_pad = w->K_pad;
  p.r_tot = w->r_tot;
  p.r_pad = w->r_pad;
  p.N_pad = w->N_pad;
  p.num_m_blocks = (M + 127) / 128;
  p.num_n_blocks = w->N_pad / 128;   // the INT4 kernel's tiles are 128 wide
  p.nk = w->K_pad / 128;
  p.nl = lowrank ? w->r_pad / 64 : 0;
  p.sX = static_cast<const float*>(sX);
  p.sR = reinterpret_cast<const float*>(w->sR);
  p.bias = w->bias_f;
  p.epi = (int)epi;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.err = dev_err(d);
  return from_cuda(launch_gemm_int4(tmX8, w->tm_qR8, tmLR, w->tm_L2a_i4, p, d->num_sms, stream));
}

}  // namespace

struct svdq_awq_weights {
  int dev;
  int K, N, N_pad;
  uint8_t* code;
  __half* scale;
  uint8_t* zero;
  float* inv_s;
  float* bias_f;
  CUtensorMap tm_code, tm_scale, tm_zero;   // the GEMV's TMA views of the three
  CUtensorMap tm_code_g, tm_scale_g, tm_zero_g;   // the tensor-core GEMM's (256-feature boxes)
  bool has_s;                                // an AWQ scale was given (the GEMM rescales X)
};

namespace {

void free_awq(svdq_awq_weights* w) {
  cudaFree(w->code);
  cudaFree(w->scale);
  cudaFree(w->zero);
  cudaFree(w->inv_s);
  cudaFree(w->bias_f);
}

void free_buffers(svdq_weights* w) {
  cudaFree(w->qR);
  cudaFree(w->sR);
  cudaFree(w->sR_rep);
  cudaFree(w->qR8);
  cudaFree(w->L1t);
  cudaFree(w->L2a);
  cudaFree(w->bias_f);
  cudaFree(w->lambda_inv);
  cudaFree(w->lambda_inv_k1);
}

}  // namespace

extern "C" {

const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_SHAPE: return "unsupported shape";
    case SVDQ_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case SVDQ_ERR_UNSUPPORTED_DEVICE: return "unsupported device: compute capability 10.0 (B200) required";
    case SVDQ_ERR_WORKSPACE: return "workspace missing or too small";
    case SVDQ_ERR_CUDA: return "CUDA call failed";
    case SVDQ_ERR_TIMEOUT: return "device-side wait exceeded its time limit";
    case SVDQ_ERR_DEVICE_FAULT: return "device-side check failed";
    case SVDQ_ERR_NO_MEMORY: return "device allocation failed";
  }
  return "unknown status";
}

void svdq_debug_override_cc(int major, int minor) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_cc_override_major = major;
  g_cc_override_minor = minor;
}

size_t svdq_calibrate_workspace_bytes(int K) { return K > 0 ? align256((2 * (size_t)K + 1) * 4) : 0; }

svdq_status svdq_calibrate(int M, int K, int N, const void* X, const void* W_t, float alpha,
                           float* lambda_out, float* act_scale_out, void* workspace, size_t ws_bytes,
                           cudaStream_t stream) {
  if (!W_t || !lambda_out || !act_scale_out || (M > 0 && !X)) return SVDQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.f && alpha <= 1.f)) return SVDQ_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || K % 64 || N <= 0 || N % 16) return SVDQ_ERR_SHAPE;
  if ((X && !aligned16(X)) || !aligned16(W_t) || !aligned16(lambda_out) || !aligned16(workspace))
    return SVDQ_ERR_ALIGNMENT;
  if (!workspace || ws_bytes < svdq_calibrate_workspace_bytes(K)) return SVDQ_ERR_WORKSPACE;
  DevState* d = nullptr;
  svdq_status s = current_device(&d);
  if (s != SVDQ_OK) return s;
  return from_cuda(launch_calibrate(M, K, N, static_cast<const __nv_bfloat16*>(X),
                                    static_cast<const __nv_bfloat16*>(W_t), alpha, lambda_out, act_scale_out,
                                    static_cast<unsigned*>(workspace), stream));
}

svdq_status svdq_prepare_weights(svdq_format fmt, int K, int N, int rank, const void* W_t, const float* lambda,
                                 const void* L1f, const void* L2, const void* bias, const void* lora_A,
                                 const void* lora_B, int lora_rank, float act_scale, cudaStream_t stream,
                                 svdq_weights** out) {
  if (out) *out = nullptr;
  if (!out || !W_t || !lambda || (!L1f) != (!L2)) return SVDQ_ERR_INVALID_ARG;
  if (fmt != SVDQ_NVFP4 && fmt != SVDQ_INT4) return SVDQ_ERR_INVALID_ARG;
  if (lora_rank < 0 || (lora_rank > 0) != (lora_A != nullptr) || (lora_rank > 0) != (lora_B != nullptr))
    return SVDQ_ERR_INVALID_ARG;
  if (fmt == SVDQ_NVFP4 && !(std::isfinite(act_scale) && act_scale > 0.f)) return SVDQ_ERR_INVALID_ARG;
  const int r_tot = rank + lora_rank;
  if (K <= 0 || K % 64 || N <= 0 || N % 16 || rank < 1 || r_tot % 16 || r_tot > 256) return SVDQ_ERR_SHAPE;
  if (!aligned16(W_t) || !aligned16(lambda) || !aligned16(L1f) || !aligned16(L2) || !aligned16(bias) ||
      !aligned16(lora_A) || !aligned16(lora_B))
    return SVDQ_ERR_ALIGNMENT;
  DevState* d = nullptr;
  svdq_status s = current_device(&d);
  if (s != SVDQ_OK) return s;
  if (!L1f) {
    // no factors given: the library's randomized split of diag(lambda) W
    if (rank > std::min(K, N)) return SVDQ_ERR_SHAPE;
    void *f1 = nullptr, *f2 = nullptr;
    if (cudaMalloc(&f1, (size_t)K * rank * 2) != cudaSuccess || cudaMalloc(&f2, (size_t)rank * N * 2) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(f1);
      cudaFree(f2);
      return SVDQ_ERR_NO_MEMORY;
    }
    s = from_cuda(lowrank_factors(K, N, rank, static_cast<const __nv_bfloat16*>(W_t), lambda, SVDQ_SPLIT_SEED,
                                  static_cast<__nv_bfloat16*>(f1), static_cast<__nv_bfloat16*>(f2), nullptr, stream));
    if (s == SVDQ_OK)
      s = svdq_prepare_weights(fmt, K, N, rank, W_t, lambda, f1, f2, bias, lora_A, lora_B, lora_rank, act_scale,
                               stream, out);
    cudaFree(f1);
    cudaFree(f2);
    return s;
  }

  svdq_weights* w = new (std::nothrow) svdq_weights();
  if (!w) return SVDQ_ERR_NO_MEMORY;
  cudaGetDevice(&w->dev);
  w->fmt = fmt;
  w->K = K;
  w->N = N;
  w->rank = rank;
  w->lora_rank = lora_rank;
  w->r_tot = r_tot;
  w->K_pad = round_up(K, 256);
  w->N_pad = round_up(N, 256);
  w->r_pad = round_up(r_tot, 64);
  const size_t qr_b = (size_t)w->N_pad * (w->K_pad / 2);
  const size_t sr_b = fmt == SVDQ_NVFP4 ? (size_t)w->N_pad * (w->K_pad / 16) : (size_t)w->N_pad * (w->K_pad / 64) * 4;
  float* R = nullptr;
  unsigned* amax = nullptr;
  bool ok = cudaMalloc(&w->qR, qr_b) == cudaSuccess && cudaMalloc(&w->sR, sr_b) == cudaSuccess &&
            (fmt != SVDQ_NVFP4 || cudaMalloc(&w->sR_rep, 4 * sr_b) == cudaSuccess) &&
            (fmt != SVDQ_INT4 || cudaMalloc(&w->qR8, 2 * qr_b) == cudaSuccess) &&
            cudaMalloc(&w->L1t, (size_t)r_tot * w->K_pad * 2) == cudaSuccess &&
            cudaMalloc(&w->L2a, (size_t)w->N_pad * w->r_pad * 2) == cudaSuccess &&
            cudaMalloc(&w->bias_f, (size_t)w->N_pad * 4) == cudaSuccess &&
            cudaMalloc(&w->lambda_inv, (size_t)K * 4) == cudaSuccess &&
            cudaMalloc(&w->lambda_inv_k1, (size_t)w->K_pad * 4) == cudaSuccess &&
            cudaMalloc(&R, (size_t)N * K * 4) == cudaSuccess && cudaMalloc(&amax, 256) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_buffers(w);
    cudaFree(R);
    cudaFree(amax);
    delete w;
    return SVDQ_ERR_NO_MEMORY;
  }
  PrepParams p;
  p.fmt = (int)fmt;
  p.K = K;
  p.N = N;
  p.K_pad = w->K_pad;
  p.N_pad = w->N_pad;
  p.rank = rank;
  p.lora_rank = lora_rank;
  p.r_tot = r_tot;
  p.r_pad = w->r_pad;
  p.Wt = static_cast<const __nv_bfloat16*>(W_t);
  p.lambda = lambda;
  p.L1f = static_cast<const __nv_bfloat16*>(L1f);
  p.L2 = static_cast<const __nv_bfloat16*>(L2);
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.loraA = static_cast<const __nv_bfloat16*>(lora_A);
  p.loraB = static_cast<const __nv_bfloat16*>(lora_B);
  p.R = R;
  p.amax_bits = amax;
  p.qR = w->qR;
  p.sR = w->sR;
  p.sR_rep = w->sR_rep;
  p.qR8 = w->qR8;
  p.L1t = w->L1t;
  p.L2a = w->L2a;
  p.bias_f = w->bias_f;
  p.lambda_inv = w->lambda_inv;
  p.lambda_inv_k1 = w->lambda_inv_k1;

  unsigned amax_host = 0;
  cudaError_t e = launch_prepare_residual(p, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&amax_host, amax, sizeof(unsigned), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess) {
    float a;
    std::memcpy(&a, &amax_host, 4);
    if (fmt == SVDQ_NVFP4) {
      // k: the smallest integer with 2^k >= s_tX amax(|R|) / 2688; then
      // s_tR = fl32(2^k / s_tX), so alpha = s_tX s_tR is the power of two 2^k
      // (to one float32 rounding) and L2 / alpha below is exact in bf16.
      const double x = (a > 0.f ? (double)a : 2688.0) * (double)act_scale / 2688.0;
      int e = 0;
      const double m = std::frexp(x, &e);
      const int k = (m == 0.5) ? e - 1 : e;
      w->s_tX = act_scale;
      w->s_tR = std::ldexp(1.0f, k) / act_scale;
      w->alpha = std::ldexp(1.0f, k);
    } else {
      w->s_tR = 1.f;
      w->s_tX = 1.f;
      w->alpha = 1.f;
    }
    e = launch_prepare_quantize(p, w->s_tR, w->alpha, stream);
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  cudaFree(R);
  cudaFree(amax);
  bool maps = e == cudaSuccess &&
              tmap_2d(&w->tm_qR, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->qR, w->K_pad / 2, w->N_pad, w->K_pad / 2,
                      128, K2_NV_ROWS_B) &&
              tmap_2d(&w->tm_L2a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L2a, w->r_pad, w->N_pad,
                      (uint64_t)w->r_pad * 2, 64, K2_NV_ROWS_B) &&
              tmap_2d(&w->tm_L2a_i4, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->L2a, w->r_pad, w->N_pad,
                      (uint64_t)w->r_pad * 2, 64, K2_I4_ROWS) &&
              (fmt != SVDQ_INT4 || tmap_2d(&w->tm_qR8, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->qR8, w->K_pad, w->N_pad,
                                           w->K_pad, 128, K2_I4_ROWS));
  if (!maps) {
    free_buffers(w);
    delete w;
    return e != cudaSuccess ? from_cuda(e) : SVDQ_ERR_CUDA;
  }
  *out = w;
  return SVDQ_OK;
}

svdq_status svdq_lowrank_factors(int K, int N, int rank, const void* W_t, const float* lambda,
                                 unsigned long long seed, void* L1f, void* L2, double* sigma, cudaStream_t stream) {
  if (!W_t || !lambda || !L1f || !L2) return SVDQ_ERR_INVALID_ARG;
  if (K <= 0 || N <= 0 || rank < 1 || rank > std::min(K, N)) return SVDQ_ERR_SHAPE;
  if (!aligned16(W_t) || !aligned16(lambda) || !aligned16(L1f) || !aligned16(L2)) return SVDQ_ERR_ALIGNMENT;
  DevState* d = nullptr;
  svdq_status s = current_device(&d);
  if (s != SVDQ_OK) return s;
  cudaError_t e = lowrank_factors(K, N, rank, static_cast<const __nv_bfloat16*>(W_t), lambda, seed,
                                  static_cast<__nv_bfloat16*>(L1f), static_cast<__nv_bfloat16*>(L2), sigma, stream);
  if (e == cudaErrorMemoryAllocation) {
    cudaGetLastError();
    return SVDQ_ERR_NO_MEMORY;
  }
  return from_cuda(e);
}

svdq_status svdq_free_weights(svdq_weights* w) {
  if (!w) return SVDQ_OK;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(w->dev);
  cudaDeviceSynchronize();
  free_buffers(w);
  if (prev >= 0) cudaSetDevice(prev);
  delete w;
  cudaGetLastError();
  return SVDQ_OK;
}

svdq_status svdq_weights_view(const svdq_weights* w, svdq_weights_info* info) {
  if (!w || !info) return SVDQ_ERR_INVALID_ARG;
  info->fmt = (int)w->fmt;
  info->K = w->K;
  info->N = w->N;
  info->rank = w->rank;
  info->lora_rank = w->lora_rank;
  info->r_tot = w->r_tot;
  info->K_pad = w->K_pad;
  info->N_pad = w->N_pad;
  info->r_pad = w->r_pad;
  info->qR = w->qR;
  info->sR = w->sR;
  info->L1t = w->L1t;
  info->L2a = w->L2a;
  info->bias = w->bias_f;
  info->lambda_inv = w->lambda_inv;
  info->s_tR = w->s_tR;
  info->s_tX = w->s_tX;
  info->alpha = w->alpha;
  return SVDQ_OK;
}

svdq_status svdq_act_buffer_sizes(const svdq_weights* w, int M, size_t* qx, size_t* sx, size_t* lr) {
  if (!w) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (qx) *qx = qx_bytes(w, M);
  if (sx) *sx = sx_bytes(w, M);
  if (lr) *lr = lr_bytes(w, M);
  return SVDQ_OK;
}

svdq_status svdq_quantize_act_lowrank_down(const svdq_weights* w, int M, const void* X, void* qX, void* sX,
                                           void* LR, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !qX || !sX || !LR))) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(qX) || !aligned16(sX) || !aligned16(LR)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  return run_k1(w, M, X, qX, sX, LR, 1, 1, stream);
}

svdq_status svdq_w4a4_gemm_lowrank_up(const svdq_weights* w, int M, const void* qX, const void* sX,
                                      const void* LR, svdq_epilogue epi, void* Y, cudaStream_t stream) {
  if (!w || (M > 0 && (!qX || !sX || !LR || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(qX) || !aligned16(sX) || !aligned16(LR) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  return run_k2(w, M, qX, sX, LR, epi, Y, true, stream);
}

size_t svdq_linear_workspace_bytes(const svdq_weights* w, int M) {
  if (!w || M < 0) return 0;
  return align256(qx_bytes(w, M)) + align256(sx_bytes(w, M)) + align256(lr_bytes(w, M));
}

static svdq_status carve(const svdq_weights* w, int M, void* ws, size_t ws_bytes, void** qX, void** sX,
                         void** LR) {
  if (!ws || ws_bytes < svdq_linear_workspace_bytes(w, M)) return SVDQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return SVDQ_ERR_ALIGNMENT;
  uint8_t* b = static_cast<uint8_t*>(ws);
  *qX = b;
  *sX = b + align256(qx_bytes(w, M));
  *LR = b + align256(qx_bytes(w, M)) + align256(sx_bytes(w, M));
  return SVDQ_OK;
}

svdq_status svdq_linear(const svdq_weights* w, int M, const void* X, svdq_epilogue epi, void* Y, void* workspace,
                        size_t ws_bytes, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  void *qX, *sX, *LR;
  svdq_status s = carve(w, M, workspace, ws_bytes, &qX, &sX, &LR);
  if (s != SVDQ_OK) return s;
  s = run_k1(w, M, X, qX, sX, LR, 1, 1, stream);
  if (s != SVDQ_OK) return s;
  return run_k2(w, M, qX, sX, LR, epi, Y, true, stream);
}

// [svdq_linear's workspace | 256-byte record | amax slots]
size_t svdq_linear_dynamic_workspace_bytes(const svdq_weights* w, int M) {
  if (!w || M < 0) return 0;
  return svdq_linear_workspace_bytes(w, M) + 256 + align256((size_t)AMAX_MAX_PARTS * 4);
}

svdq_status svdq_linear_dynamic(const svdq_weights* w, int M, const void* X, svdq_epilogue epi, void* Y,
                                void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  if (!workspace || ws_bytes < svdq_linear_dynamic_workspace_bytes(w, M)) return SVDQ_ERR_WORKSPACE;
  void *qX, *sX, *LR;
  svdq_status s = carve(w, M, workspace, ws_bytes, &qX, &sX, &LR);
  if (s != SVDQ_OK) return s;
  if (w->fmt != SVDQ_NVFP4) {   // INT4 has no tensor scale: the static layer
    if ((s = run_k1(w, M, X, qX, sX, LR, 1, 1, stream)) != SVDQ_OK) return s;
    return run_k2(w, M, qX, sX, LR, epi, Y, true, stream);
  }
  DevState* d = nullptr;
  if ((s = check_handle_device(w, &d)) != SVDQ_OK) return s;
  uint8_t* tail = static_cast<uint8_t*>(workspace) + svdq_linear_workspace_bytes(w, M);
  DynScale dyn;
  dyn.record = reinterpret_cast<float*>(tail);
  dyn.parts = reinterpret_cast<const uint32_t*>(tail + 256);
  dyn.n_parts = act_amax_num_parts(w->K, d->num_sms);
  if (dyn.n_parts <= 0) return SVDQ_ERR_SHAPE;
  s = from_cuda(launch_act_amax(static_cast<const __nv_bfloat16*>(X), M, w->K, w->lambda_inv,
                                reinterpret_cast<uint32_t*>(tail + 256), d->num_sms, stream));
  if (s != SVDQ_OK) return s;
  if ((s = run_k1(w, M, X, qX, sX, LR, 1, 1, stream, &dyn)) != SVDQ_OK) return s;
  return run_k2(w, M, qX, sX, LR, epi, Y, true, stream, &dyn);
}

// ---------------------------------------------------------------- one layer into the next
// [layer 1's workspace | the next layer's LR partials]
static size_t emit_part_bytes(const svdq_weights* w1, const svdq_weights* w2, int M) {
  return align256((size_t)(w1->N_pad / 256) * round_up(M, 128) * LR_PART_STRIDE * 4);
}

static svdq_status check_pair(const svdq_weights* w1, const svdq_weights* w2) {
  if (!w1 || !w2) return SVDQ_ERR_INVALID_ARG;
  if (w1->fmt != SVDQ_NVFP4 || w2->fmt != SVDQ_NVFP4) return SVDQ_ERR_INVALID_ARG;
  if (w2->K != w1->N || w2->K_pad != w1->N_pad || w2->r_tot > 64) return SVDQ_ERR_SHAPE;
  return w1->dev == w2->dev ? SVDQ_OK : SVDQ_ERR_INVALID_ARG;
}

size_t svdq_linear_emit_next_workspace_bytes(const svdq_weights* w1, const svdq_weights* w2, int M) {
  if (check_pair(w1, w2) != SVDQ_OK || M < 0) return 0;
  return svdq_linear_workspace_bytes(w1, M) + emit_part_bytes(w1, w2, M);
}

svdq_status svdq_linear_emit_next(const svdq_weights* w1, const svdq_weights* w2, int M, const void* X,
                                  svdq_epilogue epi, void* qX2, void* sX2, void* LR2, void* workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
  svdq_status s = check_pair(w1, w2);
  if (s != SVDQ_OK) return s;
  if (M > 0 && (!X || !qX2 || !sX2 || !LR2)) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned32(qX2) || !aligned16(sX2) || !aligned16(LR2)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  if (!workspace || ws_bytes < svdq_linear_emit_next_workspace_bytes(w1, w2, M)) return SVDQ_ERR_WORKSPACE;
  void *qX, *sX, *LR;
  if ((s = carve(w1, M, workspace, ws_bytes, &qX, &sX, &LR)) != SVDQ_OK) return s;
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + svdq_linear_workspace_bytes(w1, M));
  if ((s = run_k1(w1, M, X, qX, sX, LR, 1, 1, stream)) != SVDQ_OK) return s;
  K2Params::Next nx;
  nx.inv_lambda = w2->lambda_inv;
  nx.L1t = w2->L1t;
  nx.s_t = w2->s_tX;
  nx.six_st = 6.0f * w2->s_tX;   // one IEEE float32 multiply, as for kernel 1
  nx.r_tot = w2->r_tot;
  nx.qX = static_cast<uint8_t*>(qX2);
  nx.sX = static_cast<uint8_t*>(sX2);
  nx.part = part;
  if ((s = run_k2(w1, M, qX, sX, LR, epi, nullptr, true, stream, nullptr, &nx)) != SVDQ_OK) return s;
  return from_cuda(launch_next_lr_reduce(part, w1->N_pad / 256, M, round_up(M, 128), w2->r_tot, w2->r_pad,
                                         static_cast<__nv_bfloat16*>(LR2), stream));
}

size_t svdq_mlp_workspace_bytes(const svdq_weights* w1, const svdq_weights* w2, int M) {
  if (check_pair(w1, w2) != SVDQ_OK || M < 0) return 0;
  return svdq_linear_emit_next_workspace_bytes(w1, w2, M) + svdq_linear_workspace_bytes(w2, M);
}

svdq_status svdq_mlp(const svdq_weights* w1, const svdq_weights* w2, int M, const void* X, svdq_epilogue epi1,
                     svdq_epilogue epi2, void* Y, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  svdq_status s = check_pair(w1, w2);
  if (s != SVDQ_OK) return s;
  if (M > 0 && (!X || !Y)) return SVDQ_ERR_INVALID_ARG;
  if (epi2 != SVDQ_EPI_NONE && epi2 != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  if (!workspace || ws_bytes < svdq_mlp_workspace_bytes(w1, w2, M)) return SVDQ_ERR_WORKSPACE;
  const size_t e1 = svdq_linear_emit_next_workspace_bytes(w1, w2, M);
  void *qX2, *sX2, *LR2;
  if ((s = carve(w2, M, static_cast<uint8_t*>(workspace) + e1, ws_bytes - e1, &qX2, &sX2, &LR2)) != SVDQ_OK) return s;
  if ((s = svdq_linear_emit_next(w1, w2, M, X, epi1, qX2, sX2, LR2, workspace, e1, stream)) != SVDQ_OK) return s;
  return run_k2(w2, M, qX2, sX2, LR2, epi2, Y, true, stream);
}

svdq_status svdq_quantize_act(const svdq_weights* w, int M, const void* X, void* qX, void* sX,
                              cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !qX || !sX))) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(qX) || !aligned16(sX)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  return run_k1(w, M, X, qX, sX, nullptr, 1, 0, stream);
}

svdq_status svdq_lowrank_down(const svdq_weights* w, int M, const void* X, void* LR, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !LR))) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(LR)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  return run_k1(w, M, X, nullptr, nullptr, LR, 0, 1, stream);
}

svdq_status svdq_w4a4_gemm(const svdq_weights* w, int M, const void* qX, const void* sX, void* Y,
                           cudaStream_t stream) {
  if (!w || (M > 0 && (!qX || !sX || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(qX) || !aligned16(sX) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  return run_k2(w, M, qX, sX, nullptr, SVDQ_EPI_NONE, Y, false, stream);
}

svdq_status svdq_lowrank_up(const svdq_weights* w, int M, const void* LR, svdq_epilogue epi, void* Y,
                            cudaStream_t stream) {
  if (!w || (M > 0 && (!LR || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(LR) || !aligned16(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  DevState* d = nullptr;
  svdq_status s = check_handle_device(w, &d);
  if (s != SVDQ_OK) return s;
  UpParams p;
  p.M = M;
  p.N = w->N;
  p.r_tot = w->r_tot;
  p.r_pad = w->r_pad;
  p.LR = static_cast<const __nv_bfloat16*>(LR);
  p.L2a = w->L2a;
  p.alpha = w->alpha;
  p.epi = (int)epi;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  return from_cuda(launch_lowrank_up(p, stream));
}

svdq_status svdq_linear_unfused(const svdq_weights* w, int M, const void* X, svdq_epilogue epi, void* Y,
                                void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (epi != SVDQ_EPI_NONE && epi != SVDQ_EPI_GELU_TANH) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  void *qX, *sX, *LR;
  svdq_status s = carve(w, M, workspace, ws_bytes, &qX, &sX, &LR);
  if (s != SVDQ_OK) return s;
  if ((s = svdq_quantize_act(w, M, X, qX, sX, stream)) != SVDQ_OK) return s;
  if ((s = svdq_lowrank_down(w, M, X, LR, stream)) != SVDQ_OK) return s;
  if ((s = svdq_w4a4_gemm(w, M, qX, sX, Y, stream)) != SVDQ_OK) return s;
  return svdq_lowrank_up(w, M, LR, epi, Y, stream);
}

svdq_status svdq_awq_prepare(int K, int N, const void* W_t, const float* s, const void* bias, cudaStream_t stream,
                             svdq_awq_weights** out) {
  if (out) *out = nullptr;
  if (!out || !W_t) return SVDQ_ERR_INVALID_ARG;
  if (K <= 0 || K % 64 || N <= 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(W_t) || !aligned16(s) || !aligned16(bias)) return SVDQ_ERR_ALIGNMENT;
  DevState* d = nullptr;
  svdq_status st = current_device(&d);
  if (st != SVDQ_OK) return st;
  svdq_awq_weights* w = new (std::nothrow) svdq_awq_weights();
  if (!w) return SVDQ_ERR_NO_MEMORY;
  cudaGetDevice(&w->dev);
  w->K = K;
  w->N = N;
  w->N_pad = round_up(N, 32);
  const size_t G = (size_t)K / 64;
  const bool ok = cudaMalloc(&w->code, (size_t)w->N_pad * K / 2) == cudaSuccess &&
                  cudaMalloc(&w->scale, G * w->N_pad * 2) == cudaSuccess &&
                  cudaMalloc(&w->zero, G * w->N_pad) == cudaSuccess &&
                  cudaMalloc(&w->inv_s, (size_t)K * 4) == cudaSuccess &&
                  cudaMalloc(&w->bias_f, (size_t)w->N_pad * 4) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_awq(w);
    delete w;
    return SVDQ_ERR_NO_MEMORY;
  }
  AwqPrepParams p;
  p.K = K;
  p.N = N;
  p.N_pad = w->N_pad;
  p.Wt = static_cast<const __nv_bfloat16*>(W_t);
  p.s = s;
  p.bias = static_cast<const __nv_bfloat16*>(bias);
  p.code = w->code;
  p.scale = w->scale;
  p.zero = w->zero;
  p.inv_s = w->inv_s;
  p.bias_f = w->bias_f;
  cudaError_t e = launch_awq_quantize(p, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    free_awq(w);
    delete w;
    return from_cuda(e);
  }
  // stage boxes: 16 code chunks x 32 features x 16 bytes; 8 groups x 32 features of scales and zero points
  w->has_s = s != nullptr;
  const bool maps =
      tmap_3d_u8(&w->tm_code, w->code, 16, w->N_pad, (uint64_t)K / 32, 16, (uint64_t)w->N_pad * 16, 16, 32, 16) &&
      tmap_3d_u8(&w->tm_code_g, w->code, 16, w->N_pad, (uint64_t)K / 32, 16, (uint64_t)w->N_pad * 16, 16, 256, 2) &&
      tmap_2d(&w->tm_scale_g, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w->scale, w->N_pad, G, (uint64_t)w->N_pad * 2, 256, 1,
              CU_TENSOR_MAP_SWIZZLE_NONE) &&
      tmap_2d(&w->tm_zero_g, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->zero, w->N_pad, G, w->N_pad, 256, 1,
              CU_TENSOR_MAP_SWIZZLE_NONE) &&
      tmap_2d(&w->tm_scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, w->scale, w->N_pad, G, (uint64_t)w->N_pad * 2, 32, 8,
              CU_TENSOR_MAP_SWIZZLE_NONE) &&
      tmap_2d(&w->tm_zero, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->zero, w->N_pad, G, w->N_pad, 32, 8,
              CU_TENSOR_MAP_SWIZZLE_NONE);
  if (!maps) {
    free_awq(w);
    delete w;
    return SVDQ_ERR_CUDA;
  }
  *out = w;
  return SVDQ_OK;
}

svdq_status svdq_awq_free(svdq_awq_weights* w) {
  if (!w) return SVDQ_OK;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(w->dev);
  cudaDeviceSynchronize();
  free_awq(w);
  if (prev >= 0) cudaSetDevice(prev);
  delete w;
  cudaGetLastError();
  return SVDQ_OK;
}

svdq_status svdq_awq_view(const svdq_awq_weights* w, svdq_awq_info* info) {
  if (!w || !info) return SVDQ_ERR_INVALID_ARG;
  info->K = w->K;
  info->N = w->N;
  info->N_pad = w->N_pad;
  info->code = w->code;
  info->scale = w->scale;
  info->zero = w->zero;
  info->inv_s = w->inv_s;
  info->bias = w->bias_f;
  return SVDQ_OK;
}

svdq_status svdq_awq_linear(const svdq_awq_weights* w, int M, const void* X, void* Y, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned16(Y)) return SVDQ_ERR_ALIGNMENT;
  if (M == 0) return SVDQ_OK;
  DevState* d = nullptr;
  svdq_status st = current_device(&d);
  if (st != SVDQ_OK) return st;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != w->dev) return SVDQ_ERR_INVALID_ARG;
  AwqParams p;
  p.M = M;
  p.K = w->K;
  p.N = w->N;
  p.N_pad = w->N_pad;
  p.mb = awq_rows_per_block(w->K, M);
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.code = w->code;
  p.scale = w->scale;
  p.zero = w->zero;
  p.inv_s = w->inv_s;
  p.bias = w->bias_f;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.err = dev_err(d);
  return from_cuda(launch_awq_gemv(w->tm_code, w->tm_scale, w->tm_zero, p, d->num_sms, stream));
}

svdq_status svdq_awq_gemm(const svdq_awq_weights* w, int M, const void* X, void* Y, cudaStream_t stream) {
  if (!w || (M > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (M < 0 || w->N % 16) return SVDQ_ERR_SHAPE;
  if (!aligned16(X) || !aligned32(Y)) return SVDQ_ERR_ALIGNMENT;
  DevState* d = nullptr;
  svdq_status st = current_device(&d);
  if (st != SVDQ_OK) return st;
  int dev = -1;
  cudaGetDevice(&dev);
  if (dev != w->dev) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  CUtensorMap tmX;
  if (!tmap_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, w->K, M, (uint64_t)w->K * 2, 64, 128))
    return SVDQ_ERR_CUDA;
  AwqGemmParams p;
  p.M = M;
  p.K = w->K;
  p.N = w->N;
  p.N_pad = w->N_pad;
  p.num_m_blocks = (M + 127) / 128;
  p.num_n_blocks = (w->N + 255) / 256;
  p.inv_s = w->inv_s;
  p.bias = w->bias_f;
  p.Y = static_cast<__nv_bfloat16*>(Y);
  p.err = dev_err(d);
  return from_cuda(launch_awq_gemm(tmX, w->tm_code_g, w->tm_scale_g, w->tm_zero_g, p, w->has_s, d->num_sms, stream));
}

svdq_status svdq_poll_device_error(cudaStream_t stream) {
  DevState* d = nullptr;
  svdq_status s = current_device(&d);
  if (s != SVDQ_OK) return s;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  unsigned v = 0;
  if (cudaMemcpy(&v, d->err_word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess)
    return from_cuda(cudaErrorUnknown);
  if (v && cudaMemset(d->err_word, 0, sizeof(unsigned)) != cudaSuccess) return from_cuda(cudaErrorUnknown);
  if (v & ERR_TIMEOUT) return SVDQ_ERR_TIMEOUT;
  if (v & ERR_BOUNDS) return SVDQ_ERR_DEVICE_FAULT;
  return SVDQ_OK;
}

svdq_status svdq_selftest_wait_timeout(unsigned limit_us, cudaStream_t stream) {
  if (limit_us == 0 || limit_us > 10000000u) return SVDQ_ERR_INVALID_ARG;
  DevState* d = nullptr;
  svdq_status s = current_device(&d);
  if (s != SVDQ_OK) return s;
  DeviceErr e{d->err_word, (unsigned long long)limit_us * 1000ull};
  return from_cuda(launch_selftest_timeout(e, stream));
}

}  // extern "C"
