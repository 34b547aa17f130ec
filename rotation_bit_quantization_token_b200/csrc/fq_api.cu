// Host layer of libfq: the C ABI declared in include/fq.h.
//
// Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
// quantization fusion" (http://www.zwxr.cn/news/277566). fq_create is the plan phase of
// the page's two-phase interface (GetWorkspaceSize: validation, shape checks, tiling);
// fq_quantize_* is the execute phase (launch on a stream). The checks follow the page's
// parameter table and error-code table.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <new>

#include "fq.h"
#include "fq_internal.h"

struct fq_handle {
  int64_t K;
  int M, N;
  fq_dtype dtype;
  int device;
  int num_sms;
  fq_kernel pref;
  fq_kernel last;
  int last_launches;
  uint32_t* d_status;  // 256-byte device block; word 0 = status
  uint64_t debug_timeout_ns;  // one-shot test hook for the next tensor-core launch
  int debug_stall;
  int round_x1;  // intermediate rounding of x' (general kernel only)
};

namespace {

thread_local int g_last_cuda_error = 0;

fq_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = int(e);
  return FQ_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The tensor-core kernel moves x with TMA, P1 / P2 with 16-byte loads and the outputs
// with bulk copies, so all of them must be 16-byte aligned.
bool use_tc(const fq_handle* h, const void* x, const void* P1, const void* P2, const void* out,
            const void* scales) {
  if (h->pref == FQ_KERNEL_GENERAL || h->round_x1) return false;
  if (!fq::tc_supported(h->K, h->M, h->N)) return false;
  return aligned(x, 16) && aligned(P1, 16) && (P2 == nullptr || aligned(P2, 16)) &&
         aligned(out, 16) && (scales == nullptr || aligned(scales, 16));
}

int general_grid(const fq_handle* h) {
  const int64_t want = int64_t(h->num_sms) * 4;
  return int(h->K < want ? h->K : want);
}

fq_status launch(fq_handle* h, int mode, const void* x, const void* P1, const void* P2,
                 double clip, fq::MxRule rule, uint8_t* out, float* qs, uint8_t* scales,
                 float* x2, cudaStream_t s) {
  const bool fp16_in = h->dtype == FQ_FP16;
  const void* out_probe = (mode == fq::kModeRotate) ? static_cast<const void*>(x2) : out;
  if (use_tc(h, x, P1, P2, out_probe, mode == fq::kModeMx ? scales : nullptr)) {
    fq::TcParams p{};
    p.x = x; p.P1 = P1; p.P2 = P2; p.K = h->K; p.M = h->M; p.N = h->N; p.mode = mode;
    p.clip_ratio = clip; p.rule = rule; p.out = out; p.quant_scale = qs; p.scales = scales;
    p.x2 = x2; p.status = h->d_status;
    p.timeout_ns = h->debug_timeout_ns; p.stall_loads = h->debug_stall;
    h->debug_timeout_ns = 0;
    h->debug_stall = 0;
    cudaError_t e = fq::launch_tc(p, fp16_in, h->num_sms, s);
    if (e != cudaSuccess) return cuda_fail(e);
    h->last = FQ_KERNEL_TCGEN05;
    h->last_launches = 1;
    return FQ_OK;
  }
  if (h->pref == FQ_KERNEL_TCGEN05) return FQ_ERR_UNSUPPORTED;
  fq::GeneralParams p{};
  p.x = x; p.P1 = P1; p.P2 = P2; p.K = h->K; p.M = h->M; p.N = h->N; p.mode = mode;
  p.clip_ratio = clip; p.rule = rule; p.out = out; p.quant_scale = qs; p.scales = scales;
  p.x2 = x2;
  p.round_x1 = h->round_x1;
  cudaError_t e = fq::launch_general(p, fp16_in, general_grid(h), s);
  if (e != cudaSuccess) return cuda_fail(e);
  h->last = FQ_KERNEL_GENERAL;
  h->last_launches = 1;
  return FQ_OK;
}

}  // namespace

void fq::record_cuda_error(int e) { g_last_cuda_error = e; }

bool fq::mx_rule_from(double d, fq::MxRule* r) {
  if (!(d == 0.0 || (d >= 6.0 && d <= 12.0))) return false;
  if (d == 0.0) r->mode = fq::kMxFloor;
  else if (d == 6.0) r->mode = fq::kMxMantissa6;
  else if (d == 7.0) r->mode = fq::kMxMantissa7;
  else r->mode = fq::kMxRatio;
  r->dst_max = float(d);
  r->inv_dst = d > 0.0 ? float(1.0 / double(float(d))) : 0.0f;
  return true;
}

extern "C" {

fq_status fq_create(fq_handle** h, int64_t K, int64_t M, int64_t N, fq_dtype dtype) {
  if (h == nullptr) return FQ_ERR_NULLPTR;
  *h = nullptr;
  // page, parameter table: K in [1, 262144], M and N in [1, 256]
  if (K < 1 || K > 262144 || M < 1 || M > 256 || N < 1 || N > 256) return FQ_ERR_INVALID;
  if (dtype != FQ_BF16 && dtype != FQ_FP16) return FQ_ERR_INVALID;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (fq::general_smem_bytes(int(M), int(N), 2) > size_t(optin)) return FQ_ERR_UNSUPPORTED;
  fq_handle* hh = new (std::nothrow) fq_handle();
  if (hh == nullptr) return FQ_ERR_CUDA;
  hh->K = K; hh->M = int(M); hh->N = int(N); hh->dtype = dtype; hh->device = dev;
  hh->num_sms = sms; hh->pref = FQ_KERNEL_AUTO; hh->last = FQ_KERNEL_AUTO; hh->last_launches = 0;
  e = cudaMalloc(reinterpret_cast<void**>(&hh->d_status), 256);
  if (e == cudaSuccess) e = cudaMemset(hh->d_status, 0, 256);
  if (e != cudaSuccess) {
    if (hh->d_status) cudaFree(hh->d_status);
    delete hh;
    return cuda_fail(e);
  }
  *h = hh;
  return FQ_OK;
}

fq_status fq_destroy(fq_handle* h) {
  if (h == nullptr) return FQ_OK;
  cudaError_t e = cudaFree(h->d_status);
  delete h;
  return e == cudaSuccess ? FQ_OK : cuda_fail(e);
}

fq_status fq_quantize_per_token(fq_handle* h, const void* x, const void* P1, const void* P2,
                                double clipRatio, fq_int_out fmt, void* out,
                                float* quantScale, struct CUstream_st* stream) {
  if (h == nullptr || x == nullptr || P1 == nullptr || P2 == nullptr || out == nullptr ||
      quantScale == nullptr)
    return FQ_ERR_NULLPTR;
  // page: clipRatio in (0, 1]
  if (!(clipRatio > 0.0 && clipRatio <= 1.0)) return FQ_ERR_INVALID;
  // page: INT4 needs N even, INT32 needs N % 8 == 0
  if (fmt == FQ_OUT_INT4) {
    if (h->N % 2 != 0) return FQ_ERR_INVALID;
  } else if (fmt == FQ_OUT_INT32) {
    if (h->N % 8 != 0 || !aligned(out, 4)) return FQ_ERR_INVALID;
  } else {
    return FQ_ERR_INVALID;
  }
  if (!aligned(x, 2) || !aligned(P1, 2) || !aligned(P2, 2) || !aligned(quantScale, 4))
    return FQ_ERR_INVALID;
  fq::MxRule rule{fq::kMxFloor, 0.0f, 0.0f};
  return launch(h, fq::kModePerToken, x, P1, P2, clipRatio, rule, static_cast<uint8_t*>(out),
                quantScale, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

fq_status fq_quantize_mx(fq_handle* h, const void* x, const void* P1, const void* P2,
                         double dstTypeMax, void* out_fp4, uint8_t* scale_e8m0,
                         struct CUstream_st* stream) {
  if (h == nullptr || x == nullptr || P1 == nullptr || out_fp4 == nullptr ||
      scale_e8m0 == nullptr)
    return FQ_ERR_NULLPTR;
  fq::MxRule rule;
  if (!fq::mx_rule_from(dstTypeMax, &rule)) return FQ_ERR_INVALID;
  if (h->N % 2 != 0) return FQ_ERR_INVALID;  // page: FLOAT4_E2M1 needs N even
  if (!aligned(x, 2) || !aligned(P1, 2) || (P2 != nullptr && !aligned(P2, 2)))
    return FQ_ERR_INVALID;
  return launch(h, fq::kModeMx, x, P1, P2, 1.0, rule, static_cast<uint8_t*>(out_fp4), nullptr,
                scale_e8m0, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

fq_status fq_debug_rotate(fq_handle* h, const void* x, const void* P1, const void* P2,
                          float* x2, struct CUstream_st* stream) {
  if (h == nullptr || x == nullptr || P1 == nullptr || x2 == nullptr) return FQ_ERR_NULLPTR;
  if (!aligned(x, 2) || !aligned(P1, 2) || (P2 != nullptr && !aligned(P2, 2)) || !aligned(x2, 4))
    return FQ_ERR_INVALID;
  fq::MxRule rule{fq::kMxFloor, 0.0f, 0.0f};
  return launch(h, fq::kModeRotate, x, P1, P2, 1.0, rule, nullptr, nullptr, nullptr, x2,
                reinterpret_cast<cudaStream_t>(stream));
}

fq_status fq_mx_matmul(int64_t T, int64_t O, int64_t L, const void* a_fp4, const uint8_t* a_scale_e8m0,
                       const void* w_fp4, const uint8_t* w_scale_e8m0, float* C, uint32_t* status,
                       struct CUstream_st* stream) {
  if (a_fp4 == nullptr || a_scale_e8m0 == nullptr || w_fp4 == nullptr || w_scale_e8m0 == nullptr ||
      C == nullptr)
    return FQ_ERR_NULLPTR;
  // L is the flattened token M*N of the operator (M, N in [1, 256]), whole groups of 32;
  // T and O are token counts (page: K in [1, 262144])
  if (T < 1 || T > 262144 || O < 1 || O > 262144 || L < 32 || L > 65536 || L % 32 != 0)
    return FQ_ERR_INVALID;
  if (!aligned(a_fp4, 16) || !aligned(w_fp4, 16) || !aligned(C, 4) || (status && !aligned(status, 4)))
    return FQ_ERR_INVALID;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  fq::MxGemmParams p{a_fp4, a_scale_e8m0, w_fp4, w_scale_e8m0, C, status, T, O, L};
  e = fq::launch_mxgemm(p, sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FQ_OK : cuda_fail(e);
}

fq_status fq_set_kernel(fq_handle* h, fq_kernel kernel) {
  if (h == nullptr) return FQ_ERR_NULLPTR;
  if (kernel != FQ_KERNEL_AUTO && kernel != FQ_KERNEL_GENERAL && kernel != FQ_KERNEL_TCGEN05)
    return FQ_ERR_INVALID;
  if (kernel == FQ_KERNEL_TCGEN05 && !fq::tc_supported(h->K, h->M, h->N))
    return FQ_ERR_UNSUPPORTED;
  h->pref = kernel;
  return FQ_OK;
}

fq_status fq_set_intermediate_rounding(fq_handle* h, int enable) {
  if (h == nullptr) return FQ_ERR_NULLPTR;
  if (enable != 0 && enable != 1) return FQ_ERR_INVALID;
  h->round_x1 = enable;
  return FQ_OK;
}

fq_kernel fq_last_kernel(const fq_handle* h) { return h ? h->last : FQ_KERNEL_AUTO; }

int fq_last_launch_count(const fq_handle* h) { return h ? h->last_launches : 0; }

fq_status fq_debug_arm_stall(fq_handle* h, double wait_limit_s) {
  if (h == nullptr) return FQ_ERR_NULLPTR;
  if (!(wait_limit_s > 0.0 && wait_limit_s <= 10.0)) return FQ_ERR_INVALID;
  h->debug_timeout_ns = uint64_t(wait_limit_s * 1e9);
  h->debug_stall = 1;
  return FQ_OK;
}

fq_status fq_device_status(fq_handle* h, uint32_t* status) {
  if (h == nullptr || status == nullptr) return FQ_ERR_NULLPTR;
  uint32_t v = 0;
  cudaError_t e = cudaMemcpy(&v, h->d_status, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  *status = v;
  if (v != 0) {
    e = cudaMemset(h->d_status, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e);
    return FQ_ERR_DEVICE_TIMEOUT;
  }
  return FQ_OK;
}

int fq_last_cuda_error(void) { return g_last_cuda_error; }

const char* fq_status_string(fq_status s) {
  switch (s) {
    case FQ_OK: return "FQ_OK";
    case FQ_ERR_NULLPTR: return "FQ_ERR_NULLPTR: a required pointer is NULL";
    case FQ_ERR_INVALID: return "FQ_ERR_INVALID: a shape, range, type or alignment rule is violated";
    case FQ_ERR_CUDA: return "FQ_ERR_CUDA: a CUDA call or kernel launch failed";
    case FQ_ERR_UNSUPPORTED: return "FQ_ERR_UNSUPPORTED: not supported on this device or shape";
    case FQ_ERR_DEVICE_TIMEOUT: return "FQ_ERR_DEVICE_TIMEOUT: a bounded wait inside a kernel gave up";
  }
  return "unknown fq_status";
}

}  // extern "C"
