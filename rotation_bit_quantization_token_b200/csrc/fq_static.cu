// Per-group quantization without any device allocation.
//
// fq_quantize_mx needs a handle from fq_create, which cudaMallocs the handle's device
// status block (the word a kernel writes when one of its bounded waits gives up). Some
// callers cannot allocate: code whose device memory is owned by another allocator or a
// fixed budget (a framework's caching pool, an inference server that reserves all
// memory at start-up), code that must not trigger the implicit device synchronization
// of cudaMalloc / cudaFree on a latency-critical path, and plug-ins that are not allowed
// to create allocations of their own. fq_quantize_mx_static serves them: the status word
// lives in a file-scope static device array, loaded with the library's module and held
// on every GPU that uses it until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fq.h"
#include "fq_internal.h"

// 256 bytes: 64 status words. One call uses word 0 only (one word per launch), so every
// shape the page allows fits.
static __device__ __align__(256) uint32_t fq_static_scratch[64];

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kScratchBytesPerCall = sizeof(uint32_t);

std::mutex g_setup_mutex;
uint32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device. In host code the array's
// name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
cudaError_t scratch_on_current_device(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, fq_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fq_status fail(cudaError_t e) {
  fq::record_cuda_error(int(e));
  return FQ_ERR_CUDA;
}

}  // namespace

extern "C" fq_status fq_quantize_mx_static(int64_t K, int64_t M, int64_t N, fq_dtype dtype,
                                           const void* x, const void* P1, const void* P2,
                                           double dstTypeMax, void* out_fp4, uint8_t* scale_e8m0,
                                           struct CUstream_st* stream) {
  if (x == nullptr || P1 == nullptr || out_fp4 == nullptr || scale_e8m0 == nullptr)
    return FQ_ERR_NULLPTR;
  if (K < 1 || K > 262144 || M < 1 || M > 256 || N < 1 || N > 256) return FQ_ERR_INVALID;
  if (dtype != FQ_BF16 && dtype != FQ_FP16) return FQ_ERR_INVALID;
  if (N % 2 != 0) return FQ_ERR_INVALID;
  if (!(dstTypeMax == 0.0 || (dstTypeMax >= 6.0 && dstTypeMax <= 12.0))) return FQ_ERR_INVALID;
  if (!aligned_to(x, 2) || !aligned_to(P1, 2) || (P2 != nullptr && !aligned_to(P2, 2)))
    return FQ_ERR_INVALID;
  if (kScratchBytesPerCall > sizeof(fq_static_scratch)) return FQ_ERR_INVALID;

  int dev = 0, sms = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return fail(e);
  if (fq::general_smem_bytes(int(M), int(N), 2) > size_t(optin)) return FQ_ERR_UNSUPPORTED;

  uint32_t* status = nullptr;
  e = scratch_on_current_device(&status);
  if (e != cudaSuccess) return fail(e);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the status word must start at zero; the array keeps whatever the last call left
  e = cudaMemsetAsync(status, 0, kScratchBytesPerCall, s);
  if (e != cudaSuccess) return fail(e);

  fq::MxRule rule;
  rule.mode = dstTypeMax == 0.0 ? fq::kMxFloor
              : dstTypeMax == 6.0 ? fq::kMxMantissa6
              : dstTypeMax == 7.0 ? fq::kMxMantissa7
                                  : fq::kMxRatio;
  rule.dst_max = float(dstTypeMax);
  rule.inv_dst = dstTypeMax > 0.0 ? float(1.0 / dstTypeMax) : 0.0f;
  const bool fp16_in = dtype == FQ_FP16;
  const bool tc = fq::tc_supported(K, int(M), int(N)) && aligned_to(x, 16) && aligned_to(P1, 16) &&
                  (P2 == nullptr || aligned_to(P2, 16)) && aligned_to(out_fp4, 16) &&
                  aligned_to(scale_e8m0, 16);
  if (tc) {
    fq::TcParams p{};
    p.x = x; p.P1 = P1; p.P2 = P2; p.K = K; p.M = int(M); p.N = int(N); p.mode = fq::kModeMx;
    p.clip_ratio = 1.0; p.rule = rule; p.out = static_cast<uint8_t*>(out_fp4); p.scales = scale_e8m0;
    p.status = status;
    e = fq::launch_tc(p, fp16_in, sms, s);
  } else {
    fq::GeneralParams p{};
    p.x = x; p.P1 = P1; p.P2 = P2; p.K = K; p.M = int(M); p.N = int(N); p.mode = fq::kModeMx;
    p.clip_ratio = 1.0; p.rule = rule; p.out = static_cast<uint8_t*>(out_fp4); p.scales = scale_e8m0;
    const int64_t want = int64_t(sms) * 4;
    e = fq::launch_general(p, fp16_in, int(K < want ? K : want), s);
  }
  return e == cudaSuccess ? FQ_OK : fail(e);
}
