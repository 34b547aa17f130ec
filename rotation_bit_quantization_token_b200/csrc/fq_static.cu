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
// on every GPU that uses it until the process exits. fq_static_device_status reads it
// back.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "fq.h"
#include "fq_internal.h"

// 256 bytes: 64 status words. One call uses word 0 only (one word per launch), so every
// shape the page allows fits.
static __device__ __align__(256) uint32_t fq_static_scratch[64];

namespace {

constexpr size_t kScratchBytesPerCall = sizeof(uint32_t);

// One-shot test hook (fq_static_debug_arm_stall): 0 = off, else the wait limit in ns for
// the next tensor-core launch made by fq_quantize_mx_static in this process.
std::atomic<uint64_t> g_stall_ns{0};

// Device address of the static scratch in the current context. In host code the array's
// name is only a host-side stand-in, so the address comes from cudaGetSymbolAddress, with
// the device of the call current. The lookup is a host-side table query, so it runs on
// every call: an address cached by device ordinal would go stale when the context it
// belongs to is destroyed (cudaDeviceReset) or when a caller runs under a context of its
// own.
cudaError_t scratch_on_current_device(uint32_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, fq_static_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<uint32_t*>(p);
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
  fq::MxRule rule;
  if (!fq::mx_rule_from(dstTypeMax, &rule)) return FQ_ERR_INVALID;
  if (!aligned_to(x, 2) || !aligned_to(P1, 2) || (P2 != nullptr && !aligned_to(P2, 2)))
    return FQ_ERR_INVALID;
  if (kScratchBytesPerCall > sizeof(fq_static_scratch)) return FQ_ERR_INVALID;

  int dev = 0, sms = 0, optin = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return fail(e);
  if (fq::general_smem_bytes(int(M), int(N), 2) > size_t(optin)) return FQ_ERR_UNSUPPORTED;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool fp16_in = dtype == FQ_FP16;
  const bool tc = fq::tc_supported(K, int(M), int(N)) && aligned_to(x, 16) && aligned_to(P1, 16) &&
                  (P2 == nullptr || aligned_to(P2, 16)) && aligned_to(out_fp4, 16) &&
                  aligned_to(scale_e8m0, 16);
  if (tc) {
    // only the tensor-core kernel has bounded waits, so only its launch uses the word
    uint32_t* status = nullptr;
    e = scratch_on_current_device(&status);
    if (e != cudaSuccess) return fail(e);
    // the status word must start at zero; the array keeps whatever the last call left
    e = cudaMemsetAsync(status, 0, kScratchBytesPerCall, s);
    if (e != cudaSuccess) return fail(e);
    fq::TcParams p{};
    p.x = x; p.P1 = P1; p.P2 = P2; p.K = K; p.M = int(M); p.N = int(N); p.mode = fq::kModeMx;
    p.clip_ratio = 1.0; p.rule = rule; p.out = static_cast<uint8_t*>(out_fp4); p.scales = scale_e8m0;
    p.status = status;
    const uint64_t stall = g_stall_ns.exchange(0);
    p.timeout_ns = stall;
    p.stall_loads = stall != 0;
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

extern "C" fq_status fq_static_device_status(uint32_t* status) {
  if (status == nullptr) return FQ_ERR_NULLPTR;
  uint32_t* word = nullptr;
  cudaError_t e = scratch_on_current_device(&word);
  if (e != cudaSuccess) return fail(e);
  uint32_t v = 0;
  e = cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(e);
  *status = v;
  if (v != 0) {
    e = cudaMemset(word, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return fail(e);
    return FQ_ERR_DEVICE_TIMEOUT;
  }
  return FQ_OK;
}

extern "C" fq_status fq_static_debug_arm_stall(double wait_limit_s) {
  if (!(wait_limit_s > 0.0 && wait_limit_s <= 10.0)) return FQ_ERR_INVALID;
  g_stall_ns.store(uint64_t(wait_limit_s * 1e9));
  return FQ_OK;
}
