// Internal declarations shared by the host layer and the kernels of libfq.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "fq_quant.cuh"

namespace fq {

enum Mode : int { kModePerToken = 0, kModeMx = 1, kModeRotate = 2 };

struct GeneralParams {
  const void* x;       // [K, M, N] 16-bit
  const void* P1;      // [M, M]
  const void* P2;      // [N, N] or nullptr (skip the right multiply)
  int64_t K;
  int M, N;
  int mode;            // Mode
  double clip_ratio;   // per-token
  MxRule rule;         // per-group
  uint8_t* out;        // packed codes, K*M*N/2 bytes
  float* quant_scale;  // [K] per-token
  uint8_t* scales;     // [K, 2*ceilDiv(M*N,64)] per-group
  float* x2;           // [K, M, N] rotate-only
  int round_x1;        // round x' = x . P2 to the input type (RNE) before the left product
};

size_t general_smem_bytes(int M, int N, int elem_bytes);
cudaError_t launch_general(const GeneralParams& p, bool fp16_in, int grid, cudaStream_t stream);

// Tensor-core kernel: M in {32, 64, 128} (128/M tokens per 128-row tile), N a multiple
// of 16 in [64, 128], 16-byte aligned x / out / scales, M*N a multiple of 32.
struct TcParams {
  const void* x;
  const void* P1;
  const void* P2;      // nullptr: identity right multiply
  int64_t K;
  int M, N;
  int mode;
  double clip_ratio;
  MxRule rule;
  uint8_t* out;
  float* quant_scale;
  uint8_t* scales;
  float* x2;
  uint32_t* status;    // device status word (bounded waits)
  uint64_t timeout_ns; // limit of every bounded wait; 0 = the default (4 s)
  int stall_loads;     // test hook: the producer issues no x loads (see fq_debug_arm_stall)
};

bool tc_supported(int64_t K, int M, int N);

// Per-group rule from dstTypeMax (page: per-group mode, cases 1-3). Returns false for a
// value outside {0} U [6, 12] (parameter table: "0.0 disables, 6.0~12.0 customizes").
// The one decoding used by every per-group entry point.
bool mx_rule_from(double dst_type_max, MxRule* rule);

// Block-scaled FP4 x FP4 contraction of two per-group outputs (see fq_mxgemm.cu):
// C [T, O] float32 = A_hat [T, L] . W_hat [O, L]^T.
struct MxGemmParams {
  const void* a_codes;      // [T, L/2] bytes, 16-byte aligned
  const uint8_t* a_scales;  // [T, 2*ceilDiv(L,64)] E8M0 bytes
  const void* w_codes;      // [O, L/2]
  const uint8_t* w_scales;  // [O, 2*ceilDiv(L,64)]
  float* C;                 // [T, O]
  uint32_t* status;         // bounded-wait status word, or nullptr
  int64_t T, O, L;
};
cudaError_t launch_mxgemm(const MxGemmParams& p, int num_sms, cudaStream_t stream);

// Keeps a CUDA error code for fq_last_cuda_error() (thread-local).
void record_cuda_error(int e);
cudaError_t launch_tc(const TcParams& p, bool fp16_in, int num_sms, cudaStream_t stream);

}  // namespace fq
