// General fused rotate + quantize kernel: any M, N in [1, 256], float32 FFMA.
//
// Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
// quantization fusion" (http://www.zwxr.cn/news/277566), "How it works" (two-level
// small matmul) and the per-token / per-group quantizers.
//
// One CTA of 256 threads handles one token at a time (grid-stride over tokens). The
// token's x is staged in shared memory once; x'' is produced in column blocks of 32:
//     x'[:, blk] = x . P2[:, blk]        (float32 FMA, P2 block staged in shared memory)
//     x''[:, blk] = P1 . x'[:, blk]      (float32 FMA, P1 read through the L1 cache)
// The quantizer needs a reduction over the token (per-token absmax) or over groups that
// may straddle rows and column blocks, so x'' is produced twice: pass 0 reduces, pass 1
// recomputes the identical values and encodes them. Nothing but the outputs reaches
// global memory. This kernel serves the small shapes (M, N = 16), every shape the
// tensor-core kernel does not cover, and the intermediate-rounding mode (x' rounded to the
// input type between the two products, for comparison with implementations that store it
// so); x' is one float32 FMA chain over j in index order.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "fq_internal.h"
#include "fq_quant.cuh"

namespace fq {

namespace {

constexpr int kThreads = 256;
constexpr int kCol = 32;  // column block width

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// v rounded to the 16-bit input type (nearest, ties to even) and widened back
template <typename T>
__device__ __forceinline__ float round_to(float v);
template <>
__device__ __forceinline__ float round_to<__nv_bfloat16>(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }
template <>
__device__ __forceinline__ float round_to<__half>(float v) { return __half2float(__float2half_rn(v)); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
general_kernel(const GeneralParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int M = p.M, N = p.N;
  const int MN = M * N;
  const int G = (MN + 31) / 32;
  T* xs = reinterpret_cast<T*>(smem);                                   // [M*N]
  size_t off = (size_t(MN) * sizeof(T) + 15) & ~size_t(15);
  float* p2s = reinterpret_cast<float*>(smem + off);                    // [N][32]
  off += size_t(N) * kCol * sizeof(float);
  float* xp = reinterpret_cast<float*>(smem + off);                     // [M][32]
  off += size_t(M) * kCol * sizeof(float);
  uint32_t* gmax = reinterpret_cast<uint32_t*>(smem + off);             // [G]
  off += size_t(G) * sizeof(uint32_t);
  float* gR = reinterpret_cast<float*>(smem + off);                     // [G]
  off += size_t(G) * sizeof(float);
  float* red = reinterpret_cast<float*>(smem + off);                    // [kThreads/32]
  __shared__ float s_inv_scale;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const T* __restrict__ P1 = static_cast<const T*>(p.P1);
  const T* __restrict__ P2 = static_cast<const T*>(p.P2);
  const int passes = (p.mode == kModeRotate) ? 1 : 2;

  for (int64_t k = blockIdx.x; k < p.K; k += gridDim.x) {
    const T* __restrict__ xk = static_cast<const T*>(p.x) + k * MN;
    for (int i = tid; i < MN; i += kThreads) xs[i] = xk[i];
    if (p.mode == kModeMx)
      for (int g = tid; g < G; g += kThreads) gmax[g] = 0u;
    float tmax = 0.0f;
    __syncthreads();

    for (int pass = 0; pass < passes; ++pass) {
      for (int cb = 0; cb < N; cb += kCol) {
        const int nc = min(kCol, N - cb);
        // x'[:, cb:cb+nc] = x . P2[:, cb:cb+nc], or x itself when P2 is absent
        if (P2 != nullptr) {
          for (int i = tid; i < N * kCol; i += kThreads) {
            const int j = i >> 5, c = i & 31;
            p2s[i] = (c < nc) ? to_f32(P2[j * N + cb + c]) : 0.0f;
          }
          __syncthreads();
          for (int o = tid; o < M * kCol; o += kThreads) {
            const int m = o >> 5, c = o & 31;
            float acc = 0.0f;
            const T* xr = xs + m * N;
            for (int j = 0; j < N; ++j) acc = fmaf(to_f32(xr[j]), p2s[j * kCol + c], acc);
            // with intermediate rounding, x' is stored in the input type between the products
            xp[o] = p.round_x1 ? round_to<T>(acc) : acc;
          }
        } else {
          for (int o = tid; o < M * kCol; o += kThreads) {
            const int m = o >> 5, c = o & 31;
            xp[o] = (c < nc) ? to_f32(xs[m * N + cb + c]) : 0.0f;
          }
        }
        __syncthreads();
        // x''[:, cb:cb+nc] = P1 . x'[:, cb:cb+nc]; a warp owns one row m, lane = column
        for (int o = tid; o < M * kCol; o += kThreads) {
          const int m = o >> 5, c = o & 31;
          float acc = 0.0f;
          const T* p1r = P1 + m * M;
          for (int i = 0; i < M; ++i) acc = fmaf(to_f32(__ldg(p1r + i)), xp[i * kCol + c], acc);
          const bool valid = c < nc;
          const int f = m * N + cb + c;  // flat index inside the token
          if (p.mode == kModeRotate) {
            if (valid) p.x2[k * MN + f] = acc;
          } else if (pass == 0) {
            if (valid) {
              if (p.mode == kModePerToken) tmax = fmaxf(tmax, fabsf(acc));
              else atomicMax(&gmax[f >> 5], __float_as_uint(fabsf(acc)));
            }
          } else {
            // encode; lanes (c, c+1) hold flat elements (f, f+1) because cb and N are even
            float v = (p.mode == kModePerToken) ? acc * s_inv_scale : acc * gR[valid ? (f >> 5) : 0];
            const float v_hi = __shfl_down_sync(0xffffffffu, v, 1);
            if (valid && (c & 1) == 0) {
              uint32_t byte;
              if (p.mode == kModePerToken) byte = int4_nibble(v) | (int4_nibble(v_hi) << 4);
              else byte = e2m1_canonical_zero(e2m1x2_raw(v, v_hi));
              p.out[(k * MN + f) >> 1] = uint8_t(byte);
            }
          }
        }
        __syncthreads();
      }

      if (pass == 0 && p.mode == kModePerToken) {
        tmax = warp_max(tmax);
        if (lane == 0) red[tid >> 5] = tmax;
        __syncthreads();
        if (tid == 0) {
          float a = 0.0f;
          for (int w = 0; w < kThreads / 32; ++w) a = fmaxf(a, red[w]);
          const float qs = per_token_scale(a, p.clip_ratio);
          p.quant_scale[k] = qs;
          s_inv_scale = (qs > 0.0f) ? __frcp_rn(qs) : 0.0f;
        }
        __syncthreads();
      } else if (pass == 0 && p.mode == kModeMx) {
        const int gs = 2 * ((MN + 63) / 64);  // scale bytes per token, with the spare slot
        for (int g = tid; g < gs; g += kThreads) {
          uint32_t byte = 0x7Fu;  // the spare slot of an odd group count: 2^0
          if (g < G) {
            const MxScale s = mx_scale(__uint_as_float(gmax[g]), p.rule);
            byte = s.byte;
            gR[g] = s.R;
          }
          p.scales[k * gs + g] = uint8_t(byte);
        }
        __syncthreads();
      }
    }
    __syncthreads();
  }
}

}  // namespace

size_t general_smem_bytes(int M, int N, int elem_bytes) {
  const int MN = M * N;
  const int G = (MN + 31) / 32;
  size_t off = (size_t(MN) * elem_bytes + 15) & ~size_t(15);
  off += size_t(N) * kCol * 4 + size_t(M) * kCol * 4 + size_t(G) * 8 + (kThreads / 32) * 4;
  return off;
}

cudaError_t launch_general(const GeneralParams& p, bool fp16_in, int grid, cudaStream_t stream) {
  const size_t smem = general_smem_bytes(p.M, p.N, 2);
  if (fp16_in) {
    cudaError_t e = cudaFuncSetAttribute(general_kernel<__half>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    general_kernel<__half><<<grid, kThreads, smem, stream>>>(p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(general_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    general_kernel<__nv_bfloat16><<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fq
