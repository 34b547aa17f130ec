/*
 * fq.h - C ABI of the fused rotate + quantize library (libfq.so), sm_100a.
 *
 * The operator is the one defined by the page "aclnnFlatQuantV2 complete guide: from
 * two-level matmul to FP4 E2M1 quantization fusion" (http://www.zwxr.cn/news/277566):
 * for each token k of x[K, M, N]
 *
 *     x'' = P1 . (x[k] . P2)                       ("How it works", two-level matmul)
 *
 * with P1 an [M, M] and P2 an [N, N] matrix, followed by one of two quantizers that
 * never write x'' to memory:
 *
 *   per-token ("per-token mode"): quantScale[k] = max|x''| / (7 / clipRatio) (float32),
 *       out = round_half_even(x'' / quantScale) clamped to [-8, 7], as INT4 (two per
 *       byte) or INT4 packed eight per INT32 word (the same bytes);
 *   per-group ("per-group mode", cases 1-3): x'' viewed as [K, M*N] in groups of 32;
 *       one E8M0 exponent per group in a [K, ceilDiv(M*N, 64), 2] byte tensor, and one
 *       E2M1 code per element, two per byte, out [K, M*N / 2] bytes.
 *
 * Conventions shared by every call:
 *   - All tensors are dense, row-major, contiguous DEVICE buffers owned by the caller
 *     (x [K,M,N], P1 [M,M], P2 [N,N] in the handle's 16-bit type; outputs as stated).
 *     The library never allocates, frees, copies or synchronizes inside the
 *     fq_quantize_* / fq_debug_rotate calls.
 *   - Nibble order is LSB-first: element 2b of the flattened token sits in bits 0-3 of
 *     byte b, element 2b+1 in bits 4-7. INT4 values are two's complement nibbles; E2M1
 *     codes carry the sign in bit 3.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and deterministic: the same inputs give the same bytes.
 *   - Status codes mirror the page's error table ("Error code quick reference"):
 *     FQ_ERR_NULLPTR (161001) for a required NULL pointer, FQ_ERR_INVALID (161002) for a
 *     shape / range / type rule the page lists. A launch failure is FQ_ERR_CUDA; the
 *     CUDA error is kept and returned by fq_last_cuda_error(). Execution faults surface
 *     on the stream as usual.
 *   - Inputs are finite numbers. For a group whose float32 absmax is not finite, the
 *     ratio rule (case 3) gives the byte 0xFF (the rule applied to an infinite S) and the
 *     codes of that group are unspecified; a NaN in x is outside the contract.
 *   - Pointers need the alignment of their element type; 16-byte aligned x, out and
 *     scale pointers (and M*N a multiple of 32) let the tensor-core kernel run, other
 *     cases take the general kernel.
 */
#ifndef FQ_H
#define FQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

#if defined(__GNUC__)
#define FQ_API __attribute__((visibility("default")))
#else
#define FQ_API
#endif

typedef enum {
    FQ_OK = 0,
    FQ_ERR_NULLPTR = 161001,     /* a required pointer is NULL (page: ACLNN_ERR_PARAM_NULLPTR) */
    FQ_ERR_INVALID = 161002,     /* a page rule is violated (page: ACLNN_ERR_PARAM_INVALID) */
    FQ_ERR_CUDA = 161003,        /* a CUDA runtime call or a kernel launch failed */
    FQ_ERR_UNSUPPORTED = 161004, /* well-formed but not supported on this device */
    FQ_ERR_DEVICE_TIMEOUT = 161005 /* a bounded wait inside a kernel gave up (see fq_device_status) */
} fq_status;

typedef enum { FQ_BF16 = 0, FQ_FP16 = 1 } fq_dtype;          /* x, P1, P2 share one type */
typedef enum { FQ_OUT_INT4 = 0, FQ_OUT_INT32 = 1 } fq_int_out;

/* Kernel selection, for tests and benchmarks. AUTO picks the tensor-core kernel where
 * the shape allows it and the general kernel elsewhere. */
typedef enum { FQ_KERNEL_AUTO = 0, FQ_KERNEL_GENERAL = 1, FQ_KERNEL_TCGEN05 = 2 } fq_kernel;

typedef struct fq_handle fq_handle;

/* Plan phase (page: aclnnFlatQuantV2GetWorkspaceSize, "two-phase interface").
 * Validates the shape, queries the CURRENT device (SM count, shared memory) and
 * allocates a 256-byte device status block owned by the handle.
 *   K in [1, 262144]; M, N in [1, 256] (page: parameter table, x).
 * Returns FQ_ERR_NULLPTR if h is NULL, FQ_ERR_INVALID for a shape out of range or an
 * unknown dtype, FQ_ERR_CUDA if the device query or the allocation fails. On success *h
 * owns the plan; release it with fq_destroy. A handle is tied to the device that was
 * current at creation. */
FQ_API fq_status fq_create(fq_handle **h, int64_t K, int64_t M, int64_t N, fq_dtype dtype);

/* Releases the plan and its device status block. NULL is accepted. Not safe while a
 * launch made with the handle may still be reading its status block on the device. */
FQ_API fq_status fq_destroy(fq_handle *h);

/* Per-token mode (page: "per-token mode"; parameter table, out INT4 / INT32).
 *   x          [K, M, N]  16-bit input
 *   P1         [M, M]     left matrix (kroneckerP1)
 *   P2         [N, N]     right matrix (kroneckerP2); must not be NULL in this mode
 *   clipRatio  in (0, 1]
 *   fmt        FQ_OUT_INT4: out is [K, M, N] INT4, K*M*N/2 bytes (N even);
 *              FQ_OUT_INT32: out is [K, M, N/8] int32 (N % 8 == 0), the same bytes
 *   quantScale [K] float32
 * Errors: FQ_ERR_NULLPTR (h, x, P1, P2, out, quantScale), FQ_ERR_INVALID (clipRatio out
 * of range, N odd, N % 8 != 0 for INT32, unknown fmt, misaligned pointer), FQ_ERR_CUDA. */
FQ_API fq_status fq_quantize_per_token(fq_handle *h, const void *x, const void *P1, const void *P2,
                                double clipRatio, fq_int_out fmt, void *out,
                                float *quantScale, struct CUstream_st *stream);

/* Per-group mode (page: "per-group mode", cases 1-3; parameter table, FLOAT4_E2M1).
 *   x          [K, M, N]  16-bit input (N even)
 *   P1         [M, M]
 *   P2         [N, N], or NULL to skip the right multiply (page: kroneckerP2 may be
 *              [0, 0] in per-group mode only)
 *   dstTypeMax 0.0 (case 1), 6.0 or 7.0 (case 2), any other value in [6, 12] (case 3)
 *   out_fp4    [K, M*N] E2M1 codes, two per byte: K*M*N/2 bytes
 *   scale_e8m0 [K, ceilDiv(M*N, 64), 2] E8M0 bytes; group g of token k at byte
 *              k*2*ceilDiv(M*N,64) + g; the spare byte of an odd group count is 0x7F (2^0)
 * Errors: FQ_ERR_NULLPTR (h, x, P1, out_fp4, scale_e8m0), FQ_ERR_INVALID (dstTypeMax
 * outside {0} U [6, 12], N odd, misaligned pointer), FQ_ERR_CUDA. */
FQ_API fq_status fq_quantize_mx(fq_handle *h, const void *x, const void *P1, const void *P2,
                         double dstTypeMax, void *out_fp4, uint8_t *scale_e8m0,
                         struct CUstream_st *stream);

/* Consumer of two per-group outputs: the FP4 x FP4 contraction with E8M0 block scales.
 * The page ("per-token mode"; its summary on FP4 E2M1 compression of weights and
 * activations) says the quantized data and scales are emitted for later dequantization
 * and low-precision compute; this is that compute for activations A and weights W that
 * both come out of fq_quantize_mx (or fq_quantize_mx_static) with the same L = M*N:
 *
 *     C[t, o] = sum_i  A_hat[t, i] * W_hat[o, i],   X_hat[r, i] = e2m1(code) * 2^(byte - 127)
 *
 * with byte the E8M0 scale of group i / 32 of row r. It runs on the tensor cores' block-scaled
 * FP4 MMA (kind::mxf4, one E8M0 scale per 32 elements), which reads the codes and scale bytes
 * as the operator stores them. Products of E2M1 values and powers of two are exact; the sum
 * is accumulated in float32 (order unspecified).
 *   T, O       rows of A and of W, in [1, 262144]
 *   L          elements per row, a multiple of 32 in [32, 65536]
 *   a_fp4      [T, L/2] bytes, 16-byte aligned; a_scale_e8m0 [T, ceilDiv(L, 64), 2] bytes
 *   w_fp4      [O, L/2] bytes, 16-byte aligned; w_scale_e8m0 [O, ceilDiv(L, 64), 2] bytes
 *   C          [T, O] float32, row-major (4-byte aligned; O % 4 == 0 with a 16-byte aligned C
 *              takes the vector stores)
 *   (the scale arrays need no alignment; 16-byte aligned ones whose row stride
 *   2 * ceilDiv(L, 64) is a multiple of 16 bytes are read 16 bytes at a time, others word
 *   by word)
 *   status     a device word, or NULL: a bounded wait that gives up ORs a nonzero code into
 *              it and leaves C undefined (with NULL nothing reports that)
 * Allocates nothing; asynchronous on stream. Errors: FQ_ERR_NULLPTR (a_fp4, a_scale_e8m0,
 * w_fp4, w_scale_e8m0, C), FQ_ERR_INVALID (a size out of range, L % 32 != 0, misaligned
 * pointer), FQ_ERR_CUDA. */
FQ_API fq_status fq_mx_matmul(int64_t T, int64_t O, int64_t L, const void *a_fp4,
                              const uint8_t *a_scale_e8m0, const void *w_fp4,
                              const uint8_t *w_scale_e8m0, float *C, uint32_t *status,
                              struct CUstream_st *stream);

/* Per-group mode (as fq_quantize_mx) for callers that cannot allocate device memory.
 * The paper has no counterpart: this entry point is an addition of this library.
 *
 * fq_create allocates a small device status block with cudaMalloc. Callers whose device
 * memory is owned by another allocator or a fixed budget, callers that must not pay the
 * implicit device synchronization of cudaMalloc / cudaFree on a latency-critical path,
 * and plug-ins that may not create allocations of their own use this call instead. It
 * takes the shape and dtype directly (no handle), allocates nothing and frees nothing:
 * no cudaMalloc, cudaFree or allocating library routine runs in it.
 *
 * Its only scratch is one 32-bit status word (the word the tensor-core kernel sets when
 * one of its bounded waits gives up) inside a 256-byte static device array of the
 * library. That array is loaded with the library's device code and held on every GPU that
 * uses it until the process exits. A call that launches the tensor-core kernel clears the
 * word with cudaMemsetAsync on `stream` before the launch; the array otherwise keeps what
 * the last call left. All calls in the process share the array, so calls that overlap on
 * the GPU race on that word. fq_static_device_status reads the word back: a wait that
 * gave up leaves the outputs of that call undefined, and this reader is the only way to
 * learn of it on this path.
 *
 * Every call looks up the array's device address in the current context
 * (cudaGetSymbolAddress, a host-side query). The first call in a process or context may
 * also load the library's device code, so make it before any stream capture. Arguments,
 * layouts and errors are those of fq_quantize_mx plus the plan-phase checks of fq_create
 * (K in [1, 262144], M, N in [1, 256], dtype): FQ_ERR_NULLPTR, FQ_ERR_INVALID (including
 * a call whose scratch would exceed the static array, which no allowed shape does),
 * FQ_ERR_UNSUPPORTED, FQ_ERR_CUDA. */
FQ_API fq_status fq_quantize_mx_static(int64_t K, int64_t M, int64_t N, fq_dtype dtype,
                                       const void *x, const void *P1, const void *P2,
                                       double dstTypeMax, void *out_fp4, uint8_t *scale_e8m0,
                                       struct CUstream_st *stream);

/* Reads and clears the status word of fq_quantize_mx_static on the current device (the
 * paper has no counterpart). *status = 0 when no launch of that entry point gave up a
 * bounded wait since the word was last cleared, else the code of the wait (and the call
 * returns FQ_ERR_DEVICE_TIMEOUT). Synchronizes with the device (a blocking copy) and
 * allocates nothing. Returns FQ_ERR_NULLPTR for a NULL status, FQ_ERR_CUDA if the copy
 * fails. */
FQ_API fq_status fq_static_device_status(uint32_t *status);

/* Test hook for the failure path of fq_quantize_mx_static (the paper has no counterpart):
 * process-wide and one-shot, like fq_debug_arm_stall for a handle. The next call of
 * fq_quantize_mx_static in this process that takes the tensor-core kernel issues no x loads
 * and gives every bounded wait a limit of wait_limit_s seconds (0 < wait_limit_s <= 10), so
 * its first stage-A wait runs out, the kernel sets the status word and returns; the outputs
 * of that call are undefined. Returns FQ_ERR_INVALID for a limit out of range. */
FQ_API fq_status fq_static_debug_arm_stall(double wait_limit_s);

/* Test hook: writes x'' = P1 . (x . P2) ("How it works", the two-level matmul) as float32
 * [K, M, N] (P2 may be NULL), computed the way the selected kernel computes it before
 * quantization. The page exposes no such output; it lets tests compare the rotation alone.
 * Errors: FQ_ERR_NULLPTR (h, x, P1, x2), FQ_ERR_INVALID (misaligned pointer), FQ_ERR_CUDA. */
FQ_API fq_status fq_debug_rotate(fq_handle *h, const void *x, const void *P1, const void *P2,
                          float *x2, struct CUstream_st *stream);

/* Selects the kernel for later calls on h (default FQ_KERNEL_AUTO). Returns
 * FQ_ERR_UNSUPPORTED if FQ_KERNEL_TCGEN05 is asked for a shape it does not cover. */
FQ_API fq_status fq_set_kernel(fq_handle *h, fq_kernel kernel);

/* Intermediate rounding (the page's "How it works" leaves open whether x' = x . P2 is kept
 * in the input type before P1 . x'; the default keeps it exact). With enable = 1, later
 * calls on h round every x' element to the handle's 16-bit type (nearest, ties to even)
 * after summing its products in float32 in index order, then form x'' = P1 . x' from the
 * rounded values. This is meant for comparison with implementations that store x' so, not
 * for speed: it runs the general kernel (FQ_ERR_UNSUPPORTED if FQ_KERNEL_TCGEN05 is
 * selected). enable = 0 restores the default. Returns FQ_ERR_NULLPTR for a null handle and
 * FQ_ERR_INVALID for enable other than 0 or 1. */
FQ_API fq_status fq_set_intermediate_rounding(fq_handle *h, int enable);

/* The kernel the last successful call on h launched (FQ_KERNEL_GENERAL or
 * FQ_KERNEL_TCGEN05), or FQ_KERNEL_AUTO before any call. */
FQ_API fq_kernel fq_last_kernel(const fq_handle *h);

/* Number of kernel launches the last successful call on h made. */
FQ_API int fq_last_launch_count(const fq_handle *h);

/* Test hook for the failure path (the page has no counterpart). Arms the handle so that
 * its next tensor-core launch issues no x loads and gives every bounded wait a limit of
 * wait_limit_s seconds (0 < wait_limit_s <= 10): the first stage-A wait can then only end
 * by running out, after which the kernel sets the abort flag and a status bit, lets every
 * role leave its loop, frees its TMEM and returns (the outputs of that call are
 * undefined). fq_device_status then reports the expiry, and the next call runs normally.
 * One-shot; calls that take the general kernel ignore it. Returns FQ_ERR_NULLPTR or
 * FQ_ERR_INVALID for a bad argument. */
FQ_API fq_status fq_debug_arm_stall(fq_handle *h, double wait_limit_s);

/* Reads and clears the handle's device status word: 0 when no kernel gave up a bounded
 * wait since the last read, else a nonzero code naming the wait (and the call returns
 * FQ_ERR_DEVICE_TIMEOUT). Synchronizes the device. */
FQ_API fq_status fq_device_status(fq_handle *h, uint32_t *status);

/* The CUDA error code kept by the last call that returned FQ_ERR_CUDA in this thread. */
FQ_API int fq_last_cuda_error(void);

/* Static description of a status code (the codes follow the page's "Error code quick
 * reference"; the page has no such function). Never NULL; unknown codes give
 * "unknown fq_status". */
FQ_API const char *fq_status_string(fq_status s);

#ifdef __cplusplus
}
#endif

#endif /* FQ_H */
