// Tensor-core fused rotate + quantize kernel for sm_100a (tcgen05 / TMEM / TMA).
//
// Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
// quantization fusion" (http://www.zwxr.cn/news/277566): x'' = P1 . (x . P2) per token
// ("How it works"), then the per-token or per-group quantizer.
//
// Layout of the work. Tokens are stacked into 128-row tiles of the [K*M, N] row view of
// x (128/M tokens per tile, M in {32, 64, 128}). The product is associative, so each
// tile is computed as
//     stage A:  Y   = BD(P1) . X        bf16 x bf16 -> fp32 (TMEM), K = 128
//     stage B:  X'' = Y . P2            Y split as fp16 hi + fp16 lo, fp32 accumulate
// where BD(P1) is the block-diagonal matrix holding 128/M copies of P1, so one M=128
// MMA serves every token of the tile. The products of stage A are exact; stage B needs
// Y, an fp32 value, as a 16-bit operand: each row of Y is scaled by a power of two that
// puts its largest magnitude in [2^14, 2^15), then split into fp16 hi = rn(y) and
// lo = rn(y - hi), so hi + lo carries 22 significant bits and the two MMAs of stage B
// lose nothing beyond float32 rounding. In TMEM each 16-column block of a row of Y is
// replaced by the 8 words of hi followed by the 8 words of lo of the same 16 elements. P2 is scaled by one power of two into the same
// range, converted to fp16 and transposed to K-major once per CTA. The powers of two
// are undone exactly in the epilogue.
//
// Roles (one CTA per SM, persistent over tiles, 640 threads = 5 warpgroups):
//   warps 0-15  four epilogue warpgroups; group g takes the local tiles i = g (mod 4): it
//               reads Y from TMEM (lane = row), scales each row by a power of two and writes
//               fp16 hi / lo back into the same TMEM columns for stage B; then it reads the
//               row of X'' (twice: block maxima, then the codes, so that a thread never
//               holds a whole row), releases the buffer, forms per-token or per-group scales
//               and codes, stages them in shared memory and stores them with bulk copies
//   warp 16     TMA producer: x tiles (128 rows x N, 128B-swizzled) into a 3- to 5-stage ring
//   warp 17     MMA issuer of stage A (A = BD(P1) in TMEM, or in SMEM when N = 128; B = x
//               tile, MN-major); it also owns the TMEM allocation
//   warp 18     MMA issuer of stage B (A = hi/lo Y in TMEM, B = P2^T in SMEM); at
//   warp 19     N = 96 and 112, warps 18 and 19 take the even and the odd local tiles
//   warp 19     idle after the prologue
// TMEM holds D_A slots (Y, then its hi / lo) and D_B slots (X''), two of each for N >= 96,
// so stage A of the next tile runs while an epilogue group still encodes this one.
// Every wait is bounded in time; on expiry the kernel records a code in the status word,
// drains its copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "fq_internal.h"
#include "fq_quant.cuh"

namespace fq {
namespace {

constexpr int kStagesMax = 5;
constexpr int kThreads = 640;  // five warpgroups
// Register split (setmaxnreg): launched at kLaunchRegs per thread; the four epilogue
// warpgroups rise to kEpiRegs and the producer / MMA warpgroup drops to kLowRegs. The shares add up to no more than the registers the block was
// launched with, so setmaxnreg.inc always finds what it asks for.
constexpr int kEpi = 4;  // epilogue warpgroups (warps 0-15)
constexpr int kLaunchRegs = 96, kEpiRegs = 104, kLowRegs = 56;
constexpr int kWarpProducer = 16, kWarpMmaA = 17, kWarpMmaB = 18, kWarpMmaB2 = 19;
static_assert(128 * (kEpi * kEpiRegs + kLowRegs) <= kThreads * kLaunchRegs, "register split");
constexpr uint64_t kTimeoutNs = 4000000000ull;  // 4 s: far beyond any legitimate wait (default)

// status bits (device status word)
enum : uint32_t {
  kStProducerEmpty = 1u << 0, kStMmaXFull = 1u << 1, kStMmaTmemEmpty = 1u << 2,
  kStMmaYsFull = 1u << 3, kStEpiAFull = 1u << 4, kStEpiBFull = 1u << 5,
  kStMmaDone = 1u << 6, kStDrain = 1u << 7
};

template <int N>
struct Geo {
  static_assert(N % 16 == 0 && N >= 64 && N <= 128, "tensor-core kernel covers N in [64,128], N % 16 == 0");
  static constexpr int kAtoms = (N + 63) / 64;              // 64-element swizzle atoms along N
  static constexpr int kXStage = kAtoms * 128 * 128;        // bytes per x stage
  // x ring depth: five stages at N = 80 .. 112 (two to five measure within noise of one
  // another at 128 x 112: the loads land well ahead), four at N = 64 (eight measured
  // slower: the longer first round of loads delays the first tile), three at N = 128
  // where BD(P1) stays in shared memory
  static constexpr int kStages = N == 128 ? 3 : (N == 64 ? 4 : 5);
  // BD(P1) sits in TMEM (64 columns; stage A is then a TS MMA that reads only the x tile
  // from shared memory, 3.5 KB instead of 7.5 KB per MMA at N = 112) when four N-column
  // slots still fit beside it; otherwise in shared memory, 128 x 128, two K atoms (SS).
  static constexpr bool kP1Tmem = (512 - 64) / N >= 4;
  static constexpr uint32_t kP1Col = 448;                   // its first TMEM column
  static constexpr int kP1Bytes = kP1Tmem ? 0 : 2 * 128 * 128;
  static constexpr int kP2Bytes = kAtoms * N * 128;         // P2^T: N rows, kAtoms K atoms
  static constexpr int kCodeBytes = 128 * N / 2;
  static constexpr int kScaleBytes = 4 * N;                 // 128 rows x N/32 groups
  static constexpr int kOutStride = (kCodeBytes + kScaleBytes + 1023) & ~1023;
  static constexpr int kOffP1 = 0;
  static constexpr int kOffP2 = kOffP1 + kP1Bytes;
  static constexpr int kOffX = kOffP2 + kP2Bytes;
  static constexpr int kOffOut = kOffX + kStages * kXStage;
  static constexpr int kOffBar = kOffOut + kEpi * kOutStride;
  static constexpr int kSmem = kOffBar + 4096 + 1024;       // barriers + alignment slack
  // TMEM: kNA slots of N columns for D_A (Y, then its hi / lo) and kNB slots for D_B (X''),
  // as many as fit in 512 columns, D_B first. Tile i uses D_A slot i % kNA and D_B slot
  // i % kNB. Both are at most kEpi (see the MMA issuers).
  static constexpr int kSlots = (kP1Tmem ? 448 : 512) / N;
  static constexpr int kNB = kSlots / 2 < kEpi ? kSlots / 2 : kEpi;
  static constexpr int kNA = kSlots - kNB < kEpi ? kSlots - kNB : kEpi;
  static_assert(kNA >= 2 && kNB >= 1 && kNA <= kEpi && kNB <= kEpi, "TMEM slots");
  static constexpr int kBlocks = N / 16;          // 16-column blocks of a row
  static constexpr int kGroups = (kBlocks + 1) / 2;  // published two blocks at a time
  static constexpr uint32_t kTmemCols = (!kP1Tmem && (kNA + kNB) * N <= 256) ? 256u : 512u;
  // stage-B issuer warps: two (18 and 19, even and odd local tiles) where issuing a tile's
  // 2N/16 MMAs and its barrier operations keeps one warp busy for the whole tile (N = 96,
  // 112). Both slot counts must then be even, so that every slot's barriers are waited for
  // by one of the two warps only: with an odd count one warp could reach tile b + kNA
  // while the other has not yet been given tile b, and its parity wait would pass two
  // phases early. One warp at N = 64 (no gain measured) and N = 128 (measured slower).
  static constexpr int kBIss = (N == 96 || N == 112) ? 2 : 1;
  static_assert(kBIss == 1 || (kNA % 2 == 0 && kNB % 2 == 0), "two stage-B warps need even slot counts");
};

struct Bars {
  uint64_t x_full[kStagesMax];
  uint64_t x_empty[kStagesMax];
  // Every barrier below is waited for by one thread or one warpgroup, phase after phase.
  uint64_t da_full[kEpi];   // stage A of tile i done (barrier of its epilogue group i % kEpi)
  uint64_t db_full[kEpi];   // stage B of tile i done (same)
  uint64_t ys_full[4][4];   // D_A slot: hi / lo of column group g (two 16-column blocks) written
  uint64_t da_free[4];      // D_A slot: stage B that read it has completed
  uint64_t tm_empty[4];     // D_B slot: X'' read out by the epilogue
  uint64_t mma_done[3];
  uint32_t tmem_base;
  int abort;
  uint64_t timeout_ns;  // limit of every bounded wait of this launch
  int group_exit[kEpi][2];  // per epilogue group: exit decision, one slot per use parity
  float red[kEpi][4];
  float wmax[kThreads / 32];
};
static_assert(sizeof(Bars) <= 4096, "barrier block");
template <int N>
constexpr bool smem_fits() { return Geo<N>::kSmem <= 232448; }  // 227 KB opt-in per block
static_assert(smem_fits<64>() && smem_fits<80>() && smem_fits<96>() && smem_fits<112>() && smem_fits<128>(),
              "shared memory");

// ------------------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
// Waits for a phase to complete, the thread suspended in hardware until it does or a
// limit the hardware chooses passes. (An explicit suspend-time hint of 1 ms or of 2-20 us
// measured 1-4 % slower over the whole kernel: the waiters woke later.)
__device__ __forceinline__ bool mbar_try_wait(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(b), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// Every descriptor here shares its high word: stride byte offset 1024 (8 rows of 128 B),
// version 1, 128-byte swizzle. The low word holds the start address (>> 4) and the
// leading byte offset (>> 4); shared-memory addresses are below 2^18, so no masking.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo) { return (saddr >> 4) | ((lbo >> 4) << 16); }
// Warp-wide forms for the issuing warp: every lane runs the same code (so descriptors stay
// warp-uniform) and one elected lane issues the instruction.
__device__ __forceinline__ void mma_ss_e(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Stage B of one 16-column block: the hi MMA (A at a_hi, accumulate flag acc_first) then
// the lo MMA (A 8 columns further, always accumulating), both with B = b_desc, under one
// election: the issuing warp shares its sub-partition with busy epilogue warps, so every
// instruction it saves brings the next MMA to the tensor pipe sooner.
__device__ __forceinline__ void mma_ts_block_e(uint32_t d, uint32_t a_hi, uint64_t b, uint32_t idesc,
                                               uint32_t acc_first) {
  asm volatile(
      "{\n\t.reg .pred p, q, e;\n\t.reg .b32 r, a1;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 q, %4, %4;\n\t"
      "add.u32 a1, %1, 8;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], %2, %3, q;\n\t}" ::"r"(d),
      "r"(a_hi), "l"(b), "r"(idesc), "r"(acc_first)
      : "memory");
}
// Stage A of one tile as eight K = 16 MMAs under one election: A = BD(P1) in TMEM at a
// (8 columns per K step), B = the x tile at b_desc (2048 bytes per K step, 128 in the
// descriptor's 16-byte units); the first MMA overwrites D.
__device__ __forceinline__ void mma_ts_stage_a_e(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred f, t, e;\n\t.reg .b32 r, a1, a2, a3, a4, a5, a6, a7;\n\t"
      ".reg .b64 b1, b2, b3, b4, b5, b6, b7;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "setp.ne.b32 f, %1, %1;\n\t"
      "setp.eq.b32 t, %1, %1;\n\t"
      "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\tadd.u32 a4, %1, 32;\n\t"
      "add.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\tadd.u32 a7, %1, 56;\n\t"
      "add.s64 b1, %2, 128;\n\tadd.s64 b2, %2, 256;\n\tadd.s64 b3, %2, 384;\n\tadd.s64 b4, %2, 512;\n\t"
      "add.s64 b5, %2, 640;\n\tadd.s64 b6, %2, 768;\n\tadd.s64 b7, %2, 896;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, f;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b4, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b5, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b6, %3, t;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b7, %3, t;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void mma_commit_e(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ uint64_t desc64(uint32_t saddr, uint32_t lbo) {
  return (uint64_t(kDescHi) << 32) | desc_lo(saddr, lbo);
}

// Instruction descriptor, kind::f16, fp32 accumulate, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(bool a_bf16, bool b_bf16, bool b_mn_major, int n) {
  return (1u << 4) | (uint32_t(a_bf16) << 7) | (uint32_t(b_bf16) << 10) |
         (uint32_t(b_mn_major) << 16) | (uint32_t(n >> 3) << 17) | (uint32_t(128 >> 4) << 24);
}

// 2^e as float32 for e in [-149, 127] (clamped).
__device__ __forceinline__ float exp2i(int e) {
  e = e < -149 ? -149 : (e > 127 ? 127 : e);
  return e >= -126 ? __int_as_float((e + 127) << 23) : __int_as_float(1 << (e + 149));
}

// Exponent s with m * 2^s in [2^14, 2^15) for a positive normal m (clamped to the
// normal range of the factor); 0 for zero or non-finite m.
__device__ __forceinline__ int prescale_exp(float m) {
  const uint32_t E = (__float_as_uint(m) >> 23) & 0xFFu;
  if (m == 0.0f || E == 0xFFu) return 0;
  int s = 141 - int(E == 0 ? 1 : E);
  return s < -126 ? -126 : (s > 127 ? 127 : s);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// max(|a|, |b|, |c|) in one instruction
__device__ __forceinline__ float max3abs(float a, float b, float c) {
  float r;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// largest magnitude of n values (n a multiple of 16) as a shallow tree
template <int n>
__device__ __forceinline__ float absmax(const float* v) {
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
#pragma unroll
  for (int e = 0; e < n; e += 2) acc[(e >> 1) & 7] = max3abs(acc[(e >> 1) & 7], v[e], v[e + 1]);
  const float a = max3abs(acc[0], acc[1], acc[2]);
  const float b = max3abs(acc[3], acc[4], acc[5]);
  return max3abs(a, b, fmaxf(acc[6], acc[7]));
}
__device__ __forceinline__ float absmax16(const float* v) {
  const float a = max3abs(v[0], v[1], v[2]), b = max3abs(v[3], v[4], v[5]);
  const float c = max3abs(v[6], v[7], v[8]), d = max3abs(v[9], v[10], v[11]);
  const float e = max3abs(v[12], v[13], v[14]);
  return fmaxf(max3abs(a, b, c), max3abs(d, e, v[15]));
}
// eight E2M1 codes (round to nearest even, saturate) in one word: element 0 in bits 0-3
__device__ __forceinline__ uint32_t e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t r;
  // cvt puts its first source in the upper nibble of each byte
  asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, %8, %7;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
  return r;
}
template <int n>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(n) : "memory");
}

template <int n>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(n));
}
template <int n>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(n));
}
// v - float(h) for both halves, exact (h is v rounded to fp16), with one mixed-precision
// FMA per half: h * (-1) + v, the fp16 operand widened inside the FMA.
__device__ __forceinline__ float2 residual2(__half2 h, float2 v) {
  float2 r;
  const uint32_t hb = *reinterpret_cast<uint32_t*>(&h);
  asm("{\n\t.reg .b16 lo, hi, m1;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "mov.b16 m1, 0xBC00;\n\t"  // -1.0 in fp16
      "fma.rn.f32.f16 %0, lo, m1, %3;\n\t"
      "fma.rn.f32.f16 %1, hi, m1, %4;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "r"(hb), "f"(v.x), "f"(v.y));
  return r;
}
// Bounded wait on an mbarrier phase. On expiry sets the abort flag and a status bit. Each
// unsuccessful try lasts up to kSuspendNs, so the abort flag and the clock are checked
// after every one.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, Bars* bars, uint32_t* status,
                                          uint32_t code) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(b, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&bars->abort)) return false;
    if (globaltimer() - t0 > bars->timeout_ns) {
      *reinterpret_cast<volatile int*>(&bars->abort) = 1;
      atomicOr(status, code);
      return false;
    }
  }
}

// Bounded wait used by whole warps: uniform result across the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars* bars, uint32_t* status,
                                          uint32_t code) {
  const bool ok = wait_bounded(bar, parity, bars, status, code);
  return __all_sync(0xffffffffu, ok);
}

template <bool kF16>
__device__ __forceinline__ float ld16f(const void* base, int i) {
  const uint16_t u = static_cast<const uint16_t*>(base)[i];
  if constexpr (kF16) return __half2float(__ushort_as_half(u));
  else return __bfloat162float(__ushort_as_bfloat16(u));
}

template <bool kF16>
__device__ __forceinline__ void unpack8(const uint4& q, float* f) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (kF16) {
      const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    } else {
      const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------
// kRatio (per-group mode only): the group rule is case 3 (a separate instantiation, so that
// the kernels of cases 1 and 2 carry none of its code)
template <int N, bool kF16, int kMode, bool kRatio>
__global__ void __launch_bounds__(kThreads, 1)
tc_kernel(const __grid_constant__ CUtensorMap tmap, const TcParams p) {
  using G = Geo<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + G::kOffBar);
  const uint32_t sbase = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = p.M;
  const int64_t rows_total = p.K * int64_t(M);
  const int num_tiles = int((rows_total + 127) / 128);

  // ---- prologue: P2 scale, BD(P1) and P2^T operands, barriers, TMEM ----
  // TMEM first, so that BD(P1) can go there right after the first barrier. Every global
  // read of P1 and P2 is then issued at once (one round trip), into one register buffer
  // whatever the thread's part: threads 256 .. 256 + (N/8)^2 - 1 each hold an 8 x 8 block
  // of P2 (whose maximum is taken from the same registers); threads 128 .. 255 a row of
  // BD(P1) for TMEM (warps 4-7: each row's TMEM lane lies in its warp's lane quarter);
  // threads 0 .. 255 store the chunks of BD(P1)'s shared-memory form as they arrive.
  if (warp == kWarpMmaA) tmem_alloc(&bars->tmem_base, G::kTmemCols);
  // The producer thread initializes the barriers and at once issues its first round of x
  // loads: nothing in the prologue writes the x ring, so their latency overlaps all of it
  // (a small launch spends a good part of its time there). The other threads use the
  // barriers only after the first __syncthreads.
  const int n_early = (warp == kWarpProducer && lane == 0 && !p.stall_loads && int(blockIdx.x) < num_tiles)
                          ? min((num_tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1, G::kStages)
                          : 0;
  if (warp == kWarpProducer && lane == 0) {
    for (int s = 0; s < G::kStages; ++s) {
      mbar_init(&bars->x_full[s], 1);
      mbar_init(&bars->x_empty[s], 1);
    }
    for (int a = 0; a < 4; ++a) {
      for (int g = 0; g < 4; ++g) mbar_init(&bars->ys_full[a][g], 4);
      mbar_init(&bars->da_free[a], 1);
      mbar_init(&bars->tm_empty[a], 4);
    }
    for (int g = 0; g < kEpi; ++g) {
      mbar_init(&bars->da_full[g], 1);
      mbar_init(&bars->db_full[g], 1);
    }
    mbar_init(&bars->mma_done[0], 1);
    mbar_init(&bars->mma_done[1], 1);
    mbar_init(&bars->mma_done[2], 1);
    bars->abort = 0;
    bars->timeout_ns = p.timeout_ns != 0 ? p.timeout_ns : kTimeoutNs;
    for (int g = 0; g < kEpi; ++g) bars->group_exit[g][0] = bars->group_exit[g][1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_proxy_async();  // the initialized barriers, before the bulk copies that complete on them
    for (int i = 0; i < n_early; ++i) {
      mbar_arrive_expect_tx(&bars->x_full[i], G::kXStage);
#pragma unroll
      for (int a = 0; a < G::kAtoms; ++a)
        tma_load_2d(sbase + G::kOffX + i * G::kXStage + a * 16384, &tmap, a * 64,
                    (int(blockIdx.x) + i * int(gridDim.x)) * 128, &bars->x_full[i]);
    }
  }
  constexpr int NB = N / 8;
  static_assert(256 + NB * NB <= kThreads, "one P2 block per thread");
  const int pb = tid - 256;
  const bool has_pb = pb >= 0 && pb < NB * NB;
  const bool has_p1row = G::kP1Tmem && tid >= 128 && tid < 256;
  uint4 buf[16];
  if (has_pb && p.P2 != nullptr) {
    const int jb = pb / NB, nb = pb % NB;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj)
      buf[jj] = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.P2) + (jb * 8 + jj) * N + nb * 8);
  } else if (has_p1row) {
    const int r = tid - 128;
#pragma unroll
    for (int kc = 0; kc < 16; ++kc) {
      const int k = kc * 8;
      buf[kc] = r / M == k / M
                    ? *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.P1) + (r % M) * M + (k % M))
                    : make_uint4(0u, 0u, 0u, 0u);
    }
  } else if (!G::kP1Tmem && tid < 256) {
    // BD(P1): 128 x 128, K-major, 128B swizzle; element (r, k) = P1[r % M][k % M] on the
    // diagonal blocks (r / M == k / M), else 0. All eight loads first, then the stores: a
    // store between them would keep the compiler from issuing the next load (it cannot
    // tell the two pointers apart), one round trip each.
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = tid + 256 * q;
      const int r = c >> 4, kc = c & 15, k = kc * 8;
      buf[q] = r / M == k / M
                   ? *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.P1) + (r % M) * M + (k % M))
                   : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int c = tid + 256 * q;
      const int r = c >> 4, kc = c & 15;
      const uint32_t off = G::kOffP1 + (kc >> 3) * 16384 + r * 128 + ((((kc & 7) ^ (r & 7))) << 4);
      *reinterpret_cast<uint4*>(smem + off) = buf[q];
    }
  }
  float lmax = 0.0f;
  if (has_pb && p.P2 != nullptr) {
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      float f[8];
      unpack8<kF16>(buf[jj], f);
#pragma unroll
      for (int nn = 0; nn < 8; ++nn) lmax = fmaxf(lmax, fabsf(f[nn]));
    }
  }
  lmax = warp_max(lmax);
  if (lane == 0) bars->wmax[warp] = lmax;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  if (has_p1row) {
    // BD(P1) into TMEM as the A operand of stage A: lane r holds row r, column c the
    // elements (r, 2c) and (r, 2c + 1) in its low and high halves
    const uint32_t t_row = tmem + (uint32_t((warp & 3) * 32) << 16) + G::kP1Col;
#pragma unroll
    for (int j = 0; j < 4; ++j) tmem_st16(t_row + 16 * j, reinterpret_cast<const uint32_t*>(buf + 4 * j));
    tmem_wait_st();
  }
  float p2max = 0.0f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) p2max = fmaxf(p2max, bars->wmax[w]);
  if (p.P2 == nullptr) p2max = 1.0f;  // P2 skipped: the identity
  const int t_exp = prescale_exp(p2max);
  const float p2scale = exp2i(t_exp);

  // P2^T scaled by 2^t as fp16: N rows (n), K = N (j), K-major, 128B swizzle.
  if (has_pb) {
    const int jb = pb / NB, nb = pb % NB;
    float v[8][8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = jb * 8 + jj;
      if (p.P2 != nullptr) {
        unpack8<kF16>(buf[jj], v[jj]);
      } else {
#pragma unroll
        for (int nn = 0; nn < 8; ++nn) v[jj][nn] = (j == nb * 8 + nn) ? 1.0f : 0.0f;
      }
    }
#pragma unroll
    for (int nn = 0; nn < 8; ++nn) {
      const int n = nb * 8 + nn;
      uint32_t w[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        w[jj] = h2_bits(__floats2half2_rn(v[2 * jj][nn] * p2scale, v[2 * jj + 1][nn] * p2scale));
      const uint32_t off = G::kOffP2 + (jb >> 3) * (N * 128) + n * 128 + ((((jb & 7) ^ (n & 7))) << 4);
      *reinterpret_cast<uint4*>(smem + off) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == kWarpProducer) {
    // ---------------- TMA producer ----------------
    setmaxnreg_dec<kLowRegs>();
    // (test hook) with stall_loads the producer issues nothing, so the first stage-A wait can
    // only end by running out
    if (lane == 0 && !p.stall_loads) {
      int last_i[G::kStages];
#pragma unroll
      for (int s = 0; s < G::kStages; ++s) last_i[s] = s < n_early ? s : -1;
      int i = n_early;  // the first round went out in the prologue
      for (int tile = blockIdx.x + n_early * gridDim.x; tile < num_tiles; tile += gridDim.x, ++i) {
        const int s = i % G::kStages;
        if (!wait_bounded(&bars->x_empty[s], ((i / G::kStages) & 1) ^ 1, bars, p.status, kStProducerEmpty)) break;
        mbar_arrive_expect_tx(&bars->x_full[s], G::kXStage);
#pragma unroll
        for (int a = 0; a < G::kAtoms; ++a)
          tma_load_2d(sbase + G::kOffX + s * G::kXStage + a * 16384, &tmap, a * 64, tile * 128,
                      &bars->x_full[s]);
        last_i[s] = i;
      }
      // drain: every issued load has landed before the CTA may exit
      for (int s = 0; s < G::kStages; ++s) {
        if (last_i[s] < 0) continue;
        const uint32_t b = smem_u32(&bars->x_full[s]);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(b, (last_i[s] / G::kStages) & 1)) {
          if (globaltimer() - t0 > bars->timeout_ns) { atomicOr(p.status, kStDrain); break; }
        }
      }
    }
  } else if (warp == kWarpMmaA || warp == kWarpMmaB || (G::kBIss == 2 && warp == kWarpMmaB2)) {
    // ---------------- MMA issuers ----------------
    // Warp 17 issues stage A of every tile in tile order; stage B is issued by warp 18, or
    // by warps 18 and 19 taking every other tile (kBIss), each in its own tile order; all
    // with blocking waits. The whole warp runs the loop, so descriptors stay warp-uniform,
    // and one elected lane issues; each warp commits only its own MMAs.
    //   stage A of tile a: x tile landed; D_A slot free (stage B of tile a - kNA done).
    //   stage B of tile b: D_B slot free (tile b - kNB read out); then each pair of
    //                      16-column blocks of hi / lo as soon as it is published.
    // Every barrier has one waiter that takes its phases in order, and none is ever two
    // phases behind: stage A of tile i + kEpi waits for stage B of tile i + kEpi - kNA,
    // which waits for the split of tile i + kEpi - kNA, issued after that of tile i; a
    // stage-B warp waits for the split of tile b (phase b / kNA of a D_A slot) and for the
    // read-out of tile b - kNB, and the next phase of either barrier needs stage B of tile
    // b itself. With two stage-B warps both slot counts are even, so the tiles of a slot
    // all belong to one of them.
    setmaxnreg_dec<kLowRegs>();
    const int n_local = (blockIdx.x < num_tiles) ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int mb = warp - kWarpMmaA;
    if (mb == 0) {
      constexpr uint32_t kIdA = idesc_f16(!kF16, !kF16, true, N);
      const uint64_t p1_desc = desc64(sbase + G::kOffP1, 16);
      for (int a = 0; a < n_local; ++a) {
        const int s = a % G::kStages, sa = a % G::kNA;
        if (!warp_wait(&bars->x_full[s], (a / G::kStages) & 1, bars, p.status, kStMmaXFull)) break;
        if (a >= G::kNA && !warp_wait(&bars->da_free[sa], ((a / G::kNA) - 1) & 1, bars, p.status, kStMmaTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(sa * N);
        const uint64_t x_desc = desc64(sbase + G::kOffX + s * G::kXStage, 16384);
        if constexpr (G::kP1Tmem) {
          mma_ts_stage_a_e(d, tmem + G::kP1Col, x_desc, kIdA);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_e(d, p1_desc + uint64_t(((kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                     x_desc + uint64_t((kk * 2048) >> 4), kIdA, kk > 0 ? 1u : 0u);
        }
        mma_commit_e(&bars->x_empty[s]);
        mma_commit_e(&bars->da_full[a % kEpi]);
      }
    } else {
      constexpr uint32_t kIdB = idesc_f16(false, false, false, N);
      const uint64_t p2_desc = desc64(sbase + G::kOffP2, 16);
      bool ok = true;
      for (int b = mb - 1; ok && b < n_local; b += G::kBIss) {
        const int sa = b % G::kNA;
        if (b >= G::kNB &&
            !warp_wait(&bars->tm_empty[b % G::kNB], ((b / G::kNB) - 1) & 1, bars, p.status, kStMmaTmemEmpty))
          break;
        const uint32_t d = tmem + uint32_t((G::kNA + b % G::kNB) * N);
        const uint32_t a0 = tmem + uint32_t(sa * N);
#pragma unroll
        for (int g = 0; g < G::kGroups; ++g) {
          ok = warp_wait(&bars->ys_full[sa][g], (b / G::kNA) & 1, bars, p.status, kStMmaYsFull);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 2 * g; kk < 2 * g + 2 && kk < G::kBlocks; ++kk)
            mma_ts_block_e(d, a0 + uint32_t(kk * 16),
                           p2_desc + uint64_t(((kk >> 2) * (N * 128) + (kk & 3) * 32) >> 4), kIdB,
                           kk != 0 ? 1u : 0u);
        }
        if (!ok) break;
        mma_commit_e(&bars->db_full[b % kEpi]);
        mma_commit_e(&bars->da_free[sa]);
      }
    }
    // every MMA issued by this warp has completed before TMEM is released
    mma_commit_e(&bars->mma_done[mb]);
    if (lane == 0) {
      const uint32_t bd = smem_u32(&bars->mma_done[mb]);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(bd, 0)) {
        if (globaltimer() - t0 > bars->timeout_ns) { atomicOr(p.status, kStMmaDone); break; }
      }
    }
    __syncwarp();
  } else if (warp == kWarpMmaB2) {
    setmaxnreg_dec<kLowRegs>();  // idle warp of the producer / MMA warpgroup (N = 128)
  } else {
    // ---------------- epilogue warpgroups: split, then quantize, the same tile ----------------
    // Group eg takes the local tiles i = eg (mod kEpi). For its tile it first splits Y
    // (D_A) into fp16 hi / lo for stage B, publishing each pair of 16-column blocks as
    // soon as it is in TMEM, then waits for stage B and turns X'' (D_B) into codes and
    // scales. A thread owns one row (TMEM lane) throughout, so its row exponent stays in
    // a register. Both phases read their row from TMEM twice (maxima first, then the
    // values again for the conversion or the codes), so a thread never holds a whole row:
    // that keeps four groups within the registers of 640 threads, and reads from TMEM do
    // not slow the MMAs.
    setmaxnreg_inc<kEpiRegs>();
    const int eg = warp >> 2;              // group: tile residue and staging buffer
    const int q = warp & 3;                // TMEM lane quarter of this warp
    const int row = q * 32 + lane;
    const uint32_t t_lane = tmem + (uint32_t(q * 32) << 16);
    const bool leader = (q == 0) && lane == 0;
    const int bar_id = 1 + eg;
    const int tok_in_tile = row / M;
    const int m_row = row % M;
    uint8_t* s_out = smem + G::kOffOut + eg * G::kOutStride;
    const uint32_t s_out_u32 = sbase + G::kOffOut + eg * G::kOutStride;
    constexpr int NS = N / 16;                 // 16-column segments
    constexpr int kB1 = (NS + 1) / 2, kB2 = NS - kB1;  // the two batches of a row, in blocks

    int jj = 0;  // tiles done by this group
    for (int i = eg, tile = blockIdx.x + eg * gridDim.x; tile < num_tiles;
         i += kEpi, tile += kEpi * gridDim.x, ++jj) {
      const int64_t grow = int64_t(tile) * 128 + row;
      const int64_t rows_left = rows_total - int64_t(tile) * 128;
      const int valid_rows = rows_left < 128 ? int(rows_left) : 128;
      const bool row_valid = grow < rows_total;
      const int sa = i % G::kNA, sb = i % G::kNB;

      // ---- split: Y -> per-row power-of-two scale -> fp16 hi / lo in place ----
      const uint32_t colA = uint32_t(sa * N);
      int s_exp = 0;
      // tile i is phase jj of this group's stage-A barrier; the group waited for the
      // previous phase itself, and the next one (tile i + kEpi) cannot complete before this
      // split is published (see the MMA issuers)
      bool ok = warp_wait(&bars->da_full[eg], jj & 1, bars, p.status, kStEpiAFull);
      if (ok) {
        tc_fence_after();
        // pass 1: the row maximum, in two batches
        float m;
        {
          float y[kB1 * 16];
#pragma unroll
          for (int c = 0; c < kB1; ++c) tmem_ld16(t_lane + colA + c * 16, y + c * 16);
          tmem_wait_ld();
          m = absmax<kB1 * 16>(y);
        }
        {
          float y[kB2 * 16];
#pragma unroll
          for (int c = 0; c < kB2; ++c) tmem_ld16(t_lane + colA + (kB1 + c) * 16, y + c * 16);
          tmem_wait_ld();
          m = fmaxf(m, absmax<kB2 * 16>(y));
        }
        s_exp = prescale_exp(m);
        const float sc = exp2i(s_exp);
        const float2 sc2 = make_float2(sc, sc);
        // pass 2: each pair of 16-column blocks comes out of TMEM again (the next pair is
        // loaded while this one is converted), becomes 8 words of hi then 8 words of lo per
        // block, and is published on its own barrier as soon as its stores have landed
        float ya[32], yb[32];
        auto load_pair = [&](int g, float* y) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
            if (2 * g + c < NS) tmem_ld16(t_lane + colA + (2 * g + c) * 16, y + c * 16);
        };
        load_pair(0, ya);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < G::kGroups; ++g) {
          float* cur = (g & 1) ? yb : ya;
          float* nxt = (g & 1) ? ya : yb;
          if (g + 1 < G::kGroups) load_pair(g + 1, nxt);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if (2 * g + c < NS) {
              uint32_t hl[16];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float2 v = __fmul2_rn(make_float2(cur[c * 16 + 2 * e], cur[c * 16 + 2 * e + 1]), sc2);
                const __half2 hv = __float22half2_rn(v);
                hl[e] = h2_bits(hv);
                hl[8 + e] = h2_bits(__float22half2_rn(residual2(hv, v)));
              }
              tmem_st16(t_lane + colA + (2 * g + c) * 16, hl);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->ys_full[sa][g]);
          if (g + 1 < G::kGroups) tmem_wait_ld();
        }
      } else {
        // a failed wait still publishes every group, so the MMA issuer is not left waiting
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
          for (int g = 0; g < G::kGroups; ++g) mbar_arrive(&bars->ys_full[sa][g]);
      }

      // keeps the compiler from moving work of one phase into the other
      asm volatile("" ::: "memory");
      // ---- quantize: X'' = D * 2^crow -> codes and scales ----
      // phase jj of this group's stage-B barrier; stage B of tile i + kEpi cannot complete
      // before this group has read D_B out (see the MMA issuers)
      const uint32_t colB = uint32_t((G::kNA + sb) * N);
      ok = ok && warp_wait(&bars->db_full[eg], jj & 1, bars, p.status, kStEpiBFull);
      const int crow = -(s_exp + t_exp);
      const float fcrow = exp2i(crow);
      // codes (or x'' in rotate mode) of blocks [c0, c0 + nbk), read again from TMEM
      auto block_pass = [&](auto nbk_c, int c0, const float* Fseg) {
        constexpr int nbk = decltype(nbk_c)::value;
        float d[nbk * 16];
        if (ok) {
#pragma unroll
          for (int c = 0; c < nbk; ++c) tmem_ld16(t_lane + colB + (c0 + c) * 16, d + c * 16);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < nbk * 16; ++e) d[e] = 0.0f;
        }
        if constexpr (kMode == kModeRotate) {
          if (row_valid) {
            float4* dst = reinterpret_cast<float4*>(p.x2 + grow * N + c0 * 16);
#pragma unroll
            for (int e = 0; e < nbk * 16; e += 4)
              dst[e / 4] = make_float4(d[e] * fcrow, d[e + 1] * fcrow, d[e + 2] * fcrow, d[e + 3] * fcrow);
          }
        } else {
#pragma unroll
          for (int c = 0; c < nbk; ++c) {
            const int sg = c0 + c;
            const float2 F2 = make_float2(Fseg[sg], Fseg[sg]);
            uint32_t words[2];
#pragma unroll
            for (int wd = 0; wd < 2; ++wd) {
              const float* w = d + c * 16 + wd * 8;
              if constexpr (kMode == kModePerToken) {
                // integer nearest (ties to even), then clamped to [-8, 7] and packed by the
                // saturating pack: it puts its second operand in the low nibble, its first
                // above it, and the carried word above both, so the highest pair goes first
                uint32_t acc = 0u;
#pragma unroll
                for (int e = 6; e >= 0; e -= 2) {
                  const float2 t = __fmul2_rn(make_float2(w[e], w[e + 1]), F2);
                  const int lo = __float2int_rn(t.x), hi = __float2int_rn(t.y);
                  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(acc) : "r"(hi), "r"(lo), "r"(acc));
                }
                words[wd] = acc;
              } else {
                const float2 a = __fmul2_rn(make_float2(w[0], w[1]), F2);
                const float2 b = __fmul2_rn(make_float2(w[2], w[3]), F2);
                const float2 cc = __fmul2_rn(make_float2(w[4], w[5]), F2);
                const float2 dd = __fmul2_rn(make_float2(w[6], w[7]), F2);
                words[wd] = e2m1_canonical_zero(e2m1x8(a, b, cc, dd));
              }
            }
            *reinterpret_cast<uint2*>(s_out + row * (N / 2) + sg * 8) = make_uint2(words[0], words[1]);
          }
        }
      };
      if (ok) tc_fence_after();

      if constexpr (kMode == kModeRotate) {
        block_pass(std::integral_constant<int, kB1>(), 0, nullptr);
        block_pass(std::integral_constant<int, kB2>(), kB1, nullptr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->tm_empty[sb]);
        if (leader) bars->group_exit[eg][jj & 1] = *reinterpret_cast<volatile int*>(&bars->abort) | int(!ok);
        named_bar(bar_id, 128);
        if (bars->group_exit[eg][jj & 1]) break;
        continue;
      } else {
        // pass 1: the maximum of each 16-column block, in two batches
        float smax[NS];
#pragma unroll
        for (int sg = 0; sg < NS; ++sg) smax[sg] = 0.0f;
        if (ok) {
          {
            float d[kB1 * 16];
#pragma unroll
            for (int c = 0; c < kB1; ++c) tmem_ld16(t_lane + colB + c * 16, d + c * 16);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < kB1; ++c) smax[c] = absmax16(d + c * 16);
          }
          {
            float d[kB2 * 16];
#pragma unroll
            for (int c = 0; c < kB2; ++c) tmem_ld16(t_lane + colB + (kB1 + c) * 16, d + c * 16);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < kB2; ++c) smax[kB1 + c] = absmax16(d + c * 16);
          }
        }
        if (leader) bulk_wait_read<0>();  // this group's previous store has left the staging buffer
        float Fseg[NS];
        if constexpr (kMode == kModePerToken) {
          float rmax = 0.0f;
#pragma unroll
          for (int sg = 0; sg < NS; ++sg) rmax = fmaxf(rmax, smax[sg]);
          const float wm = warp_max(rmax * fcrow);
          if (lane == 0) bars->red[eg][q] = wm;
          named_bar(bar_id, 128);
          float amax = 0.0f;
          const int q0 = (tok_in_tile * M) >> 5, nq = (M + 31) >> 5;
          for (int qq = 0; qq < nq; ++qq) amax = fmaxf(amax, bars->red[eg][q0 + qq]);
          const float qs = per_token_scale(amax, p.clip_ratio);
          const float inv = qs > 0.0f ? __frcp_rn(qs) : 0.0f;
          if (row_valid && m_row == 0) p.quant_scale[grow / M] = qs;
#pragma unroll
          for (int sg = 0; sg < NS; ++sg) Fseg[sg] = inv * fcrow;
        } else {
          named_bar(bar_id, 128);
          // bytes by each rule's common path; a ratio-rule group next to a power of two is
          // decided again exactly, by the whole warp when any lane has one (rare)
          constexpr int GR = (N % 32) == 0 ? NS / 2 : (N - 16) / 32 + 1;  // groups met by a row
          float gam[GR];
          uint32_t gb[GR];
          const bool odd = (row & 1) != 0;
          if constexpr ((N % 32) == 0) {
#pragma unroll
            for (int gi = 0; gi < GR; ++gi) gam[gi] = fmaxf(smax[2 * gi], smax[2 * gi + 1]) * fcrow;
          } else {
            // groups of 32 straddle rows: the last 16 columns of an even row and the first
            // 16 of the next row form one group (the pair sits in adjacent lanes); it is
            // group GR - 1 here
            constexpr int GF = GR - 1;  // full groups per row
            const float part = (odd ? smax[0] : smax[NS - 1]) * fcrow;
            const float other = __shfl_xor_sync(0xffffffffu, part, 1);
#pragma unroll
            for (int gi = 0; gi < GF; ++gi)
              gam[gi] = (odd ? fmaxf(smax[2 * gi + 1], smax[2 * gi + 2]) : fmaxf(smax[2 * gi], smax[2 * gi + 1])) * fcrow;
            gam[GF] = fmaxf(part, other);
          }
          bool any_rare = false;
#pragma unroll
          for (int gi = 0; gi < GR; ++gi) {
            bool r;
            gb[gi] = mx_byte_common<kRatio ? kMxRatio : 0>(gam[gi], p.rule, &r);
            any_rare |= r;
          }
          if constexpr (kRatio) {
            if (__any_sync(0xffffffffu, any_rare)) {
#pragma unroll
              for (int gi = 0; gi < GR; ++gi) {
                bool r;
                mx_byte_common<kMxRatio>(gam[gi], p.rule, &r);
                if (r) gb[gi] = mx_byte_rare(gam[gi], p.rule);
              }
            }
          }
          uint8_t* s_scale = s_out + G::kCodeBytes;
          if constexpr ((N % 32) == 0) {
#pragma unroll
            for (int gi = 0; gi < GR; ++gi) {
              const float F = exp2i(127 - int(gb[gi]) + crow);
              Fseg[2 * gi] = F;
              Fseg[2 * gi + 1] = F;
              s_scale[row * (N / 32) + gi] = uint8_t(gb[gi]);
            }
          } else {
            constexpr int GF = GR - 1;
            const float Fst = exp2i(127 - int(gb[GF]) + crow);
            const int pair_base = (row >> 1) * (N / 16);
            float Ff[GF];
#pragma unroll
            for (int gi = 0; gi < GF; ++gi) {
              Ff[gi] = exp2i(127 - int(gb[gi]) + crow);
              s_scale[pair_base + (odd ? GF + 1 : 0) + gi] = uint8_t(gb[gi]);
            }
            if (!odd) s_scale[pair_base + GF] = uint8_t(gb[GF]);
#pragma unroll
            for (int sg = 0; sg < NS; ++sg) {
              const float fe = (sg == NS - 1) ? Fst : Ff[sg >> 1];
              const float fo = (sg == 0) ? Fst : Ff[(sg - 1) >> 1];
              Fseg[sg] = odd ? fo : fe;
            }
          }
        }
        // pass 2: the codes, in the same two batches
        block_pass(std::integral_constant<int, kB1>(), 0, Fseg);
        block_pass(std::integral_constant<int, kB2>(), kB1, Fseg);
        // D_B is free for stage B of tile i + NB
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->tm_empty[sb]);
        fence_proxy_async();
        if (leader) bars->group_exit[eg][jj & 1] = *reinterpret_cast<volatile int*>(&bars->abort) | int(!ok);
        named_bar(bar_id, 128);
        if (leader) {
          const int64_t row0 = int64_t(tile) * 128;
          bulk_store(p.out + row0 * (N / 2), s_out_u32, uint32_t(valid_rows * (N / 2)));
          if constexpr (kMode == kModeMx)
            bulk_store(p.scales + (row0 * N) / 32, s_out_u32 + G::kCodeBytes, uint32_t((valid_rows * N) / 32));
          bulk_commit();
        }
        if (bars->group_exit[eg][jj & 1]) break;
      }
    }
    if (leader) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMmaA) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

template <int N, bool kF16, int kMode, bool kRatio = false>
cudaError_t launch_n(const TcParams& p, int num_sms, cudaStream_t stream) {
  using G = Geo<N>;
  auto enc = get_encode();
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap map;
  const cuuint64_t dims[2] = {cuuint64_t(N), cuuint64_t(p.K * p.M)};
  const cuuint64_t strides[1] = {cuuint64_t(N) * 2};
  const cuuint32_t box[2] = {64u, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = enc(&map, kF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                         const_cast<void*>(p.x), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = tc_kernel<N, kF16, kMode, kRatio>;
  // The register split is sized for kLaunchRegs per thread; a kernel built with fewer
  // would make setmaxnreg.inc wait for registers that do not exist, so refuse it.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kSmem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (p.K * p.M + 127) / 128;
  const int grid = int(tiles < num_sms ? tiles : num_sms);
  kern<<<grid, kThreads, G::kSmem, stream>>>(map, p);
  return cudaGetLastError();
}

template <int N>
cudaError_t launch_mode(const TcParams& p, bool f16, int sms, cudaStream_t s) {
  if (p.mode == kModePerToken)
    return f16 ? launch_n<N, true, kModePerToken>(p, sms, s) : launch_n<N, false, kModePerToken>(p, sms, s);
  if (p.mode == kModeMx)
  {
    if (p.rule.mode == kMxRatio)
      return f16 ? launch_n<N, true, kModeMx, true>(p, sms, s) : launch_n<N, false, kModeMx, true>(p, sms, s);
    return f16 ? launch_n<N, true, kModeMx, false>(p, sms, s) : launch_n<N, false, kModeMx, false>(p, sms, s);
  }
  return f16 ? launch_n<N, true, kModeRotate>(p, sms, s) : launch_n<N, false, kModeRotate>(p, sms, s);
}

}  // namespace

bool tc_supported(int64_t K, int M, int N) {
  (void)K;
  return (M == 32 || M == 64 || M == 128) && (N % 16 == 0) && N >= 64 && N <= 128;
}

cudaError_t launch_tc(const TcParams& p, bool fp16_in, int num_sms, cudaStream_t stream) {
  switch (p.N) {
    case 64: return launch_mode<64>(p, fp16_in, num_sms, stream);
    case 80: return launch_mode<80>(p, fp16_in, num_sms, stream);
    case 96: return launch_mode<96>(p, fp16_in, num_sms, stream);
    case 112: return launch_mode<112>(p, fp16_in, num_sms, stream);
    case 128: return launch_mode<128>(p, fp16_in, num_sms, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace fq
