// Consumer of the per-group outputs: FP4 x FP4 contraction with block scales, sm_100a.
//
// Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
// quantization fusion" (http://www.zwxr.cn/news/277566). "per-token mode" says the
// quantized data and its scales are emitted for later dequantization and low-precision
// compute, and the page's summary presents the operator as the FP4 E2M1 compression of
// weights and activations. This kernel is that later compute for two per-group outputs
// of the operator, activations A [T, L] and weights W [O, L] (L = M*N, the flattened
// token), each as packed E2M1 codes (two per byte, element 2b in bits 0-3 of byte b) and
// E8M0 bytes in the operator's [rows, ceilDiv(L, 64), 2] layout (group g of a row at
// byte g):
//     C[t, o] = sum_i  e2m1(A[t, i]) 2^(sa[t, i/32] - 127)  e2m1(W[o, i]) 2^(sw[o, i/32] - 127)
// in float32. Each 32-element group of both operands carries its own power of two, which
// is exactly what the tensor cores' block-scaled FP4 MMA (kind::mxf4, one E8M0 scale per
// 32 elements) computes, so the codes and scale bytes are consumed as they are stored.
//
// Layout of the work: persistent CTAs (one per SM), 128 x 256 output tiles (A rows on the
// TMEM lanes, W rows along the MMA's N), K in stages of 256 elements (128 code bytes per
// row, one 128-byte swizzle atom). Roles, 384 threads:
//   warp 0       TMA producer: code tiles of A (128 rows) and W (256 rows) into a 4-stage ring
//   warp 1       MMA issuer (owns the TMEM allocation): per stage, six tcgen05.cp of the
//                stage's scale words from shared memory into its scale columns of TMEM,
//                then four K = 64 MMAs (the copies and MMAs of one thread run in issue
//                order) and one commit, which frees the stage's codes and scale slot; one
//                wait per stage, on a barrier that takes the TMA bytes and the four scale
//                warps' arrivals
//   warps 4-7    scale producer: reads the tile rows' E8M0 words (32 bytes of a row, four
//                stages, per load, two loads ahead) and stores each stage's words into the
//                stage's scale slot in shared memory in the order tcgen05.cp reads them
//   warps 8-11   epilogue: reads the float32 accumulator out of TMEM and stores C
// Scale layout in TMEM (what the MMA reads): for a pair of K = 64 steps (four groups of
// 32), row r of an operand with R rows has its four scale bytes in one 32-bit word at
// lane r % 32 of every 32-lane sub-partition, column (pair base) + r / 32; the first MMA of
// the pair reads bytes 0-1, the second bytes 2-3 (selected by the scale-factor id). The
// operator's scale bytes of groups 4c .. 4c + 3 of a row are one 32-bit word, so the words
// move unchanged; only their places change. A tcgen05.cp of shape 32x128b with .warpx4
// writes 32 shared-memory rows of 16 bytes to lanes 0-31 of all four sub-partitions, four
// columns wide, so one 512-byte block whose row l holds, at bytes 4j .. 4j + 3, the word of
// operand row 32j + l fills four columns of that layout: two blocks per stage for A (one
// per K pair), four for W (two per K pair).
// Every wait is bounded in time; on expiry the kernel sets a bit in the caller's status
// word (if one is given), lets every role leave, waits for its copies and MMAs, frees
// TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "fq_internal.h"

namespace fq {
namespace {

constexpr int kBM = 128;            // A rows per tile (TMEM lanes)
constexpr int kBN = 256;            // W rows per tile (MMA N)
constexpr int kBKBytes = 128;       // code bytes per row per stage (256 elements)
constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr int kWarpProducer = 0, kWarpMma = 1, kWarpSf0 = 4, kWarpEpi0 = 8;
constexpr int kABytes = kBM * kBKBytes;   // 16 KB
constexpr int kBBytes = kBN * kBKBytes;   // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColD = 0;             // accumulator: 256 columns
constexpr uint32_t kColSf = 256;          // scale columns: kSfCols per stage
constexpr int kSfaCols = 2 * (kBM / 32);  // two K pairs per stage, one column per 32 rows
constexpr int kSfbCols = 2 * (kBN / 32);
constexpr int kSfCols = kSfaCols + kSfbCols;  // 24
static_assert(kColSf + kStages * kSfCols <= kTmemCols, "TMEM columns");
// Scale slot of a stage in shared memory: 512-byte blocks of 32 rows x 16 bytes, in the
// order tcgen05.cp reads them: A groups 0-3, A groups 4-7, W rows 0-127 groups 0-3, W rows
// 128-255 groups 0-3, W rows 0-127 groups 4-7, W rows 128-255 groups 4-7.
constexpr int kSfBlockBytes = 512;
constexpr int kSfSlotBytes = 6 * kSfBlockBytes;
static_assert(kSfSlotBytes == (kBM + kBN) * 8, "8 scale bytes per row and stage");
// One scale slot per code stage: the stage's commit releases both, so the MMA thread issues
// one commit and waits once per stage (a separate, deeper scale ring with its own commit and
// barrier measured 5-10 % slower: the barrier round trips in the MMA thread's loop pace the
// pipe, not its instruction count).
constexpr int kSfStages = kStages;
constexpr int kSfUnit = 4;  // stages of scale words per row read at once (32 bytes, one sector)
constexpr int kOffSf = kStages * kStageBytes;
constexpr int kSmem = kOffSf + kSfStages * kSfSlotBytes + 1024 /*barriers*/ + 1024 /*alignment*/;
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
constexpr uint64_t kTimeoutNs = 4000000000ull;

enum : uint32_t {
  kStFull = 1u << 0, kStEmpty = 1u << 1, kStDFull = 1u << 3,
  kStDEmpty = 1u << 4, kStDrain = 1u << 5
};

struct Bars {
  uint64_t full[kStages];     // TMA bytes of stage s landed and its scale slot filled
  uint64_t empty[kStages];    // the MMAs (and scale copies) that read stage s completed
  uint64_t d_full;            // accumulator of the tile complete
  uint64_t d_empty;           // accumulator read out (one arrive per epilogue warp)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

struct GemmParams {
  const uint8_t* a_scales;
  const uint8_t* w_scales;
  float* C;
  uint32_t* status;
  int64_t T, O, L;
  int64_t sf_stride;   // scale bytes per row: 2 * ceilDiv(L, 64)
  int tiles_n, num_tiles, nk;
  int sf_vec;          // scale rows 16-byte aligned: read 16 bytes (two stages) at a time
};

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
__device__ __forceinline__ bool mbar_try_wait(uint32_t b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(b), "r"(parity), "n"(1000000)
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
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Bounded wait on a phase; on expiry sets the abort flag and a status bit.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, Bars* bars,
                                             uint32_t* status, uint32_t code) {
  const uint32_t b = smem_u32(bar);
  if (mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(b, parity)) return true;
    if (*reinterpret_cast<volatile int*>(&bars->abort)) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      *reinterpret_cast<volatile int*>(&bars->abort) = 1;
      if (status != nullptr) atomicOr(status, code);
      return false;
    }
  }
}
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars* bars, uint32_t* status,
                                          uint32_t code) {
  return __all_sync(0xffffffffu, wait_bounded(bar, parity, bars, status, code));
}

// Shared-memory descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  const uint32_t lo = (saddr >> 4) | (1u << 16);
  const uint32_t hi = (1024u >> 4) | (1u << 14) | (2u << 29);
  return (uint64_t(hi) << 32) | lo;
}

// Shared-memory descriptor without swizzle: 8-row groups of 16-byte rows, 128 bytes apart
// (rows contiguous), the source form of tcgen05.cp. The rows are one core matrix wide, so
// only the 8-row-group stride is used; both offset fields carry it.
__device__ __forceinline__ uint64_t plain_desc(uint32_t saddr) {
  const uint32_t lo = (saddr >> 4) | ((128u >> 4) << 16);
  const uint32_t hi = (128u >> 4) | (1u << 14);
  return (uint64_t(hi) << 32) | lo;
}

// Instruction descriptor of kind::mxf4 with E8M0 scales, M = 128, N = kBN, both operands
// K-major E2M1; the scale-factor ids (byte offset of the K pair's half) are set per MMA.
__host__ __device__ constexpr uint32_t idesc_mxf4(uint32_t sf_id) {
  return (sf_id << 4) |            // B scale-factor id
         (1u << 7) | (1u << 10) |  // A and B format: E2M1
         (uint32_t(kBN >> 3) << 17) |
         (1u << 23) |              // scale format: E8M0
         (uint32_t(kBM >> 4) << 24) |
         (sf_id << 29);            // A scale-factor id
}

// The three below are issued by one thread (the MMA warp's leader), so that the copies, the
// MMAs and the commit that tracks them all belong to the same thread.
__device__ __forceinline__ void mma_mxf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
      : "memory");
}
// 32 rows x 16 bytes of shared memory to lanes 0-31 of every sub-partition, four columns.
__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t src) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src) : "memory");
}
__device__ __forceinline__ void mma_commit_one(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred e;\n\t.reg .b32 r;\n\t"
      "elect.sync r|e, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, e;\n\t}"
      : "=r"(e));
  return e != 0;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Scale word of groups g0 .. g0 + 3 of one row (g0 a multiple of 4); bytes beyond the row
// (a partial last word, or a row past the end) read as 0.
__device__ __forceinline__ uint32_t load_sf_word(const uint8_t* sc, int64_t rows, int64_t row,
                                                 int64_t stride, int64_t g0) {
  if (row >= rows || g0 >= stride) return 0u;
  const uint8_t* p = sc + row * stride + g0;
  if (g0 + 4 <= stride && (reinterpret_cast<uintptr_t>(p) & 3u) == 0)
    return __ldg(reinterpret_cast<const uint32_t*>(p));
  uint32_t w = 0;
  for (int b = 0; b < 4 && g0 + b < stride; ++b) w |= uint32_t(__ldg(p + b)) << (8 * b);
  return w;
}

__global__ void __launch_bounds__(kThreads, 1)
mxgemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_w,
              const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffSf + kSfStages * kSfSlotBytes);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1 + 4);  // the producer's bytes and one arrive per scale warp
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->d_full, 1);
    mbar_init(&bars->d_empty, 4);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_local = (int(blockIdx.x) < p.num_tiles) ? (p.num_tiles - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

  if (warp == kWarpProducer) {
    if (lane == 0) {
      int it = 0;
      int last_it[kStages];
      for (int s = 0; s < kStages; ++s) last_it[s] = -1;
      bool ok = true;
      for (int i = 0; ok && i < n_local; ++i) {
        const int tile = int(blockIdx.x) + i * int(gridDim.x);
        const int m0 = (tile / p.tiles_n) * kBM, n0 = (tile % p.tiles_n) * kBN;
        for (int kb = 0; kb < p.nk; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !wait_bounded(&bars->empty[s], ((it / kStages) - 1) & 1, bars, p.status, kStEmpty)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
          const uint32_t dst = sbase + s * kStageBytes;
          tma_load_2d(dst, &map_a, kb * kBKBytes, m0, &bars->full[s]);
          tma_load_2d(dst + kABytes, &map_w, kb * kBKBytes, n0, &bars->full[s]);
          last_it[s] = it;
        }
      }
      // every issued load has landed before the CTA may exit
      for (int s = 0; s < kStages; ++s) {
        if (last_it[s] < 0) continue;
        const uint32_t b = smem_u32(&bars->full[s]);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(b, (last_it[s] / kStages) & 1)) {
          if (globaltimer() - t0 > kTimeoutNs) {
            if (p.status != nullptr) atomicOr(p.status, kStDrain);
            break;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    const bool leader = elect_one();
    int it = 0;
    bool ok = true;
    for (int i = 0; ok && i < n_local; ++i) {
      if (i > 0 && !warp_wait(&bars->d_empty, (i - 1) & 1, bars, p.status, kStDEmpty)) break;
      tc_fence_after();
      for (int kb = 0; kb < p.nk; ++kb, ++it) {
        const int s = it % kStages;
        const int j = it % kSfStages;
        if (!warp_wait(&bars->full[s], (it / kStages) & 1, bars, p.status, kStFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (leader) {
          const uint32_t a_addr = sbase + s * kStageBytes;
          const uint64_t a_desc = sw128_desc(a_addr);
          const uint64_t b_desc = sw128_desc(a_addr + kABytes);
          const uint32_t sfa_col = tmem + kColSf + uint32_t(s * kSfCols);
          const uint32_t sfb_col = sfa_col + kSfaCols;
          const uint32_t slot = sbase + kOffSf + uint32_t(j * kSfSlotBytes);
#pragma unroll
          for (int pr = 0; pr < 2; ++pr) {  // K pair pr: groups 4pr .. 4pr + 3
            sf_copy(sfa_col + uint32_t(pr * (kBM / 32)), plain_desc(slot + uint32_t(pr * kSfBlockBytes)));
#pragma unroll
            for (int hb = 0; hb < 2; ++hb)
              sf_copy(sfb_col + uint32_t(pr * (kBN / 32) + 4 * hb),
                      plain_desc(slot + uint32_t((2 + 2 * pr + hb) * kSfBlockBytes)));
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t id = uint32_t(2 * (k & 1));  // byte offset of this K step in its pair's words
            const uint32_t sfa = (sfa_col + uint32_t((k >> 1) * (kBM / 32))) | (id << 30);
            const uint32_t sfb = (sfb_col + uint32_t((k >> 1) * (kBN / 32))) | (id << 30);
            // 64 elements = 32 bytes further along K inside the swizzle atom
            mma_mxf4(tmem + kColD, a_desc + uint64_t((k * 32) >> 4), b_desc + uint64_t((k * 32) >> 4),
                     idesc_mxf4(id), sfa, sfb, (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit_one(&bars->empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (leader) mma_commit_one(&bars->d_full);
      __syncwarp();
    }
    // every MMA issued here has completed before TMEM is released
    if (leader) mma_commit_one(&bars->mma_done);
    __syncwarp();
    if (lane == 0) {
      const uint32_t bd = smem_u32(&bars->mma_done);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(bd, 0)) {
        if (globaltimer() - t0 > kTimeoutNs) {
          if (p.status != nullptr) atomicOr(p.status, kStDrain);
          break;
        }
      }
    }
    __syncwarp();
  } else if (warp >= kWarpSf0 && warp < kWarpSf0 + 4) {
    // thread st carries row 32c + l of the A tile and rows 32c + l, 128 + 32c + l of the W
    // tile (c = st % 4, l = st / 4), each going to row l, bytes 4c .. 4c + 3, of its block:
    // a warp's stores cover 128 contiguous bytes
    const int st = threadIdx.x - kWarpSf0 * 32;
    const int rr = 32 * (st & 3) + (st >> 2);
    const uint32_t off = uint32_t(16 * (st >> 2) + 4 * (st & 3));
    const uint8_t* bases[3] = {p.a_scales, p.w_scales, p.w_scales};
    const int64_t lim[3] = {p.T, p.O, p.O};
    auto tile_row = [&](int i, int r) {
      const int tile = int(blockIdx.x) + i * int(gridDim.x);
      return r == 0 ? int64_t(tile / p.tiles_n) * kBM + rr : int64_t(tile % p.tiles_n) * kBN + 128 * (r - 1) + rr;
    };
    bool ok = true;
    // one stage's words (groups 0-3 and 4-7 of the stage for the three rows) into scale slot
    // j; every writer fences its stores for the async proxy, then one lane per warp arrives
    auto put = [&](int it, const uint32_t (&w)[3][2]) {
      const int j = it % kSfStages;
      if (it >= kSfStages &&
          !warp_wait(&bars->empty[j], ((it / kSfStages) - 1) & 1, bars, p.status, kStEmpty)) {
        ok = false;
        return;
      }
      const uint32_t slot = sbase + kOffSf + uint32_t(j * kSfSlotBytes);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int r = 0; r < 3; ++r) {
          const int blk = r == 0 ? h : 2 + 2 * h + (r - 1);
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(slot + uint32_t(blk * kSfBlockBytes) + off), "r"(w[r][h])
                       : "memory");
        }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->full[j]);
    };
    if (p.sf_vec) {
      // kSfUnit stages (8 kSfUnit bytes of a row) per load unit, issued two units ahead of
      // use; unit n = stages kSfUnit v .. kSfUnit v + kSfUnit - 1 of local tile n / upt
      // (v = n % upt); 16-byte pieces past the row's end read as 0
      constexpr int kQ = kSfUnit / 2;  // 16-byte pieces per row and unit
      const int upt = (p.nk + kSfUnit - 1) / kSfUnit;
      const int n_units = n_local * upt;
      auto load = [&](int n, uint4 (&b)[3][kQ]) {
        if (n >= n_units) return;
        const int i = n / upt;
        const int64_t g0 = int64_t(n - i * upt) * (8 * kSfUnit);
#pragma unroll
        for (int r = 0; r < 3; ++r) {
          const int64_t row = tile_row(i, r);
#pragma unroll
          for (int q = 0; q < kQ; ++q)
            b[r][q] = row < lim[r] && g0 + 16 * (q + 1) <= p.sf_stride
                          ? __ldg(reinterpret_cast<const uint4*>(bases[r] + row * p.sf_stride + g0 + 16 * q))
                          : make_uint4(0u, 0u, 0u, 0u);
        }
      };
      auto store = [&](int n, const uint4 (&b)[3][kQ]) {
        const int i = n / upt, v = n - i * upt;
#pragma unroll
        for (int q = 0; q < kQ; ++q) {
          const int kb = kSfUnit * v + 2 * q;
          if (!ok || kb >= p.nk) return;
          const uint32_t w0[3][2] = {{b[0][q].x, b[0][q].y}, {b[1][q].x, b[1][q].y}, {b[2][q].x, b[2][q].y}};
          put(i * p.nk + kb, w0);
          if (!ok || kb + 1 >= p.nk) return;
          const uint32_t w1[3][2] = {{b[0][q].z, b[0][q].w}, {b[1][q].z, b[1][q].w}, {b[2][q].z, b[2][q].w}};
          put(i * p.nk + kb + 1, w1);
        }
      };
      uint4 b0[3][kQ], b1[3][kQ];
      load(0, b0);
      load(1, b1);
      for (int n = 0; ok && n < n_units; n += 2) {
        store(n, b0);
        load(n + 2, b0);
        if (!ok || n + 1 >= n_units) break;
        store(n + 1, b1);
        load(n + 3, b1);
      }
    } else {
      // any row stride or alignment: word by word, bytes past the row read as 0
      int it = 0;
      for (int i = 0; ok && i < n_local; ++i)
        for (int kb = 0; ok && kb < p.nk; ++kb, ++it) {
          uint32_t w[3][2];
#pragma unroll
          for (int r = 0; r < 3; ++r)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              w[r][h] = load_sf_word(bases[r], lim[r], tile_row(i, r), p.sf_stride, int64_t(kb) * 8 + 4 * h);
          put(it, w);
        }
    }
  } else if (warp >= kWarpEpi0 && warp < kWarpEpi0 + 4) {
    const int q = warp - kWarpEpi0;
    const uint32_t t_lane = tmem + (uint32_t(q * 32) << 16);
    const bool vec_ok = (p.O % 4) == 0 && (reinterpret_cast<uintptr_t>(p.C) & 15u) == 0;
    for (int i = 0; i < n_local; ++i) {
      const int tile = int(blockIdx.x) + i * int(gridDim.x);
      const int64_t row = int64_t(tile / p.tiles_n) * kBM + q * 32 + lane;
      const int64_t n0 = int64_t(tile % p.tiles_n) * kBN;
      const bool ok = warp_wait(&bars->d_full, i & 1, bars, p.status, kStDFull);
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_lane + kColD + uint32_t(c * 32), r);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
          if (c == kBN / 32 - 1) {
            // the accumulator is free for the next tile once its last columns are in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->d_empty);
          }
          const int64_t col0 = n0 + c * 32;
          if (row < p.T) {
            float* dst = p.C + row * p.O + col0;
            if (vec_ok && col0 + 32 <= p.O) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(dst + e) =
                    make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                                __uint_as_float(r[e + 3]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (col0 + e < p.O) dst[e] = __uint_as_float(r[e]);
            }
          }
        }
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->d_empty);
        break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

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

// 2-D byte tensor [rows, L / 2] of packed codes, boxes of 128 bytes x box_rows, 128B swizzle.
bool encode_codes(CUtensorMap* map, const void* codes, int64_t rows, int64_t L, uint32_t box_rows) {
  auto enc = get_encode();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cuuint64_t(L / 2), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(L / 2)};
  const cuuint32_t box[2] = {uint32_t(kBKBytes), box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_mxgemm(const MxGemmParams& g, int num_sms, cudaStream_t stream) {
  CUtensorMap map_a, map_w;
  if (!encode_codes(&map_a, g.a_codes, g.T, g.L, kBM) || !encode_codes(&map_w, g.w_codes, g.O, g.L, kBN))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.a_scales = g.a_scales;
  p.w_scales = g.w_scales;
  p.C = g.C;
  p.status = g.status;
  p.T = g.T;
  p.O = g.O;
  p.L = g.L;
  p.sf_stride = 2 * ((g.L + 63) / 64);
  p.tiles_n = int((g.O + kBN - 1) / kBN);
  p.num_tiles = int((g.T + kBM - 1) / kBM) * p.tiles_n;
  p.nk = int((g.L / 2 + kBKBytes - 1) / kBKBytes);
  p.sf_vec = (p.sf_stride % 16) == 0 && (reinterpret_cast<uintptr_t>(g.a_scales) & 15u) == 0 &&
             (reinterpret_cast<uintptr_t>(g.w_scales) & 15u) == 0;
  cudaError_t e = cudaFuncSetAttribute(mxgemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < num_sms ? p.num_tiles : num_sms;
  mxgemm_kernel<<<grid, kThreads, kSmem, stream>>>(map_a, map_w, p);
  return cudaGetLastError();
}

}  // namespace fq
