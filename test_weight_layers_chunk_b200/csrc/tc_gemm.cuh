// tcgen05 tensor-core GEMM core for sm_100a.
//
// One CTA computes one 128 x BN output tile of D_i = A_i * B^T (i < NUM_A; the
// A_i share the B operand), bf16 operands, fp32 accumulators in tensor memory:
//   warp 0      TMA producer: 64-wide K blocks of A_i and B into a STAGES-deep
//               ring of 128B-swizzled shared-memory tiles (mbarrier complete_tx)
//   warp 1      allocates TMEM, issues tcgen05.mma (kind::f16, M=128, N=BN,
//               K=16) from one thread, releases ring slots with tcgen05.commit
//   warps 2..   epilogue: tcgen05.ld 32x32b from the warp's TMEM lane quadrant,
//               then a phase-specific fused epilogue (Epi::run)
// Every mbarrier wait is bounded (about one second of globaltimer); on expiry
// the CTA records an error code in a device status word, stops issuing work,
// waits (bounded) for its own copies and MMAs in flight, frees TMEM and exits.
// No TMA multicast is used anywhere.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace e2ttt {
namespace tc {

constexpr int BM = 128;  // rows per tile (TMEM lanes)
constexpr int BK = 64;   // K elements per ring slot (128 B of bf16 = one swizzle atom row)
constexpr uint32_t kTileA = BM * BK * 2;  // bytes of one A slot
constexpr unsigned long long kWaitNs = 1000000000ull;  // bounded waits: 1 s

enum : int { kErrTimeoutProducer = 1, kErrTimeoutMma = 2, kErrTimeoutEpilogue = 3 };

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0 && globaltimer() - t0 > kWaitNs) return false;
  }
}
// Bounded wait for the hot producer / MMA loops: try_wait with a short
// suspend-time hint (20 ns), so a thread whose phase completes while it is
// suspended resumes promptly instead of after the default suspend interval.
__device__ __forceinline__ bool mbar_wait_hint(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer();
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(20u)
        : "memory");
    if (ok) return true;
    if ((i & 255) == 255 && globaltimer() - t0 > kWaitNs) return false;
  }
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// TMA stores from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1,
                                             int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
// L2 eviction-priority policies for the cache-hinted copies below.
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int c0, int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, const void* src, int c0,
                                                  int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d_hint(const CUtensorMap* map, const void* src, int c0,
                                                  int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make generic-proxy shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major, 128B-swizzled bf16 tile whose
// rows are 128 B apart (8-row swizzle atoms 1024 B apart): start address,
// leading offset 16 B (unused by this layout), stride offset 1024 B, the
// sm_100 descriptor version bit, and the 128B swizzle mode.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor for kind::f16: D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- job description
// Up to two tile classes per launch (e.g. query rows and key rows, or the
// W1/W3 and the W2 aggregations); each has its own operand maps and sizes.
struct Class {
  int tiles_m, tiles_n, kblocks;
  int a_row_head, a_row_base;  // A row coordinate = z * a_row_head + a_row_base + m0
  int b_row_head, b_row_base;  // B row coordinate = z * b_row_head + b_row_base + n0
};
struct Maps {
  CUtensorMap a0, a1, b;
};
struct Job {
  Maps maps[2];
  Class cls[2];
  int n_cls;
  int heads;
  int* status;  // device status word (0 = ok)
};

// What a fused epilogue sees for one thread: its tile, its accumulator row and
// its share of the tile's columns.
template <int BN>
struct EpiCtx {
  int cls, z, m0, n0;  // tile origin inside the class problem (rows, columns)
  int row;             // this thread's row inside the tile (its TMEM lane)
  int part, nparts;    // this thread's column share: [part, part+1) of nparts equal parts
  uint32_t taddr;      // TMEM address of (this warp's lane quadrant, column 0)
  __device__ __forceinline__ void ld(int acc, int col, float (&v)[32]) const {
    tmem_ld32(taddr + (uint32_t)(acc * BN + col), v);
  }
};

template <int BN, int NUM_A>
struct Cfg {
  static constexpr uint32_t kTileB = BN * BK * 2;
  static constexpr uint32_t kStageBytes = NUM_A * kTileA + kTileB;
  static constexpr uint32_t kCols0 = NUM_A * BN;
  static constexpr uint32_t kTmemCols = kCols0 <= 32 ? 32 : kCols0 <= 64 ? 64 : kCols0 <= 128 ? 128
                                        : kCols0 <= 256 ? 256 : 512;
  // CTAs that fit on one SM by TMEM; shared memory is padded so that no more
  // than this many are resident (tcgen05.alloc then never has to wait).
  static constexpr int kMaxResident = 512 / kTmemCols;
  static constexpr uint32_t kSmemFloor = 233472u / (kMaxResident + 1) - 1024u + 1u;
};

template <int BN, int NUM_A, int STAGES>
constexpr size_t smem_bytes() {
  size_t s = 1024 + (size_t)STAGES * Cfg<BN, NUM_A>::kStageBytes + 256;
  return s < Cfg<BN, NUM_A>::kSmemFloor ? Cfg<BN, NUM_A>::kSmemFloor : s;
}

template <int BN, int NUM_A, int STAGES, int EPI_WARPS, class Epi, class P>
__global__ void __launch_bounds__((2 + EPI_WARPS) * 32, 1)
gemm_kernel(const __grid_constant__ Job job, const __grid_constant__ P prm) {
  using C_ = Cfg<BN, NUM_A>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)STAGES * C_::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  __shared__ int s_err;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // tile -> (class, head, m tile, n tile)
  int t = blockIdx.x, c = 0;
  const int per0 = job.cls[0].tiles_m * job.cls[0].tiles_n * job.heads;
  if (job.n_cls > 1 && t >= per0) { t -= per0; c = 1; }
  const Class& K = job.cls[c];
  const Maps& M = job.maps[c];
  const int per_head = K.tiles_m * K.tiles_n;
  const int z = t / per_head;
  const int r = t - z * per_head;
  const int mt = r / K.tiles_n, nt = r - mt * K.tiles_n;
  const int m0 = mt * BM, n0 = nt * BN;

  if (threadIdx.x == 0) {
    s_err = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&M.a0);
    if (NUM_A > 1) prefetch_tmap(&M.a1);
    prefetch_tmap(&M.b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C_::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    const int a_row = z * K.a_row_head + K.a_row_base + m0;
    const int b_row = z * K.b_row_head + K.b_row_base + n0;
    int issued = 0;
    for (int kb = 0; kb < K.kblocks; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
      if (kb >= STAGES && !mbar_wait(&empty[s], ph ^ 1u)) {
        atomicExch(job.status, kErrTimeoutProducer);
        s_err = 1;
        break;
      }
      uint8_t* st = ring + (size_t)s * C_::kStageBytes;
      mbar_expect_tx(&full[s], C_::kStageBytes);
      tma_load_2d(st, &M.a0, &full[s], kb * BK, a_row);
      if (NUM_A > 1) tma_load_2d(st + kTileA, &M.a1, &full[s], kb * BK, a_row);
      tma_load_2d(st + NUM_A * kTileA, &M.b, &full[s], kb * BK, b_row);
      ++issued;
    }
    // make sure no copy of ours is still in flight before the CTA can exit
    for (int kb = issued - STAGES < 0 ? 0 : issued - STAGES; kb < issued; ++kb)
      (void)mbar_wait(&full[kb % STAGES], (uint32_t)(kb / STAGES) & 1u);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16(BM, BN);
    for (int kb = 0; kb < K.kblocks; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
      if (!mbar_wait(&full[s], ph)) {
        atomicExch(job.status, kErrTimeoutMma);
        s_err = 1;
        break;
      }
      tc_fence_after();
      const uint32_t st = smem_u32(ring + (size_t)s * C_::kStageBytes);
#pragma unroll
      for (int k = 0; k < BK / 16; ++k) {
        const uint64_t bdesc = sdesc_k_sw128(st + NUM_A * kTileA + k * 32);
        const uint32_t acc = (kb | k) != 0;
        mma_bf16(tmem, sdesc_k_sw128(st + k * 32), bdesc, idesc, acc);
        if (NUM_A > 1) mma_bf16(tmem + BN, sdesc_k_sw128(st + kTileA + k * 32), bdesc, idesc, acc);
      }
      mma_commit(&empty[s]);
      mma_issued = true;
    }
    mma_commit(accf);
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;
    EpiCtx<BN> ctx;
    ctx.cls = c;
    ctx.z = z;
    ctx.m0 = m0;
    ctx.n0 = n0;
    ctx.row = quad * 32 + lane;
    ctx.nparts = EPI_WARPS / 4;
    ctx.part = ew >> 2;
    ctx.taddr = tmem + ((uint32_t)(quad * 32) << 16);
    if (mbar_wait(accf, 0)) {
      tc_fence_after();
      if (!s_err) Epi::run(prm, ctx);
    } else {
      atomicExch(job.status, kErrTimeoutEpilogue);
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && mma_issued) (void)mbar_wait(accf, 0);  // no MMA of ours in flight
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C_::kTmemCols);
  }
}

}  // namespace tc
}  // namespace e2ttt
