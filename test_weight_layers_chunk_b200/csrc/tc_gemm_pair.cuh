// Persistent tcgen05 GEMM core on CTA pairs (sm_100a, cta_group::2), used by the
// forward's G1-G3 when E2TTT_PAIRS=1 (measured slower than the one-CTA core on
// the shapes tried, so not the default).
//
// A cluster of two CTAs on the two SMs of a TPC computes 256 x BN output tiles:
// each CTA holds its own 128 rows of the A tile and half (BN/2 rows) of the B
// tile in its shared memory; the MMA, issued by the even CTA of the pair
// (tcgen05.mma.cta_group::2, M = 256), reads both halves and writes each CTA's
// 128 x BN accumulator into that CTA's tensor memory. Per output element the
// operands are the same as in the one-CTA core, so each CTA streams half the B
// bytes per tile from L2.
//   warp 0   both CTAs: TMA loads of the CTA's own A rows and B half into its
//            own ring slot (each CTA reads only its own tiles); the transaction
//            bytes of both land on the even CTA's full barrier (.cta_group::2)
//   warp 1   both CTAs allocate the pair's tensor memory (cta_group::2); the even
//            CTA's lane 0 issues the MMAs and commits them to both CTAs' empty
//            and accumulator barriers (multicast commit)
//   warps 2..  both CTAs: epilogue of the CTA's 128 rows; the release of an
//            accumulator set is counted on the even CTA's barrier
// Every mbarrier wait is bounded; the pair synchronises (barrier.cluster) after
// the set-up and before tensor memory is freed.
#pragma once
#include "tc_gemm2.cuh"

namespace e2ttt {
namespace tcp {

using namespace tc2;
using tc::BM;
using tc::BK;
using tc::smem_u32;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the mbarrier at this shared-memory offset in both CTAs of the
// pair when the pair's earlier MMAs have completed.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\t"
      "mov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}
// TMA tile load into this CTA's shared memory whose transaction bytes count on
// the mbarrier at cluster address `bar` (the even CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar, int c0,
                                                 int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// Bounded wait with acquire at cluster scope (phases completed by the other CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  const unsigned long long t0 = tc::globaltimer();
  for (uint32_t i = 0;; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    if (ok) return true;
    if ((i & 63) == 63 && tc::globaltimer() - t0 > limit_ns) return false;
  }
}

template <bool MN, int ROWS>
__device__ __forceinline__ void load_opnd_pair(uint8_t* dst, const CUtensorMap* map, uint32_t bar, const Opnd& o,
                                               int z, int origin, int kb) {
  if (!MN) {
    tma_load_2d_pair(dst, map, bar, o.x_base + kb * BK, z * o.y_head + o.y_base + origin);
  } else {
#pragma unroll
    for (int blk = 0; blk < ROWS / 64; ++blk)
      tma_load_2d_pair(dst + blk * 8192, map, bar, o.x_base + origin + blk * 64, z * o.y_head + o.y_base + kb * BK);
  }
}

template <int BN, bool A_MN, bool B_MN, int STAGES, int EPI_WARPS>
constexpr size_t pair_smem_bytes(int epi_smem) {
  return 1024 + (size_t)STAGES * ((size_t)BM * BK * 2 + (size_t)(BN / 2) * BK * 2) + (size_t)EPI_WARPS * epi_smem +
         256 + 8 * kEpiBars * EPI_WARPS;
}

// One accumulator per tile; Class.tiles_m counts 256-row tiles. Launched with a
// cluster of two CTAs and an even grid.
template <int BN, bool A_MN, bool B_MN, int STAGES, int EPI_WARPS, class Epi, class P, int EPI_SMEM = 0>
__global__ void __launch_bounds__((2 + EPI_WARPS) * 32, 1)
gemm_pair(const __grid_constant__ Job job, const __grid_constant__ P prm) {
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair tile width");
  static_assert(!EpiPrefetch<Epi>::value, "epilogue input prefetch is not supported on pairs");
  static_assert(EPI_SMEM % 1024 == 0, "epilogue buffers stay 1024-byte aligned");
  constexpr uint32_t kTileA = BM * BK * 2;
  constexpr uint32_t kTileB = (BN / 2) * BK * 2;
  constexpr uint32_t kStage = kTileA + kTileB;
  constexpr uint32_t kAccCols = BN;
  constexpr uint32_t kTmemCols = 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* epi_smem = smem + (size_t)STAGES * kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + (size_t)EPI_WARPS * EPI_SMEM);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2] (counted on the even CTA)
  uint64_t* epi_bar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + kEpiBars * EPI_WARPS);
  __shared__ int s_err;
  __shared__ uint64_t never;  // the stall hook's mbarrier: nothing ever arrives on it
  const unsigned long long lim = job.wait_ns ? job.wait_ns : tc::kWaitNs;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    s_err = 0;
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], 2 * EPI_WARPS);
    }
    for (int w = 0; w < kEpiBars * EPI_WARPS; ++w) tc::mbar_init(&epi_bar[w], 1);
    tc::mbar_init(&never, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < job.n_cls; ++c) {
      tc::prefetch_tmap(&job.maps[c].op0);
      tc::prefetch_tmap(&job.maps[c].op2);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc::tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int mma_tiles = 0;
  griddep_wait();

  if (warp == 0 && lane == 0) {
    // ---------------- producer (both CTAs)
    int it = 0;
    bool ok = true;
    for (int t = pair; t < job.total_tiles && ok; t += npairs) {
      int c, z, mt, nt;
      decode_tile(job, t, c, z, mt, nt);
      const Class& K = job.cls[c];
      const Maps& M = job.maps[c];
      for (int kb = 0; kb < K.kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (it >= STAGES && !tc::mbar_wait_hint(&empty[s], ph ^ 1u, lim)) {
          atomicExch(job.status, kErrProducer);
          s_err = 1;
          ok = false;
          break;
        }
        const uint32_t fb = mapa(smem_u32(&full[s]), 0);
        if (lead) tc::mbar_expect_tx(&full[s], 2 * kStage);
        uint8_t* st = ring + (size_t)s * kStage;
        load_opnd_pair<A_MN, BM>(st, &M.op0, fb, K.a, z, mt * 2 * BM + (int)rank * BM, kb);
        load_opnd_pair<B_MN, BN / 2>(st + kTileA, &M.op2, fb, K.b, z, nt * BN + (int)rank * (BN / 2), kb);
      }
    }
    // the even CTA's full barriers count both CTAs' bytes: once its last
    // phases completed, no copy of either CTA is in flight
    if (lead)
      for (int j = it - STAGES < 0 ? 0 : it - STAGES; j < it; ++j)
        (void)tc::mbar_wait(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, lim);
  } else if (warp == 1 && lane == 0 && lead) {
    // ---------------- MMA issuer (even CTA)
    constexpr uint32_t id = idesc(2 * BM, BN, A_MN, B_MN);
    constexpr uint32_t kStepA = (A_MN ? 2048 : 32) >> 4;
    constexpr uint32_t kStepB = (B_MN ? 2048 : 32) >> 4;
    const uint64_t dA0 = sdesc(smem_u32(ring), A_MN);
    const uint64_t dB0 = sdesc(smem_u32(ring), B_MN);
    int it = 0, i = 0;
    bool ok = true;
    if (job.stall && pair == 0 && !tc::mbar_wait(&never, 0u, lim)) {  // failure-detection hook
      atomicExch(job.status, kErrMma);
      s_err = 1;
      ok = false;
    }
    for (int t = pair; t < job.total_tiles && ok; t += npairs, ++i) {
      int c, z, mt, nt;
      decode_tile(job, t, c, z, mt, nt);
      const int kblocks = job.cls[c].kblocks;
      const int b = i & 1;
      if (!mbar_wait_cluster(&acc_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, lim)) {
        atomicExch(job.status, kErrMma);
        s_err = 1;
        break;
      }
      tc::tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * kAccCols);
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!mbar_wait_cluster(&full[s], ph, lim)) {
          atomicExch(job.status, kErrMma);
          s_err = 1;
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t so = ((uint32_t)s * kStage) >> 4;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          mma_pair(acc, dA0 + (so + k * kStepA), dB0 + (so + (kTileA >> 4) + k * kStepB), id, (kb | k) != 0);
        commit_pair(&empty[s]);
      }
      commit_pair(&acc_full[b]);
      ++mma_tiles;
    }
  } else if (warp >= 2) {
    // ---------------- epilogue (both CTAs, this CTA's 128 rows)
    const int ew = warp - 2;
    const int quad = warp & 3;
    uint32_t uses[kEpiBars] = {0u, 0u, 0u, 0u};
    const uint32_t empty_lead[2] = {mapa(smem_u32(&acc_empty[0]), 0), mapa(smem_u32(&acc_empty[1]), 0)};
    int i = 0;
    for (int t = pair; t < job.total_tiles; t += npairs, ++i) {
      const int b = i & 1;
      int c, z, mt, nt;
      decode_tile(job, t, c, z, mt, nt);
      EpiCtx<BN> ctx;
      ctx.cls = c;
      ctx.z = z;
      ctx.m0 = mt * 2 * BM + (int)rank * BM;
      ctx.n0 = nt * BN;
      ctx.row = quad * 32 + lane;
      ctx.quad = quad;
      ctx.nparts = EPI_WARPS / 4;
      ctx.part = ew >> 2;
      ctx.taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * kAccCols);
      ctx.wsmem = epi_smem + (size_t)ew * EPI_SMEM;
      ctx.wbar = epi_bar + kEpiBars * ew;
      ctx.uses = uses;
      ctx.slot = b;
      ctx.iter = i;
      ctx.seq = i;
      ctx.pre = i > 0;
      ctx.ci = job.ci;
      ctx.t0 = job.t0;
      ctx.clen = job.clen;
      ctx.wshadow = job.wshadow;
      ctx.nxt_valid = t + npairs < job.total_tiles;
      ctx.nxt_cls = ctx.nxt_z = ctx.nxt_m0 = ctx.nxt_n0 = 0;
      ctx.nxt_ci = job.ci;
      if (ctx.nxt_valid) {
        int c2, z2, mt2, nt2;
        decode_tile(job, t + npairs, c2, z2, mt2, nt2);
        ctx.nxt_cls = c2;
        ctx.nxt_z = z2;
        ctx.nxt_m0 = mt2 * 2 * BM + (int)rank * BM;
        ctx.nxt_n0 = nt2 * BN;
      }
      if (!tc::mbar_wait(&acc_full[b], (uint32_t)(i >> 1) & 1u, lim)) {
        atomicExch(job.status, kErrEpilogue);
        s_err = 1;
        break;
      }
      tc::tc_fence_after();
      if (!s_err) Epi::run(prm, ctx);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(empty_lead[b]);
    }
    if (EPI_SMEM > 0 && lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1 && lane == 0 && lead && mma_tiles > 0) {
    const int last = mma_tiles - 1;
    (void)tc::mbar_wait(&acc_full[last & 1], (uint32_t)(last >> 1) & 1u, lim);
  }
  __syncwarp();
  cluster_sync();  // no CTA frees the pair's tensor memory or exits while the other still uses it
  if (warp == 1) {
    tc::tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace tcp
}  // namespace e2ttt
