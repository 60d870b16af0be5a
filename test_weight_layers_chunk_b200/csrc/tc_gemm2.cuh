// Persistent tcgen05 GEMM core for sm_100a (one CTA per SM).
//
// Each CTA walks a static list of 128 x BN output tiles (tile = blockIdx.x,
// blockIdx.x + gridDim.x, ...), bf16 operands, fp32 accumulators in tensor
// memory. One accumulator: D = A B^T. Two accumulators (BN = 128), chosen per
// tile class: D_i = A_i B^T (two A operands share B) or D_i = A B_i^T (one A
// shared by two B operands).
//   warp 0      TMA producer over (tile, k-block) pairs into a STAGES-deep ring
//               of 128B-swizzled shared-memory tiles; operands may be K-major
//               (box 64 K x rows) or MN-major (boxes of 64 MN x 64 K)
//   warp 1      allocates TMEM (two accumulator sets, so the epilogue of tile i
//               overlaps the MMAs of tile i+1) and issues tcgen05.mma
//               (kind::f16, M=128, N=BN, K=16) from one thread
//   warps 2..   epilogue: tcgen05.ld 32x32b from the warp's lane quadrant, the
//               phase's fused epilogue, then release of the accumulator set
// Every mbarrier wait is bounded (about 1 s of globaltimer). On expiry the CTA
// records a code in the device status word, stops, waits (bounded) for its own
// copies and MMAs in flight, frees TMEM and exits. No TMA multicast anywhere.
// Launched with programmatic stream serialization: the set-up (barriers, TMEM,
// tensor-map prefetch) overlaps the tail of the previous kernel on the stream,
// and every thread waits for that kernel (griddep_wait) before its first global
// access; the CTA at once lets the next kernel start its own set-up.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include <type_traits>

#include "common.cuh"
#include "tc_gemm.cuh"

namespace e2ttt {
namespace tc2 {

using tc::BM;
using tc::BK;
using tc::smem_u32;
using tc::mbar_init;
using tc::mbar_wait;
using tc::mbar_wait_hint;
using tc::mbar_try_wait;
using tc::mbar_expect_tx;
using tc::fence_mbar_init;
using tc::prefetch_tmap;
using tc::tma_load_2d;
using tc::tmem_alloc;
using tc::tmem_relinquish;
using tc::tmem_dealloc;
using tc::tc_fence_before;
using tc::tc_fence_after;
using tc::mma_bf16;
using tc::mma_commit;
using tc::tmem_ld32;

enum : int { kErrProducer = 1, kErrMma = 2, kErrEpilogue = 3 };
constexpr int kEpiBars = 4;  // epilogue-load mbarriers per epilogue warp

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Shared-memory descriptor, 128B swizzle, sm_100 version bit.
//  K-major tile (rows of 64 K elements, 128 B each): LBO 16 B (unused), SBO 1024 B
//    between 8-row atoms; a K=16 step advances the start by 32 B.
//  MN-major tile (64-element MN blocks of 64 K rows each, 8 KB apart): LBO 8 KB
//    between MN blocks, SBO 1024 B between 8-row K groups; a K=16 step advances
//    the start by 16 rows = 2048 B.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, bool mn_major) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(mn_major ? (8192 >> 4) : 1) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// kind::f16 instruction descriptor: D fp32, A/B bf16, majors, N, M.
__host__ __device__ constexpr uint32_t idesc(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Where an operand's tiles live in its 2-D tensor map (x = inner coordinate).
//   K-major:  x = x_base + k,            y = z * y_head + y_base + tile_origin
//   MN-major: x = x_base + tile_origin,  y = z * y_head + y_base + k
struct Opnd {
  int y_head, y_base, x_base;
};
enum : int { kModeA2B1 = 0, kModeA1B2 = 1 };
struct Class {
  int tiles_m, tiles_n, kblocks;
  Opnd a, b;
  int mode;  // two-accumulator kernels: kModeA2B1 or kModeA1B2
};
// op0 = A (A0), op2 = B (B1); op1 = A1 in mode A2B1, B0 in mode A1B2.
struct Maps {
  CUtensorMap op0, op1, op2;
};
struct Job {
  Maps maps[2];
  Class cls[2];
  int n_cls;
  int heads;
  int total_tiles;
  int* status;
  // Failure-detection test hook (0 = off): CTA 0's MMA issuer first waits on an
  // mbarrier that nothing completes, and every wait of the launch gives up
  // after wait_ns; the launch then reports a timeout in *status and exits.
  int stall;
  unsigned long long wait_ns;  // 0: the default limit (tc::kWaitNs)
  // chunk of this launch, handed to the epilogues: index, first token, tokens in
  // the chunk, and whether the bf16 operand copy of the end state is written
  int ci, t0, clen, wshadow;
};

template <int BN>
struct EpiCtx {
  int cls, z, m0, n0;
  int row;            // this thread's row inside the tile (its TMEM lane)
  int quad;           // this warp's lane quadrant (rows [32 quad, 32 quad + 32))
  int part, nparts;   // this warp's column share
  uint32_t taddr;     // TMEM address of (this warp's lane quadrant, this tile's accumulator set)
  uint8_t* wsmem;     // this warp's epilogue shared memory (EPI_SMEM bytes, 1024-aligned)
  uint64_t* wbar;     // kEpiBars mbarriers owned by this warp (epilogue TMA loads)
  uint32_t* uses;     // completed-phase counters of wbar[], kept across tiles
  int slot;           // this tile's epilogue input buffer / wbar index (tile ordinal & 1)
  int iter;           // ordinal of this tile among the CTA's tiles
  int seq;            // ordinal among the CTA's tiles of this epilogue type
  int pre;            // 1 if the CTA's previous tile already issued this tile's first input loads
  int ci, t0, clen, wshadow;  // the tile's chunk (see Job)
  // the CTA's next tile (nxt_valid = 0 if this is its last), for epilogues that
  // start loading the next tile's inputs while finishing this one
  int nxt_valid, nxt_cls, nxt_z, nxt_m0, nxt_n0, nxt_ci;
  __device__ __forceinline__ void ld(int acc, int col, float (&v)[32]) const {
    tmem_ld32(taddr + (uint32_t)(acc * BN + col), v);
  }
};

// Epilogues that define kPrefetch = true also provide bool prefetch(prm, ctx):
// TMA loads of the tile's epilogue inputs into input buffer ctx.slot, signalled
// on ctx.wbar[ctx.slot]; it returns (warp-uniformly) whether it issued any. The
// core issues them one tile ahead, before it waits for the previous tile's
// accumulator, so the loads overlap that tile's epilogue.
template <class E, class = void>
struct EpiPrefetch : std::false_type {};
template <class E>
struct EpiPrefetch<E, std::void_t<decltype(E::kPrefetch)>> : std::bool_constant<E::kPrefetch> {};

template <int BN, int NUM_ACC, bool A_MN, bool B_MN>
struct Cfg {
  static_assert(NUM_ACC == 1 || BN <= BM, "two-accumulator tiles are 128 x 128 or 128 x 64");
  static constexpr uint32_t kTileA = BM * BK * 2;
  static constexpr uint32_t kTileB = BN * BK * 2;
  // stage layout: [A][B] for one accumulator; for two, [A0][A1][B] (two A
  // operands share B) or [A][B0][B1] (one A shared by two B operands)
  static constexpr uint32_t kOffA1B = kTileA;                  // A2B1: A1 at kTileA, B at 2 kTileA
  static constexpr uint32_t kOffB1 = kTileA + kTileB;         // A1B2: B0 at kTileA, B1 here
  static constexpr uint32_t kStage =
      NUM_ACC == 1 ? kTileA + kTileB
                   : (2 * kTileA + kTileB > kTileA + 2 * kTileB ? 2 * kTileA + kTileB : kTileA + 2 * kTileB);
  static constexpr uint32_t kAccCols = NUM_ACC * BN;  // one accumulator set
  static_assert(2 * kAccCols <= 512, "two accumulator sets must fit in TMEM");
  static constexpr uint32_t kTmemCols = 2 * kAccCols <= 128 ? 128 : 2 * kAccCols <= 256 ? 256 : 512;
};

template <int BN, int NUM_ACC, bool A_MN, bool B_MN, int STAGES, int EPI_WARPS = 8, int EPI_SMEM = 0,
          int KG = 1>
constexpr size_t smem_bytes() {
  // ring + per-warp epilogue buffers + barriers; at least 116 KB so that one
  // CTA is resident per SM
  size_t s = 1024 + (size_t)STAGES * KG * Cfg<BN, NUM_ACC, A_MN, B_MN>::kStage +
             (size_t)EPI_WARPS * EPI_SMEM + 256 + 8 * kEpiBars * EPI_WARPS;
  return s < 118784 ? 118784 : s;
}

__device__ __forceinline__ void decode_tile(const Job& job, int t, int& c, int& z, int& mt, int& nt) {
  c = 0;
  const int per0 = job.cls[0].tiles_m * job.cls[0].tiles_n * job.heads;
  if (job.n_cls > 1 && t >= per0) {
    t -= per0;
    c = 1;
  }
  const Class& K = job.cls[c];
  const int per_head = K.tiles_m * K.tiles_n;
  z = t / per_head;
  const int r = t - z * per_head;
  mt = r / K.tiles_n;
  nt = r - mt * K.tiles_n;
}

// Load one operand tile (rows = 128 or BN in the MN direction, 64 K) into smem.
template <bool MN, int ROWS>
__device__ __forceinline__ void load_opnd(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                          const Opnd& o, int z, int origin, int kb) {
  if (!MN) {
    tma_load_2d(dst, map, bar, o.x_base + kb * BK, z * o.y_head + o.y_base + origin);
  } else {
#pragma unroll
    for (int blk = 0; blk < ROWS / 64; ++blk)
      tma_load_2d(dst + blk * 8192, map, bar, o.x_base + origin + blk * 64,
                  z * o.y_head + o.y_base + kb * BK);
  }
}

template <int BN, int NUM_ACC, bool A_MN, bool B_MN, int STAGES, int EPI_WARPS, class Epi, class P,
          int EPI_SMEM = 0, int KG = 1>
__global__ void __launch_bounds__((2 + EPI_WARPS) * 32, 1)
gemm_persistent(const __grid_constant__ Job job, const __grid_constant__ P prm) {
  using C_ = Cfg<BN, NUM_ACC, A_MN, B_MN>;
  static_assert(EPI_SMEM % 1024 == 0, "epilogue buffers stay 1024-byte aligned");
  // One ring slot holds KG consecutive 64-wide k-blocks (one full/empty handshake
  // per KG k-blocks); every class's k-block count is a multiple of KG.
  constexpr uint32_t kSlot = KG * C_::kStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* epi_smem = smem + (size_t)STAGES * kSlot;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi_smem + (size_t)EPI_WARPS * EPI_SMEM);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* epi_bar = acc_empty + 2;     // [kEpiBars per epilogue warp]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + kEpiBars * EPI_WARPS);
  __shared__ int s_err;
  __shared__ uint64_t never;  // the stall hook's mbarrier: nothing ever arrives on it
  const unsigned long long lim = job.wait_ns ? job.wait_ns : tc::kWaitNs;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    s_err = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    for (int w = 0; w < kEpiBars * EPI_WARPS; ++w) mbar_init(&epi_bar[w], 1);
    mbar_init(&never, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < job.n_cls; ++c) {
      prefetch_tmap(&job.maps[c].op0);
      if (NUM_ACC > 1) prefetch_tmap(&job.maps[c].op1);
      prefetch_tmap(&job.maps[c].op2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C_::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  int mma_tiles = 0;
  griddep_wait();  // the previous kernel's results are complete and visible

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < job.total_tiles && ok; t += gridDim.x) {
      int c, z, mt, nt;
      decode_tile(job, t, c, z, mt, nt);
      const Class& K = job.cls[c];
      const Maps& M = job.maps[c];
      for (int kb = 0; kb < K.kblocks; kb += KG, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (it >= STAGES && !mbar_wait_hint(&empty[s], ph ^ 1u, lim)) {
          atomicExch(job.status, kErrProducer);
          s_err = 1;
          ok = false;
          break;
        }
        mbar_expect_tx(&full[s], kSlot);
#pragma unroll
        for (int g = 0; g < KG; ++g) {
          uint8_t* st = ring + (size_t)s * kSlot + g * C_::kStage;
          load_opnd<A_MN, BM>(st, &M.op0, &full[s], K.a, z, mt * BM, kb + g);
          if (NUM_ACC == 1) {
            load_opnd<B_MN, BN>(st + C_::kTileA, &M.op2, &full[s], K.b, z, nt * BN, kb + g);
          } else if (K.mode == kModeA2B1) {
            load_opnd<A_MN, BM>(st + C_::kOffA1B, &M.op1, &full[s], K.a, z, mt * BM, kb + g);
            load_opnd<B_MN, BN>(st + 2 * C_::kTileA, &M.op2, &full[s], K.b, z, nt * BN, kb + g);
          } else {
            load_opnd<B_MN, BN>(st + C_::kTileA, &M.op1, &full[s], K.b, z, nt * BN, kb + g);
            load_opnd<B_MN, BN>(st + C_::kOffB1, &M.op2, &full[s], K.b, z, nt * BN, kb + g);
          }
        }
      }
    }
    // no copy of ours may still be in flight when the CTA exits
    for (int j = it - STAGES < 0 ? 0 : it - STAGES; j < it; ++j)
      (void)mbar_wait(&full[j % STAGES], (uint32_t)(j / STAGES) & 1u, lim);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    constexpr uint32_t id = idesc(BM, BN, A_MN, B_MN);
    // descriptors = ring-base descriptor + (byte offset >> 4): the start-address
    // field is the low 14 bits and every operand lies below 256 KB of smem
    constexpr uint32_t kStepA = (A_MN ? 2048 : 32) >> 4;
    constexpr uint32_t kStepB = (B_MN ? 2048 : 32) >> 4;
    const uint64_t dA0 = sdesc(smem_u32(ring), A_MN);
    const uint64_t dB0 = sdesc(smem_u32(ring), B_MN);
    int it = 0, i = 0;
    bool ok = true;
    if (job.stall && blockIdx.x == 0 && !mbar_wait(&never, 0u, lim)) {
      atomicExch(job.status, kErrMma);
      s_err = 1;
      ok = false;
    }
    for (int t = blockIdx.x; t < job.total_tiles && ok; t += gridDim.x, ++i) {
      int c, z, mt, nt;
      decode_tile(job, t, c, z, mt, nt);
      const int kblocks = job.cls[c].kblocks;
      const bool a1b2 = NUM_ACC > 1 && job.cls[c].mode == kModeA1B2;
      const int b = i & 1;
      if (!mbar_wait(&acc_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, lim)) {
        atomicExch(job.status, kErrMma);
        s_err = 1;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * C_::kAccCols);
      for (int kb = 0; kb < kblocks; kb += KG, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!mbar_wait_hint(&full[s], ph, lim)) {
          atomicExch(job.status, kErrMma);
          s_err = 1;
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < KG; ++g) {
          const uint32_t so = ((uint32_t)s * kSlot + (uint32_t)g * C_::kStage) >> 4;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t accum = ((kb + g) | k) != 0;
            const uint64_t ad = dA0 + (so + k * kStepA);
            if (NUM_ACC == 1) {
              mma_bf16(acc, ad, dB0 + (so + (C_::kTileA >> 4) + k * kStepB), id, accum);
            } else if (!a1b2) {
              const uint64_t bd = dB0 + (so + ((2 * C_::kTileA) >> 4) + k * kStepB);
              mma_bf16(acc, ad, bd, id, accum);
              mma_bf16(acc + BN, dA0 + (so + (C_::kOffA1B >> 4) + k * kStepA), bd, id, accum);
            } else {
              mma_bf16(acc, ad, dB0 + (so + (C_::kTileA >> 4) + k * kStepB), id, accum);
              mma_bf16(acc + BN, ad, dB0 + (so + (C_::kOffB1 >> 4) + k * kStepB), id, accum);
            }
          }
        }
        mma_commit(&empty[s]);
      }
      mma_commit(&acc_full[b]);
      ++mma_tiles;
    }
  } else if (warp >= 2) {
    // ---------------- epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;
    uint32_t uses[kEpiBars] = {0u, 0u, 0u, 0u};
    bool pend[2] = {false, false};  // prefetched input buffers not yet consumed
    auto make_ctx = [&](int t, int i) {
      int c, z, mt, nt;
      decode_tile(job, t, c, z, mt, nt);
      EpiCtx<BN> ctx;
      ctx.cls = c;
      ctx.z = z;
      ctx.m0 = mt * BM;
      ctx.n0 = nt * BN;
      ctx.row = quad * 32 + lane;
      ctx.quad = quad;
      ctx.nparts = EPI_WARPS / 4;
      ctx.part = ew >> 2;
      ctx.taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)((i & 1) * C_::kAccCols);
      ctx.wsmem = epi_smem + (size_t)ew * EPI_SMEM;
      ctx.wbar = epi_bar + kEpiBars * ew;
      ctx.uses = uses;
      ctx.slot = i & 1;
      ctx.iter = i;
      ctx.seq = i;
      ctx.pre = i > 0;
      ctx.ci = job.ci;
      ctx.t0 = job.t0;
      ctx.clen = job.clen;
      ctx.wshadow = job.wshadow;
      ctx.nxt_valid = t + (int)gridDim.x < job.total_tiles;
      ctx.nxt_cls = ctx.nxt_z = ctx.nxt_m0 = ctx.nxt_n0 = 0;
      ctx.nxt_ci = job.ci;
      if (ctx.nxt_valid) {
        int c2, z2, mt2, nt2;
        decode_tile(job, t + gridDim.x, c2, z2, mt2, nt2);
        ctx.nxt_cls = c2;
        ctx.nxt_z = z2;
        ctx.nxt_m0 = mt2 * BM;
        ctx.nxt_n0 = nt2 * BN;
      }
      return ctx;
    };
    constexpr bool kPre = EpiPrefetch<Epi>::value;
    if constexpr (kPre) {
      if ((int)blockIdx.x < job.total_tiles) pend[0] = Epi::prefetch(prm, make_ctx(blockIdx.x, 0));
    }
    int i = 0;
    for (int t = blockIdx.x; t < job.total_tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      const EpiCtx<BN> ctx = make_ctx(t, i);
      if constexpr (kPre) {
        if (t + (int)gridDim.x < job.total_tiles && !s_err)
          pend[(i + 1) & 1] = Epi::prefetch(prm, make_ctx(t + gridDim.x, i + 1));
      }
      if (!mbar_wait(&acc_full[b], (uint32_t)(i >> 1) & 1u, lim)) {
        atomicExch(job.status, kErrEpilogue);
        s_err = 1;
        break;
      }
      tc_fence_after();
      if (!s_err) {
        Epi::run(prm, ctx);
        pend[b] = false;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
    // no prefetch of ours may still be in flight when the CTA exits
    for (int k = 0; k < 2; ++k)
      if (kPre && pend[k]) (void)mbar_wait(&epi_bar[kEpiBars * ew + k], uses[k] & 1u, lim);
    if (EPI_SMEM > 0 && lane == 0) tc::bulk_wait_all();  // our TMA stores have completed
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && mma_tiles > 0) {
      // wait (bounded) until the last committed accumulator set is complete
      const int last = mma_tiles - 1;
      (void)mbar_wait(&acc_full[last & 1], (uint32_t)(last >> 1) & 1u, lim);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C_::kTmemCols);
  }
}

}  // namespace tc2
}  // namespace e2ttt

namespace e2ttt {
namespace tc2 {

// tcgen05.ld of 32 columns without waiting; call tmem_wait_ld() before use.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
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
}
// Wait for this thread's outstanding tcgen05.ld, then pin the registers after
// the wait so no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; i += 8)
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]),
                 "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7]));
}
__device__ __forceinline__ void tmem_wait_ld2(uint32_t (&r)[32], uint32_t (&s)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; i += 8) {
    asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]),
                 "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7]));
    asm volatile("" : "+r"(s[i]), "+r"(s[i + 1]), "+r"(s[i + 2]), "+r"(s[i + 3]), "+r"(s[i + 4]),
                 "+r"(s[i + 5]), "+r"(s[i + 6]), "+r"(s[i + 7]));
  }
}

}  // namespace tc2
}  // namespace e2ttt
