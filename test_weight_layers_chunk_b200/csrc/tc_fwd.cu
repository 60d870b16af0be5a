// tcgen05 tensor-core forward of the chunk scan (bf16 activations, fp32 state).
//
// Per chunk (all heads at once), "Rethinking Expressivity and Efficiency in
// Test-Time Training" (abstract: closed-form chunk transition with chunk-start
// gradients; atlas "Approach": two weighted gradient aggregations; arxivlens
// "Limitations": output at the chunk-start weights), SwiGLU fast weight:
//   G1  H = [Q; K] [W1; W3]^T     epilogue: A = silu(H1) * H3 for both row sets,
//                                 silu(H1_k) and H3_k silu'(H1_k)
//   G2  Y = A W2^T                epilogue: out = Y_q; E = Y_k - V and its a-/b-
//                                 scaled copies
//   G3  dA = E W2                 epilogue: dH1 = dA H3 silu'(H1), dH3 = dA silu(H1)
//   G4  [dM | dW] of [W1; W3] = dH^T [diag(a) K | diag(b) K]  (one A, two B)
//       [dM | dW] of W2       = [diag(a) E | diag(b) E]^T A_k  (two A, one B)
//                                 epilogue: M_end = U M0 - dM, W_end = L W0 + c M0 - dW
//                                 in fp32, plus the bf16 operand copies of W_end
// Linear fast weight: G1 gives out and the scaled E; G4 aggregates them with K.
// All intermediates are stored token-major (natural rows); the aggregations read
// them as MN-major operands, so nothing is ever transposed.
#include <cuda.h>

#include <stdlib.h>

#include <atomic>

#include "paths.h"
#include "state.cuh"
#include "tc_gemm2.cuh"
#include "tc_gemm_pair.cuh"
#include "trace.h"

namespace e2ttt {
namespace {

using tc2::EpiCtx;
using tc2::tmem_ld32_nowait;
using tc2::tmem_wait_ld;
using tc2::tmem_wait_ld2;

constexpr int kEpiWarps = 8;
constexpr int HB = 128;  // hidden units per G1 tile (its 256 columns hold h1 then h3)

struct FwdP {
  // fp32 state tiles of the aggregation epilogue (3-D maps: columns, rows, heads)
  // and the bf16 operand copies it writes; second index = tile class (0: [W1; W3]
  // or W, 1: W2); first index of the source maps: 0 = the tile's chunk is the
  // call's first (it reads W0, M0), 1 = a later chunk. The per-phase launches
  // rebuild them for every chunk and fill both entries alike.
  CUtensorMap srcW[2][2], srcM[2][2], dstW[2], dstM[2], shadow[2];
  int hasM[2];  // whether the source momentum of variant 0 / 1 exists (M0 may be NULL)
  // 32 x 32 bf16 tiles (64B swizzle) moved by the other epilogues; mOut and mV
  // are 3-D (columns, tokens, heads), so a box past a head's last token is
  // clipped on store and reads as zero
  CUtensorMap mA, mSk, mOut, mV, mE, mEa, mEb, mdH;
  Dims d;
  int nomom;  // no momentum: no a-scaled operands, W-only aggregation epilogue
  int* status;
  const bf16 *q, *k, *v;
  bf16* out;
  const float *ca, *cb, *scal;
  bf16 *Wsh13, *W2sh;  // bf16 copies of the chunk-start weights (Wsh13 = W for linear)
  bf16 *A, *Sk, *E, *Ea, *Eb, *dH, *Ka, *Kb;
};

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float fast_sigmoid(float z) { return __fdividef(1.0f, 1.0f + __expf(-z)); }
// Row of the interleaved [W1; W3] operand copy that holds row r of W1 (which=0) or W3 (which=1).
__device__ __forceinline__ int w13_row(int r, int which) {
  return (r / HB) * (2 * HB) + which * HB + (r % HB);
}
// Staging tile = one TMA box of make_map_box32: 32 rows x 32 bf16, row r at
// r * 64 bytes with its 16-byte chunks permuted by the 64B swizzle.
__device__ __forceinline__ int sw64(int r, int q) { return r * 64 + ((q ^ ((r >> 1) & 3)) << 4); }
__device__ __forceinline__ void stage32(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(buf + sw64(r, q)) =
        make_uint4(pack2(v[8 * q], v[8 * q + 1]), pack2(v[8 * q + 2], v[8 * q + 3]),
                   pack2(v[8 * q + 4], v[8 * q + 5]), pack2(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void unstage32(const uint8_t* buf, int r, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = *reinterpret_cast<const uint4*>(buf + sw64(r, q));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      v[8 * q + 2 * j] = f.x;
      v[8 * q + 2 * j + 1] = f.y;
    }
  }
}
// Before refilling staging tiles: this warp's earlier TMA stores must have read them.
__device__ __forceinline__ void staging_free(int lane) {
  if (lane == 0) tc::bulk_wait_read<0>();
  __syncwarp();
}
// After filling staging tiles: make them visible to the TMA (async) proxy.
__device__ __forceinline__ void staging_ready() {
  tc::fence_async_smem();
  __syncwarp();
}

template <int BN>
__device__ __forceinline__ void ld2(const EpiCtx<BN>& c, int acc0, int col0, int acc1, int col1,
                                    float (&x)[32], float (&y)[32]) {
  uint32_t r[32], s[32];
  tmem_ld32_nowait(c.taddr + (uint32_t)(acc0 * BN + col0), r);
  tmem_ld32_nowait(c.taddr + (uint32_t)(acc1 * BN + col1), s);
  tmem_wait_ld2(r, s);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = __uint_as_float(r[i]);
    y[i] = __uint_as_float(s[i]);
  }
}
template <int BN>
__device__ __forceinline__ void ld1(const EpiCtx<BN>& c, int acc, int col, float (&x)[32]) {
  uint32_t r[32];
  tmem_ld32_nowait(c.taddr + (uint32_t)(acc * BN + col), r);
  tmem_wait_ld(r);
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------- epilogues
// Epilogues of G1-G3: each warp owns 32 rows (its TMEM lane quadrant) and a
// share of the tile's columns; results are staged in shared memory and written
// with TMA stores, inputs they need (V, silu factors) are prefetched with TMA.

// G1, SwiGLU. Class 0 = query rows, class 1 = key rows of the chunk.
struct EpiG1 {
  static constexpr int kSmem = 6144;  // A | silu(H1) | H3 silu'(H1) staging
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;  // first token row of this warp
    const int j0 = (c.n0 / (2 * HB)) * HB;
    const int per = HB / c.nparts;
    const int yA = c.z * 2 * d.C + c.cls * d.C + r0;
    const int ySk = c.z * d.C + r0;
    uint8_t* S = c.wsmem;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      float h1[32], h3[32];
      ld2(c, 0, g, 0, HB + g, h1, h3);
      if (c.cls == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) h1[i] = h1[i] * fast_sigmoid(h1[i]) * h3[i];
        staging_free(lane);
        stage32(S, lane, h1);
      } else {
        float s2[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sg = fast_sigmoid(h1[i]);
          const float s1 = h1[i] * sg;
          s2[i] = h3[i] * sg * (1.0f + h1[i] * (1.0f - sg));
          h3[i] = s1 * h3[i];  // u
          h1[i] = s1;
        }
        staging_free(lane);
        stage32(S, lane, h3);
        stage32(S + 2048, lane, h1);
        stage32(S + 4096, lane, s2);
      }
      staging_ready();
      if (lane == 0) {
        const uint64_t keep = tc::l2_evict_last();  // read by the next phases of the chunk
        tc::tma_store_2d_hint(&p.mA, S, j0 + g, yA, keep);
        if (c.cls == 1) {
          tc::tma_store_2d_hint(&p.mSk, S + 2048, j0 + g, ySk, keep);
          tc::tma_store_2d_hint(&p.mSk, S + 4096, d.d_h + j0 + g, ySk, keep);
        }
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};

// G1, GELU MLP: H = X W1^T -> A = gelu(H) (query and key rows) and the key rows'
// gelu'(H) (the factor G3 needs). Class 0 = query rows, class 1 = key rows.
struct EpiG1Gelu {
  static constexpr int kSmem = 4096;  // gelu(H) | gelu'(H) staging
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;
    const int per = BN / c.nparts;
    const int yA = c.z * 2 * d.C + c.cls * d.C + r0;
    const int ySk = c.z * d.C + r0;
    uint8_t* S = c.wsmem;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      const int j = c.n0 + g;
      float h[32], gp[32];
      ld1(c, 0, g, h);
      if (c.cls == 1) {  // key rows: gelu and gelu'
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          gp[i] = dgelu_f(h[i]);
          h[i] = gelu_f(h[i]);
        }
      } else {  // query rows: gelu alone
#pragma unroll
        for (int i = 0; i < 32; ++i) h[i] = gelu_f(h[i]);
      }
      staging_free(lane);
      stage32(S, lane, h);
      if (c.cls == 1) stage32(S + 2048, lane, gp);
      staging_ready();
      if (lane == 0) {
        const uint64_t keep = tc::l2_evict_last();  // read by the next phases of the chunk
        tc::tma_store_2d_hint(&p.mA, S, j, yA, keep);
        if (c.cls == 1) tc::tma_store_2d_hint(&p.mSk, S + 2048, j, ySk, keep);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};

// G3, GELU MLP: dA = E W2 -> dH = dA gelu'(H_k) (rows: key tokens).
struct EpiG3Gelu {
  static constexpr int kSmem = 6144;  // gelu'(H) [2 groups] | dH staging
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;
    const int per = BN / c.nparts;
    const int col0 = c.n0 + c.part * per;
    static_assert(BN <= 128, "factor buffers for at most two column groups per warp");
    const int ngroups = per / 32;
    const int y = c.z * d.C + r0;
    uint8_t* F = c.wsmem;
    uint8_t* S = c.wsmem + 4096;
    if (lane == 0) {
      tc::mbar_expect_tx(&c.wbar[0], 2048u * ngroups);
      for (int gi = 0; gi < ngroups; ++gi)
        tc::tma_load_2d(F + gi * 2048, &p.mSk, &c.wbar[0], col0 + gi * 32, y);
    }
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      float da[32], gp[32];
      ld1(c, 0, c.part * per + gi * 32, da);
      if (gi == 0) {
        const bool ok = tc::mbar_wait(&c.wbar[0], c.uses[0] & 1u);
        c.uses[0] += 1;
        if (!ok) {
          if (lane == 0) atomicExch(p.status, tc2::kErrEpilogue);
          return;
        }
      }
      unstage32(F + gi * 2048, lane, gp);
#pragma unroll
      for (int i = 0; i < 32; ++i) da[i] *= gp[i];
      staging_free(lane);
      stage32(S, lane, da);
      staging_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mdH, S, col0 + gi * 32, y);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};

// Query rows -> out, key rows -> E (optional) and its a-/b-scaled copies, for a
// warp's 32 rows and its column groups; V of the key rows is prefetched.
// PAD: the chunk may be shorter than C (a last chunk with T % C != 0), so rows at
// or past its length are padding (compiled separately: the per-row masking
// slows the full-chunk epilogue measurably).
template <bool PAD, int BN>
__device__ __forceinline__ void out_or_residual(const FwdP& p, const EpiCtx<BN>& c, bool key_rows,
                                                int r0, bool write_e) {
  const Dims& d = p.d;
  const int lane = c.row & 31;
  const int per = BN / c.nparts;
  const int col0 = c.n0 + c.part * per;
  const int ngroups = per / 32;
  uint8_t* V = c.wsmem;            // [2][2 KB]: V of a pair of column groups
  uint8_t* S = c.wsmem + 4096;     // E | Ea | Eb staging
  const int ttok = c.t0 + r0;      // first token (within the head) of this warp's rows
  const int yrow = c.z * d.C + r0;
  const uint64_t keep = tc::l2_evict_last();    // E, aE, bE: read by the next phases
  const uint64_t stream = tc::l2_evict_first(); // out: never read again
  // Padding rows: no output, and E = a E = b E = 0, so they add nothing to any
  // later sum over tokens.
  const bool real = !PAD || lane < c.clen - r0;
  if (PAD && !key_rows && c.clen - r0 <= 0) return;  // no query row of this warp is real
  // V of key rows arrives by TMA, a pair of 32-column groups at a time
  auto load_pair = [&](int g0) {
    if (lane == 0) {
      const int n = ngroups - g0 < 2 ? ngroups - g0 : 2;
      tc::fence_async_smem();  // the previous pair's reads of V precede the refill
      tc::mbar_expect_tx(&c.wbar[0], 2048u * n);
      for (int j = 0; j < n; ++j)
        tc::tma_load_3d(V + j * 2048, &p.mV, &c.wbar[0], col0 + (g0 + j) * 32, ttok, c.z);
    }
    __syncwarp();
  };
  if (key_rows) load_pair(0);
  float at = 0.f, bt = 0.f;
  if (key_rows && real) {
    const size_t tok = (size_t)c.z * d.T + ttok + lane;
    at = p.ca[tok];
    bt = p.cb[tok];
  }
  for (int gi = 0; gi < ngroups; ++gi) {
    const int col = col0 + gi * 32;
    float y[32];
    ld1(c, 0, c.part * per + gi * 32, y);
    if (!key_rows) {
      staging_free(lane);
      stage32(S, lane, y);
      staging_ready();
      if (lane == 0) {
        tc::tma_store_3d_hint(&p.mOut, S, col, ttok, c.z, stream);
        tc::bulk_commit();
      }
      __syncwarp();
      continue;
    }
    if ((gi & 1) == 0) {
      if (gi > 0) load_pair(gi);
      const bool ok = tc::mbar_wait(&c.wbar[0], c.uses[0] & 1u);
      c.uses[0] += 1;
      if (!ok) {
        if (lane == 0) atomicExch(p.status, tc2::kErrEpilogue);
        return;
      }
    }
    float vv[32];
    unstage32(V + (gi & 1) * 2048, lane, vv);
#pragma unroll
    for (int i = 0; i < 32; ++i) y[i] = (PAD && !real) ? 0.f : d.loss == 0 ? y[i] - vv[i] : -vv[i];
    staging_free(lane);
    if (write_e) stage32(S, lane, y);
    if (!p.nomom) {
#pragma unroll
      for (int i = 0; i < 32; ++i) vv[i] = at * y[i];
      stage32(S + 2048, lane, vv);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) vv[i] = bt * y[i];
    stage32(S + 4096, lane, vv);
    staging_ready();
    if (lane == 0) {
      if (write_e) tc::tma_store_2d_hint(&p.mE, S, col, yrow, keep);
      if (!p.nomom) tc::tma_store_2d_hint(&p.mEa, S + 2048, col, yrow, keep);
      tc::tma_store_2d_hint(&p.mEb, S + 4096, col, yrow, keep);
      tc::bulk_commit();
    }
    __syncwarp();
  }
}

// G2, SwiGLU: rows [0, C) are queries (-> out), [C, 2C) keys (-> E). PAD: a
// shorter last chunk.
template <bool PAD>
struct EpiG2T {
  static constexpr int kSmem = 10240;  // V[2] | E | Ea | Eb
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const int r0 = c.m0 + c.quad * 32;
    const bool key_rows = c.m0 >= p.d.C;
    out_or_residual<PAD>(p, c, key_rows, key_rows ? r0 - p.d.C : r0, true);
  }
};
using EpiG2 = EpiG2T<false>;
using EpiG2Pad = EpiG2T<true>;

// G1, linear: class 0 = queries (-> out), class 1 = keys (-> scaled E).
template <bool PAD>
struct EpiG1LinT {
  static constexpr int kSmem = 10240;
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    out_or_residual<PAD>(p, c, c.cls == 1, c.m0 + c.quad * 32, false);
  }
};
using EpiG1Lin = EpiG1LinT<false>;
using EpiG1LinPad = EpiG1LinT<true>;

// G3, SwiGLU: dA -> dH1 = dA H3 silu'(H1), dH3 = dA silu(H1) (rows: tokens).
// The silu factors of a column group arrive by TMA in a 4 KB buffer; once read
// into registers, the same buffer stages that group's dH1 | dH3 for the TMA
// stores (each lane reads and then writes only its own row).
struct EpiG3 {
  static constexpr int kSmem = 8192;  // [2 groups][silu(H1) | H3 silu'(H1), then dH1 | dH3]
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;
    const int per = BN / c.nparts;
    const int col0 = c.n0 + c.part * per;
    const int ngroups = per / 32;
    const int y = c.z * d.C + r0;
    const uint64_t keep = tc::l2_evict_last();  // dH: read by the aggregation next
    uint8_t* F = c.wsmem;  // [group of the pair][s1 | s2] 2 KB each
    auto load_pair = [&](int g0) {
      if (lane == 0) {
        tc::bulk_wait_read<0>();  // earlier stores have read the buffers
        const int n = ngroups - g0 < 2 ? ngroups - g0 : 2;
        tc::mbar_expect_tx(&c.wbar[0], 4096u * n);
        for (int j = 0; j < n; ++j) {
          tc::tma_load_2d(F + j * 4096, &p.mSk, &c.wbar[0], col0 + (g0 + j) * 32, y);
          tc::tma_load_2d(F + j * 4096 + 2048, &p.mSk, &c.wbar[0], d.d_h + col0 + (g0 + j) * 32, y);
        }
      }
      __syncwarp();
    };
    load_pair(0);
    for (int gi = 0; gi < ngroups; ++gi) {
      float da[32], s1[32], s2[32];
      ld1(c, 0, c.part * per + gi * 32, da);
      if ((gi & 1) == 0) {
        if (gi > 0) load_pair(gi);
        const bool ok = tc::mbar_wait(&c.wbar[0], c.uses[0] & 1u);
        c.uses[0] += 1;
        if (!ok) {
          if (lane == 0) atomicExch(p.status, tc2::kErrEpilogue);
          return;
        }
      }
      uint8_t* G = F + (gi & 1) * 4096;
      unstage32(G, lane, s1);
      unstage32(G + 2048, lane, s2);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        s2[i] *= da[i];  // dH1
        s1[i] *= da[i];  // dH3
      }
      stage32(G, lane, s2);
      stage32(G + 2048, lane, s1);
      staging_ready();
      if (lane == 0) {
        tc::tma_store_2d_hint(&p.mdH, G, col0 + gi * 32, y, keep);
        tc::tma_store_2d_hint(&p.mdH, G + 2048, d.d_h + col0 + gi * 32, y, keep);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};

// G4: accumulator 0 = dM = sum_t a_t g_t, accumulator 1 = dW = sum_t b_t g_t.
// Class 0 covers rows of [W1; W3] (or W for linear), class 1 the rows of W2.
// Each of the four epilogue warps owns 32 rows x 128 columns of the tile and
// moves the fp32 state with TMA through two 10 KB slots of its shared memory, in
// one sequence of 32-column groups q that continues across the CTA's tiles: the
// W0/M0 tiles of group q + 2 load into group q's slot once its stores have read
// it, so they arrive while group q + 1 is computed (the first groups of the next
// tile load during the last groups of this one). Results are written back into
// the slot (W, M fp32 and the bf16 copy of W) and stored with TMA, so the state
// never passes through the load/store units. (Three slots, which would let a
// store's read overlap the next group's math, only fit beside a two-slot k-block
// ring, and the shallower ring costs more than they save.)
struct EpiG4 {
  static constexpr int kSlot = 10240;  // W 4 KB | M 4 KB | bf16 copy 2 KB
  static constexpr int kSlots = 2;
  static constexpr int kSmem = kSlots * kSlot;
  static __device__ __forceinline__ void issue(const FwdP& p, const uint8_t* wsmem, uint64_t* wbar,
                                               int q, int g, int cls, int z, int r0, int n0, int var) {
    const int sidx = q % kSlots;
    uint8_t* slot = const_cast<uint8_t*>(wsmem) + sidx * kSlot;
    const bool hasM = p.hasM[var];
    tc::mbar_expect_tx(&wbar[sidx], hasM ? 8192u : 4096u);
    tc::tma_load_3d(slot, &p.srcW[var][cls], &wbar[sidx], n0 + g * 32, r0, z);
    if (hasM) tc::tma_load_3d(slot + 4096, &p.srcM[var][cls], &wbar[sidx], n0 + g * 32, r0, z);
  }
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;  // first state row of this warp
    constexpr int kGroups = BN / 32;
    static_assert(kGroups >= 2, "two groups ahead");
    const int var = c.ci == 0 ? 0 : 1;
    const bool hasM = p.hasM[var];
    const size_t plane = (size_t)d.BH * d.NC;
    const size_t so = (size_t)c.z * d.NC + c.ci;
    const float PU = p.scal[so], PL = p.scal[plane + so], cc = p.scal[2 * plane + so];
    int sh_row;
    if (c.cls == 0 && d.kind == 1) {
      const int which = r0 / d.d_h, rr = r0 % d.d_h;
      sh_row = c.z * 2 * d.d_h + w13_row(rr, which);
    } else if (c.cls == 0 && d.kind == 2) {
      sh_row = c.z * d.d_h + r0;  // W1 of the GELU MLP, not interleaved
    } else {
      sh_row = c.z * d.d_v + r0;
    }
    const int q0 = c.seq * kGroups;
    if (!c.pre && lane == 0) {
      issue(p, c.wsmem, c.wbar, q0, 0, c.cls, c.z, r0, c.n0, var);
      issue(p, c.wsmem, c.wbar, q0 + 1, 1, c.cls, c.z, r0, c.n0, var);
    }
    __syncwarp();
    for (int g = 0; g < kGroups; ++g) {
      const int q = q0 + g, sidx = q % kSlots;
      uint8_t* slot = c.wsmem + sidx * kSlot;
      float dM[32], dW[32];
      ld2(c, 0, g * 32, 1, g * 32, dM, dW);
      const bool ok = tc::mbar_wait(&c.wbar[sidx], c.uses[sidx] & 1u);
      c.uses[sidx] += 1;
      if (!ok) {
        if (lane == 0) {
          atomicExch(p.status, tc2::kErrEpilogue);
          const int s1 = (q + 1) % kSlots;  // group q + 1's loads may still be in flight
          if (g + 1 < kGroups || c.nxt_valid) (void)tc::mbar_wait(&c.wbar[s1], c.uses[s1] & 1u);
        }
        return;
      }
      // row `lane` of the 128B-swizzled fp32 tiles; 64B-swizzled bf16 row
      uint8_t* wrow = slot + lane * 128;
      uint8_t* mrow = slot + 4096 + lane * 128;
      uint8_t* srow = slot + 8192 + lane * 64;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int off = (k ^ (lane & 7)) << 4;
        const float4 w = *reinterpret_cast<const float4*>(wrow + off);
        const float4 m = hasM ? *reinterpret_cast<const float4*>(mrow + off) : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 wn, mn;
        mn.x = PU * m.x - dM[4 * k + 0];
        mn.y = PU * m.y - dM[4 * k + 1];
        mn.z = PU * m.z - dM[4 * k + 2];
        mn.w = PU * m.w - dM[4 * k + 3];
        wn.x = PL * w.x + cc * m.x - dW[4 * k + 0];
        wn.y = PL * w.y + cc * m.y - dW[4 * k + 1];
        wn.z = PL * w.z + cc * m.z - dW[4 * k + 2];
        wn.w = PL * w.w + cc * m.w - dW[4 * k + 3];
        *reinterpret_cast<float4*>(wrow + off) = wn;
        *reinterpret_cast<float4*>(mrow + off) = mn;
        *reinterpret_cast<uint2*>(srow + ((((k >> 1) ^ ((lane >> 1) & 3)) << 4) | ((k & 1) << 3))) =
            make_uint2(pack2(wn.x, wn.y), pack2(wn.z, wn.w));
      }
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc::tma_store_3d(&p.dstW[c.cls], slot, c.n0 + g * 32, r0, c.z);
        tc::tma_store_3d(&p.dstM[c.cls], slot + 4096, c.n0 + g * 32, r0, c.z);
        if (c.wshadow)  // the next chunk's first phases read the bf16 copy at once
          tc::tma_store_2d_hint(&p.shadow[c.cls], slot + 8192, c.n0 + g * 32, sh_row, tc::l2_evict_last());
        tc::bulk_commit();
        tc::bulk_wait_read<0>();  // group q's stores have read the slot of group q + 2
        const int gn = g + 2;
        if (gn < kGroups) {
          issue(p, c.wsmem, c.wbar, q + 2, gn, c.cls, c.z, r0, c.n0, var);
        } else if (c.nxt_valid) {
          issue(p, c.wsmem, c.wbar, q + 2, gn - kGroups, c.nxt_cls, c.nxt_z,
                c.nxt_m0 + c.quad * 32, c.nxt_n0, c.nxt_ci == 0 ? 0 : 1);
        }
      }
      __syncwarp();
    }
  }
};

// G4 without momentum: one accumulator dW = sum_t b_t g_t and the update
// W_end = L(1,n) W0 - dW; the fp32 W (no M) moves through three 6 KB slots per
// warp in one sequence of 32-column groups across the CTA's tiles, as in EpiG4.
struct EpiG4W {
  static constexpr int kSlot = 6144;  // W 4 KB | bf16 copy 2 KB
  static constexpr int kSlots = 3;
  static constexpr int kSmem = kSlots * kSlot;
  static __device__ __forceinline__ void issue(const FwdP& p, const uint8_t* wsmem, uint64_t* wbar,
                                               int q, int g, int cls, int z, int r0, int n0, int var) {
    const int sidx = q % kSlots;
    uint8_t* slot = const_cast<uint8_t*>(wsmem) + sidx * kSlot;
    tc::mbar_expect_tx(&wbar[sidx], 4096u);
    tc::tma_load_3d(slot, &p.srcW[var][cls], &wbar[sidx], n0 + g * 32, r0, z);
  }
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;
    constexpr int kGroups = BN / 32;
    static_assert(kGroups >= 2, "two groups ahead");
    const size_t plane = (size_t)d.BH * d.NC;
    const float PL = p.scal[plane + (size_t)c.z * d.NC + c.ci];
    const int var = c.ci == 0 ? 0 : 1;
    int sh_row;
    if (c.cls == 0 && d.kind == 1) {
      const int which = r0 / d.d_h, rr = r0 % d.d_h;
      sh_row = c.z * 2 * d.d_h + w13_row(rr, which);
    } else if (c.cls == 0 && d.kind == 2) {
      sh_row = c.z * d.d_h + r0;  // W1 of the GELU MLP, not interleaved
    } else {
      sh_row = c.z * d.d_v + r0;
    }
    const int q0 = c.seq * kGroups;
    if (!c.pre && lane == 0) {
      issue(p, c.wsmem, c.wbar, q0, 0, c.cls, c.z, r0, c.n0, var);
      issue(p, c.wsmem, c.wbar, q0 + 1, 1, c.cls, c.z, r0, c.n0, var);
    }
    __syncwarp();
    for (int g = 0; g < kGroups; ++g) {
      const int q = q0 + g, sidx = q % kSlots;
      uint8_t* slot = c.wsmem + sidx * kSlot;
      float dW[32];
      ld1(c, 0, g * 32, dW);
      const bool ok = tc::mbar_wait(&c.wbar[sidx], c.uses[sidx] & 1u);
      c.uses[sidx] += 1;
      if (!ok) {
        if (lane == 0) atomicExch(p.status, tc2::kErrEpilogue);
        return;
      }
      uint8_t* wrow = slot + lane * 128;
      uint8_t* srow = slot + 4096 + lane * 64;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int off = (k ^ (lane & 7)) << 4;
        const float4 w = *reinterpret_cast<const float4*>(wrow + off);
        float4 wn;
        wn.x = PL * w.x - dW[4 * k + 0];
        wn.y = PL * w.y - dW[4 * k + 1];
        wn.z = PL * w.z - dW[4 * k + 2];
        wn.w = PL * w.w - dW[4 * k + 3];
        *reinterpret_cast<float4*>(wrow + off) = wn;
        *reinterpret_cast<uint2*>(srow + ((((k >> 1) ^ ((lane >> 1) & 3)) << 4) | ((k & 1) << 3))) =
            make_uint2(pack2(wn.x, wn.y), pack2(wn.z, wn.w));
      }
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc::tma_store_3d(&p.dstW[c.cls], slot, c.n0 + g * 32, r0, c.z);
        if (c.wshadow)
          tc::tma_store_2d_hint(&p.shadow[c.cls], slot + 4096, c.n0 + g * 32, sh_row, tc::l2_evict_last());
        tc::bulk_commit();
        tc::bulk_wait_read<1>();  // the slot of group q - 1 is free for group q + 2
        const int gn = g + 2;
        if (gn < kGroups) {
          issue(p, c.wsmem, c.wbar, q + 2, gn, c.cls, c.z, r0, c.n0, var);
        } else if (c.nxt_valid) {
          issue(p, c.wsmem, c.wbar, q + 2, gn - kGroups, c.nxt_cls, c.nxt_z,
                c.nxt_m0 + c.quad * 32, c.nxt_n0, c.nxt_ci == 0 ? 0 : 1);
        }
      }
      __syncwarp();
    }
  }
};

template <class Epi> struct EpiName;
template <> struct EpiName<EpiG1> { static constexpr const char* v = "tc_g1_h_act"; };
template <> struct EpiName<EpiG2> { static constexpr const char* v = "tc_g2_y_out_e"; };
template <> struct EpiName<EpiG2Pad> { static constexpr const char* v = "tc_g2_y_out_e"; };
template <> struct EpiName<EpiG3> { static constexpr const char* v = "tc_g3_da_dh"; };
template <> struct EpiName<EpiG4> { static constexpr const char* v = "tc_g4_aggregate_state"; };
template <> struct EpiName<EpiG4W> { static constexpr const char* v = "tc_g4_aggregate_w"; };
template <> struct EpiName<EpiG1Gelu> { static constexpr const char* v = "tc_g1_gelu"; };
template <> struct EpiName<EpiG3Gelu> { static constexpr const char* v = "tc_g3_gelu_dh"; };
template <> struct EpiName<EpiG1Lin> { static constexpr const char* v = "tc_g1_linear_out_e"; };
template <> struct EpiName<EpiG1LinPad> { static constexpr const char* v = "tc_g1_linear_out_e"; };

// ---------------------------------------------------------------- fused G1 + G2
// SwiGLU: one launch per chunk computes G1 and G2 together. A CTA takes a
// 128-row tile of [q; k] rows of one head and, per block of 128 hidden units j,
//   H_j = X [W1; W3]_j^T          (tensor memory, 256 columns: h1 | h3)
//   u_j = silu(h1) h3             (epilogue warps -> shared memory, bf16, laid
//                                  out as the K-major operand of the next MMA)
//   Y  += u_j W2_j^T              (tensor memory, d_v columns)
// and after the last block turns Y into out (query rows) or E, aE, bE (key
// rows). The query rows' u never leaves the chip; the key rows' u (for the W2
// aggregation) and their silu factors (for G3) are written once. The MMA of
// H_{j+1} starts as soon as the epilogue has read H_j into registers, so the
// silu math of block j overlaps it; Y_j is issued after H_{j+1}. Each u value
// and each Y element is computed with the same operations in the same order as
// by G1 then G2, so the results are the same bit for bit.
// Named barrier of the eight epilogue warps (warps 2..9) of the fused and the
// persistent kernels.
__device__ __forceinline__ void epi_barrier() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

namespace ff {
constexpr int kStages = 3;
constexpr uint32_t kStage = 49152;   // X k-block 16 KB + W13 k-block 32 KB, or a W2 k-block
constexpr int kEW = 8;
constexpr uint32_t kU = 32768;       // u of one block: 128 rows x 128 units, two 64-column tiles
constexpr uint32_t kEpi = 81920;     // [u buffer 0 | u buffer 1 | 16 KB]: 8 x 10 KB of staging at the end
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStage + kEpi + 1024;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(EpiG2::kSmem <= (int)(kEpi / kEW), "the Y epilogue's staging fits");
}  // namespace ff

struct FfJob {
  CUtensorMap mX[2];  // query rows, key rows: [BH T, d_k], box 64 x 128
  CUtensorMap mW13;   // interleaved [W1; W3] copy: [BH 2 d_h, d_k], box 64 x 256
  CUtensorMap mW2;    // W2 copy: [BH d_v, d_h], box 64 x d_v
  CUtensorMap mU;     // A = [u_q; u_k] per head: [BH 2C, d_h], box 64 x 32 (128B swizzle)
  int mtiles;         // 128-row tiles per head and row class: C / 128
  int nblk, kbh;      // hidden blocks (d_h / 128), k-blocks of H (d_k / 64)
  int total;          // tiles: BH x 2 x mtiles (key-row tiles first)
  int* status;
  int ci, t0, clen;
  int stall;          // failure-detection test hook, as in tc2::Job
  unsigned long long wait_ns;
};

// The fused kernel's final epilogue (Y -> out, or E, aE, bE), kept out of line
// so that its registers and those of the H epilogue are not live together.
template <int DV>
__device__ __noinline__ void ff_y_epilogue(const FwdP& p, const tc2::EpiCtx<DV>& c, bool key_rows,
                                           int r0, int pad) {
  if (pad) out_or_residual<true, DV>(p, c, key_rows, r0, true);
  else out_or_residual<false, DV>(p, c, key_rows, r0, true);
}

template <int DV>
__global__ void __launch_bounds__((2 + ff::kEW) * 32, 1)
ff12_kernel(const __grid_constant__ FfJob J, const __grid_constant__ FwdP prm) {
  using namespace ff;
  constexpr uint32_t kW2Bytes = (uint32_t)DV * 128;  // one W2 k-block: DV rows x 64 bf16
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* epi = smem + (size_t)kStages * kStage;  // u buffers, then Y-epilogue staging
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ uint64_t h_full, h_empty, u_full[2], u_empty[2], y_full, y_empty;
  __shared__ uint64_t epi_bar[tc2::kEpiBars * kEW];
  __shared__ uint64_t never;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_err_;
  volatile int& s_err = s_err_;
  const unsigned long long lim = J.wait_ns ? J.wait_ns : tc::kWaitNs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = prm.d;
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    s_err = 0;
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(&h_full, 1);
    tc::mbar_init(&h_empty, kEW);
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&u_full[b], kEW);
      tc::mbar_init(&u_empty[b], 1);
    }
    tc::mbar_init(&y_full, 1);
    tc::mbar_init(&y_empty, kEW);
    for (int w = 0; w < tc2::kEpiBars * kEW; ++w) tc::mbar_init(&epi_bar[w], 1);
    tc::mbar_init(&never, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&J.mX[0]);
    tc::prefetch_tmap(&J.mX[1]);
    tc::prefetch_tmap(&J.mW13);
    tc::prefetch_tmap(&J.mW2);
  }
  if (warp == 1) {
    tc::tmem_alloc(&tmem_slot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;  // H at columns [0, 256), Y at [256, 256 + DV)
  griddep_wait();
  const int per_class = J.total / 2;
  auto decode = [&](int t, int& cls, int& z, int& mt) {
    cls = t < per_class ? 1 : 0;  // key-row tiles first (their epilogues do more)
    const int r = cls ? t : t - per_class;
    z = r / J.mtiles;
    mt = r - z * J.mtiles;
  };
  int mma_done = 0;

  if (warp == 0 && lane == 0) {
    // ---------------- producer: per tile, the H k-blocks of block j, then W2 of block j - 1
    int it = 0;
    bool ok = true;
    auto stage = [&](uint32_t bytes) -> uint8_t* {
      const int s = it % kStages;
      const uint32_t ph = (uint32_t)(it / kStages) & 1u;
      if (it >= kStages && !tc::mbar_wait_hint(&empty[s], ph ^ 1u, lim)) {
        atomicExch(J.status, tc2::kErrProducer);
        s_err = 1;
        ok = false;
        return nullptr;
      }
      tc::mbar_expect_tx(&full[s], bytes);
      return ring + (size_t)s * kStage;
    };
    for (int t = blockIdx.x; t < J.total && ok; t += gridDim.x) {
      int cls, z, mt;
      decode(t, cls, z, mt);
      const int xrow = z * d.T + J.t0 + mt * 128;
      auto w2 = [&](int jj) {
        for (int kb = 0; kb < 2 && ok; ++kb) {
          uint8_t* st = stage(kW2Bytes);
          if (!st) break;
          tc::tma_load_2d(st, &J.mW2, &full[it % kStages], jj * 128 + kb * 64, z * DV);
          ++it;
        }
      };
      for (int j = 0; j < J.nblk && ok; ++j) {
        for (int kb = 0; kb < J.kbh && ok; ++kb) {
          uint8_t* st = stage(49152u);
          if (!st) break;
          tc::tma_load_2d(st, &J.mX[cls], &full[it % kStages], kb * 64, xrow);
          tc::tma_load_2d(st + 16384, &J.mW13, &full[it % kStages], kb * 64, z * 2 * d.d_h + j * 256);
          ++it;
        }
        if (j >= 1) w2(j - 1);
      }
      if (ok) w2(J.nblk - 1);
    }
    for (int j = it - kStages < 0 ? 0 : it - kStages; j < it; ++j)
      (void)tc::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, lim);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint64_t dR = tc2::sdesc(tc::smem_u32(ring), false);
    const uint64_t dU = tc2::sdesc(tc::smem_u32(epi), false);
    constexpr uint32_t idH = tc2::idesc(128, 256, false, false);
    constexpr uint32_t idY = tc2::idesc(128, DV, false, false);
    int it = 0, gb = 0, ti = 0;
    bool ok = !(J.stall && blockIdx.x == 0 && !tc::mbar_wait(&never, 0u, lim));
    if (!ok) {
      atomicExch(J.status, tc2::kErrMma);
      s_err = 1;
    }
    auto take = [&]() -> uint32_t {  // the next ring stage, filled; returns its offset >> 4
      const int s = it % kStages;
      const uint32_t ph = (uint32_t)(it / kStages) & 1u;
      if (!tc::mbar_wait_hint(&full[s], ph, lim)) {
        atomicExch(J.status, tc2::kErrMma);
        s_err = 1;
        ok = false;
        return 0;
      }
      tc::tc_fence_after();
      return ((uint32_t)s * kStage) >> 4;
    };
    auto release = [&]() {
      tc::mma_commit(&empty[it % kStages]);
      ++it;
    };
    auto issue_y = [&](int jj) {  // Y += u_jj W2_jj^T
      const int g = gb + jj, b = g & 1;
      if (!tc::mbar_wait(&u_full[b], (uint32_t)(g >> 1) & 1u, lim) ||
          (jj == 0 && !tc::mbar_wait(&y_empty, ((uint32_t)ti & 1u) ^ 1u, lim))) {
        atomicExch(J.status, tc2::kErrMma);
        s_err = 1;
        ok = false;
        return;
      }
      tc::tc_fence_after();
      for (int kb = 0; kb < 2 && ok; ++kb) {
        const uint32_t so = take();
        if (!ok) break;
        const uint32_t uo = ((uint32_t)b * kU + (uint32_t)kb * 16384) >> 4;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_bf16(tmem + 256, dU + (uo + k * 2), dR + (so + k * 2), idY, (jj | kb | k) != 0);
        release();
      }
      tc::mma_commit(&u_empty[b]);
    };
    for (int t = blockIdx.x; t < J.total && ok; t += gridDim.x, ++ti) {
      for (int j = 0; j < J.nblk && ok; ++j) {
        if (!tc::mbar_wait(&h_empty, ((uint32_t)(gb + j) & 1u) ^ 1u, lim)) {
          atomicExch(J.status, tc2::kErrMma);
          s_err = 1;
          ok = false;
          break;
        }
        tc::tc_fence_after();
        for (int kb = 0; kb < J.kbh && ok; ++kb) {
          const uint32_t so = take();
          if (!ok) break;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16(tmem, dR + (so + k * 2), dR + (so + (16384 >> 4) + k * 2), idH, (kb | k) != 0);
          release();
        }
        tc::mma_commit(&h_full);
        if (j >= 1 && ok) issue_y(j - 1);
      }
      if (ok) issue_y(J.nblk - 1);
      if (ok) {
        tc::mma_commit(&y_full);
        ++mma_done;
      }
      gb += J.nblk;
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: every warp runs the same barriers on every tile,
    // also after a failure (it then skips the work)
    const int ew = warp - 2, quad = warp & 3, part = ew >> 2;
    const int row = quad * 32 + lane;  // TMEM lane = row of the tile
    const uint32_t tl = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t uses[tc2::kEpiBars] = {0u, 0u, 0u, 0u};
    int gb = 0, ti = 0;
    for (int t = blockIdx.x; t < J.total; t += gridDim.x, ++ti) {
      int cls, z, mt;
      decode(t, cls, z, mt);
      const int r0 = mt * 128 + quad * 32;  // first row (within the chunk) of this warp
      // the previous tile's staged stores have read the epilogue region
      if (lane == 0) tc::bulk_wait_read<0>();
      __syncwarp();
      epi_barrier();
      for (int j = 0; j < J.nblk; ++j) {
        const int g = gb + j, b = g & 1;
        bool ok = !s_err;
        if (ok && !tc::mbar_wait(&h_full, (uint32_t)g & 1u, lim)) {
          if (lane == 0) atomicExch(J.status, tc2::kErrEpilogue);
          s_err = 1;
          ok = false;
        }
        tc::tc_fence_after();
        // buffer b is free once the MMA of its previous use and our store of it are done
        if (ok && !tc::mbar_wait(&u_empty[b], ((uint32_t)(g >> 1) & 1u) ^ 1u, lim)) {
          if (lane == 0) atomicExch(J.status, tc2::kErrEpilogue);
          s_err = 1;
          ok = false;
        }
        if (ok && lane == 0) tc::bulk_wait_read<0>();
        __syncwarp();
        uint8_t* ut = epi + (size_t)b * kU + (size_t)part * 16384;  // this warp's 64-column tile
        uint8_t* urow = ut + row * 128;
        bf16* sk = prm.Sk + ((size_t)z * d.C + r0 + lane) * (2 * d.d_h) + j * 128 + part * 64;
        // u (and for key rows the silu factors s1 = silu(h1), s2 = h3 silu'(h1)),
        // formed exactly as G1's epilogue forms them, in two halves of 32 units:
        // H is released for the next block's MMA once the second half is read
        for (int half = 0; half < 2; ++half) {
          float h1[32], h3[32];
          if (ok) {
            const int cs = part * 64 + half * 32;
            uint32_t a[32], c3[32];
            tmem_ld32_nowait(tl + (uint32_t)cs, a);
            tmem_ld32_nowait(tl + (uint32_t)(128 + cs), c3);
            tmem_wait_ld2(a, c3);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              h1[i] = __uint_as_float(a[i]);
              h3[i] = __uint_as_float(c3[i]);
            }
          }
          if (half == 1) {
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc2::mbar_arrive(&h_empty);  // the next block's MMA may overwrite H
          }
          if (!ok) continue;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = half * 4 + kk;
            float uu[8], f1[8], f2[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float x1 = h1[8 * kk + i], x3 = h3[8 * kk + i];
              if (cls == 0) {
                uu[i] = x1 * fast_sigmoid(x1) * x3;
              } else {
                const float sg = fast_sigmoid(x1);
                const float s1 = x1 * sg;
                f2[i] = x3 * sg * (1.0f + x1 * (1.0f - sg));
                uu[i] = s1 * x3;
                f1[i] = s1;
              }
            }
            *reinterpret_cast<uint4*>(urow + ((k ^ (row & 7)) << 4)) =
                make_uint4(pack2(uu[0], uu[1]), pack2(uu[2], uu[3]), pack2(uu[4], uu[5]), pack2(uu[6], uu[7]));
            if (cls == 1) {
              reinterpret_cast<uint4*>(sk)[k] =
                  make_uint4(pack2(f1[0], f1[1]), pack2(f1[2], f1[3]), pack2(f1[4], f1[5]), pack2(f1[6], f1[7]));
              reinterpret_cast<uint4*>(sk + d.d_h)[k] =
                  make_uint4(pack2(f2[0], f2[1]), pack2(f2[2], f2[3]), pack2(f2[4], f2[5]), pack2(f2[6], f2[7]));
            }
          }
        }
        tc::fence_async_smem();  // the MMA (async proxy) reads what the threads wrote
        __syncwarp();
        if (lane == 0) tc2::mbar_arrive(&u_full[b]);
        if (ok && cls == 1 && lane == 0) {
          // key rows: u for the W2 aggregation (TMA store of this warp's 32 x 64 block)
          tc::tma_store_2d_hint(&J.mU, ut + quad * 32 * 128, j * 128 + part * 64,
                                z * 2 * d.C + d.C + r0, tc::l2_evict_last());
          tc::bulk_commit();
        }
        __syncwarp();
      }
      gb += J.nblk;
      // Y -> out (query rows) or E, aE, bE (key rows), staged through the epilogue
      // region once every warp's u stores have read it
      bool ok = !s_err;
      if (ok && !tc::mbar_wait(&y_full, (uint32_t)ti & 1u, lim)) {
        if (lane == 0) atomicExch(J.status, tc2::kErrEpilogue);
        s_err = 1;
        ok = false;
      }
      tc::tc_fence_after();
      if (lane == 0) tc::bulk_wait_read<0>();
      __syncwarp();
      epi_barrier();
      if (ok) {
        tc2::EpiCtx<DV> c;
        c.cls = cls;
        c.z = z;
        c.m0 = mt * 128;
        c.n0 = 0;
        c.row = row;
        c.quad = quad;
        c.part = part;
        c.nparts = 2;
        c.taddr = tl + 256u;
        c.wsmem = epi + (size_t)ew * (kEpi / kEW);
        c.wbar = epi_bar + tc2::kEpiBars * ew;
        c.uses = uses;
        c.slot = 0;
        c.iter = ti;
        c.seq = ti;
        c.pre = 0;
        c.ci = J.ci;
        c.t0 = J.t0;
        c.clen = J.clen;
        c.wshadow = 0;
        c.nxt_valid = 0;
        c.nxt_cls = c.nxt_z = c.nxt_m0 = c.nxt_n0 = c.nxt_ci = 0;
        ff_y_epilogue<DV>(prm, c, cls == 1, r0, J.clen < d.C);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc2::mbar_arrive(&y_empty);
    }
    if (lane == 0) tc::bulk_wait_all();
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && mma_done > 0) (void)tc::mbar_wait(&y_full, (uint32_t)(mma_done - 1) & 1u, lim);
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- persistent forward
// The whole SwiGLU forward (every chunk, G1 to G4) in one cooperative launch.
// Each CTA (one per SM) walks a static list of the tiles of all four GEMM phases
// of all chunks: chunk by chunk, and inside a chunk group by group of hg heads,
// phase after phase within a group. A tile of phase p for head z and chunk ci
// may start once the tiles its inputs come from are done: G1 after every G4
// tile of (z, ci - 1) (the bf16 copy of the chunk-start weights, and no reader of
// the previous chunk's scratch is left), G2 after G1 of (z, ci), G3 after G2, G4
// after G3. Completed tiles are counted per (phase, head) in global counters
// (release increments after the tile's stores have completed; bounded acquire
// spins before the first read of a tile's inputs). Dependencies only point to
// earlier tiles of the list, and every CTA is resident (cooperative launch), so
// the earliest unfinished tile can always run. Heads of a later group (or a
// later chunk) run while an earlier group aggregates: the HBM-bound state
// epilogue of G4 overlaps the tensor-core phases of other heads, and no kernel
// boundary separates the phases.
//
// One configuration serves the four phases: a ring of three 48 KB stages (G1:
// A 16 KB + B 32 KB; G4: three 16 KB operand tiles; G2, G3: 32 KB), two TMEM
// accumulator sets of 256 columns (G1: one 128 x 256 accumulator; G4: two 128 x
// 128; G2, G3: one 128 x 128), eight epilogue warps of 10 KB (G4: four warps of
// 20 KB, the other four idle for its tiles).
namespace mk {
constexpr int kStages = 3;
constexpr uint32_t kSlot = 49152;
constexpr int kEW = 8;
constexpr int kEpiSmem = 10240;
constexpr int kEpiSmemG4 = 20480;
constexpr uint32_t kAcc = 256;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kSlot + (size_t)kEW * kEpiSmem + 1024;
static_assert(EpiG1::kSmem <= kEpiSmem && EpiG2::kSmem <= kEpiSmem && EpiG3::kSmem <= kEpiSmem,
              "epilogue buffers of G1-G3 fit the 10 KB per warp");
static_assert(4 * kEpiSmemG4 <= kEW * kEpiSmem && EpiG4::kSmem <= kEpiSmemG4, "G4 epilogue buffers fit");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
enum : int { kErrDep = 4 };
}  // namespace mk

struct MegaJob {
  tc2::Job ph[4];   // maps and tile classes of G1..G4 (y_base of every operand 0)
  int tph[4];       // tiles per head of each phase
  int BH, NC, C, hg;
  int per_group;    // tiles of one group of hg heads in one chunk (all phases)
  int per_chunk;    // tiles of one chunk
  int total;        // tiles of the call
  int* cnt;         // [4][BH] completed tiles per (phase, head), zero at launch
  int* status;
  unsigned long long wait_ns;
  int stall;        // failure-detection test hook, as in tc2::Job
};

struct MkTile {
  int ph, ci, z, cls, mt, nt;
};

__device__ __forceinline__ MkTile mk_decode(const MegaJob& J, int t) {
  MkTile r;
  r.ci = t / J.per_chunk;
  int x = t - r.ci * J.per_chunk;
  const int g = x / J.per_group;
  x -= g * J.per_group;
  r.ph = 0;
  while (r.ph < 3 && x >= J.hg * J.tph[r.ph]) {
    x -= J.hg * J.tph[r.ph];
    ++r.ph;
  }
  const tc2::Job& P = J.ph[r.ph];
  r.cls = 0;
  const int per0 = P.cls[0].tiles_m * P.cls[0].tiles_n * J.hg;
  if (P.n_cls > 1 && x >= per0) {
    x -= per0;
    r.cls = 1;
  }
  const tc2::Class& K = P.cls[r.cls];
  const int per_head = K.tiles_m * K.tiles_n;
  const int zl = x / per_head;
  x -= zl * per_head;
  r.z = g * J.hg + zl;
  r.mt = x / K.tiles_n;
  r.nt = x - r.mt * K.tiles_n;
  return r;
}
// Completed tiles of the producing phase that tile T needs (dphase < 0: none).
__device__ __forceinline__ void mk_need(const MegaJob& J, const MkTile& T, int& dphase, int& target) {
  if (T.ph == 0) {
    dphase = T.ci > 0 ? 3 : -1;
    target = T.ci * J.tph[3];
  } else {
    dphase = T.ph - 1;
    target = (T.ci + 1) * J.tph[T.ph - 1];
  }
}
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Bounded wait until the tile's inputs are complete; then order the async-proxy
// (TMA) reads that follow after the acquire.
__device__ __forceinline__ bool mk_dep_wait(const MegaJob& J, const MkTile& T, unsigned long long lim) {
  int dp, tg;
  mk_need(J, T, dp, tg);
  if (dp >= 0) {
    const int* c = J.cnt + (size_t)dp * J.BH + T.z;
    if (ld_acquire(c) < tg) {
      const unsigned long long t0 = tc::globaltimer();
      for (uint32_t i = 1;; ++i) {
        __nanosleep(64);
        if (ld_acquire(c) >= tg) break;
        if ((i & 15) == 0 && tc::globaltimer() - t0 > lim) return false;
      }
    }
  }
  fence_proxy_async_global();
  return true;
}
__device__ __forceinline__ bool mk_dep_ready(const MegaJob& J, const MkTile& T) {
  int dp, tg;
  mk_need(J, T, dp, tg);
  return dp < 0 || ld_acquire(J.cnt + (size_t)dp * J.BH + T.z) >= tg;
}

template <bool MN, int ROWS>
__device__ __forceinline__ void mk_load(uint8_t* dst, const CUtensorMap* map, uint64_t* bar,
                                        const tc2::Opnd& o, int yoff, int z, int origin, int kb) {
  tc2::Opnd q = o;
  q.y_base += yoff;
  tc2::load_opnd<MN, ROWS>(dst, map, bar, q, z, origin, kb);
}

__global__ void __launch_bounds__((2 + mk::kEW) * 32, 1)
fwd_persistent(const __grid_constant__ MegaJob J, const __grid_constant__ FwdP prm) {
  using namespace mk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* epi_smem = smem + (size_t)kStages * kSlot;
  __shared__ uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2];
  __shared__ uint64_t epi_bar[tc2::kEpiBars * kEW];
  __shared__ uint64_t never;  // the stall hook's mbarrier: nothing ever arrives on it
  __shared__ uint32_t tmem_slot;
  __shared__ int s_err_;
  volatile int& s_err = s_err_;  // set by any role on failure, read by all
  const unsigned long long lim = J.wait_ns ? J.wait_ns : tc::kWaitNs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    s_err = 0;
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], kEW);
    }
    for (int w = 0; w < tc2::kEpiBars * kEW; ++w) tc::mbar_init(&epi_bar[w], 1);
    tc::mbar_init(&never, 1);
    tc::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < 4; ++p) {
      tc::prefetch_tmap(&J.ph[p].maps[0].op0);
      tc::prefetch_tmap(&J.ph[p].maps[0].op2);
    }
  }
  if (warp == 1) {
    tc::tmem_alloc(&tmem_slot, 2 * kAcc);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  int mma_tiles = 0;

  if (warp == 0 && lane == 0) {
    // ---------------- producer
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < J.total && ok; t += gridDim.x) {
      const MkTile T = mk_decode(J, t);
      if (!mk_dep_wait(J, T, lim)) {
        atomicExch(J.status, kErrDep);
        s_err = 1;
        break;
      }
      const tc2::Job& P = J.ph[T.ph];
      const tc2::Class& K = P.cls[T.cls];
      const tc2::Maps& M = P.maps[T.cls];
      const int aoff = T.ph == 0 ? T.ci * J.C : 0;                // query / key rows of the chunk
      const int boff = (T.ph == 3 && T.cls == 0) ? T.ci * J.C : 0;  // key rows (K dim) of the chunk
      const uint32_t bytes = (T.ph == 1 || T.ph == 2) ? 32768u : 49152u;
      for (int kb = 0; kb < K.kblocks; ++kb, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (it >= kStages && !tc::mbar_wait_hint(&empty[s], ph ^ 1u, lim)) {
          atomicExch(J.status, tc2::kErrProducer);
          s_err = 1;
          ok = false;
          break;
        }
        uint8_t* st = ring + (size_t)s * kSlot;
        tc::mbar_expect_tx(&full[s], bytes);
        const int m0 = T.mt * tc::BM;
        switch (T.ph) {
          case 0:  // [q; k] rows x [W1; W3] (interleaved), both K-major, N = 256
            mk_load<false, 128>(st, &M.op0, &full[s], K.a, aoff, T.z, m0, kb);
            mk_load<false, 256>(st + 16384, &M.op2, &full[s], K.b, 0, T.z, T.nt * 256, kb);
            break;
          case 1:  // A = [u_q; u_k], B = W2, K-major, N = 128
            mk_load<false, 128>(st, &M.op0, &full[s], K.a, 0, T.z, m0, kb);
            mk_load<false, 128>(st + 16384, &M.op2, &full[s], K.b, 0, T.z, T.nt * 128, kb);
            break;
          case 2:  // A = E (K-major), B = W2 read MN-major, N = 128
            mk_load<false, 128>(st, &M.op0, &full[s], K.a, 0, T.z, m0, kb);
            mk_load<true, 128>(st + 16384, &M.op2, &full[s], K.b, 0, T.z, T.nt * 128, kb);
            break;
          default:  // the two aggregations, all operands MN-major
            if (K.mode == tc2::kModeA2B1) {
              mk_load<true, 128>(st, &M.op0, &full[s], K.a, 0, T.z, m0, kb);
              mk_load<true, 128>(st + 16384, &M.op1, &full[s], K.a, 0, T.z, m0, kb);
              mk_load<true, 128>(st + 32768, &M.op2, &full[s], K.b, boff, T.z, T.nt * 128, kb);
            } else {
              mk_load<true, 128>(st, &M.op0, &full[s], K.a, 0, T.z, m0, kb);
              mk_load<true, 128>(st + 16384, &M.op1, &full[s], K.b, boff, T.z, T.nt * 128, kb);
              mk_load<true, 128>(st + 32768, &M.op2, &full[s], K.b, boff, T.z, T.nt * 128, kb);
            }
            break;
        }
      }
    }
    for (int j = it - kStages < 0 ? 0 : it - kStages; j < it; ++j)
      (void)tc::mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, lim);
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint64_t dK = tc2::sdesc(tc::smem_u32(ring), false);
    const uint64_t dN = tc2::sdesc(tc::smem_u32(ring), true);
    constexpr uint32_t kA = 16384 >> 4, kB2 = 32768 >> 4;
    int it = 0, i = 0;
    bool ok = true;
    if (J.stall && blockIdx.x == 0 && !tc::mbar_wait(&never, 0u, lim)) {
      atomicExch(J.status, tc2::kErrMma);
      s_err = 1;
      ok = false;
    }
    for (int t = blockIdx.x; t < J.total && ok; t += gridDim.x, ++i) {
      const MkTile T = mk_decode(J, t);
      const tc2::Class& K = J.ph[T.ph].cls[T.cls];
      const int b = i & 1;
      if (!tc::mbar_wait(&acc_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, lim)) {
        atomicExch(J.status, tc2::kErrMma);
        s_err = 1;
        break;
      }
      tc::tc_fence_after();
      const uint32_t acc = tmem + (uint32_t)(b * kAcc);
      for (int kb = 0; kb < K.kblocks; ++kb, ++it) {
        const int s = it % kStages;
        const uint32_t ph = (uint32_t)(it / kStages) & 1u;
        if (!tc::mbar_wait_hint(&full[s], ph, lim)) {
          atomicExch(J.status, tc2::kErrMma);
          s_err = 1;
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t so = ((uint32_t)s * kSlot) >> 4;
#pragma unroll
        for (int k = 0; k < tc::BK / 16; ++k) {
          const uint32_t accum = (kb | k) != 0;
          switch (T.ph) {
            case 0:
              tc::mma_bf16(acc, dK + (so + k * 2), dK + (so + kA + k * 2), tc2::idesc(128, 256, false, false), accum);
              break;
            case 1:
              tc::mma_bf16(acc, dK + (so + k * 2), dK + (so + kA + k * 2), tc2::idesc(128, 128, false, false), accum);
              break;
            case 2:
              tc::mma_bf16(acc, dK + (so + k * 2), dN + (so + kA + k * 128), tc2::idesc(128, 128, false, true), accum);
              break;
            default: {
              constexpr uint32_t id = tc2::idesc(128, 128, true, true);
              if (K.mode == tc2::kModeA2B1) {
                const uint64_t bd = dN + (so + kB2 + k * 128);
                tc::mma_bf16(acc, dN + (so + k * 128), bd, id, accum);
                tc::mma_bf16(acc + 128, dN + (so + kA + k * 128), bd, id, accum);
              } else {
                const uint64_t ad = dN + (so + k * 128);
                tc::mma_bf16(acc, ad, dN + (so + kA + k * 128), id, accum);
                tc::mma_bf16(acc + 128, ad, dN + (so + kB2 + k * 128), id, accum);
              }
              break;
            }
          }
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(&acc_full[b]);
      ++mma_tiles;
    }
  } else if (warp >= 2) {
    // ---------------- epilogue
    // Every epilogue warp runs the same number of iterations and named barriers,
    // also after a failure (then it only skips the work), so no warp can wait
    // at the barrier for one that left.
    const int ew = warp - 2;
    const int quad = warp & 3;
    uint32_t uses[tc2::kEpiBars] = {0u, 0u, 0u, 0u};
    int seq4 = 0;    // G4 tiles this warp has finished
    int pre4 = 0;    // the previous G4 tile issued this one's first state loads
    int i = 0;
    for (int t = blockIdx.x; t < J.total; t += gridDim.x, ++i) {
      const MkTile T = mk_decode(J, t);
      const int b = i & 1;
      bool ok = !s_err;
      if (ok && !tc::mbar_wait(&acc_full[b], (uint32_t)(i >> 1) & 1u, lim)) {
        if (lane == 0) atomicExch(J.status, tc2::kErrEpilogue);
        s_err = 1;
        ok = false;
      }
      tc::tc_fence_after();
      if (ok) {
        int dep_ok = 1;
        if (lane == 0) dep_ok = mk_dep_wait(J, T, lim) ? 1 : 0;  // satisfied already: the producer waited
        dep_ok = __shfl_sync(0xffffffffu, dep_ok, 0);
        if (!dep_ok) {
          if (lane == 0) atomicExch(J.status, kErrDep);
          s_err = 1;
          ok = false;
        }
      }
      const int chunk_t0 = T.ci * J.C;
      const int clen = T.ci == J.NC - 1 ? prm.d.T - chunk_t0 : J.C;
      if (ok) {
        auto fill = [&](auto& c, int nparts, int part, uint8_t* ws) {
          c.cls = T.cls;
          c.z = T.z;
          c.m0 = T.mt * tc::BM;
          c.row = quad * 32 + lane;
          c.quad = quad;
          c.nparts = nparts;
          c.part = part;
          c.taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * kAcc);
          c.wsmem = ws;
          c.wbar = epi_bar + tc2::kEpiBars * ew;
          c.uses = uses;
          c.slot = i & 1;
          c.iter = i;
          c.seq = i;
          c.pre = 0;
          c.ci = T.ci;
          c.t0 = chunk_t0;
          c.clen = clen;
          c.wshadow = T.ci + 1 < J.NC;
          c.nxt_valid = 0;
          c.nxt_cls = c.nxt_z = c.nxt_m0 = c.nxt_n0 = c.nxt_ci = 0;
        };
        switch (T.ph) {
          case 0: {
            tc2::EpiCtx<256> c;
            fill(c, 2, ew >> 2, epi_smem + (size_t)ew * kEpiSmem);
            c.n0 = T.nt * 256;
            EpiG1::run(prm, c);
            break;
          }
          case 1: {
            tc2::EpiCtx<128> c;
            fill(c, 2, ew >> 2, epi_smem + (size_t)ew * kEpiSmem);
            c.n0 = T.nt * 128;
            if (clen < J.C) EpiG2Pad::run(prm, c);
            else EpiG2::run(prm, c);
            break;
          }
          case 2: {
            tc2::EpiCtx<128> c;
            fill(c, 2, ew >> 2, epi_smem + (size_t)ew * kEpiSmem);
            c.n0 = T.nt * 128;
            EpiG3::run(prm, c);
            break;
          }
          default:
            if (ew < 4) {
              tc2::EpiCtx<128> c;
              fill(c, 1, 0, epi_smem + (size_t)ew * kEpiSmemG4);
              c.n0 = T.nt * 128;
              c.seq = seq4;
              c.pre = pre4;
              // the CTA's next tile: its first state groups load during this
              // tile's last groups if it is a G4 tile whose inputs are complete
              int nv = 0, ncls = 0, nz = 0, nmt = 0, nnt = 0, nci = 0;
              const int tn = t + (int)gridDim.x;
              if (lane == 0 && tn < J.total) {
                const MkTile N = mk_decode(J, tn);
                nv = N.ph == 3 && mk_dep_ready(J, N);
                if (nv) fence_proxy_async_global();
                ncls = N.cls; nz = N.z; nmt = N.mt; nnt = N.nt; nci = N.ci;
              }
              nv = __shfl_sync(0xffffffffu, nv, 0);
              if (nv) {
                c.nxt_valid = 1;
                c.nxt_cls = __shfl_sync(0xffffffffu, ncls, 0);
                c.nxt_z = __shfl_sync(0xffffffffu, nz, 0);
                c.nxt_m0 = __shfl_sync(0xffffffffu, nmt, 0) * tc::BM;
                c.nxt_n0 = __shfl_sync(0xffffffffu, nnt, 0) * 128;
                c.nxt_ci = __shfl_sync(0xffffffffu, nci, 0);
              }
              EpiG4::run(prm, c);
              seq4 += 1;
              pre4 = nv;
            }
            break;
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc2::mbar_arrive(&acc_empty[b]);
        tc::bulk_wait_all();             // this warp's stores of the tile have completed
        fence_proxy_async_global();
      }
      __syncwarp();
      epi_barrier();                     // ... and those of every epilogue warp
      if (ew == 0 && lane == 0 && ok && !s_err) {
        __threadfence();
        asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(J.cnt + (size_t)T.ph * J.BH + T.z)
                     : "memory");
      }
    }
    // a G4 tile that prefetched for a next one that never ran (after a failure):
    // its two state loads must land before the CTA exits
    if (pre4 && lane == 0) {
      (void)tc::mbar_wait(&epi_bar[tc2::kEpiBars * ew + 0], uses[0] & 1u, lim);
      (void)tc::mbar_wait(&epi_bar[tc2::kEpiBars * ew + 1], uses[1] & 1u, lim);
    }
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && mma_tiles > 0) {
      const int last = mma_tiles - 1;
      (void)tc::mbar_wait(&acc_full[last & 1], (uint32_t)(last >> 1) & 1u, lim);
    }
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 2 * kAcc);
  }
}

// ---------------------------------------------------------------- prep kernel
// bf16 operand copies of the caller's W0 (W1/W3 rows interleaved in 128-row blocks).
// Block `bid` of `nblk` blocks (256 threads) of the bf16 copy of W0.
__device__ __forceinline__ void shadow_init_blocks(const FwdP& p, const float* __restrict__ W0, int bid,
                                                   int nblk) {
  // One warp per state row, two rows per pass with both rows' loads issued first:
  // rows [0, 2 d_h) of a head are W1 then W3 (d_k wide; GELU MLP: [0, d_h) are
  // W1), the next d_v rows are W2 (d_h wide); the linear state is d_v rows of d_k.
  const Dims& d = p.d;
  const int lane = threadIdx.x & 31;
  const int r13 = d.kind == 1 ? 2 * d.d_h : d.kind == 2 ? d.d_h : d.d_v;
  const int rows = d.kind != 0 ? r13 + d.d_v : r13;
  const long long total = (long long)d.BH * rows;
  const long long nwarps = (long long)nblk * (blockDim.x / 32);
  auto row_of = [&](long long gr, const float*& src, bf16*& dst, int& len) {
    const int z = (int)(gr / rows), r = (int)(gr - (long long)z * rows);
    if (r < r13) {
      src = W0 + (size_t)z * d.S + (size_t)r * d.d_k;
      const int sr = d.kind == 1 ? w13_row(r % d.d_h, r / d.d_h) : r;
      dst = p.Wsh13 + ((size_t)z * r13 + sr) * d.d_k;
      len = d.d_k;
    } else {
      src = W0 + (size_t)z * d.S + (size_t)r13 * d.d_k + (size_t)(r - r13) * d.d_h;
      dst = p.W2sh + ((size_t)z * d.d_v + (r - r13)) * d.d_h;
      len = d.d_h;
    }
  };
  for (long long gr = (long long)bid * (blockDim.x / 32) + (threadIdx.x >> 5); gr < total;
       gr += 2 * nwarps) {
    const float *s0, *s1 = nullptr;
    bf16 *d0, *d1 = nullptr;
    int n0, n1 = 0;
    row_of(gr, s0, d0, n0);
    if (gr + nwarps < total) row_of(gr + nwarps, s1, d1, n1);
    // row lengths are multiples of 128: every lane moves whole 8-float groups
    for (int c = lane * 8; c < (n0 > n1 ? n0 : n1); c += 256) {
      float4 f[4];
      const bool h0 = c < n0, h1 = c < n1;
      if (h0) {
        f[0] = *reinterpret_cast<const float4*>(s0 + c);
        f[1] = *reinterpret_cast<const float4*>(s0 + c + 4);
      }
      if (h1) {
        f[2] = *reinterpret_cast<const float4*>(s1 + c);
        f[3] = *reinterpret_cast<const float4*>(s1 + c + 4);
      }
      if (h0)
        *reinterpret_cast<uint4*>(d0 + c) = make_uint4(pack2(f[0].x, f[0].y), pack2(f[0].z, f[0].w),
                                                       pack2(f[1].x, f[1].y), pack2(f[1].z, f[1].w));
      if (h1)
        *reinterpret_cast<uint4*>(d1 + c) = make_uint4(pack2(f[2].x, f[2].y), pack2(f[2].z, f[2].w),
                                                       pack2(f[3].x, f[3].y), pack2(f[3].z, f[3].w));
    }
  }
}

// diag(a) K and diag(b) K for every token (B operands of the W1/W3 aggregation).
// Each thread moves kScaleVec 8-element groups per pass (all loads issued before
// the stores), consecutive threads consecutive groups.
constexpr int kScaleVec = 4;
// Block `bid` of `nblk` blocks (256 threads) of the key scaling.
__device__ __forceinline__ void scale_keys_blocks(const bf16* __restrict__ k, const float* __restrict__ ca,
                                                  const float* __restrict__ cb, bf16* __restrict__ Ka,
                                                  bf16* __restrict__ Kb, long long tokens, int d_k,
                                                  int bid, int nblk) {
  const long long n8 = tokens * d_k / 8;
  const long long step = (long long)nblk * blockDim.x * kScaleVec;
  for (long long base = (long long)bid * blockDim.x * kScaleVec + threadIdx.x; base < n8;
       base += step) {
    uint4 u[kScaleVec];
    float a[kScaleVec], b[kScaleVec];
#pragma unroll
    for (int j = 0; j < kScaleVec; ++j) {
      const long long e8 = base + (long long)j * blockDim.x;
      if (e8 < n8) {
        const long long tok = e8 * 8 / d_k;
        u[j] = reinterpret_cast<const uint4*>(k)[e8];
        a[j] = ca[tok];
        b[j] = cb[tok];
      }
    }
#pragma unroll
    for (int j = 0; j < kScaleVec; ++j) {
      const long long e8 = base + (long long)j * blockDim.x;
      if (e8 >= n8) continue;
      const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
      uint32_t oa[4], ob[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        oa[i] = pack2(a[j] * f.x, a[j] * f.y);
        ob[i] = pack2(b[j] * f.x, b[j] * f.y);
      }
      if (Ka) reinterpret_cast<uint4*>(Ka)[e8] = make_uint4(oa[0], oa[1], oa[2], oa[3]);  // NULL: no momentum
      reinterpret_cast<uint4*>(Kb)[e8] = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
  }
}

// The two prep jobs of a call in one launch: of every three blocks two copy W0
// to bf16 and one scales the keys (k NULL: the copy alone), so both streams of
// HBM traffic run side by side and the step has one prep launch, not two.
// Launched with programmatic stream serialization behind K1: the copy blocks
// read only W0, which every earlier operation of the stream has finished
// writing (K1 itself is a plain launch), and write the bf16 shadow, which no
// kernel still running reads, so they start while K1 runs; the key-scaling
// blocks wait for K1's a and b. The next kernel (G1, which waits for this one
// to finish) is released once this block's work is issued, so its CTAs do not
// take registers from the copy while it runs.
__global__ void __launch_bounds__(256) prep_kernel(FwdP p, const float* __restrict__ W0,
                                                   const bf16* __restrict__ k,
                                                   const float* __restrict__ ca,
                                                   const float* __restrict__ cb, bf16* Ka, bf16* Kb,
                                                   long long tokens, int d_k) {
  const int b = blockIdx.x, n = gridDim.x;
  if (k == nullptr) {
    shadow_init_blocks(p, W0, b, n);
  } else if (b % 3 == 2) {
    griddep_wait();  // K1's a_t and b_t are complete and visible
    scale_keys_blocks(k, ca, cb, Ka, Kb, tokens, d_k, b / 3, n / 3);
  } else {
    shadow_init_blocks(p, W0, b - b / 3, n - n / 3);
  }
  griddep_launch_dependents();
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix; box = 64 columns x box_rows
// rows, 128B swizzle (K-major operand: box_rows = tile rows; MN-major: 64).
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D fp32 map over the state rows [rows, cols] of every head (head stride in
// elements), box 32 x 32 x 1, 128B swizzle.
bool make_state_map(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols, uint64_t heads,
                    uint64_t head_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, heads};
  cuuint64_t strides[2] = {cols * 4, head_stride * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 map over per-head token rows [heads][T][cols], box 32 x 32 x 1, 64B
// swizzle: rows past a head's T are clipped on stores and read as zero on loads.
bool make_tok_map_box32(CUtensorMap* m, const void* base, uint64_t T, uint64_t cols, uint64_t heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, T, heads};
  cuuint64_t strides[2] = {cols * 2, T * cols * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 map, box 32 columns x 32 rows, 64B swizzle (epilogue stores).
bool make_map_box32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <int BN, int NUM_ACC, bool A_MN, bool B_MN, int STAGES, class Epi, int EW = kEpiWarps,
          int ESM = 0>
cudaError_t launch(tc2::Job& job, const FwdP& p, cudaStream_t st) {
  constexpr size_t smem = tc2::smem_bytes<BN, NUM_ACC, A_MN, B_MN, STAGES, EW, ESM>();
  static_assert(smem <= 232448, "shared memory per CTA");
  auto kern = tc2::gemm_persistent<BN, NUM_ACC, A_MN, B_MN, STAGES, EW, Epi, FwdP, ESM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  job.total_tiles = 0;
  for (int c = 0; c < job.n_cls; ++c) job.total_tiles += job.cls[c].tiles_m * job.cls[c].tiles_n * job.heads;
  const int grid = job.total_tiles < num_sms() ? job.total_tiles : num_sms();
  E2TTT_TRACE(EpiName<Epi>::v, st);
  return launch_pdl(kern, dim3(grid), dim3((2 + EW) * 32), smem, st, job, p);
}

// CTA-pair launch: a cluster of two CTAs per 256-row tile (cta_group::2 MMAs,
// each CTA holding half of the B tile), with programmatic stream serialization.
template <int BN, bool A_MN, bool B_MN, int STAGES, class Epi, int EW = kEpiWarps, int ESM = 0>
cudaError_t launch_pair(tc2::Job& job, const FwdP& p, cudaStream_t st) {
  constexpr size_t smem = tcp::pair_smem_bytes<BN, A_MN, B_MN, STAGES, EW>(ESM);
  static_assert(smem <= 232448, "shared memory per CTA");
  auto kern = tcp::gemm_pair<BN, A_MN, B_MN, STAGES, EW, Epi, FwdP, ESM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  job.total_tiles = 0;
  for (int c = 0; c < job.n_cls; ++c) job.total_tiles += job.cls[c].tiles_m * job.cls[c].tiles_n * job.heads;
  const int sms = num_sms() & ~1;
  const int grid = 2 * job.total_tiles < sms ? 2 * job.total_tiles : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((2 + EW) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  E2TTT_TRACE(EpiName<Epi>::v, st);
  return cudaLaunchKernelEx(&cfg, kern, job, p);
}

// Heads per group in the persistent forward's tile order: the largest divisor
// of B*H whose group (all four phases of one chunk) has no more tiles than the
// GPU has SMs, at least one head.
int mega_group_heads(int BH, int tiles_per_head, int sms) {
  int hg = 1;
  for (int h = 1; h <= BH; ++h)
    if (BH % h == 0 && h * tiles_per_head <= sms) hg = h;
  return hg;
}

cudaError_t launch_mega(const MegaJob& J, const FwdP& p, cudaStream_t st) {
  constexpr size_t smem = mk::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(fwd_persistent, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fwd_persistent, (2 + mk::kEW) * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  const int grid = J.total < num_sms() ? J.total : num_sms();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3((2 + mk::kEW) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: tiles wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  E2TTT_TRACE("tc_fwd_persistent", st);
  return cudaLaunchKernelEx(&cfg, fwd_persistent, J, p);
}

template <int DV>
cudaError_t launch_ff12(const FfJob& J, const FwdP& p, cudaStream_t st) {
  constexpr size_t smem = ff::kSmemBytes;
  auto kern = ff12_kernel<DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = J.total < num_sms() ? J.total : num_sms();
  E2TTT_TRACE("tc_ff12_h_y", st);
  return launch_pdl(kern, dim3(grid), dim3((2 + ff::kEW) * 32), smem, st, J, p);
}

struct Scratch {
  bf16 *Wsh13, *W2sh, *A, *Sk, *E, *Ea, *Eb, *dH, *Ka, *Kb;
  int* cnt;  // persistent forward: completed tiles per (phase, head)
};

size_t carve(const Dims& d, char* base, Scratch* s) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = (off + bytes + 255) & ~size_t(255);
    return (bf16*)p;
  };
  const size_t e = sizeof(bf16), BH = d.BH;
  Scratch t{};
  if (d.kind == 0) {
    t.Wsh13 = take(BH * d.d_v * d.d_k * e);
  } else {
    const size_t nf = d.kind == 1 ? 2 : 1;  // activation factors per hidden unit
    t.Wsh13 = take(BH * nf * d.d_h * d.d_k * e);
    t.W2sh = take(BH * d.d_v * d.d_h * e);
    t.A = take(BH * 2 * d.C * d.d_h * e);
    t.Sk = take(BH * d.C * nf * d.d_h * e);
    t.E = take(BH * d.C * d.d_v * e);
    t.dH = take(BH * d.C * nf * d.d_h * e);
    t.Ka = take(BH * d.T * d.d_k * e);
    t.Kb = take(BH * d.T * d.d_k * e);
  }
  t.Ea = take(BH * d.C * d.d_v * e);
  t.Eb = take(BH * d.C * d.d_v * e);
  t.cnt = (int*)take(4 * BH * sizeof(int));
  if (s) *s = t;
  return off;
}

// Failure-detection test hook (e2ttt_test_stall_next_forward): armed, it makes
// the first GEMM launch of the next tensor-core forward stall one CTA on an
// mbarrier nothing completes, with every wait of that launch limited to 1 ms.
std::atomic<int> g_stall_next{0};
constexpr unsigned long long kStallWaitNs = 1000000ull;

}  // namespace

void arm_forward_stall(bool on) { g_stall_next.store(on ? 1 : 0); }

bool tc_fwd_supported(const Dims& d, bool bf16_act) {
  if (!bf16_act || d.fp32_gemm) return false;
  if (d.C % 128 != 0) return false;  // a shorter last chunk runs padded to C tokens
  if (d.d_k % 128 != 0 || d.d_v % 128 != 0) return false;
  if (d.kind != 0 && d.d_h % 128 != 0) return false;
  return encode_fn() != nullptr;
}

size_t tc_fwd_scratch_bytes(const Dims& d) { return carve(d, nullptr, nullptr); }

cudaError_t tc_fwd(const Dims& d, const bf16* q, const bf16* k, const bf16* v, bf16* out,
                   const float* ca, const float* cb, const float* scal, const float* W0,
                   const float* M0, float* W_end, float* M_end, float* saved, void* scratch,
                   int* status, cudaStream_t st, bf16* acts_e, bf16* acts_dh) {
  Scratch s;
  carve(d, (char*)scratch, &s);
  FwdP p;
  p.d = d;
  p.q = q; p.k = k; p.v = v; p.out = out;
  p.ca = ca; p.cb = cb; p.scal = scal;
  p.status = status;
  p.nomom = d.nomom;
  p.Wsh13 = s.Wsh13; p.W2sh = s.W2sh;
  p.A = s.A; p.Sk = s.Sk; p.E = s.E; p.Ea = s.Ea; p.Eb = s.Eb; p.dH = s.dH; p.Ka = s.Ka;
  p.Kb = s.Kb;
  const int BH = d.BH, T = d.T, C = d.C, NC = d.NC, dk = d.d_k, dv = d.d_v, dh = d.d_h;
  const int nf = d.kind == 1 ? 2 : 1;           // activation factors per hidden unit
  const int r13 = d.kind == 0 ? dv : nf * dh;   // rows of the first state block

  cudaError_t e = save_initial_state(d, W0, M0, saved, st);
  if (e != cudaSuccess) return e;
  {
    // the bf16 copy of W0 and (MLP fast weights) the scaled keys: 12 blocks per
    // SM, a multiple of 3 (8 copy the state, 4 scale keys)
    E2TTT_TRACE("tc_prep", st);
    e = launch_pdl(prep_kernel, dim3(12 * num_sms()), dim3(256), 0, st, p, W0,
                   d.kind != 0 ? k : nullptr, ca, cb, d.nomom ? nullptr : s.Ka, s.Kb,
                   (long long)BH * T, dk);
    if (e != cudaSuccess) return e;
  }

  // G2 and G3 run 128 x 256 tiles where their N (d_v, resp. d_h) allows: half
  // the A-operand reloads and half the ring handshakes per FLOP of 128 x 128.
  const char* env_p = getenv("E2TTT_PERSISTENT");
  // the persistent kernel (below) runs 128 x 128 tiles in G2 and G3
  const bool persistent = d.kind == 1 && !d.nomom && saved == nullptr && env_p && env_p[0] == '1';
  const bool wide_ok = !persistent;
  // (only while the wide tiles still fill every SM at least once: with few
  // heads the narrower tiles keep more SMs busy)
  const int sms = num_sms();
  const bool wide2 = wide_ok && d.kind == 1 && dv % 256 == 0 && BH * (2 * C / 128) * (dv / 256) >= sms;
  const bool wide3 = wide_ok && d.kind == 1 && dh % 256 == 0 && BH * (C / 128) * (dh / 256) >= sms;
  // Operand maps (chunk-independent; the chunk offset goes into the coordinates).
  tc2::Job g1{}, g2{}, g3{}, g4{};
  bool ok = true;
  for (tc2::Job* j : {&g1, &g2, &g3, &g4}) {
    j->heads = BH;
    j->status = status;
  }
  using tc2::kModeA1B2;
  using tc2::kModeA2B1;
  if (d.kind != 0) {
    ok &= make_map(&g1.maps[0].op0, q, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[1].op0, k, (uint64_t)BH * T, dk, 128);
    g1.n_cls = 2;
    if (d.kind == 1) {
      // G1: classes = query rows, key rows; B = interleaved [W1; W3]
      ok &= make_map(&g1.maps[0].op2, s.Wsh13, (uint64_t)BH * 2 * dh, dk, 256);
      for (int c = 0; c < 2; ++c)
        g1.cls[c] = tc2::Class{C / 128, 2 * dh / 256, dk / 64, {T, 0, 0}, {2 * dh, 0, 0}, 0};
    } else {
      // G1, GELU MLP: B = W1 (N = d_h), 128-wide tiles
      ok &= make_map(&g1.maps[0].op2, s.Wsh13, (uint64_t)BH * dh, dk, 128);
      for (int c = 0; c < 2; ++c)
        g1.cls[c] = tc2::Class{C / 128, dh / 128, dk / 64, {T, 0, 0}, {dh, 0, 0}, 0};
    }
    g1.maps[1].op2 = g1.maps[0].op2;
    // G2: A = [A_q; A_k], B = W2 (N = d_v)
    ok &= make_map(&g2.maps[0].op0, s.A, (uint64_t)BH * 2 * C, dh, 128);
    ok &= make_map(&g2.maps[0].op2, s.W2sh, (uint64_t)BH * dv, dh, wide2 ? 256 : 128);
    g2.n_cls = 1;
    g2.cls[0] = tc2::Class{2 * C / 128, dv / (wide2 ? 256 : 128), dh / 64, {2 * C, 0, 0}, {dv, 0, 0}, 0};
    // G3: A = E, B = W2 read MN-major (N = d_h, K = d_v)
    ok &= make_map(&g3.maps[0].op0, s.E, (uint64_t)BH * C, dv, 128);
    ok &= make_map(&g3.maps[0].op2, s.W2sh, (uint64_t)BH * dv, dh, 64);
    g3.n_cls = 1;
    g3.cls[0] = tc2::Class{C / 128, dh / (wide3 ? 256 : 128), dv / 64, {C, 0, 0}, {dv, 0, 0}, 0};
    // G4 class 0: A = dH (M = [W1; W3] rows, or W1 rows for GELU; K = tokens),
    // B0 = diag(a) K, B1 = diag(b) K
    ok &= make_map(&g4.maps[0].op0, s.dH, (uint64_t)BH * C, r13, 64);
    ok &= make_map(&g4.maps[0].op1, s.Ka, (uint64_t)BH * T, dk, 64);
    ok &= make_map(&g4.maps[0].op2, s.Kb, (uint64_t)BH * T, dk, 64);
    // G4 class 1: A0 = diag(a) E, A1 = diag(b) E (M = W2 rows), B = A_k (rows [C, 2C) of A)
    ok &= make_map(&g4.maps[1].op0, s.Ea, (uint64_t)BH * C, dv, 64);
    ok &= make_map(&g4.maps[1].op1, s.Eb, (uint64_t)BH * C, dv, 64);
    ok &= make_map(&g4.maps[1].op2, s.A, (uint64_t)BH * 2 * C, dh, 64);
    g4.n_cls = 2;
    g4.cls[0] = tc2::Class{r13 / 128, dk / 128, C / 64, {C, 0, 0}, {T, 0, 0}, kModeA1B2};
    g4.cls[1] = tc2::Class{dv / 128, dh / 128, C / 64, {C, 0, 0}, {2 * C, C, 0}, kModeA2B1};
  } else {
    ok &= make_map(&g1.maps[0].op0, q, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[1].op0, k, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[0].op2, s.Wsh13, (uint64_t)BH * dv, dk, 128);
    g1.maps[1].op2 = g1.maps[0].op2;
    g1.n_cls = 2;
    for (int c = 0; c < 2; ++c)
      g1.cls[c] = tc2::Class{C / 128, dv / 128, dk / 64, {T, 0, 0}, {dv, 0, 0}, 0};
    // G4: A0 = diag(a) E, A1 = diag(b) E (M = rows of W), B = K (N = d_k, K = tokens)
    ok &= make_map(&g4.maps[0].op0, s.Ea, (uint64_t)BH * C, dv, 64);
    ok &= make_map(&g4.maps[0].op1, s.Eb, (uint64_t)BH * C, dv, 64);
    ok &= make_map(&g4.maps[0].op2, k, (uint64_t)BH * T, dk, 64);
    g4.n_cls = 1;
    g4.cls[0] = tc2::Class{dv / 128, dk / 128, C / 64, {C, 0, 0}, {T, 0, 0}, kModeA2B1};
  }
  // Without momentum: one accumulator (the b-weighted aggregation), W only.
  tc2::Job g4w{};
  g4w.heads = BH;
  g4w.status = status;
  if (d.nomom) {
    if (d.kind != 0) {
      ok &= make_map(&g4w.maps[0].op0, s.dH, (uint64_t)BH * C, r13, 64);
      ok &= make_map(&g4w.maps[0].op2, s.Kb, (uint64_t)BH * T, dk, 64);
      ok &= make_map(&g4w.maps[1].op0, s.Eb, (uint64_t)BH * C, dv, 64);
      ok &= make_map(&g4w.maps[1].op2, s.A, (uint64_t)BH * 2 * C, dh, 64);
      g4w.n_cls = 2;
      g4w.cls[0] = tc2::Class{r13 / 128, dk / 128, C / 64, {C, 0, 0}, {T, 0, 0}, 0};
      g4w.cls[1] = tc2::Class{dv / 128, dh / 128, C / 64, {C, 0, 0}, {2 * C, C, 0}, 0};
    } else {
      ok &= make_map(&g4w.maps[0].op0, s.Eb, (uint64_t)BH * C, dv, 64);
      ok &= make_map(&g4w.maps[0].op2, k, (uint64_t)BH * T, dk, 64);
      g4w.n_cls = 1;
      g4w.cls[0] = tc2::Class{dv / 128, dk / 128, C / 64, {C, 0, 0}, {T, 0, 0}, 0};
    }
  }
  // 32 x 32 tiles of the epilogues (bf16, 64B swizzle)
  ok &= make_tok_map_box32(&p.mOut, out, T, dv, BH);
  ok &= make_tok_map_box32(&p.mV, v, T, dv, BH);
  ok &= make_map_box32(&p.mEa, s.Ea, (uint64_t)BH * C, dv);
  ok &= make_map_box32(&p.mEb, s.Eb, (uint64_t)BH * C, dv);
  if (d.kind != 0) {
    ok &= make_map_box32(&p.mA, s.A, (uint64_t)BH * 2 * C, dh);
    ok &= make_map_box32(&p.mSk, s.Sk, (uint64_t)BH * C, nf * dh);
    ok &= make_map_box32(&p.mE, s.E, (uint64_t)BH * C, dv);
    ok &= make_map_box32(&p.mdH, s.dH, (uint64_t)BH * C, nf * dh);
  }
  if (!ok) return cudaErrorInvalidValue;

  // SwiGLU with E2TTT_PAIRS=1: G1, G2 and G3 on CTA pairs (256-row tiles, each
  // CTA of a pair loading half of the B tile), where the 128 x 256 tiles fill the
  // GPU. Bit-identical to the one-CTA launches; measured slower on the 1.3B layer
  // (G1 31 -> 38 us, G2 25 -> 25, G3 24 -> 27 per chunk), so not the default.
  const char* env_pr = getenv("E2TTT_PAIRS");
  const char* env_f0 = getenv("E2TTT_FUSED");
  const bool pairs = d.kind == 1 && !persistent && C % 256 == 0 && wide2 && wide3 && env_pr &&
                     env_pr[0] == '1' && !(env_f0 && env_f0[0] == '1');
  tc2::Job p1 = g1, p2 = g2, p3 = g3;
  if (pairs) {
    ok &= make_map(&p1.maps[0].op2, s.Wsh13, (uint64_t)BH * 2 * dh, dk, 128);
    p1.maps[1].op2 = p1.maps[0].op2;
    for (int c = 0; c < 2; ++c) p1.cls[c].tiles_m = C / 256;
    ok &= make_map(&p2.maps[0].op2, s.W2sh, (uint64_t)BH * dv, dh, 128);
    p2.cls[0].tiles_m = 2 * C / 256;
    p3.cls[0].tiles_m = C / 256;
    if (!ok) return cudaErrorInvalidValue;
  }

  // SwiGLU: G1 and G2 as one fused launch per chunk (u of the query rows stays
  // on chip), selected with E2TTT_FUSED=1 in the environment. Not the default:
  // on the 1.3B layer it is slower than the two launches it replaces (each
  // 128-row tile streams its head's whole W1, W3 and W2 through a three-stage
  // ring, behind a single H accumulator).
  const char* env_f = getenv("E2TTT_FUSED");
  const bool fused = d.kind == 1 && !persistent && (dv == 128 || dv == 256) && dh % 128 == 0 &&
                     env_f && env_f[0] == '1';
  FfJob fj{};
  if (fused) {
    fj.mX[0] = g1.maps[0].op0;
    fj.mX[1] = g1.maps[1].op0;
    fj.mW13 = g1.maps[0].op2;
    ok &= make_map(&fj.mW2, s.W2sh, (uint64_t)BH * dv, dh, (uint32_t)dv);
    ok &= make_map(&fj.mU, s.A, (uint64_t)BH * 2 * C, dh, 32);
    fj.mtiles = C / 128;
    fj.nblk = dh / 128;
    fj.kbh = dk / 64;
    fj.total = BH * 2 * fj.mtiles;
    fj.status = status;
    if (!ok) return cudaErrorInvalidValue;
  }

  // SwiGLU with momentum and no saved states may run every chunk in one
  // persistent, cooperative launch; it is selected with E2TTT_PERSISTENT=1 in
  // the environment (the per-phase launches are faster on the shapes measured).
  if (persistent) {
    MegaJob J{};
    J.ph[0] = g1;
    J.ph[1] = g2;
    J.ph[2] = g3;
    J.ph[3] = g4;
    for (int ph = 0; ph < 4; ++ph) {
      J.tph[ph] = 0;
      for (int c = 0; c < J.ph[ph].n_cls; ++c)
        J.tph[ph] += J.ph[ph].cls[c].tiles_m * J.ph[ph].cls[c].tiles_n;
    }
    const int tph_all = J.tph[0] + J.tph[1] + J.tph[2] + J.tph[3];
    J.BH = BH;
    J.NC = NC;
    J.C = C;
    const char* env_hg = getenv("E2TTT_PERSISTENT_HG");
    J.hg = env_hg ? atoi(env_hg) : mega_group_heads(BH, tph_all, num_sms());
    if (J.hg < 1 || BH % J.hg != 0) J.hg = 1;
    J.per_group = J.hg * tph_all;
    J.per_chunk = BH * tph_all;
    J.total = NC * J.per_chunk;
    J.cnt = s.cnt;
    J.status = status;
    J.stall = g_stall_next.exchange(0) != 0;
    J.wait_ns = J.stall ? kStallWaitNs : 0;
    // state maps: variant 0 = W0, M0 (first chunk), 1 = W_end, M_end in place
    p.hasM[0] = M0 != nullptr;
    p.hasM[1] = 1;
    for (int c = 0; c < 2; ++c) {
      const long long off = c == 0 ? 0 : (long long)r13 * dk;
      const uint64_t rows = c == 0 ? r13 : dv;
      const uint64_t cols = c == 0 ? dk : dh;
      ok &= make_state_map(&p.srcW[0][c], W0 + off, rows, cols, BH, d.S);
      if (M0) ok &= make_state_map(&p.srcM[0][c], M0 + off, rows, cols, BH, d.S);
      ok &= make_state_map(&p.srcW[1][c], W_end + off, rows, cols, BH, d.S);
      ok &= make_state_map(&p.srcM[1][c], M_end + off, rows, cols, BH, d.S);
      ok &= make_state_map(&p.dstW[c], W_end + off, rows, cols, BH, d.S);
      ok &= make_state_map(&p.dstM[c], M_end + off, rows, cols, BH, d.S);
    }
    ok &= make_map_box32(&p.shadow[0], s.Wsh13, (uint64_t)BH * r13, dk);
    ok &= make_map_box32(&p.shadow[1], s.W2sh, (uint64_t)BH * dv, dh);
    if (!ok) return cudaErrorInvalidValue;
    e = cudaMemsetAsync(s.cnt, 0, 4 * (size_t)BH * sizeof(int), st);
    if (e != cudaSuccess) return e;
    return launch_mega(J, p, st);
  }

  for (int ci = 0; ci < NC; ++ci) {
    const int clen = T - ci * C < C ? T - ci * C : C;
    for (tc2::Job* j : {&g1, &g2, &g3, &g4, &g4w}) {
      j->ci = ci;
      j->t0 = ci * C;
      j->clen = clen;
      j->wshadow = ci + 1 < NC;
    }
    StateIn src;
    StateOut dst;
    chunk_states(d, ci, W0, M0, W_end, M_end, saved, &src, &dst);
    {
      const int ncls = d.kind != 0 ? 2 : 1;
      p.hasM[0] = p.hasM[1] = src.M != nullptr;
      for (int c = 0; c < ncls; ++c) {
        const long long off = c == 0 ? 0 : (long long)r13 * dk;
        const uint64_t rows = c == 0 ? r13 : dv;
        const uint64_t cols = c == 0 ? dk : dh;
        ok &= make_state_map(&p.srcW[0][c], src.W + off, rows, cols, BH, src.stride);
        if (src.M) ok &= make_state_map(&p.srcM[0][c], src.M + off, rows, cols, BH, src.stride);
        p.srcW[1][c] = p.srcW[0][c];
        p.srcM[1][c] = p.srcM[0][c];
        ok &= make_state_map(&p.dstW[c], dst.W + off, rows, cols, BH, dst.stride);
        if (dst.M) ok &= make_state_map(&p.dstM[c], dst.M + off, rows, cols, BH, dst.stride);
      }
      if (ci == 0) {
        ok &= make_map_box32(&p.shadow[0], s.Wsh13, (uint64_t)BH * r13, dk);
        if (d.kind != 0) ok &= make_map_box32(&p.shadow[1], s.W2sh, (uint64_t)BH * dv, dh);
      }
      if (acts_e && d.kind != 0) {
        // saved activations: this chunk's E and dH go to its slots of saved_states
        // (same layouts as the scratch they replace), where G3 and G4 read them
        bf16* Ec = acts_e + (size_t)ci * BH * C * dv;
        bf16* Dc = acts_dh + (size_t)ci * BH * C * r13;
        ok &= make_map_box32(&p.mE, Ec, (uint64_t)BH * C, dv);
        ok &= make_map(&g3.maps[0].op0, Ec, (uint64_t)BH * C, dv, 128);
        ok &= make_map_box32(&p.mdH, Dc, (uint64_t)BH * C, r13);
        ok &= make_map(&g4.maps[0].op0, Dc, (uint64_t)BH * C, r13, 64);
        g4w.maps[0].op0 = g4.maps[0].op0;  // no momentum: the W-only aggregation reads dH too
        p3.maps[0].op0 = g3.maps[0].op0;
      }
      if (!ok) return cudaErrorInvalidValue;
    }
    g1.cls[0].a.y_base = g1.cls[1].a.y_base = ci * C;  // query / key rows of this chunk
    g1.stall = ci == 0 && g_stall_next.exchange(0) ? 1 : 0;
    g1.wait_ns = g1.stall ? kStallWaitNs : 0;
    g4.cls[0].b.y_base = ci * C;                        // key rows (K dimension) of this chunk
    g4w.cls[0].b.y_base = ci * C;
    if (d.kind != 0) {
      if (fused) {
        fj.ci = ci;
        fj.t0 = ci * C;
        fj.clen = clen;
        fj.stall = g1.stall;  // the stall hook, armed for this chunk's first launch
        fj.wait_ns = g1.wait_ns;
        e = dv == 256 ? launch_ff12<256>(fj, p, st) : launch_ff12<128>(fj, p, st);
      } else if (pairs) {
        for (tc2::Job* j : {&p1, &p2, &p3}) {
          j->ci = ci;
          j->t0 = ci * C;
          j->clen = clen;
          j->wshadow = ci + 1 < NC;
        }
        p1.cls[0].a.y_base = p1.cls[1].a.y_base = ci * C;
        p1.stall = g1.stall;
        p1.wait_ns = g1.wait_ns;
        e = launch_pair<256, false, false, 5, EpiG1, kEpiWarps, EpiG1::kSmem>(p1, p, st);
        if (e == cudaSuccess)
          e = clen < C ? launch_pair<256, false, false, 4, EpiG2Pad, kEpiWarps, EpiG2Pad::kSmem>(p2, p, st)
                       : launch_pair<256, false, false, 4, EpiG2, kEpiWarps, EpiG2::kSmem>(p2, p, st);
        if (e == cudaSuccess) e = launch_pair<256, false, true, 5, EpiG3, kEpiWarps, EpiG3::kSmem>(p3, p, st);
      } else if (d.kind == 1) {
        e = launch<256, 1, false, false, 3, EpiG1, kEpiWarps, EpiG1::kSmem>(g1, p, st);
      } else {
        e = launch<128, 1, false, false, 4, EpiG1Gelu, kEpiWarps, EpiG1Gelu::kSmem>(g1, p, st);
      }
      if (e == cudaSuccess && !fused && !pairs) {
        if (wide2)
          e = clen < C ? launch<256, 1, false, false, 3, EpiG2Pad, kEpiWarps, EpiG2Pad::kSmem>(g2, p, st)
                         : launch<256, 1, false, false, 3, EpiG2, kEpiWarps, EpiG2::kSmem>(g2, p, st);
        else
          e = clen < C ? launch<128, 1, false, false, 4, EpiG2Pad, kEpiWarps, EpiG2Pad::kSmem>(g2, p, st)
                         : launch<128, 1, false, false, 4, EpiG2, kEpiWarps, EpiG2::kSmem>(g2, p, st);
      }
      if (e == cudaSuccess && !pairs) {
        e = d.kind != 1 ? launch<128, 1, false, true, 3, EpiG3Gelu, kEpiWarps, EpiG3Gelu::kSmem>(g3, p, st)
            : wide3     ? launch<256, 1, false, true, 3, EpiG3, kEpiWarps, EpiG3::kSmem>(g3, p, st)
                        : launch<128, 1, false, true, 3, EpiG3, kEpiWarps, EpiG3::kSmem>(g3, p, st);
      }
      if (e == cudaSuccess) {
        e = d.nomom ? launch<128, 1, true, true, 4, EpiG4W, 4, EpiG4W::kSmem>(g4w, p, st)
                    : launch<128, 2, true, true, 3, EpiG4, 4, EpiG4::kSmem>(g4, p, st);
      }
    } else {
      e = clen < C ? launch<128, 1, false, false, 4, EpiG1LinPad, kEpiWarps, EpiG1LinPad::kSmem>(g1, p, st)
                     : launch<128, 1, false, false, 4, EpiG1Lin, kEpiWarps, EpiG1Lin::kSmem>(g1, p, st);
      if (e == cudaSuccess) {
        e = d.nomom ? launch<128, 1, true, true, 4, EpiG4W, 4, EpiG4W::kSmem>(g4w, p, st)
                    : launch<128, 2, true, true, 3, EpiG4, 4, EpiG4::kSmem>(g4, p, st);
      }
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace e2ttt
