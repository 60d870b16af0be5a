// tcgen05 tensor-core backward of the chunk scan (SwiGLU and GELU MLP, bf16
// activations).
//
// Same mathematics as the CUDA-core backward (bwd.cu): the adjoint of the
// closed-form chunk transition ("Rethinking Expressivity and Efficiency in
// Test-Time Training": abstract, fully parallelized chunk-level training),
// chunks in reverse, second-order terms through the loss gradient included.
// Per chunk, all heads at once (token-major bf16 operands and epilogue data between
// phases, fp32 accumulation):
//   R1  [K; Q] -> H1 = X W1^T, H3 = X W3^T (two accumulators) ; u = silu(H1) H3
//   R2  E = U_k W2^T - V            R3  du = E W2 -> dH1 = du H3 silu'(H1), dH3 = du silu(H1)
//   D1  K [D_M13 | D_W13]^T -> dh1b/dh3b = -(a P_M + b P_W) and the abar/bbar dot products
//   D2  U_k [D_M2 | D_W2]^T -> G2u = -(a P_M + b P_W) and the abar/bbar dot products
//   E3  E [D_M2 | D_W2] -> -(a . + b .) ; dub = dh1b H3 silu'(H1) + dh3b silu(H1)
//   E4  eb = dub W2^T + G2u (dv = -eb)    E5  [E; EB] W2: du again, ub = E3 term + eb W2 -> h1b, h3b
//   Q1  dout W2 -> query-row h1b, h3b
//   dk = -(a dH D_M13 + b dH D_W13) + [h1b | h3b] [W1; W3] ;  dq = query-row [h1b | h3b] [W1; W3]
//   dW13 += [h1b | h3b]^T [K; Q] ,  dW2 += [E; EB; dout]^T [dub; U_k; U_q]  (into D_W in place)
//   dM0 = U(1,n) D_M + c D_W ; abar, bbar and the chunk-scalar adjoints for the gate gradients.
// Launches per chunk: the shadow pass, R1, R2, R3 + Q1, D1 + D2, E3 + dk1, E4, E5,
// dk2 + dq, the sums (abar, bbar and the chunk-scalar adjoints), dW (a "+" joins
// two phases in one launch). With the forward's E and dH saved (save_acts), R2
// and the R3 half of R3 + Q1 are not run: E is copied into Z3 and dH read in
// place from the saved activations.
// GELU MLP (h = W1 k, u = gelu(h); one activation factor per hidden unit, so the
// [W1; W3] blocks above are W1 alone and h1 | h3 is h):
//   R1  h = X W1^T ; u = gelu(h)     R3  dH = du gelu'(h)     E3  dub = dhb gelu'(h)
//   E5  hb = dhb du gelu''(h) + ub gelu'(h)     Q1  query-row hb = (dout W2) gelu'(h)
// and D1, D2, E4, dk, dq, dW as above with hw = d_h columns instead of 2 d_h.
#include <cuda.h>

#include <algorithm>
#include <type_traits>

#include "paths.h"
#include "state.cuh"
#include "tc_gemm2.cuh"
#include "trace.h"

namespace e2ttt {
namespace {

using tc2::EpiCtx;

constexpr int kEW = 8;  // epilogue warps

struct BwdP {
  // 32 x 32 boxes for the epilogues' TMA-staged I/O (bf16: 64B swizzle, fp32: 128B)
  CUtensorMap mHc, mY3, mDH, mHB, fDB, fUBd;
  CUtensorMap mZ3, mv, mdv, mdk, mdq, fG2U, fdkp, fDW[2];
  // mv, mdv, mdk, mdq are 3-D (columns, tokens, heads): a box past a head's last
  // token reads as zero and is clipped on store
  Dims d;
  int ci, t0;
  int hw;  // hidden columns of the first state block: 2 d_h (SwiGLU h1 | h3) or d_h (GELU h)
  // tokens of this chunk: C, or T - t0 for a shorter last chunk, whose padding
  // rows carry zero keys, queries, dout and v and a_t = b_t = 0, so every
  // per-token term of theirs vanishes
  int clen;
  const bf16 *v;
  bf16 *dq, *dk, *dv;
  const float *ca, *cb, *scal;
  float *DW, *DM;  // fp32 state adjoints (head stride S), in place
  // bf16 token-major operands (per head)
  bf16 *X;    // [2C, d_k]   rows: keys, then queries
  bf16 *Y3;   // [3C, d_h]   rows: dub | u_k | u_q
  bf16 *Z3;   // [3C, d_v]   rows: E | EB | dout
  bf16 *Hc;   // [2C, hw] h1 | h3 (GELU: h) (keys, then queries)
  bf16 *DH;   // [C, hw]  dH1 | dH3 (GELU: dH)
  bf16 *HB;   // [2C, hw] h1b | h3b (GELU: hb) (keys, then queries)
  // bf16 epilogue data between phases (per head)
  bf16 *DB;      // [C, hw]  dh1b | dh3b (GELU: dhb)
  bf16 *G2U;     // [C, d_v]
  bf16 *UBd;     // [C, d_h]
  bf16 *dkp;     // [C, d_k]
  float *part;   // [C, NG]   partial dot products for abar (and bbar at + BH*C*NG)
  int NG;
  int per0;  // two-phase launches (EpiPair): tiles of the first phase
  int* status;
};

// ---------------------------------------------------------------- row helpers
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <int BN>
__device__ __forceinline__ void acc1(const EpiCtx<BN>& c, int col, float (&x)[32]) {
  uint32_t r[32];
  tc2::tmem_ld32_nowait(c.taddr + (uint32_t)col, r);
  tc2::tmem_wait_ld(r);
#pragma unroll
  for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
}
template <int BN>
__device__ __forceinline__ void acc2(const EpiCtx<BN>& c, int col, float (&x)[32], float (&y)[32]) {
  uint32_t r[32], s[32];
  tc2::tmem_ld32_nowait(c.taddr + (uint32_t)col, r);
  tc2::tmem_ld32_nowait(c.taddr + (uint32_t)(BN + col), s);
  tc2::tmem_wait_ld2(r, s);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = __uint_as_float(r[i]);
    y[i] = __uint_as_float(s[i]);
  }
}
// sigmoid with the fast exponential and reciprocal; silu, silu', silu'' from it.
struct Act {
  float s, d1, d2;  // silu(z), silu'(z), silu''(z)
  __device__ __forceinline__ explicit Act(float z) {
    const float sg = __fdividef(1.0f, 1.0f + __expf(-z));
    s = z * sg;
    d1 = sg * (1.0f + z * (1.0f - sg));
    d2 = sg * (1.0f - sg) * (2.0f + z * (1.0f - 2.0f * sg));
  }
};
__device__ __forceinline__ float fsilu(float z) { return z * __fdividef(1.0f, 1.0f + __expf(-z)); }
// ---------------------------------------------------------------- staged tile I/O
// A warp's 32 rows x 32 columns move between global memory and shared memory as
// one TMA box: bf16 boxes (2 KB) use the 64B swizzle, fp32 boxes (4 KB) the 128B
// swizzle; lane r reads or writes row r. Buffers are 1024-byte aligned.
__device__ __forceinline__ int swz64(int r, int q) { return r * 64 + ((q ^ ((r >> 1) & 3)) << 4); }
__device__ __forceinline__ int swz128(int r, int q) { return r * 128 + ((q ^ (r & 7)) << 4); }
__device__ __forceinline__ void stage_h(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(buf + swz64(r, q)) =
        make_uint4(pack2(v[8 * q], v[8 * q + 1]), pack2(v[8 * q + 2], v[8 * q + 3]),
                   pack2(v[8 * q + 4], v[8 * q + 5]), pack2(v[8 * q + 6], v[8 * q + 7]));
}
__device__ __forceinline__ void unstage_h(const uint8_t* buf, int r, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = *reinterpret_cast<const uint4*>(buf + swz64(r, q));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
      v[8 * q + 2 * j] = f.x;
      v[8 * q + 2 * j + 1] = f.y;
    }
  }
}
// The 8 bf16 values of 16-byte chunk q of row r of a 64B-swizzled tile.
__device__ __forceinline__ void unpack8(const uint8_t* buf, int r, int q, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(buf + swz64(r, q));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
    v[2 * j] = f.x;
    v[2 * j + 1] = f.y;
  }
}
__device__ __forceinline__ void stage_f(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(buf + swz128(r, q)) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
__device__ __forceinline__ void unstage_f(const uint8_t* buf, int r, float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(buf + swz128(r, q));
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
}
// Before refilling the output staging: this warp's earlier TMA stores have read it.
__device__ __forceinline__ void out_free(int lane) {
  if (lane == 0) tc::bulk_wait_read<0>();
  __syncwarp();
}
// After filling the output staging: visible to the TMA (async) proxy.
__device__ __forceinline__ void out_ready() {
  tc::fence_async_smem();
  __syncwarp();
}
// Input loads are single-buffered and chained: group g + 1's boxes (or the next
// tile's first group) are requested as soon as group g's are in registers, on the
// warp's barrier 0. in_wait() consumes one completed load set.
template <int BN>
__device__ __forceinline__ bool in_wait(const BwdP& p, const EpiCtx<BN>& c) {
  const bool ok = tc::mbar_wait(&c.wbar[0], c.uses[0] & 1u);
  c.uses[0] += 1;
  if (!ok && (c.row & 31) == 0) atomicExch(p.status, tc2::kErrEpilogue);
  return ok;
}
// Where a warp's group gi (of ngroups) lies: this tile, or the next tile's first group.
struct GroupAt {
  int valid, cls, z, m0, col;
};
template <int BN>
__device__ __forceinline__ GroupAt group_at(const EpiCtx<BN>& c, int gi) {
  const int per = BN / c.nparts;
  if (gi < per / 32) return GroupAt{1, c.cls, c.z, c.m0, c.n0 + c.part * per + gi * 32};
  return GroupAt{c.nxt_valid, c.nxt_cls, c.nxt_z, c.nxt_m0, c.nxt_n0 + c.part * per};
}

// Column groups of 32 owned by this thread inside the tile.
#define FOR_GROUPS(c, BN, g) \
  for (int g = (c).part * ((BN) / (c).nparts); g < ((c).part + 1) * ((BN) / (c).nparts); g += 32)

// ---------------------------------------------------------------- epilogues
// R1: rows of X (keys then queries); h1 = acc0, h3 = acc1 -> Hc, u = silu(h1) h3 -> Y3.
struct EpiR1 {
  static constexpr int kSmem = 6144;  // h1 | h3 | u staging (bf16)
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;
    const int yH = c.z * 2 * d.C + r0, yU = c.z * 3 * d.C + d.C + r0;
    uint8_t* S = c.wsmem;
    FOR_GROUPS(c, BN, g) {
      const int j = c.n0 + g;
      float h1[32], h3[32];
      acc2(c, g, h1, h3);
      out_free(lane);
      stage_h(S, lane, h1);
      stage_h(S + 2048, lane, h3);
#pragma unroll
      for (int i = 0; i < 32; ++i) h1[i] = fsilu(h1[i]) * h3[i];
      stage_h(S + 4096, lane, h1);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mHc, S, j, yH);
        tc::tma_store_2d(&p.mHc, S + 2048, d.d_h + j, yH);
        tc::tma_store_2d(&p.mY3, S + 4096, j, yU);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// R2: E = y - v (or -v) of the key rows -> rows [0, C) of Z3.
struct EpiR2 {
  static constexpr int kIn = 2048;           // v (bf16)
  static constexpr int kSmem = kIn + 2048;   // | E (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_3d(c.wsmem, &p.mv, &c.wbar[0], ga.col, p.t0 + ga.m0 + c.quad * 32, ga.z);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int yE = c.z * 3 * d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, col = c.n0 + g;
      float y[32], vv[32];
      acc1(c, g, y);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, vv);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = d.loss == 0 ? y[i] - vv[i] : -vv[i];
      out_free(lane);
      stage_h(OUT, lane, y);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mZ3, OUT, col, yE);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// R3: du = E W2 -> dH1 = du H3 silu'(H1), dH3 = du silu(H1) (key rows). du itself
// is not stored: E5 forms it again in a second accumulator of its own GEMM.
struct EpiR3 {
  static constexpr int kIn = 4096;            // h1 | h3 (bf16)
  static constexpr int kSmem = kIn + 4096;    // | dH1 | dH3 (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    const int y = ga.z * 2 * p.d.C + ga.m0 + c.quad * 32;
    tc::mbar_expect_tx(&c.wbar[0], 4096u);
    tc::tma_load_2d(c.wsmem, &p.mHc, &c.wbar[0], ga.col, y);
    tc::tma_load_2d(c.wsmem + 2048, &p.mHc, &c.wbar[0], p.d.d_h + ga.col, y);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int yD = c.z * d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* Hs = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float du[32], h1[32], h3[32];
      acc1(c, g, du);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, h1);
      unstage_h(IN + 2048, lane, h3);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const Act f(h1[i]);
        const float dh1 = du[i] * h3[i] * f.d1;
        h3[i] = du[i] * f.s;  // dH3
        h1[i] = dh1;
      }
      out_free(lane);
      stage_h(Hs, lane, h1);
      stage_h(Hs + 2048, lane, h3);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mDH, Hs, j, yD);
        tc::tma_store_2d(&p.mDH, Hs + 2048, d.d_h + j, yD);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// D1: acc0 = K D_M13^T, acc1 = K D_W13^T over columns [0, 2 d_h) -> DB = -(a P_M + b P_W)
// (bf16) and the abar / bbar partial dot products with dH.
struct EpiD1 {
  static constexpr int kIn = 2048;           // dH (bf16)
  static constexpr int kSmem = kIn + 2048;   // | DB (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_2d(c.wsmem, &p.mDH, &c.wbar[0], ga.col, ga.z * p.d.C + ga.m0 + c.quad * 32);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int t = c.m0 + c.row;
    const size_t tok = (size_t)c.z * d.T + p.t0 + t;
    const float a = t < p.clen ? p.ca[tok] : 0.f, b = t < p.clen ? p.cb[tok] : 0.f;
    const int yD = c.z * d.C + c.m0 + c.quad * 32;
    float* pa = p.part + ((size_t)c.z * d.C + t) * p.NG;
    float* pb = pa + (size_t)d.BH * d.C * p.NG;
    const uint8_t* IN = c.wsmem;
    uint8_t* F = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, jj = c.n0 + g;
      float pm[32], pw[32], dh[32];
      acc2(c, g, pm, pw);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, dh);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
      float sa = 0.f, sb = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sa += dh[i] * pm[i];
        sb += dh[i] * pw[i];
        pm[i] = -(a * pm[i] + b * pw[i]);
      }
      out_free(lane);
      stage_h(F, lane, pm);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.fDB, F, jj, yD);
        tc::bulk_commit();
      }
      __syncwarp();
      pa[jj / 32] = sa;
      pb[jj / 32] = sb;
    }
  }
};
// D2: acc0 = U_k D_M2^T, acc1 = U_k D_W2^T over columns [0, d_v) -> G2u = -(a P_M + b P_W)
// (bf16) and the abar / bbar partial dot products with E.
struct EpiD2 {
  static constexpr int kIn = 2048;           // E (bf16)
  static constexpr int kSmem = kIn + 2048;   // | G2u (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_2d(c.wsmem, &p.mZ3, &c.wbar[0], ga.col, ga.z * 3 * p.d.C + ga.m0 + c.quad * 32);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int t = c.m0 + c.row;
    const size_t tok = (size_t)c.z * d.T + p.t0 + t;
    const float a = t < p.clen ? p.ca[tok] : 0.f, b = t < p.clen ? p.cb[tok] : 0.f;
    const int yG = c.z * d.C + c.m0 + c.quad * 32;
    float* pa = p.part + ((size_t)c.z * d.C + t) * p.NG + p.hw / 32;
    float* pb = pa + (size_t)d.BH * d.C * p.NG;
    const uint8_t* IN = c.wsmem;
    uint8_t* F = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, col = c.n0 + g;
      float pm[32], pw[32], e[32];
      acc2(c, g, pm, pw);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, e);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
      float sa = 0.f, sb = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        sa += e[i] * pm[i];
        sb += e[i] * pw[i];
        pm[i] = -(a * pm[i] + b * pw[i]);
      }
      out_free(lane);
      stage_h(F, lane, pm);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.fG2U, F, col, yG);
        tc::bulk_commit();
      }
      __syncwarp();
      pa[col / 32] = sa;
      pb[col / 32] = sb;
    }
  }
};
// E3: acc0 = E D_M2, acc1 = E D_W2 (columns = hidden units) -> UBd = -(a . + b .)
// (bf16) and dub = dh1b H3 silu'(H1) + dh3b silu(H1) (bf16, rows [0, C) of Y3).
struct EpiE3 {
  static constexpr int kWarps = 4;
  static constexpr int kIn = 8192;           // dh1b | dh3b | h1 | h3 (bf16)
  static constexpr int kSmem = kIn + 4096;   // | UBd | dub (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    const Dims& d = p.d;
    const int r = ga.m0 + c.quad * 32;
    uint64_t* bar = &c.wbar[0];
    tc::mbar_expect_tx(bar, 8192u);
    tc::tma_load_2d(c.wsmem, &p.fDB, bar, ga.col, ga.z * d.C + r);
    tc::tma_load_2d(c.wsmem + 2048, &p.fDB, bar, d.d_h + ga.col, ga.z * d.C + r);
    tc::tma_load_2d(c.wsmem + 4096, &p.mHc, bar, ga.col, ga.z * 2 * d.C + r);
    tc::tma_load_2d(c.wsmem + 6144, &p.mHc, bar, d.d_h + ga.col, ga.z * 2 * d.C + r);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int t = c.m0 + c.row;
    const size_t tok = (size_t)c.z * d.T + p.t0 + t;
    const float a = t < p.clen ? p.ca[tok] : 0.f, b = t < p.clen ? p.cb[tok] : 0.f;
    const int r0 = c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* F = c.wsmem + kIn;
    uint8_t* Hs = c.wsmem + kIn + 2048;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float m[32], w[32];
      acc2(c, g, m, w);
#pragma unroll
      for (int i = 0; i < 32; ++i) m[i] = -(a * m[i] + b * w[i]);
      out_free(lane);
      stage_h(F, lane, m);
      if (!in_wait(p, c)) return;
      float b1[32], b3[32];
      unstage_h(IN, lane, b1);
      unstage_h(IN + 2048, lane, b3);
      unstage_h(IN + 4096, lane, m);       // h1
      unstage_h(IN + 6144, lane, w);       // h3
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const Act f(m[i]);
        b1[i] = b1[i] * w[i] * f.d1 + b3[i] * f.s;
      }
      stage_h(Hs, lane, b1);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.fUBd, F, j, c.z * d.C + r0);
        tc::tma_store_2d(&p.mY3, Hs, j, c.z * 3 * d.C + r0);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// E4: eb = dub W2^T + G2u; EB row (zero for the dot loss) -> rows [C, 2C) of Z3, dv = -eb.
struct EpiE4 {
  static constexpr int kIn = 2048;           // G2u (bf16)
  static constexpr int kSmem = kIn + 4096;   // | dv | EB (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_2d(c.wsmem, &p.fG2U, &c.wbar[0], ga.col, ga.z * p.d.C + ga.m0 + c.quad * 32);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int r0 = c.m0 + c.quad * 32;
    const int tV = p.t0 + r0, yB = c.z * 3 * d.C + d.C + r0;
    const bool any_real = r0 < p.clen;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, col = c.n0 + g;
      float eb[32], gu[32];
      acc1(c, g, eb);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, gu);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        eb[i] += gu[i];
        gu[i] = -eb[i];
      }
      if (d.loss != 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) eb[i] = 0.f;
      }
      out_free(lane);
      stage_h(OUT, lane, gu);
      stage_h(OUT + 2048, lane, eb);
      out_ready();
      if (lane == 0) {
        if (any_real) tc::tma_store_3d(&p.mdv, OUT, col, tV, c.z);
        tc::tma_store_2d(&p.mZ3, OUT + 2048, col, yB);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// E5: two accumulators over the same W2 tile: du = E W2 (acc0) and eb W2 (acc1);
// ub = UBd + eb W2 (MSE); the key rows' h1b, h3b (8 columns at a time).
struct EpiE5 {
  static constexpr int kWarps = 4;
  static constexpr int kIn = 10240;          // UBd | dh1b | dh3b | h1 | h3 (bf16)
  static constexpr int kSmem = kIn + 4096;   // | h1b | h3b (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    const Dims& d = p.d;
    const int r = ga.m0 + c.quad * 32;
    const int yC = ga.z * d.C + r, yH = ga.z * 2 * d.C + r;
    uint64_t* bar = &c.wbar[0];
    tc::mbar_expect_tx(bar, 10240u);
    tc::tma_load_2d(c.wsmem, &p.fUBd, bar, ga.col, yC);
    tc::tma_load_2d(c.wsmem + 2048, &p.fDB, bar, ga.col, yC);
    tc::tma_load_2d(c.wsmem + 4096, &p.fDB, bar, d.d_h + ga.col, yC);
    tc::tma_load_2d(c.wsmem + 6144, &p.mHc, bar, ga.col, yH);
    tc::tma_load_2d(c.wsmem + 8192, &p.mHc, bar, d.d_h + ga.col, yH);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int yH = c.z * 2 * d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float dua[32], acc[32];
      acc2(c, g, dua, acc);
      if (!in_wait(p, c)) return;
      out_free(lane);
#pragma unroll
      for (int s8 = 0; s8 < 4; ++s8) {
        // 8 consecutive columns: one 16-byte chunk of each bf16 row
        float ubd[8], b1[8], b3[8], h1[8], h3[8];
        unpack8(IN, lane, s8, ubd);
        unpack8(IN + 2048, lane, s8, b1);
        unpack8(IN + 4096, lane, s8, b3);
        unpack8(IN + 6144, lane, s8, h1);
        unpack8(IN + 8192, lane, s8, h3);
        const float* du = dua + 8 * s8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float ub = ubd[i] + (d.loss == 0 ? acc[8 * s8 + i] : 0.f);
          const Act f(h1[i]);
          const float sb = b3[i] * du[i] + ub * h3[i];
          const float h3b = b1[i] * du[i] * f.d1 + ub * f.s;
          const float h1b = b1[i] * du[i] * h3[i] * f.d2 + sb * f.d1;
          h1[i] = h1b;
          h3[i] = h3b;
        }
        *reinterpret_cast<uint4*>(OUT + swz64(lane, s8)) =
            make_uint4(pack2(h1[0], h1[1]), pack2(h1[2], h1[3]), pack2(h1[4], h1[5]), pack2(h1[6], h1[7]));
        *reinterpret_cast<uint4*>(OUT + 2048 + swz64(lane, s8)) =
            make_uint4(pack2(h3[0], h3[1]), pack2(h3[2], h3[3]), pack2(h3[4], h3[5]), pack2(h3[6], h3[7]));
      }
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mHB, OUT, j, yH);
        tc::tma_store_2d(&p.mHB, OUT + 2048, d.d_h + j, yH);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// Q1: ub_q = dout W2 -> query-row h1b = ub H3 silu'(H1), h3b = ub silu(H1).
struct EpiQ1 {
  static constexpr int kIn = 4096;           // query h1 | h3 (bf16)
  static constexpr int kSmem = kIn + 4096;   // | h1b | h3b (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    const int y = ga.z * 2 * p.d.C + p.d.C + ga.m0 + c.quad * 32;
    tc::mbar_expect_tx(&c.wbar[0], 4096u);
    tc::tma_load_2d(c.wsmem, &p.mHc, &c.wbar[0], ga.col, y);
    tc::tma_load_2d(c.wsmem + 2048, &p.mHc, &c.wbar[0], p.d.d_h + ga.col, y);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int y = c.z * 2 * d.C + d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float ub[32], h1[32], h3[32];
      acc1(c, g, ub);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, h1);
      unstage_h(IN + 2048, lane, h3);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const Act f(h1[i]);
        const float a1 = ub[i] * h3[i] * f.d1;
        h3[i] = ub[i] * f.s;
        h1[i] = a1;
      }
      out_free(lane);
      stage_h(OUT, lane, h1);
      stage_h(OUT + 2048, lane, h3);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mHB, OUT, j, y);
        tc::tma_store_2d(&p.mHB, OUT + 2048, d.d_h + j, y);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// ---- GELU MLP variants of R1, R3, E3, E5, Q1 (one activation factor per hidden unit)
// R1: rows of X (keys then queries); h = acc -> Hc, u = gelu(h) -> Y3.
struct EpiR1G {
  static constexpr int kSmem = 4096;  // h | u staging (bf16)
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int r0 = c.m0 + c.quad * 32;
    const int yH = c.z * 2 * d.C + r0, yU = c.z * 3 * d.C + d.C + r0;
    uint8_t* S = c.wsmem;
    FOR_GROUPS(c, BN, g) {
      const int j = c.n0 + g;
      float h[32];
      acc1(c, g, h);
      out_free(lane);
      stage_h(S, lane, h);
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = gelu_f(h[i]);
      stage_h(S + 2048, lane, h);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mHc, S, j, yH);
        tc::tma_store_2d(&p.mY3, S + 2048, j, yU);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// R3: du = E W2 -> dH = du gelu'(h) (key rows); du is formed again in E5.
struct EpiR3G {
  static constexpr int kIn = 2048;            // h (bf16)
  static constexpr int kSmem = kIn + 2048;    // | dH (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_2d(c.wsmem, &p.mHc, &c.wbar[0], ga.col, ga.z * 2 * p.d.C + ga.m0 + c.quad * 32);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int yD = c.z * d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* Hs = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float du[32], h[32];
      acc1(c, g, du);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, h);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = du[i] * dgelu_f(h[i]);
      out_free(lane);
      stage_h(Hs, lane, h);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mDH, Hs, j, yD);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// E3: acc0 = E D_M2, acc1 = E D_W2 (columns = hidden units) -> UBd = -(a . + b .)
// (bf16) and dub = dhb gelu'(h) (bf16, rows [0, C) of Y3).
struct EpiE3G {
  static constexpr int kWarps = 4;
  static constexpr int kIn = 4096;           // dhb | h (bf16)
  static constexpr int kSmem = kIn + 4096;   // | UBd | dub (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    const Dims& d = p.d;
    const int r = ga.m0 + c.quad * 32;
    uint64_t* bar = &c.wbar[0];
    tc::mbar_expect_tx(bar, 4096u);
    tc::tma_load_2d(c.wsmem, &p.fDB, bar, ga.col, ga.z * d.C + r);
    tc::tma_load_2d(c.wsmem + 2048, &p.mHc, bar, ga.col, ga.z * 2 * d.C + r);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int t = c.m0 + c.row;
    const size_t tok = (size_t)c.z * d.T + p.t0 + t;
    const float a = t < p.clen ? p.ca[tok] : 0.f, b = t < p.clen ? p.cb[tok] : 0.f;
    const int r0 = c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* F = c.wsmem + kIn;
    uint8_t* Hs = c.wsmem + kIn + 2048;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float m[32], w[32];
      acc2(c, g, m, w);
#pragma unroll
      for (int i = 0; i < 32; ++i) m[i] = -(a * m[i] + b * w[i]);
      out_free(lane);
      stage_h(F, lane, m);
      if (!in_wait(p, c)) return;
      float bh[32];
      unstage_h(IN, lane, bh);
      unstage_h(IN + 2048, lane, w);   // h
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) bh[i] *= dgelu_f(w[i]);
      stage_h(Hs, lane, bh);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.fUBd, F, j, c.z * d.C + r0);
        tc::tma_store_2d(&p.mY3, Hs, j, c.z * 3 * d.C + r0);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// E5: du = E W2 (acc0) and eb W2 (acc1); ub = UBd + eb W2 (MSE); the key rows'
// hb = dhb du gelu''(h) + ub gelu'(h).
struct EpiE5G {
  static constexpr int kWarps = 4;
  static constexpr int kIn = 6144;           // UBd | dhb | h (bf16)
  static constexpr int kSmem = kIn + 2048;   // | hb (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    const Dims& d = p.d;
    const int r = ga.m0 + c.quad * 32;
    const int yC = ga.z * d.C + r, yH = ga.z * 2 * d.C + r;
    uint64_t* bar = &c.wbar[0];
    tc::mbar_expect_tx(bar, 6144u);
    tc::tma_load_2d(c.wsmem, &p.fUBd, bar, ga.col, yC);
    tc::tma_load_2d(c.wsmem + 2048, &p.fDB, bar, ga.col, yC);
    tc::tma_load_2d(c.wsmem + 4096, &p.mHc, bar, ga.col, yH);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int yH = c.z * 2 * d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float acc[32], ubd[32], du[32], bh[32], h[32];
      acc2(c, g, du, acc);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, ubd);
      unstage_h(IN + 2048, lane, bh);
      unstage_h(IN + 4096, lane, h);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float ub = ubd[i] + (d.loss == 0 ? acc[i] : 0.f);
        h[i] = bh[i] * du[i] * d2gelu_f(h[i]) + ub * dgelu_f(h[i]);
      }
      out_free(lane);
      stage_h(OUT, lane, h);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mHB, OUT, j, yH);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// Q1: ub_q = dout W2 -> query-row hb = ub gelu'(h).
struct EpiQ1G {
  static constexpr int kIn = 2048;           // query h (bf16)
  static constexpr int kSmem = kIn + 2048;   // | hb (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_2d(c.wsmem, &p.mHc, &c.wbar[0], ga.col, ga.z * 2 * p.d.C + p.d.C + ga.m0 + c.quad * 32);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int y = c.z * 2 * d.C + d.C + c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, j = c.n0 + g;
      float ub[32], h[32];
      acc1(c, g, ub);
      if (!in_wait(p, c)) return;
      unstage_h(IN, lane, h);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = ub[i] * dgelu_f(h[i]);
      out_free(lane);
      stage_h(OUT, lane, h);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.mHB, OUT, j, y);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// dk part 1: -(a dH D_M13 + b dH D_W13) -> dkp (bf16).
struct EpiDk1 {
  static constexpr int kSmem = 2048;  // dkp staging (bf16)
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int t = c.m0 + c.row;
    const size_t tok = (size_t)c.z * d.T + p.t0 + t;
    const float a = t < p.clen ? p.ca[tok] : 0.f, b = t < p.clen ? p.cb[tok] : 0.f;
    const int y = c.z * d.C + c.m0 + c.quad * 32;
    uint8_t* F = c.wsmem;
    FOR_GROUPS(c, BN, g) {
      float m[32], w[32];
      acc2(c, g, m, w);
#pragma unroll
      for (int i = 0; i < 32; ++i) m[i] = -(a * m[i] + b * w[i]);
      out_free(lane);
      stage_h(F, lane, m);
      out_ready();
      if (lane == 0) {
        tc::tma_store_2d(&p.fdkp, F, c.n0 + g, y);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// dk part 2 (adds part 1) and dq: [h1b | h3b] [W1; W3] -> the activation-dtype output.
template <bool KEYS>
struct EpiDkq {
  static constexpr int kIn = KEYS ? 2048 : 0;  // dkp (bf16)
  static constexpr int kSmem = kIn + 2048;     // | dk or dq (bf16)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 2048u);
    tc::tma_load_2d(c.wsmem, &p.fdkp, &c.wbar[0], ga.col, ga.z * p.d.C + ga.m0 + c.quad * 32);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const int tO = p.t0 + c.m0 + c.quad * 32;
    const bool any_real = c.m0 + c.quad * 32 < p.clen;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (KEYS && c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32, col = c.n0 + g;
      float x[32];
      acc1(c, g, x);
      if (KEYS) {
        float y[32];
        if (!in_wait(p, c)) return;
        unstage_h(IN, lane, y);
        __syncwarp();
        if (lane == 0) {
          tc::fence_async_smem();
          issue(p, c, gi + 1);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] += y[i];
      }
      out_free(lane);
      stage_h(OUT, lane, x);
      out_ready();
      if (lane == 0) {
        if (any_real) tc::tma_store_3d(KEYS ? &p.mdk : &p.mdq, OUT, col, tO, c.z);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};
// dW: D_W <- L(1,n) D_W + acc in place, class 0 = rows of [W1; W3], class 1 = rows
// of W2; the fp32 rows of D_W move through shared memory with TMA.
struct EpiDW {
  static constexpr int kIn = 4096;           // D_W block (fp32)
  static constexpr int kSmem = kIn + 4096;   // | updated block (fp32)
  template <int BN>
  static __device__ __forceinline__ void issue(const BwdP& p, const EpiCtx<BN>& c, int gi) {
    const GroupAt ga = group_at(c, gi);
    if (!ga.valid) return;
    tc::mbar_expect_tx(&c.wbar[0], 4096u);
    tc::tma_load_3d(c.wsmem, &p.fDW[ga.cls], &c.wbar[0], ga.col, ga.m0 + c.quad * 32, ga.z);
  }
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int lane = c.row & 31;
    const int per = BN / c.nparts, ngroups = per / 32;
    const size_t plane = (size_t)d.BH * d.NC;
    const float PL = p.scal[plane + (size_t)c.z * d.NC + p.ci];
    const int r0 = c.m0 + c.quad * 32;
    const uint8_t* IN = c.wsmem;
    uint8_t* OUT = c.wsmem + kIn;
    if (c.iter == 0 && lane == 0) issue(p, c, 0);
    __syncwarp();
    for (int gi = 0; gi < ngroups; ++gi) {
      const int g = c.part * per + gi * 32;
      float x[32], y[32];
      acc1(c, g, x);
      if (!in_wait(p, c)) return;
      unstage_f(IN, lane, y);
      __syncwarp();
      if (lane == 0) {
        tc::fence_async_smem();
        issue(p, c, gi + 1);
      }
#pragma unroll
      for (int q = 0; q < 32; ++q) y[q] = PL * y[q] + x[q];
      out_free(lane);
      stage_f(OUT, lane, y);
      out_ready();
      if (lane == 0) {
        tc::tma_store_3d(&p.fDW[c.cls], OUT, c.n0 + g, r0, c.z);
        tc::bulk_commit();
      }
      __syncwarp();
    }
  }
};

template <class Epi> struct Name { static constexpr const char* v = "tc_bwd"; };
template <> struct Name<EpiR1> { static constexpr const char* v = "tcb_r1_h"; };
template <> struct Name<EpiR2> { static constexpr const char* v = "tcb_r2_e"; };
template <> struct Name<EpiR3> { static constexpr const char* v = "tcb_r3_du"; };
template <> struct Name<EpiD1> { static constexpr const char* v = "tcb_d1_dir13"; };
template <> struct Name<EpiD2> { static constexpr const char* v = "tcb_d2_dir2"; };
template <> struct Name<EpiE3> { static constexpr const char* v = "tcb_e3_ub_dub"; };
template <> struct Name<EpiE4> { static constexpr const char* v = "tcb_e4_eb"; };
template <> struct Name<EpiE5> { static constexpr const char* v = "tcb_e5_hb"; };
template <> struct Name<EpiQ1> { static constexpr const char* v = "tcb_q1_hbq"; };
template <> struct Name<EpiDk1> { static constexpr const char* v = "tcb_dk1"; };
template <> struct Name<EpiDkq<true>> { static constexpr const char* v = "tcb_dk2"; };
template <> struct Name<EpiDkq<false>> { static constexpr const char* v = "tcb_dq"; };
template <> struct Name<EpiDW> { static constexpr const char* v = "tcb_dw"; };
template <> struct Name<EpiR1G> { static constexpr const char* v = "tcb_r1_h"; };
template <> struct Name<EpiR3G> { static constexpr const char* v = "tcb_r3_du"; };
template <> struct Name<EpiE3G> { static constexpr const char* v = "tcb_e3_ub_dub"; };
template <> struct Name<EpiE5G> { static constexpr const char* v = "tcb_e5_hb"; };
template <> struct Name<EpiQ1G> { static constexpr const char* v = "tcb_q1_hbq"; };

// ---------------------------------------------------------------- elementwise kernels
// bf16 copies of the chunk-start weights and of the state adjoints, each split
// into a [W1; W3] block [BH, 2 d_h, d_k] (GELU: W1, [BH, d_h, d_k]) and a W2 block
// [BH, d_v, d_h]; the
// partial sums of <D_M, M0>, <D_W, W0>, <D_W, M0> (64 blocks per head); and,
// once the old D_M is read, D_M <- U(1,n) D_M + c D_W in place (the chunk-start
// adjoint of M; the GEMM phases read only the bf16 copies).
__device__ __forceinline__ void shadow4(const float4 w, const float4 m, const float4 a, const float4 b,
                                        long long i, long long n13, long long S, int z, bf16* W13,
                                        bf16* W2, bf16* DW13, bf16* DW2, bf16* DM13, bf16* DM2,
                                        float& s0, float& s1, float& s2) {
  s0 += b.x * m.x + b.y * m.y + b.z * m.z + b.w * m.w;
  s1 += a.x * w.x + a.y * w.y + a.z * w.z + a.w * w.w;
  s2 += a.x * m.x + a.y * m.y + a.z * m.z + a.w * m.w;
  size_t o;
  bf16 *pw, *pa, *pb;
  if (i < n13) {
    o = (size_t)z * n13 + i;
    pw = W13 + o; pa = DW13 + o; pb = DM13 + o;
  } else {
    o = (size_t)z * (S - n13) + (i - n13);
    pw = W2 + o; pa = DW2 + o; pb = DM2 + o;
  }
  *reinterpret_cast<uint2*>(pw) = make_uint2(pack2(w.x, w.y), pack2(w.z, w.w));
  *reinterpret_cast<uint2*>(pa) = make_uint2(pack2(a.x, a.y), pack2(a.z, a.w));
  *reinterpret_cast<uint2*>(pb) = make_uint2(pack2(b.x, b.y), pack2(b.z, b.w));
}
__global__ void __launch_bounds__(256, 4) bwd_shadow_kernel(  // 4 blocks (64 registers) per SM
    const float* __restrict__ W0, const float* __restrict__ M0, long long sst,
    const float* __restrict__ DW, float* __restrict__ DM, bf16* W13, bf16* W2, bf16* DW13,
    bf16* DW2, bf16* DM13, bf16* DM2, float* part, const float* __restrict__ scal, Dims d, int ci) {
  griddep_launch_dependents();  // the next kernel's set-up may start
  const int z = blockIdx.y, blk = blockIdx.x;
  const long long S = d.S, n13 = (d.kind == 1 ? 2LL : 1LL) * d.d_h * d.d_k;
  const size_t plane = (size_t)d.BH * d.NC, so = (size_t)z * d.NC + ci;
  const float U = scal[so], cc = scal[2 * plane + so];
  const float4* w0 = reinterpret_cast<const float4*>(W0 + z * sst);
  const float4* m0 = reinterpret_cast<const float4*>(M0 + z * sst);
  const float4* dw = reinterpret_cast<const float4*>(DW + z * S);
  float4* dm = reinterpret_cast<float4*>(DM + z * S);
  float s0 = 0.f, s1 = 0.f, s2 = 0.f;
  const long long n4 = S / 4, step = (long long)gridDim.x * blockDim.x;
  long long i4 = (long long)blk * blockDim.x + threadIdx.x;
  // two float4 groups per thread and iteration: eight 16-byte loads in flight
  for (; i4 + step < n4; i4 += 2 * step) {
    const long long j4 = i4 + step;
    const float4 w = w0[i4], m = m0[i4], a = dw[i4], b = dm[i4];
    const float4 w2 = w0[j4], m2 = m0[j4], a2 = dw[j4], b2 = dm[j4];
    dm[i4] = make_float4(U * b.x + cc * a.x, U * b.y + cc * a.y, U * b.z + cc * a.z, U * b.w + cc * a.w);
    dm[j4] = make_float4(U * b2.x + cc * a2.x, U * b2.y + cc * a2.y, U * b2.z + cc * a2.z,
                         U * b2.w + cc * a2.w);
    shadow4(w, m, a, b, i4 * 4, n13, S, z, W13, W2, DW13, DW2, DM13, DM2, s0, s1, s2);
    shadow4(w2, m2, a2, b2, j4 * 4, n13, S, z, W13, W2, DW13, DW2, DM13, DM2, s0, s1, s2);
  }
  if (i4 < n4) {
    const float4 w = w0[i4], m = m0[i4], a = dw[i4], b = dm[i4];
    dm[i4] = make_float4(U * b.x + cc * a.x, U * b.y + cc * a.y, U * b.z + cc * a.z, U * b.w + cc * a.w);
    shadow4(w, m, a, b, i4 * 4, n13, S, z, W13, W2, DW13, DW2, DM13, DM2, s0, s1, s2);
  }
  __shared__ float red[3][256];
  red[0][threadIdx.x] = s0;
  red[1][threadIdx.x] = s1;
  red[2][threadIdx.x] = s2;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o)
      for (int q = 0; q < 3; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0)
    for (int q = 0; q < 3; ++q) part[((size_t)q * d.BH + z) * 64 + blk] = red[q][0];  // blk < 64
}
// Sum over the 32 lanes of a warp in a fixed order (butterfly), every lane
// receiving the total.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}
// The chunk's sums, one warp each, the lanes reading consecutive partials in a
// fixed order: warps [0, BH C) form abar_t, bbar_t = -(sum of the row's partial
// dot products of D1 and D2); the next 3 BH warps the chunk-scalar adjoints
// from the shadow pass's partials (nb per head and scalar).
__global__ void bwd_sums_kernel(const float* part, float* abar, float* bbar, const float* spart,
                                float* sbar, Dims d, int ci, int t0, int clen, int NG, int nb) {
  griddep_launch_dependents();  // the next kernel's set-up may start
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)d.BH * d.C;
  if (r >= rows) {
    const int w = (int)(r - rows);
    if (w >= 3 * d.BH) return;  // warp-uniform
    const int q = w / d.BH, z = w - q * d.BH;
    const float* pp = spart + ((size_t)q * d.BH + z) * 64;
    float s = 0.f;
    for (int b = lane; b < nb; b += 32) s += pp[b];
    s = warp_sum(s);
    if (lane == 0) {
      const size_t plane = (size_t)d.BH * d.NC, o = (size_t)z * d.NC + ci;
      sbar[q * plane + o] = s;
    }
    return;
  }
  const int z = (int)(r / d.C), t = (int)(r % d.C);
  if (t >= clen) return;  // padding of a shorter last chunk (warp-uniform)
  const float* pa = part + (size_t)r * NG;
  const float* pb = pa + (size_t)d.BH * d.C * NG;
  float sa = 0.f, sb = 0.f;
  for (int g = lane; g < NG; g += 32) {
    sa += pa[g];
    sb += pb[g];
  }
  sa = warp_sum(sa);
  sb = warp_sum(sb);
  if (lane == 0) {
    abar[(size_t)z * d.T + t0 + t] = -sa;
    bbar[(size_t)z * d.T + t0 + t] = -sb;
  }
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
// 2-D bf16 map over [rows, cols]; box 64 columns x box_rows, 128B swizzle.
bool mk(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
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
// 2-D map, box 32 columns x 32 rows: bf16 with 64B swizzle, fp32 with 128B swizzle
// (the epilogues' staged I/O).
bool box32(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, bool f32) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * es};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t el[2] = {1, 1};
  return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, el, CU_TENSOR_MAP_INTERLEAVE_NONE,
            f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D bf16 map over per-head token rows [heads][T][cols], box 32 x 32 x 1, 64B
// swizzle: rows past a head's T read as zero and are clipped on store.
bool tok_box32(CUtensorMap* m, const void* base, uint64_t T, uint64_t cols, uint64_t heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, T, heads};
  cuuint64_t strides[2] = {cols * 2, T * cols * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t el[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, el,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// 3-D fp32 map over [heads, rows, cols] of one block of every head's state
// (head stride S), box 32 x 32 x 1, 128B swizzle.
bool state_box32(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols, uint64_t heads,
                 uint64_t head_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, rows, heads};
  cuuint64_t strides[2] = {cols * 4, head_stride * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t el[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, el,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}
// Per-epilogue launch shape: shared memory per epilogue warp (kSmem, default 0)
// and epilogue warps (kWarps, default 8).
template <class E, class = void>
struct EpiSmemOf { static constexpr int v = 0; };
template <class E>
struct EpiSmemOf<E, std::void_t<decltype(E::kSmem)>> { static constexpr int v = E::kSmem; };
template <class E, class = void>
struct EpiWarpsOf { static constexpr int v = kEW; };
template <class E>
struct EpiWarpsOf<E, std::void_t<decltype(E::kWarps)>> { static constexpr int v = E::kWarps; };

// Two independent GEMM phases of a chunk in one launch (one launch ramp instead
// of two): class 0 tiles run E0's epilogue, class 1 tiles E1's. All class-0
// tiles precede the class-1 tiles in the tile order, so a CTA switches class at
// most once. The epilogues chain their input loads from tile to tile within a
// class only: a class-0 tile whose successor is of class 1 requests nothing for
// it, and a CTA's first class-1 tile starts its own chain. The launch has E0's
// epilogue warp count; the epilogues split a tile's columns over however many
// warps there are.
template <class E0, class E1>
struct EpiPair {
  static constexpr int kWarps = EpiWarpsOf<E0>::v;
  static constexpr int kSmem = EpiSmemOf<E0>::v > EpiSmemOf<E1>::v ? EpiSmemOf<E0>::v : EpiSmemOf<E1>::v;
  template <int BN>
  static __device__ void run(const BwdP& p, const EpiCtx<BN>& c) {
    EpiCtx<BN> x = c;
    if (x.nxt_valid && x.nxt_cls != x.cls) x.nxt_valid = 0;
    if (c.cls == 0) {
      E0::run(p, x);
    } else {
      const int t = (int)blockIdx.x + c.iter * (int)gridDim.x;  // this tile's index
      if (t - (int)gridDim.x < p.per0) x.iter = 0;              // the CTA's first class-1 tile
      E1::run(p, x);
    }
  }
};
template <> struct Name<EpiPair<EpiR3, EpiQ1>> { static constexpr const char* v = "tcb_r3_q1"; };
template <> struct Name<EpiPair<EpiR3G, EpiQ1G>> { static constexpr const char* v = "tcb_r3_q1"; };
template <> struct Name<EpiPair<EpiD1, EpiD2>> { static constexpr const char* v = "tcb_d1_d2"; };
template <> struct Name<EpiPair<EpiE3, EpiDk1>> { static constexpr const char* v = "tcb_e3_dk1"; };
template <> struct Name<EpiPair<EpiE3G, EpiDk1>> { static constexpr const char* v = "tcb_e3_dk1"; };
template <> struct Name<EpiPair<EpiDkq<true>, EpiDkq<false>>> { static constexpr const char* v = "tcb_dk2_dq"; };

template <int NUM_ACC, bool A_MN, bool B_MN, class Epi, int BN = 128>
cudaError_t run_gemm(tc2::Job& job, const BwdP& p, cudaStream_t st) {
  constexpr int EW = EpiWarpsOf<Epi>::v;
  constexpr int ESM = EpiSmemOf<Epi>::v;
  constexpr uint32_t kStage = tc2::Cfg<BN, NUM_ACC, A_MN, B_MN>::kStage;
  // Epilogues without staging buffers: two 64-wide k-blocks per ring slot (one
  // producer/MMA handshake per 128 of K). With staging: single k-block slots, as
  // many (up to 4) as the shared memory left over holds.
  constexpr int KG = ESM == 0 ? 2 : 1;
  constexpr long long kFree = 232448LL - 1024 - 256 - 8LL * tc2::kEpiBars * EW - (long long)EW * ESM;
  constexpr int kFit = (int)(kFree / ((long long)KG * kStage));
  constexpr int STAGES = ESM == 0 ? (NUM_ACC == 1 ? 3 : 2) : (kFit > 4 ? 4 : kFit);
  static_assert(STAGES >= 2, "at least two ring slots");
  constexpr size_t smem = tc2::smem_bytes<BN, NUM_ACC, A_MN, B_MN, STAGES, EW, ESM, KG>();
  static_assert(smem <= 232448, "shared memory per CTA");
  auto kern = tc2::gemm_persistent<BN, NUM_ACC, A_MN, B_MN, STAGES, EW, Epi, BwdP, ESM, KG>;
  job.total_tiles = 0;
  for (int c = 0; c < job.n_cls; ++c) {
    if (job.cls[c].kblocks % KG != 0) return cudaErrorInvalidValue;
    job.total_tiles += job.cls[c].tiles_m * job.cls[c].tiles_n * job.heads;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = job.total_tiles < num_sms() ? job.total_tiles : num_sms();
  E2TTT_TRACE(Name<Epi>::v, st);
  return launch_pdl(kern, dim3(grid), dim3((2 + EW) * 32), smem, st, job, p);
}

struct Buf {
  int* status;
  bf16 *X, *Y3, *Z3, *Hc, *DH, *HB, *W13, *W2, *DW13, *DW2, *DM13, *DM2;
  float *a, *b, *scal, *abar, *bbar, *sbar, *spart, *part;
  bf16 *DB, *G2U, *UBd, *dkp;
  size_t total;
};
Buf carve(const Dims& d, char* base) {
  Buf B{};
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* p = base ? base + off : nullptr;
    off = (off + bytes + 255) & ~size_t(255);
    return p;
  };
  const size_t BH = d.BH, C = d.C, dk = d.d_k, dv = d.d_v, dh = d.d_h, h = 2, f = 4;
  const size_t hw = (d.kind == 1 ? 2 : 1) * dh;  // SwiGLU h1 | h3, GELU h
  const int NG = (int)(hw / 32 + dv / 32);
  B.status = (int*)take(256);  // first bytes of the workspace (read by e2ttt_workspace_status)
  B.a = (float*)take(BH * d.T * f);
  B.b = (float*)take(BH * d.T * f);
  B.scal = (float*)take(3 * BH * d.NC * f);
  B.abar = (float*)take(BH * d.T * f);
  B.bbar = (float*)take(BH * d.T * f);
  B.sbar = (float*)take(3 * BH * d.NC * f);
  B.spart = (float*)take(3 * BH * 64 * f);
  B.X = (bf16*)take(BH * 2 * C * dk * h);
  B.Y3 = (bf16*)take(BH * 3 * C * dh * h);
  B.Z3 = (bf16*)take(BH * 3 * C * dv * h);
  B.Hc = (bf16*)take(BH * 2 * C * hw * h);
  B.DH = (bf16*)take(BH * C * hw * h);
  B.HB = (bf16*)take(BH * 2 * C * hw * h);
  B.W13 = (bf16*)take(BH * hw * dk * h);
  B.W2 = (bf16*)take(BH * dv * dh * h);
  B.DW13 = (bf16*)take(BH * hw * dk * h);
  B.DW2 = (bf16*)take(BH * dv * dh * h);
  B.DM13 = (bf16*)take(BH * hw * dk * h);
  B.DM2 = (bf16*)take(BH * dv * dh * h);
  B.DB = (bf16*)take(BH * C * hw * h);
  B.G2U = (bf16*)take(BH * C * dv * h);
  B.UBd = (bf16*)take(BH * C * dh * h);
  B.dkp = (bf16*)take(BH * C * dk * h);
  B.part = (float*)take(2 * BH * C * NG * f);
  B.total = off;
  return B;
}

tc2::Class cls(int tm, int tn, int kb, tc2::Opnd a, tc2::Opnd b, int mode = 0) {
  return tc2::Class{tm, tn, kb, a, b, mode};
}

}  // namespace

bool tc_bwd_supported(const Dims& d, bool bf16_act) {
  return (d.kind == 1 || d.kind == 2) && tc_fwd_supported(d, bf16_act);
}
size_t tc_bwd_workspace_bytes(const Dims& d) { return carve(d, nullptr).total; }

cudaError_t tc_bwd(const BwdArgs& A) {
  const Dims& d = A.d;
  const int BH = d.BH, T = d.T, C = d.C, NC = d.NC, dk = d.d_k, dv = d.d_v, dh = d.d_h;
  Buf B = carve(d, (char*)A.ws);
  cudaStream_t st = A.st;
  const size_t sbytes = (size_t)BH * d.S * sizeof(float);
  cudaError_t e = cudaMemsetAsync(B.status, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  e = launch_chunk_coeffs(A.lr, A.mom, A.decay, B.a, B.b, B.scal, BH, T, C, NC, d.coef, st);
  if (e != cudaSuccess) return e;
  e = A.dW_end ? cudaMemcpyAsync(A.dW0, A.dW_end, sbytes, cudaMemcpyDeviceToDevice, st)
               : cudaMemsetAsync(A.dW0, 0, sbytes, st);
  if (e == cudaSuccess)
    e = A.dM_end ? cudaMemcpyAsync(A.dM0, A.dM_end, sbytes, cudaMemcpyDeviceToDevice, st)
                 : cudaMemsetAsync(A.dM0, 0, sbytes, st);
  if (e != cudaSuccess) return e;

  BwdP p{};
  p.d = d;
  p.v = (const bf16*)A.v;
  p.dq = (bf16*)A.dq; p.dk = (bf16*)A.dk; p.dv = (bf16*)A.dv;
  p.ca = B.a; p.cb = B.b; p.scal = B.scal;
  p.DW = A.dW0; p.DM = A.dM0;
  p.X = B.X; p.Y3 = B.Y3; p.Z3 = B.Z3; p.Hc = B.Hc; p.DH = B.DH; p.HB = B.HB;
  p.DB = B.DB; p.G2U = B.G2U; p.UBd = B.UBd; p.dkp = B.dkp; p.part = B.part;
  const bool gelu = d.kind == 2;
  const int hw = (gelu ? 1 : 2) * dh;  // columns of the first state block's hidden side
  p.hw = hw;
  p.NG = hw / 32 + dv / 32;
  p.status = B.status;
  {
    const uint64_t rC = (uint64_t)BH * C;
    bool mok = box32(&p.mHc, B.Hc, 2 * rC, hw, false);
    mok &= box32(&p.mY3, B.Y3, 3 * rC, dh, false);
    mok &= box32(&p.mDH, B.DH, rC, hw, false);
    mok &= box32(&p.mHB, B.HB, 2 * rC, hw, false);
    mok &= box32(&p.fDB, B.DB, rC, hw, false);
    mok &= box32(&p.fUBd, B.UBd, rC, dh, false);
    mok &= box32(&p.mZ3, B.Z3, 3 * rC, dv, false);
    mok &= tok_box32(&p.mv, A.v, T, dv, BH);
    mok &= tok_box32(&p.mdv, A.dv, T, dv, BH);
    mok &= tok_box32(&p.mdk, A.dk, T, dk, BH);
    mok &= tok_box32(&p.mdq, A.dq, T, dk, BH);
    mok &= box32(&p.fG2U, B.G2U, rC, dv, false);
    mok &= box32(&p.fdkp, B.dkp, rC, dk, false);
    mok &= state_box32(&p.fDW[0], A.dW0, hw, dk, BH, d.S);
    mok &= state_box32(&p.fDW[1], A.dW0 + (size_t)hw * dk, dv, dh, BH, d.S);
    if (!mok) return cudaErrorInvalidValue;
  }

  // operand maps (per call; the chunk only changes the copies and the epilogue data)
  tc2::Job r1{}, r2{}, r3{}, d1{}, d2{}, e3{}, e4{}, e5{}, q1{}, k1{}, k2{}, dq{}, dw{};
  bool ok = true;
  const uint64_t rX = (uint64_t)BH * 2 * C, rY = (uint64_t)BH * 3 * C, rZ = rY;
  const uint64_t rH = (uint64_t)BH * 2 * C, rD = (uint64_t)BH * C;
  const uint64_t r13 = (uint64_t)BH * hw, r2w = (uint64_t)BH * dv;
  for (tc2::Job* j : {&r1, &r2, &r3, &d1, &d2, &e3, &e4, &e5, &q1, &k1, &k2, &dq, &dw}) {
    j->heads = BH;
    j->n_cls = 1;
    j->status = B.status;
  }
  // R1: X [2C x dk] x {W1, W3}^T (two B operands; GELU: W1 alone)
  ok &= mk(&r1.maps[0].op0, B.X, rX, dk, 128);
  if (gelu) {
    ok &= mk(&r1.maps[0].op2, B.W13, r13, dk, 128);
    r1.cls[0] = cls(2 * C / 128, dh / 128, dk / 64, {2 * C, 0, 0}, {hw, 0, 0});
  } else {
    ok &= mk(&r1.maps[0].op1, B.W13, r13, dk, 128);
    ok &= mk(&r1.maps[0].op2, B.W13 + (size_t)dh * dk, r13 - dh, dk, 128);
    r1.cls[0] = cls(2 * C / 128, dh / 128, dk / 64, {2 * C, 0, 0}, {hw, 0, 0}, tc2::kModeA1B2);
  }
  // R2: U_k (rows [C, 2C) of Y3) x W2^T
  ok &= mk(&r2.maps[0].op0, B.Y3, rY, dh, 128);
  ok &= mk(&r2.maps[0].op2, B.W2, r2w, dh, 128);
  r2.cls[0] = cls(C / 128, dv / 128, dh / 64, {3 * C, C, 0}, {dv, 0, 0});
  // R3: E (rows [0, C) of Z3) x W2 (MN-major)
  ok &= mk(&r3.maps[0].op0, B.Z3, rZ, dv, 128);
  ok &= mk(&r3.maps[0].op2, B.W2, r2w, dh, 64);
  r3.cls[0] = cls(C / 128, dh / 128, dv / 64, {3 * C, 0, 0}, {dv, 0, 0});
  // D1: keys (rows [0, C) of X) x {D_M13, D_W13}^T
  ok &= mk(&d1.maps[0].op0, B.X, rX, dk, 128);
  ok &= mk(&d1.maps[0].op1, B.DM13, r13, dk, 128);
  ok &= mk(&d1.maps[0].op2, B.DW13, r13, dk, 128);
  d1.cls[0] = cls(C / 128, hw / 128, dk / 64, {2 * C, 0, 0}, {hw, 0, 0}, tc2::kModeA1B2);
  // D2: U_k x {D_M2, D_W2}^T
  ok &= mk(&d2.maps[0].op0, B.Y3, rY, dh, 128);
  ok &= mk(&d2.maps[0].op1, B.DM2, r2w, dh, 128);
  ok &= mk(&d2.maps[0].op2, B.DW2, r2w, dh, 128);
  d2.cls[0] = cls(C / 128, dv / 128, dh / 64, {3 * C, C, 0}, {dv, 0, 0}, tc2::kModeA1B2);
  // E3: E x {D_M2, D_W2} (MN-major)
  ok &= mk(&e3.maps[0].op0, B.Z3, rZ, dv, 128);
  ok &= mk(&e3.maps[0].op1, B.DM2, r2w, dh, 64);
  ok &= mk(&e3.maps[0].op2, B.DW2, r2w, dh, 64);
  e3.cls[0] = cls(C / 128, dh / 128, dv / 64, {3 * C, 0, 0}, {dv, 0, 0}, tc2::kModeA1B2);
  // E4: dub (rows [0, C) of Y3) x W2^T
  ok &= mk(&e4.maps[0].op0, B.Y3, rY, dh, 128);
  ok &= mk(&e4.maps[0].op2, B.W2, r2w, dh, 128);
  e4.cls[0] = cls(C / 128, dv / 128, dh / 64, {3 * C, 0, 0}, {dv, 0, 0});
  // E5: [E; EB] (rows [0, C) and [C, 2C) of Z3; the second map starts C rows
  // into Z3, so both A operands share one set of coordinates) x W2 (MN-major);
  // Q1: dout (rows [2C, 3C)) x W2
  ok &= mk(&e5.maps[0].op0, B.Z3, rZ, dv, 128);
  ok &= mk(&e5.maps[0].op1, B.Z3 + (size_t)C * dv, rZ - C, dv, 128);
  ok &= mk(&e5.maps[0].op2, B.W2, r2w, dh, 64);
  e5.cls[0] = cls(C / 128, dh / 128, dv / 64, {3 * C, 0, 0}, {dv, 0, 0}, tc2::kModeA2B1);
  q1.maps[0] = e5.maps[0];
  q1.cls[0] = cls(C / 128, dh / 128, dv / 64, {3 * C, 2 * C, 0}, {dv, 0, 0});
  // dk1: dH x {D_M13, D_W13} (MN-major: N = d_k, K = 2 d_h)
  ok &= mk(&k1.maps[0].op0, B.DH, rD, hw, 128);
  ok &= mk(&k1.maps[0].op1, B.DM13, r13, dk, 64);
  ok &= mk(&k1.maps[0].op2, B.DW13, r13, dk, 64);
  k1.cls[0] = cls(C / 128, dk / 128, hw / 64, {C, 0, 0}, {hw, 0, 0}, tc2::kModeA1B2);
  // dk2 / dq: [h1b | h3b] (rows [0, C) / [C, 2C) of HB) x [W1; W3] (MN-major)
  ok &= mk(&k2.maps[0].op0, B.HB, rH, hw, 128);
  ok &= mk(&k2.maps[0].op2, B.W13, r13, dk, 64);
  k2.cls[0] = cls(C / 128, dk / 128, hw / 64, {2 * C, 0, 0}, {hw, 0, 0});
  dq.maps[0] = k2.maps[0];
  dq.cls[0] = cls(C / 128, dk / 128, hw / 64, {2 * C, C, 0}, {hw, 0, 0});
  // dW: class 0 = [h1b | h3b]^T [K; Q] (2C tokens), class 1 = [E; EB; dout]^T [dub; u_k; u_q]
  ok &= mk(&dw.maps[0].op0, B.HB, rH, hw, 64);
  ok &= mk(&dw.maps[0].op2, B.X, rX, dk, 64);
  ok &= mk(&dw.maps[1].op0, B.Z3, rZ, dv, 64);
  ok &= mk(&dw.maps[1].op2, B.Y3, rY, dh, 64);
  dw.n_cls = 2;
  // 128 x 256 tiles where d_k and d_h allow and they still fill every SM: a
  // quarter fewer operand bytes per FLOP than 128 x 128 (the phase streams its
  // operands from L2) and 512-cycle MMAs per ring slot
  const int dwn = dk % 256 == 0 && dh % 256 == 0 && BH * (hw / 128 * dk / 256 + dv / 128 * dh / 256) >= num_sms()
                      ? 256 : 128;
  dw.cls[0] = cls(hw / 128, dk / dwn, 2 * C / 64, {2 * C, 0, 0}, {2 * C, 0, 0});
  dw.cls[1] = cls(dv / 128, dh / dwn, 3 * C / 64, {3 * C, 0, 0}, {3 * C, 0, 0});
  if (!ok) return cudaErrorInvalidValue;
  // two-phase launches: R3 with Q1 (both x W2), D1 with D2 and E3 with dk1 (both
  // two-accumulator products with the bf16 state adjoints), dk2 with dq
  auto pair = [](const tc2::Job& j0, const tc2::Job& j1) {
    tc2::Job j = j0;
    j.n_cls = 2;
    j.maps[1] = j1.maps[0];
    j.cls[1] = j1.cls[0];
    return j;
  };
  tc2::Job r3q1 = pair(r3, q1), d12 = pair(d1, d2), e3k1 = pair(e3, k1), kq = pair(k2, dq);
  auto tiles0 = [](const tc2::Job& j) { return j.cls[0].tiles_m * j.cls[0].tiles_n * j.heads; };

  const size_t per_chunk = (size_t)BH * 2 * d.S;
  const Dims dd = d;
  // blocks per head of the shadow kernel: one resident wave (4 blocks per SM)
  // over all heads, at most 64 (the partial-sum slots per head); fixed for a
  // given device, so the partial sums keep their order from call to call
  const int shadow_nb = std::max(1, std::min(64, 4 * num_sms() / BH));
  for (int ci = NC - 1; ci >= 0; --ci) {
    const int t0 = ci * C;
    const int cl = T - t0 < C ? T - t0 : C;  // tokens of this chunk
    p.ci = ci;
    p.t0 = t0;
    p.clen = cl;
    const float* W0 = A.saved + ci * per_chunk;
    const float* M0 = W0 + d.S;
    // chunk rows of keys, queries, dout into the stacked operands (zero padding
    // rows after a shorter last chunk's tokens)
    e = cudaMemcpy2DAsync(B.X, (size_t)2 * C * dk * 2, (const bf16*)A.k + (size_t)t0 * dk,
                          (size_t)T * dk * 2, (size_t)cl * dk * 2, BH, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(B.X + (size_t)C * dk, (size_t)2 * C * dk * 2,
                            (const bf16*)A.q + (size_t)t0 * dk, (size_t)T * dk * 2, (size_t)cl * dk * 2,
                            BH, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(B.Z3 + (size_t)2 * C * dv, (size_t)3 * C * dv * 2,
                            (const bf16*)A.dout + (size_t)t0 * dv, (size_t)T * dv * 2,
                            (size_t)cl * dv * 2, BH, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && A.acts_e) {
      // saved activations: the forward's E of this chunk into rows [0, C) of Z3
      // (its padding rows are zero), its dH read in place
      const bf16* Ec = A.acts_e + (size_t)ci * BH * C * dv;
      const bf16* Dc = A.acts_dh + (size_t)ci * BH * C * hw;
      e = cudaMemcpy2DAsync(B.Z3, (size_t)3 * C * dv * 2, Ec, (size_t)C * dv * 2, (size_t)C * dv * 2, BH,
                            cudaMemcpyDeviceToDevice, st);
      bool mok = box32(&p.mDH, Dc, (uint64_t)BH * C, hw, false);
      mok &= mk(&k1.maps[0].op0, Dc, rD, hw, 128);
      if (!mok) return cudaErrorInvalidValue;
      e3k1 = pair(e3, k1);
    }
    if (e == cudaSuccess && cl < C) {
      const size_t pk = (size_t)(C - cl) * dk * 2, pv = (size_t)(C - cl) * dv * 2;
      e = cudaMemset2DAsync(B.X + (size_t)cl * dk, (size_t)2 * C * dk * 2, 0, pk, BH, st);
      if (e == cudaSuccess)
        e = cudaMemset2DAsync(B.X + (size_t)(C + cl) * dk, (size_t)2 * C * dk * 2, 0, pk, BH, st);
      if (e == cudaSuccess)
        e = cudaMemset2DAsync(B.Z3 + (size_t)(2 * C + cl) * dv, (size_t)3 * C * dv * 2, 0, pv, BH, st);
    }
    if (e != cudaSuccess) return e;
    {
      E2TTT_TRACE("tcb_shadow", st);
      bwd_shadow_kernel<<<dim3(shadow_nb, BH), 256, 0, st>>>(W0, M0, 2 * d.S, A.dW0, A.dM0, B.W13,
                                                              B.W2, B.DW13, B.DW2, B.DM13, B.DM2,
                                                              B.spart, B.scal, dd, ci);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    using tc2::kModeA1B2;
    e = gelu ? run_gemm<1, false, false, EpiR1G>(r1, p, st) : run_gemm<2, false, false, EpiR1>(r1, p, st);
    if (e != cudaSuccess) return e;
    if (A.acts_e) {
      // E and dH come from the forward: no R2, and of R3 + Q1 only Q1
      e = gelu ? run_gemm<1, false, true, EpiQ1G>(q1, p, st) : run_gemm<1, false, true, EpiQ1>(q1, p, st);
      if (e != cudaSuccess) return e;
    } else {
      if ((e = run_gemm<1, false, false, EpiR2>(r2, p, st)) != cudaSuccess) return e;
      p.per0 = tiles0(r3q1);
      e = gelu ? run_gemm<1, false, true, EpiPair<EpiR3G, EpiQ1G>>(r3q1, p, st)
               : run_gemm<1, false, true, EpiPair<EpiR3, EpiQ1>>(r3q1, p, st);
      if (e != cudaSuccess) return e;
    }
    p.per0 = tiles0(d12);
    if ((e = run_gemm<2, false, false, EpiPair<EpiD1, EpiD2>>(d12, p, st)) != cudaSuccess) return e;
    p.per0 = tiles0(e3k1);
    e = gelu ? run_gemm<2, false, true, EpiPair<EpiE3G, EpiDk1>>(e3k1, p, st)
             : run_gemm<2, false, true, EpiPair<EpiE3, EpiDk1>>(e3k1, p, st);
    if (e != cudaSuccess) return e;
    if ((e = run_gemm<1, false, false, EpiE4>(e4, p, st)) != cudaSuccess) return e;
    e = gelu ? run_gemm<2, false, true, EpiE5G>(e5, p, st) : run_gemm<2, false, true, EpiE5>(e5, p, st);
    if (e != cudaSuccess) return e;
    p.per0 = tiles0(kq);
    if ((e = run_gemm<1, false, true, EpiPair<EpiDkq<true>, EpiDkq<false>>>(kq, p, st)) != cudaSuccess) return e;
    {
      E2TTT_TRACE("tcb_sums", st);
      const long long warps = (long long)BH * C + 3 * BH;
      bwd_sums_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(
          B.part, B.abar, B.bbar, B.spart, B.sbar, dd, ci, t0, cl, p.NG, shadow_nb);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    e = dwn == 256 ? run_gemm<1, true, true, EpiDW, 256>(dw, p, st) : run_gemm<1, true, true, EpiDW>(dw, p, st);
    if (e != cudaSuccess) return e;
  }
  return launch_chunk_coeffs_bwd(A.lr, A.mom, A.decay, B.abar, B.bbar, B.sbar, A.dlr, A.dmom,
                                 A.ddecay, BH, T, C, NC, d.coef, st);
}

}  // namespace e2ttt
