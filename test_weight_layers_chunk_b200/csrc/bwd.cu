// Backward of the chunk scan on fp32 CUDA cores (any shape; fp32 or bf16 activations).
//
// Adjoint of the closed-form chunk transition ("Rethinking Expressivity and
// Efficiency in Test-Time Training": abstract, training through the closed form
// with all tokens of a chunk in parallel), chunks in reverse. For the scalar
//   L = sum_t <dout_t, out_t> + <dW_end, W_end> + <dM_end, M_end>,
// with D_W, D_M the adjoints of a chunk's end states and G_t = a_t D_M + b_t D_W:
//   dM0   = U(1,n) D_M + c D_W
//   dW0   = L(1,n) D_W + grad_W0 sum_t <dout_t, f_W0(q_t)> - sum_t VJP_W0[g_t](G_t)
//   abar_t = -<D_M, g_t>,  bbar_t = -<D_W, g_t>
//   (U(1,n), L(1,n), c)bar = (<D_M, M0>, <D_W, W0>, <D_W, M0>)
// and dk, dv from -sum_t <G_t, g_t(W0; k_t, v_t)> (second-order terms through the
// loss gradient), dq from the output path. The gate gradients follow from the
// adjoint of the scalar kernels (scan.cu) once every chunk is done.
// SwiGLU per key row (h1 = W1 k, h3 = W3 k, s = silu(h1), u = s h3, e = W2 u - v,
// du = W2^T e, dh1 = du h3 s', dh3 = du s) the VJP of g = (dh1 k^T, dh3 k^T, e u^T)
// along -G gives, with P1 = G1 k, P3 = G3 k, P2 = G2 u (G split like W):
//   dh1b = -P1, dh3b = -P3, dub = dh1b h3 s' + dh3b s,  eb = W2 dub - P2,
//   ub = -G2^T e + W2^T eb (MSE),  sb = dh3b du + ub h3,  h3b = dh1b du s' + ub s,
//   h1b = dh1b du h3 s'' + sb s',  dv = -eb,
//   dk = -(G1^T dh1 + G3^T dh3) + W1^T h1b + W3^T h3b,
//   dW2 += e dub^T + eb u^T (MSE),  dW1 += h1b k^T,  dW3 += h3b k^T.
// GELU MLP (h = W1 k, u = gelu(h), dh = du gelu'(h)), with P1 = G1 k, P2 = G2 u:
//   dhb = -P1, dub = dhb gelu'(h), eb = W2 dub - P2, ub = -G2^T e + W2^T eb (MSE),
//   hb = dhb du gelu''(h) + ub gelu'(h), dv = -eb, dk = -G1^T dh + W1^T hb,
//   dW2 += e dub^T + eb u^T (MSE), dW1 += hb k^T.
// Both MLPs share the code below with nf = 2 (SwiGLU: h1 | h3) or 1 (GELU: h)
// activation factors per hidden unit.
#include <stdint.h>

#include <initializer_list>

#include "paths.h"
#include "simt.cuh"
#include "state.cuh"

namespace e2ttt {
namespace {

// Scratch of the backward (fp32), per head, C rows per chunk.
struct BwdWs {
  size_t status, a, b, scal, abar, bbar, sbar, part;
  size_t H, E, dA, P, P2, UB, DUB, EB, UB5, HB, GK;
  size_t total;
};

BwdWs bwd_layout(const Dims& d) {
  size_t off = 0;
  auto take = [&](size_t floats) {
    size_t o = off;
    off = (off + floats * sizeof(float) + 255) & ~size_t(255);
    return o;
  };
  const size_t BH = d.BH, C = d.C, dh = d.d_h, dv = d.d_v;
  BwdWs L{};
  L.status = take(64);  // status word (read by e2ttt_workspace_status; always 0 here)
  L.a = take(BH * d.T);
  L.b = take(BH * d.T);
  L.scal = take(3 * BH * d.NC);
  L.abar = take(BH * d.T);
  L.bbar = take(BH * d.T);
  L.sbar = take(3 * BH * d.NC);
  L.part = take(3 * BH * 64);
  if (d.kind != 0) {
    const size_t nf = d.kind == 1 ? 2 : 1;
    L.H = take(BH * 2 * C * nf * dh);
    L.E = take(BH * C * dv);
    L.dA = take(BH * C * dh);
    L.P = take(BH * C * 2 * nf * dh);
    L.P2 = take(BH * C * 2 * dv);
    L.UB = take(BH * C * 2 * dh);
    L.DUB = take(BH * C * dh);
    L.EB = take(BH * C * dv);
    L.UB5 = take(BH * C * dh);
    L.HB = take(BH * 2 * C * nf * dh);
  } else {
    L.E = take(BH * C * dv);
    L.P = take(BH * C * 2 * dv);
    L.GK = take(BH * C * dv);
  }
  L.total = off;
  return L;
}

template <typename TA>
struct Bwd {
  Dims d;
  const TA *q, *k, *v, *dout;
  TA *dq, *dk, *dv;
  const float *ca, *cb;
  float *abar, *bbar, *sbar, *part;
  const float *scal;
  const float *W0, *M0;  // chunk-start states
  long long sst;         // their head stride
  float *DW, *DM;        // state adjoints (head stride S), updated in place
  float *H, *E, *dA, *P, *P2, *UB, *DUB, *EB, *UB5, *HB, *GK;
  int ci, t0, n;
  __device__ __forceinline__ size_t tok(int z, int t) const { return (size_t)z * d.T + t0 + t; }
  __device__ __forceinline__ float coef_a(int z, int t) const { return ca[tok(z, t)]; }
  __device__ __forceinline__ float coef_b(int z, int t) const { return cb[tok(z, t)]; }
  __device__ __forceinline__ const float* w0(int z) const { return W0 + z * sst; }
  __device__ __forceinline__ const float* dWp(int z) const { return DW + z * d.S; }
  __device__ __forceinline__ const float* dMp(int z) const { return DM + z * d.S; }
  // activation factors per hidden unit (SwiGLU h1 | h3: 2, GELU h: 1) and the
  // row width nf d_h of H and HB
  __device__ __forceinline__ int nf() const { return d.kind == 2 ? 1 : 2; }
  __device__ __forceinline__ int hw() const { return nf() * d.d_h; }
  // key-row quantities at (t, j): h1 (GELU: h), h3 (SwiGLU only), the activation u
  __device__ __forceinline__ float h1k(int z, int t, int j) const {
    return H[((size_t)z * 2 * d.C + n + t) * hw() + j];
  }
  __device__ __forceinline__ float h3k(int z, int t, int j) const {
    return H[((size_t)z * 2 * d.C + n + t) * hw() + d.d_h + j];
  }
  __device__ __forceinline__ float act_row(const float* h, int j) const {
    return d.kind == 2 ? gelu_f(h[j]) : silu_f(h[j]) * h[d.d_h + j];
  }
  __device__ __forceinline__ float uk(int z, int t, int j) const {
    return act_row(H + ((size_t)z * 2 * d.C + n + t) * hw(), j);
  }
};

// ------------------------------------------------------------------ loaders
template <typename TA> struct LX {  // rows of [q; k] of the chunk
  Bwd<TA> c;
  __device__ float operator()(int z, int r, int kk) const {
    const TA* p = r < c.n ? c.q + c.tok(z, r) * c.d.d_k : c.k + c.tok(z, r - c.n) * c.d.d_k;
    return to_f(p[kk]);
  }
};
template <typename TA> struct LRowAct {  // token rows of an activation tensor (q, k or dout)
  Bwd<TA> c;
  const TA* base;
  int ld;
  __device__ float operator()(int z, int t, int kk) const { return to_f(base[c.tok(z, t) * ld + kk]); }
};
template <typename TA> struct LBufRow {  // A(t, kk) = buf[z][t][kk]
  const float* base;
  int C, ld;
  __device__ float operator()(int z, int t, int kk) const { return base[((size_t)z * C + t) * ld + kk]; }
};
template <typename TA> struct LStateT {  // B(kk, col) = state matrix [col][kk] of W0
  Bwd<TA> c;
  long long off;
  int ld;
  __device__ float operator()(int z, int kk, int col) const { return c.w0(z)[off + (long long)col * ld + kk]; }
};
template <typename TA> struct LState {  // B(kk, col) = state matrix [kk][col] of W0
  Bwd<TA> c;
  long long off;
  int ld;
  __device__ float operator()(int z, int kk, int col) const { return c.w0(z)[off + (long long)kk * ld + col]; }
};
template <typename TA> struct LActK {  // u of key rows (t, j) from H
  Bwd<TA> c;
  __device__ float operator()(int z, int t, int j) const { return c.uk(z, t, j); }
};
// B(kk, col) over [DM rows | DW rows] of a block with row length ld: col < half -> DM
template <typename TA> struct LDirT {
  Bwd<TA> c;
  long long off;
  int ld, half;
  __device__ float operator()(int z, int kk, int col) const {
    return col < half ? c.dMp(z)[off + (long long)col * ld + kk]
                      : c.dWp(z)[off + (long long)(col - half) * ld + kk];
  }
};
// B(kk, col) = [DM2 | DW2][kk][col]: col < half -> DM2[kk][col]
template <typename TA> struct LDir {
  Bwd<TA> c;
  long long off;
  int ld, half;
  __device__ float operator()(int z, int kk, int col) const {
    return col < half ? c.dMp(z)[off + (long long)kk * ld + col]
                      : c.dWp(z)[off + (long long)kk * ld + col - half];
  }
};

// ------------------------------------------------------------------ epilogues
template <typename TA> struct EStore {  // buf[z][r][col] = acc
  float* base;
  int C2, ld;
  __device__ void operator()(int z, int r, int col, const float* acc) const {
    base[((size_t)z * C2 + r) * ld + col] = acc[0];
  }
};
template <typename TA> struct EResid {  // E = y - v (or -v)
  Bwd<TA> c;
  __device__ void operator()(int z, int t, int col, const float* acc) const {
    const float vv = to_f(c.v[c.tok(z, t) * c.d.d_v + col]);
    c.E[((size_t)z * c.d.C + t) * c.d.d_v + col] = c.d.loss == 0 ? acc[0] - vv : -vv;
  }
};
template <typename TA> struct EActOut {  // act tensor [token][col] = acc
  Bwd<TA> c;
  TA* base;
  int ld;
  __device__ void operator()(int z, int t, int col, const float* acc) const {
    base[c.tok(z, t) * ld + col] = from_f<TA>(acc[0]);
  }
};
// eb = W2 dub - (a P2M + b P2W); EB stored, dv = -eb.
template <typename TA> struct EEb {
  Bwd<TA> c;
  __device__ void operator()(int z, int t, int col, const float* acc) const {
    const int dv = c.d.d_v;
    const float* p2 = c.P2 + ((size_t)z * c.d.C + t) * 2 * dv;
    const float eb = acc[0] - (c.coef_a(z, t) * p2[col] + c.coef_b(z, t) * p2[dv + col]);
    c.EB[((size_t)z * c.d.C + t) * dv + col] = eb;
    c.dv[c.tok(z, t) * dv + col] = from_f<TA>(-eb);
  }
};
// query rows: ub_q = dout W2 -> h1b_q = ub h3 s', h3b_q = ub s (GELU: hb_q = ub
// gelu'(h)) (rows [0, C) of HB)
template <typename TA> struct EQrows {
  Bwd<TA> c;
  __device__ void operator()(int z, int t, int j, const float* acc) const {
    const int dh = c.d.d_h;
    const float* h = c.H + ((size_t)z * 2 * c.d.C + t) * c.hw();
    float* o = c.HB + ((size_t)z * 2 * c.d.C + t) * c.hw();
    if (c.d.kind == 2) {
      o[j] = acc[0] * dgelu_f(h[j]);
      return;
    }
    o[j] = acc[0] * h[dh + j] * dsilu_f(h[j]);
    o[dh + j] = acc[0] * silu_f(h[j]);
  }
};
// D_W <- L(1,n) D_W + acc  (in place; the state-gradient aggregation of a block)
template <typename TA> struct EdW {
  Bwd<TA> c;
  long long off;
  int ld;
  __device__ void operator()(int z, int i, int j, const float* acc) const {
    const size_t plane = (size_t)c.d.BH * c.d.NC;
    const float PL = c.scal[plane + (size_t)z * c.d.NC + c.ci];
    float* p = c.DW + (size_t)z * c.d.S + off + (long long)i * ld + j;
    *p = PL * *p + acc[0];
  }
};

// ------------------------------------------------------------------ SwiGLU stacked loaders
// dk: A(t, kk') over [-a dh1 | -a dh3 | -b dh1 | -b dh3 | h1b | h3b] (6 d_h;
// GELU: [-a dh | -b dh | hb], 3 d_h)
template <typename TA> struct LdkA {
  Bwd<TA> c;
  __device__ float operator()(int z, int t, int kk) const {
    const int dh = c.d.d_h, nf = c.nf();
    const int seg = kk / dh, j = kk - seg * dh;
    if (seg >= 2 * nf)
      return c.HB[((size_t)z * 2 * c.d.C + c.d.C + t) * c.hw() + (seg - 2 * nf) * dh + j];
    const float h1 = c.h1k(z, t, j);
    const float du = c.dA[((size_t)z * c.d.C + t) * dh + j];
    float dh_;
    if (nf == 1) dh_ = du * dgelu_f(h1);
    else dh_ = (seg & 1) ? du * silu_f(h1) : du * c.h3k(z, t, j) * dsilu_f(h1);
    const float sc = seg < nf ? c.coef_a(z, t) : c.coef_b(z, t);
    return -sc * dh_;
  }
};
// dk: B(kk', col) over [DM1; DM3; DW1; DW3; W1; W3] rows (each d_h x d_k; GELU:
// [DM1; DW1; W1])
template <typename TA> struct LdkB {
  Bwd<TA> c;
  __device__ float operator()(int z, int kk, int col) const {
    const int dh = c.d.d_h, dk = c.d.d_k, nf = c.nf();
    const int seg = kk / dh, j = kk - seg * dh;
    const long long o = (long long)((seg % nf) * dh + j) * dk + col;  // W1 (or W3) block row j
    if (seg < nf) return c.dMp(z)[o];
    if (seg < 2 * nf) return c.dWp(z)[o];
    return c.w0(z)[o];
  }
};
// dW1/dW3: A(i, t') = HB (t' < n: key rows, else query rows), column i of [h1b | h3b]
template <typename TA> struct LdW13A {
  Bwd<TA> c;
  __device__ float operator()(int z, int i, int tt) const {
    const int row = tt < c.n ? c.d.C + tt : tt - c.n;
    return c.HB[((size_t)z * 2 * c.d.C + row) * c.hw() + i];
  }
};
template <typename TA> struct LdW13B {  // B(t', col) = k (t' < n) or q
  Bwd<TA> c;
  __device__ float operator()(int z, int tt, int col) const {
    const TA* p = tt < c.n ? c.k + c.tok(z, tt) * c.d.d_k : c.q + c.tok(z, tt - c.n) * c.d.d_k;
    return to_f(p[col]);
  }
};
// dW2: A(v, t') over [E | EB (MSE) | dout], B(t', j) over [dub | u_k | u_q]
template <typename TA> struct LdW2A {
  Bwd<TA> c;
  __device__ float operator()(int z, int vv, int tt) const {
    const int n = c.n, dv = c.d.d_v;
    if (tt < n) return c.E[((size_t)z * c.d.C + tt) * dv + vv];
    if (tt < 2 * n) return c.d.loss == 0 ? c.EB[((size_t)z * c.d.C + tt - n) * dv + vv] : 0.f;
    return to_f(c.dout[c.tok(z, tt - 2 * n) * dv + vv]);
  }
};
template <typename TA> struct LdW2B {
  Bwd<TA> c;
  __device__ float operator()(int z, int tt, int j) const {
    const int n = c.n, dh = c.d.d_h;
    if (tt < n) return c.DUB[((size_t)z * c.d.C + tt) * dh + j];
    if (tt < 2 * n) return c.uk(z, tt - n, j);
    return c.act_row(c.H + ((size_t)z * 2 * c.d.C + tt - 2 * n) * c.hw(), j);
  }
};

// ------------------------------------------------------------------ linear stacked loaders
// dk: A(t, kk') over [-a e | -b e | -gk (MSE)] (3 d_v), B over [DM; DW; W0] rows
template <typename TA> struct LLinDkA {
  Bwd<TA> c;
  __device__ float operator()(int z, int t, int kk) const {
    const int dv = c.d.d_v;
    const int seg = kk / dv, j = kk - seg * dv;
    const size_t r = ((size_t)z * c.d.C + t) * dv + j;
    if (seg == 0) return -c.coef_a(z, t) * c.E[r];
    if (seg == 1) return -c.coef_b(z, t) * c.E[r];
    return c.d.loss == 0 ? -c.GK[r] : 0.f;
  }
};
template <typename TA> struct LLinDkB {
  Bwd<TA> c;
  __device__ float operator()(int z, int kk, int col) const {
    const int dv = c.d.d_v, dk = c.d.d_k;
    const int seg = kk / dv, j = kk - seg * dv;
    const long long o = (long long)j * dk + col;
    if (seg == 0) return c.dMp(z)[o];
    if (seg == 1) return c.dWp(z)[o];
    return c.w0(z)[o];
  }
};
// dW: A(v, t') over [dout | -gk (MSE)], B(t', col) over [q | k]
template <typename TA> struct LLinDwA {
  Bwd<TA> c;
  __device__ float operator()(int z, int vv, int tt) const {
    const int n = c.n, dv = c.d.d_v;
    if (tt < n) return to_f(c.dout[c.tok(z, tt) * dv + vv]);
    return c.d.loss == 0 ? -c.GK[((size_t)z * c.d.C + tt - n) * dv + vv] : 0.f;
  }
};
template <typename TA> struct LLinDwB {
  Bwd<TA> c;
  __device__ float operator()(int z, int tt, int col) const {
    const TA* p = tt < c.n ? c.q + c.tok(z, tt) * c.d.d_k : c.k + c.tok(z, tt - c.n) * c.d.d_k;
    return to_f(p[col]);
  }
};

// ------------------------------------------------------------------ row / element kernels
// SwiGLU: abar_t, bbar_t (one warp per key row)
template <typename TA>
__global__ void swiglu_rows_kernel(Bwd<TA> c) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= c.d.BH * c.n) return;
  const int z = w / c.n, t = w - z * c.n;
  const int dh = c.d.d_h, dv = c.d.d_v, hw = c.hw();
  const float* P = c.P + ((size_t)z * c.d.C + t) * 2 * hw;
  const float* P2 = c.P2 + ((size_t)z * c.d.C + t) * 2 * dv;
  const float* du = c.dA + ((size_t)z * c.d.C + t) * dh;
  const float* e = c.E + ((size_t)z * c.d.C + t) * dv;
  float am = 0.f, bw = 0.f;
  for (int j = lane; j < dh; j += 32) {
    const float h1 = c.h1k(z, t, j);
    if (c.d.kind == 2) {
      const float dhj = du[j] * dgelu_f(h1);
      am += dhj * P[j];
      bw += dhj * P[hw + j];
      continue;
    }
    const float h3 = c.h3k(z, t, j);
    const float dh1 = du[j] * h3 * dsilu_f(h1), dh3 = du[j] * silu_f(h1);
    am += dh1 * P[j] + dh3 * P[dh + j];
    bw += dh1 * P[2 * dh + j] + dh3 * P[3 * dh + j];
  }
  for (int j = lane; j < dv; j += 32) {
    am += e[j] * P2[j];
    bw += e[j] * P2[dv + j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    am += __shfl_xor_sync(0xffffffffu, am, o);
    bw += __shfl_xor_sync(0xffffffffu, bw, o);
  }
  if (lane == 0) {
    c.abar[c.tok(z, t)] = -am;
    c.bbar[c.tok(z, t)] = -bw;
  }
}

// SwiGLU: dub (stage 1) or the final h1b, h3b of the key rows (stage 2)
template <typename TA>
__global__ void swiglu_elem_kernel(Bwd<TA> c, int stage) {
  const int dh = c.d.d_h;
  const long long total = (long long)c.d.BH * c.n * dh;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(e % dh);
    const long long r = e / dh;
    const int t = (int)(r % c.n), z = (int)(r / c.n);
    const float a = c.coef_a(z, t), b = c.coef_b(z, t);
    const size_t row = (size_t)z * c.d.C + t;
    if (c.d.kind == 2) {  // GELU MLP
      const float* P = c.P + row * 2 * dh;
      const float dhb = -(a * P[j] + b * P[dh + j]);
      const float h = c.h1k(z, t, j), gp = dgelu_f(h);
      if (stage == 1) {
        c.DUB[row * dh + j] = dhb * gp;
        continue;
      }
      const float du = c.dA[row * dh + j];
      float ub = -(a * c.UB[row * 2 * dh + j] + b * c.UB[row * 2 * dh + dh + j]);
      if (c.d.loss == 0) ub += c.UB5[row * dh + j];
      c.HB[((size_t)z * 2 * c.d.C + c.d.C + t) * dh + j] = dhb * du * d2gelu_f(h) + ub * gp;
      continue;
    }
    const float* P = c.P + row * 4 * dh;
    const float dh1b = -(a * P[j] + b * P[2 * dh + j]);
    const float dh3b = -(a * P[dh + j] + b * P[3 * dh + j]);
    const float h1 = c.h1k(z, t, j), h3 = c.h3k(z, t, j);
    const float s = silu_f(h1), s1 = dsilu_f(h1);
    if (stage == 1) {
      c.DUB[row * dh + j] = dh1b * h3 * s1 + dh3b * s;
      continue;
    }
    const float du = c.dA[row * dh + j];
    float ub = -(a * c.UB[row * 2 * dh + j] + b * c.UB[row * 2 * dh + dh + j]);
    if (c.d.loss == 0) ub += c.UB5[row * dh + j];
    const float sb = dh3b * du + ub * h3;
    const float h3b = dh1b * du * s1 + ub * s;
    const float h1b = dh1b * du * h3 * d2silu_f(h1) + sb * s1;
    float* o = c.HB + ((size_t)z * 2 * c.d.C + c.d.C + t) * 2 * dh;
    o[j] = h1b;
    o[dh + j] = h3b;
  }
}

// Linear: abar, bbar, gk = a P_M + b P_W, dv = gk (one warp per key row)
template <typename TA>
__global__ void linear_rows_kernel(Bwd<TA> c) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= c.d.BH * c.n) return;
  const int z = w / c.n, t = w - z * c.n;
  const int dv = c.d.d_v;
  const size_t row = (size_t)z * c.d.C + t;
  const float* P = c.P + row * 2 * dv;
  const float* e = c.E + row * dv;
  const float a = c.coef_a(z, t), b = c.coef_b(z, t);
  float am = 0.f, bw = 0.f;
  for (int j = lane; j < dv; j += 32) {
    am += e[j] * P[j];
    bw += e[j] * P[dv + j];
    const float gk = a * P[j] + b * P[dv + j];
    c.GK[row * dv + j] = gk;
    c.dv[c.tok(z, t) * dv + j] = from_f<TA>(gk);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    am += __shfl_xor_sync(0xffffffffu, am, o);
    bw += __shfl_xor_sync(0xffffffffu, bw, o);
  }
  if (lane == 0) {
    c.abar[c.tok(z, t)] = -am;
    c.bbar[c.tok(z, t)] = -bw;
  }
}

// Chunk-scalar adjoints <D_M, M0>, <D_W, W0>, <D_W, M0>: 64 blocks per head
// write partial sums, then one thread per head adds them in a fixed order.
template <typename TA>
__global__ void scalar_adjoint_partials(Bwd<TA> c) {
  const int z = blockIdx.y, blk = blockIdx.x;
  const long long S = c.d.S;
  const float* dm = c.dMp(z);
  const float* dw = c.dWp(z);
  const float* w0 = c.w0(z);
  const float* m0 = c.M0 ? c.M0 + z * c.sst : nullptr;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f;
  for (long long i = (long long)blk * blockDim.x + threadIdx.x; i < S; i += (long long)gridDim.x * blockDim.x) {
    const float m = m0 ? m0[i] : 0.f;
    s0 += dm[i] * m;
    s1 += dw[i] * w0[i];
    s2 += dw[i] * m;
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
    for (int q = 0; q < 3; ++q) c.part[((size_t)q * c.d.BH + z) * 64 + blk] = red[q][0];
}
template <typename TA>
__global__ void scalar_adjoint_final(Bwd<TA> c) {
  const int z = blockIdx.x * blockDim.x + threadIdx.x;
  if (z >= c.d.BH) return;
  const size_t plane = (size_t)c.d.BH * c.d.NC, o = (size_t)z * c.d.NC + c.ci;
  for (int q = 0; q < 3; ++q) {
    float s = 0.f;
    for (int b = 0; b < 64; ++b) s += c.part[((size_t)q * c.d.BH + z) * 64 + b];
    // order of chunk_scalars: U(1,n), L(1,n), c  <->  <D_M,M0>, <D_W,W0>, <D_W,M0>
    c.sbar[q * plane + o] = s;
  }
}
// dM0 = U(1,n) D_M + c D_W  (in place into D_M)
template <typename TA>
__global__ void dm_update_kernel(Bwd<TA> c) {
  const long long total = (long long)c.d.BH * c.d.S;
  const size_t plane = (size_t)c.d.BH * c.d.NC;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int z = (int)(e / c.d.S);
    const size_t o = (size_t)z * c.d.NC + c.ci;
    c.DM[e] = c.scal[o] * c.DM[e] + c.scal[2 * plane + o] * c.DW[e];
  }
}

template <typename TA>
cudaError_t chunk_bwd(const Bwd<TA>& c, cudaStream_t st) {
  const Dims& d = c.d;
  const int n = c.n, BH = d.BH, dk = d.d_k, dv = d.d_v, dh = d.d_h;
  cudaError_t e;
#define E2_CHECK(x) do { e = (x); if (e != cudaSuccess) return e; } while (0)
  {
    E2TTT_TRACE("bwd_scalar_adjoints", st);
    scalar_adjoint_partials<TA><<<dim3(64, BH), 256, 0, st>>>(c);
    scalar_adjoint_final<TA><<<(BH + 127) / 128, 128, 0, st>>>(c);
    E2_CHECK(cudaGetLastError());
  }
  const int row_blocks = (BH * n + 7) / 8;
  if (d.kind == 0) {
    // e = K W0^T - v ; P = K [D_M; D_W]^T
    E2_CHECK(simt_gemm<1>(BH, n, dv, dk, LRowAct<TA>{c, c.k, dk}, LStateT<TA>{c, 0, dk}, UnitScale{},
                          EResid<TA>{c}, st, "bwd_linear_residual"));
    E2_CHECK(simt_gemm<1>(BH, n, 2 * dv, dk, LRowAct<TA>{c, c.k, dk}, LDirT<TA>{c, 0, dk, dv},
                          UnitScale{}, EStore<TA>{c.P, d.C, 2 * dv}, st, "bwd_linear_directions"));
    {
      E2TTT_TRACE("bwd_linear_rows", st);
      linear_rows_kernel<TA><<<row_blocks, 256, 0, st>>>(c);
      E2_CHECK(cudaGetLastError());
    }
    E2_CHECK(simt_gemm<1>(BH, n, dk, 3 * dv, LLinDkA<TA>{c}, LLinDkB<TA>{c}, UnitScale{},
                          EActOut<TA>{c, c.dk, dk}, st, "bwd_linear_dk"));
    E2_CHECK(simt_gemm<1>(BH, n, dk, dv, LRowAct<TA>{c, c.dout, dv}, LState<TA>{c, 0, dk}, UnitScale{},
                          EActOut<TA>{c, c.dq, dk}, st, "bwd_linear_dq"));
    {
      E2TTT_TRACE("bwd_dm_update", st);
      dm_update_kernel<TA><<<1184, 256, 0, st>>>(c);
      E2_CHECK(cudaGetLastError());
    }
    return simt_gemm<1>(BH, dv, dk, 2 * n, LLinDwA<TA>{c}, LLinDwB<TA>{c}, UnitScale{},
                        EdW<TA>{c, 0, dk}, st, "bwd_linear_dw");
  }
  const int nf = d.kind == 2 ? 1 : 2;   // activation factors per hidden unit
  const int hw = nf * dh;                // rows of W1 (GELU) or [W1; W3]
  const long long o2 = (long long)hw * dk;
  // recompute the forward internals at W0
  E2_CHECK(simt_gemm<1>(BH, 2 * n, hw, dk, LX<TA>{c}, LStateT<TA>{c, 0, dk}, UnitScale{},
                        EStore<TA>{c.H, 2 * d.C, hw}, st, "bwd_h"));
  E2_CHECK(simt_gemm<1>(BH, n, dv, dh, LActK<TA>{c}, LStateT<TA>{c, o2, dh}, UnitScale{}, EResid<TA>{c},
                        st, "bwd_residual"));
  E2_CHECK(simt_gemm<1>(BH, n, dh, dv, LBufRow<TA>{c.E, d.C, dv}, LState<TA>{c, o2, dh}, UnitScale{},
                        EStore<TA>{c.dA, d.C, dh}, st, "bwd_da"));
  // directional products with the state adjoints
  E2_CHECK(simt_gemm<1>(BH, n, 2 * hw, dk, LRowAct<TA>{c, c.k, dk}, LDirT<TA>{c, 0, dk, hw},
                        UnitScale{}, EStore<TA>{c.P, d.C, 2 * hw}, st, "bwd_dir_w13"));
  E2_CHECK(simt_gemm<1>(BH, n, 2 * dv, dh, LActK<TA>{c}, LDirT<TA>{c, o2, dh, dv}, UnitScale{},
                        EStore<TA>{c.P2, d.C, 2 * dv}, st, "bwd_dir_w2"));
  E2_CHECK(simt_gemm<1>(BH, n, 2 * dh, dv, LBufRow<TA>{c.E, d.C, dv}, LDir<TA>{c, o2, dh, dh},
                        UnitScale{}, EStore<TA>{c.UB, d.C, 2 * dh}, st, "bwd_ub_dir"));
  {
    E2TTT_TRACE("bwd_rows", st);
    swiglu_rows_kernel<TA><<<row_blocks, 256, 0, st>>>(c);
    swiglu_elem_kernel<TA><<<1184, 256, 0, st>>>(c, 1);
    E2_CHECK(cudaGetLastError());
  }
  // eb = W2 dub - P2 (dv = -eb);  ub += W2^T eb (MSE)
  E2_CHECK(simt_gemm<1>(BH, n, dv, dh, LBufRow<TA>{c.DUB, d.C, dh}, LStateT<TA>{c, o2, dh}, UnitScale{},
                        EEb<TA>{c}, st, "bwd_eb"));
  if (d.loss == 0)
    E2_CHECK(simt_gemm<1>(BH, n, dh, dv, LBufRow<TA>{c.EB, d.C, dv}, LState<TA>{c, o2, dh}, UnitScale{},
                          EStore<TA>{c.UB5, d.C, dh}, st, "bwd_ub_eb"));
  // query rows: ub_q = dout W2 -> h1b_q, h3b_q
  E2_CHECK(simt_gemm<1>(BH, n, dh, dv, LRowAct<TA>{c, c.dout, dv}, LState<TA>{c, o2, dh}, UnitScale{},
                        EQrows<TA>{c}, st, "bwd_q_rows"));
  {
    E2TTT_TRACE("bwd_elem", st);
    swiglu_elem_kernel<TA><<<1184, 256, 0, st>>>(c, 2);
    E2_CHECK(cudaGetLastError());
  }
  // input gradients
  E2_CHECK(simt_gemm<1>(BH, n, dk, 3 * hw, LdkA<TA>{c}, LdkB<TA>{c}, UnitScale{},
                        EActOut<TA>{c, c.dk, dk}, st, "bwd_dk"));
  E2_CHECK(simt_gemm<1>(BH, n, dk, hw, LBufRow<TA>{c.HB, 2 * d.C, hw}, LState<TA>{c, 0, dk},
                        UnitScale{}, EActOut<TA>{c, c.dq, dk}, st, "bwd_dq"));
  {
    E2TTT_TRACE("bwd_dm_update", st);
    dm_update_kernel<TA><<<1184, 256, 0, st>>>(c);
    E2_CHECK(cudaGetLastError());
  }
  // state-gradient aggregations (in place into D_W)
  E2_CHECK(simt_gemm<1>(BH, hw, dk, 2 * n, LdW13A<TA>{c}, LdW13B<TA>{c}, UnitScale{},
                        EdW<TA>{c, 0, dk}, st, "bwd_dw13"));
  return simt_gemm<1>(BH, dv, dh, 3 * n, LdW2A<TA>{c}, LdW2B<TA>{c}, UnitScale{}, EdW<TA>{c, o2, dh},
                      st, "bwd_dw2");
#undef E2_CHECK
}

}  // namespace

size_t bwd_workspace_bytes(const Dims& d, bool bf16_act) {
  size_t n = bwd_layout(d).total;
  if (tc_bwd_supported(d, bf16_act)) {
    const size_t t = tc_bwd_workspace_bytes(d);
    if (t > n) n = t;
  }
  return n;
}

static bool aligned16(std::initializer_list<const void*> ps) {
  for (const void* q : ps)
    if (((uintptr_t)q) & 15) return false;
  return true;
}

template <typename TA>
cudaError_t bwd_run(const BwdArgs& A) {
  const Dims& d = A.d;
  if (sizeof(TA) == 2 && tc_bwd_supported(d, true) &&
      aligned16({A.q, A.k, A.v, A.dout, A.dq, A.dk, A.dv, A.saved, A.dW0, A.dM0}))
    return tc_bwd(A);
  BwdWs L = bwd_layout(d);
  char* w = (char*)A.ws;
  Bwd<TA> c;
  c.d = d;
  c.q = (const TA*)A.q; c.k = (const TA*)A.k; c.v = (const TA*)A.v; c.dout = (const TA*)A.dout;
  c.dq = (TA*)A.dq; c.dk = (TA*)A.dk; c.dv = (TA*)A.dv;
  float* ca = (float*)(w + L.a);
  float* cb = (float*)(w + L.b);
  float* scal = (float*)(w + L.scal);
  c.ca = ca; c.cb = cb; c.scal = scal;
  c.abar = (float*)(w + L.abar); c.bbar = (float*)(w + L.bbar);
  c.sbar = (float*)(w + L.sbar); c.part = (float*)(w + L.part);
  auto F = [&](size_t off) { return off ? (float*)(w + off) : nullptr; };
  c.H = F(L.H); c.E = F(L.E); c.dA = F(L.dA); c.P = F(L.P); c.P2 = F(L.P2); c.UB = F(L.UB);
  c.DUB = F(L.DUB); c.EB = F(L.EB); c.UB5 = F(L.UB5); c.HB = F(L.HB); c.GK = F(L.GK);
  c.DW = A.dW0;
  c.DM = A.dM0;
  cudaStream_t st = A.st;
  const size_t sbytes = (size_t)d.BH * d.S * sizeof(float);
  cudaError_t e = cudaMemsetAsync(w + L.status, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  e = launch_chunk_coeffs(A.lr, A.mom, A.decay, ca, cb, scal, d.BH, d.T, d.C, d.NC, d.coef, st);
  if (e != cudaSuccess) return e;
  e = A.dW_end ? cudaMemcpyAsync(A.dW0, A.dW_end, sbytes, cudaMemcpyDeviceToDevice, st)
               : cudaMemsetAsync(A.dW0, 0, sbytes, st);
  if (e != cudaSuccess) return e;
  e = A.dM_end ? cudaMemcpyAsync(A.dM0, A.dM_end, sbytes, cudaMemcpyDeviceToDevice, st)
               : cudaMemsetAsync(A.dM0, 0, sbytes, st);
  if (e != cudaSuccess) return e;
  const size_t per_chunk = (size_t)d.BH * 2 * d.S;
  for (int ci = d.NC - 1; ci >= 0; --ci) {
    c.ci = ci;
    c.t0 = ci * d.C;
    c.n = d.T - c.t0 < d.C ? d.T - c.t0 : d.C;
    c.W0 = A.saved + ci * per_chunk;
    c.M0 = A.saved + ci * per_chunk + d.S;
    c.sst = 2 * d.S;
    e = chunk_bwd(c, st);
    if (e != cudaSuccess) return e;
  }
  return launch_chunk_coeffs_bwd(A.lr, A.mom, A.decay, c.abar, c.bbar, c.sbar, A.dlr, A.dmom,
                                 A.ddecay, d.BH, d.T, d.C, d.NC, d.coef, st);
}

template cudaError_t bwd_run<float>(const BwdArgs&);
template cudaError_t bwd_run<bf16>(const BwdArgs&);

}  // namespace e2ttt
