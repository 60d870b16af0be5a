// Forward chunk scan on fp32 CUDA cores (any shape; fp32 or bf16 activations).
//
// Per chunk of n tokens and per head z, with W0/M0 the chunk-start states
// ("Rethinking Expressivity and Efficiency in Test-Time Training": abstract,
// closed-form chunk transition; atlas "Approach", two weighted gradient
// aggregations; "Limitations", output at the chunk-start weights):
//   linear:  [out; Y_k] = [Q; K] W0^T,  E = Y_k - V
//            dM = E^T diag(a) K,  dW = E^T diag(b) K
//   SwiGLU:  H = [Q; K] [W1; W3]^T,  A = silu(H1) * H3,  [out; Y_k] = A W2^T,
//            E = Y_k - V,  dA = E W2,  dH1 = dA * H3_k * silu'(H1_k),
//            dH3 = dA * silu(H1_k)
//            d[W1; W3] = [dH1 | dH3]^T diag(.) K,   dW2 = E^T diag(.) A_k
//   GELU MLP: H = [Q; K] W1^T,  A = gelu(H),  [out; Y_k] = A W2^T,  E = Y_k - V,
//            dH = (E W2) * gelu'(H_k),  dW1 = dH^T diag(.) K,  dW2 = E^T diag(.) A_k
//   epilogue (fp32): M_end = U(1,n) M0 - dM,  W_end = L(1,n) W0 + c M0 - dW
// (E = -V for the dot-product loss.)
#include "simt.cuh"
#include "state.cuh"

namespace e2ttt {
namespace {

template <typename TA>
struct Fwd {
  Dims d;
  const TA *q, *k, *v;
  TA* out;
  const float *ca, *cb, *scal;
  StateIn src;
  StateOut dst;
  float *H, *E, *dH;
  int ci, t0, n;
  __device__ __forceinline__ size_t tok(int z, int t) const { return (size_t)z * d.T + t0 + t; }
  // row length of H and dH: [h1 | h3] (SwiGLU) or h (GELU MLP)
  __device__ __forceinline__ int hld() const { return d.kind == 2 ? d.d_h : 2 * d.d_h; }
};
// the activation of hidden unit j of one row of H
__device__ __forceinline__ float act_of(const Dims& d, const float* h, int j) {
  return d.kind == 2 ? gelu_f(h[j]) : silu_f(h[j]) * h[d.d_h + j];
}

// rows of [Q_chunk; K_chunk]
template <typename TA> struct LoadX {
  Fwd<TA> c;
  __device__ __forceinline__ float operator()(int z, int r, int kk) const {
    const TA* p = r < c.n ? c.q + c.tok(z, r) * c.d.d_k : c.k + c.tok(z, r - c.n) * c.d.d_k;
    return to_f(p[kk]);
  }
};
// B(kk, col) = Wmat[col, kk] for a row-major block of the chunk-start state
template <typename TA> struct LoadWT {
  Fwd<TA> c;
  long long off;  // element offset of the matrix inside the state
  int ld;         // its row length
  __device__ __forceinline__ float operator()(int z, int kk, int col) const {
    return c.src.W[z * c.src.stride + off + (long long)col * ld + kk];
  }
};
// B(kk, j) = Wmat[kk, j]
template <typename TA> struct LoadW {
  Fwd<TA> c;
  long long off;
  int ld;
  __device__ __forceinline__ float operator()(int z, int kk, int j) const {
    return c.src.W[z * c.src.stride + off + (long long)kk * ld + j];
  }
};
// A = silu(H1) * H3 (or gelu(H)) on the [q; k] rows
template <typename TA> struct LoadAct {
  Fwd<TA> c;
  int row0;
  __device__ __forceinline__ float operator()(int z, int r, int j) const {
    return act_of(c.d, c.H + ((size_t)z * 2 * c.d.C + row0 + r) * c.hld(), j);
  }
};
// A(t, kk) = L[t, kk] with L [C, ld] per head in workspace
template <typename TA> struct LoadRow {
  const float* base;
  int C, ld;
  __device__ __forceinline__ float operator()(int z, int t, int kk) const {
    return base[((size_t)z * C + t) * ld + kk];
  }
};
// For the aggregations, A(i, t) = L[t, i] with L [C, ld] per head in workspace
template <typename TA> struct LoadTok {
  const float* base;
  int C, ld;
  __device__ __forceinline__ float operator()(int z, int i, int t) const {
    return base[((size_t)z * C + t) * ld + i];
  }
};
// B(t, j) = k_t[j]
template <typename TA> struct LoadK {
  Fwd<TA> c;
  __device__ __forceinline__ float operator()(int z, int t, int j) const {
    return to_f(c.k[c.tok(z, t) * c.d.d_k + j]);
  }
};
// B(t, j) = A_k[t, j], the activation of the key rows
template <typename TA> struct LoadActK {
  Fwd<TA> c;
  __device__ __forceinline__ float operator()(int z, int t, int j) const {
    return act_of(c.d, c.H + ((size_t)z * 2 * c.d.C + c.n + t) * c.hld(), j);
  }
};
template <typename TA> struct ScaleAB {
  Fwd<TA> c;
  __device__ __forceinline__ float operator()(int z, int t, int i) const {
    size_t o = c.tok(z, t);
    return i == 0 ? c.ca[o] : c.cb[o];
  }
};

// y rows: out for query rows, E = y - v (or -v) for key rows
template <typename TA> struct EpiOutE {
  Fwd<TA> c;
  __device__ __forceinline__ void operator()(int z, int r, int col, const float* acc) const {
    const int dv = c.d.d_v;
    if (r < c.n) {
      c.out[c.tok(z, r) * dv + col] = from_f<TA>(acc[0]);
    } else {
      int t = r - c.n;
      float vv = to_f(c.v[c.tok(z, t) * dv + col]);
      c.E[((size_t)z * c.d.C + t) * dv + col] = (c.d.loss == 0) ? acc[0] - vv : -vv;
    }
  }
};
template <typename TA> struct EpiStoreH {
  Fwd<TA> c;
  __device__ __forceinline__ void operator()(int z, int r, int col, const float* acc) const {
    c.H[((size_t)z * 2 * c.d.C + r) * c.hld() + col] = acc[0];
  }
};
template <typename TA> struct EpiDH {
  Fwd<TA> c;
  __device__ __forceinline__ void operator()(int z, int t, int j, const float* acc) const {
    const int dh = c.d.d_h;
    const float* h = c.H + ((size_t)z * 2 * c.d.C + c.n + t) * c.hld();
    float* o = c.dH + ((size_t)z * c.d.C + t) * c.hld();
    if (c.d.kind == 2) {
      o[j] = acc[0] * dgelu_f(h[j]);
      return;
    }
    float h1 = h[j], h3 = h[dh + j];
    o[j] = acc[0] * h3 * dsilu_f(h1);
    o[dh + j] = acc[0] * silu_f(h1);
  }
};
template <typename TA> struct EpiState {
  Fwd<TA> c;
  long long off;
  int ld;
  __device__ __forceinline__ void operator()(int z, int i, int j, const float* acc) const {
    state_update(c.src, c.dst, c.scal, c.d.BH, c.d.NC, c.ci, z, off + (long long)i * ld + j,
                 acc[0], acc[1]);
  }
};

template <typename TA>
cudaError_t fwd_chunk(const Fwd<TA>& c, cudaStream_t st) {
  const Dims& d = c.d;
  const int n = c.n;
  cudaError_t e;
  if (d.kind == 0) {
    e = simt_gemm<1>(d.BH, 2 * n, d.d_v, d.d_k, LoadX<TA>{c}, LoadWT<TA>{c, 0, d.d_k}, UnitScale{},
                     EpiOutE<TA>{c}, st, "simt_linear_out_e");
    if (e != cudaSuccess) return e;
    return simt_gemm<2>(d.BH, d.d_v, d.d_k, n, LoadTok<TA>{c.E, d.C, d.d_v}, LoadK<TA>{c},
                        ScaleAB<TA>{c}, EpiState<TA>{c, 0, d.d_k}, st, "simt_aggregate_state");
  }
  const int r13 = d.kind == 2 ? d.d_h : 2 * d.d_h;  // rows of W1 (GELU) or [W1; W3]
  const long long o2 = (long long)r13 * d.d_k;
  e = simt_gemm<1>(d.BH, 2 * n, r13, d.d_k, LoadX<TA>{c}, LoadWT<TA>{c, 0, d.d_k},
                   UnitScale{}, EpiStoreH<TA>{c}, st, "simt_g1_h");
  if (e != cudaSuccess) return e;
  e = simt_gemm<1>(d.BH, 2 * n, d.d_v, d.d_h, LoadAct<TA>{c, 0}, LoadWT<TA>{c, o2, d.d_h},
                   UnitScale{}, EpiOutE<TA>{c}, st, "simt_g2_y_out_e");
  if (e != cudaSuccess) return e;
  e = simt_gemm<1>(d.BH, n, d.d_h, d.d_v, LoadRow<TA>{c.E, d.C, d.d_v}, LoadW<TA>{c, o2, d.d_h},
                   UnitScale{}, EpiDH<TA>{c}, st, "simt_g3_da_dh");
  if (e != cudaSuccess) return e;
  e = simt_gemm<2>(d.BH, r13, d.d_k, n, LoadTok<TA>{c.dH, d.C, r13}, LoadK<TA>{c},
                   ScaleAB<TA>{c}, EpiState<TA>{c, 0, d.d_k}, st, "simt_g4_aggregate_w13");
  if (e != cudaSuccess) return e;
  return simt_gemm<2>(d.BH, d.d_v, d.d_h, n, LoadTok<TA>{c.E, d.C, d.d_v}, LoadActK<TA>{c},
                      ScaleAB<TA>{c}, EpiState<TA>{c, o2, d.d_h}, st, "simt_g4_aggregate_w2");
}

}  // namespace

template <typename TA>
cudaError_t simt_fwd(const Dims& d, const TA* q, const TA* k, const TA* v, TA* out,
                     const float* ca, const float* cb, const float* scal, const float* W0,
                     const float* M0, float* W_end, float* M_end, float* saved, float* H,
                     float* E, float* dH, cudaStream_t st) {
  Fwd<TA> c;
  c.d = d;
  c.q = q; c.k = k; c.v = v; c.out = out;
  c.ca = ca; c.cb = cb; c.scal = scal;
  c.H = H; c.E = E; c.dH = dH;
  cudaError_t e = save_initial_state(d, W0, M0, saved, st);
  if (e != cudaSuccess) return e;
  for (int ci = 0; ci < d.NC; ++ci) {
    c.ci = ci;
    c.t0 = ci * d.C;
    c.n = d.T - c.t0 < d.C ? d.T - c.t0 : d.C;
    chunk_states(d, ci, W0, M0, W_end, M_end, saved, &c.src, &c.dst);
    e = fwd_chunk(c, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template cudaError_t simt_fwd<float>(const Dims&, const float*, const float*, const float*, float*,
                                     const float*, const float*, const float*, const float*,
                                     const float*, float*, float*, float*, float*, float*, float*,
                                     cudaStream_t);
template cudaError_t simt_fwd<bf16>(const Dims&, const bf16*, const bf16*, const bf16*, bf16*,
                                    const float*, const float*, const float*, const float*,
                                    const float*, float*, float*, float*, float*, float*, float*,
                                    cudaStream_t);

}  // namespace e2ttt
