// K1: the two scalar kernels of E2-TTT and their adjoint.
//
// "Rethinking Expressivity and Efficiency in Test-Time Training", atlas.scime.ai
// summary, "Approach": unrolling the token-wise recurrence with momentum and
// decay over a chunk gives a momentum kernel and a weight kernel, computed from
// sums of logarithms; arxivlens summary, "Results": the added cost is sums over
// later tokens in log space and sums of ratios of gate products. Per chunk of n
// tokens (1-based t), with
// U(i,j) = prod mu, L(i,j) = prod lam over tokens i..j:
//   SU_t = sum_{s>t} log mu_s,  SL_t = sum_{s>t} log lam_s     (suffix log-sums)
//   a_t  = eta_t exp(SU_t)                                     (momentum kernel)
//   R_t  = exp(SL_t) + mu_{t+1} R_{t+1},  R_n = 1              (ratio sum; affine scan)
//   b_t  = eta_t R_t                                           (weight kernel)
//   U(1,n) = exp(SU_0), L(1,n) = exp(SL_0), c = mu_1 R_1        (chunk scalars)
// No prefix sum is ever subtracted from another, so mu = 0 or lam = 0 (log = -inf)
// gives exact zeros instead of NaN. The logarithms and exponentials are taken in
// base 2 (log2f, exp2f: the identities above hold in any base, at the same
// documented accuracy, 1 and 2 ulp, for fewer instructions). A thread's segment
// of consecutive tokens enters the suffix log-sums through the log of its gate
// product (one log per gate stream and segment), and inside the segment
// U(t+1, n) and L(t+1, n) are the exponentials of the exclusive log-sums times
// the segment's later gates: products of at most a segment's gates, no
// division. Per token that leaves a few multiplications, so the scan is bound
// by its 20 bytes per token rather than by its arithmetic.
//
// Layout: one 128-thread block per (head, chunk) for chunks up to 8192 tokens
// (thread i owns a contiguous segment of ceil(n/128) tokens; segment results are
// combined with warp shuffles, then across warps), else one warp per (head,
// chunk) with segments of ceil(n/32) tokens.
#include "common.cuh"
#include "trace.h"

namespace e2ttt {

namespace {

constexpr int kWarpsPerBlock = 4;

__device__ __forceinline__ void seg_bounds(int n, int lane, int& s0, int& s1) {
  int per = (n + 31) >> 5;
  s0 = min(n, lane * per);
  s1 = min(n, s0 + per);
}

// Inclusive suffix sum across lanes (lane l gets sum over lanes >= l).
__device__ __forceinline__ float warp_suffix_sum(float x, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float y = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x += y;
  }
  return x;
}

// Momentum gate of token t (mu == nullptr: no-momentum mode, mu = 0).
__device__ __forceinline__ float mu_at(const float* mu, int t) { return mu ? mu[t] : 0.f; }

// Per chunk: exclusive suffix log-sums at the end of this lane's segment and
// the chunk totals (lane-uniform).
struct LogSums {
  float su_excl, sl_excl;  // sum over tokens after this lane's segment
  float su_all, sl_all;    // sum over the whole chunk
};

__device__ __forceinline__ LogSums chunk_log_sums(const float* mu, const float* lam, int s0, int s1,
                                                  int lane) {
  float pu = 1.f, pl = 1.f;  // the segment's gate products, one log each
  for (int t = s1 - 1; t >= s0; --t) {
    pu *= mu_at(mu, t);
    pl *= lam[t];
  }
  const float su = log2f(pu), sl = log2f(pl);
  float su_inc = warp_suffix_sum(su, lane);
  float sl_inc = warp_suffix_sum(sl, lane);
  LogSums r;
  r.su_excl = __shfl_down_sync(0xffffffffu, su_inc, 1);
  r.sl_excl = __shfl_down_sync(0xffffffffu, sl_inc, 1);
  if (lane == 31) { r.su_excl = 0.f; r.sl_excl = 0.f; }
  r.su_all = __shfl_sync(0xffffffffu, su_inc, 0);
  r.sl_all = __shfl_sync(0xffffffffu, sl_inc, 0);
  return r;
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
chunk_coeffs_kernel(const float* __restrict__ lr, const float* __restrict__ mom,
                    const float* __restrict__ decay, float* __restrict__ a_out,
                    float* __restrict__ b_out, float* __restrict__ scal, int BH, int T, int C,
                    int NC, int coef) {
  const int lane = threadIdx.x & 31;
  const int wid = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (wid >= BH * NC) return;  // warp-uniform
  const int bh = wid / NC, ci = wid % NC;
  const int t0 = ci * C;
  const int n = min(C, T - t0);
  const size_t base = (size_t)bh * T + t0;
  const float* eta = lr + base;
  const float* mu = mom ? mom + base : nullptr;
  const float* lam = decay + base;
  int s0, s1;
  seg_bounds(n, lane, s0, s1);

  LogSums ls = chunk_log_sums(mu, lam, s0, s1, lane);

  // Reverse walk 1: momentum kernel a_t and the segment's ratio-sum map. The
  // products U(t+1, n), L(t+1, n) start from the exponential of the exclusive
  // log-sum and pick up one gate per token inside the segment.
  const float L_excl = exp2f(ls.sl_excl);
  float U = exp2f(ls.su_excl), L = L_excl;
  float Mseg = 1.f, Cseg = 0.f;
  float asum = 0.f, bsum = 0.f;  // segment sums (chunk means for coef = 1)
  for (int t = s1 - 1; t >= s0; --t) {
    const float at = eta[t] * U;
    a_out[base + t] = at;
    asum += at;
    float m = (t + 1 < n) ? mu_at(mu, t + 1) : 0.f;
    Cseg = L + m * Cseg;
    Mseg = m * Mseg;
    U *= mu_at(mu, t);
    L *= lam[t];
  }
  float M = Mseg, Cc = Cseg;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float Mr = __shfl_down_sync(0xffffffffu, M, off);
    float Cr = __shfl_down_sync(0xffffffffu, Cc, off);
    if (lane + off < 32) {
      Cc = Cc + M * Cr;
      M = M * Mr;
    }
  }
  float r_next = __shfl_down_sync(0xffffffffu, Cc, 1);
  if (lane == 31) r_next = 0.f;

  // Reverse walk 2: R_t and the weight kernel b_t.
  L = L_excl;
  float r1 = 0.f;
  for (int t = s1 - 1; t >= s0; --t) {
    float m = (t + 1 < n) ? mu_at(mu, t + 1) : 0.f;
    float r = L + m * r_next;
    const float bt = eta[t] * r;
    b_out[base + t] = bt;
    bsum += bt;
    r_next = r;
    if (t == 0) r1 = r;
    L *= lam[t];
  }
  if (coef) {  // the chunk-averaged variant: every token carries the chunk means
    const float am = __shfl_sync(0xffffffffu, warp_suffix_sum(asum, lane), 0) / (float)n;
    const float bm = __shfl_sync(0xffffffffu, warp_suffix_sum(bsum, lane), 0) / (float)n;
    for (int t = s0; t < s1; ++t) {
      a_out[base + t] = am;
      b_out[base + t] = bm;
    }
  }
  if (s0 == 0 && s1 > 0) {  // lane 0 holds token 1
    const size_t plane = (size_t)BH * NC;
    const size_t o = (size_t)bh * NC + ci;
    scal[o] = exp2f(ls.su_all);
    scal[plane + o] = exp2f(ls.sl_all);
    scal[2 * plane + o] = mu_at(mu, 0) * r1;
  }
}

// Block version of chunk_coeffs_kernel: one 128-thread block per (head, chunk),
// thread i owning a contiguous segment of ceil(n/128) tokens. The gates are
// staged in shared memory; each segment's log-sums are the logs of its gate
// products (one log per gate stream and segment); the segment
// log-sums and the segment maps of the ratio-sum recurrence are combined with
// warp shuffles and then across the four warps, suffix-wise and by additions and
// products only (never by subtracting a prefix), as in the warp version.
constexpr int kK1Threads = 128;
constexpr int kK1Warps = kK1Threads / 32;
constexpr int kK1MaxC = 8192;  // 3 C floats of shared memory

__global__ void __launch_bounds__(kK1Threads)
chunk_coeffs_block_kernel(const float* __restrict__ lr, const float* __restrict__ mom,
                          const float* __restrict__ decay, float* __restrict__ a_out,
                          float* __restrict__ b_out, float* __restrict__ scal, int BH, int T, int C,
                          int NC, int coef) {
  extern __shared__ float k1s[];
  float* s_eta = k1s;
  float* s_mu = k1s + C;
  float* s_lam = k1s + 2 * C;
  __shared__ float w_su[kK1Warps], w_sl[kK1Warps], w_M[kK1Warps], w_C[kK1Warps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x / NC, ci = blockIdx.x % NC;
  const int t0 = ci * C;
  const int n = min(C, T - t0);
  const size_t base = (size_t)bh * T + t0;
  for (int t = tid; t < n; t += kK1Threads) {
    const float mu = mom ? mom[base + t] : 0.f;  // NULL: no-momentum mode
    s_eta[t] = lr[base + t];
    s_mu[t] = mu;
    s_lam[t] = decay[base + t];
  }
  __syncthreads();
  const int per = (n + kK1Threads - 1) / kK1Threads;
  const int s0 = min(n, tid * per), s1 = min(n, s0 + per);

  // suffix log-sums: exclusive (tokens after this segment) and chunk totals
  float pu = 1.f, pl = 1.f;  // the segment's gate products
  for (int t = s1 - 1; t >= s0; --t) {
    pu *= s_mu[t];
    pl *= s_lam[t];
  }
  const float su = log2f(pu), sl = log2f(pl);
  const float su_inc = warp_suffix_sum(su, lane), sl_inc = warp_suffix_sum(sl, lane);
  if (lane == 0) {
    w_su[warp] = su_inc;
    w_sl[warp] = sl_inc;
  }
  __syncthreads();
  float su_later = 0.f, sl_later = 0.f;  // warps after this one
  for (int w = kK1Warps - 1; w > warp; --w) {
    su_later += w_su[w];
    sl_later += w_sl[w];
  }
  float su_excl = __shfl_down_sync(0xffffffffu, su_inc, 1);
  float sl_excl = __shfl_down_sync(0xffffffffu, sl_inc, 1);
  if (lane == 31) {
    su_excl = 0.f;
    sl_excl = 0.f;
  }
  su_excl += su_later;
  sl_excl += sl_later;
  float su_all = 0.f, sl_all = 0.f;
  for (int w = kK1Warps - 1; w >= 0; --w) {
    su_all += w_su[w];
    sl_all += w_sl[w];
  }

  // reverse walk 1: momentum kernel a_t and the segment's ratio-sum map; the
  // products U(t+1, n), L(t+1, n) start from the exponentials of the exclusive
  // log-sums and pick up one gate per token inside the segment
  const float L_excl = exp2f(sl_excl);
  float U = exp2f(su_excl), L = L_excl;
  float Mseg = 1.f, Cseg = 0.f;
  float asum = 0.f, bsum = 0.f;  // segment sums (chunk means for coef = 1)
  for (int t = s1 - 1; t >= s0; --t) {
    const float at = s_eta[t] * U;
    a_out[base + t] = at;
    asum += at;
    const float m = (t + 1 < n) ? s_mu[t + 1] : 0.f;
    Cseg = L + m * Cseg;
    Mseg = m * Mseg;
    U *= s_mu[t];
    L *= s_lam[t];
  }
  // inclusive suffix composition of the maps within the warp, then across warps
  float M = Mseg, Cc = Cseg;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Mr = __shfl_down_sync(0xffffffffu, M, off);
    const float Cr = __shfl_down_sync(0xffffffffu, Cc, off);
    if (lane + off < 32) {
      Cc = Cc + M * Cr;
      M = M * Mr;
    }
  }
  if (lane == 0) {
    w_M[warp] = M;
    w_C[warp] = Cc;
  }
  __syncthreads();
  float r_end = 0.f;  // R at the first token after this warp's segments
  for (int w = kK1Warps - 1; w > warp; --w) r_end = w_C[w] + w_M[w] * r_end;
  const float Cn = __shfl_down_sync(0xffffffffu, Cc, 1);
  const float Mn = __shfl_down_sync(0xffffffffu, M, 1);
  float r_next = lane == 31 ? r_end : Cn + Mn * r_end;

  // reverse walk 2: R_t and the weight kernel b_t
  L = L_excl;
  float r1 = 0.f;
  for (int t = s1 - 1; t >= s0; --t) {
    const float m = (t + 1 < n) ? s_mu[t + 1] : 0.f;
    const float r = L + m * r_next;
    const float bt = s_eta[t] * r;
    b_out[base + t] = bt;
    bsum += bt;
    r_next = r;
    if (t == 0) r1 = r;
    L *= s_lam[t];
  }
  if (coef) {  // the chunk-averaged variant: every token carries the chunk means
    const float ai = warp_suffix_sum(asum, lane), bi = warp_suffix_sum(bsum, lane);
    __syncthreads();  // w_su / w_sl are free again
    if (lane == 0) {
      w_su[warp] = ai;
      w_sl[warp] = bi;
    }
    __syncthreads();
    float at = 0.f, bt = 0.f;
    for (int w = kK1Warps - 1; w >= 0; --w) {
      at += w_su[w];
      bt += w_sl[w];
    }
    const float am = at / (float)n, bm = bt / (float)n;
    for (int t = s0; t < s1; ++t) {
      a_out[base + t] = am;
      b_out[base + t] = bm;
    }
  }
  if (s0 == 0 && s1 > 0) {  // the thread holding token 1
    const size_t plane = (size_t)BH * NC;
    const size_t o = (size_t)bh * NC + ci;
    scal[o] = exp2f(su_all);
    scal[plane + o] = exp2f(sl_all);
    scal[2 * plane + o] = s_mu[0] * r1;
  }
}

// Vectorised block version for full chunks of C = PER x 128 tokens: thread i
// owns tokens [PER i, PER i + PER) of its chunk, loads its gates with one
// PER-wide vector load per gate (all of them in flight at once), keeps them and
// their logs in registers, and writes a_t, b_t with one vector store each. The
// arithmetic, its order and the cross-thread combination are those of
// chunk_coeffs_block_kernel, so the results are the same bit for bit; only the
// memory access differs (the block kernel's per-token loop waited on one load
// round trip per token).
template <int PER>
__device__ __forceinline__ void load_vec(const float* __restrict__ p, float (&v)[PER]) {
  if constexpr (PER == 1) {
    v[0] = p[0];
  } else if constexpr (PER == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
#pragma unroll
    for (int j = 0; j < PER; j += 4) {
      const float4 x = *reinterpret_cast<const float4*>(p + j);
      v[j] = x.x; v[j + 1] = x.y; v[j + 2] = x.z; v[j + 3] = x.w;
    }
  }
}
template <int PER>
__device__ __forceinline__ void store_vec(float* __restrict__ p, const float (&v)[PER]) {
  if constexpr (PER == 1) {
    p[0] = v[0];
  } else if constexpr (PER == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
#pragma unroll
    for (int j = 0; j < PER; j += 4)
      *reinterpret_cast<float4*>(p + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
  }
}

template <int PER>
__global__ void __launch_bounds__(kK1Threads, PER >= 8 ? 8 : 16)  // 16 blocks (2048 threads) per SM
chunk_coeffs_vec_kernel(const float* __restrict__ lr, const float* __restrict__ mom,
                        const float* __restrict__ decay, float* __restrict__ a_out,
                        float* __restrict__ b_out, float* __restrict__ scal, int BH, int T, int C,
                        int NC, int coef) {
  // A successor launched with programmatic stream serialization (the forward's
  // prep launch) may start now: it waits (griddepcontrol.wait) before it reads
  // a, b or the chunk scalars; plain launches still wait for this grid to end.
  griddep_launch_dependents();
  __shared__ float s_mu_first[kK1Threads + 1];  // first mu of every segment, then 0
  __shared__ float w_su[kK1Warps], w_sl[kK1Warps], w_M[kK1Warps], w_C[kK1Warps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x / NC, ci = blockIdx.x % NC;
  const size_t base = (size_t)bh * T + (size_t)ci * C + (size_t)tid * PER;
  float eta[PER], mu[PER], lam[PER];
  load_vec<PER>(lr + base, eta);
  if (mom) {
    load_vec<PER>(mom + base, mu);
  } else {  // no-momentum mode: mu = 0
#pragma unroll
    for (int i = 0; i < PER; ++i) mu[i] = 0.f;
  }
  load_vec<PER>(decay + base, lam);
  s_mu_first[tid] = mu[0];
  if (tid == 0) s_mu_first[kK1Threads] = 0.f;  // no token after the chunk's last

  // suffix log-sums: exclusive (tokens after this segment) and chunk totals
  float pu = 1.f, pl = 1.f;  // the segment's gate products
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    pu *= mu[i];
    pl *= lam[i];
  }
  const float su = log2f(pu), sl = log2f(pl);
  const float su_inc = warp_suffix_sum(su, lane), sl_inc = warp_suffix_sum(sl, lane);
  if (lane == 0) {
    w_su[warp] = su_inc;
    w_sl[warp] = sl_inc;
  }
  __syncthreads();
  float su_later = 0.f, sl_later = 0.f;  // warps after this one
  for (int w = kK1Warps - 1; w > warp; --w) {
    su_later += w_su[w];
    sl_later += w_sl[w];
  }
  float su_excl = __shfl_down_sync(0xffffffffu, su_inc, 1);
  float sl_excl = __shfl_down_sync(0xffffffffu, sl_inc, 1);
  if (lane == 31) {
    su_excl = 0.f;
    sl_excl = 0.f;
  }
  su_excl += su_later;
  sl_excl += sl_later;
  float su_all = 0.f, sl_all = 0.f;
  for (int w = kK1Warps - 1; w >= 0; --w) {
    su_all += w_su[w];
    sl_all += w_sl[w];
  }
  const float mu_next = s_mu_first[tid + 1];

  // reverse walk 1: momentum kernel a_t and the segment's ratio-sum map
  const float L_excl = exp2f(sl_excl);
  float U = exp2f(su_excl), L = L_excl;
  float Mseg = 1.f, Cseg = 0.f;
  float asum = 0.f, bsum = 0.f;
  float av[PER], bv[PER];
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    av[i] = eta[i] * U;
    asum += av[i];
    const float m = i + 1 < PER ? mu[i + 1] : mu_next;
    Cseg = L + m * Cseg;
    Mseg = m * Mseg;
    U *= mu[i];
    L *= lam[i];
  }
  float M = Mseg, Cc = Cseg;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Mr = __shfl_down_sync(0xffffffffu, M, off);
    const float Cr = __shfl_down_sync(0xffffffffu, Cc, off);
    if (lane + off < 32) {
      Cc = Cc + M * Cr;
      M = M * Mr;
    }
  }
  if (lane == 0) {
    w_M[warp] = M;
    w_C[warp] = Cc;
  }
  __syncthreads();
  float r_end = 0.f;
  for (int w = kK1Warps - 1; w > warp; --w) r_end = w_C[w] + w_M[w] * r_end;
  const float Cn = __shfl_down_sync(0xffffffffu, Cc, 1);
  const float Mn = __shfl_down_sync(0xffffffffu, M, 1);
  float r_next = lane == 31 ? r_end : Cn + Mn * r_end;

  // reverse walk 2: R_t and the weight kernel b_t
  L = L_excl;
  float r1 = 0.f;
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    const float m = i + 1 < PER ? mu[i + 1] : mu_next;
    const float r = L + m * r_next;
    bv[i] = eta[i] * r;
    bsum += bv[i];
    r_next = r;
    if (i == 0) r1 = r;
    L *= lam[i];
  }
  if (coef) {  // the chunk-averaged variant: every token carries the chunk means
    const float ai = warp_suffix_sum(asum, lane), bi = warp_suffix_sum(bsum, lane);
    __syncthreads();  // w_su / w_sl are free again
    if (lane == 0) {
      w_su[warp] = ai;
      w_sl[warp] = bi;
    }
    __syncthreads();
    float at = 0.f, bt = 0.f;
    for (int w = kK1Warps - 1; w >= 0; --w) {
      at += w_su[w];
      bt += w_sl[w];
    }
    const float n = (float)(PER * kK1Threads);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      av[i] = at / n;
      bv[i] = bt / n;
    }
  }
  store_vec<PER>(a_out + base, av);
  store_vec<PER>(b_out + base, bv);
  if (tid == 0) {  // the thread holding token 1
    const size_t plane = (size_t)BH * NC;
    const size_t o = (size_t)bh * NC + ci;
    scal[o] = exp2f(su_all);
    scal[plane + o] = exp2f(sl_all);
    scal[2 * plane + o] = mu[0] * r1;
  }
}

// Adjoint of chunk_coeffs_kernel. Given abar, bbar (per token) and the chunk
// scalar adjoints (PUbar, PLbar, cbar), with
//   X_1 = PUbar, X_{s+1} = mu_s X_s + abar_s eta_s
//   Y_1 = cbar,  Y_{s+1} = mu_s Y_s + bbar_s eta_s
//   V_1 = PLbar, V_{s+1} = lam_s V_s + Y_{s+1}
// the gate gradients are
//   deta_t = abar_t U(t+1,n) + bbar_t R_t
//   dmu_s  = U(s+1,n) X_s + R_s Y_s
//   dlam_s = L(s+1,n) V_s
// (derivatives of the product definitions with the factor s removed; no gate
// is ever divided by). X and (Y, V) are forward affine scans.
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
chunk_coeffs_bwd_kernel(const float* __restrict__ lr, const float* __restrict__ mom,
                        const float* __restrict__ decay, const float* __restrict__ abar,
                        const float* __restrict__ bbar, const float* __restrict__ scal_bar,
                        float* __restrict__ deta, float* __restrict__ dmu,
                        float* __restrict__ dlam, int BH, int T, int C, int NC, int coef) {
  extern __shared__ float sm[];
  const int lane = threadIdx.x & 31;
  const int wl = threadIdx.x >> 5;
  const int wid = blockIdx.x * kWarpsPerBlock + wl;
  if (wid >= BH * NC) return;
  float* sR = sm + (size_t)wl * 3 * C;
  float* sU = sR + C;
  float* sL = sU + C;
  const int bh = wid / NC, ci = wid % NC;
  const int t0 = ci * C;
  const int n = min(C, T - t0);
  const size_t base = (size_t)bh * T + t0;
  const float* eta = lr + base;
  const float* mu = mom ? mom + base : nullptr;
  const float* lam = decay + base;
  const float* ab = abar + base;
  const float* bb = bbar + base;
  int s0, s1;
  seg_bounds(n, lane, s0, s1);
  LogSums ls = chunk_log_sums(mu, lam, s0, s1, lane);
  // The chunk-averaged variant: each token's per-token kernel receives the
  // chunk mean of the adjoints of the (averaged) factors.
  float abm = 0.f, bbm = 0.f;
  if (coef) {
    float sa = 0.f, sb = 0.f;
    for (int t = s0; t < s1; ++t) {
      sa += ab[t];
      sb += bb[t];
    }
    abm = __shfl_sync(0xffffffffu, warp_suffix_sum(sa, lane), 0) / (float)n;
    bbm = __shfl_sync(0xffffffffu, warp_suffix_sum(sb, lane), 0) / (float)n;
  }
  auto AB = [&](int t) { return coef ? abm : ab[t]; };
  auto BB = [&](int t) { return coef ? bbm : bb[t]; };

  // Reverse walks: U(t+1,n), L(t+1,n), R_t into shared memory; deta.
  float su = ls.su_excl, sl = ls.sl_excl;
  float Mseg = 1.f, Cseg = 0.f;
  for (int t = s1 - 1; t >= s0; --t) {
    float m = (t + 1 < n) ? mu_at(mu, t + 1) : 0.f;
    float cl = exp2f(sl);
    sU[t] = exp2f(su);
    sL[t] = cl;
    Cseg = cl + m * Cseg;
    Mseg = m * Mseg;
    su += log2f(mu_at(mu, t));
    sl += log2f(lam[t]);
  }
  float M = Mseg, Cc = Cseg;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float Mr = __shfl_down_sync(0xffffffffu, M, off);
    float Cr = __shfl_down_sync(0xffffffffu, Cc, off);
    if (lane + off < 32) {
      Cc = Cc + M * Cr;
      M = M * Mr;
    }
  }
  float r_next = __shfl_down_sync(0xffffffffu, Cc, 1);
  if (lane == 31) r_next = 0.f;
  for (int t = s1 - 1; t >= s0; --t) {
    float m = (t + 1 < n) ? mu_at(mu, t + 1) : 0.f;
    float r = sL[t] + m * r_next;
    sR[t] = r;
    deta[base + t] = AB(t) * sU[t] + BB(t) * r;
    r_next = r;
  }

  // Forward scans. Segment maps: X -> pX X + uX ;  (Y, V) -> [[p,0],[q,r]] (Y,V) + (u,w).
  float pX = 1.f, uX = 0.f;
  float p = 1.f, q = 0.f, r = 1.f, u = 0.f, w = 0.f;
  for (int s = s0; s < s1; ++s) {
    float m_ = mu_at(mu, s), l_ = lam[s];
    float al = AB(s) * eta[s], be = BB(s) * eta[s];
    uX = m_ * uX + al;
    pX = m_ * pX;
    float q2 = m_ * p + l_ * q;
    float w2 = m_ * u + l_ * w + be;
    p = m_ * p;
    r = l_ * r;
    u = m_ * u + be;
    q = q2;
    w = w2;
  }
  // inclusive prefix composition (later o earlier) across lanes
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    float pXe = __shfl_up_sync(0xffffffffu, pX, off);
    float uXe = __shfl_up_sync(0xffffffffu, uX, off);
    float pe = __shfl_up_sync(0xffffffffu, p, off);
    float qe = __shfl_up_sync(0xffffffffu, q, off);
    float re = __shfl_up_sync(0xffffffffu, r, off);
    float ue = __shfl_up_sync(0xffffffffu, u, off);
    float we = __shfl_up_sync(0xffffffffu, w, off);
    if (lane >= off) {
      // self o earlier
      uX = pX * uXe + uX;
      pX = pX * pXe;
      float np = p * pe;
      float nq = q * pe + r * qe;
      float nr = r * re;
      float nu = p * ue + u;
      float nw = q * ue + r * we + w;
      p = np; q = nq; r = nr; u = nu; w = nw;
    }
  }
  // exclusive: the composition of all earlier lanes, applied to the initial values
  float epX = __shfl_up_sync(0xffffffffu, pX, 1), euX = __shfl_up_sync(0xffffffffu, uX, 1);
  float ep = __shfl_up_sync(0xffffffffu, p, 1), eq = __shfl_up_sync(0xffffffffu, q, 1);
  float er = __shfl_up_sync(0xffffffffu, r, 1), eu = __shfl_up_sync(0xffffffffu, u, 1);
  float ew = __shfl_up_sync(0xffffffffu, w, 1);
  if (lane == 0) { epX = 1.f; euX = 0.f; ep = 1.f; eq = 0.f; er = 1.f; eu = 0.f; ew = 0.f; }
  const size_t plane = (size_t)BH * NC;
  const size_t o = (size_t)bh * NC + ci;
  const float PUb = scal_bar[o], PLb = scal_bar[plane + o], cb = scal_bar[2 * plane + o];
  float X = epX * PUb + euX;
  float Y = ep * cb + eu;
  float V = eq * cb + er * PLb + ew;
  for (int s = s0; s < s1; ++s) {
    if (dmu) dmu[base + s] = sU[s] * X + sR[s] * Y;  // NULL in no-momentum mode
    dlam[base + s] = sL[s] * V;
    float m_ = mu_at(mu, s), l_ = lam[s];
    X = m_ * X + AB(s) * eta[s];
    float Yn = m_ * Y + BB(s) * eta[s];
    V = l_ * V + Yn;
    Y = Yn;
  }
}

// Block version of chunk_coeffs_bwd_kernel for full chunks of C = PER x 128
// tokens: one 128-thread block per (head, chunk), thread i owning tokens
// [PER i, PER i + PER) with its gates and adjoints in registers (one vector
// load each). U(t+1, n) and L(t+1, n) are the exponentials of the exclusive
// suffix log-sums times the segment's later gates and R_t comes from the
// segments' ratio-sum maps combined across lanes and warps, as in
// chunk_coeffs_vec_kernel; the forward scans X and (Y, V) compose each
// thread's segment map across lanes by shuffles and across the four warps
// through shared memory. The same quantities as the warp kernel (one warp per
// chunk, which leaves most of the GPU idle); the rounding differs.
template <int PER>
__global__ void __launch_bounds__(kK1Threads)
chunk_coeffs_bwd_vec_kernel(const float* __restrict__ lr, const float* __restrict__ mom,
                            const float* __restrict__ decay, const float* __restrict__ abar,
                            const float* __restrict__ bbar, const float* __restrict__ scal_bar,
                            float* __restrict__ deta, float* __restrict__ dmu,
                            float* __restrict__ dlam, int BH, int T, int C, int NC, int coef) {
  __shared__ float s_mu_first[kK1Threads + 1];  // first mu of every segment, then 0
  __shared__ float w_su[kK1Warps], w_sl[kK1Warps], w_M[kK1Warps], w_C[kK1Warps];
  __shared__ float w_map[kK1Warps][7];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.x / NC, ci = blockIdx.x % NC;
  const size_t base = (size_t)bh * T + (size_t)ci * C + (size_t)tid * PER;
  float eta[PER], mu[PER], lam[PER], ab[PER], bb[PER];
  load_vec<PER>(lr + base, eta);
  if (mom) {
    load_vec<PER>(mom + base, mu);
  } else {  // no-momentum mode: mu = 0
#pragma unroll
    for (int i = 0; i < PER; ++i) mu[i] = 0.f;
  }
  load_vec<PER>(decay + base, lam);
  load_vec<PER>(abar + base, ab);
  load_vec<PER>(bbar + base, bb);
  s_mu_first[tid] = mu[0];
  if (tid == 0) s_mu_first[kK1Threads] = 0.f;  // no token after the chunk's last
  if (coef) {  // the chunk-averaged variant: every token takes the chunk means
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      sa += ab[i];
      sb += bb[i];
    }
    const float ai = warp_suffix_sum(sa, lane), bi = warp_suffix_sum(sb, lane);
    if (lane == 0) {
      w_M[warp] = ai;
      w_C[warp] = bi;
    }
    __syncthreads();
    float at = 0.f, bt = 0.f;
    for (int w = kK1Warps - 1; w >= 0; --w) {
      at += w_M[w];
      bt += w_C[w];
    }
    __syncthreads();  // w_M and w_C are written again below
    const float n = (float)(PER * kK1Threads);
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      ab[i] = at / n;
      bb[i] = bt / n;
    }
  }

  // exclusive suffix log-sums of the gates after this thread's segment
  float pu = 1.f, pl = 1.f;
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    pu *= mu[i];
    pl *= lam[i];
  }
  const float su_inc = warp_suffix_sum(log2f(pu), lane), sl_inc = warp_suffix_sum(log2f(pl), lane);
  if (lane == 0) {
    w_su[warp] = su_inc;
    w_sl[warp] = sl_inc;
  }
  __syncthreads();
  float su_excl = __shfl_down_sync(0xffffffffu, su_inc, 1);
  float sl_excl = __shfl_down_sync(0xffffffffu, sl_inc, 1);
  if (lane == 31) {
    su_excl = 0.f;
    sl_excl = 0.f;
  }
  for (int w = kK1Warps - 1; w > warp; --w) {
    su_excl += w_su[w];
    sl_excl += w_sl[w];
  }
  const float mu_next = s_mu_first[tid + 1];

  // reverse walk 1: U(t+1, n), L(t+1, n) and the segment's ratio-sum map
  float U = exp2f(su_excl), L = exp2f(sl_excl);
  float Ut[PER], Lt[PER];
  float Mseg = 1.f, Cseg = 0.f;
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    Ut[i] = U;
    Lt[i] = L;
    const float m = i + 1 < PER ? mu[i + 1] : mu_next;
    Cseg = L + m * Cseg;
    Mseg = m * Mseg;
    U *= mu[i];
    L *= lam[i];
  }
  float M = Mseg, Cc = Cseg;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Mr = __shfl_down_sync(0xffffffffu, M, off);
    const float Cr = __shfl_down_sync(0xffffffffu, Cc, off);
    if (lane + off < 32) {
      Cc = Cc + M * Cr;
      M = M * Mr;
    }
  }
  if (lane == 0) {
    w_M[warp] = M;
    w_C[warp] = Cc;
  }
  __syncthreads();
  float r_end = 0.f;
  for (int w = kK1Warps - 1; w > warp; --w) r_end = w_C[w] + w_M[w] * r_end;
  const float Cn = __shfl_down_sync(0xffffffffu, Cc, 1);
  const float Mn = __shfl_down_sync(0xffffffffu, M, 1);
  float r_next = lane == 31 ? r_end : Cn + Mn * r_end;

  // reverse walk 2: R_t and deta_t = abar_t U(t+1, n) + bbar_t R_t
  float Rt[PER], out[PER];
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    const float m = i + 1 < PER ? mu[i + 1] : mu_next;
    const float r = Lt[i] + m * r_next;
    Rt[i] = r;
    out[i] = ab[i] * Ut[i] + bb[i] * r;
    r_next = r;
  }
  store_vec<PER>(deta + base, out);

  // Forward scans. The segment's map: X -> pX X + uX; (Y, V) -> (p Y + u, q Y + r V + w).
  float pX = 1.f, uX = 0.f, p = 1.f, q = 0.f, r = 1.f, u = 0.f, w = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const float m_ = mu[i], l_ = lam[i];
    const float al = ab[i] * eta[i], be = bb[i] * eta[i];
    uX = m_ * uX + al;
    pX = m_ * pX;
    const float q2 = m_ * p + l_ * q;
    const float w2 = m_ * u + l_ * w + be;
    p = m_ * p;
    r = l_ * r;
    u = m_ * u + be;
    q = q2;
    w = w2;
  }
  // inclusive prefix composition across lanes (this lane's map after the earlier ones)
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float pXe = __shfl_up_sync(0xffffffffu, pX, off);
    const float uXe = __shfl_up_sync(0xffffffffu, uX, off);
    const float pe = __shfl_up_sync(0xffffffffu, p, off);
    const float qe = __shfl_up_sync(0xffffffffu, q, off);
    const float re = __shfl_up_sync(0xffffffffu, r, off);
    const float ue = __shfl_up_sync(0xffffffffu, u, off);
    const float we = __shfl_up_sync(0xffffffffu, w, off);
    if (lane >= off) {
      uX = pX * uXe + uX;
      pX = pX * pXe;
      const float np = p * pe;
      const float nq = q * pe + r * qe;
      const float nr = r * re;
      const float nu = p * ue + u;
      const float nw = q * ue + r * we + w;
      p = np; q = nq; r = nr; u = nu; w = nw;
    }
  }
  if (lane == 31) {  // the warp's whole map
    w_map[warp][0] = pX; w_map[warp][1] = uX; w_map[warp][2] = p; w_map[warp][3] = q;
    w_map[warp][4] = r; w_map[warp][5] = u; w_map[warp][6] = w;
  }
  __syncthreads();
  // the chunk's initial values X_1 = PUbar, Y_1 = cbar, V_1 = PLbar, carried
  // through the earlier warps' maps, then through this warp's earlier lanes
  const size_t plane = (size_t)BH * NC;
  const size_t o = (size_t)bh * NC + ci;
  float X = scal_bar[o], Y = scal_bar[2 * plane + o], V = scal_bar[plane + o];
  for (int wi = 0; wi < warp; ++wi) {
    const float* mp = w_map[wi];
    const float Xn = mp[0] * X + mp[1];
    const float Yn = mp[2] * Y + mp[5];
    V = mp[3] * Y + mp[4] * V + mp[6];
    X = Xn;
    Y = Yn;
  }
  {
    float epX = __shfl_up_sync(0xffffffffu, pX, 1), euX = __shfl_up_sync(0xffffffffu, uX, 1);
    float ep = __shfl_up_sync(0xffffffffu, p, 1), eq = __shfl_up_sync(0xffffffffu, q, 1);
    float er = __shfl_up_sync(0xffffffffu, r, 1), eu = __shfl_up_sync(0xffffffffu, u, 1);
    float ew = __shfl_up_sync(0xffffffffu, w, 1);
    if (lane == 0) { epX = 1.f; euX = 0.f; ep = 1.f; eq = 0.f; er = 1.f; eu = 0.f; ew = 0.f; }
    const float Xn = epX * X + euX;
    const float Yn = ep * Y + eu;
    V = eq * Y + er * V + ew;
    X = Xn;
    Y = Yn;
  }
  float om[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    om[i] = Ut[i] * X + Rt[i] * Y;
    out[i] = Lt[i] * V;
    X = mu[i] * X + ab[i] * eta[i];
    const float Yn = mu[i] * Y + bb[i] * eta[i];
    V = lam[i] * V + Yn;
    Y = Yn;
  }
  if (dmu) store_vec<PER>(dmu + base, om);  // NULL in no-momentum mode
  store_vec<PER>(dlam + base, out);
}

}  // namespace

cudaError_t launch_chunk_coeffs(const float* lr, const float* mom, const float* decay, float* a,
                                float* b, float* scal, int BH, int T, int C, int NC, int coef,
                                cudaStream_t st) {
  E2TTT_TRACE("k1_chunk_coeffs", st);
  // Full chunks of 128, 256, 512 or 1024 tokens with vector-aligned gates and
  // outputs: the vectorised kernel (same results as the block kernel).
  const int per = C / kK1Threads;
  const int vb = per >= 4 ? 16 : per * 4;  // alignment of one vector access in bytes
  auto vec_ok = [&](const void* p) { return p == nullptr || ((uintptr_t)p % vb) == 0; };
  if (T % C == 0 && C % kK1Threads == 0 && (per == 1 || per == 2 || per == 4 || per == 8) &&
      vec_ok(lr) && vec_ok(mom) && vec_ok(decay) && vec_ok(a) && vec_ok(b)) {
    switch (per) {
      case 1: chunk_coeffs_vec_kernel<1><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, a, b, scal, BH, T, C, NC, coef); break;
      case 2: chunk_coeffs_vec_kernel<2><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, a, b, scal, BH, T, C, NC, coef); break;
      case 4: chunk_coeffs_vec_kernel<4><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, a, b, scal, BH, T, C, NC, coef); break;
      default: chunk_coeffs_vec_kernel<8><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, a, b, scal, BH, T, C, NC, coef); break;
    }
    return cudaGetLastError();
  }
  if (C <= kK1MaxC) {
    const size_t smem = (size_t)3 * C * sizeof(float);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(chunk_coeffs_block_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    chunk_coeffs_block_kernel<<<BH * NC, kK1Threads, smem, st>>>(lr, mom, decay, a, b, scal, BH, T,
                                                                 C, NC, coef);
    return cudaGetLastError();
  }
  int warps = BH * NC;
  int blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
  chunk_coeffs_kernel<<<blocks, kWarpsPerBlock * 32, 0, st>>>(lr, mom, decay, a, b, scal, BH, T,
                                                               C, NC, coef);
  return cudaGetLastError();
}

cudaError_t launch_chunk_coeffs_bwd(const float* lr, const float* mom, const float* decay,
                                    const float* abar, const float* bbar, const float* scal_bar,
                                    float* deta, float* dmu, float* dlam, int BH, int T, int C,
                                    int NC, int coef, cudaStream_t st) {
  // Full chunks of 128, 256, 512 or 1024 tokens with vector-aligned buffers:
  // one block per chunk.
  const int per = C / kK1Threads;
  const int vb = per >= 4 ? 16 : per * 4;  // alignment of one vector access in bytes
  auto vec_ok = [&](const void* p) { return p == nullptr || ((uintptr_t)p % vb) == 0; };
  if (T % C == 0 && C % kK1Threads == 0 && (per == 1 || per == 2 || per == 4 || per == 8) &&
      vec_ok(lr) && vec_ok(mom) && vec_ok(decay) && vec_ok(abar) && vec_ok(bbar) &&
      vec_ok(deta) && vec_ok(dmu) && vec_ok(dlam)) {
    E2TTT_TRACE("k1_chunk_coeffs_bwd", st);
    switch (per) {
      case 1: chunk_coeffs_bwd_vec_kernel<1><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, abar, bbar, scal_bar, deta, dmu, dlam, BH, T, C, NC, coef); break;
      case 2: chunk_coeffs_bwd_vec_kernel<2><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, abar, bbar, scal_bar, deta, dmu, dlam, BH, T, C, NC, coef); break;
      case 4: chunk_coeffs_bwd_vec_kernel<4><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, abar, bbar, scal_bar, deta, dmu, dlam, BH, T, C, NC, coef); break;
      default: chunk_coeffs_bwd_vec_kernel<8><<<BH * NC, kK1Threads, 0, st>>>(lr, mom, decay, abar, bbar, scal_bar, deta, dmu, dlam, BH, T, C, NC, coef); break;
    }
    return cudaGetLastError();
  }
  int warps = BH * NC;
  int blocks = (warps + kWarpsPerBlock - 1) / kWarpsPerBlock;
  size_t smem = (size_t)kWarpsPerBlock * 3 * C * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(chunk_coeffs_bwd_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  E2TTT_TRACE("k1_chunk_coeffs_bwd", st);
  chunk_coeffs_bwd_kernel<<<blocks, kWarpsPerBlock * 32, smem, st>>>(
      lr, mom, decay, abar, bbar, scal_bar, deta, dmu, dlam, BH, T, C, NC, coef);
  return cudaGetLastError();
}

}  // namespace e2ttt
