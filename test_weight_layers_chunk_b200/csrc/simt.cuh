// Tiled fp32 CUDA-core GEMM with pluggable operand loaders and epilogue.
//
//   acc_i[m, n] = sum_k A(z, m, k) * B(z, k, n) * s_i(z, k),   i < NACC
//
// z = blockIdx.z (one head), 64x64 output tile per 256-thread block, 4x4 outputs
// per thread per accumulator. Loaders return float, so the same kernel serves
// fp32 and bf16 activations, transposed operands and operands computed on the
// fly (e.g. silu(h1) * h3). Used for fp32 activations and for shapes the
// tensor-core path does not tile.
#pragma once
#include "common.cuh"
#include "trace.h"

namespace e2ttt {

constexpr int kSimtBM = 64, kSimtBN = 64, kSimtBK = 16;

struct UnitScale {
  __device__ __forceinline__ float operator()(int, int, int) const { return 1.f; }
};

template <int NACC, class LA, class LB, class SC, class EPI>
__global__ void __launch_bounds__(256)
simt_gemm_kernel(int M, int N, int K, LA la, LB lb, SC sc, EPI epi) {
  __shared__ float As[kSimtBK][kSimtBM + 4];
  __shared__ float Bs[NACC][kSimtBK][kSimtBN + 4];
  const int z = blockIdx.z;
  const int m0 = blockIdx.y * kSimtBM, n0 = blockIdx.x * kSimtBN;
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[NACC][4][4];
#pragma unroll
  for (int i = 0; i < NACC; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][r][c] = 0.f;

  for (int k0 = 0; k0 < K; k0 += kSimtBK) {
#pragma unroll
    for (int e = tid; e < kSimtBM * kSimtBK; e += 256) {
      int kk = e & (kSimtBK - 1), mm = e >> 4;  // consecutive threads walk k
      int m = m0 + mm, k = k0 + kk;
      As[kk][mm] = (m < M && k < K) ? la(z, m, k) : 0.f;
    }
#pragma unroll
    for (int e = tid; e < kSimtBN * kSimtBK; e += 256) {
      int nn = e & (kSimtBN - 1), kk = e >> 6;  // consecutive threads walk n
      int n = n0 + nn, k = k0 + kk;
      float bv = (n < N && k < K) ? lb(z, k, n) : 0.f;
#pragma unroll
      for (int i = 0; i < NACC; ++i) Bs[i][kk][nn] = (k < K) ? bv * sc(z, k, i) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSimtBK; ++kk) {
      float a[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = As[kk][ty * 4 + r];
#pragma unroll
      for (int i = 0; i < NACC; ++i) {
        float b[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) b[c] = Bs[i][kk][tx * 4 + c];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[i][r][c] = fmaf(a[r], b[c], acc[i][r][c]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      int m = m0 + ty * 4 + r, n = n0 + tx * 4 + c;
      if (m < M && n < N) {
        float v[NACC];
#pragma unroll
        for (int i = 0; i < NACC; ++i) v[i] = acc[i][r][c];
        epi(z, m, n, v);
      }
    }
}

template <int NACC, class LA, class LB, class SC, class EPI>
cudaError_t simt_gemm(int Z, int M, int N, int K, LA la, LB lb, SC sc, EPI epi, cudaStream_t st,
                      const char* name = "simt_gemm") {
  if (M <= 0 || N <= 0 || Z <= 0) return cudaSuccess;
  E2TTT_TRACE(name, st);
  dim3 grid((N + kSimtBN - 1) / kSimtBN, (M + kSimtBM - 1) / kSimtBM, Z);
  simt_gemm_kernel<NACC><<<grid, 256, 0, st>>>(M, N, K, la, lb, sc, epi);
  return cudaGetLastError();
}

}  // namespace e2ttt
