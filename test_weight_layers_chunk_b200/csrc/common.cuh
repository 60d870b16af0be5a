// Shared device helpers of the E2-TTT chunk-scan library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace e2ttt {

typedef __nv_bfloat16 bf16;

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<bf16>(bf16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// silu(z) = z * sigmoid(z) and its first two derivatives (SwiGLU fast MLP).
__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float silu_f(float z) { return z * sigmoid_f(z); }
__device__ __forceinline__ float dsilu_f(float z) {
  float s = sigmoid_f(z);
  return s * (1.0f + z * (1.0f - s));
}
__device__ __forceinline__ float d2silu_f(float z) {
  float s = sigmoid_f(z);
  return s * (1.0f - s) * (2.0f + z * (1.0f - 2.0f * s));
}

// Sizes of one problem as the kernels see them.
struct Dims {
  int BH;      // batch rows x heads
  int T, C, NC;
  int d_k, d_v, d_h;
  int kind, loss;
  int coef;    // 0: per-token kernels, 1: chunk means (the chunk-averaged variant)
  int nomom;   // 1: no momentum (mu = 0, no M state)
  int fp32_gemm;  // 1: the fp32 CUDA-core kernels even where the tensor cores apply
  int save_acts;  // 1: per-chunk E and dH kept in saved_states after the states
  long long S; // state elements per head
};

// The standard normal CDF Phi(z) and density phi(z) for the GELU MLP fast
// weight (GELU z Phi(z), not the tanh form). Phi comes from erfc(|z| / sqrt 2)
// by the rational approximation of Abramowitz and Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (after Hastings; absolute error at
// most 1.5e-7 in erf): erfc(x) ~ t (a1 + t (a2 + t (a3 + t (a4 + t a5))))
// exp(-x^2) with t = 1 / (1 + p x). At x = |z| / sqrt 2 its exponential is
// exp(-z^2 / 2), which phi needs too, so one exponential and one reciprocal
// give both. The negative side is taken as Phi(-|z|) = erfc(|z| / sqrt 2) / 2
// directly, without the cancellation in 1 + erf.
struct NormCdfPdf {
  float cdf, pdf;
};
__device__ __forceinline__ NormCdfPdf norm_cdf_pdf(float z) {
  const float e = exp2f(-0.72134752044448170f * z * z);  // exp(-z^2 / 2): -log2(e) / 2
  const float x = fabsf(z) * 0.70710678118654752f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, x, 1.0f));
  float s = fmaf(t, 1.061405429f, -1.453152027f);
  s = fmaf(t, s, 1.421413741f);
  s = fmaf(t, s, -0.284496736f);
  s = fmaf(t, s, 0.254829592f);
  const float tail = 0.5f * t * s * e;  // Phi(-|z|)
  return {z >= 0.0f ? 1.0f - tail : tail, 0.39894228040143268f * e};
}
__device__ __forceinline__ float gelu_f(float z) { return z * norm_cdf_pdf(z).cdf; }
// gelu'(z) = Phi(z) + z phi(z)
__device__ __forceinline__ float dgelu_f(float z) {
  const NormCdfPdf n = norm_cdf_pdf(z);
  return fmaf(z, n.pdf, n.cdf);
}
// gelu''(z) = phi(z) (2 - z^2)
__device__ __forceinline__ float d2gelu_f(float z) { return norm_cdf_pdf(z).pdf * (2.0f - z * z); }

// Programmatic dependent launch (sm_90 and later). A kernel launched with the
// programmatic stream serialization attribute (launch_pdl) may start while its
// predecessor on the stream still runs: griddep_wait() blocks until that
// predecessor has completed and its memory operations are visible, so it comes
// before the kernel's first global memory access. griddep_launch_dependents()
// lets the successor start early (its own griddep_wait() still orders it).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with programmatic stream serialization: the kernel must call
// griddep_wait() before touching global memory.
template <class... Params, class... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace e2ttt
