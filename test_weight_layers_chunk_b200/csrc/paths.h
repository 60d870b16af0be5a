// Internal interfaces between the C ABI layer and the compute paths.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace e2ttt {

// K1 (scan.cu): scalar kernels of every chunk, and their adjoint. coef = 1 gives
// every token of a chunk the chunk means of a_t, b_t (and, in the adjoint, the
// chunk means of abar, bbar).
cudaError_t launch_chunk_coeffs(const float* lr, const float* mom, const float* decay, float* a,
                                float* b, float* scal, int BH, int T, int C, int NC, int coef,
                                cudaStream_t st);
cudaError_t launch_chunk_coeffs_bwd(const float* lr, const float* mom, const float* decay,
                                    const float* abar, const float* bbar, const float* scal_bar,
                                    float* deta, float* dmu, float* dlam, int BH, int T, int C,
                                    int NC, int coef, cudaStream_t st);

// fp32 CUDA-core forward (simt_fwd.cu).
template <typename TA>
cudaError_t simt_fwd(const Dims& d, const TA* q, const TA* k, const TA* v, TA* out,
                     const float* ca, const float* cb, const float* scal, const float* W0,
                     const float* M0, float* W_end, float* M_end, float* saved, float* H,
                     float* E, float* dH, cudaStream_t st);

// saved_states: the chunk-start states, then (save_acts) the per-chunk
// activations of the tensor-core forward, bf16: E [NC][BH][C][d_v] (the key
// rows' residual) and dH [NC][BH][C][hw] (the inner loss's hidden gradient),
// each region 256-byte aligned.
struct SavedLayout {
  size_t states, e, dh, total;  // byte offsets of E and dH; total bytes
};
inline SavedLayout saved_layout(const Dims& d) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  SavedLayout L{};
  L.states = (size_t)d.NC * d.BH * 2 * (size_t)d.S * sizeof(float);
  L.total = L.states;
  L.e = L.dh = 0;
  if (d.save_acts && d.kind != 0) {
    const size_t hw = (size_t)(d.kind == 1 ? 2 : 1) * d.d_h;
    L.e = up(L.states);
    L.dh = up(L.e + (size_t)d.NC * d.BH * d.C * d.d_v * 2);
    L.total = L.dh + (size_t)d.NC * d.BH * d.C * hw * 2;
  }
  return L;
}

// tcgen05 tensor-core forward for bf16 activations (tc_fwd.cu). acts_e / acts_dh:
// the saved activations' E and dH regions (save_acts), else NULL.
bool tc_fwd_supported(const Dims& d, bool bf16_act);
size_t tc_fwd_scratch_bytes(const Dims& d);
cudaError_t tc_fwd(const Dims& d, const bf16* q, const bf16* k, const bf16* v, bf16* out,
                   const float* ca, const float* cb, const float* scal, const float* W0,
                   const float* M0, float* W_end, float* M_end, float* saved, void* scratch,
                   int* status, cudaStream_t st, bf16* acts_e = nullptr, bf16* acts_dh = nullptr);

// Test hook behind e2ttt_test_stall_next_forward (tc_fwd.cu).
void arm_forward_stall(bool on);

// Backward (bwd.cu).
struct BwdArgs {
  Dims d;
  const void *q, *k, *v;
  const float *lr, *mom, *decay, *saved;
  const void* dout;
  const float *dW_end, *dM_end;
  void *dq, *dk, *dv;
  float *dlr, *dmom, *ddecay, *dW0, *dM0;
  void* ws;
  cudaStream_t st;
  const bf16 *acts_e, *acts_dh;  // saved activations (save_acts, read only), else NULL
};
size_t bwd_workspace_bytes(const Dims& d, bool bf16_act);
template <typename TA>
cudaError_t bwd_run(const BwdArgs& a);

// tcgen05 tensor-core backward (tc_bwd.cu): SwiGLU, bf16, tile-aligned shapes.
bool tc_bwd_supported(const Dims& d, bool bf16_act);
size_t tc_bwd_workspace_bytes(const Dims& d);
cudaError_t tc_bwd(const BwdArgs& a);

}  // namespace e2ttt
