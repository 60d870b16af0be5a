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

// tcgen05 tensor-core forward for bf16 activations (tc_fwd.cu).
bool tc_fwd_supported(const Dims& d, bool bf16_act);
size_t tc_fwd_scratch_bytes(const Dims& d);
cudaError_t tc_fwd(const Dims& d, const bf16* q, const bf16* k, const bf16* v, bf16* out,
                   const float* ca, const float* cb, const float* scal, const float* W0,
                   const float* M0, float* W_end, float* M_end, float* saved, void* scratch,
                   int* status, cudaStream_t st);

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
};
size_t bwd_workspace_bytes(const Dims& d, bool bf16_act);
template <typename TA>
cudaError_t bwd_run(const BwdArgs& a);

// tcgen05 tensor-core backward (tc_bwd.cu): SwiGLU, bf16, tile-aligned shapes.
bool tc_bwd_supported(const Dims& d, bool bf16_act);
size_t tc_bwd_workspace_bytes(const Dims& d);
cudaError_t tc_bwd(const BwdArgs& a);

}  // namespace e2ttt
