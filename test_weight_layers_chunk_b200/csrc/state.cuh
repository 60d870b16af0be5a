// Fast-weight state plumbing shared by every forward path.
//
// Chunk i reads the chunk-start state (W, M) and writes the chunk-end state,
// which is the start state of chunk i+1 (abstract of "Rethinking Expressivity
// and Efficiency in Test-Time Training": chunk-end fast-weight and momentum
// states). Where the states live:
//   with saved_states [NC, BH, 2, S]: chunk 0 reads the caller's W0/M0 (a copy
//     goes to saved[0]); chunk i writes saved[i+1]; the last chunk writes
//     W_end/M_end;
//   without: chunk 0 reads W0/M0 and writes W_end/M_end; later chunks update
//     W_end/M_end in place.
#pragma once
#include "common.cuh"

namespace e2ttt {

struct StateIn {
  const float* W;
  const float* M;   // nullptr means a zero momentum state
  long long stride; // elements between consecutive heads
};
struct StateOut {
  float* W;
  float* M;
  long long stride;
};

// The closed-form chunk transition for one state element:
//   M_end = U(1,n) M0 - dM,   W_end = L(1,n) W0 + c M0 - dW
__device__ __forceinline__ void state_update(const StateIn& src, const StateOut& dst,
                                             const float* scal, int BH, int NC, int ci, int z,
                                             long long idx, float dM, float dW) {
  const size_t plane = (size_t)BH * NC;
  const size_t o = (size_t)z * NC + ci;
  const float PU = scal[o], PL = scal[plane + o], cc = scal[2 * plane + o];
  const float m0 = src.M ? src.M[z * src.stride + idx] : 0.f;
  const float w0 = src.W[z * src.stride + idx];
  dst.M[z * dst.stride + idx] = PU * m0 - dM;
  dst.W[z * dst.stride + idx] = PL * w0 + cc * m0 - dW;
}

inline void chunk_states(const Dims& d, int ci, const float* W0, const float* M0, float* W_end,
                         float* M_end, float* saved, StateIn* src, StateOut* dst) {
  const long long S = d.S;
  const size_t per_chunk = (size_t)d.BH * 2 * S;
  if (saved) {
    if (ci == 0) *src = StateIn{W0, M0, S};
    else *src = StateIn{saved + ci * per_chunk, saved + ci * per_chunk + S, 2 * S};
    if (ci + 1 < d.NC) *dst = StateOut{saved + (ci + 1) * per_chunk, saved + (ci + 1) * per_chunk + S, 2 * S};
    else *dst = StateOut{W_end, M_end, S};
    return;
  }
  // In place after the first chunk: every state element is read and then
  // written by the same thread, and no other kernel of the chunk reads the
  // fp32 state while the aggregation kernel updates it.
  if (ci == 0) *src = StateIn{W0, M0, S};
  else *src = StateIn{W_end, M_end, S};
  *dst = StateOut{W_end, M_end, S};
}

inline cudaError_t save_initial_state(const Dims& d, const float* W0, const float* M0, float* saved,
                                      cudaStream_t st) {
  if (!saved) return cudaSuccess;
  const size_t row = (size_t)d.S * sizeof(float);
  cudaError_t e = cudaMemcpy2DAsync(saved, 2 * row, W0, row, row, d.BH, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return e;
  if (M0) return cudaMemcpy2DAsync(saved + d.S, 2 * row, M0, row, row, d.BH, cudaMemcpyDeviceToDevice, st);
  return cudaMemset2DAsync(saved + d.S, 2 * row, 0, row, d.BH, st);
}

}  // namespace e2ttt
