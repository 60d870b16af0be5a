// Forward entry point for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand over a workspace: an application
// whose device memory is already claimed up front by its own pool allocator
// (a cudaMalloc would fail or fragment that pool), a C host program with no
// device allocator of its own, or a latency-critical loop where cudaMalloc's
// implicit device synchronisation is not acceptable. This file gives them
// e2ttt_chunk_scan_fwd_noalloc: the same forward as e2ttt_chunk_scan_fwd, with
// its scratch taken from a fixed, library-owned device array instead of a
// caller workspace.
//
// The array is a file-scope __device__ variable of kStaticScratchBytes (32 MiB),
// so every GPU on which the library's kernels are loaded holds it until the
// process exits. Host code cannot use the array's name as a device address
// (it names a host-side stand-in); the device address is fetched once per
// device with cudaGetSymbolAddress, with that device current, on the first call
// made on that device. Make that first call before any stream capture.
// All calls share the one array and its contents persist between calls; the
// forward resets the only part that must start at zero (its status word) on
// every call. Calls that overlap on the GPU (other streams, other host threads)
// race on the array and must be serialised by the caller.
#include <stdio.h>

#include <mutex>

#include "../../include/e2ttt.h"

namespace e2ttt {
void set_last_error(const char* msg);
}

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" e2ttt_status e2ttt_chunk_scan_fwd_noalloc(
    const e2ttt_shape* shape, const void* q, const void* k, const void* v, const float* lr,
    const float* mom, const float* decay, const float* W0, const float* M0, void* out,
    float* W_end, float* M_end, float* saved_states, void* stream) {
  const size_t need = e2ttt_workspace_bytes(shape, 0);
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "e2ttt_chunk_scan_fwd_noalloc: this shape needs %zu bytes of scratch, the library's "
             "static scratch holds %zu; use e2ttt_chunk_scan_fwd with a caller workspace",
             need, kStaticScratchBytes);
    e2ttt::set_last_error(msg);
    return E2TTT_ERR_INVALID_ARG;
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    e2ttt::set_last_error("e2ttt_chunk_scan_fwd_noalloc: no usable current CUDA device");
    return E2TTT_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_static_scratch);
      if (e != cudaSuccess || !p) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "e2ttt_chunk_scan_fwd_noalloc: cudaGetSymbolAddress of the static scratch failed "
                 "on device %d: %s", dev, cudaGetErrorString(e));
        e2ttt::set_last_error(msg);
        return E2TTT_ERR_CUDA;
      }
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  // An invalid shape (need == 0) is reported by the regular entry point.
  return e2ttt_chunk_scan_fwd(shape, q, k, v, lr, mom, decay, W0, M0, out, W_end, M_end,
                              saved_states, scratch, kStaticScratchBytes, stream);
}
