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
// (it names a host-side stand-in); the device address is fetched with
// cudaGetSymbolAddress, with the device current, by the first call made on that
// device, so make that first call before any stream capture. A call that is not
// being captured looks the address up again (a cheap host-side query), so a
// context created anew on the device, after cudaDeviceReset for instance, gets
// its own address; a call under capture uses the address the last uncaptured
// call on that device found, so after a reset make one uncaptured call before
// capturing again.
// All calls share the one array and its contents persist between calls; the
// forward resets the only part that must start at zero (its status word) on
// every call. Calls that overlap on the GPU (other streams, other host threads)
// race on the array and must be serialised by the caller. The status word of
// the device-side bounded waits is the first word of the array:
// e2ttt_noalloc_status reads it.
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

// Device address of the static scratch on the current device: looked up again
// unless `stream` is being captured, in which case the address found by the
// last uncaptured call on this device is used (an error if there was none).
e2ttt_status scratch_address(void* stream, void** out, const char* who) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    char msg[160];
    snprintf(msg, sizeof(msg), "%s: no usable current CUDA device", who);
    e2ttt::set_last_error(msg);
    return E2TTT_ERR_CUDA;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing((cudaStream_t)stream, &cap);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "%s: cudaStreamIsCapturing failed: %s", who, cudaGetErrorString(e));
    e2ttt::set_last_error(msg);
    return E2TTT_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      char msg[256];
      snprintf(msg, sizeof(msg), "%s: cudaGetSymbolAddress of the static scratch failed on device %d: %s",
               who, dev, cudaGetErrorString(e));
      e2ttt::set_last_error(msg);
      return E2TTT_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  } else if (!g_scratch_addr[dev]) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "%s: first call on device %d is under stream capture; make one call outside capture first",
             who, dev);
    e2ttt::set_last_error(msg);
    return E2TTT_ERR_INVALID_ARG;
  }
  *out = g_scratch_addr[dev];
  return E2TTT_OK;
}

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
  void* scratch = nullptr;
  const e2ttt_status st = scratch_address(stream, &scratch, "e2ttt_chunk_scan_fwd_noalloc");
  if (st != E2TTT_OK) return st;
  // An invalid shape (need == 0) is reported by the regular entry point.
  return e2ttt_chunk_scan_fwd(shape, q, k, v, lr, mom, decay, W0, M0, out, W_end, M_end,
                              saved_states, scratch, kStaticScratchBytes, stream);
}

extern "C" e2ttt_status e2ttt_noalloc_status(void* stream) {
  void* scratch = nullptr;
  const e2ttt_status st = scratch_address(stream, &scratch, "e2ttt_noalloc_status");
  if (st != E2TTT_OK) return st;
  return e2ttt_workspace_status(scratch, stream);
}
