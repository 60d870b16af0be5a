// C ABI of the E2-TTT chunk-scan library: argument checks, workspace layout,
// dispatch to the tensor-core or CUDA-core path. See include/e2ttt.h.
#include <stdarg.h>
#include <stdint.h>
#include <string.h>

#include <cstdio>
#include <initializer_list>
#include <string>

#include "../../include/e2ttt.h"
#include "common.cuh"
#include "paths.h"

namespace e2ttt {
namespace {

thread_local std::string g_last_error;

e2ttt_status fail(e2ttt_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
e2ttt_status fail(e2ttt_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

e2ttt_status cuda_fail(cudaError_t e, const char* where) {
  return fail(E2TTT_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

bool shape_ok(const e2ttt_shape* s, std::string* why) {
  char buf[256];
  if (!s) { *why = "shape is NULL"; return false; }
  if (s->B < 1 || s->H < 1 || s->T < 1 || s->C < 1 || s->d_k < 1 || s->d_v < 1) {
    snprintf(buf, sizeof(buf), "sizes must be >= 1 (B=%d H=%d T=%d C=%d d_k=%d d_v=%d)", s->B, s->H,
             s->T, s->C, s->d_k, s->d_v);
    *why = buf;
    return false;
  }
  if (s->kind != E2TTT_LINEAR && s->kind != E2TTT_SWIGLU && s->kind != E2TTT_GELU_MLP) { *why = "unknown fast-weight kind"; return false; }
  if (s->act != E2TTT_F32 && s->act != E2TTT_BF16) { *why = "unknown activation dtype"; return false; }
  if (s->loss != E2TTT_LOSS_MSE && s->loss != E2TTT_LOSS_NEG_DOT) { *why = "unknown loss"; return false; }
  if (s->coef != E2TTT_COEF_PER_TOKEN && s->coef != E2TTT_COEF_CHUNK_MEAN) { *why = "unknown coef"; return false; }
  if (s->momentum != E2TTT_MOMENTUM && s->momentum != E2TTT_NO_MOMENTUM) { *why = "unknown momentum mode"; return false; }
  if (s->gemm != E2TTT_GEMM_AUTO && s->gemm != E2TTT_GEMM_FP32) { *why = "unknown gemm precision"; return false; }
  if (s->save_acts != E2TTT_RECOMPUTE_ACTS && s->save_acts != E2TTT_SAVE_ACTS) { *why = "unknown save_acts mode"; return false; }
  if (s->kind != E2TTT_LINEAR && s->d_h < 1) { *why = "SwiGLU and the GELU MLP need d_h >= 1"; return false; }
  if (s->C > 1024) { *why = "chunk size C must be <= 1024"; return false; }
  long long BH = (long long)s->B * s->H;
  if (BH > 65535) { *why = "B*H must be <= 65535"; return false; }
  long long dmax = s->d_k;
  if (s->d_v > dmax) dmax = s->d_v;
  if (s->kind != E2TTT_LINEAR && 2LL * s->d_h > dmax) dmax = 2LL * s->d_h;
  if (BH * s->T * dmax >= (1LL << 31)) { *why = "B*H*T*max(d) must be < 2^31"; return false; }
  return true;
}

Dims make_dims(const e2ttt_shape* s) {
  Dims d;
  d.BH = s->B * s->H;
  d.T = s->T;
  d.C = s->C;
  d.NC = (s->T + s->C - 1) / s->C;
  d.d_k = s->d_k;
  d.d_v = s->d_v;
  d.d_h = s->kind != E2TTT_LINEAR ? s->d_h : 0;
  d.kind = s->kind;
  d.loss = s->loss;
  d.coef = s->coef;
  d.nomom = s->momentum == E2TTT_NO_MOMENTUM;
  d.fp32_gemm = s->gemm == E2TTT_GEMM_FP32;
  d.save_acts = s->save_acts == E2TTT_SAVE_ACTS;
  d.S = s->kind == E2TTT_LINEAR     ? (long long)s->d_v * s->d_k
        : s->kind == E2TTT_GELU_MLP ? (long long)s->d_h * s->d_k + (long long)s->d_v * s->d_h
                                    : 2LL * s->d_h * s->d_k + (long long)s->d_v * s->d_h;
  return d;
}

// ------------------------------------------------------------------ workspace layout
struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes);
    return o;
  }
};

struct FwdWs {
  size_t status;                    // device status word (bounded waits)
  size_t a, b, scal, H, E, dH;      // fp32 CUDA-core path
  size_t mscr;                      // no-momentum mode: the CUDA-core path's M_end scratch
  size_t tc;                        // tensor-core path scratch
  size_t total;
};

// Status word and coefficients, then one region shared by the tensor-core
// scratch and the CUDA-core scratch (only one path runs per call).
FwdWs fwd_layout(const Dims& d, bool tc_shape) {
  Bump w;
  FwdWs L{};
  const size_t f = sizeof(float);
  L.status = w.take(256);
  L.a = w.take((size_t)d.BH * d.T * f);
  L.b = w.take((size_t)d.BH * d.T * f);
  L.scal = w.take((size_t)3 * d.BH * d.NC * f);
  const size_t region = w.off;
  Bump s;
  s.off = region;
  const size_t nf = d.kind == 1 ? 2 : 1;  // activation factors per hidden unit
  if (d.kind != 0) L.H = s.take((size_t)d.BH * 2 * d.C * nf * d.d_h * f);
  L.E = s.take((size_t)d.BH * d.C * d.d_v * f);
  if (d.kind != 0) L.dH = s.take((size_t)d.BH * d.C * nf * d.d_h * f);
  size_t end = s.off;
  L.tc = region;
  if (tc_shape) {
    size_t tend = align_up(region + tc_fwd_scratch_bytes(d));
    if (tend > end) end = tend;
  }
  L.mscr = 0;
  if (d.nomom) {
    L.mscr = align_up(end);
    end = L.mscr + (size_t)d.BH * d.S * sizeof(float);
  }
  L.total = end;
  return L;
}
// The backward's workspace; in no-momentum mode followed by the scratch that
// stands in for dM0 (the momentum adjoint, identically zero there).
size_t bwd_total_bytes(const Dims& d, bool bf, size_t* dm_off) {
  size_t n = bwd_workspace_bytes(d, bf);
  *dm_off = 0;
  if (d.nomom) {
    *dm_off = align_up(n);
    n = *dm_off + (size_t)d.BH * d.S * sizeof(float);
  }
  return n;
}

bool aligned16(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (((uintptr_t)p) & 15) return false;
  return true;
}

struct Range {
  const void* p;
  size_t n;
  const char* name;
};

bool overlaps(const Range& a, const Range& b) {
  if (!a.p || !b.p || !a.n || !b.n) return false;
  uintptr_t a0 = (uintptr_t)a.p, b0 = (uintptr_t)b.p;
  return a0 < b0 + b.n && b0 < a0 + a.n;
}

// Every output must be disjoint from every input and every other output.
bool check_overlaps(const Range* in, int nin, const Range* out, int nout, std::string* why) {
  for (int i = 0; i < nout; ++i) {
    for (int j = 0; j < nin; ++j)
      if (overlaps(out[i], in[j])) { *why = std::string(out[i].name) + " overlaps input " + in[j].name; return false; }
    for (int j = i + 1; j < nout; ++j)
      if (overlaps(out[i], out[j])) { *why = std::string(out[i].name) + " overlaps output " + out[j].name; return false; }
  }
  return true;
}

}  // namespace

// Lets other translation units of the library report a failure through
// e2ttt_last_error().
void set_last_error(const char* msg) { g_last_error = msg; }

}  // namespace e2ttt

using namespace e2ttt;

extern "C" {

size_t e2ttt_state_elems(const e2ttt_shape* s) {
  std::string why;
  if (!shape_ok(s, &why)) return 0;
  return (size_t)make_dims(s).S;
}

int e2ttt_num_chunks(const e2ttt_shape* s) {
  std::string why;
  if (!shape_ok(s, &why)) return 0;
  return make_dims(s).NC;
}

size_t e2ttt_saved_bytes(const e2ttt_shape* s) {
  std::string why;
  if (!shape_ok(s, &why)) return 0;
  return saved_layout(make_dims(s)).total;
}

int e2ttt_fwd_uses_tensor_cores(const e2ttt_shape* s) {
  std::string why;
  if (!shape_ok(s, &why)) return -1;
  return tc_fwd_supported(make_dims(s), s->act == E2TTT_BF16) ? 1 : 0;
}

size_t e2ttt_workspace_bytes(const e2ttt_shape* s, int for_bwd) {
  std::string why;
  if (!shape_ok(s, &why)) return 0;
  Dims d = make_dims(s);
  size_t dm_off;
  if (for_bwd) return bwd_total_bytes(d, s->act == E2TTT_BF16, &dm_off);
  return fwd_layout(d, tc_fwd_supported(d, s->act == E2TTT_BF16)).total;
}

const char* e2ttt_status_string(e2ttt_status st) {
  switch (st) {
    case E2TTT_OK: return "E2TTT_OK";
    case E2TTT_ERR_INVALID_ARG: return "E2TTT_ERR_INVALID_ARG: invalid argument";
    case E2TTT_ERR_UNSUPPORTED: return "E2TTT_ERR_UNSUPPORTED: valid but not implemented";
    case E2TTT_ERR_CUDA: return "E2TTT_ERR_CUDA: a CUDA call or kernel launch failed";
    case E2TTT_ERR_TIMEOUT: return "E2TTT_ERR_TIMEOUT: a device-side bounded wait gave up";
  }
  return "unknown e2ttt_status";
}

const char* e2ttt_last_error(void) { return g_last_error.c_str(); }

e2ttt_status e2ttt_workspace_status(const void* ws, void* stream) {
  g_last_error.clear();
  if (!ws) return fail(E2TTT_ERR_INVALID_ARG, "workspace is NULL");
  int word = 0;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the workspace status word");
  if (word != 0)
    return fail(E2TTT_ERR_TIMEOUT, "a device-side wait gave up (code %d: 1 = TMA producer, 2 = MMA issuer, 3 = epilogue)", word);
  return E2TTT_OK;
}

void e2ttt_test_stall_next_forward(int on) { arm_forward_stall(on != 0); }

e2ttt_status e2ttt_chunk_coeffs(const e2ttt_shape* s, const float* lr, const float* mom,
                                const float* decay, float* a, float* b, float* scal,
                                void* stream) {
  g_last_error.clear();
  std::string why;
  if (!shape_ok(s, &why)) return fail(E2TTT_ERR_INVALID_ARG, "%s", why.c_str());
  if (!lr || !decay || !a || !b || !scal)
    return fail(E2TTT_ERR_INVALID_ARG, "e2ttt_chunk_coeffs: NULL pointer argument");
  Dims d = make_dims(s);
  if (d.nomom != (mom == nullptr))
    return fail(E2TTT_ERR_INVALID_ARG, d.nomom ? "no-momentum mode: mom must be NULL"
                                               : "e2ttt_chunk_coeffs: mom is NULL");
  size_t g = (size_t)d.BH * d.T * sizeof(float);
  Range in[] = {{lr, g, "lr"}, {mom, g, "mom"}, {decay, g, "decay"}};
  Range out[] = {{a, g, "a"}, {b, g, "b"}, {scal, (size_t)3 * d.BH * d.NC * sizeof(float), "chunk_scalars"}};
  if (!check_overlaps(in, 3, out, 3, &why)) return fail(E2TTT_ERR_INVALID_ARG, "%s", why.c_str());
  cudaError_t e = launch_chunk_coeffs(lr, mom, decay, a, b, scal, d.BH, d.T, d.C, d.NC, d.coef,
                                      (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "chunk coefficient kernel");
  return E2TTT_OK;
}

e2ttt_status e2ttt_chunk_scan_fwd(const e2ttt_shape* s, const void* q, const void* k, const void* v,
                                  const float* lr, const float* mom, const float* decay,
                                  const float* W0, const float* M0, void* out, float* W_end,
                                  float* M_end, float* saved, void* ws, size_t ws_bytes,
                                  void* stream) {
  g_last_error.clear();
  std::string why;
  if (!shape_ok(s, &why)) return fail(E2TTT_ERR_INVALID_ARG, "%s", why.c_str());
  if (!q || !k || !v || !lr || !decay || !W0 || !out || !W_end)
    return fail(E2TTT_ERR_INVALID_ARG, "e2ttt_chunk_scan_fwd: NULL pointer argument (only M0 and saved_states may be NULL)");
  Dims d = make_dims(s);
  if (d.nomom && (mom || M0 || M_end))
    return fail(E2TTT_ERR_INVALID_ARG, "no-momentum mode: mom, M0 and M_end must be NULL");
  if (!d.nomom && (!mom || !M_end))
    return fail(E2TTT_ERR_INVALID_ARG, "e2ttt_chunk_scan_fwd: mom and M_end are required");
  const bool bf = s->act == E2TTT_BF16;
  const bool tc_shape = tc_fwd_supported(d, bf);
  FwdWs L = fwd_layout(d, tc_shape);
  const bool tc = tc_shape && aligned16({q, k, v, out, W0, M0, W_end, M_end, saved});
  if (d.save_acts) {
    if (d.kind == E2TTT_LINEAR)
      return fail(E2TTT_ERR_UNSUPPORTED, "save_acts: only the SwiGLU and GELU MLP fast weights save activations");
    if (!saved) return fail(E2TTT_ERR_INVALID_ARG, "save_acts needs saved_states");
    if (!tc)
      return fail(E2TTT_ERR_UNSUPPORTED, "save_acts needs the tensor-core path (bf16 activations, gemm auto, "
                                         "tile-aligned sizes, 16-byte aligned pointers)");
  }
  const SavedLayout SL = saved_layout(d);
  if (!ws) return fail(E2TTT_ERR_INVALID_ARG, "workspace is NULL (needs %zu bytes)", L.total);
  if (ws_bytes < L.total)
    return fail(E2TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", ws_bytes, L.total);
  if (((uintptr_t)ws) & 255) return fail(E2TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t es = bf ? 2 : 4;
  const size_t nq = (size_t)d.BH * d.T * d.d_k * es, nv = (size_t)d.BH * d.T * d.d_v * es;
  const size_t ng = (size_t)d.BH * d.T * sizeof(float), ns = (size_t)d.BH * d.S * sizeof(float);
  Range in[] = {{q, nq, "q"}, {k, nq, "k"}, {v, nv, "v"}, {lr, ng, "lr"}, {mom, ng, "mom"},
                {decay, ng, "decay"}, {W0, ns, "W0"}, {M0, ns, "M0"}};
  Range outr[] = {{out, nv, "out"}, {W_end, ns, "W_end"}, {M_end, ns, "M_end"},
                  {saved, SL.total, "saved_states"}, {ws, L.total, "workspace"}};
  if (!check_overlaps(in, 8, outr, 5, &why)) return fail(E2TTT_ERR_INVALID_ARG, "%s", why.c_str());

  cudaStream_t st = (cudaStream_t)stream;
  char* w = (char*)ws;
  float* ca = (float*)(w + L.a);
  float* cb = (float*)(w + L.b);
  float* scal = (float*)(w + L.scal);
  int* status = (int*)(w + L.status);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "status word reset");
  e = launch_chunk_coeffs(lr, mom, decay, ca, cb, scal, d.BH, d.T, d.C, d.NC, d.coef, st);
  if (e != cudaSuccess) return cuda_fail(e, "chunk coefficient kernel");
  if (d.nomom && saved) {
    // no momentum state: the saved M parts hold zeros (the backward reads them)
    const size_t row = (size_t)d.S * sizeof(float);
    e = cudaMemset2DAsync(saved + d.S, 2 * row, 0, row, (size_t)d.NC * d.BH, st);
    if (e != cudaSuccess) return cuda_fail(e, "saved-state reset");
  }
  if (tc) {
    bf16* acts_e = d.save_acts ? (bf16*)((char*)saved + SL.e) : nullptr;
    bf16* acts_dh = d.save_acts ? (bf16*)((char*)saved + SL.dh) : nullptr;
    e = tc_fwd(d, (const bf16*)q, (const bf16*)k, (const bf16*)v, (bf16*)out, ca, cb, scal, W0, M0,
               W_end, M_end, saved, w + L.tc, status, st, acts_e, acts_dh);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core forward");
    return E2TTT_OK;
  }
  float* H = (float*)(w + L.H);
  float* E = (float*)(w + L.E);
  float* dH = (float*)(w + L.dH);
  if (d.nomom) M_end = (float*)(w + L.mscr);  // the CUDA-core path's momentum scratch
  if (bf)
    e = simt_fwd<bf16>(d, (const bf16*)q, (const bf16*)k, (const bf16*)v, (bf16*)out, ca, cb, scal,
                       W0, M0, W_end, M_end, saved, H, E, dH, st);
  else
    e = simt_fwd<float>(d, (const float*)q, (const float*)k, (const float*)v, (float*)out, ca, cb,
                        scal, W0, M0, W_end, M_end, saved, H, E, dH, st);
  if (e != cudaSuccess) return cuda_fail(e, "CUDA-core forward");
  return E2TTT_OK;
}

e2ttt_status e2ttt_chunk_scan_bwd(const e2ttt_shape* s, const void* q, const void* k, const void* v,
                                  const float* lr, const float* mom, const float* decay,
                                  const float* saved, const void* dout, const float* dW_end,
                                  const float* dM_end, void* dq, void* dk, void* dv, float* dlr,
                                  float* dmom, float* ddecay, float* dW0, float* dM0, void* ws,
                                  size_t ws_bytes, void* stream) {
  g_last_error.clear();
  std::string why;
  if (!shape_ok(s, &why)) return fail(E2TTT_ERR_INVALID_ARG, "%s", why.c_str());
  if (!q || !k || !v || !lr || !decay || !saved || !dout || !dq || !dk || !dv || !dlr ||
      !ddecay || !dW0)
    return fail(E2TTT_ERR_INVALID_ARG, "e2ttt_chunk_scan_bwd: NULL pointer argument (only dW_end and dM_end may be NULL)");
  Dims d = make_dims(s);
  if (d.nomom && (mom || dM_end || dmom || dM0))
    return fail(E2TTT_ERR_INVALID_ARG, "no-momentum mode: mom, dM_end, dmom and dM0 must be NULL");
  if (!d.nomom && (!mom || !dmom || !dM0))
    return fail(E2TTT_ERR_INVALID_ARG, "e2ttt_chunk_scan_bwd: mom, dmom and dM0 are required");
  const bool bf = s->act == E2TTT_BF16;
  size_t dm_off = 0;
  size_t need = bwd_total_bytes(d, bf, &dm_off);
  if (!ws) return fail(E2TTT_ERR_INVALID_ARG, "workspace is NULL (needs %zu bytes)", need);
  if (ws_bytes < need) return fail(E2TTT_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  if (((uintptr_t)ws) & 255) return fail(E2TTT_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const size_t es = bf ? 2 : 4;
  const size_t nq = (size_t)d.BH * d.T * d.d_k * es, nv = (size_t)d.BH * d.T * d.d_v * es;
  const size_t ng = (size_t)d.BH * d.T * sizeof(float), ns = (size_t)d.BH * d.S * sizeof(float);
  const SavedLayout SL = saved_layout(d);
  Range in[] = {{q, nq, "q"}, {k, nq, "k"}, {v, nv, "v"}, {lr, ng, "lr"}, {mom, ng, "mom"},
                {decay, ng, "decay"}, {saved, SL.total, "saved_states"},
                {dout, nv, "dout"}, {dW_end, ns, "dW_end"}, {dM_end, ns, "dM_end"}};
  Range outr[] = {{dq, nq, "dq"}, {dk, nq, "dk"}, {dv, nv, "dv"}, {dlr, ng, "dlr"},
                  {dmom, ng, "dmom"}, {ddecay, ng, "ddecay"}, {dW0, ns, "dW0"}, {dM0, ns, "dM0"},
                  {ws, need, "workspace"}};
  if (!check_overlaps(in, 10, outr, 9, &why)) return fail(E2TTT_ERR_INVALID_ARG, "%s", why.c_str());
  if (d.nomom) dM0 = (float*)((char*)ws + dm_off);  // zero momentum adjoint, kept internal
  const bool acts = d.save_acts && d.kind != E2TTT_LINEAR;
  const bf16* acts_e = acts ? (const bf16*)((const char*)saved + SL.e) : nullptr;
  const bf16* acts_dh = acts ? (const bf16*)((const char*)saved + SL.dh) : nullptr;
  BwdArgs A{d, q, k, v, lr, mom, decay, saved, dout, dW_end, dM_end, dq, dk, dv,
            dlr, dmom, ddecay, dW0, dM0, ws, (cudaStream_t)stream, acts_e, acts_dh};
  cudaError_t e = bf ? bwd_run<bf16>(A) : bwd_run<float>(A);
  if (e == cudaErrorNotSupported)
    return fail(E2TTT_ERR_UNSUPPORTED, "backward path not available for this shape");
  if (e != cudaSuccess) return cuda_fail(e, "backward");
  return E2TTT_OK;
}

}  // extern "C"
