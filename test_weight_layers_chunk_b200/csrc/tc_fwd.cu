// tcgen05 tensor-core forward of the chunk scan (bf16 activations, fp32 state).
//
// Per chunk (all heads at once), "Rethinking Expressivity and Efficiency in
// Test-Time Training" (abstract: closed-form chunk transition with chunk-start
// gradients; atlas "Approach": two weighted gradient aggregations; arxivlens
// "Limitations": output at the chunk-start weights), SwiGLU fast weight:
//   G1  H = [Q; K] [W1; W3]^T     epilogue: A = silu(H1) * H3 (bf16, both row
//                                 sets), A_k^T, and silu(H1_k), H3_k silu'(H1_k)
//   G2  Y = A W2^T                epilogue: out = Y_q; E = Y_k - V, and the
//                                 transposed, a- and b-scaled copies of E
//   G3  dA = E W2                 epilogue: dH1 = dA H3 silu'(H1), dH3 = dA
//                                 silu(H1), transposed and a-/b-scaled
//   G4  [dM | dW] = [Da | Db]^T K  and  [Ea | Eb]^T A_k   (two accumulators)
//                                 epilogue: M_end = U M0 - dM, W_end = L W0 + c M0 - dW
//                                 in fp32, plus the bf16 operand copies of W_end
//                                 that the next chunk's GEMMs read.
// Linear fast weight: G1 gives out and the scaled E^T; G4 aggregates E^T K.
// Every GEMM operand is K-major in global memory: the epilogues write the
// transposed operands directly, and the keys are transposed once per call.
#include <cuda.h>

#include "paths.h"
#include "state.cuh"
#include "tc_gemm.cuh"
#include "trace.h"

namespace e2ttt {
namespace {

using tc::EpiCtx;

constexpr int kEpiWarps = 8;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr int HB = 128;  // hidden units per G1 tile (its 256 columns hold h1 then h3)

struct FwdP {
  Dims d;
  int ci, t0, write_shadow;
  const bf16 *q, *k, *v;
  bf16* out;
  const float *ca, *cb, *scal;
  StateIn src;
  StateOut dst;
  bf16 *Wsh13, *W2sh, *W2Tsh;  // bf16 copies of the chunk-start weights (Wsh13 = W for linear)
  bf16 *KT, *A, *AkT, *Sk, *E, *EaT, *EbT, *DaT, *DbT;
};

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void st_row32(bf16* dst, const float (&v)[32]) {
  uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    p[i] = make_uint4(pack2(v[8 * i], v[8 * i + 1]), pack2(v[8 * i + 2], v[8 * i + 3]),
                      pack2(v[8 * i + 4], v[8 * i + 5]), pack2(v[8 * i + 6], v[8 * i + 7]));
}
__device__ __forceinline__ void ld_row32(const bf16* src, float (&v)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u = p[i];
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&w[j]);
      float2 f = __bfloat1622float2(h);
      v[8 * i + 2 * j] = f.x;
      v[8 * i + 2 * j + 1] = f.y;
    }
  }
}
__device__ __forceinline__ void ld_row32_f(const float* src, float (&v)[32]) {
  const float4* p = reinterpret_cast<const float4*>(src);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 f = p[i];
    v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
  }
}
__device__ __forceinline__ void st_row32_f(float* dst, const float (&v)[32]) {
  float4* p = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}
// Row of the interleaved [W1; W3] operand copy that holds row r of W1 (which=0) or W3 (which=1).
__device__ __forceinline__ int w13_row(int r, int which) {
  return (r / HB) * (2 * HB) + which * HB + (r % HB);
}

// ---------------------------------------------------------------- epilogues
// G1, SwiGLU. Class 0 = query rows, class 1 = key rows of the chunk.
struct EpiG1 {
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int t = c.m0 + c.row;
    const int j0 = (c.n0 / (2 * HB)) * HB;
    const int per = HB / c.nparts;
    const size_t arow = ((size_t)c.z * 2 * d.C + (size_t)c.cls * d.C + t) * d.d_h;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      float h1[32], h3[32], u[32];
      c.ld(0, g, h1);
      c.ld(0, HB + g, h3);
      if (c.cls == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = silu_f(h1[i]) * h3[i];
        st_row32(p.A + arow + j0 + g, u);
      } else {
        float s1[32], s2[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sg = sigmoid_f(h1[i]);
          s1[i] = h1[i] * sg;
          s2[i] = h3[i] * sg * (1.0f + h1[i] * (1.0f - sg));
          u[i] = s1[i] * h3[i];
        }
        st_row32(p.A + arow + j0 + g, u);
        const size_t srow = ((size_t)c.z * d.C + t) * 2 * d.d_h;
        st_row32(p.Sk + srow + j0 + g, s1);
        st_row32(p.Sk + srow + d.d_h + j0 + g, s2);
        bf16* akt = p.AkT + ((size_t)c.z * d.d_h + j0 + g) * d.C + t;
#pragma unroll
        for (int i = 0; i < 32; ++i) akt[(size_t)i * d.C] = __float2bfloat16_rn(u[i]);
      }
    }
  }
};

// Key-row epilogue shared by G2 (SwiGLU) and G1 (linear): e = y - v (or -v);
// writes E (if requested) and the a-/b-scaled transposes.
template <int BN>
__device__ __forceinline__ void key_rows_epilogue(const FwdP& p, const EpiCtx<BN>& c, int t, int col0,
                                                  const float (&y)[32], bool write_e) {
  const Dims& d = p.d;
  const size_t tok = (size_t)c.z * d.T + p.t0 + t;
  float vv[32], e[32];
  ld_row32(p.v + tok * d.d_v + col0, vv);
#pragma unroll
  for (int i = 0; i < 32; ++i) e[i] = d.loss == 0 ? y[i] - vv[i] : -vv[i];
  if (write_e) st_row32(p.E + ((size_t)c.z * d.C + t) * d.d_v + col0, e);
  const float at = p.ca[tok], bt = p.cb[tok];
  const size_t o = ((size_t)c.z * d.d_v + col0) * d.C + t;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    p.EaT[o + (size_t)i * d.C] = __float2bfloat16_rn(at * e[i]);
    p.EbT[o + (size_t)i * d.C] = __float2bfloat16_rn(bt * e[i]);
  }
}

// G2, SwiGLU: rows [0, C) are queries (-> out), [C, 2C) keys (-> E).
struct EpiG2 {
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int m = c.m0 + c.row;
    const int per = BN / c.nparts;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      float y[32];
      c.ld(0, g, y);
      const int col = c.n0 + g;
      if (m < d.C) {
        st_row32(p.out + ((size_t)c.z * d.T + p.t0 + m) * d.d_v + col, y);
      } else {
        key_rows_epilogue(p, c, m - d.C, col, y, true);
      }
    }
  }
};

// G1, linear: class 0 = queries (-> out), class 1 = keys (-> scaled E^T).
struct EpiG1Lin {
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int t = c.m0 + c.row;
    const int per = BN / c.nparts;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      float y[32];
      c.ld(0, g, y);
      const int col = c.n0 + g;
      if (c.cls == 0) st_row32(p.out + ((size_t)c.z * d.T + p.t0 + t) * d.d_v + col, y);
      else key_rows_epilogue(p, c, t, col, y, false);
    }
  }
};

// G3, SwiGLU: dA -> dH1, dH3, transposed and scaled by a_t and b_t.
struct EpiG3 {
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int t = c.m0 + c.row;
    const size_t tok = (size_t)c.z * d.T + p.t0 + t;
    const float at = p.ca[tok], bt = p.cb[tok];
    const int per = BN / c.nparts;
    const size_t srow = ((size_t)c.z * d.C + t) * 2 * d.d_h;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      float da[32], s1[32], s2[32];
      c.ld(0, g, da);
      const int j = c.n0 + g;
      ld_row32(p.Sk + srow + j, s1);
      ld_row32(p.Sk + srow + d.d_h + j, s2);
      const size_t o1 = ((size_t)c.z * 2 * d.d_h + j) * d.C + t;
      const size_t o3 = o1 + (size_t)d.d_h * d.C;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float dh1 = da[i] * s2[i], dh3 = da[i] * s1[i];
        p.DaT[o1 + (size_t)i * d.C] = __float2bfloat16_rn(at * dh1);
        p.DbT[o1 + (size_t)i * d.C] = __float2bfloat16_rn(bt * dh1);
        p.DaT[o3 + (size_t)i * d.C] = __float2bfloat16_rn(at * dh3);
        p.DbT[o3 + (size_t)i * d.C] = __float2bfloat16_rn(bt * dh3);
      }
    }
  }
};

// G4: accumulator 0 = dM = sum_t a_t g_t, accumulator 1 = dW = sum_t b_t g_t.
// Class 0 covers rows of [W1; W3] (or W for linear), class 1 the rows of W2.
struct EpiG4 {
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    const Dims& d = p.d;
    const int i = c.m0 + c.row;
    const size_t plane = (size_t)d.BH * d.NC;
    const size_t so = (size_t)c.z * d.NC + p.ci;
    const float PU = p.scal[so], PL = p.scal[plane + so], cc = p.scal[2 * plane + so];
    const bool swiglu = d.kind == 1;
    const int ld = c.cls == 0 ? d.d_k : d.d_h;
    const long long base = c.cls == 0 ? 0 : 2LL * d.d_h * d.d_k;
    const int per = BN / c.nparts;
    for (int g = c.part * per; g < (c.part + 1) * per; g += 32) {
      float dM[32], dW[32], w0[32], m0[32];
      c.ld(0, g, dM);
      c.ld(1, g, dW);
      const int j = c.n0 + g;
      const long long idx = base + (long long)i * ld + j;
      ld_row32_f(p.src.W + c.z * p.src.stride + idx, w0);
      if (p.src.M) ld_row32_f(p.src.M + c.z * p.src.stride + idx, m0);
      else {
#pragma unroll
        for (int q = 0; q < 32; ++q) m0[q] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        const float mn = PU * m0[q] - dM[q];
        const float wn = PL * w0[q] + cc * m0[q] - dW[q];
        dM[q] = mn;
        dW[q] = wn;
      }
      st_row32_f(p.dst.M + c.z * p.dst.stride + idx, dM);
      st_row32_f(p.dst.W + c.z * p.dst.stride + idx, dW);
      if (!p.write_shadow) continue;
      if (c.cls == 0) {
        const int row = swiglu ? w13_row(i % d.d_h, i / d.d_h) : i;
        const int rows = swiglu ? 2 * d.d_h : d.d_v;
        st_row32(p.Wsh13 + ((size_t)c.z * rows + row) * d.d_k + j, dW);
      } else {
        st_row32(p.W2sh + ((size_t)c.z * d.d_v + i) * d.d_h + j, dW);
        bf16* wt = p.W2Tsh + ((size_t)c.z * d.d_h + j) * d.d_v + i;
#pragma unroll
        for (int q = 0; q < 32; ++q) wt[(size_t)q * d.d_v] = __float2bfloat16_rn(dW[q]);
      }
    }
  }
};

template <class Epi>
struct EpiAdapter {
  template <int BN>
  static __device__ __forceinline__ void run(const FwdP& p, const EpiCtx<BN>& c) {
    Epi::template run<BN>(p, c);
  }
};

// ---------------------------------------------------------------- prep kernels
// K [BH, T, d_k] -> per-chunk transposes KT [BH, NC, d_k, C] (32x32 tiles).
__global__ void transpose_keys_kernel(const bf16* __restrict__ k, bf16* __restrict__ KT, int T, int C,
                                      int NC, int d_k) {
  __shared__ bf16 tile[32][33];
  const int z = blockIdx.z;
  const int t0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
  for (int r = threadIdx.y; r < 32; r += 8)
    tile[r][threadIdx.x] = k[((size_t)z * T + t0 + r) * d_k + j0 + threadIdx.x];
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int j = j0 + r, t = t0 + threadIdx.x;
    KT[(((size_t)z * NC + t / C) * d_k + j) * C + (t % C)] = tile[threadIdx.x][r];
  }
}

// bf16 operand copies of the caller's W0.
__global__ void shadow_init_kernel(FwdP p, const float* __restrict__ W0) {
  const Dims& d = p.d;
  const long long total = (long long)d.BH * d.S;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int z = (int)(e / d.S);
    const long long idx = e - (long long)z * d.S;
    const bf16 w = __float2bfloat16_rn(W0[e]);
    if (d.kind == 0) {
      p.Wsh13[e] = w;
      continue;
    }
    const long long n13 = 2LL * d.d_h * d.d_k;
    if (idx < n13) {
      const int i = (int)(idx / d.d_k), j = (int)(idx % d.d_k);
      p.Wsh13[((size_t)z * 2 * d.d_h + w13_row(i % d.d_h, i / d.d_h)) * d.d_k + j] = w;
    } else {
      const long long r2 = idx - n13;
      const int i = (int)(r2 / d.d_h), j = (int)(r2 % d.d_h);
      p.W2sh[((size_t)z * d.d_v + i) * d.d_h + j] = w;
      p.W2Tsh[((size_t)z * d.d_h + j) * d.d_v + i] = w;
    }
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix; box = 64 columns x box_rows rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class Epi> struct EpiName;
template <> struct EpiName<struct EpiG1> { static constexpr const char* v = "tc_g1_h_act"; };
template <> struct EpiName<struct EpiG2> { static constexpr const char* v = "tc_g2_y_out_e"; };
template <> struct EpiName<struct EpiG3> { static constexpr const char* v = "tc_g3_da_dh"; };
template <> struct EpiName<struct EpiG4> { static constexpr const char* v = "tc_g4_aggregate_state"; };
template <> struct EpiName<struct EpiG1Lin> { static constexpr const char* v = "tc_g1_linear_out_e"; };

template <int BN, int NUM_A, int STAGES, class Epi>
cudaError_t launch(const tc::Job& job, const FwdP& p, cudaStream_t st) {
  constexpr size_t smem = tc::smem_bytes<BN, NUM_A, STAGES>();
  auto kern = tc::gemm_kernel<BN, NUM_A, STAGES, kEpiWarps, EpiAdapter<Epi>, FwdP>;
  cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)smem);
  if (attr != cudaSuccess) return attr;
  int tiles = 0;
  for (int c = 0; c < job.n_cls; ++c) tiles += job.cls[c].tiles_m * job.cls[c].tiles_n * job.heads;
  E2TTT_TRACE(EpiName<Epi>::v, st);
  kern<<<tiles, kThreads, smem, st>>>(job, p);
  return cudaGetLastError();
}

// BN = 256 when N allows, else 128 (N is always a multiple of 128 here).
template <int NUM_A, int STAGES256, int STAGES128, class Epi>
cudaError_t launch_bn(bool bn256, const tc::Job& job, const FwdP& p, cudaStream_t st) {
  if (bn256) return launch<256, NUM_A, STAGES256, Epi>(job, p, st);
  return launch<128, NUM_A, STAGES128, Epi>(job, p, st);
}

struct Scratch {
  bf16 *Wsh13, *W2sh, *W2Tsh, *KT, *A, *AkT, *Sk, *E, *EaT, *EbT, *DaT, *DbT;
};

size_t carve(const Dims& d, char* base, Scratch* s) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = (off + bytes + 255) & ~size_t(255);
    return p;
  };
  const size_t e = sizeof(bf16), BH = d.BH;
  Scratch t;
  if (d.kind == 0) {
    t.Wsh13 = (bf16*)take(BH * d.d_v * d.d_k * e);
    t.W2sh = t.W2Tsh = t.A = t.AkT = t.Sk = t.E = t.DaT = t.DbT = nullptr;
  } else {
    t.Wsh13 = (bf16*)take(BH * 2 * d.d_h * d.d_k * e);
    t.W2sh = (bf16*)take(BH * d.d_v * d.d_h * e);
    t.W2Tsh = (bf16*)take(BH * d.d_h * d.d_v * e);
    t.A = (bf16*)take(BH * 2 * d.C * d.d_h * e);
    t.AkT = (bf16*)take(BH * d.d_h * d.C * e);
    t.Sk = (bf16*)take(BH * d.C * 2 * d.d_h * e);
    t.E = (bf16*)take(BH * d.C * d.d_v * e);
    t.DaT = (bf16*)take(BH * 2 * d.d_h * d.C * e);
    t.DbT = (bf16*)take(BH * 2 * d.d_h * d.C * e);
  }
  t.KT = (bf16*)take(BH * d.T * d.d_k * e);
  t.EaT = (bf16*)take(BH * d.d_v * d.C * e);
  t.EbT = (bf16*)take(BH * d.d_v * d.C * e);
  if (s) *s = t;
  return off;
}

}  // namespace

bool tc_fwd_supported(const Dims& d, bool bf16_act) {
  if (!bf16_act) return false;
  if (d.T % d.C != 0 || d.C % 128 != 0) return false;
  if (d.d_k % 128 != 0 || d.d_v % 128 != 0) return false;
  if (d.kind == 1 && d.d_h % 128 != 0) return false;
  return encode_fn() != nullptr;
}

size_t tc_fwd_scratch_bytes(const Dims& d) { return carve(d, nullptr, nullptr); }

cudaError_t tc_fwd(const Dims& d, const bf16* q, const bf16* k, const bf16* v, bf16* out,
                   const float* ca, const float* cb, const float* scal, const float* W0,
                   const float* M0, float* W_end, float* M_end, float* saved, float* stbuf,
                   void* scratch, int* status, cudaStream_t st) {
  Scratch s;
  carve(d, (char*)scratch, &s);
  FwdP p;
  p.d = d;
  p.q = q; p.k = k; p.v = v; p.out = out;
  p.ca = ca; p.cb = cb; p.scal = scal;
  p.Wsh13 = s.Wsh13; p.W2sh = s.W2sh; p.W2Tsh = s.W2Tsh;
  p.KT = s.KT; p.A = s.A; p.AkT = s.AkT; p.Sk = s.Sk; p.E = s.E;
  p.EaT = s.EaT; p.EbT = s.EbT; p.DaT = s.DaT; p.DbT = s.DbT;
  const int BH = d.BH, T = d.T, C = d.C, NC = d.NC, dk = d.d_k, dv = d.d_v, dh = d.d_h;

  cudaError_t e = save_initial_state(d, W0, M0, saved, st);
  if (e != cudaSuccess) return e;
  {
    E2TTT_TRACE("tc_transpose_keys", st);
    transpose_keys_kernel<<<dim3(T / 32, dk / 32, BH), dim3(32, 8), 0, st>>>(k, s.KT, T, C, NC, dk);
  }
  {
    E2TTT_TRACE("tc_shadow_init", st);
    shadow_init_kernel<<<1184, 256, 0, st>>>(p, W0);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // Operand maps (chunk-independent: coordinates carry the chunk offset).
  tc::Job g1{}, g2{}, g3{}, g4{};
  bool ok = true;
  const bool bn_v = dv % 256 == 0, bn_k = dk % 256 == 0, bn_h = dh % 256 == 0;
  for (tc::Job* j : {&g1, &g2, &g3, &g4}) {
    j->heads = BH;
    j->status = status;
  }
  if (d.kind == 1) {
    // G1: classes = query rows, key rows; B = interleaved [W1; W3]
    ok &= make_map(&g1.maps[0].a0, q, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[1].a0, k, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[0].b, s.Wsh13, (uint64_t)BH * 2 * dh, dk, 256);
    g1.maps[1].b = g1.maps[0].b;
    g1.n_cls = 2;
    for (int c = 0; c < 2; ++c) g1.cls[c] = tc::Class{C / 128, 2 * dh / 256, dk / 64, T, 0, 2 * dh, 0};
    // G2: A = [A_q; A_k] (2C rows per head), B = W2 (N = d_v)
    ok &= make_map(&g2.maps[0].a0, s.A, (uint64_t)BH * 2 * C, dh, 128);
    ok &= make_map(&g2.maps[0].b, s.W2sh, (uint64_t)BH * dv, dh, bn_v ? 256 : 128);
    g2.n_cls = 1;
    g2.cls[0] = tc::Class{2 * C / 128, dv / (bn_v ? 256 : 128), dh / 64, 2 * C, 0, dv, 0};
    // G3: A = E, B = W2^T (N = d_h)
    ok &= make_map(&g3.maps[0].a0, s.E, (uint64_t)BH * C, dv, 128);
    ok &= make_map(&g3.maps[0].b, s.W2Tsh, (uint64_t)BH * dh, dv, bn_h ? 256 : 128);
    g3.n_cls = 1;
    g3.cls[0] = tc::Class{C / 128, dh / (bn_h ? 256 : 128), dv / 64, C, 0, dh, 0};
    // G4: class 0 = [W1; W3] rows (A = Da/Db, B = K^T), class 1 = W2 rows (A = Ea/Eb, B = A_k^T)
    const bool bn4 = bn_k && bn_h;
    const uint32_t b4 = bn4 ? 256 : 128;
    ok &= make_map(&g4.maps[0].a0, s.DaT, (uint64_t)BH * 2 * dh, C, 128);
    ok &= make_map(&g4.maps[0].a1, s.DbT, (uint64_t)BH * 2 * dh, C, 128);
    ok &= make_map(&g4.maps[0].b, s.KT, (uint64_t)BH * NC * dk, C, b4);
    ok &= make_map(&g4.maps[1].a0, s.EaT, (uint64_t)BH * dv, C, 128);
    ok &= make_map(&g4.maps[1].a1, s.EbT, (uint64_t)BH * dv, C, 128);
    ok &= make_map(&g4.maps[1].b, s.AkT, (uint64_t)BH * dh, C, b4);
    g4.n_cls = 2;
    g4.cls[0] = tc::Class{2 * dh / 128, dk / (int)b4, C / 64, 2 * dh, 0, NC * dk, 0};
    g4.cls[1] = tc::Class{dv / 128, dh / (int)b4, C / 64, dv, 0, dh, 0};
  } else {
    ok &= make_map(&g1.maps[0].a0, q, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[1].a0, k, (uint64_t)BH * T, dk, 128);
    ok &= make_map(&g1.maps[0].b, s.Wsh13, (uint64_t)BH * dv, dk, bn_v ? 256 : 128);
    g1.maps[1].b = g1.maps[0].b;
    g1.n_cls = 2;
    for (int c = 0; c < 2; ++c) g1.cls[c] = tc::Class{C / 128, dv / (bn_v ? 256 : 128), dk / 64, T, 0, dv, 0};
    ok &= make_map(&g4.maps[0].a0, s.EaT, (uint64_t)BH * dv, C, 128);
    ok &= make_map(&g4.maps[0].a1, s.EbT, (uint64_t)BH * dv, C, 128);
    ok &= make_map(&g4.maps[0].b, s.KT, (uint64_t)BH * NC * dk, C, bn_k ? 256 : 128);
    g4.n_cls = 1;
    g4.cls[0] = tc::Class{dv / 128, dk / (bn_k ? 256 : 128), C / 64, dv, 0, NC * dk, 0};
  }
  if (!ok) return cudaErrorInvalidValue;

  for (int ci = 0; ci < NC; ++ci) {
    p.ci = ci;
    p.t0 = ci * C;
    p.write_shadow = ci + 1 < NC;
    chunk_states(d, ci, W0, M0, W_end, M_end, saved, stbuf, &p.src, &p.dst);
    for (int c = 0; c < g1.n_cls; ++c) g1.cls[c].a_row_base = ci * C;
    for (int c = 0; c < g4.n_cls; ++c)
      if (c == 0) g4.cls[c].b_row_base = ci * dk;
    if (d.kind == 1) {
      e = launch<256, 1, 2, EpiG1>(g1, p, st);
      if (e == cudaSuccess) e = launch_bn<1, 2, 3, EpiG2>(bn_v, g2, p, st);
      if (e == cudaSuccess) e = launch_bn<1, 2, 3, EpiG3>(bn_h, g3, p, st);
      if (e == cudaSuccess) e = launch_bn<2, 3, 2, EpiG4>(bn_k && bn_h, g4, p, st);
    } else {
      e = launch_bn<1, 2, 3, EpiG1Lin>(bn_v, g1, p, st);
      if (e == cudaSuccess) e = launch_bn<2, 3, 2, EpiG4>(bn_k, g4, p, st);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace e2ttt
