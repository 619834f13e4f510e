// scan2d_proj.cu -- the input-dependent scan parameters, computed from x in one pass.
//
// The pages say the selective parameters are set by the current input ("2DMamba 精读：从小白到
// 博士", section 四.4: A_t and B_t are modulated by x_t; papernotes.org notes, "方法详解 /
// 关键设计": the 2D scan extends Mamba's 1D selective scan).  The projection itself is not
// printed there; the plainest reading is Mamba's: per position p, with the channels of x[p]
// contracted against two small weight matrices,
//   u[p]     = Wx · x[p]                          (R + 2N values: dt part, B, C)
//   B[n, p]  = u[R + n],   C[n, p] = u[R + N + n]
//   delta[d, p] = softplus(Wdt[d, :] · u[0:R] + bdt[d])
// written straight into the layouts scan2d_fwd reads (delta like x, B and C as (batch, N, H, W)).
//
// Roofline (fp32, D = 128, R = 8, N = 16): per position 128 x 40 + 8 x 128 = 6144 FMAs and
// 128 softplus against 512 B of x read and 512 + 128 B written; 12 FMA per byte, which B200's
// FP32 lanes (37 T FMA/s) and HBM (6.5 TB/s) serve in about the same time.  A tensor-core GEMM
// would not shorten it, so the contraction runs on the FP32 pipes with packed f32x2 FMAs:
// a thread owns two adjacent positions, the weights sit in shared memory (transposed so that
// one 16-byte load feeds four outputs) and every global access is a coalesced run of positions.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/scan2d.h"

namespace {

constexpr int kThreads = 128;
constexpr int kPos = 2;                  // positions per thread
constexpr int kNB = 16;                  // B and C rows reserved in u (N <= 16)

struct ProjArgs {
  const void* x;
  const float* Wx;       // (R + 2N, D)
  const float* Wdt;      // (D, R)
  const float* bdt;      // (D)
  void* delta;
  void* B;
  void* C;
  int batch, D, HW, N, R;
  int pairs;             // HW even and buffers aligned: a thread's two positions move as one access
};

__device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld(const uint16_t* p) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(p))) << 16);
}
__device__ __forceinline__ void st(float* p, float v) { *p = v; }
__device__ __forceinline__ void st(uint16_t* p, float v) { *p = __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

// two adjacent positions in one access (8 bytes fp32, 4 bytes bf16)
__device__ __forceinline__ float2 ld2(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
__device__ __forceinline__ float2 ld2(const uint16_t* p) {
  const unsigned v = __ldg(reinterpret_cast<const unsigned*>(p));
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ void st2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void st2(uint16_t* p, float2 v) {
  const unsigned lo = __bfloat16_as_ushort(__float2bfloat16_rn(v.x));
  const unsigned hi = __bfloat16_as_ushort(__float2bfloat16_rn(v.y));
  *reinterpret_cast<unsigned*>(p) = lo | (hi << 16);
}

template <typename T>
__device__ __forceinline__ void put(T* p, float2 v, bool ok1, bool pairs) {
  if (pairs && ok1) {
    st2(p, v);
  } else {
    st(p, v.x);
    if (ok1) st(p + 1, v.y);
  }
}

__device__ __forceinline__ float softplus(float z) { return z > 20.f ? z : log1pf(expf(z)); }

// RP: dt rows of u padded to a multiple of 4; u has RP + 2*kNB rows, the unused ones with zero
// weights.  Shared memory: WxT [D][RP + 2*kNB], then Wdt [D][RP], then bdt [D].
template <typename T, int RP>
__global__ void __launch_bounds__(kThreads) k_proj(const ProjArgs a) {
  constexpr int NU = RP + 2 * kNB;
  extern __shared__ __align__(16) float sm[];
  float* wxt = sm;
  float* wdt = sm + (size_t)a.D * NU;
  float* bdt = wdt + (size_t)a.D * RP;
  for (int e = threadIdx.x; e < a.D * NU; e += kThreads) {
    const int c = e / NU, j = e % NU;          // u row j, channel c
    int row = -1;
    if (j < RP) row = j < a.R ? j : -1;
    else if (j < RP + kNB) row = (j - RP) < a.N ? a.R + (j - RP) : -1;
    else row = (j - RP - kNB) < a.N ? a.R + a.N + (j - RP - kNB) : -1;
    wxt[e] = row >= 0 ? a.Wx[(size_t)row * a.D + c] : 0.f;
  }
  for (int e = threadIdx.x; e < a.D * RP; e += kThreads) {
    const int d = e / RP, r = e % RP;
    wdt[e] = r < a.R ? a.Wdt[(size_t)d * a.R + r] : 0.f;
  }
  for (int e = threadIdx.x; e < a.D; e += kThreads) bdt[e] = a.bdt[e];
  __syncthreads();

  const long long tiles_per_map = ((long long)a.HW + kThreads * kPos - 1) / (kThreads * kPos);
  const int b = static_cast<int>(blockIdx.x / tiles_per_map);
  const long long p0 = (blockIdx.x % tiles_per_map) * (kThreads * kPos) + (long long)threadIdx.x * kPos;
  if (p0 >= a.HW) return;
  const bool ok1 = p0 + 1 < a.HW;
  const bool pairs = a.pairs && ok1;
  const T* x = static_cast<const T*>(a.x) + (size_t)b * a.D * a.HW + p0;

  float2 u[NU];
#pragma unroll
  for (int j = 0; j < NU; ++j) u[j] = make_float2(0.f, 0.f);
  // kBatch channels of x are loaded before any is used, so their loads are in flight together
  // (fp32 gains from 8; the bf16 rows, half the bytes, measured faster with 2)
  constexpr int kBatch = sizeof(T) == 4 ? 8 : 2;
  for (int c0 = 0; c0 < a.D; c0 += kBatch) {
    float2 xv[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const T* xc = x + (size_t)(c0 + k) * a.HW;
      const bool okc = c0 + k < a.D;
      if (pairs) xv[k] = okc ? ld2(xc) : make_float2(0.f, 0.f);
      else xv[k] = make_float2(okc ? ld(xc) : 0.f, (okc && ok1) ? ld(xc + 1) : 0.f);
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (c0 + k >= a.D) break;
      const float4* w = reinterpret_cast<const float4*>(wxt + (size_t)(c0 + k) * NU);
#pragma unroll
      for (int j4 = 0; j4 < NU / 4; ++j4) {
        const float4 wv = w[j4];
        u[4 * j4 + 0] = __ffma2_rn(make_float2(wv.x, wv.x), xv[k], u[4 * j4 + 0]);
        u[4 * j4 + 1] = __ffma2_rn(make_float2(wv.y, wv.y), xv[k], u[4 * j4 + 1]);
        u[4 * j4 + 2] = __ffma2_rn(make_float2(wv.z, wv.z), xv[k], u[4 * j4 + 2]);
        u[4 * j4 + 3] = __ffma2_rn(make_float2(wv.w, wv.w), xv[k], u[4 * j4 + 3]);
      }
    }
  }
  // B and C
  T* Bo = static_cast<T*>(a.B) + (size_t)b * a.N * a.HW + p0;
  T* Co = static_cast<T*>(a.C) + (size_t)b * a.N * a.HW + p0;
#pragma unroll
  for (int n = 0; n < kNB; ++n) {
    if (n < a.N) {
      put(Bo + (size_t)n * a.HW, u[RP + n], ok1, pairs);
      put(Co + (size_t)n * a.HW, u[RP + kNB + n], ok1, pairs);
    }
  }
  // delta = softplus(Wdt u_dt + bdt)
  T* Do = static_cast<T*>(a.delta) + (size_t)b * a.D * a.HW + p0;
#pragma unroll 2
  for (int d = 0; d < a.D; ++d) {
    const float bd = bdt[d];
    float2 z = make_float2(bd, bd);
    const float4* w = reinterpret_cast<const float4*>(wdt + (size_t)d * RP);
#pragma unroll
    for (int r4 = 0; r4 < RP / 4; ++r4) {
      const float4 wv = w[r4];
      z = __ffma2_rn(make_float2(wv.x, wv.x), u[4 * r4 + 0], z);
      z = __ffma2_rn(make_float2(wv.y, wv.y), u[4 * r4 + 1], z);
      z = __ffma2_rn(make_float2(wv.z, wv.z), u[4 * r4 + 2], z);
      z = __ffma2_rn(make_float2(wv.w, wv.w), u[4 * r4 + 3], z);
    }
    put(Do + (size_t)d * a.HW, make_float2(softplus(z.x), ok1 ? softplus(z.y) : 0.f), ok1, pairs);
  }
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// an sm_100 device is current (the library is built for it alone)
int device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_DEVICE;
  }
  return major == 10 ? SCAN2D_OK : SCAN2D_E_DEVICE;
}

template <typename T, int RP>
int launch(const ProjArgs& a, cudaStream_t st) {
  constexpr int NU = RP + 2 * kNB;
  const size_t smem = ((size_t)a.D * NU + (size_t)a.D * RP + a.D) * sizeof(float);
  if (smem > 227 * 1024) return SCAN2D_E_DIMS;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(k_proj<T, RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  const long long tiles = ((long long)a.HW + kThreads * kPos - 1) / (kThreads * kPos);
  const long long blocks = tiles * a.batch;
  if (blocks > 0x7fffffffLL) return SCAN2D_E_DIMS;
  k_proj<T, RP><<<static_cast<unsigned>(blocks), kThreads, smem, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? SCAN2D_OK : SCAN2D_E_LAUNCH;
}

template <typename T>
int launch_r(const ProjArgs& a, cudaStream_t st) {
  if (a.R <= 8) return launch<T, 8>(a, st);
  if (a.R <= 16) return launch<T, 16>(a, st);
  return launch<T, 32>(a, st);
}

}  // namespace

extern "C" {

int scan2d_proj(const void* x, const float* Wx, const float* Wdt, const float* bdt, void* delta, void* B,
                void* C, int batch, int channels, int H, int W, int N, int R, unsigned flags, void* stream) {
  if (flags & ~SCAN2D_BF16) return SCAN2D_E_FLAGS;
  if (batch < 1 || channels < 1 || H < 1 || W < 1 || R < 1 || R > SCAN2D_PROJ_MAX_R) return SCAN2D_E_DIMS;
  if (N < 1 || N > kNB) return SCAN2D_E_N;
  const unsigned long long hw = static_cast<unsigned long long>(H) * W;
  if (hw > (1ull << 31) - 1 || hw * channels * batch > (1ull << 40)) return SCAN2D_E_DIMS;
  if (!x || !Wx || !Wdt || !bdt || !delta || !B || !C) return SCAN2D_E_NULL;
  const size_t el = (flags & SCAN2D_BF16) ? 2 : 4;
  if (!aligned(x, el) || !aligned(delta, el) || !aligned(B, el) || !aligned(C, el) || !aligned(Wx, 4) ||
      !aligned(Wdt, 4) || !aligned(bdt, 4))
    return SCAN2D_E_ALIGN;
  const bool pairs = hw % 2 == 0 && aligned(x, 2 * el) && aligned(delta, 2 * el) && aligned(B, 2 * el) &&
                     aligned(C, 2 * el);
  if (const int rc = device_ok()) return rc;
  ProjArgs a{x, Wx, Wdt, bdt, delta, B, C, batch, channels, static_cast<int>(hw), N, R, pairs ? 1 : 0};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return el == 2 ? launch_r<uint16_t>(a, st) : launch_r<float>(a, st);
}

}  // extern "C"
