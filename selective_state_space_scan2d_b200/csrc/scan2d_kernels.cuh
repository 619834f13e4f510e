// scan2d_kernels.cuh -- sm_100a kernel of the 2D selective-scan forward (2DMamba).
//
// What is computed ("2DMamba 精读：从小白到博士", section 四.5 (1) and (2)):
//   Abar = exp(delta*A[d,n]),  Bbar = delta*B[n],
//   hh[i,j] = Abar[i,j]*hh[i,j-1] + Bbar[i,j]*x[i,j]      (horizontal, hh[i,-1] = 0)
//   h[i,j]  = Abar[i,j]*h[i-1,j]  + hh[i,j]               (vertical,   h[-1,j]  = 0)
//   y[i,j]  = sum_n C[n,i,j]*h[n,i,j] + Dskip[d]*x[i,j]
// The N states never leave the chip: they are reduced against C in registers and only y
// is written (papernotes "关键设计": O(L) memory traffic instead of O(N L)).
//
// Work mapping (designed for the B200 SM, not a translation of SegmentedBlockScan):
//   * The scan is bound by the SFU (one ex2 per (position, state, channel)) and, close
//     behind, by how many values shared memory can hand to the lanes (32 lane-words per
//     clock).  A lane therefore owns an outer-product block of G channels x NG states:
//     per position it reads G values of x and delta and NG values of B and C and does
//     G*NG updates, and the G = 2 channels pair up into packed f32x2 FMAs.
//   * lane = (channel group cg = lane>>2) x (state group q = lane&3); lane q holds states
//     n = q, q+4, q+8, ...; a warp covers 8*G channels and a strip of CMAX columns.
//   * A warp walks all rows of its strip in scan order.  The vertical state of every
//     (column, channel, state) it owns stays in registers for the whole walk, so the
//     vertical scan needs no communication.
//   * The horizontal scan crosses strips.  Inside a block the warps of one chain run
//     skewed by one row (warp w is on row tau-w at step tau) and hand over the carry
//     through shared memory; between the blocks of a chain the carry goes through a ring
//     in global memory with release/acquire flags.  Blocks take (chain, segment) from a
//     ticket counter, so a block only waits on blocks that started before it, and every
//     wait is bounded in time.
//   * Each warp stages the row tiles of its strip (x, delta for its channels, B, C for all
//     states) into a private shared-memory ring, by TMA (cp.async.bulk.tensor, mbarrier
//     completion) when the strides allow, else by plain loads prefetched one row ahead.
//   * The per-lane partial outputs are reduced over the 4 state-group lanes with a
//     reduce-scatter, so each lane stores a contiguous run of one channel's columns.
//   * Orientations: scan position (r, s) is stored position (flipH ? H-1-r : r,
//     flipW ? W-1-s : s).  Strips are fixed in stored columns; a W-reversed orientation
//     walks the strips and the columns inside them backwards.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/scan2d.h"

namespace scan2d {

constexpr int kQ = 4;                  // state-group lanes per channel group
constexpr int kGroups = 8;             // channel groups per warp
constexpr int kRing = 16;              // carry rows buffered between blocks
constexpr int kMaxWarps = 8;           // warps per block
constexpr int kDepth = 3;              // rows staged ahead per warp (TMA path)
constexpr float kLog2e = 1.4426950408889634f;

enum Mode : int {
  kSingle = 0,       // one orientation: y = acc + D x
  kSmemMulti = 1,    // every orientation inside the block, fp32 partial sums in shared memory
  kGlobalFirst = 2,  // first of several launches: yacc = acc + D x
  kGlobalMid = 3,    // yacc += acc
  kGlobalLast = 4,   // y = yacc + acc
};

struct Params {
  const void* x;
  const void* delta;
  const float* A;
  const void* B;
  const void* C;
  const float* Dskip;
  void* y;
  float* yacc;              // fp32 accumulator of the kGlobal* modes (may equal y)
  int batch, channels, H, W, N, K;
  int n_cgroups;            // ceil(channels / channels-per-warp)
  int n_chains;             // batch * n_cgroups
  int strips;               // ceil(W / CMAX)
  int wpc;                  // warps (strips) per chain inside one block
  int chains_per_block;     // > 1 only when nseg == 1
  int nseg;                 // blocks per chain
  int orient_count;         // orientations handled by this launch
  int orient_code[4];       // orientation number (bit0 = flip W, bit1 = flip H)
  int orient_k[4];          // index of the orientation's B_k, C_k
  int mode;
  int yacc_stride;          // kSmemMulti: floats per channel in shared memory
  int vec_store;            // rows of y are aligned for 4-column vector stores
  int out_f32;              // y is fp32 (else bf16)
  unsigned long long* ctrl;   // [0] ticket counter, [1] finished blocks, [2] aborted generation
  unsigned long long* flags;  // [n_chains*nseg] rows published by a segment (tagged)
  unsigned long long* acks;   // [n_chains*nseg] rows consumed by a segment (tagged)
  float* carry;               // [n_chains*nseg][kRing][32][G*NG]
  unsigned long long gen;     // launch generation, tags flags and acks
  long long timeout_ns;
};

struct TmaMaps {
  CUtensorMap x, d, b, c;     // (W, H, channels, batch) and (W, H, N, batch*K)
};

// First device-side error of the device (0 = none); read and cleared by the host.  This
// header is compiled into exactly one translation unit, which owns the definition.
__device__ int g_device_error = 0;

// ---- small device helpers --------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(unsigned long long* p, unsigned long long v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ long long global_ns() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ unsigned long long tag(unsigned long long gen, int v) {
  return (gen << 32) | static_cast<unsigned>(v);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Records a device error once and marks this launch generation aborted (every other wait
// of the launch then gives up at once).
__device__ __noinline__ void report_timeout(unsigned long long* ctrl, unsigned long long gen) {
  atomicCAS(&g_device_error, 0, SCAN2D_E_TIMEOUT);
  if (ctrl != nullptr) st_release(&ctrl[2], gen);
}

// Bounded wait (one lane) until *p >= want.  False on time-out or when the launch is aborted.
__device__ __noinline__ bool wait_geq(const unsigned long long* p, unsigned long long want,
                                      unsigned long long* ctrl, unsigned long long gen,
                                      long long timeout_ns) {
  long long t0 = 0;
  for (unsigned it = 0;; ++it) {
    if (ld_acquire(p) >= want) return true;
    if ((it & 31u) == 0u) {
      if (ld_acquire(&ctrl[2]) == gen) return false;
      const long long now = global_ns();
      if (it == 0u) t0 = now;
      if (now - t0 > timeout_ns || it > (1u << 30)) {
        report_timeout(ctrl, gen);
        return false;
      }
    }
    __nanosleep(64);
  }
}

// Bounded wait for phase `parity` of a TMA mbarrier.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned long long* ctrl,
                                       unsigned long long gen, long long timeout_ns) {
  long long t0 = 0;
  for (unsigned it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0u) {
      const long long now = global_ns();
      if (it == 0u) t0 = now;
      if (now - t0 > timeout_ns || it > (1u << 28)) {
        report_timeout(ctrl, gen);
        return false;
      }
    }
  }
}

// ---- G-wide vectors: G = 2 channels per lane pair into packed f32x2 instructions --------
template <int G> struct VecT;
template <> struct VecT<1> { using T = float; };
template <> struct VecT<2> { using T = float2; };

__device__ __forceinline__ float vmul(float a, float b) { return a * b; }
__device__ __forceinline__ float vfma(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ float vex2(float a) { return ex2_approx(a); }
__device__ __forceinline__ float vget(float a, int) { return a; }

__device__ __forceinline__ float2 vmul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 vfma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 vex2(float2 a) { return make_float2(ex2_approx(a.x), ex2_approx(a.y)); }
__device__ __forceinline__ float vget(float2 a, int c) { return c == 0 ? a.x : a.y; }

template <int G> __device__ __forceinline__ typename VecT<G>::T vsplat(float a);
template <> __device__ __forceinline__ float vsplat<1>(float a) { return a; }
template <> __device__ __forceinline__ float2 vsplat<2>(float a) { return make_float2(a, a); }

template <int G> __device__ __forceinline__ typename VecT<G>::T vmake(const float* a);
template <> __device__ __forceinline__ float vmake<1>(const float* a) { return a[0]; }
template <> __device__ __forceinline__ float2 vmake<2>(const float* a) { return make_float2(a[0], a[1]); }

// ---- staged-row element access ------------------------------------------------------------
// A 16-byte vector holds 4 fp32 or 8 bf16 values of consecutive columns.
template <typename Tin> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerVec = 4;
  static __device__ __forceinline__ float get(const uint4& v, int j) {
    const unsigned w = j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
    return __uint_as_float(w);
  }
};
template <> struct Elem<uint16_t> {
  static constexpr int kPerVec = 8;
  static __device__ __forceinline__ float get(const uint4& v, int j) {
    const unsigned w = (j >> 1) == 0 ? v.x : ((j >> 1) == 1 ? v.y : ((j >> 1) == 2 ? v.z : v.w));
    return __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
  }
};

__device__ __forceinline__ uint16_t load_raw(const uint16_t* p) {
  return __ldg(reinterpret_cast<const unsigned short*>(p));
}
__device__ __forceinline__ float load_raw(const float* p) { return __ldg(p); }

__device__ __forceinline__ void store_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_f(uint16_t* p, float v) {
  *reinterpret_cast<unsigned short*>(p) = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
__device__ __forceinline__ void store4(float* p, const float* v) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(uint16_t* p, const float* v) {
  const unsigned lo = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v[0]))) |
                      (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v[1]))) << 16);
  const unsigned hi = static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2]))) |
                      (static_cast<unsigned>(__bfloat16_as_ushort(__float2bfloat16_rn(v[3]))) << 16);
  *reinterpret_cast<uint2*>(p) = make_uint2(lo, hi);
}

// y element idx <- v, in the output type of the call
__device__ __forceinline__ void store_out(void* y, size_t idx, float v, bool f32) {
  if (f32) store_f(static_cast<float*>(y) + idx, v);
  else store_f(static_cast<uint16_t*>(y) + idx, v);
}
__device__ __forceinline__ void store_out4(void* y, size_t idx, const float* v, bool f32) {
  if (f32) store4(static_cast<float*>(y) + idx, v);
  else store4(static_cast<uint16_t*>(y) + idx, v);
}

// ---- shared-memory tile of one strip row ------------------------------------------------------
template <typename Tin, int NG, int G, int CMAX>
struct Layout {
  static constexpr int ESZ = static_cast<int>(sizeof(Tin));
  static constexpr int CPW = kGroups * G;                    // channels per warp
  static constexpr int NB = kQ * NG;                         // states covered by the 4 q lanes
  static constexpr int X_BYTES = CPW * CMAX * ESZ;           // [CPW][CMAX]
  static constexpr int B_BYTES = NB * CMAX * ESZ;            // [NB][CMAX]
  static constexpr int r128(int v) { return (v + 127) / 128 * 128; }
  // every region starts on a 128-byte boundary (TMA destination alignment)
  static constexpr int X_OFF = 0;                                        // element offsets
  static constexpr int D_OFF = r128(X_BYTES) / ESZ;
  static constexpr int B_OFF = D_OFF + r128(X_BYTES) / ESZ;
  static constexpr int C_OFF = B_OFF + r128(B_BYTES) / ESZ;
  static constexpr int BYTES = (C_OFF * ESZ) + r128(B_BYTES);
  static constexpr int TX_BYTES = 2 * X_BYTES + 2 * B_BYTES;
  static constexpr int DENSE = (2 * CPW + 2 * NB) * CMAX;    // tile values without padding
  static constexpr int E = CMAX * G;                         // partial outputs per lane per row
  static constexpr int PLAIN_PER_LANE = DENSE / 32;          // plain-load path: values per lane
};

// ---- the kernel ------------------------------------------------------------------------------
template <typename Tin, int NG, int G, int CMAX, bool TMA>
__global__ void __launch_bounds__(kMaxWarps * 32)
scan2d_kernel(const __grid_constant__ Params p, const __grid_constant__ TmaMaps tm) {
  using L = Layout<Tin, NG, G, CMAX>;
  using V = typename VecT<G>::T;
  constexpr int PV = Elem<Tin>::kPerVec;
  static_assert(CMAX % PV == 0, "strip width must hold whole 16-byte vectors");
  static_assert(L::E % 4 == 0, "reduce-scatter needs 4 | CMAX*G");
  static_assert(L::DENSE % 32 == 0, "plain-load path needs 32 | tile values");
  constexpr int DEPTH = TMA ? kDepth : 1;
  constexpr int NVEC = CMAX / PV;                            // 16-byte vectors per strip row
  constexpr int E = L::E;

  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t s_bar[kMaxWarps][kDepth];
  __shared__ int s_item;

  const unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int slot = warp / p.wpc;            // chain slot inside the block
  const int w = warp - slot * p.wpc;        // strip inside the segment
  const int cg = lane >> 2;                 // channel group
  const int q = lane & 3;                   // state group

  // ---- which chain and segment -------------------------------------------------------
  int chain, seg;
  if (p.nseg > 1) {
    if (threadIdx.x == 0) s_item = static_cast<int>(atomicAdd(&p.ctrl[0], 1ull));
    __syncthreads();
    chain = s_item / p.nseg;
    seg = s_item - chain * p.nseg;
  } else {
    chain = blockIdx.x * p.chains_per_block + slot;
    seg = 0;
  }
  const bool chain_ok = chain < p.n_chains && slot < p.chains_per_block;
  const int b = chain_ok ? chain / p.n_cgroups : 0;
  const int grp = chain_ok ? chain - b * p.n_cgroups : 0;
  const int u_scan = seg * p.wpc + w;                        // strip position in scan order
  const bool strip_ok = chain_ok && u_scan < p.strips;       // warp-uniform

  const int H = p.H, W = p.W, N = p.N;
  const size_t HW = static_cast<size_t>(H) * W;
  const int ch0 = grp * L::CPW + cg * G;                     // first channel of this lane

  // per-lane constants: A * log2(e) per (channel, state), Dskip per channel
  V A2[NG];
  V Dd;
  {
    float dd[G];
#pragma unroll
    for (int c = 0; c < G; ++c) {
      const int d = ch0 + c;
      dd[c] = (chain_ok && d < p.channels && p.Dskip != nullptr) ? __ldg(p.Dskip + d) : 0.f;
    }
    Dd = vmake<G>(dd);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float a[G];
      const int n = q + kQ * g;
#pragma unroll
      for (int c = 0; c < G; ++c) {
        const int d = ch0 + c;
        a[c] = (chain_ok && d < p.channels && n < N) ? __ldg(p.A + static_cast<size_t>(d) * N + n) * kLog2e : 0.f;
      }
      A2[g] = vmake<G>(a);
    }
  }

  // ---- shared memory: carries | staged rows | output accumulator ----------------------------
  const int carry_floats = p.wpc > 1 ? 2 * kMaxWarps * 32 * G * NG : 0;
  float* carry_s = reinterpret_cast<float*>(smem);
  unsigned char* slots = smem + carry_floats * sizeof(float) + warp * DEPTH * L::BYTES;
  float* yacc_s = reinterpret_cast<float*>(smem + carry_floats * sizeof(float) +
                                           (p.wpc * p.chains_per_block) * DEPTH * L::BYTES);

  if (TMA) {
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < DEPTH; ++s) mbar_init(&s_bar[warp][s], 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  __syncthreads();

  const int item = chain * p.nseg + seg;
  const bool consumer = (w == 0) && seg > 0;
  const bool producer = (w == p.wpc - 1) && seg < p.nseg - 1;
  const int U = p.orient_count * H;                          // rows this warp walks

  // row u of the walk -> (orientation index, stored row, stored strip)
  auto row_coords = [&](int uu, int& oi, int& i, int& t) {
    oi = uu / H;
    const int r = uu - oi * H;
    const int o = p.orient_code[oi];
    i = (o & 2) ? H - 1 - r : r;
    t = (o & 1) ? p.strips - 1 - u_scan : u_scan;
  };

  auto issue_tma = [&](int uu) {
    int oi, i, t;
    row_coords(uu, oi, i, t);
    const int k = p.orient_k[oi];
    const int s = uu % DEPTH;
    unsigned char* dst = slots + s * L::BYTES;
    uint64_t* bar = &s_bar[warp][s];
    mbar_expect_tx(bar, L::TX_BYTES);
    tma_load_4d(dst + L::X_OFF * L::ESZ, &tm.x, bar, t * CMAX, i, grp * L::CPW, b);
    tma_load_4d(dst + L::D_OFF * L::ESZ, &tm.d, bar, t * CMAX, i, grp * L::CPW, b);
    tma_load_4d(dst + L::B_OFF * L::ESZ, &tm.b, bar, t * CMAX, i, 0, b * p.K + k);
    tma_load_4d(dst + L::C_OFF * L::ESZ, &tm.c, bar, t * CMAX, i, 0, b * p.K + k);
  };

  // plain-load path: this lane's share of row u's tile, zero outside the tensors.  Value
  // e of the dense tile goes to tile offset plain_dst(e).
  auto plain_split = [&](int e, int& region, int& rr, int& cc) {
    if (e < 2 * L::CPW * CMAX) {
      region = e / (L::CPW * CMAX);
      rr = (e - region * L::CPW * CMAX) / CMAX;
    } else {
      const int f = e - 2 * L::CPW * CMAX;
      region = 2 + f / (L::NB * CMAX);
      rr = (f - (region - 2) * L::NB * CMAX) / CMAX;
    }
    cc = e % CMAX;
  };
  auto plain_dst = [&](int e) {
    int region, rr, cc;
    plain_split(e, region, rr, cc);
    const int off = region == 0 ? L::X_OFF : (region == 1 ? L::D_OFF : (region == 2 ? L::B_OFF : L::C_OFF));
    return off + rr * CMAX + cc;
  };
  Tin pre[L::PLAIN_PER_LANE];
  auto plain_load = [&](int uu) {
    int oi, i, t;
    row_coords(uu, oi, i, t);
    const int k = p.orient_k[oi];
#pragma unroll
    for (int m = 0; m < L::PLAIN_PER_LANE; ++m) {
      int region, rr, cc;
      plain_split(lane + 32 * m, region, rr, cc);
      const int col = t * CMAX + cc;
      Tin val = Tin(0);
      if (col < W) {
        if (region < 2) {
          const int d = grp * L::CPW + rr;
          if (d < p.channels) {
            const Tin* src = static_cast<const Tin*>(region == 0 ? p.x : p.delta);
            val = load_raw(src + (static_cast<size_t>(b) * p.channels + d) * HW + static_cast<size_t>(i) * W + col);
          }
        } else if (rr < N) {
          const Tin* src = static_cast<const Tin*>(region == 2 ? p.B : p.C);
          val = load_raw(src + ((static_cast<size_t>(b) * p.K + k) * N + rr) * HW + static_cast<size_t>(i) * W + col);
        }
      }
      pre[m] = val;
    }
  };

  if (strip_ok) {
    if (TMA) {
      if (lane == 0)
        for (int uu = 0; uu < DEPTH && uu < U; ++uu) issue_tma(uu);
    } else {
      plain_load(0);
    }
  }

  int u = 0;                                                 // rows of the walk done so far
  for (int oi = 0; oi < p.orient_count; ++oi) {
    const int o = p.orient_code[oi];
    const bool flipW = (o & 1) != 0, flipH = (o & 2) != 0;
    const int t = flipW ? p.strips - 1 - u_scan : u_scan;   // stored strip
    const int col0 = t * CMAX;
    const bool add_dx = (p.mode == kSingle || p.mode == kGlobalFirst || (p.mode == kSmemMulti && oi == 0));

    V v[CMAX][NG];
#pragma unroll
    for (int j = 0; j < CMAX; ++j)
#pragma unroll
      for (int g = 0; g < NG; ++g) v[j][g] = vsplat<G>(0.f);

    const int steps = H + p.wpc - 1;
    for (int tau = 0; tau < steps; ++tau) {
      const int r = tau - w;
      const bool active = strip_ok && r >= 0 && r < H;      // warp-uniform
      if (active) {
        const int i = flipH ? H - 1 - r : r;
        const int s = u % DEPTH;
        const Tin* tile = reinterpret_cast<const Tin*>(slots + s * L::BYTES);

        // ---- (1) this row's tile is in shared memory -----------------------------------
        if (TMA) {
          mbar_wait(&s_bar[warp][s], static_cast<unsigned>((u / DEPTH) & 1), p.ctrl, p.gen, p.timeout_ns);
        } else {
          Tin* dst = reinterpret_cast<Tin*>(slots);
#pragma unroll
          for (int m = 0; m < L::PLAIN_PER_LANE; ++m) dst[plain_dst(lane + 32 * m)] = pre[m];
          __syncwarp();
          if (u + 1 < U) plain_load(u + 1);
        }

        // ---- (2) carry-in: hh at the column before this strip (scan order) ----------------
        V hh[NG];
        if (w > 0) {
          const float* src = carry_s + (((tau - 1) & 1) * kMaxWarps + (warp - 1)) * 32 * G * NG + lane * G * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[g] = vmake<G>(src + g * G);
        } else if (consumer) {
          const unsigned long long want = tag(p.gen, r + 1);
          if (lane == 0) wait_geq(&p.flags[item - 1], want, p.ctrl, p.gen, p.timeout_ns);
          __syncwarp();
          const bool ok = ld_acquire(&p.flags[item - 1]) >= want;   // every lane acquires
          const float* src = p.carry + ((static_cast<size_t>(item - 1) * kRing + (r % kRing)) * 32 + lane) * G * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            float tmp[G];
#pragma unroll
            for (int c = 0; c < G; ++c) tmp[c] = ok ? __ldcg(src + g * G + c) : 0.f;
            hh[g] = vmake<G>(tmp);
          }
        } else {
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[g] = vsplat<G>(0.f);
        }

        // ---- (3) the strip's columns of this row ------------------------------------------
        // per lane: G channels (x, delta) and NG states (B, C) of every column, 16-byte vectors
        V acc[CMAX];
        auto column = [&](int j, const uint4* xv, const uint4* dv, const uint4* bv, const uint4* cv, int jv) {
          float xs[G], ds[G];
#pragma unroll
          for (int c = 0; c < G; ++c) {
            xs[c] = Elem<Tin>::get(xv[c], jv);
            ds[c] = Elem<Tin>::get(dv[c], jv);
          }
          const V x2 = vmake<G>(xs);
          const V d2 = vmake<G>(ds);
          const V dx = vmul(d2, x2);
          V a_acc = (add_dx && q == 0) ? vmul(Dd, x2) : vsplat<G>(0.f);
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            const V a = vex2(vmul(d2, A2[g]));
            const V uu = vmul(dx, vsplat<G>(Elem<Tin>::get(bv[g], jv)));
            hh[g] = vfma(a, hh[g], uu);
            v[j][g] = vfma(a, v[j][g], hh[g]);
            a_acc = vfma(vsplat<G>(Elem<Tin>::get(cv[g], jv)), v[j][g], a_acc);
          }
          acc[j] = a_acc;
        };
        auto vector_group = [&](int vg, bool rev) {
          uint4 xv[G], dv[G], bv[NG], cv[NG];
#pragma unroll
          for (int c = 0; c < G; ++c) {
            xv[c] = *reinterpret_cast<const uint4*>(tile + L::X_OFF + (cg * G + c) * CMAX + vg * PV);
            dv[c] = *reinterpret_cast<const uint4*>(tile + L::D_OFF + (cg * G + c) * CMAX + vg * PV);
          }
#pragma unroll
          for (int g = 0; g < NG; ++g) {
            bv[g] = *reinterpret_cast<const uint4*>(tile + L::B_OFF + (q + kQ * g) * CMAX + vg * PV);
            cv[g] = *reinterpret_cast<const uint4*>(tile + L::C_OFF + (q + kQ * g) * CMAX + vg * PV);
          }
          if (!rev) {
#pragma unroll
            for (int jv = 0; jv < PV; ++jv) column(vg * PV + jv, xv, dv, bv, cv, jv);
          } else {
#pragma unroll
            for (int jv = PV - 1; jv >= 0; --jv) column(vg * PV + jv, xv, dv, bv, cv, jv);
          }
        };
        if (!flipW) {
#pragma unroll
          for (int vg = 0; vg < NVEC; ++vg) vector_group(vg, false);
        } else {
#pragma unroll
          for (int vg = NVEC - 1; vg >= 0; --vg) vector_group(vg, true);
        }

        // ---- (4) the tile slot is free again: stage row u + DEPTH into it ---------------------
        __syncwarp();
        if (TMA && lane == 0 && u + DEPTH < U) {
          fence_proxy_async();
          issue_tma(u + DEPTH);
        }

        // ---- (5) carry-out --------------------------------------------------------------------
        if (w < p.wpc - 1) {
          float* dst = carry_s + ((tau & 1) * kMaxWarps + warp) * 32 * G * NG + lane * G * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int c = 0; c < G; ++c) dst[g * G + c] = vget(hh[g], c);
        } else if (producer) {
          if (r >= kRing) {
            const unsigned long long want = tag(p.gen, r - kRing + 1);
            if (lane == 0) wait_geq(&p.acks[item + 1], want, p.ctrl, p.gen, p.timeout_ns);
            __syncwarp();
            (void)ld_acquire(&p.acks[item + 1]);           // orders this lane's ring writes
          }
          float* dst = p.carry + ((static_cast<size_t>(item) * kRing + (r % kRing)) * 32 + lane) * G * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g)
#pragma unroll
            for (int c = 0; c < G; ++c) __stcg(dst + g * G + c, vget(hh[g], c));
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release(&p.flags[item], tag(p.gen, r + 1));
        }
        if (consumer) st_release(&p.acks[item], tag(p.gen, r + 1));   // every lane: its loads are done

        // ---- (6) reduce over the 4 state groups; lane q keeps the q-th quarter ------------------
        // flat index e = c*CMAX + j (channel-major)
        float flat[E];
#pragma unroll
        for (int c = 0; c < G; ++c)
#pragma unroll
          for (int j = 0; j < CMAX; ++j) flat[c * CMAX + j] = vget(acc[j], c);
        float r1[E / 2];
        const bool hi2 = (q & 2) != 0, hi1 = (q & 1) != 0;
#pragma unroll
        for (int e = 0; e < E / 2; ++e) {
          const float lo = flat[e], hi = flat[e + E / 2];
          r1[e] = (hi2 ? hi : lo) + __shfl_xor_sync(FULL, hi2 ? lo : hi, 2);
        }
        float own[E / 4];
#pragma unroll
        for (int e = 0; e < E / 4; ++e) {
          const float lo = r1[e], hi = r1[e + E / 4];
          own[e] = (hi1 ? hi : lo) + __shfl_xor_sync(FULL, hi1 ? lo : hi, 1);
        }

        // ---- (7) output: channel c, columns j0 .. j0 + E/4 - 1 of the strip --------------------
        {
          const int e0 = q * (E / 4);
          const int c = e0 / CMAX;
          const int j0 = e0 - c * CMAX;
          const int d = ch0 + c;
          if (chain_ok && d < p.channels) {
            const size_t rowoff = (static_cast<size_t>(b) * p.channels + d) * HW + static_cast<size_t>(i) * W;
            const int gc = col0 + j0;
            if (p.mode == kSingle) {
              if ((E / 4) % 4 == 0 && p.vec_store && gc + E / 4 <= W) {
#pragma unroll
                for (int m = 0; m < E / 4; m += 4) store_out4(p.y, rowoff + gc + m, own + m, p.out_f32);
              } else {
#pragma unroll
                for (int m = 0; m < E / 4; ++m)
                  if (gc + m < W) store_out(p.y, rowoff + gc + m, own[m], p.out_f32);
              }
            } else if (p.mode == kSmemMulti) {
              float* a = yacc_s + (slot * L::CPW + cg * G + c) * p.yacc_stride + i * W + gc;
#pragma unroll
              for (int m = 0; m < E / 4; ++m)
                if (gc + m < W) a[m] = (oi == 0) ? own[m] : a[m] + own[m];
            } else {
#pragma unroll
              for (int m = 0; m < E / 4; ++m) {
                if (gc + m >= W) continue;
                const size_t idx = rowoff + gc + m;
                if (p.mode == kGlobalFirst) p.yacc[idx] = own[m];
                else if (p.mode == kGlobalMid) p.yacc[idx] += own[m];
                else store_out(p.y, idx, p.yacc[idx] + own[m], p.out_f32);
              }
            }
          }
        }
        ++u;
      }
      __syncthreads();
    }
  }

  // ---- kSmemMulti: write the accumulated maps of this block's chains --------------------------
  if (p.mode == kSmemMulti && chain_ok) {
    const int nthreads = p.wpc * 32;
    const int tid = w * 32 + lane;
    for (int cs = 0; cs < L::CPW; ++cs) {
      const int dd = grp * L::CPW + cs;
      if (dd >= p.channels) break;
      const float* src = yacc_s + (slot * L::CPW + cs) * p.yacc_stride;
      const size_t base = (static_cast<size_t>(b) * p.channels + dd) * HW;
      for (size_t e = tid; e < HW; e += nthreads) store_out(p.y, base + e, src[e], p.out_f32);
    }
  }

  // ---- the last block of a ticketed launch resets the counters for the next launch ----------
  if (p.nseg > 1) {
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned long long done = atomicAdd(&p.ctrl[1], 1ull);
      if (done == gridDim.x - 1) {
        p.ctrl[0] = 0ull;
        p.ctrl[1] = 0ull;
        __threadfence();
      }
    }
  }
}

}  // namespace scan2d
