// scan2d_kernels.cuh -- sm_100a kernels of the 2D selective-scan forward (2DMamba).
//
// What is computed ("2DMamba 精读：从小白到博士", section 四.5 (1) and (2)):
//   Abar = exp(delta*A[d,n]),  Bbar = delta*B[n],
//   hh[i,j] = Abar[i,j]*hh[i,j-1] + Bbar[i,j]*x[i,j]      (horizontal, hh[i,-1] = 0)
//   h[i,j]  = Abar[i,j]*h[i-1,j]  + hh[i,j]               (vertical,   h[-1,j]  = 0)
//   y[i,j]  = sum_n C[n,i,j]*h[n,i,j] + Dskip[d]*x[i,j]
// The N states never leave the chip: they are reduced against C in registers and only y
// is written (papernotes "关键设计": O(L) memory traffic instead of O(N L)).
//
// Work mapping (a B200 design, not the pages' SegmentedBlockScan):
//   * lane = (channel slot cl in 0..7) x (state group q in 0..3).  A lane owns NG states
//     n = q*NG .. q*NG+NG-1 of one channel.  B and C are shared by all channels, so the
//     8 channel slots of a warp read the same B/C addresses (broadcast loads).
//   * a warp owns a strip of up to CMAX consecutive columns (in scan order) and walks the
//     rows top to bottom in scan order; the vertical state h of every (column, state) it
//     owns stays in registers for the whole walk, so the vertical scan is sequential and
//     free of communication.
//   * the horizontal scan crosses strips: the row's last hh of strip w is the carry-in of
//     strip w+1.  Inside a block the warps of a chain run skewed by one row (warp w works
//     on row tau-w at step tau) and hand the carry over through shared memory; between
//     blocks of a chain the carry goes through a global ring buffer with release/acquire
//     flags.  Blocks take their (chain, segment) from a ticket counter, so a block only
//     ever waits on blocks that started earlier.  Every wait is bounded in time.
//   * the per-lane partial sums over its NG states are reduced across the 4 state-group
//     lanes with a reduce-scatter (each lane ends up owning every 4th column of the strip).
//   * orientations: a scan position (r, s) maps to the stored position
//     (flipH ? H-1-r : r, flipW ? W-1-s : s); everything else is orientation-blind.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/scan2d.h"

namespace scan2d {

constexpr int kStateLanes = 4;                         // lanes sharing one channel
constexpr int kChanPerWarp = 32 / kStateLanes;         // channels per warp
constexpr int kRing = 16;                              // carry rows buffered between blocks
constexpr int kMaxWarps = 8;                           // warps per block
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
  int n_cgroups;            // ceil(channels / kChanPerWarp)
  int n_chains;             // batch * n_cgroups
  int cols_per_warp;        // columns of a full strip (<= CMAX)
  int wpc;                  // warps (strips) per chain inside one block
  int chains_per_block;     // > 1 only when nseg == 1
  int nseg;                 // blocks per chain
  int orient_count;         // orientations handled by this launch
  int orient_code[4];       // orientation number (bit0 = flip W, bit1 = flip H)
  int orient_k[4];          // index of the orientation's B_k, C_k
  int mode;
  int yacc_stride;          // kSmemMulti: floats per channel slot in shared memory
  unsigned long long* ctrl;   // [0] ticket counter, [1] finished blocks, [2] aborted generation
  unsigned long long* flags;  // [n_chains*nseg] rows published by a segment (tagged)
  unsigned long long* acks;   // [n_chains*nseg] rows consumed by a segment (tagged)
  float* carry;               // [n_chains*nseg][kRing][32][NG]
  unsigned long long gen;     // launch generation, tags flags and acks
  long long timeout_ns;
};

// First device-side error of the device (0 = none); read and cleared by the host.  This
// header is compiled into exactly one translation unit, which owns the definition.
__device__ int g_device_error = 0;

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

template <typename T> __device__ __forceinline__ float load_f(const T* p);
template <> __device__ __forceinline__ float load_f<float>(const float* p) { return __ldg(p); }
template <> __device__ __forceinline__ float load_f<uint16_t>(const uint16_t* p) {
  return __uint_as_float(static_cast<unsigned>(__ldg(reinterpret_cast<const unsigned short*>(p))) << 16);
}

__device__ __forceinline__ void store_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_f(uint16_t* p, float v) {
  *reinterpret_cast<unsigned short*>(p) = __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

__device__ __forceinline__ unsigned long long tag(unsigned long long gen, int v) {
  return (gen << 32) | static_cast<unsigned>(v);
}

// Bounded wait (one lane): until *p >= want.  On time-out records SCAN2D_E_TIMEOUT, marks
// this launch generation as aborted (so every other block stops waiting at once) and
// returns false.  Returns false immediately once the launch is marked aborted.
__device__ __noinline__ bool wait_geq(const unsigned long long* p, unsigned long long want,
                                      unsigned long long* ctrl, unsigned long long gen,
                                      long long timeout_ns) {
  long long t0 = 0;
  for (unsigned it = 0;; ++it) {
    if (ld_acquire(p) >= want) return true;
    if ((it & 31u) == 0u) {
      if (ld_acquire(&ctrl[2]) == gen) return false;   // another block gave up
      const long long now = global_ns();
      if (it == 0u) t0 = now;
      if (now - t0 > timeout_ns || it > (1u << 30)) {
        atomicCAS(&g_device_error, 0, SCAN2D_E_TIMEOUT);
        st_release(&ctrl[2], gen);
        return false;
      }
    }
    __nanosleep(64);
  }
}

template <typename Tin, typename Tout, int NG, int CMAX>
__global__ void __launch_bounds__(kMaxWarps * 32)
scan2d_strip_kernel(const Params p) {
  static_assert(CMAX % 4 == 0, "strip width must be a multiple of the state-group count");
  extern __shared__ float smem[];
  __shared__ int s_item;

  const unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int slot = warp / p.wpc;            // chain slot inside the block
  const int w = warp - slot * p.wpc;        // strip inside the segment
  const int cl = lane >> 2;                 // channel slot
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
  const int d = grp * kChanPerWarp + cl;
  const bool ch_ok = chain_ok && d < p.channels;
  const int d_ld = ch_ok ? d : 0;

  const int H = p.H, W = p.W, N = p.N;
  const size_t HW = static_cast<size_t>(H) * W;
  const int seg_cols = p.wpc * p.cols_per_warp;
  const int s_begin = seg * seg_cols + w * p.cols_per_warp;
  const int c = chain_ok ? max(0, min(p.cols_per_warp, W - s_begin)) : 0;   // warp-uniform

  const Tin* __restrict__ xg = static_cast<const Tin*>(p.x) + (static_cast<size_t>(b) * p.channels + d_ld) * HW;
  const Tin* __restrict__ dg = static_cast<const Tin*>(p.delta) + (static_cast<size_t>(b) * p.channels + d_ld) * HW;
  const float Dd = (ch_ok && p.Dskip != nullptr) ? __ldg(p.Dskip + d_ld) : 0.f;

  float A2[NG];
  int n_ld[NG];
  bool n_ok[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = q * NG + g;
    n_ok[g] = n < N;
    n_ld[g] = n_ok[g] ? n : 0;
    A2[g] = (ch_ok && n_ok[g]) ? __ldg(p.A + static_cast<size_t>(d_ld) * N + n_ld[g]) * kLog2e : 0.f;
  }

  float* carry_s = smem;                                        // [2][kMaxWarps][32][NG]
  float* yacc_s = smem + (p.wpc > 1 ? 2 * kMaxWarps * 32 * NG : 0);
  const int item = chain * p.nseg + seg;
  const bool consumer = (w == 0) && seg > 0;
  const bool producer = (w == p.wpc - 1) && seg < p.nseg - 1;

  for (int oi = 0; oi < p.orient_count; ++oi) {
    const int o = p.orient_code[oi];
    const int k = p.orient_k[oi];
    const bool flipW = o & 1, flipH = (o >> 1) & 1;
    const int j0 = flipW ? W - 1 - s_begin : s_begin;
    const int dj = flipW ? -1 : 1;
    const bool add_dx = (p.mode == kSingle || p.mode == kGlobalFirst || (p.mode == kSmemMulti && oi == 0));

    const Tin* Bg[NG];
    const Tin* Cg[NG];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const size_t off = ((static_cast<size_t>(b) * p.K + k) * N + n_ld[g]) * HW;
      Bg[g] = static_cast<const Tin*>(p.B) + off;
      Cg[g] = static_cast<const Tin*>(p.C) + off;
    }

    float v[CMAX][NG];
#pragma unroll
    for (int jj = 0; jj < CMAX; ++jj)
#pragma unroll
      for (int g = 0; g < NG; ++g) v[jj][g] = 0.f;

    const int steps = H + p.wpc - 1;
    for (int tau = 0; tau < steps; ++tau) {
      const int r = tau - w;
      const bool active = c > 0 && r >= 0 && r < H;                // warp-uniform
      if (active) {
        const int i = flipH ? H - 1 - r : r;
        const int row = i * W + j0;

        // ---- carry-in: hh at the column left of this strip (scan order) -------------
        float hh[NG];
        if (w > 0) {
          const float* src = carry_s + (((tau - 1) & 1) * kMaxWarps + (warp - 1)) * 32 * NG + lane * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[g] = src[g];
        } else if (consumer) {
          bool ok = true;
          if (lane == 0) ok = wait_geq(&p.flags[item - 1], tag(p.gen, r + 1), p.ctrl, p.gen, p.timeout_ns);
          ok = __shfl_sync(FULL, ok, 0);
          const float* src = p.carry + ((static_cast<size_t>(item - 1) * kRing + (r % kRing)) * 32 + lane) * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[g] = ok ? __ldcg(src + g) : 0.f;
        } else {
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[g] = 0.f;
        }

        // ---- the strip's columns of this row ------------------------------------------
        float acc[CMAX];
#pragma unroll
        for (int jj = 0; jj < CMAX; ++jj) {
          acc[jj] = 0.f;
          if (jj < c) {
            const int pos = row + dj * jj;
            const float xv = load_f<Tin>(xg + pos);
            const float dv = load_f<Tin>(dg + pos);
            const float dx = dv * xv;
            if (add_dx && q == 0) acc[jj] = Dd * xv;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              const float a = ex2_approx(dv * A2[g]);
              const float bv = n_ok[g] ? load_f<Tin>(Bg[g] + pos) : 0.f;
              const float cv = n_ok[g] ? load_f<Tin>(Cg[g] + pos) : 0.f;
              hh[g] = fmaf(a, hh[g], dx * bv);
              v[jj][g] = fmaf(a, v[jj][g], hh[g]);
              acc[jj] = fmaf(cv, v[jj][g], acc[jj]);
            }
          }
        }

        // ---- carry-out ------------------------------------------------------------------
        if (w < p.wpc - 1) {
          float* dst = carry_s + ((tau & 1) * kMaxWarps + warp) * 32 * NG + lane * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g) dst[g] = hh[g];
        } else if (producer) {
          bool ok = true;
          if (lane == 0 && r >= kRing) ok = wait_geq(&p.acks[item + 1], tag(p.gen, r - kRing + 1), p.ctrl, p.gen, p.timeout_ns);
          ok = __shfl_sync(FULL, ok, 0);
          float* dst = p.carry + ((static_cast<size_t>(item) * kRing + (r % kRing)) * 32 + lane) * NG;
#pragma unroll
          for (int g = 0; g < NG; ++g) __stcg(dst + g, hh[g]);
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release(&p.flags[item], tag(p.gen, r + 1));
          (void)ok;
        }
        if (consumer) {
          // the carry of row r has been consumed (its loads fed this row's arithmetic)
          __syncwarp();
          if (lane == 0) st_release(&p.acks[item], tag(p.gen, r + 1));
        }

        // ---- reduce over the 4 state groups: lane q keeps columns 4m+q ----------------
        float r1[CMAX / 2];
        const bool hi2 = (q & 2) != 0, hi1 = (q & 1) != 0;
#pragma unroll
        for (int m = 0; m < CMAX / 4; ++m)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float lo = acc[4 * m + e], hi = acc[4 * m + e + 2];
            const float send = hi2 ? lo : hi;
            r1[2 * m + e] = (hi2 ? hi : lo) + __shfl_xor_sync(FULL, send, 2);
          }
        float own[CMAX / 4];
#pragma unroll
        for (int m = 0; m < CMAX / 4; ++m) {
          const float send = hi1 ? r1[2 * m] : r1[2 * m + 1];
          own[m] = (hi1 ? r1[2 * m + 1] : r1[2 * m]) + __shfl_xor_sync(FULL, send, 1);
        }

        // ---- output ---------------------------------------------------------------------
        if (ch_ok) {
          const size_t mapoff = (static_cast<size_t>(b) * p.channels + d) * HW;
#pragma unroll
          for (int m = 0; m < CMAX / 4; ++m) {
            const int jj = 4 * m + q;
            if (jj < c) {
              const int pos = row + dj * jj;
              switch (p.mode) {
                case kSingle:
                  store_f(static_cast<Tout*>(p.y) + mapoff + pos, own[m]);
                  break;
                case kSmemMulti: {
                  float* a = yacc_s + (slot * kChanPerWarp + cl) * p.yacc_stride + pos;
                  *a = (oi == 0) ? own[m] : *a + own[m];
                  break;
                }
                case kGlobalFirst:
                  p.yacc[mapoff + pos] = own[m];
                  break;
                case kGlobalMid:
                  p.yacc[mapoff + pos] += own[m];
                  break;
                default:  // kGlobalLast
                  store_f(static_cast<Tout*>(p.y) + mapoff + pos, p.yacc[mapoff + pos] + own[m]);
                  break;
              }
            }
          }
        }
      }
      __syncthreads();
    }
  }

  // ---- kSmemMulti: write the accumulated maps of this block's chains -------------------
  if (p.mode == kSmemMulti) {
    const int nthreads = p.wpc * 32;
    const int t = w * 32 + lane;
    if (chain_ok) {
      for (int cs = 0; cs < kChanPerWarp; ++cs) {
        const int dd = grp * kChanPerWarp + cs;
        if (dd >= p.channels) break;
        const float* src = yacc_s + (slot * kChanPerWarp + cs) * p.yacc_stride;
        Tout* dst = static_cast<Tout*>(p.y) + (static_cast<size_t>(b) * p.channels + dd) * HW;
        for (size_t e = t; e < HW; e += nthreads) store_f(dst + e, src[e]);
      }
    }
  }

  // ---- the last block of a ticketed launch resets the counters for the next launch -------
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
