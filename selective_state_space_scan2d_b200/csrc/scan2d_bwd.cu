// scan2d_bwd.cu -- sm_100a kernels and C entry points of the gradients of the 2D selective scan.
//
// The pages on 2DMamba describe the forward only ("2DMamba 精读：从小白到博士", section 四.5:
// (1) horizontal scan, (2) vertical scan and output).  The backward here is the chain-rule
// adjoint of those two recurrences.  For one map (b, d), one state n and one orientation, with
// p - e1 the previous position of the horizontal scan and p - e2 that of the vertical scan:
//   forward   a = exp(delta*A),  u = delta*B*x,
//             hh[p] = a*hh[p-e1] + u,   h[p] = a*h[p-e2] + hh[p],   y[p] += C*h[p]
//   adjoint   gh[p]  = C*dy + a[p+e2]*gh[p+e2]         (vertical, run backwards)
//             ghh[p] = gh[p] + a[p+e1]*ghh[p+e1]       (horizontal, run backwards)
//             dL/da = gh*h[p-e2] + ghh*hh[p-e1],   dL/du = ghh
// from which dx += ghh*delta*B, ddelta += dL/da*a*A + ghh*B*x, dA += dL/da*a*delta,
// dB += ghh*delta*x and dC += dy*h (both summed over the channels that share B and C),
// dDskip += dy*x and dx += Dskip*dy.
//
// Design.  The adjoint runs against the forward's direction in both dimensions, and needs the
// forward's vertical state h of the row before each row.  The forward keeps that state in
// registers and never stores it, so the backward first recomputes it and stores it (N floats
// per element, one orientation at a time, strip-major: the 8 columns x N states x 8 channels of
// one warp's row are one contiguous 4 KB block).  No kernel here waits on another warp:
//   1. k_pre    walks each strip's rows backwards, carrying the adjoint's vertical state in
//               registers.  For every (row, strip, channel, state) it writes what the strip
//               adds to the two horizontal carries when it starts from zero (forward: the hh
//               leaving the strip; adjoint: a*ghh leaving it) and the product of a across the
//               strip: a carry that enters the strip leaves it multiplied by that product.
//   2. k_carry  runs the two short recurrences across the strips of every row and writes the
//               carry that enters each strip.
//   3. k_states walks each strip's rows forwards from the known carries and stores h.
//   4. k_main   walks each strip's rows backwards from the known carries, with h of the row
//               before read back, and produces every gradient.
// With the vertical-first order the forward's first scan needs no carry and the adjoint's
// horizontal scan reads only C*dy, so k_states_vf (rows forwards) stores vv and writes both
// chains' strip terms, then k_carry and k_main as above: three kernels.
// A warp owns a strip of 8 columns and 8 channels; lane = (channel cg = lane>>2) x (state group
// q = lane&3), lane q holding states q, q+4, q+8, q+12.  Per-element gradients are summed over
// a channel's 4 lanes with a shuffle reduce-scatter; dB and dC over the warp's 8 channels, then
// added with vector atomics (other warps hold the other channels).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/scan2d.h"

namespace {

constexpr int kCols = 8;        // columns per warp strip
constexpr int kCh = 8;          // channels per warp
constexpr int kWarps = 8;       // warps per block
constexpr int kMaxNBwd = 16;    // states per channel supported by the backward
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

struct Args {
  const void* x;
  const void* delta;
  const float* A;
  const void* B;
  const void* C;
  const float* Dskip;
  const void* dy;
  void* dx;                 // per-element gradients, element type of y
  void* ddelta;
  float* accx;              // fp32 sums over orientations (equal to dx / ddelta when those are fp32)
  float* accd;
  float* dA;
  float* dB;
  float* dC;
  float* dDskip;            // may be null
  float* hsave;             // (batch, H, S, channels, N, 8): forward vertical state of one
                            // orientation, strip-major so that a warp's row is contiguous
  float* tf;                // (batch, H, S, channels, N): forward horizontal carry terms
  float* tb;                //   adjoint horizontal carry terms
  float* beta;              //   product of a across the strip
  float* cf;                //   forward carry entering the strip
  float* cb;                //   adjoint carry entering the strip
  long long tasks;          // warps: batch * S * channel groups
  int batch, channels, H, W, N, K, S, ncg;
  int k;                    // orientation index: B_k, C_k, dB_k, dC_k
  int flipH;
  int first, last;          // first / last orientation of the call
  int vec2;                 // W even and outputs aligned: 2-column stores and atomics
};

__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// One of the lane's 8 columns (held as 4 pairs), chosen by two lane bits (keeps the register
// arrays static): column (m2 ? 4 : 0) + (m1 ? 2 : 0) + e.
__device__ __forceinline__ float pick(const float2 (&v)[4], bool m2, bool m1, int e) {
  const float lo = m1 ? (e ? v[1].y : v[1].x) : (e ? v[0].y : v[0].x);
  const float hi = m1 ? (e ? v[3].y : v[3].x) : (e ? v[2].y : v[2].x);
  return m2 ? hi : lo;
}

struct Task {
  int b, s, cgi, d, q, j0;
  bool act;
};

// Warps of one block take adjacent channel groups of one strip (strips_first = false: they
// share B and C rows and write adjacent blocks of the workspace), or adjacent strips of one
// channel group (strips_first = true: warps running together add dB and dC at different
// places).
__device__ __forceinline__ bool decode(const Args& p, Task& t, bool strips_first = false) {
  const long long task = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (task >= p.tasks) return false;
  const int lane = threadIdx.x & 31;
  if (strips_first) {
    t.s = static_cast<int>(task % p.S);
    const long long rest = task / p.S;
    t.cgi = static_cast<int>(rest % p.ncg);
    t.b = static_cast<int>(rest / p.ncg);
  } else {
    t.cgi = static_cast<int>(task % p.ncg);
    const long long rest = task / p.ncg;
    t.s = static_cast<int>(rest % p.S);
    t.b = static_cast<int>(rest / p.S);
  }
  t.d = t.cgi * kCh + (lane >> 2);
  t.q = lane & 3;
  t.j0 = t.s * kCols;
  t.act = t.d < p.channels;
  return true;
}

// scan-order row ii of this orientation -> stored row
__device__ __forceinline__ int row_of(const Args& p, int ii) { return p.flipH ? p.H - 1 - ii : ii; }

// index of (b, row i, strip s, channel d, state n) in the strip-carry arrays; channels are
// padded to whole groups of 8, so a warp's 8 x N values start on a 32-byte boundary
__device__ __forceinline__ size_t carry_idx(const Args& p, int b, int d, int i, int s, int n) {
  return ((((size_t)b * p.H + i) * p.S + s) * (size_t)(p.ncg * kCh) + d) * p.N + n;
}

// first float of the 8 columns of (b, row i, strip s, channel d, state n) in hsave
__device__ __forceinline__ size_t hs_idx(const Args& p, int b, int d, int i, int s, int n) {
  return carry_idx(p, b, d, i, s, n) * kCols;
}

__device__ __forceinline__ void lds8(const float* src, float (&v)[kCols]) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kPairs = kCols / 2;

// 8 floats from shared memory as 4 column pairs
__device__ __forceinline__ void lds8x2(const float* src, float2 (&v)[kPairs]) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  v[0] = make_float2(a.x, a.y); v[1] = make_float2(a.z, a.w);
  v[2] = make_float2(b.x, b.y); v[3] = make_float2(b.z, b.w);
}

__device__ __forceinline__ float lo_hi(const float2 (&v)[kPairs], int c) { return (c & 1) ? v[c >> 1].y : v[c >> 1].x; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// ---- per-warp row staging -------------------------------------------------------------------------
// Each warp stages the rows it walks into two shared-memory buffers, one row ahead:
//   * the inputs (x, delta, dy of its 8 channels, B and C of all states, 8 columns each) are
//     loaded into registers while the current row is computed and stored to shared memory
//     (as fp32) after it, element by element, so any alignment works;
//   * the workspace blocks (strip carries, saved states: contiguous and 32-byte aligned by
//     construction) are copied with cp.async.
// Buffer layout, in floats:
constexpr int kOffX = 0;                                  // [8 channels][8 columns]
constexpr int kOffD = kOffX + kCh * kCols;                // delta
constexpr int kOffB = kOffD + kCh * kCols;                // [N states][8 columns]
constexpr int kOffC = kOffB + kMaxNBwd * kCols;
constexpr int kOffG = kOffC + kMaxNBwd * kCols;           // dy [8 channels][8 columns]
constexpr int kOffCF = kOffG + kCh * kCols;               // forward carries [8 channels * N]
constexpr int kOffCB = kOffCF + kCh * kMaxNBwd;           // adjoint carries
constexpr int kOffH = kOffCB + kCh * kMaxNBwd;            // saved states [8 channels * N][8 columns]
constexpr int kBufPre = kOffCF;                           // floats per buffer: k_pre
constexpr int kBufStates = kOffCB;                        //   k_states
constexpr int kBufMain = kOffH + kCh * kMaxNBwd * kCols;  //   k_main

template <typename Tin, typename Tg, int NG, bool WITH_C, bool WITH_G>
struct InputPrefetch {
  Tin x[2], dl[2];
  Tg gy[2];
  Tin bv[NG], cv[NG];
  size_t xo[2], bo[NG];        // element offsets without the row term
  bool xok[2], bok[NG];

  __device__ __forceinline__ void init(const Args& p, const Task& t, int lane) {
    const size_t HW = (size_t)p.H * p.W;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = lane + 32 * k, ch = e >> 3, col = e & 7;
      const int d = t.cgi * kCh + ch, j = t.j0 + col;
      xok[k] = d < p.channels && j < p.W;
      xo[k] = xok[k] ? ((size_t)t.b * p.channels + d) * HW + j : 0;
    }
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      const int e = lane + 32 * k, n = e >> 3, col = e & 7;
      const int j = t.j0 + col;
      bok[k] = n < p.N && j < p.W;
      bo[k] = bok[k] ? (((size_t)t.b * p.K + p.k) * p.N + n) * HW + j : 0;
    }
  }
  __device__ __forceinline__ void load(const Args& p, int i) {
    const size_t r = (size_t)i * p.W;
    const Tin* X = static_cast<const Tin*>(p.x);
    const Tin* Dl = static_cast<const Tin*>(p.delta);
    const Tg* G = static_cast<const Tg*>(p.dy);
    const Tin* Bm = static_cast<const Tin*>(p.B);
    const Tin* Cm = static_cast<const Tin*>(p.C);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      x[k] = xok[k] ? __ldg(X + xo[k] + r) : Tin(0);
      dl[k] = xok[k] ? __ldg(Dl + xo[k] + r) : Tin(0);
      if (WITH_G) gy[k] = xok[k] ? __ldg(G + xo[k] + r) : Tg(0);
    }
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      bv[k] = bok[k] ? __ldg(Bm + bo[k] + r) : Tin(0);
      if (WITH_C) cv[k] = bok[k] ? __ldg(Cm + bo[k] + r) : Tin(0);
    }
  }
  __device__ __forceinline__ void store(float* buf, int lane) const {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      buf[kOffX + lane + 32 * k] = to_f(x[k]);
      buf[kOffD + lane + 32 * k] = to_f(dl[k]);
      if (WITH_G) buf[kOffG + lane + 32 * k] = to_f(gy[k]);
    }
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      buf[kOffB + lane + 32 * k] = to_f(bv[k]);
      if (WITH_C) buf[kOffC + lane + 32 * k] = to_f(cv[k]);
    }
  }
};

// cp.async of n16 16-byte chunks from src to dst, spread over the warp's lanes
__device__ __forceinline__ void copy_block(float* dst, const float* src, int n16, int lane) {
  for (int c = lane; c < n16; c += 32) cp_async16(dst + 4 * c, src + 4 * c);
}

// ---- 1. strip terms of the two horizontal carries ---------------------------------------------
template <typename Tin, typename Tg, int NG, bool FW>
__global__ void __launch_bounds__(kWarps * 32) k_pre(const Args p) {
  extern __shared__ __align__(16) float smem[];
  Task t;
  if (!decode(p, t)) return;
  const int lane = threadIdx.x & 31, cg = lane >> 2;
  float* buf0 = smem + (threadIdx.x >> 5) * 2 * kBufPre;
  float A2[NG];
  bool nok[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    A2[g] = (t.act && nok[g]) ? p.A[(size_t)t.d * p.N + n] * kLog2e : 0.f;
  }
  float V[NG][kCols];                      // a*gh of the row after (in forward order)
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int c = 0; c < kCols; ++c) V[g][c] = 0.f;

  InputPrefetch<Tin, Tg, NG, true, true> pf;
  pf.init(p, t, lane);
  pf.load(p, row_of(p, p.H - 1));
  pf.store(buf0, lane);
  __syncwarp();
  for (int e = 0; e < p.H; ++e) {
    const int ii = p.H - 1 - e;
    const int i = row_of(p, ii);
    float* cur = buf0 + (e & 1) * kBufPre;
    if (ii > 0) pf.load(p, row_of(p, ii - 1));
    float xv[kCols], dl[kCols], gy[kCols];
    lds8(cur + kOffX + cg * kCols, xv);
    lds8(cur + kOffD + cg * kCols, dl);
    lds8(cur + kOffG + cg * kCols, gy);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float bv[kCols], cv[kCols];
      lds8(cur + kOffB + (t.q + 4 * g) * kCols, bv);
      lds8(cur + kOffC + (t.q + 4 * g) * kCols, cv);
      float a[kCols];
      float prod = 1.f;
#pragma unroll
      for (int c = 0; c < kCols; ++c) {
        a[c] = ex2_approx(dl[c] * A2[g]);
        prod *= a[c];
        V[g][c] = a[c] * fmaf(cv[c], gy[c], V[g][c]);   // a*gh of this row
      }
      float r = 0.f;                        // forward: hh leaving the strip, from zero
#pragma unroll
      for (int k = 0; k < kCols; ++k) {
        const int c = FW ? kCols - 1 - k : k;
        r = fmaf(a[c], r, (dl[c] * xv[c]) * bv[c]);
      }
      float hc = 0.f;                       // adjoint: a*ghh leaving the strip, from zero
#pragma unroll
      for (int k = 0; k < kCols; ++k) {
        const int c = FW ? k : kCols - 1 - k;
        hc = fmaf(a[c], hc, V[g][c]);       // a*(gh + hc)
      }
      if (t.act && nok[g]) {
        const size_t ci = carry_idx(p, t.b, t.d, i, t.s, t.q + 4 * g);
        p.tf[ci] = r;
        p.tb[ci] = hc;
        p.beta[ci] = prod;
      }
    }
    if (ii > 0) pf.store(buf0 + ((e + 1) & 1) * kBufPre, lane);
    __syncwarp();
  }
}

// ---- 2. carries entering each strip -----------------------------------------------------------
// One thread per (b, row, channel, state): the forward carries in the forward strip order and
// the adjoint carries in the reverse order.  Adjacent threads hold adjacent (channel, state),
// so every strip step is one coalesced access per warp; the terms of kChunk strips are loaded
// before any of them is used, so those loads are in flight together.
constexpr int kChunk = 8;

__global__ void __launch_bounds__(256) k_carry(const Args p, int fw) {
  const long long dn = (long long)p.ncg * kCh * p.N;
  const long long total = (long long)p.batch * p.H * dn;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  if ((t % dn) / p.N >= p.channels) return;        // padding channel
  const size_t base = (size_t)(t / dn) * p.S * dn + (size_t)(t % dn);
  const float* __restrict__ tf = p.tf;
  const float* __restrict__ tb = p.tb;
  const float* __restrict__ be = p.beta;
  float* __restrict__ cf = p.cf;
  float* __restrict__ cb = p.cb;
  for (int dir = 0; dir < 2; ++dir) {
    const bool rev = (dir == 0) == (fw != 0);      // strips walked from the last one
    const float* __restrict__ term = dir == 0 ? tf : tb;
    float* __restrict__ out = dir == 0 ? cf : cb;
    float carry = 0.f;
    for (int e0 = 0; e0 < p.S; e0 += kChunk) {
      float tv[kChunk], bv[kChunk];
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const int s = rev ? p.S - 1 - (e0 + e) : e0 + e;
        const bool ok = e0 + e < p.S;
        tv[e] = ok ? __ldg(term + base + (size_t)s * dn) : 0.f;
        bv[e] = ok ? __ldg(be + base + (size_t)s * dn) : 1.f;
      }
#pragma unroll
      for (int e = 0; e < kChunk; ++e) {
        const int s = rev ? p.S - 1 - (e0 + e) : e0 + e;
        if (e0 + e < p.S) out[base + (size_t)s * dn] = carry;
        carry = fmaf(bv[e], carry, tv[e]);
      }
    }
  }
}

// ---- 3. forward vertical state of every element -----------------------------------------------
template <typename Tin, int NG, bool FW>
__global__ void __launch_bounds__(kWarps * 32, 2) k_states(const Args p) {
  extern __shared__ __align__(16) float smem[];
  Task t;
  if (!decode(p, t)) return;
  const int lane = threadIdx.x & 31, cg = lane >> 2;
  float* buf0 = smem + (threadIdx.x >> 5) * 2 * kBufStates;
  float A2[NG];
  bool nok[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    A2[g] = (t.act && nok[g]) ? p.A[(size_t)t.d * p.N + n] * kLog2e : 0.f;
  }
  float2 h[NG][kPairs];
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int k = 0; k < kPairs; ++k) h[g][k] = make_float2(0.f, 0.f);
  const int n16 = 2 * p.N;                 // 8 channels x N carries, in 16-byte chunks

  InputPrefetch<Tin, float, NG, false, false> pf;
  pf.init(p, t, lane);
  pf.load(p, row_of(p, 0));
  copy_block(buf0 + kOffCF, p.cf + carry_idx(p, t.b, t.cgi * kCh, row_of(p, 0), t.s, 0), n16, lane);
  cp_commit();
  pf.store(buf0, lane);
  for (int ii = 0; ii < p.H; ++ii) {
    const int i = row_of(p, ii);
    float* cur = buf0 + (ii & 1) * kBufStates;
    float* nxt = buf0 + ((ii + 1) & 1) * kBufStates;
    if (ii + 1 < p.H) {
      pf.load(p, row_of(p, ii + 1));
      copy_block(nxt + kOffCF, p.cf + carry_idx(p, t.b, t.cgi * kCh, row_of(p, ii + 1), t.s, 0), n16, lane);
    }
    cp_commit();
    cp_wait1();
    __syncwarp();
    float2 xv[kPairs], dl[kPairs], dxp[kPairs];
    lds8x2(cur + kOffX + cg * kCols, xv);
    lds8x2(cur + kOffD + cg * kCols, dl);
#pragma unroll
    for (int k = 0; k < kPairs; ++k) dxp[k] = __fmul2_rn(dl[k], xv[k]);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const int n = t.q + 4 * g;
      float2 bv[kPairs], a[kPairs], u[kPairs], rr[kPairs];
      lds8x2(cur + kOffB + n * kCols, bv);
      const float2 A2g = make_float2(A2[g], A2[g]);
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {
        const float2 arg = __fmul2_rn(dl[k], A2g);
        a[k] = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
        u[k] = __fmul2_rn(dxp[k], bv[k]);
      }
      float r = nok[g] ? cur[kOffCF + cg * p.N + n] : 0.f;
#pragma unroll
      for (int k = 0; k < kCols; ++k) {       // horizontal, in scan order
        const int c = FW ? kCols - 1 - k : k;
        r = fmaf(lo_hi(a, c), r, lo_hi(u, c));
        if (c & 1) rr[c >> 1].y = r; else rr[c >> 1].x = r;
      }
#pragma unroll
      for (int k = 0; k < kPairs; ++k) h[g][k] = __ffma2_rn(a[k], h[g][k], rr[k]);   // vertical
      if (t.act && nok[g]) {
        float* dst = p.hsave + hs_idx(p, t.b, t.d, i, t.s, n);
        *reinterpret_cast<float4*>(dst) = make_float4(h[g][0].x, h[g][0].y, h[g][1].x, h[g][1].y);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(h[g][2].x, h[g][2].y, h[g][3].x, h[g][3].y);
      }
    }
    if (ii + 1 < p.H) pf.store(nxt, lane);
    __syncwarp();
  }
}

// ---- 3'. vertical-first order: the forward's vertical state and both carry terms ---------------
// In this order the forward's first (vertical) scan needs no carry and the adjoint's horizontal
// scan reads only C*dy, so one pass down the rows stores vv and writes the strip terms of both
// horizontal chains (the forward one over vv, the adjoint one over C*dy) and the product of Abar.
template <typename Tin, typename Tg, int NG, bool FW>
__global__ void __launch_bounds__(kWarps * 32, 2) k_states_vf(const Args p) {
  extern __shared__ __align__(16) float smem[];
  Task t;
  if (!decode(p, t)) return;
  const int lane = threadIdx.x & 31, cg = lane >> 2;
  float* buf0 = smem + (threadIdx.x >> 5) * 2 * kBufStates;
  float A2[NG];
  bool nok[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    A2[g] = (t.act && nok[g]) ? p.A[(size_t)t.d * p.N + n] * kLog2e : 0.f;
  }
  float2 vv[NG][kPairs];
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int k = 0; k < kPairs; ++k) vv[g][k] = make_float2(0.f, 0.f);

  InputPrefetch<Tin, Tg, NG, true, true> pf;
  pf.init(p, t, lane);
  pf.load(p, row_of(p, 0));
  pf.store(buf0, lane);
  __syncwarp();
  for (int ii = 0; ii < p.H; ++ii) {
    const int i = row_of(p, ii);
    float* cur = buf0 + (ii & 1) * kBufStates;
    float* nxt = buf0 + ((ii + 1) & 1) * kBufStates;
    if (ii + 1 < p.H) pf.load(p, row_of(p, ii + 1));
    float2 xv[kPairs], dl[kPairs], gy[kPairs], dxp[kPairs];
    lds8x2(cur + kOffX + cg * kCols, xv);
    lds8x2(cur + kOffD + cg * kCols, dl);
    lds8x2(cur + kOffG + cg * kCols, gy);
#pragma unroll
    for (int k = 0; k < kPairs; ++k) dxp[k] = __fmul2_rn(dl[k], xv[k]);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const int n = t.q + 4 * g;
      float2 bv[kPairs], cv[kPairs], a[kPairs], aw[kPairs];
      lds8x2(cur + kOffB + n * kCols, bv);
      lds8x2(cur + kOffC + n * kCols, cv);
      const float2 A2g = make_float2(A2[g], A2[g]);
      float2 prod2 = make_float2(1.f, 1.f);
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {
        const float2 arg = __fmul2_rn(dl[k], A2g);
        a[k] = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
        prod2 = __fmul2_rn(prod2, a[k]);
        vv[g][k] = __ffma2_rn(a[k], vv[g][k], __fmul2_rn(dxp[k], bv[k]));   // vertical, first
        aw[k] = __fmul2_rn(a[k], __fmul2_rn(cv[k], gy[k]));                // Abar*C*dy
      }
      float r = 0.f;                          // forward: h leaving the strip, from zero
#pragma unroll
      for (int k = 0; k < kCols; ++k) {
        const int c = FW ? kCols - 1 - k : k;
        r = fmaf(lo_hi(a, c), r, lo_hi(vv[g], c));
      }
      float hc = 0.f;                         // adjoint: Abar*g2 leaving the strip, from zero
#pragma unroll
      for (int k = 0; k < kCols; ++k) {
        const int c = FW ? k : kCols - 1 - k;
        hc = fmaf(lo_hi(a, c), hc, lo_hi(aw, c));
      }
      if (t.act && nok[g]) {
        float* dst = p.hsave + hs_idx(p, t.b, t.d, i, t.s, n);
        *reinterpret_cast<float4*>(dst) = make_float4(vv[g][0].x, vv[g][0].y, vv[g][1].x, vv[g][1].y);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(vv[g][2].x, vv[g][2].y, vv[g][3].x, vv[g][3].y);
        const size_t ci = carry_idx(p, t.b, t.d, i, t.s, n);
        p.tf[ci] = r;
        p.tb[ci] = hc;
        p.beta[ci] = prod2.x * prod2.y;
      }
    }
    if (ii + 1 < p.H) pf.store(nxt, lane);
    __syncwarp();
  }
}

// ---- 4. gradients -------------------------------------------------------------------------------
template <typename Tg>
__device__ __forceinline__ void put2(Tg* out, size_t idx, float v0, float v1, bool ok0, bool ok1, bool vec) {
  if constexpr (sizeof(Tg) == 4) {
    if (vec && ok1) {
      *reinterpret_cast<float2*>(reinterpret_cast<float*>(out) + idx) = make_float2(v0, v1);
    } else {
      if (ok0) reinterpret_cast<float*>(out)[idx] = v0;
      if (ok1) reinterpret_cast<float*>(out)[idx + 1] = v1;
    }
  } else {
    const uint16_t b0 = __bfloat16_as_ushort(__float2bfloat16_rn(v0));
    const uint16_t b1 = __bfloat16_as_ushort(__float2bfloat16_rn(v1));
    if (vec && ok1) {
      *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(out) + idx) =
          static_cast<uint32_t>(b0) | (static_cast<uint32_t>(b1) << 16);
    } else {
      if (ok0) reinterpret_cast<uint16_t*>(out)[idx] = b0;
      if (ok1) reinterpret_cast<uint16_t*>(out)[idx + 1] = b1;
    }
  }
}

template <typename Tin, typename Tg, int NG, bool FW, bool VF = false>
__global__ void __launch_bounds__(kWarps * 32) k_main(const Args p) {
  extern __shared__ __align__(16) float smem[];
  Task t;
  if (!decode(p, t, true)) return;
  const int lane = threadIdx.x & 31, cg = lane >> 2;
  const bool hi = lane & 16, m8 = lane & 8, m4 = lane & 4, m2 = lane & 2, m1 = lane & 1;
  float* buf0 = smem + (threadIdx.x >> 5) * 2 * kBufMain;
  const size_t HW = (size_t)p.H * p.W;
  const size_t map = ((size_t)t.b * p.channels + (t.act ? t.d : 0)) * HW;
  float A2[NG], Af[NG];
  bool nok[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    Af[g] = (t.act && nok[g]) ? p.A[(size_t)t.d * p.N + n] : 0.f;
    A2[g] = Af[g] * kLog2e;
  }
  const float Dd = (p.first && t.act && p.Dskip) ? p.Dskip[t.d] : 0.f;
  // this lane's two columns after the reduce-scatters
  const int cq = (m2 ? 4 : 0) + (m1 ? 2 : 0);           // per-element outputs
  const int cbc = (m8 ? 4 : 0) + (m4 ? 2 : 0);          // dB / dC
  float2 V[NG][kPairs];
  float2 dAacc[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    dAacc[g] = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kPairs; ++k) V[g][k] = make_float2(0.f, 0.f);
  }
  float dDacc = 0.f;
  const int n16c = 2 * p.N;                // 8 channels x N carries, in 16-byte chunks
  const int n16h = 16 * p.N;               // 8 channels x N states x 8 columns

  // stage one row (scan-order ii) into buf: inputs from pf, carries and h of row ii-1 by cp.async
  auto stage_ws = [&](float* buf, int ii) {
    const int i = row_of(p, ii);
    const size_t c0 = carry_idx(p, t.b, t.cgi * kCh, i, t.s, 0);
    copy_block(buf + kOffCF, p.cf + c0, n16c, lane);
    copy_block(buf + kOffCB, p.cb + c0, n16c, lane);
    if (ii > 0) copy_block(buf + kOffH, p.hsave + hs_idx(p, t.b, t.cgi * kCh, row_of(p, ii - 1), t.s, 0), n16h, lane);
  };
  InputPrefetch<Tin, Tg, NG, true, true> pf;
  pf.init(p, t, lane);
  pf.load(p, row_of(p, p.H - 1));
  stage_ws(buf0, p.H - 1);
  cp_commit();
  pf.store(buf0, lane);

  for (int e = 0; e < p.H; ++e) {
    const int ii = p.H - 1 - e;
    const int i = row_of(p, ii);
    float* cur = buf0 + (e & 1) * kBufMain;
    float* nxt = buf0 + ((e + 1) & 1) * kBufMain;
    if (ii > 0) {
      pf.load(p, row_of(p, ii - 1));
      stage_ws(nxt, ii - 1);
    }
    cp_commit();
    cp_wait1();
    __syncwarp();
    float2 xv[kPairs], dl[kPairs], gy[kPairs], dxp[kPairs];
    lds8x2(cur + kOffX + cg * kCols, xv);
    lds8x2(cur + kOffD + cg * kCols, dl);
    lds8x2(cur + kOffG + cg * kCols, gy);
    float2 dD2 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kPairs; ++k) {
      dxp[k] = __fmul2_rn(dl[k], xv[k]);
      dD2 = __ffma2_rn(gy[k], xv[k], dD2);
    }
    dDacc += dD2.x + dD2.y;
    float2 s1[kPairs], s2[kPairs];           // sum over the lane's states of ghh*B and dL/da*a*A
#pragma unroll
    for (int k = 0; k < kPairs; ++k) s1[k] = s2[k] = make_float2(0.f, 0.f);

#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const int n = t.q + 4 * g;
      const bool live = t.act && nok[g];
      float2 bv[kPairs], cv[kPairs], hp[kPairs];
      lds8x2(cur + kOffB + n * kCols, bv);
      lds8x2(cur + kOffC + n * kCols, cv);
      if (live && ii > 0) {
        lds8x2(cur + kOffH + (cg * p.N + n) * kCols, hp);
      } else {
#pragma unroll
        for (int k = 0; k < kPairs; ++k) hp[k] = make_float2(0.f, 0.f);
      }
      const float hin = live ? cur[kOffCF + cg * p.N + n] : 0.f;
      const float cin = live ? cur[kOffCB + cg * p.N + n] : 0.f;
      const float2 A2g = make_float2(A2[g], A2[g]);
      const float2 Afg = make_float2(Af[g], Af[g]);
      float pB[kCols], pC[kCols];
      if constexpr (!VF) {
      float2 a[kPairs], u[kPairs], gh[kPairs];
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {
        const float2 arg = __fmul2_rn(dl[k], A2g);
        a[k] = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
        u[k] = __fmul2_rn(dxp[k], bv[k]);
        gh[k] = __ffma2_rn(cv[k], gy[k], V[g][k]);          // adjoint, vertical
        V[g][k] = __fmul2_rn(a[k], gh[k]);
      }
      float2 hhp[kPairs], rr[kPairs], cpre[kPairs];
      float r = hin;
#pragma unroll
      for (int k = 0; k < kCols; ++k) {       // forward recompute: hh before and after each column
        const int c = FW ? kCols - 1 - k : k;
        if (c & 1) hhp[c >> 1].y = r; else hhp[c >> 1].x = r;
        r = fmaf(lo_hi(a, c), r, lo_hi(u, c));
        if (c & 1) rr[c >> 1].y = r; else rr[c >> 1].x = r;
      }
      float carry = cin;
#pragma unroll
      for (int k = 0; k < kCols; ++k) {       // adjoint, horizontal: carry before each column
        const int c = FW ? k : kCols - 1 - k;
        if (c & 1) cpre[c >> 1].y = carry; else cpre[c >> 1].x = carry;
        carry = fmaf(lo_hi(a, c), carry, lo_hi(V[g], c));  // a*(gh + carry)
      }
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {       // what each column adds
        const float2 hc = __ffma2_rn(a[k], hp[k], rr[k]);   // h of this row
        const float2 ghh = __fadd2_rn(gh[k], cpre[k]);
        const float2 ta = __fmul2_rn(__ffma2_rn(gh[k], hp[k], __fmul2_rn(ghh, hhp[k])), a[k]);
        s1[k] = __ffma2_rn(ghh, bv[k], s1[k]);
        s2[k] = __ffma2_rn(ta, Afg, s2[k]);
        dAacc[g] = __ffma2_rn(ta, dl[k], dAacc[g]);
        const float2 b2 = __fmul2_rn(ghh, dxp[k]);
        const float2 c2 = __fmul2_rn(gy[k], hc);
        pB[2 * k] = b2.x; pB[2 * k + 1] = b2.y;
        pC[2 * k] = c2.x; pC[2 * k + 1] = c2.y;
      }
      } else {
      // vertical first: hp holds vv of the row before; g2 is the adjoint of the horizontal
      // (second) scan, g1 that of the vertical (first) scan, carried up the column in V
      float2 a[kPairs], vvc[kPairs], w[kPairs], aw[kPairs];
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {
        const float2 arg = __fmul2_rn(dl[k], A2g);
        a[k] = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
        vvc[k] = __ffma2_rn(a[k], hp[k], __fmul2_rn(dxp[k], bv[k]));   // vv of this row
        w[k] = __fmul2_rn(cv[k], gy[k]);
        aw[k] = __fmul2_rn(a[k], w[k]);
      }
      float2 hhp[kPairs], hcur[kPairs], cpre[kPairs];
      float r = hin;
#pragma unroll
      for (int k = 0; k < kCols; ++k) {       // forward recompute: h before and after each column
        const int c = FW ? kCols - 1 - k : k;
        if (c & 1) hhp[c >> 1].y = r; else hhp[c >> 1].x = r;
        r = fmaf(lo_hi(a, c), r, lo_hi(vvc, c));
        if (c & 1) hcur[c >> 1].y = r; else hcur[c >> 1].x = r;
      }
      float carry = cin;
#pragma unroll
      for (int k = 0; k < kCols; ++k) {       // adjoint, horizontal: carry before each column
        const int c = FW ? k : kCols - 1 - k;
        if (c & 1) cpre[c >> 1].y = carry; else cpre[c >> 1].x = carry;
        carry = fmaf(lo_hi(a, c), carry, lo_hi(aw, c));    // a*(C*dy + carry)
      }
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {       // what each column adds
        const float2 g2 = __fadd2_rn(w[k], cpre[k]);
        const float2 g1 = __fadd2_rn(g2, V[g][k]);
        V[g][k] = __fmul2_rn(a[k], g1);                      // adjoint, vertical, carried up
        const float2 ta = __fmul2_rn(__ffma2_rn(g2, hhp[k], __fmul2_rn(g1, hp[k])), a[k]);
        s1[k] = __ffma2_rn(g1, bv[k], s1[k]);
        s2[k] = __ffma2_rn(ta, Afg, s2[k]);
        dAacc[g] = __ffma2_rn(ta, dl[k], dAacc[g]);
        const float2 b2 = __fmul2_rn(g1, dxp[k]);
        const float2 c2 = __fmul2_rn(gy[k], hcur[k]);
        pB[2 * k] = b2.x; pB[2 * k + 1] = b2.y;
        pC[2 * k] = c2.x; pC[2 * k + 1] = c2.y;
      }
      }
      // dB, dC: sum over the warp's 8 channels (lanes xor 16, 8, 4 share the state)
      float k1[kCols];
#pragma unroll
      for (int c = 0; c < kCols; ++c) {
        const float send = hi ? pB[c] : pC[c];
        k1[c] = (hi ? pC[c] : pB[c]) + __shfl_xor_sync(kFull, send, 16);
      }
      float k2[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float send = m8 ? k1[c] : k1[c + 4];
        k2[c] = (m8 ? k1[c + 4] : k1[c]) + __shfl_xor_sync(kFull, send, 8);
      }
      float o[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float send = m4 ? k2[c] : k2[c + 2];
        o[c] = (m4 ? k2[c + 2] : k2[c]) + __shfl_xor_sync(kFull, send, 4);
      }
      if (nok[g]) {
        const int j = t.j0 + cbc;
        float* dst = (hi ? p.dC : p.dB) + (((size_t)t.b * p.K + p.k) * p.N + n) * HW + (size_t)i * p.W + j;
        if (p.vec2 && j + 1 < p.W) {
          atomicAdd(reinterpret_cast<float2*>(dst), make_float2(o[0], o[1]));
        } else {
          if (j < p.W) atomicAdd(dst, o[0]);
          if (j + 1 < p.W) atomicAdd(dst + 1, o[1]);
        }
      }
    }
    // dx, ddelta: sum over the channel's 4 state lanes (xor 2, 1)
    float a1[4], a2[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const float s1lo = lo_hi(s1, c), s1hi = lo_hi(s1, c + 4);
      const float s2lo = lo_hi(s2, c), s2hi = lo_hi(s2, c + 4);
      a1[c] = (m2 ? s1hi : s1lo) + __shfl_xor_sync(kFull, m2 ? s1lo : s1hi, 2);
      a2[c] = (m2 ? s2hi : s2lo) + __shfl_xor_sync(kFull, m2 ? s2lo : s2hi, 2);
    }
    float f1[2], f2[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float send1 = m1 ? a1[c] : a1[c + 2];
      const float send2 = m1 ? a2[c] : a2[c + 2];
      f1[c] = (m1 ? a1[c + 2] : a1[c]) + __shfl_xor_sync(kFull, send1, 1);
      f2[c] = (m1 ? a2[c + 2] : a2[c]) + __shfl_xor_sync(kFull, send2, 1);
    }
    if (t.act) {
      const int j = t.j0 + cq;
      const bool ok0 = j < p.W, ok1 = j + 1 < p.W;
      float vx[2], vd[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        vx[k] = fmaf(pick(dl, m2, m1, k), f1[k], Dd * pick(gy, m2, m1, k));
        vd[k] = fmaf(pick(xv, m2, m1, k), f1[k], f2[k]);
      }
      const size_t idx = map + (size_t)i * p.W + j;
      if (!p.first) {                         // add what the earlier orientations left
        if (ok0) { vx[0] += p.accx[idx]; vd[0] += p.accd[idx]; }
        if (ok1) { vx[1] += p.accx[idx + 1]; vd[1] += p.accd[idx + 1]; }
      }
      if (p.last) {
        put2(static_cast<Tg*>(p.dx), idx, vx[0], vx[1], ok0, ok1, p.vec2);
        put2(static_cast<Tg*>(p.ddelta), idx, vd[0], vd[1], ok0, ok1, p.vec2);
      } else {
        put2(p.accx, idx, vx[0], vx[1], ok0, ok1, p.vec2);
        put2(p.accd, idx, vd[0], vd[1], ok0, ok1, p.vec2);
      }
    }
    if (ii > 0) pf.store(nxt, lane);
    __syncwarp();
  }
#pragma unroll
  for (int g = 0; g < NG; ++g)
    if (t.act && nok[g]) atomicAdd(p.dA + (size_t)t.d * p.N + t.q + 4 * g, dAacc[g].x + dAacc[g].y);
  if (p.first && t.act && t.q == 0 && p.dDskip) atomicAdd(p.dDskip + t.d, dDacc);
}

// ---- host ---------------------------------------------------------------------------------------
struct BwdShape {
  int batch, channels, H, W, N, K, S, ncg;
  bool bf16, out_f32;
  unsigned orient;
  size_t in_elem, out_elem, xy, bc, carries;
};

int popcount4(unsigned v) { return (v & 1) + ((v >> 1) & 1) + ((v >> 2) & 1) + ((v >> 3) & 1); }

int bwd_shape(int batch, int channels, int H, int W, int N, unsigned flags, BwdShape* s) {
  if (flags & ~SCAN2D_FLAGS_KNOWN) return SCAN2D_E_FLAGS;
  if ((flags & SCAN2D_OUT_F32) && !(flags & SCAN2D_BF16)) return SCAN2D_E_FLAGS;
  if (batch < 1 || channels < 1 || H < 1 || W < 1) return SCAN2D_E_DIMS;
  if (N < 1 || N > kMaxNBwd) return SCAN2D_E_N;
  const unsigned long long hw = static_cast<unsigned long long>(H) * W;
  if (hw > (1ull << 31) - 1) return SCAN2D_E_DIMS;
  unsigned orient = (flags >> 4) & 0xFu;
  if (orient == 0) orient = 1;
  const int K = popcount4(orient);
  const int S = (W + kCols - 1) / kCols;
  const unsigned long long xy = static_cast<unsigned long long>(batch) * channels * hw;
  const unsigned long long bc = static_cast<unsigned long long>(batch) * K * N * hw;
  const unsigned long long hs = static_cast<unsigned long long>(batch) * channels * N * hw;
  const int ncg = (channels + kCh - 1) / kCh;
  const unsigned long long cr = static_cast<unsigned long long>(batch) * ncg * kCh * H * S * N;
  if (xy > (1ull << 40) || bc > (1ull << 40) || hs > (1ull << 40) || cr > (1ull << 40)) return SCAN2D_E_DIMS;
  s->batch = batch; s->channels = channels; s->H = H; s->W = W; s->N = N; s->K = K; s->S = S;
  s->ncg = (channels + kCh - 1) / kCh;
  s->bf16 = (flags & SCAN2D_BF16) != 0;
  s->out_f32 = !s->bf16 || (flags & SCAN2D_OUT_F32) != 0;
  s->orient = orient;
  s->in_elem = s->bf16 ? 2 : 4;
  s->out_elem = s->out_f32 ? 4 : 2;
  s->xy = static_cast<size_t>(xy);
  s->bc = static_cast<size_t>(bc);
  s->carries = static_cast<size_t>(cr);
  return SCAN2D_OK;
}

size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
  size_t hsave, tf, tb, beta, cf, cb, accx, accd, total;
};

WsLayout ws_layout(const BwdShape& s) {
  WsLayout l{};
  size_t off = 0;
  l.hsave = off; off += round256(s.carries * kCols * sizeof(float));   // strips padded to 8 columns
  l.tf = off;    off += round256(s.carries * sizeof(float));
  l.tb = off;    off += round256(s.carries * sizeof(float));
  l.beta = off;  off += round256(s.carries * sizeof(float));
  l.cf = off;    off += round256(s.carries * sizeof(float));
  l.cb = off;    off += round256(s.carries * sizeof(float));
  const bool acc = !s.out_f32 && s.K > 1;    // bf16 outputs summed over orientations in fp32
  l.accx = off;  off += acc ? round256(s.xy * sizeof(float)) : 0;
  l.accd = off;  off += acc ? round256(s.xy * sizeof(float)) : 0;
  l.total = off;
  return l;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <typename K>
bool launch_warps(K kern, int floats_per_buffer, const Args& a, cudaStream_t st) {
  const long long nblocks = (a.tasks + kWarps - 1) / kWarps;
  if (nblocks > 0x7fffffffLL) return false;
  const unsigned blocks = static_cast<unsigned>(nblocks);
  const size_t smem = static_cast<size_t>(kWarps) * 2 * floats_per_buffer * sizeof(float);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return false;
  kern<<<blocks, kWarps * 32, smem, st>>>(a);
  return true;
}

template <typename Tin, typename Tg, int NG>
int launch_orientation(const Args& a, bool fw, bool vf, cudaStream_t st) {
  const long long threads = (long long)a.batch * a.H * a.ncg * kCh * a.N;
  if ((threads + 255) / 256 > 0x7fffffffLL) return SCAN2D_E_DIMS;
  const unsigned cblocks = static_cast<unsigned>((threads + 255) / 256);
  bool ok;
  if (!vf) {                   // horizontal first: terms (rows up), carries, states (rows down), gradients
    ok = fw ? launch_warps(k_pre<Tin, Tg, NG, true>, kBufPre, a, st)
            : launch_warps(k_pre<Tin, Tg, NG, false>, kBufPre, a, st);
    k_carry<<<cblocks, 256, 0, st>>>(a, fw ? 1 : 0);
    ok = ok && (fw ? launch_warps(k_states<Tin, NG, true>, kBufStates, a, st)
                   : launch_warps(k_states<Tin, NG, false>, kBufStates, a, st));
    ok = ok && (fw ? launch_warps(k_main<Tin, Tg, NG, true>, kBufMain, a, st)
                   : launch_warps(k_main<Tin, Tg, NG, false>, kBufMain, a, st));
  } else {                     // vertical first: states and terms (rows down), carries, gradients
    ok = fw ? launch_warps(k_states_vf<Tin, Tg, NG, true>, kBufStates, a, st)
            : launch_warps(k_states_vf<Tin, Tg, NG, false>, kBufStates, a, st);
    k_carry<<<cblocks, 256, 0, st>>>(a, fw ? 1 : 0);
    ok = ok && (fw ? launch_warps(k_main<Tin, Tg, NG, true, true>, kBufMain, a, st)
                   : launch_warps(k_main<Tin, Tg, NG, false, true>, kBufMain, a, st));
  }
  if (!ok) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  return cudaGetLastError() == cudaSuccess ? SCAN2D_OK : SCAN2D_E_LAUNCH;
}

template <typename Tin, typename Tg>
int launch_ng(const Args& a, bool fw, bool vf, cudaStream_t st) {
  if (a.N <= 4) return launch_orientation<Tin, Tg, 1>(a, fw, vf, st);
  if (a.N <= 8) return launch_orientation<Tin, Tg, 2>(a, fw, vf, st);
  return launch_orientation<Tin, Tg, 4>(a, fw, vf, st);
}

}  // namespace

extern "C" {

size_t scan2d_bwd_workspace_bytes(int batch, int channels, int H, int W, int N, unsigned flags) {
  BwdShape s;
  if (bwd_shape(batch, channels, H, W, N, flags, &s) != SCAN2D_OK) return 0;
  return ws_layout(s).total;
}

int scan2d_bwd(const void* x, const void* delta, const float* A, const void* B, const void* C,
               const float* Dskip, const void* dy, void* dx, void* ddelta, float* dA, float* dB,
               float* dC, float* dDskip, void* workspace, size_t workspace_bytes, int batch,
               int channels, int H, int W, int N, unsigned flags, void* stream) {
  BwdShape s;
  int rc = bwd_shape(batch, channels, H, W, N, flags, &s);
  if (rc) return rc;
  if (!x || !delta || !A || !B || !C || !dy || !dx || !ddelta || !dA || !dB || !dC || !workspace)
    return SCAN2D_E_NULL;
  if (!aligned(x, s.in_elem) || !aligned(delta, s.in_elem) || !aligned(B, s.in_elem) ||
      !aligned(C, s.in_elem) || !aligned(A, 4) || !aligned(Dskip, 4) || !aligned(dy, s.out_elem) ||
      !aligned(dx, s.out_elem) || !aligned(ddelta, s.out_elem) || !aligned(dA, 4) ||
      !aligned(dB, 4) || !aligned(dC, 4) || !aligned(dDskip, 4) || !aligned(workspace, 256))
    return SCAN2D_E_ALIGN;
  const WsLayout l = ws_layout(s);
  if (workspace_bytes < l.total) return SCAN2D_E_WORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_DEVICE;
  }
  if (major != 10) return SCAN2D_E_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);

  if (cudaMemsetAsync(dA, 0, (size_t)channels * N * sizeof(float), st) != cudaSuccess ||
      cudaMemsetAsync(dB, 0, s.bc * sizeof(float), st) != cudaSuccess ||
      cudaMemsetAsync(dC, 0, s.bc * sizeof(float), st) != cudaSuccess ||
      (dDskip && cudaMemsetAsync(dDskip, 0, (size_t)channels * sizeof(float), st) != cudaSuccess)) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }

  Args a{};
  a.x = x; a.delta = delta; a.A = A; a.B = B; a.C = C; a.Dskip = Dskip; a.dy = dy;
  a.dx = dx; a.ddelta = ddelta;
  a.accx = s.out_f32 ? static_cast<float*>(dx) : reinterpret_cast<float*>(ws + l.accx);
  a.accd = s.out_f32 ? static_cast<float*>(ddelta) : reinterpret_cast<float*>(ws + l.accd);
  a.dA = dA; a.dB = dB; a.dC = dC; a.dDskip = dDskip;
  a.hsave = reinterpret_cast<float*>(ws + l.hsave);
  a.tf = reinterpret_cast<float*>(ws + l.tf);
  a.tb = reinterpret_cast<float*>(ws + l.tb);
  a.beta = reinterpret_cast<float*>(ws + l.beta);
  a.cf = reinterpret_cast<float*>(ws + l.cf);
  a.cb = reinterpret_cast<float*>(ws + l.cb);
  a.batch = batch; a.channels = channels; a.H = H; a.W = W; a.N = N; a.K = s.K; a.S = s.S;
  a.ncg = s.ncg;
  a.tasks = (long long)batch * s.S * s.ncg;
  a.vec2 = W % 2 == 0 && aligned(dx, 2 * s.out_elem) && aligned(ddelta, 2 * s.out_elem) &&
           aligned(dB, 8) && aligned(dC, 8);

  const bool vf = (flags & SCAN2D_VFIRST) != 0;
  int k = 0;
  for (int o = 0; o < 4; ++o) {
    if (!((s.orient >> o) & 1u)) continue;
    a.k = k;
    a.flipH = (o >> 1) & 1;
    a.first = k == 0;
    a.last = k == s.K - 1;
    const bool fw = (o & 1) != 0;
    if (!s.bf16) rc = launch_ng<float, float>(a, fw, vf, st);
    else if (s.out_f32) rc = launch_ng<uint16_t, float>(a, fw, vf, st);
    else rc = launch_ng<uint16_t, uint16_t>(a, fw, vf, st);
    if (rc) return rc;
    ++k;
  }
  return SCAN2D_OK;
}

}  // extern "C"
