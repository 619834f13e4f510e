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
// per element, one orientation at a time).  No kernel here waits on another warp:
//   1. k_pre    walks each strip's rows backwards, carrying the adjoint's vertical state in
//               registers.  For every (row, strip, channel, state) it writes what the strip
//               adds to the two horizontal carries when it starts from zero (forward: the hh
//               leaving the strip; adjoint: a*ghh leaving it) and the product of a across the
//               strip: a carry that enters the strip leaves it multiplied by that product.
//   2. k_carry  runs the two short recurrences across the strips of every row and replaces
//               those terms in place by the carry that enters each strip.
//   3. k_states walks each strip's rows forwards from the known carries and stores h.
//   4. k_main   walks each strip's rows backwards from the known carries, with h of the row
//               before read back, and produces every gradient.
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
  float* hsave;             // (batch, channels, N, H, W): forward vertical state of one orientation
  float* cf;                // (batch, channels, H, S, N): forward horizontal carry terms
  float* cb;                //   adjoint horizontal carry terms
  float* beta;              //   product of a across the strip
  long long tasks;          // warps: batch * S * channel groups
  int batch, channels, H, W, N, K, S, ncg;
  int k;                    // orientation index: B_k, C_k, dB_k, dC_k
  int flipH;
  int first, last;          // first / last orientation of the call
  int vec_in;               // input rows allow 16-byte loads
  int vec_g;                // dy rows allow 16-byte loads
  int vec_h;                // hsave rows allow 16-byte access (W % 4 == 0)
  int vec2;                 // W even and outputs aligned: 2-column stores and atomics
};

__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(uint16_t v) { return __uint_as_float(static_cast<uint32_t>(v) << 16); }

// 8 consecutive values of a row starting at column j0; columns at or beyond W read as 0.
template <typename T>
__device__ __forceinline__ void load8(const T* row, int j0, int W, bool vec, float (&v)[kCols]) {
  if (vec && j0 + kCols <= W) {
    if constexpr (sizeof(T) == 4) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(row + j0));
      const float4 b = __ldg(reinterpret_cast<const float4*>(row + j0 + 4));
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(row + j0));
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w[e] << 16);
        v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < kCols; ++c) v[c] = (j0 + c < W) ? to_f(row[j0 + c]) : 0.f;
  }
}

// Plain (coherent) loads for buffers written by an earlier kernel of the same call.
__device__ __forceinline__ void load8_ws(const float* row, int j0, int W, bool vec, float (&v)[kCols]) {
  if (vec && j0 + kCols <= W) {
    const float4 a = *reinterpret_cast<const float4*>(row + j0);
    const float4 b = *reinterpret_cast<const float4*>(row + j0 + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
#pragma unroll
    for (int c = 0; c < kCols; ++c) v[c] = (j0 + c < W) ? row[j0 + c] : 0.f;
  }
}

__device__ __forceinline__ void store8_ws(float* row, int j0, int W, bool vec, const float (&v)[kCols]) {
  if (vec && j0 + kCols <= W) {
    *reinterpret_cast<float4*>(row + j0) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(row + j0 + 4) = make_float4(v[4], v[5], v[6], v[7]);
  } else {
#pragma unroll
    for (int c = 0; c < kCols; ++c)
      if (j0 + c < W) row[j0 + c] = v[c];
  }
}

// One of the lane's 8 columns, chosen by two lane bits (keeps the register arrays static).
__device__ __forceinline__ float pick(const float (&v)[kCols], bool m2, bool m1, int e) {
  const float lo = m1 ? v[2 + e] : v[e];
  const float hi = m1 ? v[6 + e] : v[4 + e];
  return m2 ? hi : lo;
}

struct Task {
  int b, s, d, q, j0;
  bool act;
};

__device__ __forceinline__ bool decode(const Args& p, Task& t) {
  const long long task = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  if (task >= p.tasks) return false;
  const int lane = threadIdx.x & 31;
  const int cgi = static_cast<int>(task % p.ncg);
  const long long rest = task / p.ncg;
  t.s = static_cast<int>(rest % p.S);
  t.b = static_cast<int>(rest / p.S);
  t.d = cgi * kCh + (lane >> 2);
  t.q = lane & 3;
  t.j0 = t.s * kCols;
  t.act = t.d < p.channels;
  return true;
}

// scan-order row ii of this orientation -> stored row
__device__ __forceinline__ int row_of(const Args& p, int ii) { return p.flipH ? p.H - 1 - ii : ii; }

// index of (b, d, row i, strip s, state n) in the strip-carry arrays
__device__ __forceinline__ size_t carry_idx(const Args& p, int b, int d, int i, int s, int n) {
  return ((((size_t)b * p.channels + d) * p.H + i) * p.S + s) * p.N + n;
}

// ---- 1. strip terms of the two horizontal carries ---------------------------------------------
template <typename Tin, typename Tg, int NG, bool FW>
__global__ void __launch_bounds__(kWarps * 32) k_pre(const Args p) {
  Task t;
  if (!decode(p, t)) return;
  const size_t HW = (size_t)p.H * p.W;
  const size_t map = ((size_t)t.b * p.channels + (t.act ? t.d : 0)) * HW;
  const Tin* xm = static_cast<const Tin*>(p.x) + map;
  const Tin* dm = static_cast<const Tin*>(p.delta) + map;
  const Tg* gm = static_cast<const Tg*>(p.dy) + map;
  float A2[NG];
  bool nok[NG];
  const Tin* Bp[NG];
  const Tin* Cp[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    A2[g] = (t.act && nok[g]) ? p.A[(size_t)t.d * p.N + n] * kLog2e : 0.f;
    const size_t plane = (((size_t)t.b * p.K + p.k) * p.N + (nok[g] ? n : 0)) * HW;
    Bp[g] = static_cast<const Tin*>(p.B) + plane;
    Cp[g] = static_cast<const Tin*>(p.C) + plane;
  }
  float V[NG][kCols];                      // a*gh of the row after (in forward order)
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int c = 0; c < kCols; ++c) V[g][c] = 0.f;

  for (int ii = p.H - 1; ii >= 0; --ii) {
    const int i = row_of(p, ii);
    float xv[kCols], dl[kCols], gy[kCols];
    if (t.act) {
      load8(xm + (size_t)i * p.W, t.j0, p.W, p.vec_in, xv);
      load8(dm + (size_t)i * p.W, t.j0, p.W, p.vec_in, dl);
      load8(gm + (size_t)i * p.W, t.j0, p.W, p.vec_g, gy);
    } else {
#pragma unroll
      for (int c = 0; c < kCols; ++c) xv[c] = dl[c] = gy[c] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      float bv[kCols], cv[kCols];
      if (nok[g]) {
        load8(Bp[g] + (size_t)i * p.W, t.j0, p.W, p.vec_in, bv);
        load8(Cp[g] + (size_t)i * p.W, t.j0, p.W, p.vec_in, cv);
      } else {
#pragma unroll
        for (int c = 0; c < kCols; ++c) bv[c] = cv[c] = 0.f;
      }
      float a[kCols];
      float prod = 1.f;
#pragma unroll
      for (int c = 0; c < kCols; ++c) {
        a[c] = ex2_approx(dl[c] * A2[g]);
        prod *= a[c];
      }
      float r = 0.f;                        // forward: hh leaving the strip, from zero
#pragma unroll
      for (int e = 0; e < kCols; ++e) {
        const int c = FW ? kCols - 1 - e : e;
        r = fmaf(a[c], r, (dl[c] * xv[c]) * bv[c]);
      }
      float hc = 0.f;                       // adjoint: a*ghh leaving the strip, from zero
#pragma unroll
      for (int e = 0; e < kCols; ++e) {
        const int c = FW ? e : kCols - 1 - e;
        const float gh = fmaf(cv[c], gy[c], V[g][c]);
        V[g][c] = a[c] * gh;
        hc = a[c] * (gh + hc);
      }
      if (t.act && nok[g]) {
        const size_t ci = carry_idx(p, t.b, t.d, i, t.s, t.q + 4 * g);
        p.cf[ci] = r;
        p.cb[ci] = hc;
        p.beta[ci] = prod;
      }
    }
  }
}

// ---- 2. carries entering each strip -----------------------------------------------------------
// One thread per (b, d, row, state): forward carries in the forward strip order, adjoint
// carries in the reverse order; each term is replaced by the carry that enters its strip.
__global__ void __launch_bounds__(256) k_carry(const Args p, int fw) {
  const long long total = (long long)p.batch * p.channels * p.H * p.N;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total) return;
  const int n = static_cast<int>(t % p.N);
  const size_t base = (size_t)(t / p.N) * p.S * p.N + n;
  float carry = 0.f;
  for (int e = 0; e < p.S; ++e) {
    const int s = fw ? p.S - 1 - e : e;
    const size_t ci = base + (size_t)s * p.N;
    const float term = p.cf[ci];
    p.cf[ci] = carry;
    carry = fmaf(p.beta[ci], carry, term);
  }
  carry = 0.f;
  for (int e = 0; e < p.S; ++e) {
    const int s = fw ? e : p.S - 1 - e;
    const size_t ci = base + (size_t)s * p.N;
    const float term = p.cb[ci];
    p.cb[ci] = carry;
    carry = fmaf(p.beta[ci], carry, term);
  }
}

// ---- 3. forward vertical state of every element -----------------------------------------------
template <typename Tin, int NG, bool FW>
__global__ void __launch_bounds__(kWarps * 32) k_states(const Args p) {
  Task t;
  if (!decode(p, t)) return;
  if (!t.act) return;                       // no shuffles in this kernel
  const size_t HW = (size_t)p.H * p.W;
  const size_t map = ((size_t)t.b * p.channels + t.d) * HW;
  const Tin* xm = static_cast<const Tin*>(p.x) + map;
  const Tin* dm = static_cast<const Tin*>(p.delta) + map;
  float A2[NG];
  bool nok[NG];
  const Tin* Bp[NG];
  float* hs[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    A2[g] = nok[g] ? p.A[(size_t)t.d * p.N + n] * kLog2e : 0.f;
    Bp[g] = static_cast<const Tin*>(p.B) + (((size_t)t.b * p.K + p.k) * p.N + (nok[g] ? n : 0)) * HW;
    hs[g] = p.hsave + (((size_t)t.b * p.channels + t.d) * p.N + (nok[g] ? n : 0)) * HW;
  }
  float h[NG][kCols];
#pragma unroll
  for (int g = 0; g < NG; ++g)
#pragma unroll
    for (int c = 0; c < kCols; ++c) h[g][c] = 0.f;

  for (int ii = 0; ii < p.H; ++ii) {
    const int i = row_of(p, ii);
    float xv[kCols], dl[kCols];
    load8(xm + (size_t)i * p.W, t.j0, p.W, p.vec_in, xv);
    load8(dm + (size_t)i * p.W, t.j0, p.W, p.vec_in, dl);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      if (!nok[g]) continue;
      float bv[kCols];
      load8(Bp[g] + (size_t)i * p.W, t.j0, p.W, p.vec_in, bv);
      float r = p.cf[carry_idx(p, t.b, t.d, i, t.s, t.q + 4 * g)];
#pragma unroll
      for (int e = 0; e < kCols; ++e) {
        const int c = FW ? kCols - 1 - e : e;
        const float a = ex2_approx(dl[c] * A2[g]);
        r = fmaf(a, r, (dl[c] * xv[c]) * bv[c]);
        h[g][c] = fmaf(a, h[g][c], r);
      }
      store8_ws(hs[g] + (size_t)i * p.W, t.j0, p.W, p.vec_h, h[g]);
    }
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

template <typename Tin, typename Tg, int NG, bool FW>
__global__ void __launch_bounds__(kWarps * 32) k_main(const Args p) {
  Task t;
  if (!decode(p, t)) return;
  const int lane = threadIdx.x & 31;
  const bool hi = lane & 16, m8 = lane & 8, m4 = lane & 4, m2 = lane & 2, m1 = lane & 1;
  const size_t HW = (size_t)p.H * p.W;
  const size_t map = ((size_t)t.b * p.channels + (t.act ? t.d : 0)) * HW;
  const Tin* xm = static_cast<const Tin*>(p.x) + map;
  const Tin* dm = static_cast<const Tin*>(p.delta) + map;
  const Tg* gm = static_cast<const Tg*>(p.dy) + map;
  float A2[NG], Af[NG];
  bool nok[NG];
  const Tin* Bp[NG];
  const Tin* Cp[NG];
  const float* hs[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const int n = t.q + 4 * g;
    nok[g] = n < p.N;
    Af[g] = (t.act && nok[g]) ? p.A[(size_t)t.d * p.N + n] : 0.f;
    A2[g] = Af[g] * kLog2e;
    const size_t plane = (((size_t)t.b * p.K + p.k) * p.N + (nok[g] ? n : 0)) * HW;
    Bp[g] = static_cast<const Tin*>(p.B) + plane;
    Cp[g] = static_cast<const Tin*>(p.C) + plane;
    hs[g] = p.hsave + (((size_t)t.b * p.channels + (t.act ? t.d : 0)) * p.N + (nok[g] ? n : 0)) * HW;
  }
  const float Dd = (p.first && t.act && p.Dskip) ? p.Dskip[t.d] : 0.f;
  // this lane's two columns after the reduce-scatters
  const int cq = (m2 ? 4 : 0) + (m1 ? 2 : 0);           // per-element outputs
  const int cbc = (m8 ? 4 : 0) + (m4 ? 2 : 0);          // dB / dC
  float V[NG][kCols];
  float dAacc[NG];
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    dAacc[g] = 0.f;
#pragma unroll
    for (int c = 0; c < kCols; ++c) V[g][c] = 0.f;
  }
  float dDacc = 0.f;

  for (int ii = p.H - 1; ii >= 0; --ii) {
    const int i = row_of(p, ii);
    float xv[kCols], dl[kCols], gy[kCols];
    if (t.act) {
      load8(xm + (size_t)i * p.W, t.j0, p.W, p.vec_in, xv);
      load8(dm + (size_t)i * p.W, t.j0, p.W, p.vec_in, dl);
      load8(gm + (size_t)i * p.W, t.j0, p.W, p.vec_g, gy);
    } else {
#pragma unroll
      for (int c = 0; c < kCols; ++c) xv[c] = dl[c] = gy[c] = 0.f;
    }
    float dxp[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      dxp[c] = dl[c] * xv[c];
      dDacc = fmaf(gy[c], xv[c], dDacc);
    }
    float s1[kCols], s2[kCols];              // sum over the lane's states of ghh*B and dL/da*a*A
#pragma unroll
    for (int c = 0; c < kCols; ++c) s1[c] = s2[c] = 0.f;

#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const bool live = t.act && nok[g];
      float bv[kCols], cv[kCols], hp[kCols];
      float hin = 0.f, cin = 0.f;
      if (nok[g]) {
        load8(Bp[g] + (size_t)i * p.W, t.j0, p.W, p.vec_in, bv);
        load8(Cp[g] + (size_t)i * p.W, t.j0, p.W, p.vec_in, cv);
      } else {
#pragma unroll
        for (int c = 0; c < kCols; ++c) bv[c] = cv[c] = 0.f;
      }
      if (live && ii > 0) {
        load8_ws(hs[g] + (size_t)row_of(p, ii - 1) * p.W, t.j0, p.W, p.vec_h, hp);
      } else {
#pragma unroll
        for (int c = 0; c < kCols; ++c) hp[c] = 0.f;
      }
      if (live) {
        const size_t ci = carry_idx(p, t.b, t.d, i, t.s, t.q + 4 * g);
        hin = p.cf[ci];
        cin = p.cb[ci];
      }
      float a[kCols], hhp[kCols], hc[kCols];
      float r = hin;
#pragma unroll
      for (int e = 0; e < kCols; ++e) {       // forward: hh before each column, and h
        const int c = FW ? kCols - 1 - e : e;
        a[c] = ex2_approx(dl[c] * A2[g]);
        hhp[c] = r;
        r = fmaf(a[c], r, dxp[c] * bv[c]);
        hc[c] = fmaf(a[c], hp[c], r);
      }
      float gh[kCols];
#pragma unroll
      for (int c = 0; c < kCols; ++c) {       // adjoint, vertical
        gh[c] = fmaf(cv[c], gy[c], V[g][c]);
        V[g][c] = a[c] * gh[c];
      }
      float pB[kCols], pC[kCols];
      float carry = cin;
#pragma unroll
      for (int e = 0; e < kCols; ++e) {       // adjoint, horizontal, and what each column adds
        const int c = FW ? e : kCols - 1 - e;
        const float ghh = gh[c] + carry;
        carry = a[c] * ghh;
        const float ta = fmaf(gh[c], hp[c], ghh * hhp[c]) * a[c];
        s1[c] = fmaf(ghh, bv[c], s1[c]);
        s2[c] = fmaf(ta, Af[g], s2[c]);
        dAacc[g] = fmaf(ta, dl[c], dAacc[g]);
        pB[c] = ghh * dxp[c];
        pC[c] = gy[c] * hc[c];
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
        float* dst = (hi ? p.dC : p.dB) + (((size_t)t.b * p.K + p.k) * p.N + t.q + 4 * g) * HW +
                     (size_t)i * p.W + j;
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
      const float send1 = m2 ? s1[c] : s1[c + 4];
      const float send2 = m2 ? s2[c] : s2[c + 4];
      a1[c] = (m2 ? s1[c + 4] : s1[c]) + __shfl_xor_sync(kFull, send1, 2);
      a2[c] = (m2 ? s2[c + 4] : s2[c]) + __shfl_xor_sync(kFull, send2, 2);
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
      for (int e = 0; e < 2; ++e) {
        vx[e] = fmaf(pick(dl, m2, m1, e), f1[e], Dd * pick(gy, m2, m1, e));
        vd[e] = fmaf(pick(xv, m2, m1, e), f1[e], f2[e]);
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
  }
#pragma unroll
  for (int g = 0; g < NG; ++g)
    if (t.act && nok[g]) atomicAdd(p.dA + (size_t)t.d * p.N + t.q + 4 * g, dAacc[g]);
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
  if (flags & SCAN2D_VFIRST) return SCAN2D_E_FLAGS;
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
  const unsigned long long cr = static_cast<unsigned long long>(batch) * channels * H * S * N;
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
  size_t hsave, cf, cb, beta, accx, accd, total;
};

WsLayout ws_layout(const BwdShape& s) {
  WsLayout l{};
  size_t off = 0;
  l.hsave = off; off += round256(s.xy * s.N * sizeof(float));
  l.cf = off;    off += round256(s.carries * sizeof(float));
  l.cb = off;    off += round256(s.carries * sizeof(float));
  l.beta = off;  off += round256(s.carries * sizeof(float));
  const bool acc = !s.out_f32 && s.K > 1;    // bf16 outputs summed over orientations in fp32
  l.accx = off;  off += acc ? round256(s.xy * sizeof(float)) : 0;
  l.accd = off;  off += acc ? round256(s.xy * sizeof(float)) : 0;
  l.total = off;
  return l;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <typename Tin, typename Tg, int NG>
int launch_orientation(const Args& a, bool fw, cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>((a.tasks + kWarps - 1) / kWarps);
  const long long threads = (long long)a.batch * a.channels * a.H * a.N;
  const unsigned cblocks = static_cast<unsigned>((threads + 255) / 256);
  if (fw) k_pre<Tin, Tg, NG, true><<<blocks, kWarps * 32, 0, st>>>(a);
  else k_pre<Tin, Tg, NG, false><<<blocks, kWarps * 32, 0, st>>>(a);
  k_carry<<<cblocks, 256, 0, st>>>(a, fw ? 1 : 0);
  if (fw) k_states<Tin, NG, true><<<blocks, kWarps * 32, 0, st>>>(a);
  else k_states<Tin, NG, false><<<blocks, kWarps * 32, 0, st>>>(a);
  if (fw) k_main<Tin, Tg, NG, true><<<blocks, kWarps * 32, 0, st>>>(a);
  else k_main<Tin, Tg, NG, false><<<blocks, kWarps * 32, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? SCAN2D_OK : SCAN2D_E_LAUNCH;
}

template <typename Tin, typename Tg>
int launch_ng(const Args& a, bool fw, cudaStream_t st) {
  if (a.N <= 4) return launch_orientation<Tin, Tg, 1>(a, fw, st);
  if (a.N <= 8) return launch_orientation<Tin, Tg, 2>(a, fw, st);
  return launch_orientation<Tin, Tg, 4>(a, fw, st);
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
  a.cf = reinterpret_cast<float*>(ws + l.cf);
  a.cb = reinterpret_cast<float*>(ws + l.cb);
  a.beta = reinterpret_cast<float*>(ws + l.beta);
  a.batch = batch; a.channels = channels; a.H = H; a.W = W; a.N = N; a.K = s.K; a.S = s.S;
  a.ncg = s.ncg;
  a.tasks = (long long)batch * s.S * s.ncg;
  const size_t row_in = (size_t)W * s.in_elem, row_out = (size_t)W * s.out_elem;
  a.vec_in = row_in % 16 == 0 && aligned(x, 16) && aligned(delta, 16) && aligned(B, 16) && aligned(C, 16);
  a.vec_g = row_out % 16 == 0 && aligned(dy, 16);
  a.vec_h = W % 4 == 0;
  a.vec2 = W % 2 == 0 && aligned(dx, 2 * s.out_elem) && aligned(ddelta, 2 * s.out_elem) &&
           aligned(dB, 8) && aligned(dC, 8);

  int k = 0;
  for (int o = 0; o < 4; ++o) {
    if (!((s.orient >> o) & 1u)) continue;
    a.k = k;
    a.flipH = (o >> 1) & 1;
    a.first = k == 0;
    a.last = k == s.K - 1;
    const bool fw = (o & 1) != 0;
    if (!s.bf16) rc = launch_ng<float, float>(a, fw, st);
    else if (s.out_f32) rc = launch_ng<uint16_t, float>(a, fw, st);
    else rc = launch_ng<uint16_t, uint16_t>(a, fw, st);
    if (rc) return rc;
    ++k;
  }
  return SCAN2D_OK;
}

}  // extern "C"
