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
//     G*NG updates.
//   * lane = (channel group cg = lane>>2) x (state group q = lane&3); lane q holds states
//     n = q, q+4, q+8, ...; a warp covers 8*G channels and a strip of CMAX columns.
//   * Everything but the horizontal recurrence is done on pairs of adjacent columns with
//     packed f32x2 instructions (adjacent columns are adjacent in shared memory, so the
//     pairs need no repacking).
//   * A warp walks all rows of its strip in scan order.  The vertical state of every
//     (column, channel, state) it owns stays in registers for the whole walk, so the
//     vertical scan needs no communication.
//   * The horizontal scan crosses strips.  Warps are not lock-stepped: the carry (the row's
//     last hh) goes to the next strip's warp through a small shared-memory ring guarded by
//     full/empty mbarriers.  The blocks of one chain form a thread-block cluster and the
//     last warp of a block writes straight into the next block's ring (distributed shared
//     memory, remote mbarrier arrive), so no compute warp ever waits on a global-memory
//     fence.  Chains longer than a cluster fall back to a ring in global memory whose
//     8-byte words carry a row tag beside each value (relaxed loads and stores, no flags or
//     fences; blocks take their place from a ticket counter, so a block only waits on
//     blocks that started before it).  Every wait is bounded in time.
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
constexpr int kRing = 16;              // carry rows buffered in global memory between blocks
constexpr int kCarryRing = 4;          // carry rows buffered in shared memory between warps
constexpr int kMaxWarps = 8;           // warps per block, except for split orientations
constexpr int kMaxWarpsSplit = 16;     // warps per block when two chains split the orientations
constexpr int kTileRows = 4;           // rows per staged tile (TMA path; the plain path stages 1)
constexpr int kTileDepth = 2;          // staged tiles in flight per warp (TMA path)
constexpr int kPublish = 4;            // global fallback: rows per flag release
constexpr float kLog2e = 1.4426950408889634f;

enum Mode : int {
  kSingle = 0,       // one orientation: y = acc + D x
  kSmemMulti = 1,    // every orientation inside the block, fp32 partial sums in shared memory
  kGlobalFirst = 2,  // first of several launches: yacc = acc + D x
  kGlobalMid = 3,    // yacc += acc
  kGlobalLast = 4,   // y = yacc + acc
};

enum Link : int {
  kLinkNone = 0,     // one block per chain
  kLinkCluster = 1,  // the chain's blocks form a cluster; carries through distributed smem
  kLinkGlobal = 2,   // carries through a ring in global memory
};

struct Params {
  const void* x;            // the map x, or with cell_patch the bag of patch features (npatch, channels)
  const int* cell_patch;    // null, or (H*W): the bag row at each cell, -1 for a non-tissue cell
  const void* pad;          // with cell_patch: the non-tissue token (channels)
  int npatch;               // with cell_patch: rows of the bag (other cell entries read pad)
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
  int link;                 // Link
  int orient_count;         // orientations handled by this launch
  int orient_code[4];       // orientation number (bit0 = flip W, bit1 = flip H)
  int orient_k[4];          // index of the orientation's B_k, C_k
  int mode;
  int yacc_stride;          // kSmemMulti: floats per channel in shared memory
  int orient_split;         // kSmemMulti: 2 when the block's two chain slots walk every other
                            // orientation of the same channels (else 1)
  int vec_store;            // rows of y are aligned for 4-column vector stores
  int out_f32;              // y is fp32 (else bf16)
  unsigned long long* ctrl;   // [0] ticket counter, [1] finished blocks, [2] aborted generation
  unsigned long long* acks;   // [n_chains*nseg] rows consumed by a segment (tagged)
  unsigned long long* carry;  // [n_chains*nseg][kRing][32][CARRY2] tagged carry words
  unsigned long long gen;     // launch generation, tags acks and carry words
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

// Global carry ring: every word is (tag << 32) | float bits, written and read as single
// 8-byte accesses, so a word is valid exactly when its tag is the one expected and no flag
// (with the fence it would need) guards the ring.  The tag is the low 20 bits of the launch
// generation and the low 12 bits of row + 1; the host zeroes the ring before the
// generation's low 20 bits wrap, and a slot is only ever refilled kRing rows later.
__device__ __forceinline__ unsigned ctag(unsigned long long gen, int r) {
  return (static_cast<unsigned>(gen & 0xFFFFFull) << 12) | (static_cast<unsigned>(r + 1) & 0xFFFu);
}

__device__ __forceinline__ unsigned long long ld_relaxed(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__device__ __forceinline__ void st_relaxed_v2(unsigned long long* p, unsigned long long a, unsigned long long b) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

__device__ __forceinline__ void ld_relaxed_v2(const unsigned long long* p, unsigned long long& a,
                                              unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned cluster_rank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the same shared-memory location in block `rank` of the cluster
__device__ __forceinline__ uint32_t map_rank(uint32_t local, unsigned rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Relaxed arrive on another block's mbarrier: orders nothing, so it never waits for this
// thread's outstanding global stores.  Used to free a carry slot once its values are in use.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// Arms this block's mbarrier for `bytes` of st.async data (arrive + expect_tx, relaxed).
__device__ __forceinline__ void mbar_arm_tx(uint32_t bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 16 bytes into another block's shared memory; their arrival completes `bytes` of the
// transaction count of that block's mbarrier `cluster_bar` (no arrive, no fence).
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d, uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];"
               ::"r"(addr), "r"(__float_as_uint(a)), "r"(__float_as_uint(b)), "r"(__float_as_uint(c)),
               "r"(__float_as_uint(d)), "r"(cluster_bar)
               : "memory");
}

// One try of phase `parity` of an mbarrier of this block; true once the phase has completed.
// CTA scope: every mbarrier waited on is this block's own, and the data it guards arrives
// either by this block's stores (release.cta arrives), by TMA or by st.async (both signalled
// through the barrier's transaction count).
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
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

// The four copies of one staged tile (x, delta, B, C boxes) and the arming of their mbarrier,
// issued by one lane chosen with elect.sync.  Called by every lane of a converged warp, so the
// operands are warp-uniform and no lane waits in a divergent branch.
__device__ __forceinline__ void tma_tile4(uint32_t bar, uint32_t dx, uint32_t dd, uint32_t db, uint32_t dc,
                                          const CUtensorMap* mx, const CUtensorMap* md, const CUtensorMap* mb,
                                          const CUtensorMap* mc, int col, int ch, int row, int bx, int bk,
                                          unsigned tx_bytes) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "@p mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %14;\n\t"
      "@p cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%1], [%5, {%9, %10, %11, %12}], [%0];\n\t"
      "@p cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%2], [%6, {%9, %10, %11, %12}], [%0];\n\t"
      "@p cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%3], [%7, {%9, %15, %11, %13}], [%0];\n\t"
      "@p cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%4], [%8, {%9, %15, %11, %13}], [%0];\n\t"
      "}" ::"r"(bar), "r"(dx), "r"(dd), "r"(db), "r"(dc),
      "l"(reinterpret_cast<uint64_t>(mx)), "l"(reinterpret_cast<uint64_t>(md)), "l"(reinterpret_cast<uint64_t>(mb)),
      "l"(reinterpret_cast<uint64_t>(mc)), "r"(col), "r"(ch), "r"(row), "r"(bx), "r"(bk), "r"(tx_bytes), "r"(0)
      : "memory");
}

// Records a device error once and marks this launch generation aborted: every other wait of
// the launch then gives up at once (checked through ctrl[2] where a ctrl block exists).
__device__ __noinline__ void report_timeout(unsigned long long* ctrl, unsigned long long gen) {
  atomicCAS(&g_device_error, 0, SCAN2D_E_TIMEOUT);
  if (ctrl != nullptr) st_release(&ctrl[2], gen);
}

// Bounded wait (one lane) until *p >= want.  False on time-out or when the launch is aborted.
__device__ __noinline__ bool wait_geq(const unsigned long long* p, unsigned long long want,
                                      unsigned long long* ctrl, unsigned long long gen,
                                      long long timeout_ns) {
  long long t0 = -1;
  for (unsigned it = 1;; ++it) {
    if (ld_acquire(p) >= want) return true;
    if ((it & 31u) == 0u) {
      if (ld_acquire(&ctrl[2]) == gen) return false;
      const long long now = global_ns();
      if (t0 < 0) t0 = now;
      else if (now - t0 > timeout_ns || it > (1u << 30)) {
        report_timeout(ctrl, gen);
        return false;
      }
    }
    __nanosleep(64);
  }
}

// Slow path of a bounded mbarrier wait: keeps trying until phase `parity` completes or the
// time runs out.  Returns false after a time-out (the error is recorded).
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, unsigned parity, unsigned long long* ctrl,
                                            unsigned long long gen, long long timeout_ns) {
  // the clock is read only every 64 tries (most waits end well before the first read)
  long long t0 = -1;
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      const long long now = global_ns();
      if (t0 < 0) t0 = now;
      else if (now - t0 > timeout_ns || it > (1u << 28)) {
        report_timeout(ctrl, gen);
        return false;
      }
    }
  }
}

// Bounded wait for phase `parity` of an mbarrier (TMA completion or a carry ring slot): one
// try inline, the rest out of line.  Once a wait of this warp has timed out (`aborted`),
// later waits return at once.  Returns the new `aborted`.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, unsigned parity, unsigned long long* ctrl,
                                          unsigned long long gen, long long timeout_ns, bool aborted) {
  if (aborted || mbar_try_wait(bar, parity)) return aborted;
  return !mbar_wait_slow(bar, parity, ctrl, gen, timeout_ns);
}

// ---- staged-row element access ------------------------------------------------------------
// A 16-byte vector holds 4 fp32 or 8 bf16 values of consecutive columns; pair(v, p) returns
// columns 2p and 2p+1 of it as a float2.
template <typename Tin> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerVec = 4;
  static __device__ __forceinline__ float2 pair(const uint4& v, int p) {
    return p == 0 ? make_float2(__uint_as_float(v.x), __uint_as_float(v.y))
                  : make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
};
template <> struct Elem<uint16_t> {
  static constexpr int kPerVec = 8;
  static __device__ __forceinline__ float2 pair(const uint4& v, int p) {
    const unsigned w = p == 0 ? v.x : (p == 1 ? v.y : (p == 2 ? v.z : v.w));
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
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

// ---- shared memory of one block ---------------------------------------------------------------
template <typename Tin, int NG, int G, int CMAX, int R = 1>
struct Layout {
  static constexpr int ESZ = static_cast<int>(sizeof(Tin));
  static constexpr int CPW = kGroups * G;                    // channels per warp
  static constexpr int NB = kQ * NG;                         // states covered by the 4 q lanes
  static constexpr int X_ROW = CPW * CMAX;                   // elements of one row: [CPW][CMAX]
  static constexpr int B_ROW = NB * CMAX;                    // [NB][CMAX]
  static constexpr int X_BYTES = R * X_ROW * ESZ;            // R rows: [R][CPW][CMAX]
  static constexpr int B_BYTES = R * B_ROW * ESZ;            // [R][NB][CMAX]
  static constexpr int r128(int v) { return (v + 127) / 128 * 128; }
  // one staged tile of R strip rows; every region starts on a 128-byte boundary (TMA
  // destinations)
  static constexpr int X_OFF = 0;                                        // element offsets
  static constexpr int D_OFF = r128(X_BYTES) / ESZ;
  static constexpr int B_OFF = D_OFF + r128(X_BYTES) / ESZ;
  static constexpr int C_OFF = B_OFF + r128(B_BYTES) / ESZ;
  static constexpr int TILE_BYTES = (C_OFF * ESZ) + r128(B_BYTES);
  static constexpr int TX_BYTES = 2 * X_BYTES + 2 * B_BYTES;
  static constexpr int DENSE = (2 * CPW + 2 * NB) * CMAX;    // values of one row without padding
  static constexpr int PLAIN_PER_LANE = DENSE / 32;          // plain-load path: values per lane
  static constexpr int CARRY = G * NG;                       // carry floats per lane
  static constexpr int CARRY_PAD = (CARRY + 3) / 4 * 4;      // ... padded to whole float4s
  static constexpr int CARRY2 = (CARRY + 1) / 2 * 2;         // tagged words per lane (global ring)
  static constexpr int CARRY_SLOT_BYTES = 32 * CARRY_PAD * 4;  // one carry row of a warp
  static constexpr int E = CMAX * G;                         // partial outputs per lane per row
  static constexpr int NP = CMAX / 2;                        // column pairs per strip
};

// Dynamic shared memory, in this order (all offsets multiples of 128 bytes):
//   carry rings   [warps][kCarryRing] carry rows          (incoming carries of each warp)
//   tile rings    [warps][depth] staged strip rows
//   accumulator   [chains_per_block][CPW][yacc_stride] floats (kSmemMulti only)
template <typename Tin, int NG, int G, int CMAX>
__host__ __device__ constexpr size_t carry_ring_bytes(int warps) {
  return static_cast<size_t>(warps) * kCarryRing * Layout<Tin, NG, G, CMAX>::CARRY_SLOT_BYTES;
}

// ---- the kernel ------------------------------------------------------------------------------
template <typename Tin, int NG, int G, int CMAX, bool TMA, int MAXW = kMaxWarps, bool VF = false, bool GX = false>
__global__ void __launch_bounds__(MAXW * 32, 1)
scan2d_kernel(const __grid_constant__ Params p, const __grid_constant__ TmaMaps tm) {
  constexpr int R = TMA ? kTileRows : 1;                     // rows per staged tile
  using L = Layout<Tin, NG, G, CMAX, R>;
  constexpr int PV = Elem<Tin>::kPerVec;
  static_assert(CMAX % PV == 0, "strip width must hold whole 16-byte vectors");
  static_assert(L::E % 4 == 0, "reduce-scatter needs 4 | CMAX*G");
  static_assert(L::DENSE % 32 == 0, "plain-load path needs 32 | tile values");
  constexpr int DEPTH = TMA ? kTileDepth : 1;
  constexpr int NVEC = CMAX / PV;                            // 16-byte vectors per strip row
  constexpr int E = L::E;
  constexpr int NP = L::NP;

  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ uint64_t s_tfull[MAXW][kTileDepth];             // staged tile landed (TMA)
  __shared__ uint64_t s_full[MAXW][kCarryRing];              // carry slot written (consumer side)
  __shared__ uint64_t s_empty[MAXW][kCarryRing];             // carry slot read (producer side)
  __shared__ int s_item;

  const unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  // every warp computes (and stages its own rows)
  const int ncomp = p.wpc * p.chains_per_block;
  const bool is_compute = warp < ncomp;
  const int slot = is_compute ? warp / p.wpc : 0;            // chain slot inside the block
  // Warp k runs on sub-partition k % 4 of the SM.  With one chain of 8 strips per block, the
  // two warps of a sub-partition take adjacent strips (strip s on warp s/2 + 4 (s % 2)): a warp
  // then computes while its partner waits for the carry it is about to hand over, instead of
  // both computing (or both waiting) at the same time.
  const bool pair_map = MAXW == kMaxWarps && p.wpc == 8 && p.chains_per_block == 1;
  auto warp_of = [&](int ws) { return pair_map ? (ws >> 1) + 4 * (ws & 1) : slot * p.wpc + ws; };
  const int w = is_compute ? (pair_map ? 2 * (warp & 3) + (warp >> 2) : warp - slot * p.wpc) : 0;  // strip
  const int next_warp = warp_of(w + 1);                      // warps of the neighbouring strips
  const int prev_warp = warp_of(w - 1);
  const int cg = lane >> 2;                 // channel group
  const int q = lane & 3;                   // state group
  const bool cluster = p.link == kLinkCluster;
  const bool global_link = p.link == kLinkGlobal;

  // ---- which chain and segment -------------------------------------------------------
  if (threadIdx.x == 0) {
    if (global_link) s_item = static_cast<int>(atomicAdd(&p.ctrl[0], 1ull));
  }
  __syncthreads();
  const int seg = cluster ? static_cast<int>(cluster_rank()) : (global_link ? s_item % p.nseg : 0);
  // chain of chain slot `sl` of this block
  auto chain_of = [&](int sl) -> int {
    if (cluster) return blockIdx.x / p.nseg;
    if (global_link) return s_item / p.nseg;
    if (p.orient_split > 1) return blockIdx.x;               // the slots share the channels
    return blockIdx.x * p.chains_per_block + sl;
  };
  const int chain = chain_of(slot);
  const bool chain_ok = is_compute && chain < p.n_chains && slot < p.chains_per_block;
  const int b = chain_ok ? chain / p.n_cgroups : 0;
  const int grp = chain_ok ? chain - b * p.n_cgroups : 0;
  const int u_scan = seg * p.wpc + w;                        // strip position in scan order
  const bool strip_ok = chain_ok && u_scan < p.strips;       // warp-uniform
  // does the next strip of the chain exist (and who owns it)?
  const bool next_local = strip_ok && w < p.wpc - 1 && u_scan + 1 < p.strips;
  const bool next_remote = strip_ok && w == p.wpc - 1 && seg < p.nseg - 1 && u_scan + 1 < p.strips;
  const bool has_left = strip_ok && u_scan > 0;              // a carry comes in
  const bool left_global = has_left && w == 0 && global_link;
  const bool left_remote = has_left && w == 0 && cluster;    // carry comes from the previous block

  const int H = p.H, W = p.W, N = p.N;
  const size_t HW = static_cast<size_t>(H) * W;
  const int ch0 = grp * L::CPW + cg * G;                     // first channel of this lane

  // per-lane constants: A * log2(e) per (channel, state) as a splat pair, Dskip per channel
  float2 A2[G][NG];
  float2 Dd[G];
#pragma unroll
  for (int c = 0; c < G; ++c) {
    const int d = ch0 + c;
    const bool dok = chain_ok && d < p.channels;
    const float dv = (dok && p.Dskip != nullptr) ? __ldg(p.Dskip + d) : 0.f;
    Dd[c] = make_float2(dv, dv);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const int n = q + kQ * g;
      const float a = (dok && n < N) ? __ldg(p.A + static_cast<size_t>(d) * N + n) * kLog2e : 0.f;
      A2[c][g] = make_float2(a, a);
    }
  }

  // ---- shared memory ---------------------------------------------------------------------
  unsigned char* carry_base = smem;
  unsigned char* tiles0 = smem + carry_ring_bytes<Tin, NG, G, CMAX>(ncomp);
  unsigned char* tiles = tiles0 + (is_compute ? warp : 0) * DEPTH * L::TILE_BYTES;
  float* yacc_s = reinterpret_cast<float*>(tiles0 + static_cast<size_t>(ncomp) * DEPTH * L::TILE_BYTES);
  const int yslot = p.orient_split > 1 ? 0 : slot;           // accumulator of this warp's chain
  if (p.mode == kSmemMulti) {
    // the orientations add into the accumulator (in any order, from any warp): start at zero
    const int ny = (p.orient_split > 1 ? 1 : p.chains_per_block) * L::CPW * p.yacc_stride;
    for (int e = threadIdx.x; e < ny; e += blockDim.x) yacc_s[e] = 0.f;
  }
  auto carry_slot = [&](int wr, int s) -> float* {
    return reinterpret_cast<float*>(carry_base + (wr * kCarryRing + s) * L::CARRY_SLOT_BYTES);
  };

  if (lane == 0 && is_compute) {
#pragma unroll
    for (int s = 0; s < DEPTH; ++s) {
      mbar_init(&s_tfull[warp][s], 1);        // the elected lane's expect_tx arrival + the bytes
    }
#pragma unroll
    for (int s = 0; s < kCarryRing; ++s) {
      // a carry from another block arrives by st.async: this warp arms the slot itself
      mbar_init(&s_full[warp][s], left_remote ? 1 : 32);
      mbar_init(&s_empty[warp][s], 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (left_remote)
#pragma unroll
      for (int s = 0; s < kCarryRing; ++s) mbar_arm_tx(smem_u32(&s_full[warp][s]), L::CARRY_SLOT_BYTES);
  }
  if (cluster) cluster_sync();      // every block's barriers exist before any remote arrive
  else __syncthreads();

  const int item = chain * p.nseg + seg;
  // orientations this warp walks: all of them, or every other one when two chains split them
  const int ostep = p.orient_split > 1 ? p.orient_split : 1;
  const int oi_first = ostep > 1 ? slot : 0;
  const int n_or = oi_first < p.orient_count ? (p.orient_count - oi_first + ostep - 1) / ostep : 0;
  const int U = n_or * H;                                    // rows each warp walks

  // row uu of the walk of the warp at scan position us -> (orientation, stored row, stored strip)
  auto row_coords_of = [&](int us, int uu, int& oi, int& i, int& t) {
    const int oj = uu / H;
    const int r = uu - oj * H;
    oi = oi_first + oj * ostep;
    const int o = p.orient_code[oi];
    i = (o & 2) ? H - 1 - r : r;
    t = (o & 1) ? p.strips - 1 - us : us;
  };
  auto row_coords = [&](int uu, int& oi, int& i, int& t) { row_coords_of(u_scan, uu, oi, i, t); };

  // plain-load path: this lane's share of row u's tile, zero outside the tensors.  Value e
  // of the dense tile goes to tile offset plain_dst(e).
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
            if (GX && region == 0) {                      // GX: x read from a bag
              // x read from the bag through the cell map (one map, b = 0)
              const int kp = __ldg(p.cell_patch + static_cast<size_t>(i) * W + col);
              val = load_raw((kp >= 0 && kp < p.npatch
                                  ? static_cast<const Tin*>(p.x) + static_cast<size_t>(kp) * p.channels
                                  : static_cast<const Tin*>(p.pad)) + d);
            } else {
              const Tin* src = static_cast<const Tin*>(region == 0 ? p.x : p.delta);
              val = load_raw(src + (static_cast<size_t>(b) * p.channels + d) * HW + static_cast<size_t>(i) * W + col);
            }
          }
        } else if (rr < N) {
          const Tin* src = static_cast<const Tin*>(region == 2 ? p.B : p.C);
          val = load_raw(src + ((static_cast<size_t>(b) * p.K + k) * N + rr) * HW + static_cast<size_t>(i) * W + col);
        }
      }
      pre[m] = val;
    }
  };

  bool aborted = false;
  if (!TMA && strip_ok) plain_load(0);

  // ---- TMA: the warp stages the tiles of its walk, DEPTH tiles ahead (one elected lane issues) ---
  // A tile is R consecutive scan rows of one orientation (the last one may reach past the map:
  // TMA fills those rows with zeros).  Walk tile wt goes to slot wt % DEPTH; the warp refills
  // a slot right after all its lanes have read the tile's last row.  Once a wait of this warp
  // has given up, nothing more is staged.
  const int TPO = (H + R - 1) / R;                           // tiles per orientation
  const int UT = n_or * TPO;                                 // tiles of the walk
  int staged = 0;                                            // tiles of the walk staged so far
  // the next tile to stage, as (orientation, tile in it), with that orientation's stored strip
  // column, flip and B/C index (every lane keeps the same copy)
  int st_oi = oi_first, st_tr = 0, st_col = 0, st_flip = 0, st_bk = 0;
  auto st_orientation = [&]() {
    const int o = p.orient_code[st_oi];
    st_flip = o & 2;
    st_col = ((o & 1) ? p.strips - 1 - u_scan : u_scan) * CMAX;
    st_bk = b * p.K + p.orient_k[st_oi];
  };
  auto stage_tile = [&]() {                                  // whole warp, converged: walk tile `staged`
    const int row0 = st_flip ? H - R - st_tr * R : st_tr * R;  // first stored row of the box
    const int s = staged % DEPTH;
    const uint32_t dst = smem_u32(tiles + s * L::TILE_BYTES);
    tma_tile4(smem_u32(&s_tfull[warp][s]), dst + L::X_OFF * L::ESZ, dst + L::D_OFF * L::ESZ,
              dst + L::B_OFF * L::ESZ, dst + L::C_OFF * L::ESZ, &tm.x, &tm.d, &tm.b, &tm.c, st_col,
              grp * L::CPW, row0, b, st_bk, L::TX_BYTES);
    if (++st_tr == TPO) {
      st_tr = 0;
      if ((st_oi += ostep) < p.orient_count) st_orientation();
    }
  };
  if (TMA && strip_ok) {
    const int first = UT < DEPTH ? UT : DEPTH;
    st_orientation();
    for (; staged < first; ++staged) stage_tile();
  }

  // where this warp's carries go: the next warp of this block, or warp 0 of the next block
  const uint32_t next_full0 = smem_u32(&s_full[next_local ? next_warp : 0][0]);
  const uint32_t my_empty0 = smem_u32(&s_empty[warp][0]);
  uint32_t next_ring_cl = 0, next_full_cl = 0, prev_empty_cl = 0;
  if (cluster) {
    if (next_remote) {
      next_ring_cl = map_rank(smem_u32(carry_slot(0, 0)), seg + 1);
      next_full_cl = map_rank(smem_u32(&s_full[0][0]), seg + 1);
    }
    if (left_remote) prev_empty_cl = map_rank(smem_u32(&s_empty[warp_of(p.wpc - 1)][0]), seg - 1);
  }

  // global ring, consumer side: this lane's tagged words of the row it will need next
  unsigned long long cw[L::CARRY2];
  auto cw_load = [&](int uu) {
    const unsigned long long* src =
        p.carry + ((static_cast<size_t>(item - 1) * kRing + (uu % kRing)) * 32 + lane) * L::CARRY2;
#pragma unroll
    for (int k = 0; k < L::CARRY2 / 2; ++k) ld_relaxed_v2(src + 2 * k, cw[2 * k], cw[2 * k + 1]);
  };
  auto cw_ready = [&](unsigned want) {
    bool ok = true;
#pragma unroll
    for (int e = 0; e < L::CARRY; ++e) ok = ok && static_cast<unsigned>(cw[e] >> 32) == want;
    return ok;
  };
  // reloads row uu until every tag is right; true if it gave up (time-out or aborted launch)
  auto cw_poll = [&](int uu) -> bool {
    const unsigned want = ctag(p.gen, uu);
    long long t0 = -1;
    for (unsigned it = 1;; ++it) {
      if (cw_ready(want)) return false;
      __nanosleep(32);
      if ((it & 15u) == 0u) {
        if (ld_acquire(&p.ctrl[2]) == p.gen) return true;
        const long long now = global_ns();
        if (t0 < 0) t0 = now;
        else if (now - t0 > p.timeout_ns || it > (1u << 26)) {
          report_timeout(p.ctrl, p.gen);
          return true;
        }
      }
      cw_load(uu);
    }
  };

  unsigned long long ack_seen = 0;                           // global ring: last ack read
  int u = 0;                                                 // rows of the walk done so far
  for (int oj = 0; oj < n_or; ++oj) {
    const int oi = oi_first + oj * ostep;
    const int o = p.orient_code[oi];
    const bool flipW = (o & 1) != 0, flipH = (o & 2) != 0;
    const int t = flipW ? p.strips - 1 - u_scan : u_scan;   // stored strip
    const int col0 = t * CMAX;
    const bool add_dx = (p.mode == kSingle || p.mode == kGlobalFirst || (p.mode == kSmemMulti && oi == 0));

    float2 v[NP][G][NG];                                     // vertical state, column pairs
#pragma unroll
    for (int pp = 0; pp < NP; ++pp)
#pragma unroll
      for (int c = 0; c < G; ++c)
#pragma unroll
        for (int g = 0; g < NG; ++g) v[pp][c][g] = make_float2(0.f, 0.f);

    if (left_global && strip_ok) {
      // start two rows behind the upstream block, so that the words of the next row are
      // already published when this warp requests them one row ahead
      const int u1 = u + 1 < U ? u + 1 : u;
      cw_load(u1);
      if (!aborted) aborted = cw_poll(u1);
      cw_load(u);
    }

    // row outputs are written one row late: the reduction of row r over the 4 state-group
    // lanes is issued together with the math of row r + 1, so the two overlap
    float2 pacc[NP][G];                                      // partial outputs of the pending row
#pragma unroll
    for (int pp = 0; pp < NP; ++pp)
#pragma unroll
      for (int c = 0; c < G; ++c) pacc[pp][c] = make_float2(0.f, 0.f);
    int p_i = -1;                                            // stored row of the pending row

    // reduce-scatter over the 4 state-group lanes of a channel group: lane q keeps the q-th
    // quarter of the flat index e = c*CMAX + j (channel-major, j = stored column in the strip)
    auto reduce_row = [&](const float2 (&ac)[NP][G], float (&own)[E / 4]) {
      float flat[E];
#pragma unroll
      for (int c = 0; c < G; ++c)
#pragma unroll
        for (int pp = 0; pp < NP; ++pp) {
          flat[c * CMAX + 2 * pp] = ac[pp][c].x;
          flat[c * CMAX + 2 * pp + 1] = ac[pp][c].y;
        }
      float r1[E / 2];
      const bool hi2 = (q & 2) != 0, hi1 = (q & 1) != 0;
#pragma unroll
      for (int e = 0; e < E / 2; ++e) {
        const float lo = flat[e], hi = flat[e + E / 2];
        r1[e] = (hi2 ? hi : lo) + __shfl_xor_sync(FULL, hi2 ? lo : hi, 2);
      }
#pragma unroll
      for (int e = 0; e < E / 4; ++e) {
        const float lo = r1[e], hi = r1[e + E / 4];
        own[e] = (hi1 ? hi : lo) + __shfl_xor_sync(FULL, hi1 ? lo : hi, 1);
      }
    };
    // output of stored row i_row: channel c, columns j0 .. j0 + E/4 - 1 of the strip
    auto write_row = [&](int i_row, const float (&own)[E / 4]) {
      const int e0 = q * (E / 4);
      const int c = e0 / CMAX;
      const int j0 = e0 - c * CMAX;
      const int d = ch0 + c;
      if (d >= p.channels) return;
      const size_t rowoff = (static_cast<size_t>(b) * p.channels + d) * HW + static_cast<size_t>(i_row) * W;
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
        float* a = yacc_s + (yslot * L::CPW + cg * G + c) * p.yacc_stride + i_row * W + gc;
#pragma unroll
        for (int m = 0; m < E / 4; ++m)
          if (gc + m < W) atomicAdd(a + m, own[m]);
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
    };

    for (int r = 0; r < H && strip_ok; ++r, ++u) {
      const int i = flipH ? H - 1 - r : r;
      const int tr = r / R, rr = r - tr * R;                 // tile of the orientation, row in it
      const int wt = oj * TPO + tr;                          // tile of the walk
      const int s = wt % DEPTH;
      const int rt = flipH ? R - 1 - rr : rr;                // this row's place in the staged tile
      const Tin* tile = reinterpret_cast<const Tin*>(tiles + s * L::TILE_BYTES);
      const int cs = u % kCarryRing;                         // carry ring slot of this row
      const unsigned cpar = static_cast<unsigned>((u / kCarryRing) & 1);

      // ---- (1) this row's tile is in shared memory -----------------------------------
      if (TMA) {
        if (rr == 0)
          aborted = mbar_wait(smem_u32(&s_tfull[warp][s]), static_cast<unsigned>((wt / DEPTH) & 1), p.ctrl,
                              p.gen, p.timeout_ns, aborted);
      } else {
        Tin* dst = reinterpret_cast<Tin*>(tiles);
#pragma unroll
        for (int m = 0; m < L::PLAIN_PER_LANE; ++m) dst[plain_dst(lane + 32 * m)] = pre[m];
        __syncwarp();
        if (u + 1 < U) plain_load(u + 1);
      }

      // ---- (2) carry-in: hh at the column before this strip (scan order) ----------------
      float hh[G][NG];
      if (left_global) {
        // this row's words were requested one row ago; every tag must be this row's
        if (!aborted) aborted = cw_poll(u);
#pragma unroll
        for (int c = 0; c < G; ++c)
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[c][g] = __uint_as_float(static_cast<unsigned>(cw[c * NG + g]));
        if (u + 1 < U) cw_load(u + 1);
      } else if (has_left) {
        aborted = mbar_wait(smem_u32(&s_full[warp][cs]), cpar, p.ctrl, p.gen, p.timeout_ns, aborted);
        const float4* src = reinterpret_cast<const float4*>(carry_slot(warp, cs)) + lane * (L::CARRY_PAD / 4);
        float in[L::CARRY_PAD];
#pragma unroll
        for (int k4 = 0; k4 < L::CARRY_PAD / 4; ++k4) {
          const float4 f = src[k4];
          in[4 * k4] = f.x;
          in[4 * k4 + 1] = f.y;
          in[4 * k4 + 2] = f.z;
          in[4 * k4 + 3] = f.w;
        }
#pragma unroll
        for (int c = 0; c < G; ++c)
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[c][g] = in[c * NG + g];
        // free the slot (a slot filled from another block is freed once its values are used)
        if (!left_remote) mbar_arrive_local(smem_u32(&s_empty[prev_warp][cs]));
      } else {
#pragma unroll
        for (int c = 0; c < G; ++c)
#pragma unroll
          for (int g = 0; g < NG; ++g) hh[c][g] = 0.f;
      }

      // ---- (3) the strip's columns of this row, two adjacent columns at a time -------------
      float2 acc[NP][G];
      // vf: vertical-first order.  The carried chain is then the second (horizontal) scan of
      // the vertical state, and the output contracts that chain's state.
      auto vec_group = [&](int vg, bool rev, bool vf) {
        uint4 xv[G], dv[G], bv[NG], cv[NG];
#pragma unroll
        for (int c = 0; c < G; ++c) {
          xv[c] = *reinterpret_cast<const uint4*>(tile + L::X_OFF + rt * L::X_ROW + (cg * G + c) * CMAX + vg * PV);
          dv[c] = *reinterpret_cast<const uint4*>(tile + L::D_OFF + rt * L::X_ROW + (cg * G + c) * CMAX + vg * PV);
        }
#pragma unroll
        for (int g = 0; g < NG; ++g) {
          bv[g] = *reinterpret_cast<const uint4*>(tile + L::B_OFF + rt * L::B_ROW + (q + kQ * g) * CMAX + vg * PV);
          cv[g] = *reinterpret_cast<const uint4*>(tile + L::C_OFF + rt * L::B_ROW + (q + kQ * g) * CMAX + vg * PV);
        }
#pragma unroll
        for (int k = 0; k < PV / 2; ++k) {
          const int kp = rev ? PV / 2 - 1 - k : k;           // pair inside the vector
          const int pp = vg * (PV / 2) + kp;                 // pair inside the strip
#pragma unroll
          for (int c = 0; c < G; ++c) {
            const float2 x2 = Elem<Tin>::pair(xv[c], kp);
            const float2 d2 = Elem<Tin>::pair(dv[c], kp);
            const float2 dx = __fmul2_rn(d2, x2);
            float2 a_acc = (add_dx && q == 0) ? __fmul2_rn(Dd[c], x2) : make_float2(0.f, 0.f);
#pragma unroll
            for (int g = 0; g < NG; ++g) {
              const float2 arg = __fmul2_rn(d2, A2[c][g]);
              const float2 a = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
              const float2 uu = __fmul2_rn(dx, Elem<Tin>::pair(bv[g], kp));
              if (vf) v[pp][c][g] = __ffma2_rn(a, v[pp][c][g], uu);          // vertical first
              const float2 in2 = vf ? v[pp][c][g] : uu;                       // input of the chain
              float2 h2;
              if (!rev) {
                h2.x = fmaf(a.x, hh[c][g], in2.x);
                h2.y = fmaf(a.y, h2.x, in2.y);
                hh[c][g] = h2.y;
              } else {
                h2.y = fmaf(a.y, hh[c][g], in2.y);
                h2.x = fmaf(a.x, h2.y, in2.x);
                hh[c][g] = h2.x;
              }
              if (!vf) v[pp][c][g] = __ffma2_rn(a, v[pp][c][g], h2);         // then vertical
              a_acc = __ffma2_rn(Elem<Tin>::pair(cv[g], kp), vf ? h2 : v[pp][c][g], a_acc);
            }
            acc[pp][c] = a_acc;
          }
        }
      };
      float own_prev[E / 4];                                 // the pending row, reduced
      if (!flipW) {
        reduce_row(pacc, own_prev);
#pragma unroll
        for (int vg = 0; vg < NVEC; ++vg) vec_group(vg, false, VF);
      } else {
        reduce_row(pacc, own_prev);
#pragma unroll
        for (int vg = NVEC - 1; vg >= 0; --vg) vec_group(vg, true, VF);
      }

      // ---- (4) carry-out to the next strip, as early as possible -----------------------------
      if (next_local || (next_remote && cluster)) {
        // the slot is free once the consumer released its previous use
        if (u >= kCarryRing)
          aborted = mbar_wait(my_empty0 + cs * 8, cpar ^ 1u, p.ctrl, p.gen, p.timeout_ns, aborted);
        float out[L::CARRY_PAD];
#pragma unroll
        for (int e = L::CARRY; e < L::CARRY_PAD; ++e) out[e] = 0.f;
#pragma unroll
        for (int c = 0; c < G; ++c)
#pragma unroll
          for (int g = 0; g < NG; ++g) out[c * NG + g] = hh[c][g];
        if (next_local) {
          float4* dst = reinterpret_cast<float4*>(carry_slot(next_warp, cs)) + lane * (L::CARRY_PAD / 4);
#pragma unroll
          for (int k4 = 0; k4 < L::CARRY_PAD / 4; ++k4)
            dst[k4] = make_float4(out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3]);
          mbar_arrive_local(next_full0 + cs * 8);
        } else {
          // st.async into the next block's slot: the bytes complete its full barrier
          const uint32_t dst = next_ring_cl + cs * L::CARRY_SLOT_BYTES + lane * L::CARRY_PAD * 4;
#pragma unroll
          for (int k4 = 0; k4 < L::CARRY_PAD / 4; ++k4)
            st_async_v4(dst + 16 * k4, out[4 * k4], out[4 * k4 + 1], out[4 * k4 + 2], out[4 * k4 + 3],
                        next_full_cl + cs * 8);
        }
      } else if (next_remote && global_link) {
        if (u >= kRing && (u % kPublish) == 0) {
          // rows up to u - kRing must have been consumed before their slots are reused; the
          // ack read kPublish rows ago usually shows that already, else wait for it (bounded)
          const unsigned long long want = tag(p.gen, u - kRing + kPublish);
          if (ack_seen < want) {
            if (lane == 0) wait_geq(&p.acks[item + 1], want, p.ctrl, p.gen, p.timeout_ns);
            __syncwarp();
          }
          ack_seen = ld_relaxed(&p.acks[item + 1]);           // for the next check, not waited on
        }
        // tagged words, no fence: the consumer checks every word's tag
        unsigned long long* dst = p.carry + ((static_cast<size_t>(item) * kRing + (u % kRing)) * 32 + lane) * L::CARRY2;
        const unsigned long long t = static_cast<unsigned long long>(ctag(p.gen, u)) << 32;
        float out[L::CARRY2];
        out[L::CARRY2 - 1] = 0.f;
#pragma unroll
        for (int c = 0; c < G; ++c)
#pragma unroll
          for (int g = 0; g < NG; ++g) out[c * NG + g] = hh[c][g];
#pragma unroll
        for (int k = 0; k < L::CARRY2 / 2; ++k)
          st_relaxed_v2(dst + 2 * k, t | __float_as_uint(out[2 * k]), t | __float_as_uint(out[2 * k + 1]));
      }
      // consumed rows, every kPublish rows (the words read so far are in use already)
      if (left_global && ((u + 1) % kPublish == 0 || u == U - 1)) {
        __syncwarp();
        if (lane == 0) st_relaxed(&p.acks[item], tag(p.gen, u + 1));
      }

      // ---- (5) refill the tile slot (every lane has read the tile's last row) ---------------
      // a wait that gave up on one lane gives up for the warp: the refill below is issued by
      // the converged warp
      __syncwarp();
      aborted = __any_sync(FULL, aborted);
      if (TMA && (rr == R - 1 || r == H - 1) && !aborted && staged < UT) {
        // every lane has read the tile's last row (its values are in use): refill the slot
        stage_tile();
        ++staged;
      }
      // a carry slot filled by the previous block: re-arm it for its next use, then free it;
      // both are relaxed, so they never wait for this warp's outstanding stores of y
      if (left_remote) {
        if (lane == 0) mbar_arm_tx(smem_u32(&s_full[warp][cs]), L::CARRY_SLOT_BYTES);
        mbar_arrive_remote_relaxed(prev_empty_cl + cs * 8);
      }

      // ---- (6) the previous row's output (its reduction was interleaved with this row's math) --
      if (p_i >= 0) write_row(p_i, own_prev);
#pragma unroll
      for (int pp = 0; pp < NP; ++pp)
#pragma unroll
        for (int c = 0; c < G; ++c) pacc[pp][c] = acc[pp][c];
      p_i = i;
    }
    // the orientation's last row
    if (p_i >= 0) {
      float own_last[E / 4];
      reduce_row(pacc, own_last);
      write_row(p_i, own_last);
    }
  }
  // ---- after a timed-out wait: let this warp's copies still in flight land (bounded) -------
  if (TMA && aborted && lane == 0) {
    bool gave_up = false;
    for (int wt = staged - DEPTH < 0 ? 0 : staged - DEPTH; wt < staged; ++wt)
      gave_up = mbar_wait(smem_u32(&s_tfull[warp][wt % DEPTH]), static_cast<unsigned>((wt / DEPTH) & 1),
                          p.ctrl, p.gen, p.timeout_ns, gave_up);
  }
  __syncthreads();

  // ---- kSmemMulti: write the accumulated maps of this block's chains --------------------------
  if (p.mode == kSmemMulti && chain_ok) {
    // every warp of the chain (both slots when they split the orientations) writes a share
    const int nthreads = (p.orient_split > 1 ? ncomp : p.wpc) * 32;
    const int tid = (p.orient_split > 1 ? warp : w) * 32 + lane;
    for (int cs = 0; cs < L::CPW; ++cs) {
      const int dd = grp * L::CPW + cs;
      if (dd >= p.channels) break;
      const float* src = yacc_s + (yslot * L::CPW + cs) * p.yacc_stride;
      const size_t base = (static_cast<size_t>(b) * p.channels + dd) * HW;
      for (size_t e = tid; e < HW; e += nthreads) store_out(p.y, base + e, src[e], p.out_f32);
    }
  }

  // ---- leave together: a cluster's shared memory must outlive the remote arrives into it ----
  if (cluster) cluster_sync();

  // ---- the last block of a ticketed launch resets the counters for the next launch ----------
  if (global_link) {
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
