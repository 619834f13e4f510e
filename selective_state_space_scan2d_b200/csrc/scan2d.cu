// scan2d.cu -- C ABI of the 2D selective-scan forward: argument checks, work planning,
// tensor maps, per-(device, stream) workspace, kernel dispatch.  The arithmetic is in
// scan2d_kernels.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "../../include/scan2d.h"
#include "scan2d_kernels.cuh"

namespace scan2d {

namespace {

constexpr long long kTimeoutNs = 2000000000LL;   // bounded inter-block waits: 2 s
constexpr size_t kAlign = 256;
constexpr size_t kSmemBudget = 200 * 1024;       // dynamic shared memory per block we plan for
constexpr size_t kSmemBudgetSplit = 220 * 1024;  // ... for blocks whose chains split the orientations

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int popcount4(unsigned v) { return ((v >> 0) & 1) + ((v >> 1) & 1) + ((v >> 2) & 1) + ((v >> 3) & 1); }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

struct Shape {
  int batch, channels, H, W, N, K;
  bool bf16, out_f32;
  bool vfirst;                 // vertical scan first (SCAN2D_VFIRST)
  unsigned orient;             // 4-bit orientation mask
  size_t in_elem, out_elem;    // bytes per element of x/delta/B/C and of y
  size_t xy_count, bc_count;   // elements of x (= y) and of B (= C)
};

int check_shape(int batch, int channels, int H, int W, int N, unsigned flags, Shape* s) {
  if (flags & ~SCAN2D_FLAGS_KNOWN) return SCAN2D_E_FLAGS;
  if ((flags & SCAN2D_OUT_F32) && !(flags & SCAN2D_BF16)) return SCAN2D_E_FLAGS;
  if (batch < 1 || channels < 1 || H < 1 || W < 1) return SCAN2D_E_DIMS;
  if (N < 1 || N > SCAN2D_MAX_N) return SCAN2D_E_N;
  const unsigned long long hw = static_cast<unsigned long long>(H) * W;
  if (hw > (1ull << 31) - 1) return SCAN2D_E_DIMS;                 // in-map offsets are int
  unsigned orient = (flags >> 4) & 0xFu;
  if (orient == 0) orient = 1;                                       // default: top-left
  const int K = popcount4(orient);
  const unsigned long long xy = static_cast<unsigned long long>(batch) * channels * hw;
  const unsigned long long bc = static_cast<unsigned long long>(batch) * K * N * hw;
  if (xy > (1ull << 40) || bc > (1ull << 40)) return SCAN2D_E_DIMS;
  s->batch = batch; s->channels = channels; s->H = H; s->W = W; s->N = N; s->K = K;
  s->bf16 = (flags & SCAN2D_BF16) != 0;
  s->out_f32 = !s->bf16 || (flags & SCAN2D_OUT_F32) != 0;
  s->vfirst = (flags & SCAN2D_VFIRST) != 0;
  s->orient = orient;
  s->in_elem = s->bf16 ? 2 : 4;
  s->out_elem = s->out_f32 ? 4 : 2;
  s->xy_count = static_cast<size_t>(xy);
  s->bc_count = static_cast<size_t>(bc);
  return SCAN2D_OK;
}

// ---- kernel variants ------------------------------------------------------------------------
using KernelFn = void (*)(const Params, const TmaMaps);

struct Variant {
  int ng, g, cmax;            // states per lane, channels per lane, strip width
  size_t tile_bytes_tma;      // one staged tile of kTileRows strip rows (TMA path)
  size_t tile_bytes_plain;    // one staged strip row (plain-load path)
  size_t carry_slot_bytes;    // one carry row of a warp
  // [scan order: 0 horizontal first, 1 vertical first]
  KernelFn fn_tma[2], fn_plain[2];
  KernelFn fn_tma16[2], fn_plain16[2];   // up to 16 warps per block (one channel per lane only)
  KernelFn fn_plain_gx[2], fn_plain16_gx[2];   // plain staging with x read from a bag of patches
};

template <typename Tin, int NG, int G, int CMAX>
Variant make_variant() {
  using LT = Layout<Tin, NG, G, CMAX, kTileRows>;
  using LP = Layout<Tin, NG, G, CMAX, 1>;
  Variant v{NG, G, CMAX, static_cast<size_t>(LT::TILE_BYTES), static_cast<size_t>(LP::TILE_BYTES),
            static_cast<size_t>(LP::CARRY_SLOT_BYTES),
            {scan2d_kernel<Tin, NG, G, CMAX, true, kMaxWarps, false>, scan2d_kernel<Tin, NG, G, CMAX, true, kMaxWarps, true>},
            {scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarps, false>, scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarps, true>},
            {nullptr, nullptr}, {nullptr, nullptr},
            {scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarps, false, true>,
             scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarps, true, true>},
            {nullptr, nullptr}};
  if constexpr (G == 1) {
    v.fn_tma16[0] = scan2d_kernel<Tin, NG, G, CMAX, true, kMaxWarpsSplit, false>;
    v.fn_tma16[1] = scan2d_kernel<Tin, NG, G, CMAX, true, kMaxWarpsSplit, true>;
    v.fn_plain16[0] = scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarpsSplit, false>;
    v.fn_plain16[1] = scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarpsSplit, true>;
    v.fn_plain16_gx[0] = scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarpsSplit, false, true>;
    v.fn_plain16_gx[1] = scan2d_kernel<Tin, NG, G, CMAX, false, kMaxWarpsSplit, true, true>;
  }
  return v;
}

int states_per_lane(int N) {
  int ng = 1;
  while (ng * kQ < N) ng *= 2;
  return ng;                       // 1, 2, 4, 8 or 16 for N <= 64
}

// G = 2 channels per lane (packed f32x2) unless the block keeps a whole-map accumulator in
// shared memory (G = 1 halves it) or the lane already holds 16 states.
template <typename Tin>
Variant pick_variant_t(int ng, bool g1) {
  constexpr bool kF32 = sizeof(Tin) == 4;
  switch (ng) {
    case 1: return g1 ? make_variant<Tin, 1, 1, 8>() : make_variant<Tin, 1, 2, 8>();
    case 2: return g1 ? make_variant<Tin, 2, 1, 8>() : make_variant<Tin, 2, 2, 8>();
    case 4: return g1 ? make_variant<Tin, 4, 1, 8>() : make_variant<Tin, 4, 2, 8>();
    case 8:
      if constexpr (kF32) return g1 ? make_variant<Tin, 8, 1, 4>() : make_variant<Tin, 8, 2, 4>();
      else
      return make_variant<Tin, 8, 1, 8>();
    default:
      if constexpr (kF32) return make_variant<Tin, 16, 1, 4>();
      else
      return make_variant<Tin, 16, 1, 8>();
  }
}

Variant pick_variant(const Shape& s, int ng, bool g1) {
  return s.bf16 ? pick_variant_t<uint16_t>(ng, g1) : pick_variant_t<float>(ng, g1);
}

// ---- work plan ---------------------------------------------------------------------------
struct Plan {
  Variant var;
  int cpw, strips, wpc, nseg, chains_per_block, n_cgroups, n_chains, warps;
  size_t carry_smem, tile_smem;   // carry rings and tile rings of all warps of a block
};

constexpr int kMaxCluster = 16;   // blocks of a chain that can share distributed shared memory

Plan make_plan(const Shape& s, int ng, bool g1, bool tma) {
  Plan pl{};
  pl.var = pick_variant(s, ng, g1);
  pl.cpw = kGroups * pl.var.g;
  pl.n_cgroups = (s.channels + pl.cpw - 1) / pl.cpw;
  pl.n_chains = s.batch * pl.n_cgroups;
  pl.strips = (s.W + pl.var.cmax - 1) / pl.var.cmax;
  if (pl.strips <= kMaxWarps) {
    pl.wpc = pl.strips;
    pl.nseg = 1;
    pl.chains_per_block = kMaxWarps / pl.wpc;
  } else {
    pl.wpc = kMaxWarps;
    pl.nseg = (pl.strips + kMaxWarps - 1) / kMaxWarps;
    pl.chains_per_block = 1;
  }
  pl.warps = pl.wpc * pl.chains_per_block;
  pl.carry_smem = static_cast<size_t>(pl.warps) * kCarryRing * pl.var.carry_slot_bytes;
  pl.tile_smem = static_cast<size_t>(pl.warps) * (tma ? kTileDepth * pl.var.tile_bytes_tma : pl.var.tile_bytes_plain);
  return pl;
}

// ---- tensor maps (cuTensorMapEncodeTiled through the runtime's driver entry point) -----------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 4-D map of a dense (d3, d2, H, W) tensor, with dimensions listed as (W, d2, H, d3), so that a
// (cmax, box2, kTileRows, 1) box lands in shared memory as kTileRows consecutive [box2][cmax]
// row tiles.
bool encode_map(CUtensorMap* m, const void* base, bool bf16, int W, int H, long long d2,
                long long d3, int cmax, int box2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const size_t e = bf16 ? 2 : 4;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(d2),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(d3)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(W) * H * e,
                                 static_cast<cuuint64_t>(W) * e,
                                 static_cast<cuuint64_t>(W) * H * e * d2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(cmax), static_cast<cuuint32_t>(box2),
                             static_cast<cuuint32_t>(kTileRows), 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// TMA needs 16-byte aligned bases and row strides (W * element) that are multiples of 16 B.
bool tma_possible(const Shape& s, const void* x, const void* delta, const void* B, const void* C) {
  if ((static_cast<size_t>(s.W) * s.in_elem) % 16 != 0) return false;
  return aligned(x, 16) && aligned(delta, 16) && aligned(B, 16) && aligned(C, 16);
}

// ---- per-(device, stream) workspace --------------------------------------------------------
// Layout: [control words: 256 B][acks: cap_items u64][carry ring: carry_cap bytes of tagged
// words][fp32 accumulator ...].  The ack and carry regions keep their place and size for the
// life of the allocation and only ever hold generation-tagged words, so a later call of
// another shape can never take an earlier call's data for its own.  The workspace is
// reallocated, zeroed, when a call needs more than it holds, and its tagged regions are
// zeroed again before the 20 generation bits of the carry tags wrap.
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
  size_t cap_items = 0;
  size_t carry_cap = 0;
  unsigned long long gen = 0;
};

std::mutex g_mu;
std::map<std::pair<int, cudaStream_t>, Workspace> g_ws;

size_t sync_bytes(size_t items) { return kAlign + round_up(items * 8, kAlign); }

// A workspace whose ack region holds `items` items, whose carry region holds `carry` bytes
// and whose tail after them holds `tail` bytes, zero-initialised when (re)created, or null.
Workspace* get_workspace(int dev, cudaStream_t st, size_t items, size_t carry, size_t tail) {
  std::lock_guard<std::mutex> lk(g_mu);
  Workspace& ws = g_ws[std::make_pair(dev, st)];
  if (ws.cap_items < items || ws.carry_cap < carry || ws.bytes < sync_bytes(ws.cap_items) + ws.carry_cap + tail) {
    size_t cap = ws.cap_items, ccap = ws.carry_cap;
    if (cap < items) cap = items > 2 * cap ? items : 2 * cap;
    if (ccap < carry) ccap = carry > 2 * ccap ? carry : 2 * ccap;
    if (ws.ptr != nullptr) {
      if (cudaStreamSynchronize(st) != cudaSuccess) return nullptr;
      cudaFree(ws.ptr);
      ws = Workspace{};
    }
    const size_t want = round_up(sync_bytes(cap) + ccap + tail, 1 << 20);
    if (cudaMalloc(&ws.ptr, want) != cudaSuccess) {
      cudaGetLastError();
      ws = Workspace{};
      return nullptr;
    }
    if (cudaMemsetAsync(ws.ptr, 0, want, st) != cudaSuccess) {
      cudaFree(ws.ptr);
      ws = Workspace{};
      return nullptr;
    }
    ws.bytes = want;
    ws.cap_items = cap;
    ws.carry_cap = ccap;
    ws.gen = 0;
  }
  return &ws;
}

int device_ok(int* dev, int* nsm) {
  if (cudaGetDevice(dev) != cudaSuccess) { cudaGetLastError(); return SCAN2D_E_DEVICE; }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
      cudaDeviceGetAttribute(nsm, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_DEVICE;
  }
  if (major != 10) return SCAN2D_E_DEVICE;
  return SCAN2D_OK;
}

// Everything a call of this shape launches, without touching memory.
struct CallPlan {
  Plan pl;
  bool tma;
  int codes[4], nk;
  bool smem_multi, global_multi, need_yacc_ws, need_ws;
  int link, yacc_stride, grid, launches;
  int orient_split;            // 2: two chain slots per block walk every other orientation
  size_t smem, items, carry_bytes, yacc_bytes, ws_bytes;
};

// Blocks a plan launches per launch.
int plan_blocks(const Plan& pl) {
  return pl.nseg > 1 ? pl.n_chains * pl.nseg : (pl.n_chains + pl.chains_per_block - 1) / pl.chains_per_block;
}

// `nsm`: streaming multiprocessors of the device the plan is for (148 on a B200).
CallPlan plan_call(const Shape& s, bool tma, bool cluster_ok, int nsm) {
  CallPlan cp{};
  cp.tma = tma;
  cp.orient_split = 1;
  const int ng = states_per_lane(s.N);
  cp.nk = 0;
  for (int o = 0; o < 4; ++o)
    if (s.orient & (1u << o)) cp.codes[cp.nk++] = o;

  // several orientations: sum them in a shared-memory accumulator when a block can hold
  // whole maps of its channels (G = 1 channel per lane keeps it small); otherwise one
  // launch per orientation with an fp32 accumulator in global memory.
  const size_t HW = static_cast<size_t>(s.H) * s.W;
  cp.smem_multi = false;
  if (s.K > 1 && HW <= (1u << 20)) {
    Plan p1 = make_plan(s, ng, true, tma);
    const int stride = static_cast<int>(round_up(HW, 32) + 4);        // +4: spread the banks
    if (p1.nseg == 1) {
      const size_t per_chain = sizeof(float) * p1.cpw * stride +
                               (p1.tile_smem + p1.carry_smem) / p1.chains_per_block;
      int cpb = p1.chains_per_block;
      while (cpb > 1 && per_chain * cpb > kSmemBudget) --cpb;
      // one chain per block: let a second chain slot walk every other orientation of the same
      // channels at the same time (twice the warps, half the walk), if that still fits
      const size_t split_smem = sizeof(float) * p1.cpw * stride + 2 * (p1.tile_smem + p1.carry_smem);
      // (up to 4 states per lane: the 16-warp variants get 128 registers a thread)
      if (p1.chains_per_block == 1 && 2 * p1.wpc <= kMaxWarpsSplit && split_smem <= kSmemBudgetSplit &&
          p1.var.fn_tma16[0] != nullptr && ng <= 4) {
        p1.tile_smem *= 2;
        p1.carry_smem *= 2;
        p1.chains_per_block = 2;
        p1.warps = 2 * p1.wpc;
        cp.pl = p1;
        cp.smem_multi = true;
        cp.orient_split = 2;
        cp.yacc_stride = stride;
        cp.smem = split_smem;
      } else if (per_chain * cpb <= kSmemBudget) {
        p1.tile_smem = p1.tile_smem / p1.chains_per_block * cpb;
        p1.carry_smem = p1.carry_smem / p1.chains_per_block * cpb;
        p1.chains_per_block = cpb;
        p1.warps = p1.wpc * cpb;
        cp.pl = p1;
        cp.smem_multi = true;
        cp.yacc_stride = stride;
        cp.smem = per_chain * cpb;
      }
    }
  }
  if (!cp.smem_multi) {
    cp.pl = make_plan(s, ng, ng >= 16, tma);
    // two channels per lane share the B, C loads, but halve the number of chains: when that
    // leaves most multiprocessors idle (few channels, e.g. batch 1 with a small map), one
    // channel per lane and twice the chains is faster
    if (plan_blocks(cp.pl) * 2 <= nsm) cp.pl = make_plan(s, ng, true, tma);
    cp.yacc_stride = 0;
    cp.smem = cp.pl.carry_smem + cp.pl.tile_smem;
  }
  const Plan& pl = cp.pl;
  cp.link = pl.nseg == 1 ? kLinkNone : (cluster_ok && pl.nseg <= kMaxCluster ? kLinkCluster : kLinkGlobal);
  cp.global_multi = s.K > 1 && !cp.smem_multi;
  cp.need_yacc_ws = cp.global_multi && !s.out_f32;
  cp.items = static_cast<size_t>(pl.n_chains) * pl.nseg;
  const size_t carry2 = (static_cast<size_t>(pl.var.g) * pl.var.ng + 1) / 2 * 2;   // tagged words per lane
  cp.carry_bytes = cp.link == kLinkGlobal ? round_up(cp.items * kRing * 32 * carry2 * 8, kAlign) : 0;
  cp.yacc_bytes = cp.need_yacc_ws ? s.xy_count * sizeof(float) : 0;
  cp.need_ws = cp.link == kLinkGlobal || cp.need_yacc_ws;
  cp.ws_bytes = cp.need_ws ? sync_bytes(cp.link == kLinkGlobal ? cp.items : 0) + cp.carry_bytes + cp.yacc_bytes : 0;
  cp.grid = cp.orient_split > 1 ? pl.n_chains : plan_blocks(pl);
  cp.launches = cp.global_multi ? cp.nk : 1;
  return cp;
}

// Raises the kernel's dynamic shared-memory limit when it needs more than the default 48 KB
// (before occupancy queries and launches).
bool allow_smem(KernelFn fn, size_t smem) {
  // static shared memory (barriers) counts against the same 48 KB default
  if (smem + 4096 <= 48 * 1024) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return true;
}

int launch(KernelFn fn, int threads, const Params& prm, const TmaMaps& tm, size_t smem, int grid,
           int cluster, cudaStream_t st) {
  if (!allow_smem(fn, smem)) return SCAN2D_E_LAUNCH;
  if (cluster <= 1) {
    fn<<<grid, threads, smem, st>>>(prm, tm);
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, prm, tm) != cudaSuccess) {
      cudaGetLastError();
      return SCAN2D_E_LAUNCH;
    }
  }
  if (cudaGetLastError() != cudaSuccess) return SCAN2D_E_LAUNCH;
  return SCAN2D_OK;
}

// Can clusters of `nseg` blocks of this kernel be resident at all on this device?
// How many clusters of `nseg` blocks of this kernel can be resident at once (0 if none).
// Cached per (kernel, threads, shared memory, cluster size): the query is not free.
int clusters_resident(KernelFn fn, int threads, size_t smem, int nseg) {
  if (nseg > kMaxCluster) return 0;
  static std::mutex mu;
  static std::map<std::pair<std::pair<const void*, int>, std::pair<size_t, int>>, int> cache;
  const auto key = std::make_pair(std::make_pair(reinterpret_cast<const void*>(fn), threads), std::make_pair(smem, nseg));
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int n = 0;
  if (allow_smem(fn, smem) &&
      (nseg <= 8 || cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nseg, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nseg;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  std::lock_guard<std::mutex> lk(mu);
  cache[key] = n;
  return n;
}

// Clusters are used when they fit and the last wave of clusters is not mostly empty: the
// blocks of a chain run at the pace of its slowest block, so a partial wave costs a whole one.
bool cluster_worth_it(KernelFn fn, int threads, size_t smem, int nseg, int chains) {
  const int n = clusters_resident(fn, threads, smem, nseg);
  if (n <= 0) return false;
  const long long waves = (chains + n - 1) / n;
  return waves == 1 || chains * 100 >= waves * n * 85;   // one wave, or >= 85% of the slots busy
}

// `fixed_scratch`, when given, is the device address of a buffer of
// SCAN2D_NOALLOC_SCRATCH_BYTES that replaces the per-stream workspace (nothing is allocated).
// `cell_patch`, when given, makes x a bag of patch features read through that cell map (one
// map, batch 1), with `pad` at the cells that hold no patch; such calls stage by plain loads.
int forward(const void* x, const void* delta, const float* A, const void* B, const void* C,
            const float* Dskip, void* y, int batch, int channels, int H, int W, int N,
            unsigned flags, cudaStream_t st, char* fixed_scratch = nullptr,
            const int* cell_patch = nullptr, const void* pad = nullptr, int npatch = 0) {
  Shape s;
  int rc = check_shape(batch, channels, H, W, N, flags, &s);
  if (rc) return rc;
  if (!x || !delta || !A || !B || !C || !y) return SCAN2D_E_NULL;
  if (!aligned(x, s.in_elem) || !aligned(delta, s.in_elem) || !aligned(B, s.in_elem) ||
      !aligned(C, s.in_elem) || !aligned(A, 4) || !aligned(Dskip, 4) || !aligned(y, s.out_elem))
    return SCAN2D_E_ALIGN;
  int dev = 0, nsm = 0;
  rc = device_ok(&dev, &nsm);
  if (rc) return rc;

  // tensor maps when the layout allows TMA, else the plain-load variant
  TmaMaps tm;
  std::memset(&tm, 0, sizeof tm);
  bool tma = cell_patch == nullptr && tma_possible(s, x, delta, B, C);
  CallPlan cp = plan_call(s, tma, true, nsm);
  if (tma) {
    const Plan& p0 = cp.pl;
    const int nb = kQ * p0.var.ng;
    tma = encode_map(&tm.x, x, s.bf16, W, H, channels, batch, p0.var.cmax, p0.cpw) &&
          encode_map(&tm.d, delta, s.bf16, W, H, channels, batch, p0.var.cmax, p0.cpw) &&
          encode_map(&tm.b, B, s.bf16, W, H, N, static_cast<long long>(batch) * s.K, p0.var.cmax, nb) &&
          encode_map(&tm.c, C, s.bf16, W, H, N, static_cast<long long>(batch) * s.K, p0.var.cmax, nb);
    if (!tma) cp = plan_call(s, false, true, nsm);
  }
  // a chain's blocks share distributed shared memory when such a cluster fits on the device
  if (cp.link == kLinkCluster &&
      !cluster_worth_it(tma ? cp.pl.var.fn_tma[s.vfirst ? 1 : 0] : cp.pl.var.fn_plain[s.vfirst ? 1 : 0], cp.pl.warps * 32, cp.smem, cp.pl.nseg,
                        cp.pl.n_chains))
    cp = plan_call(s, tma, false, nsm);
  const Plan& pl = cp.pl;
  const int vf = s.vfirst ? 1 : 0;
  const bool gx = cell_patch != nullptr;
  const KernelFn fn = cp.orient_split > 1
                          ? (tma ? pl.var.fn_tma16[vf] : (gx ? pl.var.fn_plain16_gx[vf] : pl.var.fn_plain16[vf]))
                          : (tma ? pl.var.fn_tma[vf] : (gx ? pl.var.fn_plain_gx[vf] : pl.var.fn_plain[vf]));

  Params prm;
  std::memset(&prm, 0, sizeof prm);
  prm.x = x; prm.delta = delta; prm.A = A; prm.B = B; prm.C = C; prm.Dskip = Dskip; prm.y = y;
  prm.cell_patch = cell_patch; prm.pad = pad; prm.npatch = npatch;
  prm.batch = batch; prm.channels = channels; prm.H = H; prm.W = W; prm.N = N; prm.K = s.K;
  prm.n_cgroups = pl.n_cgroups; prm.n_chains = pl.n_chains;
  prm.strips = pl.strips; prm.wpc = pl.wpc; prm.chains_per_block = pl.chains_per_block;
  prm.nseg = pl.nseg;
  prm.link = cp.link;
  prm.timeout_ns = kTimeoutNs;
  prm.yacc_stride = cp.yacc_stride;
  prm.orient_split = cp.orient_split;
  prm.out_f32 = s.out_f32 ? 1 : 0;
  prm.vec_store = (W % 4 == 0) && aligned(y, s.out_f32 ? 16 : 8);

  Workspace* ws = nullptr;
  if (cp.need_ws) {
    if (cp.link == kLinkGlobal) {
      // a chain's blocks must be able to be resident together (producer back-pressure)
      int per_sm = 0;
      if (!allow_smem(fn, cp.smem)) return SCAN2D_E_LAUNCH;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, pl.warps * 32, cp.smem) != cudaSuccess) {
        cudaGetLastError();
        return SCAN2D_E_LAUNCH;
      }
      if (static_cast<long long>(per_sm) * nsm < pl.nseg) return SCAN2D_E_DIMS;
    }
    char* base = nullptr;
    size_t cap = 0, ccap = 0;
    if (fixed_scratch != nullptr) {
      // the fixed buffer keeps the previous call's contents: its control, ack and carry
      // words are cleared for every call, which then starts again at generation 1
      if (cp.ws_bytes > SCAN2D_NOALLOC_SCRATCH_BYTES) return SCAN2D_E_SCRATCH;
      base = fixed_scratch;
      cap = cp.link == kLinkGlobal ? cp.items : 0;
      ccap = cp.carry_bytes;
      if (cudaMemsetAsync(base, 0, sync_bytes(cap) + ccap, st) != cudaSuccess) {
        cudaGetLastError();
        return SCAN2D_E_LAUNCH;
      }
    } else {
      ws = get_workspace(dev, st, cp.link == kLinkGlobal ? cp.items : 0, cp.carry_bytes, cp.yacc_bytes);
      if (!ws) return SCAN2D_E_NOMEM;
      base = static_cast<char*>(ws->ptr);
      cap = ws->cap_items;
      ccap = ws->carry_cap;
    }
    prm.ctrl = reinterpret_cast<unsigned long long*>(base);
    prm.acks = reinterpret_cast<unsigned long long*>(base + kAlign);
    prm.carry = reinterpret_cast<unsigned long long*>(base + sync_bytes(cap));
    if (cp.need_yacc_ws) prm.yacc = reinterpret_cast<float*>(base + sync_bytes(cap) + ccap);
  }
  if (cp.global_multi && s.out_f32) prm.yacc = static_cast<float*>(y);

  // generation of the next launch; before the carry tags' 20 generation bits wrap, the
  // tagged regions are zeroed (in stream order) and generation ...00000 is skipped
  auto next_gen = [&]() -> unsigned long long {
    if (!ws) return 1ull;
    std::lock_guard<std::mutex> lk(g_mu);
    if (((++ws->gen) & 0xFFFFFull) == 0ull) {
      cudaMemsetAsync(static_cast<char*>(ws->ptr) + kAlign, 0, sync_bytes(ws->cap_items) - kAlign + ws->carry_cap, st);
      ++ws->gen;
    }
    return ws->gen;
  };

  const int threads = pl.warps * 32;
  const int cluster = cp.link == kLinkCluster ? pl.nseg : 1;
  if (!cp.global_multi) {
    prm.mode = cp.smem_multi ? kSmemMulti : kSingle;
    prm.orient_count = cp.smem_multi ? cp.nk : 1;
    for (int k = 0; k < prm.orient_count; ++k) { prm.orient_code[k] = cp.codes[k]; prm.orient_k[k] = k; }
    prm.gen = next_gen();
    return launch(fn, threads, prm, tm, cp.smem, cp.grid, cluster, st);
  }
  for (int k = 0; k < cp.nk; ++k) {
    prm.mode = k == 0 ? kGlobalFirst : (k == cp.nk - 1 ? kGlobalLast : kGlobalMid);
    prm.orient_count = 1;
    prm.orient_code[0] = cp.codes[k];
    prm.orient_k[0] = k;
    prm.gen = next_gen();
    rc = launch(fn, threads, prm, tm, cp.smem, cp.grid, cluster, st);
    if (rc) return rc;
  }
  return SCAN2D_OK;
}

// ---- fixed scratch for callers that cannot allocate device memory -------------------------
// One buffer per device, allocated by the CUDA runtime when the library's module is loaded
// and held until the process exits.  Host code must not use the array's name as a device
// address: the address is looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SCAN2D_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
char* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device `dev`, or null.
char* noalloc_scratch(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_noalloc_addr[dev] = static_cast<char*>(p);
  }
  return g_noalloc_addr[dev];
}

}  // namespace scan2d

// ---- C ABI ---------------------------------------------------------------------------------
extern "C" {

int scan2d_fwd(const void* x, const void* delta, const float* A, const void* B, const void* C,
               const float* Dskip, void* y, int batch, int channels, int H, int W, int N,
               unsigned flags, void* stream) {
  return scan2d::forward(x, delta, A, B, C, Dskip, y, batch, channels, H, W, N, flags,
                         static_cast<cudaStream_t>(stream));
}

int scan2d_fwd_noalloc(const void* x, const void* delta, const float* A, const void* B,
                       const void* C, const float* Dskip, void* y, int batch, int channels, int H,
                       int W, int N, unsigned flags, void* stream) {
  scan2d::Shape s;
  int rc = scan2d::check_shape(batch, channels, H, W, N, flags, &s);
  if (rc) return rc;
  if (!x || !delta || !A || !B || !C || !y) return SCAN2D_E_NULL;
  int dev = 0, nsm = 0;
  rc = scan2d::device_ok(&dev, &nsm);
  if (rc) return rc;
  char* scratch = scan2d::noalloc_scratch(dev);
  if (scratch == nullptr) return SCAN2D_E_DEVICE;
  return scan2d::forward(x, delta, A, B, C, Dskip, y, batch, channels, H, W, N, flags,
                         static_cast<cudaStream_t>(stream), scratch);
}

int scan2d_fwd_wsi(const void* feat, const int* cell_patch, const void* pad, const void* delta,
                   const float* A, const void* B, const void* C, const float* Dskip, void* y,
                   int npatch, int channels, int H, int W, int N, unsigned flags, void* stream) {
  scan2d::Shape s;
  int rc = scan2d::check_shape(1, channels, H, W, N, flags, &s);
  if (rc) return rc;
  if (npatch < 0) return SCAN2D_E_DIMS;
  if (!cell_patch || !pad || (npatch > 0 && !feat)) return SCAN2D_E_NULL;
  if (!scan2d::aligned(cell_patch, 4) || !scan2d::aligned(pad, s.in_elem) || !scan2d::aligned(feat, s.in_elem))
    return SCAN2D_E_ALIGN;
  // a bag without patches is read at no address; any aligned pointer stands in for it
  return scan2d::forward(npatch > 0 ? feat : pad, delta, A, B, C, Dskip, y, 1, channels, H, W, N, flags,
                         static_cast<cudaStream_t>(stream), nullptr, cell_patch, pad, npatch);
}

int scan2d_query_plan(int batch, int channels, int H, int W, int N, unsigned flags,
                      long long* out, int n_out) {
  scan2d::Shape s;
  const int rc = scan2d::check_shape(batch, channels, H, W, N, flags, &s);
  if (rc) return rc;
  if (!out) return SCAN2D_E_NULL;
  // the layout decides TMA; with 16-byte aligned buffers only the row stride matters
  const bool tma = (static_cast<size_t>(W) * s.in_elem) % 16 == 0;
  // chains of up to 16 blocks are planned as clusters (the call itself falls back to the
  // global ring if such a cluster cannot be resident on the device)
  const scan2d::CallPlan cp = scan2d::plan_call(s, tma, true, 148);   // planned for a B200
  const long long v[SCAN2D_PLAN_FIELDS] = {
      cp.launches, cp.grid, cp.pl.warps * 32, static_cast<long long>(cp.smem), cp.pl.nseg,
      cp.pl.var.cmax, cp.pl.wpc, cp.smem_multi ? 1 : (cp.global_multi ? 2 : 0), cp.pl.var.ng,
      static_cast<long long>(cp.ws_bytes), cp.pl.var.g, tma ? 1 : 0, cp.link};
  for (int k = 0; k < n_out && k < SCAN2D_PLAN_FIELDS; ++k) out[k] = v[k];
  return SCAN2D_OK;
}

size_t scan2d_host_staging_bytes(int batch, int channels, int H, int W, int N, unsigned flags) {
  scan2d::Shape s;
  if (scan2d::check_shape(batch, channels, H, W, N, flags, &s)) return 0;
  const size_t a = 256;
  auto r = [&](size_t v) { return (v + a - 1) / a * a; };
  return 2 * r(s.xy_count * s.in_elem) + r(static_cast<size_t>(channels) * N * 4) +
         2 * r(s.bc_count * s.in_elem) + r(static_cast<size_t>(channels) * 4) + r(s.xy_count * s.out_elem);
}

int scan2d_fwd_host(const void* x, const void* delta, const float* A, const void* B,
                    const void* C, const float* Dskip, void* y, void* staging,
                    size_t staging_bytes, int batch, int channels, int H, int W, int N,
                    unsigned flags, void* stream) {
  scan2d::Shape s;
  int rc = scan2d::check_shape(batch, channels, H, W, N, flags, &s);
  if (rc) return rc;
  if (!x || !delta || !A || !B || !C || !y || !staging) return SCAN2D_E_NULL;
  const size_t need = scan2d_host_staging_bytes(batch, channels, H, W, N, flags);
  if (staging_bytes < need) return SCAN2D_E_STAGING;
  if (reinterpret_cast<uintptr_t>(staging) % 256) return SCAN2D_E_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t a = 256;
  auto r = [&](size_t v) { return (v + a - 1) / a * a; };
  char* p = static_cast<char*>(staging);
  const size_t bx = s.xy_count * s.in_elem, bA = static_cast<size_t>(channels) * N * 4;
  const size_t bB = s.bc_count * s.in_elem, bD = static_cast<size_t>(channels) * 4;
  const size_t by = s.xy_count * s.out_elem;
  char* dx = p;            p += r(bx);
  char* dd = p;            p += r(bx);
  char* dA = p;            p += r(bA);
  char* dB = p;            p += r(bB);
  char* dC = p;            p += r(bB);
  char* dD = p;            p += r(bD);
  char* dy = p;
  const cudaMemcpyKind h2d = cudaMemcpyHostToDevice;
  if (cudaMemcpyAsync(dx, x, bx, h2d, st) != cudaSuccess ||
      cudaMemcpyAsync(dd, delta, bx, h2d, st) != cudaSuccess ||
      cudaMemcpyAsync(dA, A, bA, h2d, st) != cudaSuccess ||
      cudaMemcpyAsync(dB, B, bB, h2d, st) != cudaSuccess ||
      cudaMemcpyAsync(dC, C, bB, h2d, st) != cudaSuccess ||
      (Dskip && cudaMemcpyAsync(dD, Dskip, bD, h2d, st) != cudaSuccess)) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  rc = scan2d::forward(dx, dd, reinterpret_cast<float*>(dA), dB, dC,
                       Dskip ? reinterpret_cast<float*>(dD) : nullptr, dy, batch, channels, H, W,
                       N, flags, st);
  if (rc) return rc;
  if (cudaMemcpyAsync(y, dy, by, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  return SCAN2D_OK;
}

int scan2d_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  int e = 0;
  if (cudaMemcpyFromSymbol(&e, scan2d::g_device_error, sizeof e) != cudaSuccess) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  if (e != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(scan2d::g_device_error, &zero, sizeof zero);
  }
  return e;
}

const char* scan2d_strerror(int code) {
  switch (code) {
    case SCAN2D_OK: return "ok";
    case SCAN2D_E_NULL: return "a required pointer is NULL";
    case SCAN2D_E_DIMS: return "invalid or too large batch/channels/H/W";
    case SCAN2D_E_N: return "N out of range (1..SCAN2D_MAX_N)";
    case SCAN2D_E_FLAGS: return "unknown or inconsistent flags";
    case SCAN2D_E_ALIGN: return "a pointer is not aligned to its element size";
    case SCAN2D_E_LAUNCH: return "the CUDA runtime rejected a launch or copy";
    case SCAN2D_E_TIMEOUT: return "device: a bounded wait on a neighbouring block timed out";
    case SCAN2D_E_NOMEM: return "workspace allocation failed";
    case SCAN2D_E_DEVICE: return "no usable sm_100 CUDA device";
    case SCAN2D_E_STAGING: return "staging buffer too small";
    case SCAN2D_E_SCRATCH: return "scan2d_fwd_noalloc: the shape needs more scratch than SCAN2D_NOALLOC_SCRATCH_BYTES";
    case SCAN2D_E_WORKSPACE: return "scan2d_bwd: workspace smaller than scan2d_bwd_workspace_bytes";
    default: return "unknown error";
  }
}

int scan2d_version(void) { return 200; }

}  // extern "C"
