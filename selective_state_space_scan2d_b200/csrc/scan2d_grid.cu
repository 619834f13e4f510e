// scan2d_grid.cu -- the 2D map of a whole-slide image from its bag of patch features.
//
// The pages' pipeline ("2DMamba 精读：从小白到博士", section 四.2, the 2DMambaMIL framework,
// steps 3 and 4; papernotes.org notes, "方法详解 / 整体框架" and "关键设计": learnable non-tissue
// padding): patch features are put back on the 2D grid at the patch's position, and every cell
// without a patch holds one learnable non-tissue token p instead of zeros.  Two steps here:
//   scan2d_grid_cells   cell map: cell_patch[i*W + j] = index of the patch at (i, j), or -1;
//   scan2d_grid_gather  x[d, i, j] = feat[cell_patch[i*W + j], d], or p[d] at non-tissue cells.
// The scan can also read x through the cell map without the map being written
// (scan2d_fwd_wsi, in scan2d.cu).
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/scan2d.h"

namespace {

constexpr int kTile = 32;     // cells x channels per gather tile
constexpr int kRowsY = 8;     // thread rows per gather block

// One thread per patch: the patch's cell gets its index; when several patches name one cell
// the highest index wins (atomicMax), so the map does not depend on the order of the writes.
__global__ void __launch_bounds__(256) k_cells(const int* __restrict__ coords, int npatch, int H, int W,
                                               int* __restrict__ cell_patch, int* __restrict__ n_skipped) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= npatch) return;
  const int r = coords[2 * k], c = coords[2 * k + 1];
  if (r >= 0 && r < H && c >= 0 && c < W) {
    atomicMax(cell_patch + (size_t)r * W + c, k);
  } else if (n_skipped != nullptr) {
    atomicAdd(n_skipped, 1);
  }
}

// A tile of 32 consecutive cells (row-major) x 32 channels: read row-wise from the bag (each
// cell's channels are contiguous there), transposed in shared memory, written channel-wise
// (each channel's cells are contiguous in x).  Both global sides move whole 32-element runs.
template <typename T>
__global__ void __launch_bounds__(kTile * kRowsY) k_gather(const T* __restrict__ feat, const int* __restrict__ cell_patch,
                                                          const T* __restrict__ pad, T* __restrict__ x, int npatch,
                                                          int channels, long long cells) {
  __shared__ T tile[kTile][kTile + 1];
  __shared__ int kp[kTile];
  const long long c0 = (long long)blockIdx.x * kTile;
  const int d0 = blockIdx.y * kTile;
  const int tx = threadIdx.x, ty = threadIdx.y;
  if (ty == 0) kp[tx] = c0 + tx < cells ? cell_patch[c0 + tx] : -1;
  __syncthreads();
  const int d = d0 + tx;
#pragma unroll
  for (int m = 0; m < kTile / kRowsY; ++m) {
    const int cc = ty + kRowsY * m;             // cell in the tile
    const int k = kp[cc];
    T v = T(0);
    if (d < channels) v = (k >= 0 && k < npatch) ? feat[(size_t)k * channels + d] : pad[d];
    tile[cc][tx] = v;
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < kTile / kRowsY; ++m) {
    const int dd = d0 + ty + kRowsY * m;        // channel in the tile
    const long long cell = c0 + tx;
    if (dd < channels && cell < cells) x[(size_t)dd * cells + cell] = tile[tx][ty + kRowsY * m];
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

}  // namespace

extern "C" {

int scan2d_grid_cells(const int* coords, int npatch, int H, int W, int* cell_patch, int* n_skipped,
                      void* stream) {
  if (npatch < 0 || H < 1 || W < 1 || static_cast<unsigned long long>(H) * W > (1ull << 31) - 1)
    return SCAN2D_E_DIMS;
  if (!cell_patch || (npatch > 0 && !coords)) return SCAN2D_E_NULL;
  if (!aligned(cell_patch, 4) || !aligned(coords, 4) || !aligned(n_skipped, 4)) return SCAN2D_E_ALIGN;
  if (const int rc = device_ok()) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(cell_patch, 0xFF, (size_t)H * W * sizeof(int), st) != cudaSuccess ||
      (n_skipped && cudaMemsetAsync(n_skipped, 0, sizeof(int), st) != cudaSuccess)) {
    cudaGetLastError();
    return SCAN2D_E_LAUNCH;
  }
  if (npatch > 0) k_cells<<<(npatch + 255) / 256, 256, 0, st>>>(coords, npatch, H, W, cell_patch, n_skipped);
  return cudaGetLastError() == cudaSuccess ? SCAN2D_OK : SCAN2D_E_LAUNCH;
}

int scan2d_grid_gather(const void* feat, const int* cell_patch, const void* pad, void* x, int npatch,
                       int channels, int H, int W, unsigned flags, void* stream) {
  if (flags & ~SCAN2D_BF16) return SCAN2D_E_FLAGS;
  if (npatch < 0 || channels < 1 || H < 1 || W < 1) return SCAN2D_E_DIMS;
  const unsigned long long cells = static_cast<unsigned long long>(H) * W;
  if (cells > (1ull << 31) - 1 || cells * channels > (1ull << 40) || (channels + kTile - 1) / kTile > 65535)
    return SCAN2D_E_DIMS;
  if (!cell_patch || !pad || !x || (npatch > 0 && !feat)) return SCAN2D_E_NULL;
  const size_t el = (flags & SCAN2D_BF16) ? 2 : 4;
  if (!aligned(feat, el) || !aligned(pad, el) || !aligned(x, el) || !aligned(cell_patch, 4)) return SCAN2D_E_ALIGN;
  if (const int rc = device_ok()) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>((cells + kTile - 1) / kTile), static_cast<unsigned>((channels + kTile - 1) / kTile));
  const dim3 block(kTile, kRowsY);
  const long long nc = static_cast<long long>(cells);
  if (el == 2)
    k_gather<uint16_t><<<grid, block, 0, st>>>(static_cast<const uint16_t*>(feat), cell_patch,
                                               static_cast<const uint16_t*>(pad), static_cast<uint16_t*>(x),
                                               npatch, channels, nc);
  else
    k_gather<float><<<grid, block, 0, st>>>(static_cast<const float*>(feat), cell_patch,
                                            static_cast<const float*>(pad), static_cast<float*>(x), npatch,
                                            channels, nc);
  return cudaGetLastError() == cudaSuccess ? SCAN2D_OK : SCAN2D_E_LAUNCH;
}

}  // extern "C"
