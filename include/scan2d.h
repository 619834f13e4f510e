/*
 * scan2d.h -- C ABI of the B200 (sm_100a) 2D selective-scan forward (2DMamba) and its
 * gradients.
 *
 * Operation (sources are web pages on 2DMamba, arXiv 2412.00678):
 *   "2DMamba 精读：从小白到博士" (juejin.cn), section 四.5 "2DMamba 如何扩展到二维？":
 *     (1) horizontal scan   hh[i,j] = Abar[i,j] * hh[i,j-1] + Bbar[i,j] * x[i,j]
 *     (2) vertical scan     h[i,j]  = Abar[i,j] * h[i-1,j]  + hh[i,j]
 *         output            y[i,j]  = C h[i,j]
 *   papernotes.org notes on the CVPR 2025 paper, "关键设计": the hardware-aware operator
 *   keeps the N states on chip and writes only the reduced output, so memory traffic is
 *   O(L) rather than O(N L).
 * For every (b, d) map and state n this library computes, with the same Abar in both scans,
 *   Abar = exp(delta[b,d,i,j] * A[d,n]),   Bbar = delta[b,d,i,j] * B[b,k,n,i,j],
 *   y[b,d,i,j] = sum_k sum_n C[b,k,n,i,j] * h_k[n,i,j] + Dskip[d] * x[b,d,i,j],
 * with zero initial states (hh[i,-1] = 0, h[-1,j] = 0).  The discretisation, the initial
 * states, the skip term and the orientation semantics are not printed on the pages; the
 * plainest readings are taken (see the design notes shipped with the repository).
 *
 * Scan order (papernotes.org notes, "消融实验要点": horizontal-then-vertical and
 * vertical-then-horizontal are both studied).  With SCAN2D_VFIRST the two recurrences run in
 * the other order, with the same Abar, Bbar, C and zero initial states:
 *     vv[i,j] = Abar[i,j] * vv[i-1,j] + Bbar[i,j] * x[i,j]      (vertical first)
 *     h[i,j]  = Abar[i,j] * h[i,j-1]  + vv[i,j]                 (then horizontal)
 * which equals the default order on the transposed map, transposed back.
 *
 * Orientations ("reverse scans" in the papernotes "局限与展望", "四象限" in the juejin
 * section 七.4): orientation TL scans from the top-left corner; TR from the top-right
 * (W reversed); BL from the bottom-left (H reversed); BR from the bottom-right.  Each
 * orientation k has its own B_k, C_k; delta, A and Dskip are shared and Dskip * x is added
 * once.  K = number of orientation bits set (default TL only, K = 1).
 *
 * Layouts: dense, contiguous, row-major with W fastest.
 *   x, delta, y : (batch, channels, H, W)
 *   A           : (channels, N)            fp32
 *   B, C        : (batch, K, N, H, W)      shared by all channels; for K = 1 this is
 *                                          (batch, N, H, W); orientations in bit order
 *                                          TL, TR, BL, BR
 *   Dskip       : (channels)               fp32, may be NULL (then 0)
 * Element types: fp32 by default; with SCAN2D_BF16, x, delta, B, C and y are bf16 (y fp32
 * instead with SCAN2D_OUT_F32).  Arithmetic is fp32 throughout.
 *
 * Ownership: the caller owns every buffer.  scan2d_fwd never frees or retains a caller
 * pointer past the call.  It keeps, per (device, stream), a small internal workspace for
 * cross-block carries (and, for several orientations on maps too large for shared memory
 * with bf16 output, an fp32 accumulator); it is created with cudaMalloc on first need and
 * grown on demand, which synchronises that stream once.  Make a first call of each shape
 * before capturing a stream into a CUDA graph.  Calls on different streams use different
 * workspaces and may run concurrently.
 *
 * Errors: every entry point returns 0 on success or a negative SCAN2D_E_* code, and never
 * aborts or throws.  Argument errors are detected on the host before anything is launched.
 * Device-side failures (a bounded wait for a neighbouring block that ran out) are reported
 * by scan2d_get_device_error() after the work has completed.
 */
#ifndef SCAN2D_H
#define SCAN2D_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- flags ----------------------------------------------------------------------- */
#define SCAN2D_BF16     0x1u   /* x, delta, B, C (and y) are bf16 instead of fp32      */
#define SCAN2D_OUT_F32  0x2u   /* with SCAN2D_BF16: y is fp32                          */
#define SCAN2D_VFIRST   0x8u   /* scan order: vertical scan first, then horizontal      */
#define SCAN2D_OR_TL    0x10u  /* orientation: from the top-left corner (default)     */
#define SCAN2D_OR_TR    0x20u  /* from the top-right corner (W reversed)              */
#define SCAN2D_OR_BL    0x40u  /* from the bottom-left corner (H reversed)            */
#define SCAN2D_OR_BR    0x80u  /* from the bottom-right corner (H and W reversed)     */
#define SCAN2D_OR_ALL   0xF0u
#define SCAN2D_FLAGS_KNOWN 0xFBu

/* ---- limits ---------------------------------------------------------------------- */
#define SCAN2D_MAX_N    64     /* states per channel                                   */
#define SCAN2D_BWD_MAX_N 16    /* states per channel of scan2d_bwd                     */
#define SCAN2D_PROJ_MAX_R 32   /* rank of the delta projection of scan2d_proj           */
#define SCAN2D_NOALLOC_SCRATCH_BYTES 33554432  /* fixed scratch of scan2d_fwd_noalloc (32 MiB) */

/* ---- error codes ----------------------------------------------------------------- */
#define SCAN2D_OK          0
#define SCAN2D_E_NULL     -1   /* a required pointer is NULL                            */
#define SCAN2D_E_DIMS     -2   /* batch, channels, H or W < 1, or a size overflows      */
#define SCAN2D_E_N        -3   /* N < 1 or N > SCAN2D_MAX_N                             */
#define SCAN2D_E_FLAGS    -4   /* unknown flag bits, or SCAN2D_OUT_F32 without BF16     */
#define SCAN2D_E_ALIGN    -5   /* a pointer is not aligned to its element size          */
#define SCAN2D_E_LAUNCH   -6   /* the CUDA runtime rejected a launch or a copy          */
#define SCAN2D_E_TIMEOUT  -7   /* device: a bounded wait on a neighbouring block gave up */
#define SCAN2D_E_NOMEM    -8   /* the internal workspace could not be allocated         */
#define SCAN2D_E_DEVICE   -9   /* no usable CUDA device, or not an sm_100 device        */
#define SCAN2D_E_STAGING -10   /* scan2d_fwd_host: staging buffer too small             */
#define SCAN2D_E_SCRATCH -11   /* scan2d_fwd_noalloc: shape needs more scratch than the
                                  fixed SCAN2D_NOALLOC_SCRATCH_BYTES                    */
#define SCAN2D_E_WORKSPACE -12 /* scan2d_bwd: workspace smaller than
                                  scan2d_bwd_workspace_bytes(...)                       */

/*
 * scan2d_fwd -- the 2D selective-scan forward on device buffers.
 *   x, delta, B, C, y : device pointers, element type per flags (see above);
 *   A, Dskip          : device pointers to fp32 (Dskip may be NULL);
 *   batch, channels, H, W >= 1;  1 <= N <= SCAN2D_MAX_N;
 *   flags             : SCAN2D_BF16 | SCAN2D_OUT_F32 | SCAN2D_VFIRST | orientation bits;
 *   stream            : a cudaStream_t (NULL = the legacy default stream).
 * Asynchronous: returns once the work is enqueued on `stream`.  y must not alias an input.
 * Repeated calls give bitwise identical y, except that when several orientations are summed
 * in shared memory (small maps) the order of those fp32 additions depends on timing, so y
 * may differ in the last bits.
 * Returns 0, or SCAN2D_E_NULL / _DIMS / _N / _FLAGS / _ALIGN / _NOMEM / _LAUNCH / _DEVICE.
 */
int scan2d_fwd(const void *x, const void *delta, const float *A, const void *B, const void *C,
               const float *Dskip, void *y, int batch, int channels, int H, int W, int N,
               unsigned flags, void *stream);

/*
 * scan2d_fwd_noalloc -- scan2d_fwd for callers that must not allocate device memory.  The
 * pages have no counterpart: this entry point exists for the host program, not the method.
 * Some callers cannot let a library call cudaMalloc: a runtime whose allocator has already
 * reserved the device memory it may use (a cudaMalloc outside it can fail or fragment it),
 * a plugin or operator interface that forbids allocating inside its execute call, or a
 * latency-bound loop that cannot afford the device-wide synchronisation cudaMalloc and
 * cudaFree may cause.  scan2d_fwd keeps a per-stream workspace that it allocates on first
 * need; this entry point instead takes its scratch (cross-block carry rings, and the fp32
 * accumulator of several orientations with bf16 output on maps too large for shared memory)
 * from one fixed device array of SCAN2D_NOALLOC_SCRATCH_BYTES that the library holds on every
 * device that loads it, until the process exits.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.  Arguments, layouts and results are those of scan2d_fwd.
 *   - The first call on a device looks up the array's device address with that device
 *     current; make that first call before any stream capture.
 *   - Every call, on every stream, shares the one array and leaves its contents behind; each
 *     call clears (cudaMemsetAsync on `stream`) the words that must start at zero.  Calls
 *     whose work overlaps on the GPU (different streams, or other threads) race on the
 *     array and give undefined results: order them, e.g. on one stream.
 *   - A shape whose scratch exceeds SCAN2D_NOALLOC_SCRATCH_BYTES (see scan2d_query_plan
 *     field [9]) is rejected with SCAN2D_E_SCRATCH before anything is enqueued.
 * Returns the scan2d_fwd codes (never SCAN2D_E_NOMEM), or SCAN2D_E_SCRATCH.
 */
int scan2d_fwd_noalloc(const void *x, const void *delta, const float *A, const void *B,
                       const void *C, const float *Dskip, void *y, int batch, int channels,
                       int H, int W, int N, unsigned flags, void *stream);

/*
 * Whole-slide images: the map x built from a bag of patch features ("2DMamba 精读", section
 * 四.2, the 2DMambaMIL framework, steps 3-4; papernotes.org notes, "方法详解 / 整体框架" and
 * "关键设计": patch features go back to the 2D grid at the patch's position, and every cell
 * without a patch holds a learnable non-tissue token p instead of zeros):
 *     x[d, i, j] = feat[k, d]  if patch k sits at cell (i, j),  else  p[d].
 *
 * scan2d_grid_cells -- the cell map of a bag.  coords: device (npatch, 2) int32 (row, column);
 * cell_patch: device (H*W) int32, written: the index of the patch at each cell, -1 where there
 * is none.  When several patches name one cell the highest index wins.  Patches outside the
 * grid are skipped and counted into *n_skipped (device int, written; may be NULL).
 * Asynchronous on `stream`.  Returns 0, SCAN2D_E_DIMS / _NULL / _ALIGN / _LAUNCH.
 */
int scan2d_grid_cells(const int *coords, int npatch, int H, int W, int *cell_patch,
                      int *n_skipped, void *stream);

/*
 * scan2d_grid_gather -- writes x (1, channels, H, W) from the bag feat (npatch, channels,
 * row-major), a cell map and the token pad (channels).  flags: 0 (fp32) or SCAN2D_BF16 (feat,
 * pad and x bf16).  Cell entries outside [0, npatch) read pad.  Asynchronous on `stream`.
 * Returns 0, SCAN2D_E_FLAGS / _DIMS / _NULL / _ALIGN / _LAUNCH.
 */
int scan2d_grid_gather(const void *feat, const int *cell_patch, const void *pad, void *x,
                       int npatch, int channels, int H, int W, unsigned flags, void *stream);

/*
 * scan2d_fwd_wsi -- scan2d_fwd of one map (batch 1) whose x is read from the bag through the
 * cell map as above, without x being written: the grid step fused in front of the scan.
 * feat (npatch, channels) and pad (channels) have the element type of x; delta, A, B, C,
 * Dskip, y, flags as for scan2d_fwd with batch = 1.  Rows are staged by plain loads (no TMA).
 * Returns the scan2d_fwd codes.
 */
int scan2d_fwd_wsi(const void *feat, const int *cell_patch, const void *pad, const void *delta,
                   const float *A, const void *B, const void *C, const float *Dskip, void *y,
                   int npatch, int channels, int H, int W, int N, unsigned flags, void *stream);

/*
 * scan2d_proj -- the input-dependent scan parameters from x, in the layouts scan2d_fwd reads.
 * The pages say the selective parameters are set by the current input ("2DMamba 精读", section
 * 四.4); the projection is read as Mamba's.  Per position p, contracting the channels of x[p]:
 *     u = Wx x[p]  (R + 2N values),   B[n,p] = u[R+n],   C[n,p] = u[R+N+n],
 *     delta[d,p] = softplus(sum_r Wdt[d,r] u[r] + bdt[d]),   softplus(z) = log(1 + e^z).
 *   x      : device (batch, channels, H, W), fp32 or bf16 (SCAN2D_BF16);
 *   Wx     : device (R + 2N, channels) fp32;  Wdt: device (channels, R) fp32;  bdt: (channels) fp32;
 *   delta  : device (batch, channels, H, W), element type of x (written);
 *   B, C   : device (batch, N, H, W), element type of x (written): the K = 1 layout of scan2d_fwd.
 * Limits: 1 <= R <= SCAN2D_PROJ_MAX_R, 1 <= N <= 16, and the weights must fit in shared memory
 * (channels * (R + N) floats, padded; 384 channels fit).  fp32 arithmetic.  Asynchronous on
 * `stream`.  Returns 0, SCAN2D_E_FLAGS / _DIMS / _N / _NULL / _ALIGN / _LAUNCH.
 */
int scan2d_proj(const void *x, const float *Wx, const float *Wdt, const float *bdt, void *delta,
                void *B, void *C, int batch, int channels, int H, int W, int N, int R,
                unsigned flags, void *stream);

/*
 * scan2d_query_plan -- how scan2d_fwd would run a call of this shape on a B200 (148
 * multiprocessors, clusters assumed resident), without launching anything or touching a device.  Writes up to n_out (<= SCAN2D_PLAN_FIELDS) values to `out`:
 *   [0] kernel launches per call        [5] columns per warp strip
 *   [1] blocks per launch               [6] warps (strips) per chain in a block
 *   [2] threads per block               [7] 0 one orientation, 1 orientations summed in
 *   [3] dynamic shared memory bytes         shared memory, 2 one launch per orientation
 *   [4] blocks per chain (segments)     [8] states per lane   [9] workspace bytes
 *   [10] channels per lane              [11] 1 if rows are staged by TMA (16-byte aligned
 *                                            row stride; buffers must also be 16-byte aligned)
 *   [12] how the blocks of a chain hand carries over: 0 one block per chain, 1 thread-block
 *        cluster (distributed shared memory), 2 ring in the internal global workspace
 * Returns 0 or the argument-check codes of scan2d_fwd.
 */
#define SCAN2D_PLAN_FIELDS 13
int scan2d_query_plan(int batch, int channels, int H, int W, int N, unsigned flags,
                      long long *out, int n_out);

/*
 * scan2d_host_staging_bytes -- device bytes scan2d_fwd_host needs for one call of this
 * shape (all inputs and the output, each rounded up to 256 bytes).  0 on bad arguments.
 */
size_t scan2d_host_staging_bytes(int batch, int channels, int H, int W, int N, unsigned flags);

/*
 * scan2d_fwd_host -- scan2d_fwd on HOST buffers.  Copies x, delta, A, B, C, Dskip from the
 * host into `staging` (a device buffer of at least scan2d_host_staging_bytes(...) bytes,
 * owned by the caller), runs scan2d_fwd there, and copies y back to the host buffer `y`,
 * all enqueued on `stream` with one cudaMemcpyAsync per tensor.  Asynchronous: host buffers
 * must stay valid until the stream has completed; use pinned host memory for the copies to
 * overlap.  Returns the scan2d_fwd codes, or SCAN2D_E_STAGING.
 */
int scan2d_fwd_host(const void *x, const void *delta, const float *A, const void *B,
                    const void *C, const float *Dskip, void *y, void *staging,
                    size_t staging_bytes, int batch, int channels, int H, int W, int N,
                    unsigned flags, void *stream);

/*
 * scan2d_bwd -- gradients of the 2D selective scan (training).  The pages give the forward
 * only ("2DMamba 精读", section 四.5); these are the chain-rule adjoints of its two recurrences.
 * For a cotangent dy of y = scan2d_fwd(x, delta, A, B, C, Dskip) they are the derivatives of
 * L = sum(dy * y):
 *     gh[p]  = C[p]*dy[p] + Abar[p+e2]*gh[p+e2]     (the vertical scan, backwards)
 *     ghh[p] = gh[p] + Abar[p+e1]*ghh[p+e1]         (the horizontal scan, backwards)
 *     dL/dAbar[p] = gh[p]*h[p-e2] + ghh[p]*hh[p-e1]
 *   dx     = sum_k sum_n ghh*delta*B + Dskip*dy     dB[b,k,n] = sum_d ghh*delta*x
 *   ddelta = sum_k sum_n (dL/dAbar*Abar*A + ghh*B*x) dC[b,k,n] = sum_d dy*h
 *   dA[d,n] = sum_{b,k,i,j} dL/dAbar*Abar*delta     dDskip[d] = sum_{b,i,j} dy*x
 * where e1 / e2 step one column / one row in the orientation's scan direction.
 *   x, delta, A, B, C, Dskip, flags, shapes : as for scan2d_fwd (Dskip may be NULL, then 0);
 *   dy, dx, ddelta : device, (batch, channels, H, W), element type of y (fp32; bf16 with
 *                    SCAN2D_BF16 unless SCAN2D_OUT_F32);
 *   dA (channels, N), dB and dC (batch, K, N, H, W), dDskip (channels): device fp32; all
 *                    are overwritten; dDskip may be NULL (not computed);
 *   workspace      : device buffer of at least scan2d_bwd_workspace_bytes(...) bytes,
 *                    256-byte aligned, owned by the caller; its contents on entry do not
 *                    matter and are left undefined.  It holds the forward's vertical state of
 *                    one orientation (N floats per element) and the strip carries.
 * With SCAN2D_VFIRST these are the gradients of the vertical-first forward (the roles of the
 * two scans swap: the horizontal adjoint reads C*dy, the vertical one adds it up the column).
 * Limits: 1 <= N <= SCAN2D_BWD_MAX_N.  Asynchronous on `stream`; outputs must not alias
 * inputs or each other.  dA, dB, dC and dDskip are sums built with atomic additions, so their
 * last bits may vary between calls.
 * Returns 0, or SCAN2D_E_NULL / _DIMS / _N / _FLAGS / _ALIGN / _WORKSPACE / _LAUNCH / _DEVICE.
 */
int scan2d_bwd(const void *x, const void *delta, const float *A, const void *B, const void *C,
               const float *Dskip, const void *dy, void *dx, void *ddelta, float *dA,
               float *dB, float *dC, float *dDskip, void *workspace, size_t workspace_bytes,
               int batch, int channels, int H, int W, int N, unsigned flags, void *stream);

/* scan2d_bwd_workspace_bytes -- workspace scan2d_bwd needs for this shape; 0 on bad arguments. */
size_t scan2d_bwd_workspace_bytes(int batch, int channels, int H, int W, int N, unsigned flags);

/*
 * scan2d_get_device_error -- synchronises `stream`, then returns and clears the first
 * device-side error recorded on the current device since the last call (0 if none;
 * SCAN2D_E_TIMEOUT if a bounded inter-block wait gave up, in which case the output of
 * the affected call is undefined), or SCAN2D_E_LAUNCH if the stream itself reports an error.
 */
int scan2d_get_device_error(void *stream);

/* Human-readable text for a SCAN2D_E_* code (static storage, never NULL). */
const char *scan2d_strerror(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
int scan2d_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SCAN2D_H */
