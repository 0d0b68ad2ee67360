/*
 * himuon.h -- C ABI of libhimuon: tiled Newton-Schulz (HiMuon) on B200.
 *
 * The library evaluates the finite Newton-Schulz (NS) map that Muon-type
 * optimizers apply to momentum matrices, in the tiled form of
 * "Hierarchical Muon: Tiled Newton-Schulz Updates for Efficient Muon
 * Optimization" (abstract): each H x W matrix is cut into T x T tiles from the
 * top-left corner, each tile gets the same NS map on its own, and the results
 * are put back in place.  Ragged edge tiles are smaller matrices under the same
 * map.  The per-tile map is Algorithm 1 of the "Gram Newton-Schulz" page
 * (sec. 3):
 *     X <- X / (||X||_F + eps);  if rows > cols: X <- X^T
 *     for t = 1..K:  A = X X^T;  B = b_t A + c_t A^2;  X = a_t X + B X
 *     undo the transpose.
 *
 * Conventions for every entry point
 *  - Matrices are row-major 2-D arrays in DEVICE memory described by
 *    himuon_mat; element (i, j) sits at data + (i * ld + j) * sizeof(dtype).
 *    All pointers inside himuon_mat must be 16-byte aligned and ld * sizeof
 *    must be a multiple of 16 bytes (the tile loads use the tensor memory
 *    accelerator).  Other struct pointers (splits, coeffs, restart lists) are
 *    HOST pointers, read during the call only.
 *  - The caller owns every buffer.  Results are written into caller buffers;
 *    `ws` is caller-provided device scratch of `ws_bytes` bytes, sized with
 *    himuon_workspace_size().  The library keeps a small cache of per-matrix
 *    tables (tensor-map descriptors and tile tables) keyed by the call's
 *    matrices and parameters; it is built and uploaded on the first call with
 *    a new key and reused afterwards.
 *  - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  Calls on one stream run in order.
 *  - Return value: HIMUON_OK (0) or a negative HIMUON_ERR_* code for invalid
 *    arguments, unsupported shapes or dtypes, a too-small workspace or a CUDA
 *    launch error.  Nothing is enqueued when an argument check fails.  Faults
 *    that only the device can see (a wait that timed out, a bad descriptor)
 *    set a device status word read by himuon_get_device_status(); kernels never
 *    trap.
 *  - Not thread-safe: serialise calls from different host threads (the plan
 *    cache is locked internally, but the device status word is shared).
 */
#ifndef HIMUON_H_
#define HIMUON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HIMUON_VERSION 2   /* 2: himuon_ns_params.tiles */

#if defined(__GNUC__)
#define HIMUON_API __attribute__((visibility("default")))
#else
#define HIMUON_API
#endif

typedef enum {
  HIMUON_BF16 = 0,   /* storage: bfloat16;  compute: bf16 tensor-core operands, fp32 accumulate */
  HIMUON_FP16 = 1,   /* storage: float16;   compute: fp16 tensor-core operands, fp32 accumulate */
  HIMUON_FP32 = 2    /* storage: float32;   compute: fp32 on CUDA cores */
} himuon_dtype;

enum {
  HIMUON_OK = 0,
  HIMUON_ERR_INVALID = -1,      /* null pointer, bad count, bad shape or ld */
  HIMUON_ERR_UNSUPPORTED = -2,  /* dtype / tile size / step count not supported */
  HIMUON_ERR_WORKSPACE = -3,    /* ws_bytes smaller than himuon_workspace_size() */
  HIMUON_ERR_ALIGNMENT = -4,    /* pointer or row pitch not 16-byte aligned */
  HIMUON_ERR_CUDA = -5,         /* a CUDA runtime/driver call failed */
  HIMUON_ERR_TIMEOUT = -6,      /* device: a bounded wait gave up (device status only) */
  HIMUON_ERR_DEVICE = -7,       /* device: inconsistent descriptor seen by a kernel */
  HIMUON_ERR_NO_DEVICE = -8,    /* no usable sm_100 device */
  HIMUON_ERR_TOO_LARGE = -9     /* himuon_ns_static: the call needs more scratch than its fixed array */
};

/* One row-major matrix in device memory. */
typedef struct {
  void *data;       /* device pointer to element (0, 0) */
  int64_t rows;     /* H >= 1 */
  int64_t cols;     /* W >= 1 */
  int64_t ld;       /* elements between consecutive rows, >= cols */
  int32_t dtype;    /* himuon_dtype of the storage */
} himuon_mat;

/*
 * CMuon split (CMuon article: split a fused tensor such as QKV or AdaLN into
 * its functional blocks before orthogonalisation; each block is treated as a
 * matrix of its own).  dim = 0 cuts the rows, dim = 1 the columns, into
 * nblocks consecutive blocks of sizes[i]; the sizes must sum to that
 * dimension.  nblocks <= 1 (or a NULL himuon_split pointer) keeps the matrix
 * whole.  `sizes` is a host pointer.
 */
typedef struct {
  int32_t dim;
  int32_t nblocks;
  const int64_t *sizes;
} himuon_split;

/* Parameters of the NS map. */
typedef struct {
  int32_t tile;            /* T in {32, 64, 128, 256, 512, ...}; T <= 0 or T >= max(rows, cols)
                              means one tile per (split block of a) matrix: full-matrix NS.      */
  int32_t steps;           /* K, 1..16                                                           */
  const float *coeffs;     /* host: K triples (a_t, b_t, c_t), step t at coeffs[3t..3t+2]       */
  float eps;               /* added to ||X||_F before dividing (Algorithm 1 uses 1e-7)          */
  int32_t compute;         /* himuon_dtype of the arithmetic (see himuon_dtype)                  */
  float safety;            /* input divided by this factor after normalisation; 1.0 = off
                              ("Gram Newton-Schulz" sec. 6 suggests 1.05); 0 is read as 1.0      */
  int32_t n_restart;       /* Gram NS only: number of entries in restart_at                      */
  const int32_t *restart_at; /* host: 1-based step indices t before which Gram NS restarts
                              (X <- Q X, R <- X X^T, Q <- I); the page restarts at t = 3         */
  int64_t chunk_bytes;     /* staged path: upper bound on the scratch one chunk of tiles may
                              use (memory-bounded chunking); 0 = use all of ws_bytes             */
  const int32_t *tiles;    /* host, NULL or one T per matrix (a runtime tile-size schedule,
                              "Hierarchical Muon" abstract): tiles[i] replaces `tile` for matrix
                              i (and all its split blocks), with the same meaning (<= 0: the
                              whole matrix).  See "Per-matrix tile sizes" below.                 */
} himuon_ns_params;

/*
 * Per-matrix tile sizes (p->tiles != NULL).  The matrices of a call are
 * grouped by their T (in first-appearance order of T, matrix order kept inside
 * a group), and each group runs as the same call would with p->tile = that T:
 * on chip for T <= 128, staged otherwise.  The groups run one after another on
 * `stream` and share `ws`, which must hold the largest group's need (what
 * himuon_workspace_size returns for the same params).  Every group's arguments
 * are checked before the first is enqueued.  himuon_ns_full ignores `tiles`
 * (every matrix is one tile); himuon_ns_static rejects it with
 * HIMUON_ERR_UNSUPPORTED.
 */

/* op codes for himuon_workspace_size */
enum { HIMUON_OP_NS_TILED = 0, HIMUON_OP_NS_FULL = 1, HIMUON_OP_GRAM_NS = 2, HIMUON_OP_MOMENTUM_STEP = 3 };

/*
 * Tiled NS (HiMuon abstract; per-tile map: Gram Newton-Schulz page, Alg. 1).
 * in[i] -> out[i] for i < n.  in and out have equal shapes; out may alias in
 * (the same pointer and ld) -- every tile is read before it is written.
 * splits: NULL or n entries (CMuon split per matrix).
 * Storage dtype of in/out: BF16 or FP16 with compute BF16/FP16, or any storage
 * with compute FP32.  All tiles of all matrices run in one batched launch per
 * tile-shape class; T <= 128 keeps each tile on chip for all K steps, larger T
 * runs HBM-staged batched GEMMs in chunks bounded by ws_bytes / chunk_bytes.
 */
HIMUON_API int himuon_ns_tiled(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                    const himuon_ns_params *p, void *ws, size_t ws_bytes, void *stream);

/* Full-matrix NS of every (split block of a) matrix: himuon_ns_tiled with T = infinity. */
HIMUON_API int himuon_ns_full(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                   const himuon_ns_params *p, void *ws, size_t ws_bytes, void *stream);

/*
 * Stabilised Gram NS ("Gram Newton-Schulz" page, sec. 6, Algorithm 3) of every
 * (split block of a) matrix, full-matrix: normalise, transpose if taller than
 * wide, R = X X^T, Q = I; per step (after a restart X <- Q X, R <- X X^T,
 * Q <- I at the steps in p->restart_at) Z = b R + c R^2, Q <- Q Z + a Q,
 * RZ <- R Z + a R, R <- Z RZ + a RZ; output Q X (transposed back).
 * Equal to himuon_ns_full in exact arithmetic.  compute: FP16 (the page's
 * advice for this variant), BF16 or FP32.  p->tile = 0 (or any T at least as
 * large as a block's sides) runs it on the whole (split block of the) matrix;
 * a smaller T applies it to each T x T tile ("Hierarchical Muon" abstract:
 * the same map per tile, ragged edge tiles smaller), on the staged path.
 */
HIMUON_API int himuon_gram_ns(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                   const himuon_ns_params *p, void *ws, size_t ws_bytes, void *stream);

/*
 * One Muon step ("Gram Newton-Schulz" page, sec. 3, Muon recap) with tiled NS:
 *     M <- mu M + G;   O = tiledNS(M);   W <- W - lr O.
 * M is updated in place (the stored momentum is the rounded mu M + G; the NS
 * input is the same value before rounding).  W may be NULL (no weight update);
 * update_out may be NULL, else it receives O.  At least one of W and
 * update_out must be given.  All matrices of index i have equal shapes.
 * Storage: BF16 (compute BF16) for the on-chip path; any storage with compute
 * FP32.  The split of matrix i applies to W[i], M[i], G[i] and update_out[i].
 */
HIMUON_API int himuon_momentum_step(const himuon_mat *W, const himuon_mat *M, const himuon_mat *G, int32_t n,
                         float mu, float lr, const himuon_split *splits, const himuon_ns_params *p,
                         const himuon_mat *update_out, void *ws, size_t ws_bytes, void *stream);

/*
 * Device scratch (bytes) that op (HIMUON_OP_*) needs for these matrices and
 * parameters; 0 when the whole call runs on chip.  Returns a negative
 * HIMUON_ERR_* code on invalid arguments.  Host-only, enqueues nothing.
 */
HIMUON_API int64_t himuon_workspace_size(const himuon_mat *mats, int32_t n, const himuon_split *splits,
                              const himuon_ns_params *p, int32_t op);

/*
 * Synchronises `stream`, returns the device status word of the current device
 * (HIMUON_OK, HIMUON_ERR_TIMEOUT or HIMUON_ERR_DEVICE) and clears it.
 */
HIMUON_API int himuon_get_device_status(void *stream);

/* Static, human-readable text for a status code. */
HIMUON_API const char *himuon_status_string(int code);

/* HIMUON_VERSION of the loaded library. */
HIMUON_API int himuon_version(void);

/*
 * Allocation-free variant of the staged (HBM) path of himuon_ns_tiled /
 * himuon_ns_full.  The paper has no counterpart to this entry point: it serves
 * callers that cannot allocate device memory themselves -- for instance code
 * running under a custom allocator or memory pool that owns all of HBM, or a
 * host runtime that forbids cudaMalloc/cudaFree (which synchronise the device)
 * during training steps -- and so cannot hand the other entry points a
 * workspace.
 *
 * Arguments are those of himuon_ns_tiled (p->tile <= 0 means full-matrix NS),
 * minus the workspace.  in/out are still caller buffers.  Every tile, of any
 * size, runs on the staged path of batched tensor-core GEMMs (or the fp32 path
 * for compute FP32).  Its scratch -- the tile tables and the chunk workspace --
 * lives in one file-scope device array of HIMUON_STATIC_SCRATCH_BYTES
 * (32 MiB) that every GPU which loads the library holds until the process
 * exits.  The call allocates no device memory (no cudaMalloc, cudaFree or
 * allocating library routine) and bypasses the plan cache.  A call whose
 * largest tile (or its tables) does not fit returns HIMUON_ERR_TOO_LARGE
 * before enqueuing anything; e.g. full-matrix NS of a 1024-row matrix fits up
 * to 1024 x 7040 in bf16 (4 bytes of scratch per element plus 4 n^2 bytes for
 * the n x n products) and 1024 x 2944 in fp32 (twice that).
 *
 * The first call on a device looks up that device's address of the array
 * (cudaGetSymbolAddress, with the device current) and keeps it for later
 * calls; make that first call before any stream capture.  A cudaDeviceReset
 * of that device invalidates the kept address: do not call himuon_ns_static
 * after resetting a device it was used on.  Thin tiles (short side <= 64) of
 * a bf16 call run in fp32, as on the workspace path.  All calls share the one
 * array and it keeps the last call's contents: calls that overlap on the GPU
 * (on different streams, or from different host threads) race on it and must
 * be serialised by the caller.  Calls on one stream are ordered and safe.
 */
#define HIMUON_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
HIMUON_API int himuon_ns_static(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                                const himuon_ns_params *p, void *stream);

/*
 * Number of CUDA kernels this library has enqueued since it was loaded, on all
 * devices and streams (a host-side counter, incremented at each launch; no
 * device synchronisation).  For accounting in benchmarks and tests.
 */
HIMUON_API int64_t himuon_launch_count(void);

/*
 * Host-side tile list of a call, for checking the planner against a reference
 * tiling.  Fills up to `cap` records of 5 int64 each:
 *     (matrix index, row0, col0, h, w)
 * in the order the tile scheduler numbers tiles (matrix by matrix, split block
 * by split block, tiles row-major from the top-left corner of each block),
 * and returns the total number of tiles (or a negative HIMUON_ERR_* code).
 * Tile size T <= 0 or T >= the block size gives one tile per block.
 */
HIMUON_API int64_t himuon_plan_tiles(const himuon_mat *mats, int32_t n, const himuon_split *splits, int32_t tile,
                          int64_t *records, int64_t cap);

#ifdef __cplusplus
}
#endif
#endif /* HIMUON_H_ */
