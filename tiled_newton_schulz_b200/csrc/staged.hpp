// staged.hpp -- HBM-staged batched path for tiles larger than 128 and for
// full-matrix NS / Gram NS, plus the fp32 CUDA-core path.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.hpp"

namespace himuon {

// A batch of equally shaped row-major matrices in workspace memory.
struct Batch {
  void *ptr;          // element (0,0) of matrix 0
  int64_t rows, cols; // each matrix
  int64_t stride;     // elements between consecutive matrices (= rows * cols)
  int32_t dtype;      // himuon_dtype
};

// Epilogue of the batched products below:
//   out32 = alpha * acc + beta * c32 + diag * I   (c32 may be null: beta ignored)
//   out16 = 16-bit copy of out32 (operand dtype), optional
struct Epilogue {
  float alpha, beta;
  float diag;       // added on the diagonal of each (square) output matrix
  const float *c32;
  const void *c16;      // the C term in 16 bits (out16_dtype) instead of c32 (nullptr: none)
  const float *alpha_batch;   // per-matrix alpha (replaces alpha; tensor-core path only)
  float *out32;
  void *out16;
  int32_t out16_dtype;
  // A second output, the same values plus diag2 on the diagonal (e.g. Q = Z + a I
  // beside Z); out2_16 has out16_dtype.
  float *out2_32;
  void *out2_16;
  float diag2;
  // The product is symmetric (M == N; and c32, if given, symmetric): the
  // tensor-core version computes only the 128 x 128 tiles on and below the
  // diagonal and writes each off-diagonal one twice, mirrored.
  int32_t sym;
  // With sym: the fp32 outputs (out32, out2_32) get only the 128 x 128 blocks
  // on and below the diagonal, not the mirrored copies above it (for a
  // matrix read only as the C term of other symmetric products, which read
  // those blocks alone).  The 16-bit outputs, read as operands, stay whole.
  int32_t lower32;
  // Scatter (tensor-core path): instead of out32/out16, matrix z of the batch
  // is the tile sc_tiles[z]; its valid h x w part (transposed back when the
  // tile is) goes straight to its block's Out role and, with sc_mode 1, into
  // W -= sc_lr * O, as launch_unpack would write it from an fp32 copy.
  const DevTile *sc_tiles;
  const DevBlock *sc_blocks;
  int32_t sc_mode;
  float sc_lr;
};

// acc = A * B^T (b_trans = 1, B is N x K) or A * B (b_trans = 0, B is K x N),
// for every matrix of the batch.  A: M x K.  Operands are 16-bit for the
// tensor-core version and fp32 for the CUDA-core version.  M, N multiples of
// 128 and K a multiple of 64 (the planner pads with zeros).
cudaError_t gemm_tc(const Batch &A, const Batch &B, int b_trans, int64_t M, int64_t N, int64_t K, int64_t batch,
                    const Epilogue &ep, int *status, cudaStream_t stream);
cudaError_t gemm_simt(const Batch &A, const Batch &B, int b_trans, int64_t M, int64_t N, int64_t K, int64_t batch,
                      const Epilogue &ep, cudaStream_t stream);

// ----------------------------------------------------------------- element passes
struct PackArgs {
  const DevBlock *blocks;
  const DevTile *tiles;   // tiles of this chunk
  int64_t n_tiles;
  int64_t n, m;           // padded iterate shape (n <= m), row-major n x m per tile
  float *x32;             // n_tiles * n * m (fp32 iterate), or nullptr when x16 takes the values
  void *x16;              // 16-bit copy instead of x32 (x16_dtype; neither: sums of squares only)
  int32_t x16_dtype;
  const float *scale;     // with x16: per-tile factor applied before rounding (the second pass
                          // of a two-pass normalisation; nullptr: the values as they are)
  float *partial;         // n_tiles * parts
  int32_t parts;          // partial sums per tile (row slices of the source tile)
  int32_t mode;           // 0: NS input; 1: momentum (M' = mu M + G written back to M)
  float mu;
};
cudaError_t launch_pack(const PackArgs &a, cudaStream_t stream);

struct NormArgs {
  int64_t n_tiles;
  int64_t elems;          // n * m per tile
  float *x32;
  void *x16;              // optional 16-bit operand copy
  int32_t x16_dtype;
  const float *partial;
  int32_t parts;
  int32_t keep32;         // also write the normalised fp32 iterate back to x32
  float eps, safety;
};
cudaError_t launch_normalize(const NormArgs &a, cudaStream_t stream);
// inv[t] = 1 / ((sqrt(sum of tile t's partial sums) + eps) * safety), inv2[t] = inv[t]^2
cudaError_t launch_tile_scales(const float *partial, int32_t parts, int64_t n_tiles, float eps, float safety,
                               float *inv, float *inv2, cudaStream_t stream);

struct UnpackArgs {
  const DevBlock *blocks;
  const DevTile *tiles;
  int64_t n_tiles;
  int64_t n, m;
  const float *x32;
  int32_t mode;           // 0: write role Out; 1: momentum: W -= lr O (if W), O to role Out (if present)
  float lr;
};
cudaError_t launch_unpack(const UnpackArgs &a, cudaStream_t stream);

}  // namespace himuon
