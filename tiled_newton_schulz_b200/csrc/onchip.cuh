// onchip.cuh -- device helpers shared by the on-chip kernels (one CTA per
// tile group, and the CTA pair for 256 x 256 tiles): tile coordinates and
// their decoder, bounded waits, 16-bit packing.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "layout.hpp"
#include "ptx.cuh"
#include "resident.hpp"

namespace himuon {
namespace onchip {

constexpr float kTinyNorm = 1.0f / 1024.0f;   // below this normalised norm a tile keeps bf16 operands

struct TileCoord {
  int32_t blk;       // -1: no tile
  int32_t x0, y0, cols;
  int32_t h, w;      // the tile's extent (edge tiles smaller)
  int32_t tm[kNumRoles];
  int32_t pad[2];
};

// What the tile decoder needs of a DevBlock, kept in shared memory (used when
// the host found that the block table fits: ResidentArgs::smem_blocks).
struct SBlock {
  int32_t tile_begin;
  int32_t cols;
  uint16_t tiles_c, T;
  int16_t tm[kNumRoles];
  int32_t rows;
};
static_assert(sizeof(SBlock) == 24, "SBlock layout");
static_assert(sizeof(TileCoord) == 48, "TileCoord layout");

// Bounded wait that also gives up as soon as another thread of the CTA has
// raised the abort flag (after its own wait timed out).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort, int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
  }
  set_status(status, HIMUON_ERR_TIMEOUT);
  *abort = 1;
  return false;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
// two values as a 16-bit operand pair of format F (0: fp16, 1: bf16)
template <int F>
__device__ __forceinline__ uint32_t pack2_op(float a, float b) {
  if (F == 1) return pack2_bf16(a, b);
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ uint4 pack8_bf16(const float *f) {
  return make_uint4(pack2_bf16(f[0], f[1]), pack2_bf16(f[2], f[3]), pack2_bf16(f[4], f[5]), pack2_bf16(f[6], f[7]));
}
template <int F>
__device__ __forceinline__ uint4 pack8_op(const float *f) {
  return make_uint4(pack2_op<F>(f[0], f[1]), pack2_op<F>(f[2], f[3]), pack2_op<F>(f[4], f[5]),
                    pack2_op<F>(f[6], f[7]));
}

// Block of `tile` by binary search over tile_begin, in the shared-memory copy
// of the block table `sb` when there is one (a few shared loads), else in global.
static __device__ __noinline__ TileCoord decode_tile(const ResidentArgs &a, const SBlock *sb, int64_t tile,
                                             int hint = -1) {
  TileCoord t;
  t.blk = -1;
  t.x0 = t.y0 = t.cols = t.h = t.w = 0;
  t.pad[0] = t.pad[1] = 0;
#pragma unroll
  for (int r = 0; r < kNumRoles; ++r) t.tm[r] = -1;
  if (tile >= a.n_tiles) return t;
  int lo = 0, hi = a.n_blocks - 1;
  if (sb) {
    if (hint >= 0) {  // the tile right after one in block `hint`: same block or a later one
      lo = hint;
      while (lo < hi && sb[lo + 1].tile_begin <= tile) ++lo;
      hi = lo;
    }
    while (lo < hi) {  // last block with tile_begin <= tile
      const int mid = (lo + hi + 1) >> 1;
      if (sb[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
    }
    const SBlock &b = sb[lo];
    const int32_t local = static_cast<int32_t>(tile) - b.tile_begin;
    t.blk = lo;
    t.y0 = (local / b.tiles_c) * b.T;
    t.x0 = (local % b.tiles_c) * b.T;
    t.cols = b.cols;
    t.h = min(static_cast<int32_t>(b.T), b.rows - t.y0);
    t.w = min(static_cast<int32_t>(b.T), b.cols - t.x0);
#pragma unroll
    for (int r = 0; r < kNumRoles; ++r) t.tm[r] = b.tm[r];
    return t;
  }
  if (hint >= 0) {  // a later tile than one in block `hint`: that block or one after it, usually
                    // the same or the next (one or two dependent loads instead of a full search)
    lo = hint;
    for (int k = 0; k < 2 && lo < hi; ++k) {
      if (a.blocks[lo + 1].tile_begin > tile) {
        hi = lo;
        break;
      }
      ++lo;
    }
  }
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.blocks[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const DevBlock &b = a.blocks[lo];
  const int64_t local = tile - b.tile_begin;
  t.blk = lo;
  t.y0 = static_cast<int32_t>(local / b.tiles_c) * b.T;
  t.x0 = static_cast<int32_t>(local % b.tiles_c) * b.T;
  t.cols = b.cols;
  t.h = min(b.T, b.rows - t.y0);
  t.w = min(b.T, b.cols - t.x0);
#pragma unroll
  for (int r = 0; r < kNumRoles; ++r) t.tm[r] = b.tmap[r];
  return t;
}

}  // namespace onchip
}  // namespace himuon
