// staged.cu -- batched products and element passes of the HBM-staged path.
//
// Used for tiles larger than 128 x 128, for full-matrix NS and Gram NS, and
// for fp32 arithmetic.  The iterate of every tile lives in workspace memory as
// an fp32 master copy (x32) plus a 16-bit operand copy; each NS step
// ("Gram Newton-Schulz" page, sec. 3, Algorithm 1) is three batched products
// with fused epilogues:
//     A  = X X^T                  -> A (fp32) and a 16-bit copy
//     B  = b A + c (A A)          -> 16-bit B
//     X  = a X + B X              -> X (fp32, in place) and a 16-bit copy
// Tiles are zero-padded to multiples of 128 on both sides and transposed when
// taller than wide; both leave the map unchanged (a zero border stays zero,
// and NS(X^T) = NS(X)^T).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"
#include "staged.hpp"

namespace himuon {

namespace {

// ---------------------------------------------------------------- element access
__device__ __forceinline__ float ld_elem(const void *p, int32_t dtype, int64_t i) {
  if (dtype == HIMUON_BF16) return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
  if (dtype == HIMUON_FP16) return __half2float(static_cast<const __half *>(p)[i]);
  return static_cast<const float *>(p)[i];
}
__device__ __forceinline__ void st_elem(void *p, int32_t dtype, int64_t i, float v) {
  if (dtype == HIMUON_BF16) static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
  else if (dtype == HIMUON_FP16) static_cast<__half *>(p)[i] = __float2half_rn(v);
  else static_cast<float *>(p)[i] = v;
}

template <int NT>
__device__ __forceinline__ float block_sum(float v, float *scratch) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) scratch[w] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < NT / 32; ++i) s += scratch[i];
  }
  return s;  // valid in thread 0
}

// ---------------------------------------------------------------- pack
// 8 consecutive 16-bit values of either type, to fp32
__device__ __forceinline__ void ld8_16(const void *p, int32_t dtype, int64_t i, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p) + i);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (dtype == HIMUON_BF16) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[k]));
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    } else {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[k]));
      v[2 * k] = f.x;
      v[2 * k + 1] = f.y;
    }
  }
}
__device__ __forceinline__ void st8_16(void *p, int32_t dtype, int64_t i, const float (&v)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (dtype == HIMUON_BF16) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t *>(&h);
    } else {
      const __half2 h = __floats2half2_rn(v[2 * k], v[2 * k + 1]);
      w[k] = *reinterpret_cast<const uint32_t *>(&h);
    }
  }
  *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p) + i) = make_uint4(w[0], w[1], w[2], w[3]);
}
// Runs of 8 elements of a role can be moved as one 16-byte access when the
// role is 16-bit, its base is 16-byte aligned and its rows and the tile's
// first column keep that alignment.
__device__ __forceinline__ bool vec8_ok(const void *p, int32_t dtype, int64_t ld, int32_t c0) {
  return p && dtype != HIMUON_FP32 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0 && (ld & 7) == 0 && (c0 & 7) == 0;
}

// grid (parts, tiles): CTA p copies source rows [p*rpp, (p+1)*rpp) of its
// tile, rpp = ceil(rows / parts), so every part of a tile has work whatever
// its orientation.  The CTA's threads run over (row, 8-column run) pairs,
// with 16-byte accesses where the roles allow them.
__global__ void __launch_bounds__(256) pack_kernel(const PackArgs a) {
  __shared__ float scratch[8];
  const int64_t t = blockIdx.y;
  const DevTile tl = a.tiles[t];
  const DevBlock &b = a.blocks[tl.block];
  const int32_t rpp = (tl.h + a.parts - 1) / a.parts;
  const int32_t i0 = blockIdx.x * rpp;
  const int32_t i1 = min(tl.h, i0 + rpp);
  float *x = a.x32 ? a.x32 + t * a.n * a.m : nullptr;
  void *xh = (a.x32 || !a.x16) ? nullptr : static_cast<void *>(static_cast<uint16_t *>(a.x16) + t * a.n * a.m);
  const float sc = a.scale ? a.scale[t] : 1.f;
  float ss = 0.f;
  if (i0 < i1) {
    const void *src = b.ptr[kRoleIn];
    const int64_t ld = b.ld[kRoleIn];
    const int32_t dt = b.dtype[kRoleIn];
    const void *gsrc = b.ptr[kRoleG];
    const int64_t ldg = b.ld[kRoleG];
    const int32_t dtg = b.dtype[kRoleG];
    const bool vec = vec8_ok(src, dt, ld, tl.c0) && (a.mode == 0 || vec8_ok(gsrc, dtg, ldg, tl.c0));
    const int32_t runs = vec ? tl.w / 8 : 0;            // whole 8-column runs per row
    const int32_t rest = tl.w - 8 * runs;                // columns left to the scalar loop
    const int32_t rows = i1 - i0;
    for (int32_t k = threadIdx.x; k < rows * runs; k += blockDim.x) {
      const int32_t i = i0 + k / runs, j = 8 * (k % runs);
      const int64_t gi = static_cast<int64_t>(tl.r0 + i) * ld + tl.c0 + j;
      float v[8];
      ld8_16(src, dt, gi, v);
      if (a.mode == 1) {
        float g[8];
        ld8_16(gsrc, dtg, static_cast<int64_t>(tl.r0 + i) * ldg + tl.c0 + j, g);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = fmaf(a.mu, v[e], g[e]);
        st8_16(b.ptr[kRoleIn], dt, gi, v);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
      if (xh) {
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = v[e] * sc;
        if (tl.transposed) {
#pragma unroll
          for (int e = 0; e < 8; ++e) st_elem(xh, a.x16_dtype, static_cast<int64_t>(j + e) * a.m + i, w[e]);
        } else {
          st8_16(xh, a.x16_dtype, static_cast<int64_t>(i) * a.m + j, w);
        }
      } else if (x && tl.transposed) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[static_cast<int64_t>(j + e) * a.m + i] = v[e];
      } else if (x) {
        float4 *xo = reinterpret_cast<float4 *>(x + static_cast<int64_t>(i) * a.m + j);
        xo[0] = make_float4(v[0], v[1], v[2], v[3]);
        xo[1] = make_float4(v[4], v[5], v[6], v[7]);
      }
    }
    for (int32_t k = threadIdx.x; k < rows * rest; k += blockDim.x) {
      const int32_t i = i0 + k / rest, j = 8 * runs + k % rest;
      const int64_t gi = static_cast<int64_t>(tl.r0 + i) * ld + tl.c0 + j;
      float v = ld_elem(src, dt, gi);
      if (a.mode == 1) {
        v = fmaf(a.mu, v, ld_elem(gsrc, dtg, static_cast<int64_t>(tl.r0 + i) * ldg + tl.c0 + j));
        st_elem(b.ptr[kRoleIn], dt, gi, v);
      }
      ss = fmaf(v, v, ss);
      const int64_t o = tl.transposed ? static_cast<int64_t>(j) * a.m + i : static_cast<int64_t>(i) * a.m + j;
      if (xh) st_elem(xh, a.x16_dtype, o, v * sc);
      else if (x) x[o] = v;
    }
  }
  const float s = block_sum<256>(ss, scratch);
  if (threadIdx.x == 0 && !a.scale) a.partial[t * a.parts + blockIdx.x] = s;   // (the second pass: already summed)
}

// grid (chunks, tiles): rho from the partial sums (fixed order), then scale,
// four elements per access (16-byte fp32 loads and stores, 8-byte 16-bit
// stores; a tile's chunk starts at a multiple of 8 elements).
__global__ void __launch_bounds__(256) normalize_kernel(const NormArgs a) {
  const int64_t t = blockIdx.y;
  float s = 0.f;
  for (int p = 0; p < a.parts; ++p) s += a.partial[t * a.parts + p];
  const float inv = 1.0f / ((sqrtf(s) + a.eps) * a.safety);
  float *x = a.x32 + t * a.elems;
  const int64_t per = ((a.elems + gridDim.x - 1) / gridDim.x + 7) / 8 * 8;
  const int64_t e0 = blockIdx.x * per, e1 = min(a.elems, e0 + per);
  // (the planner pads tiles to multiples of 128 rows and columns; any other
  // size takes the element loop below)
  const bool vec = (a.elems & 7) == 0;
  int64_t e = vec ? e0 + 4 * threadIdx.x : e0 + threadIdx.x;
  for (; vec && e + 4 <= e1; e += 4 * blockDim.x) {
    float4 v = *reinterpret_cast<const float4 *>(x + e);
    v.x *= inv;
    v.y *= inv;
    v.z *= inv;
    v.w *= inv;
    if (a.keep32) *reinterpret_cast<float4 *>(x + e) = v;
    if (a.x16) {
      uint2 u;
      if (a.x16_dtype == HIMUON_FP16) {
        __half2 *h = reinterpret_cast<__half2 *>(&u);
        h[0] = __floats2half2_rn(v.x, v.y);
        h[1] = __floats2half2_rn(v.z, v.w);
      } else {
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
        h[0] = __floats2bfloat162_rn(v.x, v.y);
        h[1] = __floats2bfloat162_rn(v.z, v.w);
      }
      *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(a.x16) + t * a.elems + e) = u;
    }
  }
  for (; e < e1; e += vec ? 1 : blockDim.x) {   // element by element when not vectorised
    const float v = x[e] * inv;
    if (a.keep32) x[e] = v;
    if (a.x16) st_elem(a.x16, a.x16_dtype, t * a.elems + e, v);
  }
}

// grid (parts, tiles), rows split as in pack_kernel; 8-column runs where the
// roles allow 16-byte accesses.
__global__ void __launch_bounds__(256) unpack_kernel(const UnpackArgs a, int32_t parts) {
  const int64_t t = blockIdx.y;
  const DevTile tl = a.tiles[t];
  const DevBlock &b = a.blocks[tl.block];
  const int32_t rpp = (tl.h + parts - 1) / parts;
  const int32_t i0 = blockIdx.x * rpp, i1 = min(tl.h, i0 + rpp);
  if (i0 >= i1) return;
  const float *x = a.x32 + t * a.n * a.m;
  void *out = b.ptr[kRoleOut];
  void *wp = a.mode == 1 ? b.ptr[kRoleW] : nullptr;
  const bool vec = (!out || vec8_ok(out, b.dtype[kRoleOut], b.ld[kRoleOut], tl.c0)) &&
                   (!wp || vec8_ok(wp, b.dtype[kRoleW], b.ld[kRoleW], tl.c0));
  const int32_t runs = vec ? tl.w / 8 : 0;
  const int32_t rest = tl.w - 8 * runs;
  const int32_t rows = i1 - i0;
  for (int32_t k = threadIdx.x; k < rows * runs; k += blockDim.x) {
    const int32_t i = i0 + k / runs, j = 8 * (k % runs);
    float o[8];
    if (tl.transposed) {
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = x[static_cast<int64_t>(j + e) * a.m + i];
    } else {
      const float4 *xi = reinterpret_cast<const float4 *>(x + static_cast<int64_t>(i) * a.m + j);
      const float4 p0 = xi[0], p1 = xi[1];
      o[0] = p0.x; o[1] = p0.y; o[2] = p0.z; o[3] = p0.w;
      o[4] = p1.x; o[5] = p1.y; o[6] = p1.z; o[7] = p1.w;
    }
    if (out) st8_16(out, b.dtype[kRoleOut], static_cast<int64_t>(tl.r0 + i) * b.ld[kRoleOut] + tl.c0 + j, o);
    if (wp) {
      const int64_t gi = static_cast<int64_t>(tl.r0 + i) * b.ld[kRoleW] + tl.c0 + j;
      float w[8];
      ld8_16(wp, b.dtype[kRoleW], gi, w);
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = fmaf(-a.lr, o[e], w[e]);
      st8_16(wp, b.dtype[kRoleW], gi, w);
    }
  }
  for (int32_t k = threadIdx.x; k < rows * rest; k += blockDim.x) {
    const int32_t i = i0 + k / rest, j = 8 * runs + k % rest;
    const int64_t xo = tl.transposed ? static_cast<int64_t>(j) * a.m + i : static_cast<int64_t>(i) * a.m + j;
    const float o = x[xo];
    if (out) st_elem(out, b.dtype[kRoleOut], static_cast<int64_t>(tl.r0 + i) * b.ld[kRoleOut] + tl.c0 + j, o);
    if (wp) {
      const int64_t gi = static_cast<int64_t>(tl.r0 + i) * b.ld[kRoleW] + tl.c0 + j;
      st_elem(wp, b.dtype[kRoleW], gi, fmaf(-a.lr, o, ld_elem(wp, b.dtype[kRoleW], gi)));
    }
  }
}

// ---------------------------------------------------------------- epilogue
struct EpiArgs {
  float alpha, beta, diag;
  const float *c32;
  const void *c16;   // 16-bit C term (out16_dtype), tensor-core path only
  const float *alpha_batch;   // per-matrix alpha (tensor-core path only; nullptr: alpha)
  float *out32;
  void *out16;
  int32_t out16_dtype;
  float *out2_32;   // the same values + diag2 on the diagonal (nullptr: none)
  void *out2_16;
  float diag2;
  int32_t sym;      // lower-triangle tiles only, off-diagonal ones mirrored
  int32_t lower32;  // with sym: no mirrored copies in the fp32 outputs
  const DevTile *sc_tiles;   // scatter to the blocks' roles (nullptr: out32/out16)
  const DevBlock *sc_blocks;
  int32_t sc_mode;
  float sc_lr;
  int64_t N;        // columns of the output matrices
  int64_t stride;   // elements per output matrix (M * N)
};

// Store 8 values v at element index `o` of an fp32 and/or a 16-bit output
// (and mirrored, see epi_store8).
__device__ __forceinline__ void epi_put8(const EpiArgs &e, float *out32, void *out16, int64_t o, const float *v,
                                         bool mirror, int64_t om) {
  if (out32) {
    *reinterpret_cast<float4 *>(out32 + o) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4 *>(out32 + o + 4) = make_float4(v[4], v[5], v[6], v[7]);
    if (mirror && !e.lower32) {
#pragma unroll
      for (int i = 0; i < 8; ++i) out32[om + i * e.N] = v[i];
    }
  }
  if (out16) {
    uint4 u;
    if (e.out16_dtype == HIMUON_FP16) {
      __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
      *reinterpret_cast<uint4 *>(static_cast<__half *>(out16) + o) = u;
    } else {
      __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out16) + o) = u;
    }
    if (mirror) {
      const uint16_t *hs = reinterpret_cast<const uint16_t *>(&u);
      uint16_t *d = static_cast<uint16_t *>(out16);
#pragma unroll
      for (int i = 0; i < 8; ++i) d[om + i * e.N] = hs[i];
    }
  }
}

// Where the scatter epilogue puts matrix z of the batch: its tile's block
// roles, resolved once per output tile.
struct ScatterDst {
  void *out, *w;
  int64_t ldo, ldw;
  int32_t dto, dtw;
  int32_t r0, c0, h, wd, transposed;
  bool vec;   // 16-byte runs allowed for every role written
};

__device__ __forceinline__ ScatterDst scatter_dst(const EpiArgs &e, int64_t z) {
  const DevTile tl = e.sc_tiles[z];
  const DevBlock &b = e.sc_blocks[tl.block];
  ScatterDst d;
  d.out = b.ptr[kRoleOut];
  d.w = e.sc_mode == 1 ? b.ptr[kRoleW] : nullptr;
  d.ldo = b.ld[kRoleOut];
  d.ldw = b.ld[kRoleW];
  d.dto = b.dtype[kRoleOut];
  d.dtw = b.dtype[kRoleW];
  d.r0 = tl.r0;
  d.c0 = tl.c0;
  d.h = tl.h;
  d.wd = tl.w;
  d.transposed = tl.transposed;
  d.vec = (!d.out || vec8_ok(d.out, d.dto, d.ldo, tl.c0)) && (!d.w || vec8_ok(d.w, d.dtw, d.ldw, tl.c0));
  return d;
}

// Scatter 8 values (row `row`, columns col..col+7 of the n x m tile operand)
// to the block they came from: the unpack pass's element map.  Straight
// tiles write a run of a block row (one 16-byte access per role where the
// alignment allows); transposed ones write column c0 + row of the block, one
// element per row col..col+7 (a warp's lanes hold consecutive rows, so each
// of these stores is coalesced).
__device__ __forceinline__ void epi_scatter8(const EpiArgs &e, const ScatterDst &d, int64_t row, int64_t col,
                                             const float (&v)[8]) {
  if (!d.transposed) {
    if (row >= d.h || col >= d.wd) return;   // zero padding of a ragged tile
    const int64_t r = d.r0 + row, c = d.c0 + col;
    if (col + 8 <= d.wd && d.vec) {
      if (d.out) st8_16(d.out, d.dto, r * d.ldo + c, v);
      if (d.w) {
        float w[8];
        ld8_16(d.w, d.dtw, r * d.ldw + c, w);
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = fmaf(-e.sc_lr, v[i], w[i]);
        st8_16(d.w, d.dtw, r * d.ldw + c, w);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (col + i >= d.wd) break;
        if (d.out) st_elem(d.out, d.dto, r * d.ldo + c + i, v[i]);
        if (d.w) st_elem(d.w, d.dtw, r * d.ldw + c + i, fmaf(-e.sc_lr, v[i], ld_elem(d.w, d.dtw, r * d.ldw + c + i)));
      }
    }
  } else {
    if (row >= d.wd) return;   // operand row `row` is block column c0 + row
    const int64_t c = d.c0 + row;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (col + i >= d.h) break;
      const int64_t r = d.r0 + col + i;
      if (d.out) st_elem(d.out, d.dto, r * d.ldo + c, v[i]);
      if (d.w) st_elem(d.w, d.dtw, r * d.ldw + c, fmaf(-e.sc_lr, v[i], ld_elem(d.w, d.dtw, r * d.ldw + c)));
    }
  }
}

// The C term's 8 values at element index `o` of the batch (c32, or c16 in
// out16_dtype), loaded ahead of the accumulator so that a group's loads are in
// flight together.
__device__ __forceinline__ void epi_load_c8(const EpiArgs &e, int64_t o, float *cc) {
  if (e.c32) {
    const float4 c0 = *reinterpret_cast<const float4 *>(e.c32 + o);
    const float4 c1 = *reinterpret_cast<const float4 *>(e.c32 + o + 4);
    cc[0] = c0.x; cc[1] = c0.y; cc[2] = c0.z; cc[3] = c0.w;
    cc[4] = c1.x; cc[5] = c1.y; cc[6] = c1.z; cc[7] = c1.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(e.c16) + o);
    if (e.out16_dtype == HIMUON_FP16) {
      const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        cc[2 * i] = f.x;
        cc[2 * i + 1] = f.y;
      }
    } else {
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        cc[2 * i] = f.x;
        cc[2 * i + 1] = f.y;
      }
    }
  }
}

// Write 8 consecutive outputs starting at element index `o` of the batch;
// they sit in row `row`, columns col..col+7 of their matrix.  With `mirror`
// (an off-diagonal tile of a symmetric product) they also go to rows
// col..col+7, column `row` (element index `om` for the first; a warp's lanes
// hold consecutive rows, so each of these scalar stores is coalesced).
// `alpha` is the product's alpha for this matrix, `cc` the C term's values
// (epi_load_c8; nullptr: none) and `sd`, with the scatter epilogue, the
// matrix's destination (alpha and sd resolved once per output tile).
__device__ __forceinline__ void epi_store8(const EpiArgs &e, int64_t o, int64_t row, int64_t col, const float *acc,
                                           bool mirror, int64_t om, float alpha, const float *cc,
                                           const ScatterDst &sd) {
  float v[8];
  if (cc) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fmaf(alpha, acc[i], e.beta * cc[i]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = alpha * acc[i];
  }
  const bool on_diag = row >= col && row < col + 8;
  if (e.diag != 0.f && on_diag) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += (col + i == row) ? e.diag : 0.f;
  }
  if (e.sc_tiles) {
    epi_scatter8(e, sd, row, col, v);
    return;
  }
  epi_put8(e, e.out32, e.out16, o, v, mirror, om);
  if (e.out2_32 || e.out2_16) {
    if (on_diag) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] += (col + i == row) ? e.diag2 : 0.f;
    }
    epi_put8(e, e.out2_32, e.out2_16, o, v, mirror, om);
  }
}

// ---------------------------------------------------------------- tcgen05 GEMM
// A persistent kernel, one CTA per SM, computes 128 x BN output tiles (BN =
// 256 when N is a multiple of 256, and at least 2048 for a symmetric product;
// else 128: a 128 x 256 x 16 MMA reads 12 KB of operands from shared memory in
// 128 cycles where two 128 x 128 x 16 ones read 16 KB, which keeps the operand
// traffic under the shared-memory bandwidth).  Warp 0 streams the operands of
// its tiles, one after the other, through a ring of stages (TMA); warp 1
// issues each tile's MMAs into one of two TMEM accumulators; warps 2..9 drain
// the other accumulator (the previous tile) meanwhile, so the epilogue runs
// under the next tile's main loop.  Two warps share each 32-lane quarter of
// the accumulator, one per half of its columns: eight warps keep enough
// stores in flight that the epilogue of a short-K tile still hides under the
// next one's MMAs.
constexpr uint32_t kStageA = 16384;
template <int BN>
__host__ __device__ constexpr uint32_t stage_bytes() { return kStageA + BN * 128u; }
template <int BN>
__host__ __device__ constexpr int gemm_stages() { return BN == 256 ? 4 : 6; }
template <int BN>
constexpr uint32_t gemm_smem() { return gemm_stages<BN>() * stage_bytes<BN>() + 256 + 1024; }
constexpr int kGemmThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue

struct GemmTcArgs {
  int64_t K;
  uint32_t idesc;
  EpiArgs ep;
  int *status;
  int64_t tiles_per_matrix;   // output tiles of one matrix of the batch
  int64_t n_tiles;            // tiles_per_matrix * batch
  int32_t gx, gy;             // output tiles along N and M (non-symmetric products)
};

// Output tile `idx` of the launch: its matrix z and corner (m0, n0).
template <int BN>
__device__ __forceinline__ void gemm_tile(const GemmTcArgs &a, int64_t idx, int32_t &m0, int32_t &n0, int32_t &z) {
  z = static_cast<int32_t>(idx / a.tiles_per_matrix);
  const int64_t k = idx - static_cast<int64_t>(z) * a.tiles_per_matrix;
  if (a.ep.sym && BN == 128) {   // the tiles (ti, tj), tj <= ti, row by row
    int32_t ti = static_cast<int32_t>((sqrtf(8.f * static_cast<float>(k) + 1.f) - 1.f) * 0.5f);
    while ((ti + 1) * (ti + 2) / 2 <= k) ++ti;
    while (ti * (ti + 1) / 2 > k) --ti;
    m0 = ti * 128;
    n0 = static_cast<int32_t>(k - ti * (ti + 1) / 2) * 128;
  } else if (a.ep.sym) {
    // 128 x 256 tiles reaching the lower triangle: row tile ti holds
    // ti / 2 + 1 of them (columns 0 .. 256 (ti / 2) + 255), row by row
    int32_t ti = 0;
    int64_t base = 0;
    while (base + ti / 2 + 1 <= k) {
      base += ti / 2 + 1;
      ++ti;
    }
    m0 = ti * 128;
    n0 = static_cast<int32_t>(k - base) * 256;
  } else {
    // Grouped order: consecutive tiles cover bands of up to 32 row tiles, row
    // tile fastest, so the tiles in flight together share each B column panel
    // among the band's rows and keep the band's A row panels in L2 while B
    // streams through once (row-major order re-read all of B for every ~2 row
    // tiles).
    const int64_t gx = a.gx, gy = a.gy;
    const int64_t G = gy < 32 ? gy : 32;
    const int64_t per = G * gx, g = k / per, r = k % per;
    const int64_t gm = (gy - g * G) < G ? (gy - g * G) : G;
    m0 = static_cast<int32_t>((g * G + r % gm) * 128);
    n0 = static_cast<int32_t>((r / gm) * BN);
  }
}

template <int B_MN, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                   const GemmTcArgs a) {
  constexpr int kStages = gemm_stages<BN>();
  constexpr uint32_t kStageBytes = stage_bytes<BN>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + kStages * kStageBytes);
  uint64_t *empty = full + kStages;
  uint64_t *acc_full = empty + kStages;    // [2] accumulator b holds a finished tile
  uint64_t *acc_empty = acc_full + 2;      // [2] accumulator b drained by the epilogue
  uint64_t *done = acc_empty + 2;          // every MMA issued has completed
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = static_cast<int>(a.K / 64);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 8);   // one arrival per epilogue warp
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch_desc(&mapA);
    tma_prefetch_desc(&mapB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // producer: k-block `it` (counted over all of this CTA's tiles) uses stage it % kStages
    int64_t it = 0;
    bool ok = true;
    for (int64_t idx = blockIdx.x; idx < a.n_tiles && ok; idx += gridDim.x) {
      int32_t m0, n0, z;
      gemm_tile<BN>(a, idx, m0, n0, z);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = static_cast<int>(it % kStages);
        const int64_t use = it / kStages;
        if (use > 0 && !(ok = mbar_wait(empty + s, static_cast<uint32_t>((use - 1) & 1), a.status))) break;
        uint8_t *As = sm + s * kStageBytes, *Bs = As + kStageA;
        mbar_arrive_expect_tx(full + s, kStageBytes);
        tma_load_3d(As, &mapA, kb * 64, m0, z, full + s);
        if (B_MN) {   // BN / 64 boxes of 64 columns x 64 k-rows
#pragma unroll
          for (int j = 0; j < BN / 64; ++j) tma_load_3d(Bs + 8192 * j, &mapB, n0 + 64 * j, kb * 64, z, full + s);
        } else {      // one box of 64 k-columns x BN rows
          tma_load_3d(Bs, &mapB, kb * 64, n0, z, full + s);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer: tile j of this CTA accumulates in TMEM columns (j % 2) * BN ..
    int64_t it = 0, j = 0;
    bool ok = true;
    for (int64_t idx = blockIdx.x; idx < a.n_tiles && ok; idx += gridDim.x, ++j) {
      const int b = static_cast<int>(j & 1);
      if (j >= 2 && !(ok = mbar_wait(acc_empty + b, static_cast<uint32_t>(((j >> 1) - 1) & 1), a.status))) break;
      tc_fence_after();
      const uint32_t d = tmem + static_cast<uint32_t>(b * BN);
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = static_cast<int>(it % kStages);
        if (!(ok = mbar_wait(full + s, static_cast<uint32_t>((it / kStages) & 1), a.status))) break;
        tc_fence_after();
        const uint32_t as = smem_u32(sm + s * kStageBytes), bs = as + kStageA;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = sw128_desc(as + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? sw128_desc(bs + kk * 2048, 8192, 1024) : sw128_desc(bs + kk * 32, 16, 1024);
          mma_ss(d, ad, bd, a.idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(empty + s);   // the stage is free once these MMAs have read it
      }
      if (ok) mma_commit(acc_full + b);
    }
    mma_commit(done);
    mbar_wait(done, 0, a.status);   // nothing of this CTA's is in flight when TMEM is released
  } else if (warp >= 2) {
    // epilogue: symmetric products write each 128-column block below the
    // diagonal also mirrored, the diagonal block as it is, and a block above
    // the diagonal (in a 256-column tile on the diagonal) not at all: its
    // mirror image comes from the tile below
    const int q = warp & 3;                    // TMEM lanes 32 q .. 32 q + 31
    const int half = (warp - 2) >> 2;          // columns half * BN / 2 ..
    const int row = q * 32 + lane;
    const bool has_c = a.ep.c32 || a.ep.c16;
    int64_t j = 0;
    for (int64_t idx = blockIdx.x; idx < a.n_tiles; idx += gridDim.x, ++j) {
      const int b = static_cast<int>(j & 1);
      if (!mbar_wait(acc_full + b, static_cast<uint32_t>((j >> 1) & 1), a.status)) break;
      tc_fence_after();
      int32_t m0, n0, z;
      gemm_tile<BN>(a, idx, m0, n0, z);
      const int32_t ti = m0 / 128;
      const float alpha = a.ep.alpha_batch ? a.ep.alpha_batch[z] : a.ep.alpha;
      ScatterDst sd{};
      if (a.ep.sc_tiles) sd = scatter_dst(a.ep, z);
      const uint32_t taddr = tmem + static_cast<uint32_t>(b * BN) + (static_cast<uint32_t>(q * 32) << 16);
      const int64_t obase = z * a.ep.stride + static_cast<int64_t>(m0 + row) * a.ep.N + n0;
#pragma unroll 1
      for (int i = half * (BN / 64); i < (half + 1) * (BN / 64); ++i) {
        const int32_t ct = (n0 + 32 * i) / 128;   // 128-column block of the output
        if (a.ep.sym && ct > ti) break;          // above the diagonal (the tile's last block)
        const bool mirror = a.ep.sym && ct < ti;
        // the group's C loads first, all four in flight (issued one by one
        // between the stores, each waited for its own trip to memory)
        float cv[32];
        if (has_c) {
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) epi_load_c8(a.ep, obase + 32 * i + 8 * jj, cv + 8 * jj);
        }
        float v[32];
        tmem_ld32(taddr + 32 * i, v);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int64_t col = n0 + 32 * i + 8 * jj;
          epi_store8(a.ep, obase + 32 * i + 8 * jj, m0 + row, col, v + 8 * jj, mirror,
                     z * a.ep.stride + col * a.ep.N + m0 + row, alpha, has_c ? cv + 8 * jj : nullptr, sd);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + b);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// ---------------------------------------------------------------- fp32 SIMT GEMM
constexpr int kSB = 64, kSK = 16;
template <int BT>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const float *A, const float *B, int64_t K, int64_t lda,
                                                        int64_t ldb, int64_t sA, int64_t sB, EpiArgs ep) {
  __shared__ float As[kSK][kSB + 4];
  __shared__ float Bs[kSK][kSB + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t n0 = blockIdx.x * kSB, m0 = blockIdx.y * kSB, z = blockIdx.z;
  A += z * sA;
  B += z * sB;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += kSK) {
    for (int e = threadIdx.x; e < kSB * kSK; e += 256) {
      const int r = e / kSK, c = e % kSK;   // A: 64 rows x 16 k
      As[c][r] = A[(m0 + r) * lda + k0 + c];
      if (BT) Bs[c][r] = B[(n0 + r) * ldb + k0 + c];
    }
    if (!BT) {
      for (int e = threadIdx.x; e < kSB * kSK; e += 256) {
        const int r = e / kSB, c = e % kSB;  // B: 16 k rows x 64 cols
        Bs[r][c] = B[(k0 + r) * ldb + n0 + c];
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kSK; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t o = z * ep.stride + (m0 + ty * 4 + i) * ep.N + n0 + tx * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v = ep.alpha * acc[i][j];
      if (ep.c32) v = fmaf(ep.beta, ep.c32[o + j], v);
      const bool d = m0 + ty * 4 + i == n0 + tx * 4 + j;
      if (d) v += ep.diag;
      if (ep.out32) ep.out32[o + j] = v;
      if (ep.out16) st_elem(ep.out16, ep.out16_dtype, o + j, v);
      if (d) v += ep.diag2;
      if (ep.out2_32) ep.out2_32[o + j] = v;
      if (ep.out2_16) st_elem(ep.out2_16, ep.out16_dtype, o + j, v);
    }
  }
}

// ---------------------------------------------------------------- host helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over a batch of row-major [batch][rows][cols] 16-bit matrices.
bool make_batch_map(CUtensorMap *m, const Batch &b, int64_t batch, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType dt =
      b.dtype == HIMUON_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(b.cols), static_cast<cuuint64_t>(b.rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(b.cols * 2), static_cast<cuuint64_t>(b.stride * 2)};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, dt, 3, b.ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

EpiArgs to_epi(const Epilogue &e, int64_t M, int64_t N) {
  EpiArgs a;
  a.alpha = e.alpha;
  a.beta = e.beta;
  a.diag = e.diag;
  a.c32 = e.c32;
  a.c16 = e.c16;
  a.alpha_batch = e.alpha_batch;
  a.out32 = e.out32;
  a.out16 = e.out16;
  a.out16_dtype = e.out16_dtype;
  a.out2_32 = e.out2_32;
  a.out2_16 = e.out2_16;
  a.diag2 = e.diag2;
  a.sym = e.sym && M == N;
  a.lower32 = a.sym && e.lower32;
  a.sc_tiles = e.sc_tiles;
  a.sc_blocks = e.sc_blocks;
  a.sc_mode = e.sc_mode;
  a.sc_lr = e.sc_lr;
  a.N = N;
  a.stride = M * N;
  return a;
}

}  // namespace

cudaError_t gemm_tc(const Batch &A, const Batch &B, int b_trans, int64_t M, int64_t N, int64_t K, int64_t batch,
                    const Epilogue &ep, int *status, cudaStream_t stream) {
  if (M % 128 || N % 128 || K % 64 || batch < 1 || batch > 65535) return cudaErrorInvalidValue;
  GemmTcArgs a;
  a.K = K;
  a.ep = to_epi(ep, M, N);
  a.status = status;
  // 256-column tiles when N allows; for a symmetric product only from N = 2048,
  // where the tiles on the diagonal, half above it, cost at most 6% extra
  // work (at N = 1024 the extra 11% outweighed the faster MMAs: measured)
  const int BN = (N % 256 == 0 && (!a.ep.sym || N >= 2048)) ? 256 : 128;
  CUtensorMap ma, mb;
  if (!make_batch_map(&ma, A, batch, 64, 128)) return cudaErrorInvalidValue;
  if (b_trans) {
    if (!make_batch_map(&mb, B, batch, 64, static_cast<uint32_t>(BN))) return cudaErrorInvalidValue;
  } else {
    if (!make_batch_map(&mb, B, batch, 64, 64)) return cudaErrorInvalidValue;
  }
  a.idesc = idesc_f16(128, static_cast<uint32_t>(BN), A.dtype == HIMUON_FP16 ? 0u : 1u, 0, b_trans ? 0u : 1u, 0);
  a.gx = static_cast<int32_t>(N / BN);
  a.gy = static_cast<int32_t>(M / 128);
  if (a.ep.sym) {   // the tiles reaching the lower triangle (see gemm_tile)
    const int64_t nt = M / 128;
    int64_t count = 0;
    for (int64_t ti = 0; ti < nt; ++ti) count += BN == 128 ? ti + 1 : ti / 2 + 1;
    a.tiles_per_matrix = count;
  } else {
    a.tiles_per_matrix = static_cast<int64_t>(a.gx) * a.gy;
  }
  a.n_tiles = a.tiles_per_matrix * batch;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const dim3 grid(static_cast<unsigned>(std::min<int64_t>(a.n_tiles, sms)));
  cudaError_t e;
  auto go = [&](auto kern, uint32_t smem) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    count_launch();
    kern<<<grid, kGemmThreads, smem, stream>>>(ma, mb, a);
    return cudaSuccess;
  };
  if (BN == 256) e = b_trans ? go(gemm_tc_kernel<0, 256>, gemm_smem<256>()) : go(gemm_tc_kernel<1, 256>, gemm_smem<256>());
  else e = b_trans ? go(gemm_tc_kernel<0, 128>, gemm_smem<128>()) : go(gemm_tc_kernel<1, 128>, gemm_smem<128>());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t gemm_simt(const Batch &A, const Batch &B, int b_trans, int64_t M, int64_t N, int64_t K, int64_t batch,
                      const Epilogue &ep, cudaStream_t stream) {
  if (M % kSB || N % kSB || K % kSK || batch < 1 || batch > 65535) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(N / kSB), static_cast<unsigned>(M / kSB), static_cast<unsigned>(batch));
  const float *pa = static_cast<const float *>(A.ptr), *pb = static_cast<const float *>(B.ptr);
  count_launch();
  if (b_trans)
    gemm_simt_kernel<1><<<grid, 256, 0, stream>>>(pa, pb, K, A.cols, B.cols, A.stride, B.stride, to_epi(ep, M, N));
  else
    gemm_simt_kernel<0><<<grid, 256, 0, stream>>>(pa, pb, K, A.cols, B.cols, A.stride, B.stride, to_epi(ep, M, N));
  return cudaGetLastError();
}

cudaError_t launch_pack(const PackArgs &a, cudaStream_t stream) {
  dim3 grid(static_cast<unsigned>(a.parts), static_cast<unsigned>(a.n_tiles));
  count_launch();
  pack_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

__global__ void tile_scales_kernel(const float *partial, int32_t parts, int64_t n_tiles, float eps, float safety,
                                   float *inv, float *inv2) {
  const int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (t >= n_tiles) return;
  float s = 0.f;
  for (int p = 0; p < parts; ++p) s += partial[t * parts + p];   // the order normalize_kernel sums in
  const float v = 1.0f / ((sqrtf(s) + eps) * safety);
  inv[t] = v;
  inv2[t] = v * v;
}

cudaError_t launch_tile_scales(const float *partial, int32_t parts, int64_t n_tiles, float eps, float safety,
                               float *inv, float *inv2, cudaStream_t stream) {
  count_launch();
  tile_scales_kernel<<<static_cast<unsigned>((n_tiles + 255) / 256), 256, 0, stream>>>(partial, parts, n_tiles, eps,
                                                                                     safety, inv, inv2);
  return cudaGetLastError();
}

cudaError_t launch_normalize(const NormArgs &a, cudaStream_t stream) {
  const int64_t chunks = (a.elems + 8191) / 8192;
  dim3 grid(static_cast<unsigned>(chunks), static_cast<unsigned>(a.n_tiles));
  count_launch();
  normalize_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const UnpackArgs &a, cudaStream_t stream) {
  const int64_t side = a.n > a.m ? a.n : a.m;   // a tile has at most max(n, m) rows
  const int64_t parts = (side + 31) / 32;
  dim3 grid(static_cast<unsigned>(parts), static_cast<unsigned>(a.n_tiles));
  count_launch();
  unpack_kernel<<<grid, 256, 0, stream>>>(a, static_cast<int32_t>(parts));
  return cudaGetLastError();
}

}  // namespace himuon
