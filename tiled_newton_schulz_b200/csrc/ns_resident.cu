// ns_resident.cu -- tiled NS with every tile kept on chip for all K steps.
//
// The map ("Gram Newton-Schulz" page, sec. 3, Algorithm 1, applied per tile as
// in the "Hierarchical Muon" abstract):
//     X <- X / (||X||_F + eps);  per step  A = X X^T,  B = b A + c A^2,  X = a X + B X.
// Tiles up to 128 x 128 are zero-padded to 128 x 128 (exactly the same map: a
// zero border stays zero through X X^T, A^2 and B X and leaves ||X||_F alone;
// and the transpose of a tall tile is not needed because NS(X^T) = NS(X)^T).
//
// One persistent CTA per SM runs two independent tile "groups" of 4 warps each
// plus one MMA-issuing warp, so that one group's tcgen05 MMAs overlap the other
// group's TMEM -> register -> shared-memory conversions.  Per group:
//   shared memory  X_s (16-bit iterate operand, 32 KB), S_s (16-bit operand, 32 KB), W_s (32 KB)
//   tensor memory  D_P (128 cols fp32: A, then B / b), D_X (128 cols fp32 iterate)
// Per step the group runs three 128x128x128 MMAs:
//   MMA1  D_P  = X X^T                               (X_s twice, K-major)
//   MMA2  D_P += sign(c/b) S S^T,  S = r(sqrt|c/b| A)    -> D_P = A + (c/b) A^2 = B / b
//   MMA3  D_X += Bop X,  Bop = r(b D_P + (a - 1) I)      (X_s read MN-major)
// r() rounds to the 16-bit operand type (fp16 or bf16, chosen per call).
// D_X holds the fp32 iterate X_t itself, so MMA3 realises X <- a X + B X as
// X + ((a - 1) I + B) X: the fp32 part is carried exactly and only the
// correction goes through 16-bit operands.  The momentum update M' = mu M + G
// is fused into the prologue (M' written back once) and W <- W - lr O into the
// epilogue, so HBM sees one read and one write per element and role.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "layout.hpp"
#include "ptx.cuh"
#include "resident.hpp"

namespace himuon {

namespace {

constexpr int kGroupThreads = 128;
constexpr int kMmaWarp = 8;
constexpr int kThreads = 9 * 32;
constexpr uint32_t kHalf = 16384;          // one 64-column, 128-row swizzled half tile
constexpr uint32_t kOffX = 0, kOffS = 32768, kOffW = 65536, kGroupBytes = 98304;
constexpr uint32_t kOffBars = 2 * kGroupBytes;
constexpr uint32_t kSmemBytes = kOffBars + 256 + 1024;   // + alignment slack

struct Smem {
  uint8_t *base;
  __device__ uint8_t *x(int g) const { return base + g * kGroupBytes + kOffX; }
  __device__ uint8_t *s(int g) const { return base + g * kGroupBytes + kOffS; }
  __device__ uint8_t *w(int g) const { return base + g * kGroupBytes + kOffW; }
  __device__ uint64_t *bar_ld(int g) const { return reinterpret_cast<uint64_t *>(base + kOffBars) + 3 * g + 0; }
  __device__ uint64_t *bar_mma(int g) const { return reinterpret_cast<uint64_t *>(base + kOffBars) + 3 * g + 1; }
  __device__ uint64_t *bar_epi(int g) const { return reinterpret_cast<uint64_t *>(base + kOffBars) + 3 * g + 2; }
  __device__ float *red(int g) const { return reinterpret_cast<float *>(base + kOffBars + 64) + 4 * g; }
  __device__ uint32_t *tmem_slot() const { return reinterpret_cast<uint32_t *>(base + kOffBars + 128); }
  __device__ volatile int *abort_flag() const { return reinterpret_cast<volatile int *>(base + kOffBars + 132); }
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, const Smem &sm, int *status) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u && *sm.abort_flag()) return false;
  }
  set_status(status, HIMUON_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
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
__device__ __forceinline__ uint4 pack8_bf16(const float *f) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
// 16-bit operand of format F (0: fp16, 1: bf16)
template <int F>
__device__ __forceinline__ uint4 pack8_op(const float *f) {
  if (F == 1) return pack8_bf16(f);
  uint4 u;
  __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

// byte offset of 16-byte chunk cg (0..15, i.e. columns 8cg..8cg+7) of row r in
// a 128x128 bf16 tile stored as two 128B-swizzled 64-column halves.
__device__ __forceinline__ uint32_t chunk_off(uint32_t r, uint32_t cg) {
  return (cg >> 3) * kHalf + sw128_off(r, cg & 7u);
}

// Row r of a 128-column fp32 TMEM region -> scale * v (+ diag on column r) as
// 16-bit operands in the swizzled tile.  With WB the scaled fp32 values are
// also written back to the TMEM region.
template <int F, bool DIAG, bool WB>
__device__ __forceinline__ void tmem_row_to_op(uint32_t taddr, uint8_t *dst, uint32_t r, float scale, float diag) {
  const uint32_t q = r >> 5, ln = r & 31u;
#pragma unroll
  for (int i = 0; i < 4; i += 2) {
    float v0[32], v1[32];
    tmem_ld32(taddr + 32 * i, v0);
    tmem_ld32(taddr + 32 * (i + 1), v1);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      v0[e] *= scale;
      v1[e] *= scale;
    }
    if (DIAG) {
      if (q == static_cast<uint32_t>(i)) {
#pragma unroll
        for (int e = 0; e < 32; ++e) v0[e] += (static_cast<uint32_t>(e) == ln) ? diag : 0.f;
      } else if (q == static_cast<uint32_t>(i + 1)) {
#pragma unroll
        for (int e = 0; e < 32; ++e) v1[e] += (static_cast<uint32_t>(e) == ln) ? diag : 0.f;
      }
    }
    if (WB) {
      tmem_st32(taddr + 32 * i, v0);
      tmem_st32(taddr + 32 * (i + 1), v1);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      *reinterpret_cast<uint4 *>(dst + chunk_off(r, 4 * i + j)) = pack8_op<F>(v0 + 8 * j);
      *reinterpret_cast<uint4 *>(dst + chunk_off(r, 4 * (i + 1) + j)) = pack8_op<F>(v1 + 8 * j);
    }
  }
  if (WB) tmem_wait_st();
}

__device__ __forceinline__ void signal_mma(uint64_t *bar) {
  fence_proxy_async_smem();
  tc_fence_before();
  mbar_arrive(bar);
}

struct TileCoord {
  const DevBlock *blk;
  int32_t x0, y0;
};

__device__ __forceinline__ TileCoord decode_tile(const ResidentArgs &a, int64_t tile) {
  int lo = 0, hi = a.n_blocks - 1;
  while (lo < hi) {  // last block with tile_begin <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (a.blocks[mid].tile_begin <= tile) lo = mid; else hi = mid - 1;
  }
  const DevBlock *b = a.blocks + lo;
  const int64_t local = tile - b->tile_begin;
  TileCoord t;
  t.blk = b;
  t.y0 = static_cast<int32_t>(local / b->tiles_c) * b->T;
  t.x0 = static_cast<int32_t>(local % b->tiles_c) * b->T;
  return t;
}

__device__ __forceinline__ void load_tile(const CUtensorMap *m, uint8_t *dst, int32_t x0, int32_t y0, uint64_t *bar) {
  tma_load_2d(dst, m, x0, y0, bar);
  tma_load_2d(dst + kHalf, m, x0 + 64, y0, bar);
}
__device__ __forceinline__ void store_tile(const CUtensorMap *m, const uint8_t *src, int32_t x0, int32_t y0,
                                           int32_t cols) {
  tma_store_2d(m, src, x0, y0);
  if (x0 + 64 < cols) tma_store_2d(m, src + kHalf, x0 + 64, y0);
}
__device__ __forceinline__ void prefetch_tile(const CUtensorMap *m, int32_t x0, int32_t y0, int32_t cols) {
  tma_prefetch_l2_2d(m, x0, y0);
  if (x0 + 64 < cols) tma_prefetch_l2_2d(m, x0 + 64, y0);
}

// ------------------------------------------------------------------ epilogue group
template <int F>
__device__ void group_main(const ResidentArgs &a, const Smem &sm, uint32_t tmem, int g) {
  const int gt = threadIdx.x - g * kGroupThreads;   // 0..127 == tile row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t r = static_cast<uint32_t>(gt);
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t tP = tmem + lane_base + 256u * g;     // D_P
  const uint32_t tX = tP + 128u;                       // D_X
  uint8_t *Xs = sm.x(g), *Ss = sm.s(g), *Ws = sm.w(g);
  const int bar_id = 1 + g;
  const bool step_mode = a.mode == 1;
  const int64_t grid = gridDim.x;
  uint32_t it = 0, job = 0;

  for (int64_t tile = blockIdx.x + g * grid; tile < a.n_tiles; tile += 2 * grid, ++it) {
    const TileCoord tc = decode_tile(a, tile);
    const DevBlock &b = *tc.blk;
    const CUtensorMap *mIn = a.tmaps + b.tmap[kRoleIn];
    if (gt == 0) {
      bulk_wait_read0();  // the previous tile's stores have finished reading X_s / W_s
      uint32_t bytes = 2 * kHalf;
      if (step_mode) bytes += 2 * kHalf + (a.has_w ? 2 * kHalf : 0);
      mbar_arrive_expect_tx(sm.bar_ld(g), bytes);
      load_tile(mIn, Xs, tc.x0, tc.y0, sm.bar_ld(g));
      if (step_mode) {
        load_tile(a.tmaps + b.tmap[kRoleG], Ss, tc.x0, tc.y0, sm.bar_ld(g));
        if (a.has_w) load_tile(a.tmaps + b.tmap[kRoleW], Ws, tc.x0, tc.y0, sm.bar_ld(g));
      }
      const int64_t nxt = tile + 2 * grid;
      if (nxt < a.n_tiles) {  // warm L2 with this group's next tile
        const TileCoord nc = decode_tile(a, nxt);
        const DevBlock &nb = *nc.blk;
        prefetch_tile(a.tmaps + nb.tmap[kRoleIn], nc.x0, nc.y0, nb.cols);
        if (step_mode) {
          prefetch_tile(a.tmaps + nb.tmap[kRoleG], nc.x0, nc.y0, nb.cols);
          if (a.has_w) prefetch_tile(a.tmaps + nb.tmap[kRoleW], nc.x0, nc.y0, nb.cols);
        }
      }
    }
    if (!wait_or_abort(sm.bar_ld(g), it & 1u, sm, a.status)) break;

    // ---- prologue: M' = mu M + G (or the plain input), ||.||_F, fp32 copy to D_X
    float sumsq = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t off = chunk_off(r, 4 * i + j);
        float m[8];
        unpack8(*reinterpret_cast<const uint4 *>(Xs + off), m);
        if (step_mode) {
          float gg[8];
          unpack8(*reinterpret_cast<const uint4 *>(Ss + off), gg);
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] = fmaf(a.mu, m[e], gg[e]);
          *reinterpret_cast<uint4 *>(Xs + off) = pack8_bf16(m);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[8 * j + e] = m[e];
          sumsq = fmaf(m[e], m[e], sumsq);
        }
      }
      tmem_st32(tX + 32 * i, v);
    }
    tmem_wait_st();
    if (step_mode) {
      fence_proxy_async_smem();
      named_bar_sync(bar_id, kGroupThreads);
      if (gt == 0) {
        store_tile(mIn, Xs, tc.x0, tc.y0, b.cols);
        bulk_commit();
      }
    }
    sumsq = warp_sum(sumsq);
    if (lane == 0) sm.red(g)[warp & 3] = sumsq;
    named_bar_sync(bar_id, kGroupThreads);
    const float total = sm.red(g)[0] + sm.red(g)[1] + sm.red(g)[2] + sm.red(g)[3];
    const float rho = (sqrtf(total) + a.eps) * a.safety;
    const float inv_rho = 1.0f / rho;
    if (step_mode && gt == 0) bulk_wait_read0();   // M' has left X_s
    named_bar_sync(bar_id, kGroupThreads);

    // ---- X_0 = M' / rho: operand copy to X_s, fp32 copy back to D_X
    tmem_row_to_op<F, false, true>(tX, Xs, r, inv_rho, 0.f);
    signal_mma(sm.bar_epi(g));

    bool ok = true;
    for (int t = 0; t < a.K && ok; ++t) {
      const ResidentStep &st = a.step[t];
      // after MMA1: S = r(s A)
      if (!(ok = wait_or_abort(sm.bar_mma(g), job++ & 1u, sm, a.status))) break;
      tc_fence_after();
      tmem_row_to_op<F, false, false>(tP, Ss, r, st.s, 0.f);
      signal_mma(sm.bar_epi(g));
      // after MMA2: Bop = r(beta D_P + (a - 1) I)
      if (!(ok = wait_or_abort(sm.bar_mma(g), job++ & 1u, sm, a.status))) break;
      tc_fence_after();
      tmem_row_to_op<F, true, false>(tP, Ss, r, st.beta, st.am1);
      signal_mma(sm.bar_epi(g));
      // after MMA3: next operand X_t = r(D_X)
      if (!(ok = wait_or_abort(sm.bar_mma(g), job++ & 1u, sm, a.status))) break;
      tc_fence_after();
      if (t + 1 < a.K) {
        tmem_row_to_op<F, false, false>(tX, Xs, r, 1.f, 0.f);
        signal_mma(sm.bar_epi(g));
      }
    }
    if (!ok) break;

    // ---- epilogue: O = D_X;  W <- W - lr O
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v[32];
      tmem_ld32(tX + 32 * i, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t off = chunk_off(r, 4 * i + j);
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = v[8 * j + e];
        if (a.has_o) *reinterpret_cast<uint4 *>(Xs + off) = pack8_bf16(o);
        if (a.has_w) {
          float w[8];
          unpack8(*reinterpret_cast<const uint4 *>(Ws + off), w);
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = fmaf(-a.lr, o[e], w[e]);
          *reinterpret_cast<uint4 *>(Ws + off) = pack8_bf16(w);
        }
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(bar_id, kGroupThreads);
    if (gt == 0) {
      if (a.has_o) store_tile(a.tmaps + b.tmap[kRoleOut], Xs, tc.x0, tc.y0, b.cols);
      if (a.has_w) store_tile(a.tmaps + b.tmap[kRoleW], Ws, tc.x0, tc.y0, b.cols);
      bulk_commit();
    }
  }
  if (gt == 0) bulk_wait0();
}

// ------------------------------------------------------------------ MMA issuer
__device__ __forceinline__ uint64_t desc_k(uint32_t base, int kk) {
  // K-major operand: 128 rows x 128 bf16, two swizzled 64-column halves;
  // k-step kk covers columns 16kk..16kk+15.
  return sw128_desc(base + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, int kk) {
  // The same storage read MN-major (rows are K): k-step kk covers rows
  // 16kk..16kk+15; the two 64-column halves are kHalf apart.
  return sw128_desc(base + kk * 2048, kHalf, 1024);
}

template <int F>
__device__ void mma_main(const ResidentArgs &a, const Smem &sm, uint32_t tmem) {
  const int64_t grid = gridDim.x;
  int64_t jobs[2], done[2] = {0, 0};
  for (int g = 0; g < 2; ++g) {
    const int64_t first = blockIdx.x + g * grid;
    const int64_t tiles = first < a.n_tiles ? (a.n_tiles - first + 2 * grid - 1) / (2 * grid) : 0;
    jobs[g] = tiles * 3 * a.K;
  }
  const uint32_t idesc1 = idesc_f16(128, 128, F, 0, 0, 0);
  const uint32_t idesc3 = idesc_f16(128, 128, F, 0, 1, 0);
  uint32_t idle = 0;
  while (done[0] < jobs[0] || done[1] < jobs[1]) {
    bool progressed = false;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      if (done[g] >= jobs[g] || !mbar_try_wait(sm.bar_epi(g), static_cast<uint32_t>(done[g] & 1))) continue;
      tc_fence_after();
      const int type = static_cast<int>(done[g] % 3);
      const int t = static_cast<int>((done[g] / 3) % a.K);
      const uint32_t xs = smem_u32(sm.x(g)), ss = smem_u32(sm.s(g));
      const uint32_t dP = tmem + 256u * g, dX = dP + 128u;
      if (type == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(dP, desc_k(xs, kk), desc_k(xs, kk), idesc1, kk > 0);
      } else if (type == 1) {
        const ResidentStep &st = a.step[t];
        const uint32_t idesc2 = idesc_f16(128, 128, F, 0, 0, st.neg2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(dP, desc_k(ss, kk), desc_k(ss, kk), idesc2, st.acc2 | (kk > 0));
      } else {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ss(dX, desc_k(ss, kk), desc_mn(xs, kk), idesc3, 1u);
      }
      mma_commit(sm.bar_mma(g));
      ++done[g];
      progressed = true;
    }
    if (progressed) {
      idle = 0;
    } else if (++idle > kSpinLimit || ((idle & 1023u) == 1023u && *sm.abort_flag())) {
      if (!*sm.abort_flag()) set_status(a.status, HIMUON_ERR_TIMEOUT);
      *sm.abort_flag() = 1;
      break;
    }
  }
}

template <int F>
__global__ void __launch_bounds__(kThreads, 1) ns_resident_kernel(const __grid_constant__ ResidentArgs args) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(sm.bar_ld(g), 1);
      mbar_init(sm.bar_mma(g), 1);
      mbar_init(sm.bar_epi(g), kGroupThreads);
    }
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sm.tmem_slot(), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();

  if (warp < kMmaWarp) {
    group_main<F>(args, sm, tmem, warp >> 2);
  } else if ((threadIdx.x & 31) == 0) {
    mma_main<F>(args, sm, tmem);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int resident_smem_bytes() { return static_cast<int>(kSmemBytes); }

void make_resident_steps(ResidentArgs &args, const float *coeffs, int K) {
  // MMA2 leaves D_P = B / beta with beta = b (beta = 1 when b = 0, in which
  // case MMA2 overwrites A with c A^2): S = r(sqrt|c / beta| A) and the sign of
  // c / beta goes on MMA2's A operand.  MMA3 then adds r(beta D_P + (a-1) I) X.
  for (int t = 0; t < K; ++t) {
    const double a = coeffs[3 * t], b = coeffs[3 * t + 1], c = coeffs[3 * t + 2];
    const double beta = (b != 0.0) ? b : 1.0;
    const double ratio = c / beta;
    ResidentStep &st = args.step[t];
    st.s = static_cast<float>(sqrt(fabs(ratio)));
    st.neg2 = ratio < 0.0 ? 1u : 0u;
    st.acc2 = (b != 0.0) ? 1u : 0u;
    st.beta = static_cast<float>(beta);
    st.am1 = static_cast<float>(a - 1.0);
  }
}

template <int F>
static cudaError_t launch_fmt(const ResidentArgs &args, int grid, cudaStream_t stream) {
  // The shared-memory opt-in is per device; setting it again is cheap.
  cudaError_t e = cudaFuncSetAttribute(ns_resident_kernel<F>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  count_launch();
  ns_resident_kernel<F><<<grid, kThreads, kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_ns_resident(const ResidentArgs &args, int grid, cudaStream_t stream) {
  return args.op_fmt == 0 ? launch_fmt<0>(args, grid, stream) : launch_fmt<1>(args, grid, stream);
}

}  // namespace himuon
