// ns_resident.cu -- tiled NS with every tile kept on chip for all K steps.
//
// The map ("Gram Newton-Schulz" page, sec. 3, Algorithm 1, applied per tile as
// in the "Hierarchical Muon" abstract):
//     X <- X / (||X||_F + eps);  per step  A = X X^T,  B = b A + c A^2,  X = a X + B X.
// Tiles up to 128 x 128 are zero-padded to 128 x 128 (exactly the same map: a
// zero border stays zero through X X^T, A^2 and B X and leaves ||X||_F alone;
// and the transpose of a tall tile is not needed because NS(X^T) = NS(X)^T).
// For T = 64 and T = 32, P = 128 / T consecutive tiles share one "super-tile",
// stacked along M as rows T j .. T j + T - 1 of a 128 x T operand, each
// normalised by its own norm.  The Gram and square products then run with
// K = T (D_P = Xs Xs^T, 128 x 128: its diagonal T x T blocks are the tiles'
// own products, the rest is never read), and the update D_X = Bop Xs with
// K = 128 and N = T, where the packed A operand Bop is block-diagonal (zeros
// outside each row's tile), so each tile goes through exactly its own map
// with 2x (T = 64) or 4x (T = 32) the MMA work of its own products.
//
// One persistent CTA per SM runs two independent tile "groups" of 8 warps
// (two per TMEM lane quarter, each owning 64 of a row's 128 columns), so that
// one group's tcgen05 MMAs overlap the other group's TMEM -> register ->
// shared-memory conversions.  Each group issues its own MMAs from one thread
// right after a group-wide named barrier (no hand-off to a separate MMA warp);
// that thread's tcgen05.commit tracks exactly its group's MMAs.  Per group:
//   shared memory  X_s (16-bit iterate operand, 32 KB), S_s (16-bit operand, 32 KB), W_s (32 KB)
//   tensor memory  D_P (128 cols fp32: A, then B / b), D_X (128 cols fp32: the iterate)
// Per step the group runs three 128x128x128 MMAs, every A operand read from
// TMEM and every B operand from shared memory.  The operand carries the
// iterate scaled, Xg = g X with g = sqrt|c/b|, which is what lets S go to
// the tensor cores without a multiply of its own:
//   MMA1  D_P  = Xg Xg^T = g^2 A                 A: Xg (packed in D_X),  B: X_s (K-major)
//   MMA2  D_P += sign(c/b) S S^T,  S = r(D_P)   A: S (packed in D_X),   B: S_s
//                                               -> D_P = g^2 (A + (c/b) A^2) = g^2 B / b
//   MMA3  D_X  = Bop Xg,  Bop = r((b/g^2) D_P + a I) = r(a I + B)
//                                               A: Bop (packed in D_P), B: X_s (MN-major)
// so D_X = g X_{t+1}, which is the next step's operand as it stands (a ratio
// g_{t+1}/g_t is applied when the coefficients change; O = D_X / g).  r()
// rounds to the 16-bit operand type (fp16 or bf16, chosen per call); every
// operand is still one rounding of an fp32 value, with the relative error
// bound of the unscaled iteration (g = 0.65 for the quintic coefficients keeps
// fp16 operands far from its range limits).  MMA3 forms the whole update
// X <- a X + B X = (a I + B) X with fp32 accumulation.  The conversions are
// partly bound by the SM's arithmetic pipes, which is why S and X carry no
// multiply and the diagonal a I is added only in the 32 columns that hold it.  A 16-bit operand is packed two per 32-bit TMEM column in
// place: each thread, having read its 64 fp32 columns of a region, writes
// their 16-bit values to the first 32 of those columns (nobody else reads
// them), or into D_X while D_X holds nothing live.  Keeping A operands out of
// shared memory halves the operand traffic there (N = 128 MMAs with both
// operands in shared memory run at the shared-memory bandwidth limit).
// Operand type.  The call asks for bf16 or fp16 operands.  A bf16 call still
// rounds to fp16 the operands of a super-tile whose tiles all have a short
// side of at most 64 (T = 64 and 32, and ragged edge tiles): rounding the
// operands of such tiles to bf16's 8 significant bits moves their output
// singular values by up to ~0.1, where fp16's 11 bits keep them within ~0.01,
// at the same tensor-core rate.  A tile whose normalised norm is below 2^-10
// (input norm far below eps) keeps bf16, whose range fp16 lacks.  The choice
// is made per super-tile at run time, after its norms are known.
//
// The momentum update M' = mu M + G is fused into the prologue (M' written
// back once) and W <- W - lr O into the epilogue, so HBM sees one read and one
// write per element and role.  The next tile's inputs are loaded (TMA) as soon
// as this tile's last MMA has released X_s / S_s, under the final epilogue; W
// lands in its own buffer.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include <vector>

#include "layout.hpp"
#include "onchip.cuh"
#include "ptx.cuh"
#include "resident.hpp"

namespace himuon {

namespace {

using namespace onchip;

constexpr int kGroupWarps = 8;
constexpr int kGroupThreads = kGroupWarps * 32;
constexpr int kIssuerWarp = 2 * kGroupWarps;          // warp 16 issues every MMA
constexpr int kThreads = 2 * kGroupThreads + 32;
constexpr uint32_t kHalf = 16384;          // one 64-column, 128-row swizzled half tile
constexpr uint32_t kOffX = 0, kOffS = 32768, kOffW = 65536, kGroupBytes = 98304;
constexpr uint32_t kOffBars = 2 * kGroupBytes;
constexpr int kMaxSmemBlocks = 256;        // block tables up to this size live in shared memory
constexpr int kMaxPack = 4;                // tiles per super-tile (T = 32)
constexpr uint32_t kOffCoords = kOffBars + 512;                    // 2 groups x 2 x kMaxPack TileCoords
constexpr uint32_t kCoordBytes = 48;
constexpr uint32_t kOffBlocks = kOffCoords + 2 * 2 * kMaxPack * kCoordBytes;
constexpr uint32_t kSmemBytes = kOffBlocks + kMaxSmemBlocks * 24 + 1024;   // + alignment slack

struct Smem {
  uint8_t *base;
  __device__ uint8_t *x(int g) const { return base + g * kGroupBytes + kOffX; }
  __device__ uint8_t *s(int g) const { return base + g * kGroupBytes + kOffS; }
  __device__ uint8_t *w(int g) const { return base + g * kGroupBytes + kOffW; }
  __device__ uint64_t *bar(int g, int i) const { return reinterpret_cast<uint64_t *>(base + kOffBars) + 8 * g + i; }
  __device__ uint64_t *bar_ld(int g) const { return bar(g, 0); }    // M (or input) and G landed
  __device__ uint64_t *bar_w(int g) const { return bar(g, 1); }     // W landed
  __device__ uint64_t *bar_mma(int g) const { return bar(g, 2); }   // the group's MMA job finished
  __device__ uint64_t *bar_never(int g) const { return bar(g, 3); } // never arrived on (stall self-test)
  __device__ uint64_t *bar_ready(int g) const { return bar(g, 4); } // the operands of the group's next job are written
  __device__ uint64_t *bar_pro(int g) const { return bar(g, 5); }   // prologue: M' and the partial norms written
  __device__ uint64_t *bar_epi(int g) const { return bar(g, 6); }   // epilogue: W' / O staged for the stores
  __device__ float *red(int g) const { return reinterpret_cast<float *>(base + kOffBars + 128) + kGroupWarps * g; }
  __device__ uint32_t *tmem_slot() const { return reinterpret_cast<uint32_t *>(base + kOffBars + 192); }
  __device__ volatile int *abort_flag() const { return reinterpret_cast<volatile int *>(base + kOffBars + 196); }
  // operand type of the group's current super-tile (1: fp16), for the issuer
  __device__ volatile int *fmt16(int g) const { return reinterpret_cast<volatile int *>(base + kOffBars + 200) + g; }
  __device__ SBlock *blocks() const { return reinterpret_cast<SBlock *>(base + kOffBlocks); }
  // current (i = 0) / next (i = 1) super-tile's tile coordinates of group g,
  // kMaxPack each (read and written by the group's issuing thread only)
  __device__ TileCoord *coord(int g, int i) const {
    return reinterpret_cast<TileCoord *>(base + kOffCoords) + (2 * g + i) * kMaxPack;
  }
};

// Bounded wait that also gives up as soon as another thread of the CTA has
// raised the abort flag (after its own wait timed out).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, const Smem &sm, int *status) {
  return onchip::wait_or_abort(bar, parity, sm.abort_flag(), status);
}

// This thread's 64 columns (half `hf`) of row r of the 128-column fp32 TMEM
// region at `src` -> r(scale * v), written twice: to the swizzled shared tile
// (B operand) and packed to TMEM columns [64 hf, 64 hf + 32) of the region at
// `pk` (A operand).  `pk` may equal `src`: the thread reads all 64 columns
// before it writes the first 32.
template <int F, bool SCALE>
__device__ __forceinline__ void tmem_row_to_op(uint32_t src, uint32_t pk, uint8_t *dst, uint32_t r, uint32_t hf,
                                               float scale) {
  // 32 columns at a time keeps the live register set small (no spills)
  uint8_t *row = dst + hf * kHalf;
  const uint32_t c0 = 64u * hf;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float v[32];
    tmem_ld32(src + c0 + 32 * i, v);
    tmem_wait_ld();
    uint32_t p[16];
#pragma unroll
    for (int e = 0; e < 16; ++e)
      p[e] = SCALE ? pack2_op<F>(v[2 * e] * scale, v[2 * e + 1] * scale) : pack2_op<F>(v[2 * e], v[2 * e + 1]);
    tmem_st16(pk + c0 + 16 * i, p);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4 *>(row + sw128_off(r, 4 * i + j)) = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
  }
  tmem_wait_st();
}

// Bop = r(beta * D_P + diag * I) for this thread's 64 columns of row r,
// packed two per 32-bit word into TMEM columns [64 hf, 64 hf + 32) of D_P
// (columns this thread has already read; nobody else reads them).
// Row r = 32 q + lane: its diagonal element lies in column half r / 64 = q / 2,
// 32-column chunk q % 2 of that half, position lane -- so whether a warp's
// chunk holds it is uniform across the warp, and only that chunk pays for
// the per-element test.
template <int F>
__device__ __forceinline__ void tmem_row_to_tmem_op(uint32_t taddr, uint32_t r, uint32_t hf, float beta, float diag) {
  const uint32_t c0 = 64u * hf;
  const uint32_t lane = r & 31u;
  const uint32_t dchunk = ((r >> 6) == hf) ? ((r >> 5) & 1u) : 2u;   // chunk holding the diagonal (2: none)
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float v[32];
    tmem_ld32(taddr + c0 + 32 * i, v);
    tmem_wait_ld();
    uint32_t p[16];
    if (dchunk == static_cast<uint32_t>(i)) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a0 = fmaf(beta, v[2 * e], lane == 2u * e ? diag : 0.f);
        const float a1 = fmaf(beta, v[2 * e + 1], lane == 2u * e + 1u ? diag : 0.f);
        p[e] = pack2_op<F>(a0, a1);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) p[e] = pack2_op<F>(beta * v[2 * e], beta * v[2 * e + 1]);
    }
    tmem_st16(taddr + c0 + 16 * i, p);   // columns [c0, c0 + 32) were read before any is written
  }
  tmem_wait_st();
}

// ---- stacked super-tiles of two 64 x 64 tiles (P = 2)
// The tiles sit on top of each other as rows 64 j .. 64 j + 63 of a 128 x 64
// operand (the TMA staging layout already is that: one 128-byte swizzled
// block).  The warp of half hf of a row covers its columns 32 hf .. 32 hf + 31.
// v (those 32 fp32 values) -> r(scale v): packed to TMEM columns
// pa + 16 hf .. pa + 16 hf + 15 (K values 32 hf .. 32 hf + 31 of the A
// operand) and K-major to row r of `dst`.
template <int F, bool SCALE>
__device__ __forceinline__ void stack_row_to_op(const float (&v)[32], uint32_t pa, uint8_t *dst, uint32_t r,
                                                uint32_t hf, float scale) {
  uint32_t p[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    p[e] = SCALE ? pack2_op<F>(v[2 * e] * scale, v[2 * e + 1] * scale) : pack2_op<F>(v[2 * e], v[2 * e + 1]);
  tmem_st16(pa + 16u * hf, p);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    *reinterpret_cast<uint4 *>(dst + sw128_off(r, 4u * hf + j)) = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
  tmem_wait_st();
}
template <int F, bool SCALE>
__device__ __forceinline__ void stack_tmem_to_op(uint32_t src, uint32_t pa, uint8_t *dst, uint32_t r, uint32_t hf,
                                                 float scale) {
  float v[32];
  tmem_ld32(src, v);
  tmem_wait_ld();
  stack_row_to_op<F, SCALE>(v, pa, dst, r, hf, scale);
}
// The block-diagonal A operand of the update, Bop = r(beta D_P + diag I) on
// row r's tile (tile r / 64, whose K values are packed at columns
// 32 (r / 64) .. + 31) and zeros on the other tile's K values.  The warp of
// half hf writes packed columns pa + 32 hf .. + 31: the Bop values when they
// are its row's tile's (read from D_P columns 64 (r / 64) .. + 63), else zeros.
template <int F>
__device__ __forceinline__ void stack_row_to_bop(uint32_t tp, uint32_t pa, uint32_t r, uint32_t hf, float beta,
                                                 float diag) {
  const uint32_t jr = r >> 6;            // the same in the whole warp
  uint32_t p[16];
  if (hf == jr) {
    const uint32_t lane = r & 31u, dchunk = (r >> 5) & 1u;   // diagonal: chunk (r % 64) / 32, position r % 32
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float v[32];
      tmem_ld32(tp + 64u * jr + 32u * i, v);
      tmem_wait_ld();
      if (dchunk == static_cast<uint32_t>(i)) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a0 = fmaf(beta, v[2 * e], lane == 2u * e ? diag : 0.f);
          const float a1 = fmaf(beta, v[2 * e + 1], lane == 2u * e + 1u ? diag : 0.f);
          p[e] = pack2_op<F>(a0, a1);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) p[e] = pack2_op<F>(beta * v[2 * e], beta * v[2 * e + 1]);
      }
      tmem_st16(pa + 32u * hf + 16u * i, p);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) p[e] = 0u;
    tmem_st16(pa + 32u * hf, p);
    tmem_st16(pa + 32u * hf + 16u, p);
  }
  tmem_wait_st();
}

// ---- stacked super-tiles of four 32 x 32 tiles (P = 4)
// Rows 32 j .. 32 j + 31 of a 128 x 32 operand, K-major with 64-byte rows and
// the 64-byte swizzle (again the TMA staging layout); the warp of half hf of a
// row covers its columns 16 hf .. 16 hf + 15.
__device__ __forceinline__ uint32_t sw64_off(uint32_t r, uint32_t c) { return r * 64u + ((c ^ ((r >> 1) & 3u)) << 4); }
template <int F>
__device__ __forceinline__ void stack4_tmem_to_op(uint32_t src, uint32_t pa, uint8_t *dst, uint32_t r, uint32_t hf,
                                                  float scale) {
  float v[16];
  tmem_ld16(src, v);
  tmem_wait_ld();
  uint32_t p[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) p[e] = pack2_op<F>(v[2 * e] * scale, v[2 * e + 1] * scale);
  tmem_st8(pa + 8u * hf, p);
#pragma unroll
  for (int j = 0; j < 2; ++j)
    *reinterpret_cast<uint4 *>(dst + sw64_off(r, 2u * hf + j)) = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
  tmem_wait_st();
}
// The block-diagonal A operand of the update for P = 4: row r's tile
// j = r / 32 has its K values packed at columns 16 j .. 16 j + 15; the warp of
// half hf writes packed columns pa + 32 hf .. + 31 (tiles 2 hf and 2 hf + 1).
template <int F>
__device__ __forceinline__ void stack4_row_to_bop(uint32_t tp, uint32_t pa, uint32_t r, uint32_t hf, float beta,
                                                  float diag) {
  const uint32_t jr = r >> 5;            // the same in the whole warp
  uint32_t z[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) z[e] = 0u;
  if ((jr >> 1) == hf) {
    const uint32_t lane = r & 31u;       // the diagonal element's column in the tile
    float v[32];
    tmem_ld32(tp + 32u * jr, v);
    tmem_wait_ld();
    uint32_t p[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float a0 = fmaf(beta, v[2 * e], lane == 2u * e ? diag : 0.f);
      const float a1 = fmaf(beta, v[2 * e + 1], lane == 2u * e + 1u ? diag : 0.f);
      p[e] = pack2_op<F>(a0, a1);
    }
    tmem_st16(pa + 32u * hf + 16u * (jr & 1u), p);
    tmem_st16(pa + 32u * hf + 16u * (1u - (jr & 1u)), z);
  } else {
    tmem_st16(pa + 32u * hf, z);
    tmem_st16(pa + 32u * hf + 16u, z);
  }
  tmem_wait_st();
}

__device__ __forceinline__ bool use_smem_blocks(const ResidentArgs &a) {
  return a.smem_blocks != 0 && a.n_blocks <= kMaxSmemBlocks;
}

__device__ __forceinline__ TileCoord decode_tile(const ResidentArgs &a, const Smem &sm, int64_t tile, int hint = -1) {
  return onchip::decode_tile(a, use_smem_blocks(a) ? sm.blocks() : nullptr, tile, hint);
}

// Staged tiles in shared memory (TMA boxes; the swizzle is applied by TMA):
//   P = 1: one 128 x 128 tile as two 64-column halves, 128-byte swizzle;
//   P = 2: sub-tile j (64 x 64) at j * 8 KB, 128-byte rows, 128-byte swizzle;
//   P = 4: sub-tile j (32 x 32) at j * 2 KB, 64-byte rows, 64-byte swizzle.
template <int P>
__device__ __forceinline__ uint32_t stage_off(uint32_t j, uint32_t row, uint32_t c) {
  if (P == 1) return (c >> 3) * kHalf + sw128_off(row, c & 7u);
  if (P == 2) return j * 8192u + sw128_off(row, c);
  return j * 2048u + row * 64u + ((c ^ ((row >> 1) & 3u)) << 4);
}
template <int P>
__device__ __forceinline__ void load_tile(const CUtensorMap *m, uint8_t *dst, const TileCoord &t, int j,
                                          uint64_t *bar) {
  if (P == 1) {
    tma_load_2d(dst, m, t.x0, t.y0, bar);
    tma_load_2d(dst + kHalf, m, t.x0 + 64, t.y0, bar);
  } else {
    tma_load_2d(dst + stage_off<P>(j, 0, 0), m, t.x0, t.y0, bar);
  }
}
template <int P>
__device__ __forceinline__ void store_tile(const CUtensorMap *m, const uint8_t *src, const TileCoord &t, int j) {
  if (P == 1) {
    tma_store_2d(m, src, t.x0, t.y0);
    if (t.x0 + 64 < t.cols) tma_store_2d(m, src + kHalf, t.x0 + 64, t.y0);
  } else {
    tma_store_2d(m, src + stage_off<P>(j, 0, 0), t.x0, t.y0);
  }
}
template <int P>
__device__ __forceinline__ void prefetch_tile(const CUtensorMap *m, const TileCoord &t) {
  tma_prefetch_l2_2d(m, t.x0, t.y0);
  if (P == 1 && t.x0 + 64 < t.cols) tma_prefetch_l2_2d(m, t.x0 + 64, t.y0);
}

// bytes one role's TMA boxes bring in for tile coordinate t
template <int P>
__device__ __forceinline__ uint32_t tile_bytes() { return P == 1 ? 2 * kHalf : (128 / P) * (128 / P) * 2; }

// M (or the NS input) -> X_s and, for a momentum step, G -> S_s, for every
// tile of the super-tile.
template <int P>
__device__ __forceinline__ void issue_mg(const ResidentArgs &a, const Smem &sm, int g, const TileCoord *t) {
  const bool step_mode = a.mode == 1;
  uint32_t bytes = 0;
#pragma unroll
  for (int j = 0; j < P; ++j)
    if (t[j].blk >= 0) bytes += (step_mode ? 2 : 1) * tile_bytes<P>();
  mbar_arrive_expect_tx(sm.bar_ld(g), bytes);
#pragma unroll
  for (int j = 0; j < P; ++j) {
    if (t[j].blk < 0) continue;
    load_tile<P>(a.tmaps + t[j].tm[kRoleIn], sm.x(g), t[j], j, sm.bar_ld(g));
    if (step_mode) load_tile<P>(a.tmaps + t[j].tm[kRoleG], sm.s(g), t[j], j, sm.bar_ld(g));
  }
}
template <int P>
__device__ __forceinline__ void issue_w(const ResidentArgs &a, const Smem &sm, int g, const TileCoord *t) {
  uint32_t bytes = 0;
#pragma unroll
  for (int j = 0; j < P; ++j)
    if (t[j].blk >= 0) bytes += tile_bytes<P>();
  mbar_arrive_expect_tx(sm.bar_w(g), bytes);
#pragma unroll
  for (int j = 0; j < P; ++j)
    if (t[j].blk >= 0) load_tile<P>(a.tmaps + t[j].tm[kRoleW], sm.w(g), t[j], j, sm.bar_w(g));
}
// coordinates of the P tiles of super-tile `st` (tile P st + j; blk = -1 past the end)
template <int P>
__device__ __forceinline__ void decode_super(const ResidentArgs &a, const Smem &sm, int64_t st, TileCoord *out) {
#pragma unroll
  for (int j = 0; j < P; ++j) out[j] = decode_tile(a, sm, P * st + j, j == 0 ? -1 : out[j - 1].blk);
}

// ------------------------------------------------------------------ MMA issue
// Shared-memory descriptors differ only in the start-address field (bits
// 0..13, address >> 4; every address here is below 256 KB), so each one is a
// fixed template plus a per-operand address and a compile-time offset.
//   K-major operand (X_s, S_s): 128 rows x 128 16-bit values, two swizzled
//   64-column halves; k-step kk covers columns 16kk..16kk+15.
//   MN-major view of X_s (its rows are K): k-step kk covers rows 16kk..16kk+15,
//   the two 64-column halves are kHalf apart.
__device__ __forceinline__ uint64_t desc_k(uint64_t tmpl, uint32_t base4, int kk) {
  return tmpl + base4 + static_cast<uint32_t>(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
}
__device__ __forceinline__ uint64_t desc_mn(uint64_t tmpl, uint32_t base4, int kk) {
  return tmpl + base4 + static_cast<uint32_t>((kk * 2048) >> 4);
}

enum Job { kJobGram = 0, kJobSquare = 1, kJobUpdate = 2 };

// All threads of the group have written (and fenced) the operands of `job`:
// one thread issues its eight 128x128x16 MMAs and commits them to bar_mma.
// f16: the operands are fp16 (else bf16).
template <int JOB, int P>
__device__ __forceinline__ void group_issue_mmas(const Smem &sm, int g, uint32_t dP, const ResidentStep *st, bool f16);

// A warp of group g has written (and fenced) its share of the operands of
// the group's next job: its lane 0 arrives on the group's ready barrier, which
// completes once all eight warps have arrived; the issuer warp then issues.
__device__ __forceinline__ void group_ready(const Smem &sm, int g, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(sm.bar_ready(g));
}

// Bounded group-wide barrier on an mbarrier of count kGroupWarps (one arrival
// per warp); unlike a named barrier it never hangs a thread whose partners
// have stopped after a failure.
__device__ __forceinline__ bool group_sync(uint64_t *bar, uint32_t parity, const Smem &sm, int lane, int *status) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  return wait_or_abort(bar, parity, sm, status);
}

template <int JOB, int P>
__device__ __forceinline__ void group_issue_mmas(const Smem &sm, int g, uint32_t dP, const ResidentStep *st, bool f16) {
  tc_fence_after();
  const uint64_t tk = sw128_desc(0, 16, 1024);
  const uint32_t dX = dP + 128u;
  if (P == 2) {
    // Two 64 x 64 tiles stacked along M (rows 64 j .. 64 j + 63 of a 128 x 64
    // operand; X_s / S_s hold it K-major, one 128-byte swizzled block):
    //   Gram / square  D_P (128 x 128) += Xs Xs^T, K = 64: the diagonal 64 x 64
    //                  blocks are the two tiles' products, the rest is unused;
    //   update         D_X (128 x 64) = Bop Xs, K = 128, Bop block-diagonal
    //                  (zeros outside the tiles' blocks), Xs read MN-major.
    // Every A operand is packed at TMEM columns dP + 192 .. dP + 255.
    const uint32_t dA = dP + 192u;
    if (JOB == kJobGram) {
      const uint32_t x4 = smem_u32(sm.x(g)) >> 4;
      const uint32_t id = f16 ? idesc_f16(128, 128, 0, 0, 0, 0) : idesc_f16(128, 128, 1, 0, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_ts(dP, dA + 8 * kk, desc_k(tk, x4, kk), id, kk > 0);
    } else if (JOB == kJobSquare) {
      const uint32_t s4 = smem_u32(sm.s(g)) >> 4;
      const uint32_t id = idesc_f16(128, 128, f16 ? 0 : 1, 0, 0, st->neg2);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) mma_ts(dP, dA + 8 * kk, desc_k(tk, s4, kk), id, st->acc2 | (kk > 0));
    } else {
      const uint32_t x4 = smem_u32(sm.x(g)) >> 4;
      const uint64_t tmn = sw128_desc(0, kHalf, 1024);
      const uint32_t id = f16 ? idesc_f16(128, 64, 0, 0, 1, 0) : idesc_f16(128, 64, 1, 0, 1, 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) mma_ts(dX, dA + 8 * kk, desc_mn(tmn, x4, kk), id, kk > 0);
    }
    mma_commit(sm.bar_mma(g));
    return;
  }
  if (P == 4) {
    // Four 32 x 32 tiles stacked along M (rows 32 j .. 32 j + 31 of a 128 x 32
    // operand, K-major with 64-byte rows and the 64-byte swizzle): Gram and
    // square products with K = 32, the update with K = 128 (Bop
    // block-diagonal) and N = 32, Xs read MN-major.
    const uint32_t dA = dP + 192u;
    const uint64_t tk64 = sw64_desc(0, 16, 512);
    if (JOB == kJobGram) {
      const uint32_t x4 = smem_u32(sm.x(g)) >> 4;
      const uint32_t id = f16 ? idesc_f16(128, 128, 0, 0, 0, 0) : idesc_f16(128, 128, 1, 0, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) mma_ts(dP, dA + 8 * kk, tk64 + x4 + 2 * kk, id, kk > 0);
    } else if (JOB == kJobSquare) {
      const uint32_t s4 = smem_u32(sm.s(g)) >> 4;
      const uint32_t id = idesc_f16(128, 128, f16 ? 0 : 1, 0, 0, st->neg2);
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) mma_ts(dP, dA + 8 * kk, tk64 + s4 + 2 * kk, id, st->acc2 | (kk > 0));
    } else {
      // K rows 16 kk .. 16 kk + 15: 1024 bytes on; one 32-column atom in N
      const uint32_t x4 = smem_u32(sm.x(g)) >> 4;
      const uint64_t tmn64 = sw64_desc(0, 8192, 512);
      const uint32_t id = f16 ? idesc_f16(128, 32, 0, 0, 1, 0) : idesc_f16(128, 32, 1, 0, 1, 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) mma_ts(dX, dA + 8 * kk, tmn64 + x4 + 64 * kk, id, kk > 0);
    }
    mma_commit(sm.bar_mma(g));
    return;
  }
  // packed A operand: K columns 0..63 at region + [0, 32), 64..127 at region + [64, 96)
  if (JOB == kJobGram) {
    const uint32_t x4 = smem_u32(sm.x(g)) >> 4;
    const uint32_t id = f16 ? idesc_f16(128, 128, 0, 0, 0, 0) : idesc_f16(128, 128, 1, 0, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) mma_ts(dP, dX + (kk >> 2) * 64 + (kk & 3) * 8, desc_k(tk, x4, kk), id, kk > 0);
  } else if (JOB == kJobSquare) {
    const uint32_t s4 = smem_u32(sm.s(g)) >> 4;
    const uint32_t id = idesc_f16(128, 128, f16 ? 0 : 1, 0, 0, st->neg2);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(dP, dX + (kk >> 2) * 64 + (kk & 3) * 8, desc_k(tk, s4, kk), id, st->acc2 | (kk > 0));
  } else {
    const uint32_t x4 = smem_u32(sm.x(g)) >> 4;
    const uint64_t tmn = sw128_desc(0, kHalf, 1024);
    const uint32_t id = f16 ? idesc_f16(128, 128, 0, 0, 1, 0) : idesc_f16(128, 128, 1, 0, 1, 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) mma_ts(dX, dP + (kk >> 2) * 64 + (kk & 3) * 8, desc_mn(tmn, x4, kk), id, kk > 0);
  }
  mma_commit(sm.bar_mma(g));
}

// ------------------------------------------------------------------ one tile group
// P tiles of edge T = 128 / P per super-tile (P = 1: one 128-tile).
//
// Synchronisation inside a group uses only mbarriers with bounded waits (no
// named barriers), so a thread whose partners stopped after a failure never
// hangs: every wait gives up after kWaitLimitNs or as soon as the CTA's abort
// flag is raised.  Warps agree on a failure among their lanes (a warp stops as
// a whole); warps of a group that are still running then stop at their next
// wait, which the abort flag ends.
template <int P>
__device__ void group_main(const ResidentArgs &a, const Smem &sm, uint32_t tmem, int g) {
  constexpr uint32_t T = 128 / P;
  const int gt = threadIdx.x - g * kGroupThreads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wig = warp - g * kGroupWarps;              // warp in group, 0..7
  const uint32_t q = static_cast<uint32_t>(warp & 3);  // TMEM lane quarter
  const uint32_t hf = static_cast<uint32_t>(wig >> 2); // column half owned by this thread
  const uint32_t r = q * 32 + lane;                    // super-tile row
  const uint32_t jr = P == 1 ? 0u : r / T;             // this row's tile (diagonal block)
  const uint32_t rr = r - jr * T;                      // ... and its row inside that tile
  const uint32_t dP = tmem + 256u * g;                 // D_P (lane 0); D_X = dP + 128
  const uint32_t tP = dP + ((q * 32) << 16);           // this warp's lanes of D_P
  const uint32_t tX = tP + 128u;                       // ... and of D_X
  const uint32_t tA = tP + 192u;                       // ... and (P = 2) of the packed A operand
  uint8_t *Xs = sm.x(g), *Ss = sm.s(g), *Ws = sm.w(g);
  const bool step_mode = a.mode == 1;
  const bool has_w = step_mode && a.has_w;
  const int64_t grid = gridDim.x;
  const int64_t n_super = (a.n_tiles + P - 1) / P;
  uint32_t it = 0, job = 0;
  bool mg_issued = false;   // (issuing thread) this super-tile's M/G loads went out during the previous one
  // (issuing thread) phases armed on / waited for on bar_ld and bar_w, so
  // that an aborted tile can wait for its own copies in flight
  uint32_t ld_armed = 0, ld_seen = 0, w_armed = 0, w_seen = 0;
  // Self-test of the timeout path: one group waits on a barrier that nothing
  // arrives on, times out, records HIMUON_ERR_TIMEOUT and makes the CTA abort.
  if (a.test_stall && blockIdx.x == 0 && g == 0) wait_or_abort(sm.bar_never(g), 0, sm, a.status);
  const bool stalled = *sm.abort_flag() != 0;
  TileCoord *cur = sm.coord(g, 0), *nxt = sm.coord(g, 1);
  if (gt == 0) decode_super<P>(a, sm, blockIdx.x + g * grid, cur);
  __syncwarp();

  for (int64_t st = blockIdx.x + g * grid; st < n_super && !stalled; st += 2 * grid, ++it) {
    // this row's tile exists (the last super-tile may hold fewer than P tiles)
    const bool row_valid = P == 1 || P * st + jr < a.n_tiles;
    if (gt == 0) {
      bulk_wait_read0();  // the previous super-tile's stores have finished reading S_s / W_s
      if (!mg_issued) {
        issue_mg<P>(a, sm, g, cur);
        ++ld_armed;
      }
      if (has_w) {
        issue_w<P>(a, sm, g, cur);
        ++w_armed;
      }
    }
    __syncwarp();
    bool bad = !wait_or_abort(sm.bar_ld(g), it & 1u, sm, a.status);
    if (gt == 0 && !bad) ++ld_seen;
    if (__any_sync(0xffffffffu, bad)) break;

    // ---- prologue: M' = mu M + G (or the plain input), ||.||_F, fp32 copy to D_X.
    // M' (bf16, for the write-back) replaces G in S_s, so X_s is free for X_0 at once.
    // Columns outside this row's diagonal block are zero.
    float sumsq = 0.f;
    if constexpr (P == 2) {   // stacked: this row's 64 columns, 32 per warp, fp32 at D_X columns 32 hf..
      float v[32];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float m[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = 0.f;
        if (row_valid) {
          const uint32_t off = stage_off<P>(jr, rr, 4 * hf + k);
          unpack8(*reinterpret_cast<const uint4 *>(Xs + off), m);
          if (step_mode) {
            float gg[8];
            unpack8(*reinterpret_cast<const uint4 *>(Ss + off), gg);
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = fmaf(a.mu, m[e], gg[e]);
            *reinterpret_cast<uint4 *>(Ss + off) = pack8_bf16(m);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[8 * k + e] = m[e];
          sumsq = fmaf(m[e], m[e], sumsq);
        }
      }
      tmem_st32(tX + 32 * hf, v);
    } else if constexpr (P == 4) {   // stacked: this row's 32 columns, 16 per warp, fp32 at D_X columns 16 hf..
      float v[16];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float m[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = 0.f;
        if (row_valid) {
          const uint32_t off = stage_off<P>(jr, rr, 2 * hf + k);
          unpack8(*reinterpret_cast<const uint4 *>(Xs + off), m);
          if (step_mode) {
            float gg[8];
            unpack8(*reinterpret_cast<const uint4 *>(Ss + off), gg);
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = fmaf(a.mu, m[e], gg[e]);
            *reinterpret_cast<uint4 *>(Ss + off) = pack8_bf16(m);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[8 * k + e] = m[e];
          sumsq = fmaf(m[e], m[e], sumsq);
        }
      }
      tmem_st16(tX + 16 * hf, *reinterpret_cast<const uint32_t(*)[16]>(v));
    } else
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float v[32];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t cg = 8 * hf + 4 * i + k;         // 8-column chunk of the super-tile row
        float m[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = 0.f;
        if (P == 1 || ((8 * cg) / T == jr && row_valid)) {
          const uint32_t off = stage_off<P>(jr, rr, cg - jr * (T / 8));
          unpack8(*reinterpret_cast<const uint4 *>(Xs + off), m);
          if (step_mode) {
            float gg[8];
            unpack8(*reinterpret_cast<const uint4 *>(Ss + off), gg);
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = fmaf(a.mu, m[e], gg[e]);
            *reinterpret_cast<uint4 *>(Ss + off) = pack8_bf16(m);
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[8 * k + e] = m[e];
          sumsq = fmaf(m[e], m[e], sumsq);
        }
      }
      tmem_st32(tX + 64 * hf + 32 * i, v);
    }
    tmem_wait_st();
    sumsq = warp_sum(sumsq);
    if (lane == 0) sm.red(g)[wig] = sumsq;
    if (step_mode) fence_proxy_async_smem();
    tc_fence_before();
    // M' complete in S_s, partial sums visible, M read
    bad = !group_sync(sm.bar_pro(g), it & 1u, sm, lane, a.status);
    if (__any_sync(0xffffffffu, bad)) break;
    tc_fence_after();
    if (step_mode && gt == 0) {
#pragma unroll
      for (int j = 0; j < P; ++j)
        if (cur[j].blk >= 0) store_tile<P>(a.tmaps + cur[j].tm[kRoleIn], Ss, cur[j], j);
      bulk_commit();
    }
    __syncwarp();
    // ||tile||^2 of every tile of the super-tile (the warps whose rows lie in it)
    float tot[P];
#pragma unroll
    for (int j = 0; j < P; ++j) tot[j] = 0.f;
#pragma unroll
    for (int w = 0; w < kGroupWarps; ++w) tot[(32u * (w & 3)) / T] += sm.red(g)[w];
    float total = tot[0];   // this row's tile (a select, not an indexed load)
#pragma unroll
    for (int j = 1; j < P; ++j) total = (jr == static_cast<uint32_t>(j)) ? tot[j] : total;
    const float rho = (sqrtf(total) + a.eps) * a.safety;
    // operand type of this super-tile (the same in every thread of the group)
    bool f16 = a.op_fmt == 0;
    if (!f16 && a.f16_small) {
      bool small = true;
      if (P == 1) small = min(cur[0].h, cur[0].w) <= 64;
      bool tiny = false;
#pragma unroll
      for (int j = 0; j < P; ++j) {
        const float nrm = sqrtf(tot[j]);
        tiny = tiny || (tot[j] > 0.f && nrm < kTinyNorm * ((nrm + a.eps) * a.safety));
      }
      f16 = small && !tiny;
    }
    if (gt == 0) *sm.fmt16(g) = f16 ? 1 : 0;   // read by the issuer after this group's next arrival

    // ---- operand g_0 X_0 = r(g_0 M' / rho) to X_s and (packed) to D_X
    if constexpr (P == 2) {
      if (f16) stack_tmem_to_op<0, true>(tX + 32 * hf, tA, Xs, r, hf, a.gamma0 / rho);
      else stack_tmem_to_op<1, true>(tX + 32 * hf, tA, Xs, r, hf, a.gamma0 / rho);
    } else if constexpr (P == 4) {
      if (f16) stack4_tmem_to_op<0>(tX + 16 * hf, tA, Xs, r, hf, a.gamma0 / rho);
      else stack4_tmem_to_op<1>(tX + 16 * hf, tA, Xs, r, hf, a.gamma0 / rho);
    } else {
      if (f16) tmem_row_to_op<0, true>(tX, tX, Xs, r, hf, a.gamma0 / rho);
      else tmem_row_to_op<1, true>(tX, tX, Xs, r, hf, a.gamma0 / rho);
    }
    // M' must have left S_s before the first conversion (after MMA1) overwrites it
    if (step_mode && gt == 0) bulk_wait_read0();
    fence_proxy_async_smem();
    tc_fence_before();
    group_ready(sm, g, lane);

    if (gt == 0) {   // next super-tile of this group, while MMA1 runs
      decode_super<P>(a, sm, st + 2 * grid, nxt);
#pragma unroll
      for (int j = 0; j < P; ++j) {
        if (nxt[j].blk < 0) continue;
        prefetch_tile<P>(a.tmaps + nxt[j].tm[kRoleIn], nxt[j]);
        if (step_mode) prefetch_tile<P>(a.tmaps + nxt[j].tm[kRoleG], nxt[j]);
        if (has_w) prefetch_tile<P>(a.tmaps + nxt[j].tm[kRoleW], nxt[j]);
      }
    }
    __syncwarp();

    bool stop = false;
    for (int t = 0; t < a.K && !stop; ++t) {
      const ResidentStep *stp = &a.step[t];
      // after MMA1: S = r(s D_P) (s = 1 unless c = 0) to S_s and (packed) to D_X
      bad = !wait_or_abort(sm.bar_mma(g), job++ & 1u, sm, a.status);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      tc_fence_after();
      if constexpr (P == 2) {   // the row's own tile block of D_P: columns 64 jr + 32 hf ..
        const uint32_t src = tP + 64 * jr + 32 * hf;
        if (f16) stack_tmem_to_op<0, true>(src, tA, Ss, r, hf, stp->s);
        else stack_tmem_to_op<1, true>(src, tA, Ss, r, hf, stp->s);
      } else if constexpr (P == 4) {   // the row's own tile block of D_P: columns 32 jr + 16 hf ..
        const uint32_t src = tP + 32 * jr + 16 * hf;
        if (f16) stack4_tmem_to_op<0>(src, tA, Ss, r, hf, stp->s);
        else stack4_tmem_to_op<1>(src, tA, Ss, r, hf, stp->s);
      } else if (f16) {
        if (stp->s == 1.f) tmem_row_to_op<0, false>(tP, tX, Ss, r, hf, 1.f);
        else tmem_row_to_op<0, true>(tP, tX, Ss, r, hf, stp->s);
      } else {
        if (stp->s == 1.f) tmem_row_to_op<1, false>(tP, tX, Ss, r, hf, 1.f);
        else tmem_row_to_op<1, true>(tP, tX, Ss, r, hf, stp->s);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      group_ready(sm, g, lane);
      // after MMA2: Bop = r(beta D_P + a I) (beta = b / g^2), packed in D_P
      bad = !wait_or_abort(sm.bar_mma(g), job++ & 1u, sm, a.status);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      tc_fence_after();
      if constexpr (P == 2) {
        if (f16) stack_row_to_bop<0>(tP, tA, r, hf, stp->beta, stp->a);
        else stack_row_to_bop<1>(tP, tA, r, hf, stp->beta, stp->a);
      } else if constexpr (P == 4) {
        if (f16) stack4_row_to_bop<0>(tP, tA, r, hf, stp->beta, stp->a);
        else stack4_row_to_bop<1>(tP, tA, r, hf, stp->beta, stp->a);
      } else {
        if (f16) tmem_row_to_tmem_op<0>(tP, r, hf, stp->beta, stp->a);
        else tmem_row_to_tmem_op<1>(tP, r, hf, stp->beta, stp->a);
      }
      tc_fence_before();
      group_ready(sm, g, lane);
      // after MMA3: next operand r(xr D_X) = g_{t+1} X_{t+1} (xr = 1 for constant coefficients)
      bad = !wait_or_abort(sm.bar_mma(g), job++ & 1u, sm, a.status);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      tc_fence_after();
      if (t + 1 < a.K) {
        if constexpr (P == 2) {
          if (f16) stack_tmem_to_op<0, true>(tX + 32 * hf, tA, Xs, r, hf, stp->xr);
          else stack_tmem_to_op<1, true>(tX + 32 * hf, tA, Xs, r, hf, stp->xr);
        } else if constexpr (P == 4) {
          if (f16) stack4_tmem_to_op<0>(tX + 16 * hf, tA, Xs, r, hf, stp->xr);
          else stack4_tmem_to_op<1>(tX + 16 * hf, tA, Xs, r, hf, stp->xr);
        } else if (f16) {
          if (stp->xr == 1.f) tmem_row_to_op<0, false>(tX, tX, Xs, r, hf, 1.f);
          else tmem_row_to_op<0, true>(tX, tX, Xs, r, hf, stp->xr);
        } else {
          if (stp->xr == 1.f) tmem_row_to_op<1, false>(tX, tX, Xs, r, hf, 1.f);
          else tmem_row_to_op<1, true>(tX, tX, Xs, r, hf, stp->xr);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        group_ready(sm, g, lane);
      }
    }
    if (stop) break;

    // X_s is free now (and S_s unless it stages O): start the next super-tile's loads
    mg_issued = false;
    if (gt == 0 && nxt[0].blk >= 0 && (!step_mode || !a.has_o)) {
      issue_mg<P>(a, sm, g, nxt);
      ++ld_armed;
      mg_issued = true;
    }
    __syncwarp();

    // ---- epilogue: O = D_X;  W <- W - lr O  (this row's diagonal block only)
    if (has_w) {
      bad = !wait_or_abort(sm.bar_w(g), it & 1u, sm, a.status);
      if (gt == 0 && !bad) ++w_seen;
      if (__any_sync(0xffffffffu, bad)) break;
    }
    // 8 values of gamma_{K-1} O for the staged tile at byte offset `off`: O and / or W'
    auto emit8 = [&](uint32_t off, const float *o) {
      if (a.has_o) {
        float ov[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ov[e] = a.oscale * o[e];
        *reinterpret_cast<uint4 *>(Ss + off) = pack8_bf16(ov);
      }
      if (has_w) {
        const float lro = -a.lr * a.oscale;
        float w[8];
        unpack8(*reinterpret_cast<const uint4 *>(Ws + off), w);
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = fmaf(lro, o[e], w[e]);
        *reinterpret_cast<uint4 *>(Ws + off) = pack8_bf16(w);
      }
    };
    if constexpr (P == 4) {   // stacked: this row's 32 columns, 16 per warp, at D_X columns 16 hf..
      if (row_valid) {
        float v[16];
        tmem_ld16(tX + 16 * hf, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 2; ++k) emit8(stage_off<P>(jr, rr, 2 * hf + k), v + 8 * k);
      }
    } else {
#pragma unroll
      for (int i = 0; i < (P == 2 ? 1 : 2); ++i) {
        // 32-column group of the super-tile row (P = 2: of the stacked row, at D_X columns 32 hf..)
        const uint32_t c32 = P == 2 ? hf : 2 * hf + i;
        if (P == 1 || row_valid) {
          float v[32];
          tmem_ld32(tX + 32 * c32, v);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 4; ++k) emit8(stage_off<P>(jr, rr, 4 * c32 + k), v + 8 * k);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    // Only the storing thread needs the whole group's W' / O in place; the
    // others go on to the next super-tile, whose loads wait for these stores.
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.bar_epi(g));
    if (gt == 0) {
      bad = !wait_or_abort(sm.bar_epi(g), it & 1u, sm, a.status);
      if (!bad) {
#pragma unroll
        for (int j = 0; j < P; ++j) {
          if (cur[j].blk < 0) continue;
          if (a.has_o) store_tile<P>(a.tmaps + cur[j].tm[kRoleOut], Ss, cur[j], j);
          if (has_w) store_tile<P>(a.tmaps + cur[j].tm[kRoleW], Ws, cur[j], j);
        }
        bulk_commit();
      }
#pragma unroll
      for (int j = 0; j < P; ++j) cur[j] = nxt[j];
    }
    if (__any_sync(0xffffffffu, bad)) break;
  }
  if (gt == 0) {
    // After an abort: wait (bounded) for this group's own loads still in
    // flight, so that no copy lands in memory the CTA is about to release
    // (the issuer waits for the group's MMAs).  Nothing is outstanding after a
    // normal finish.
    for (; ld_seen < ld_armed; ++ld_seen) mbar_wait(sm.bar_ld(g), ld_seen & 1u, a.status);
    for (; w_seen < w_armed; ++w_seen) mbar_wait(sm.bar_w(g), w_seen & 1u, a.status);
    bulk_wait0();
  }
}

// ------------------------------------------------------------------ the issuer
// One thread (lane 0 of warp 16) issues every MMA of both groups: it polls
// each group's ready barrier (non-blocking) and, when a group's operands are
// in place, issues that group's next job and commits it to the group's MMA
// barrier.  The converting warps therefore never stall in an MMA issue while
// the tensor pipe is busy with the other group's job.  Per group it walks the
// same sequence as the group: per super-tile K steps of (Gram, Square, Update).
template <int P>
__device__ void issuer_main(const ResidentArgs &a, const Smem &sm, uint32_t tmem) {
  const int64_t grid = gridDim.x;
  const int64_t n_super = (a.n_tiles + P - 1) / P;
  int64_t st0 = blockIdx.x, st1 = blockIdx.x + grid;
  int t0 = 0, t1 = 0, jb0 = kJobGram, jb1 = kJobGram;
  uint32_t rph0 = 0, rph1 = 0, issued0 = 0, issued1 = 0;
  bool done0 = st0 >= n_super, done1 = st1 >= n_super;
  uint64_t last = globaltimer_ns();
  uint32_t spin = 0;
  while (!(done0 && done1)) {
    bool any = false;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      // this group's state (named per group: no local-memory arrays)
      int64_t &st = g == 0 ? st0 : st1;
      int &t = g == 0 ? t0 : t1;
      int &jb = g == 0 ? jb0 : jb1;
      uint32_t &rph = g == 0 ? rph0 : rph1;
      uint32_t &issued = g == 0 ? issued0 : issued1;
      bool &done = g == 0 ? done0 : done1;
      if (done) continue;
      if (!mbar_test_wait(sm.bar_ready(g), rph & 1u)) continue;
      ++rph;
      tc_fence_after();
      const bool f16 = *sm.fmt16(g) != 0;
      const uint32_t dP = tmem + 256u * g;
      const ResidentStep *stp = &a.step[t];
      if (jb == kJobGram) group_issue_mmas<kJobGram, P>(sm, g, dP, nullptr, f16);
      else if (jb == kJobSquare) group_issue_mmas<kJobSquare, P>(sm, g, dP, stp, f16);
      else group_issue_mmas<kJobUpdate, P>(sm, g, dP, stp, f16);
      ++issued;
      // next job of this group: the Gram job of step t + 1, or of the next super-tile
      if (++jb == 3) {
        jb = kJobGram;
        if (++t == a.K) {
          t = 0;
          st += 2 * grid;
          done = st >= n_super;
        }
      }
      any = true;
    }
    if (any) {
      last = globaltimer_ns();
      spin = 0;
    } else if ((++spin & 63u) == 0) {
      if (*sm.abort_flag()) break;
      if (globaltimer_ns() - last > kWaitLimitNs) {
        set_status(a.status, HIMUON_ERR_TIMEOUT);
        *sm.abort_flag() = 1;
        break;
      }
    }
  }
  // Every MMA issued must have finished before the CTA frees its TMEM and
  // shared memory: wait (bounded) for each group's last job.  Jobs of a group
  // complete in order, one barrier phase each.
  if (issued0 > 0) mbar_wait(sm.bar_mma(0), (issued0 - 1u) & 1u, a.status);
  if (issued1 > 0) mbar_wait(sm.bar_mma(1), (issued1 - 1u) & 1u, a.status);
}

template <int P>
__global__ void __launch_bounds__(kThreads, 1) ns_resident_kernel(const __grid_constant__ ResidentArgs args) {
  extern __shared__ uint8_t smem_raw[];
  Smem sm;
  sm.base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(sm.bar_ld(g), 1);
      mbar_init(sm.bar_w(g), 1);
      mbar_init(sm.bar_mma(g), 1);
      mbar_init(sm.bar_never(g), 1);
      mbar_init(sm.bar_ready(g), kGroupWarps);
      mbar_init(sm.bar_pro(g), kGroupWarps);
      mbar_init(sm.bar_epi(g), kGroupWarps);
      *sm.fmt16(g) = 0;
    }
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(sm.tmem_slot(), 512);
    tmem_relinquish();
  }
  if (use_smem_blocks(args)) {
    for (int i = threadIdx.x; i < args.n_blocks; i += blockDim.x) {
      const DevBlock &b = args.blocks[i];
      SBlock &d = sm.blocks()[i];
      d.tile_begin = static_cast<int32_t>(b.tile_begin);
      d.cols = b.cols;
      d.tiles_c = static_cast<uint16_t>(b.tiles_c);
      d.T = static_cast<uint16_t>(b.T);
#pragma unroll
      for (int r = 0; r < kNumRoles; ++r) d.tm[r] = static_cast<int16_t>(b.tmap[r]);
      d.rows = b.rows;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();

  if (warp < kIssuerWarp) {
    group_main<P>(args, sm, tmem, warp / kGroupWarps);
  } else {
    if ((threadIdx.x & 31) == 0) issuer_main<P>(args, sm, tmem);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace


int resident_smem_bytes() { return static_cast<int>(kSmemBytes); }
int resident_max_smem_blocks() { return kMaxSmemBlocks; }

void make_resident_steps(ResidentArgs &args, const float *coeffs, int K) {
  // Step t with beta = b (beta = 1 when b = 0, in which case MMA2 overwrites
  // A with c A^2) and g = sqrt|c / beta|.  The operand carries the iterate as
  // gamma_t X_t with gamma_t = g (1 when c = 0), so MMA1 leaves
  // D_P = gamma_t^2 A and S = r(s D_P), s = g / gamma_t^2 ... = 1 when
  // gamma_t = g: then S S^T = g^2 gamma_t^2 A^2 and MMA2 (sign of c / beta on
  // its A operand) leaves D_P = gamma_t^2 (A + (c / beta) A^2) = gamma_t^2 B / beta.
  // Bop = r((beta / gamma_t^2) D_P + a I) = r(a I + B) as written, MMA3 leaves
  // D_X = Bop gamma_t X_t = gamma_t X_{t+1}, and the next operand is
  // r((gamma_{t+1} / gamma_t) D_X); O = D_X / gamma_{K-1}.
  std::vector<double> gam(K);
  for (int t = 0; t < K; ++t) {
    const double b = coeffs[3 * t + 1], c = coeffs[3 * t + 2];
    const double beta = (b != 0.0) ? b : 1.0;
    const double g = sqrt(fabs(c / beta));
    gam[t] = g > 0.0 ? g : 1.0;
  }
  for (int t = 0; t < K; ++t) {
    const double a = coeffs[3 * t], b = coeffs[3 * t + 1], c = coeffs[3 * t + 2];
    const double beta = (b != 0.0) ? b : 1.0;
    const double ratio = c / beta;
    ResidentStep &st = args.step[t];
    st.s = static_cast<float>(sqrt(fabs(ratio)) / gam[t]);   // exactly 1 unless c = 0 (then 0)
    if (sqrt(fabs(ratio)) == gam[t]) st.s = 1.f;
    st.neg2 = ratio < 0.0 ? 1u : 0u;
    st.acc2 = (b != 0.0) ? 1u : 0u;
    st.beta = static_cast<float>(beta / (gam[t] * gam[t]));
    st.a = static_cast<float>(a);
    st.xr = t + 1 < K ? static_cast<float>(gam[t + 1] / gam[t]) : 1.f;
    if (t + 1 < K && gam[t + 1] == gam[t]) st.xr = 1.f;
  }
  args.gamma0 = K > 0 ? static_cast<float>(gam[0]) : 1.f;
  args.oscale = K > 0 ? static_cast<float>(1.0 / gam[K - 1]) : 1.f;
}

template <int P>
static cudaError_t launch_pack(const ResidentArgs &args, int grid, cudaStream_t stream) {
  // The shared-memory opt-in is per device; setting it again is cheap.
  cudaError_t e = cudaFuncSetAttribute(ns_resident_kernel<P>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  count_launch();
  ns_resident_kernel<P><<<grid, kThreads, kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

cudaError_t launch_ns_resident(const ResidentArgs &args, int grid, cudaStream_t stream) {
  switch (args.pack) {
    case 2: return launch_pack<2>(args, grid, stream);
    case 4: return launch_pack<4>(args, grid, stream);
    default: return launch_pack<1>(args, grid, stream);
  }
}

}  // namespace himuon
