// ns_pair.cu -- tiled NS with 256 x 256 tiles kept on chip for all K steps,
// one tile per CTA pair.
//
// The map ("Gram Newton-Schulz" page, sec. 3, Algorithm 1, applied per tile as
// in the "Hierarchical Muon" abstract) on tiles of T = 256: normalise by
// (||X||_F + eps), then per step A = X X^T, B = b A + c A^2, X = a X + B X.
// Ragged edge tiles are zero-padded to 256 x 256 (the same map, as on the
// 128-tile kernel: a zero border stays zero and NS(X^T) = NS(X)^T).
//
// A 256 x 256 tile does not fit one SM's tensor memory twice (two fp32 256 x 256
// accumulators are 2 x 256 KB), so each tile runs on a pair of CTAs in a
// cluster of two: CTA c owns rows 128c .. 128c + 127 of the tile and of every
// 256 x 256 product, in its own TMEM (256 columns for D_P, 256 for D_X).  The
// even CTA issues every MMA as a pair MMA (cta_group::2, M = 256, N = 256):
// each CTA supplies its 128 rows of the A operand from its TMEM and 128 of the
// N rows of the B operand from its shared memory.  With the iterate carried
// scaled by g = sqrt|c/b| as on the 128-tile kernel:
//   MMA1  D_P  = Xg Xg^T           A: Xg (own rows, packed in D_X)   B: own rows of Xg (K-major)
//   MMA2  D_P += sign(c/b) S S^T    A: S  (own rows, packed in D_X)   B: own rows of S  (K-major)
//   MMA3  D_X  = Bop Xg             A: Bop (own rows, packed in D_P)  B: columns 128c .. 128c+127 of Xg,
//                                                                        all 256 rows (MN-major)
// so only MMA3's B operand needs the partner's rows.  Each conversion of the
// iterate writes its rows' values of the partner's column half to a local
// staging buffer, and one thread copies it (32 KB, one bulk copy in the async
// proxy) into the partner's X_mn, completing on the partner's exchange
// barrier; each tile's norm is the sum of the two CTAs' partial sums.
// Operands are ready for a job when all 16 warps of both CTAs have arrived on
// the even CTA's ready barrier and, for MMA3 (the only reader of X_mn), both
// copies have landed: the odd CTA's warp 0 arrives only after the even CTA's
// copy has landed in its X_mn, and the issuing thread waits for the odd CTA's
// copy into the even CTA's X_mn.  The copies thus overlap the next step's
// Gram and square products.  The even CTA's issuing thread then issues the
// job's 16 MMAs and commits them to the MMA barrier of both CTAs (multicast
// commit).
// Shared memory per CTA: X_s (128 rows x 256, K-major, 64 KB), S_s (same;
// also M' in the prologue and W / W' in the epilogue), X_mn (256 rows x this
// CTA's 128 columns, MN-major, 64 KB; G in the prologue), the staging buffer
// (this CTA's 128 rows of the partner's columns, 32 KB).
//
// Operand type per tile as on the 128-tile kernel: a bf16 call rounds the
// operands of a tile with a short side of at most 64 to fp16 (unless its
// normalised norm is below 2^-10).  Every wait is bounded; a CTA that gives up
// raises its own and its partner's abort flag.  At the end the pair meets in a
// cluster barrier, each CTA waits (bounded) for the copies its partner sent
// it, and after a second cluster barrier each CTA releases its TMEM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "layout.hpp"
#include "onchip.cuh"
#include "ptx.cuh"
#include "resident.hpp"

namespace himuon {

namespace {

using namespace onchip;

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kChunk = 16384;      // 128 rows x 64 columns of 16-bit values, 128-byte swizzle
constexpr uint32_t kOffX = 0;           // X_s: own rows, K-major, 4 chunks
constexpr uint32_t kOffS = 65536;       // S_s: own rows, K-major, 4 chunks
constexpr uint32_t kOffMN = 131072;     // X_mn: all 256 rows of this CTA's 128 columns, MN-major
constexpr uint32_t kMnRows = 32768;     // its two 128-row halves (row half h written by CTA h) ...
constexpr uint32_t kMnSub = 16384;      // ... each of two 64-column sub-blocks (128 rows x 128 bytes)
constexpr uint32_t kOffStage = 196608;  // staging: own rows of the partner's 128 columns (one X_mn row half)
constexpr uint32_t kOffBars = kOffStage + kMnRows;
constexpr uint32_t kSmemBytes = kOffBars + 512 + 1024;   // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

struct PairSmem {
  uint8_t *base;
  __device__ uint8_t *x() const { return base + kOffX; }
  __device__ uint8_t *s() const { return base + kOffS; }
  __device__ uint8_t *mn() const { return base + kOffMN; }
  __device__ uint8_t *stage() const { return base + kOffStage; }
  __device__ uint64_t *bar(int i) const { return reinterpret_cast<uint64_t *>(base + kOffBars) + i; }
  __device__ uint64_t *bar_ld() const { return bar(0); }     // M (or input) and G landed
  __device__ uint64_t *bar_w() const { return bar(1); }      // W landed
  __device__ uint64_t *bar_mma() const { return bar(2); }    // the pair's MMA job finished (multicast commit)
  __device__ uint64_t *bar_ready() const { return bar(3); }  // even CTA: both CTAs' operands of the next job written
  __device__ uint64_t *bar_pro() const { return bar(4); }    // prologue: M' and partial norms of this CTA written
  __device__ uint64_t *bar_norm() const { return bar(5); }   // the partner's partial norm landed
  __device__ uint64_t *bar_epi() const { return bar(6); }    // epilogue: W' / O staged
  __device__ uint64_t *bar_never() const { return bar(7); }  // never arrived on (stall self-test)
  __device__ uint64_t *bar_stage() const { return bar(8); }  // this CTA's staging buffer written
  __device__ uint64_t *bar_xin() const { return bar(9); }    // the partner's copy landed in this CTA's X_mn
  __device__ uint64_t *bar_sfree() const { return bar(10); } // S_s no longer read by the previous tile's store
  __device__ float *red() const { return reinterpret_cast<float *>(base + kOffBars + 128); }   // kWarps floats
  __device__ float *peer_norm() const { return reinterpret_cast<float *>(base + kOffBars + 192); }
  __device__ uint32_t *tmem_slot() const { return reinterpret_cast<uint32_t *>(base + kOffBars + 196); }
  __device__ volatile int *abort_flag() const { return reinterpret_cast<volatile int *>(base + kOffBars + 200); }
  __device__ volatile uint32_t *peer_sent() const {   // copies the partner sent here (written by the partner)
    return reinterpret_cast<volatile uint32_t *>(base + kOffBars + 204);
  }
  __device__ TileCoord *coord(int i) const { return reinterpret_cast<TileCoord *>(base + kOffBars + 256) + i; }
};

// Bounded wait (cluster-scope acquire: some phases complete by the partner's
// arrivals).  On a timeout it records HIMUON_ERR_TIMEOUT and raises the abort
// flag of both CTAs of the pair; it gives up as soon as the flag is raised.
__device__ __forceinline__ bool pair_wait(uint64_t *bar, uint32_t parity, const PairSmem &sm, uint32_t peer,
                                          int *status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*sm.abort_flag()) return false;
      if (globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
  }
  set_status(status, HIMUON_ERR_TIMEOUT);
  *sm.abort_flag() = 1;
  st_cluster_u32(mapa_shared(smem_u32(const_cast<int *>(sm.abort_flag())), peer), 1u);
  return false;
}

// Byte offset of 16-byte chunk `c8` (0..31) of row `r` in a K-major operand of
// 256 columns: four 64-column, 128-byte-swizzled chunks.
__device__ __forceinline__ uint32_t kmaj_off(uint32_t r, uint32_t c8) {
  return (c8 >> 3) * kChunk + sw128_off(r, c8 & 7u);
}
// Byte offset of 16-byte chunk `c8` (0..15) of row `r` (0..127) in one row
// half of X_mn, and in the staging buffer, which has the same layout.
__device__ __forceinline__ uint32_t mn_off(uint32_t r, uint32_t c8) {
  return (c8 >> 3) * kMnSub + sw128_off(r, c8 & 7u);
}

// This thread's 64 columns (chunk cb) of row r of a 256-column fp32 TMEM
// region -> r(scale * v): packed in place to TMEM columns [64 cb, 64 cb + 32)
// of `pk` (the A operand), and to the K-major shared operand `kdst`.  With MN
// the values also go, as row r of an X_mn row half, to `mn_dst`: this CTA's
// own row half of X_mn when the columns are its own (cb / 2 == c), else the
// staging buffer bound for the partner.
template <int F, bool MN>
__device__ __forceinline__ void pair_row_to_op(uint32_t src, uint32_t pk, uint8_t *kdst, uint32_t r, uint32_t cb,
                                               float scale, uint8_t *mn_dst) {
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float v[32];
    tmem_ld32(src + 64u * cb + 32u * i, v);
    tmem_wait_ld();
    uint32_t p[16];
    if (scale != 1.f) {
#pragma unroll
      for (int e = 0; e < 16; ++e) p[e] = pack2_op<F>(v[2 * e] * scale, v[2 * e + 1] * scale);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) p[e] = pack2_op<F>(v[2 * e], v[2 * e + 1]);
    }
    tmem_st16(pk + 64u * cb + 16u * i, p);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 u = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
      const uint32_t c8 = 8u * cb + 4u * i + j;            // 16-byte chunk of the 256-column row
      *reinterpret_cast<uint4 *>(kdst + kmaj_off(r, c8)) = u;
      if (MN) *reinterpret_cast<uint4 *>(mn_dst + mn_off(r, c8 & 15u)) = u;
    }
  }
  tmem_wait_st();
}

// Bop = r(beta * D_P + diag * I) for this thread's 64 columns, packed in place.
// Row r of CTA c is row 128 c + r of the tile: its diagonal element sits in
// chunk (128 c + r) / 64 at position (128 c + r) % 64.
template <int F>
__device__ __forceinline__ void pair_row_to_bop(uint32_t taddr, uint32_t grow, uint32_t cb, float beta, float diag) {
  const bool dchunk = (grow >> 6) == cb;
  const uint32_t dpos = grow & 63u;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float v[32];
    tmem_ld32(taddr + 64u * cb + 32u * i, v);
    tmem_wait_ld();
    uint32_t p[16];
    if (dchunk && (dpos >> 5) == static_cast<uint32_t>(i)) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float a0 = fmaf(beta, v[2 * e], (dpos & 31u) == 2u * e ? diag : 0.f);
        const float a1 = fmaf(beta, v[2 * e + 1], (dpos & 31u) == 2u * e + 1u ? diag : 0.f);
        p[e] = pack2_op<F>(a0, a1);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) p[e] = pack2_op<F>(beta * v[2 * e], beta * v[2 * e + 1]);
    }
    tmem_st16(taddr + 64u * cb + 16u * i, p);
  }
  tmem_wait_st();
}

enum Job { kJobGram = 0, kJobSquare = 1, kJobUpdate = 2 };

// TMEM column of the packed A operand for k-step kk (K elements 16 kk .. +15)
__device__ __forceinline__ uint32_t acol(int kk) { return 64u * (kk >> 2) + 8u * (kk & 3); }

// The even CTA's issuing thread: the job's sixteen 256x256x16 pair MMAs,
// committed to the MMA barrier of both CTAs.
template <int JOB>
__device__ __forceinline__ void pair_issue(const PairSmem &sm, uint32_t tmem, const ResidentStep *st, bool f16) {
  tc_fence_after();
  const uint32_t dP = tmem, dX = tmem + 256u;
  const uint64_t tk = sw128_desc(0, 16, 1024);
  if (JOB == kJobGram) {
    const uint32_t x4 = smem_u32(sm.x()) >> 4;
    const uint32_t id = f16 ? idesc_f16(256, 256, 0, 0, 0, 0) : idesc_f16(256, 256, 1, 0, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
      mma_ts_pair(dP, dX + acol(kk), tk + x4 + (((kk >> 2) * kChunk + (kk & 3) * 32) >> 4), id, kk > 0);
  } else if (JOB == kJobSquare) {
    const uint32_t s4 = smem_u32(sm.s()) >> 4;
    const uint32_t id = idesc_f16(256, 256, f16 ? 0 : 1, 0, 0, st->neg2);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
      mma_ts_pair(dP, dX + acol(kk), tk + s4 + (((kk >> 2) * kChunk + (kk & 3) * 32) >> 4), id, st->acc2 | (kk > 0));
  } else {
    // K rows 16 kk .. 16 kk + 15 of X_mn: row half kk / 8, 8-row groups 1024 bytes
    // apart, the two 64-column sub-blocks kMnSub apart
    const uint32_t m4 = smem_u32(sm.mn()) >> 4;
    const uint64_t tmn = sw128_desc(0, kMnSub, 1024);
    const uint32_t id = f16 ? idesc_f16(256, 256, 0, 0, 1, 0) : idesc_f16(256, 256, 1, 0, 1, 0);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
      mma_ts_pair(dX, dP + acol(kk), tmn + m4 + (((kk >> 3) * kMnRows + (kk & 7) * 2048) >> 4), id, kk > 0);
  }
  mma_commit_pair(sm.bar_mma(), 3);
}

// Boxes of this CTA's 128 rows of a tile: 64 columns x 128 rows each, at
// (x0 + 64 j, y0 + 128 c); boxes wholly past the block's last column or row
// are skipped on stores (loads read zeros there).
__device__ __forceinline__ void load_rows(const CUtensorMap *m, uint8_t *dst, const TileCoord &t, uint32_t c,
                                          uint64_t *bar) {
#pragma unroll
  for (int j = 0; j < 4; ++j) tma_load_2d(dst + j * kChunk, m, t.x0 + 64 * j, t.y0 + 128 * static_cast<int>(c), bar);
}
__device__ __forceinline__ void store_rows(const CUtensorMap *m, const uint8_t *src, const TileCoord &t, uint32_t c) {
  if (128 * static_cast<int>(c) >= t.h) return;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (64 * j < t.w) tma_store_2d(m, src + j * kChunk, t.x0 + 64 * j, t.y0 + 128 * static_cast<int>(c));
}
__device__ __forceinline__ void prefetch_rows(const CUtensorMap *m, const TileCoord &t, uint32_t c) {
  if (128 * static_cast<int>(c) >= t.h) return;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (64 * j < t.w) tma_prefetch_l2_2d(m, t.x0 + 64 * j, t.y0 + 128 * static_cast<int>(c));
}

__device__ void pair_main(const ResidentArgs &a, const PairSmem &sm, uint32_t tmem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t c = cluster_ctarank();           // 0: even CTA (issues the MMAs), 1: odd CTA
  const uint32_t peer = c ^ 1u;
  const uint32_t q = static_cast<uint32_t>(warp & 3);   // TMEM lane quarter
  const uint32_t cb = static_cast<uint32_t>(warp >> 2); // 64-column chunk of the 256-column row
  const uint32_t r = q * 32 + lane;               // row among this CTA's 128
  const uint32_t grow = 128u * c + r;             // row of the tile
  const uint32_t tP = tmem + ((q * 32) << 16);    // this warp's lanes of D_P (columns 0..255)
  const uint32_t tX = tP + 256u;                  // ... and of D_X (columns 256..511)
  uint8_t *Xs = sm.x(), *Ss = sm.s(), *Xmn = sm.mn();
  const bool step_mode = a.mode == 1;
  const bool has_w = step_mode && a.has_w;
  const bool leader = c == 0 && threadIdx.x == 0;
  const bool tma = threadIdx.x == 0;              // this CTA's TMA-issuing thread
  // This warp's columns belong to X_mn of CTA cb / 2: this CTA's own row half
  // of it, or the staging buffer that one thread copies to the partner's.
  const bool stager = (cb >> 1) != c;
  uint8_t *mn_dst = stager ? sm.stage() : Xmn + c * kMnRows;
  const bool copier = static_cast<int>(threadIdx.x) == (c == 0 ? kThreads / 2 : 0);   // lane 0 of a staging warp
  const uint32_t peer_mn = mapa_shared(smem_u32(Xmn + c * kMnRows), peer);             // this CTA's rows there
  const uint32_t peer_xin = mapa_shared(smem_u32(sm.bar_xin()), peer);
  const uint32_t xin0_addr = mapa_shared(smem_u32(sm.bar_xin()), 0);
  const uint32_t ready_addr = mapa_shared(smem_u32(sm.bar_ready()), 0);
  const uint32_t peer_norm_addr = mapa_shared(smem_u32(sm.peer_norm()), peer);
  const uint32_t peer_norm_bar = mapa_shared(smem_u32(sm.bar_norm()), peer);
  const int64_t n_pairs = gridDim.x / 2;
  const int64_t pair = blockIdx.x / 2;
  const uint32_t ld_bytes = (step_mode ? 2u : 1u) * 4u * kChunk;
  // The next tile's M (to X_s, after the last Gram product) and G (to X_mn,
  // after the last update product) are loaded during the current tile's last
  // step, unless X_s stages O for the epilogue.
  const bool prefetch = !a.has_o;
  uint32_t it = 0, job = 0, xj = 0;   // tiles, MMA jobs, exchanges of the iterate so far
  uint32_t ld_armed = 0, ld_seen = 0, w_armed = 0, w_seen = 0, mma_issued = 0;
  uint32_t sent = 0;                  // (copier) copies issued to the partner
  uint32_t xin_armed = 0, xin_seen = 0;   // (thread 0) exchange phases armed / seen complete
  uint32_t relayed = 0;               // (odd CTA's thread 0) arrivals on the even CTA's exchange barrier
  bool ld_issued = false;   // (TMA thread) the current tile's loads are out
  bool g_pending = false;   // (TMA thread) the next tile's M is out, its G not yet
  bool f16 = false;         // operand type of the current tile
  // Tile coordinates alternate between two slots: the TMA thread decodes tile
  // it + 1 into the other slot before it arms that tile's loads, so a thread
  // that has seen the loads land also sees the coordinates.
  if (a.test_stall && pair == 0) pair_wait(sm.bar_never(), 0, sm, peer, a.status);
  if (tma) *sm.coord(0) = decode_tile(a, nullptr, pair);
  __syncthreads();
  bool bad = *sm.abort_flag() != 0;

  // This warp's arrival on the even CTA's ready barrier once its operands are
  // written.  X_mn is read by MMA3 alone, so the copies of the iterate made
  // after an update product have the next step's Gram and square products to
  // land: the issuing thread waits for them (its exchange barrier) only before
  // MMA3.
  auto ready = [&]() {
    __syncwarp();
    if (lane == 0) {
      if (c == 0) mbar_arrive(sm.bar_ready());
      else mbar_arrive_cluster(ready_addr);
    }
  };
  // The odd CTA's thread 0, after its arrival for the square product: once the
  // even CTA's copy of the iterate has landed in this CTA's X_mn, it arrives on
  // the even CTA's exchange barrier (release, cluster scope), which the issuing
  // thread waits for before MMA3.
  auto relay = [&]() -> bool {
    const bool ok = pair_wait(sm.bar_xin(), xin_seen & 1u, sm, peer, a.status);
    if (ok) {
      ++xin_seen;
      mbar_arrive_cluster(xin0_addr);
      ++relayed;
    }
    return ok;
  };
  // Operand g X of the iterate from the fp32 copy in D_X: X_s, packed in D_X,
  // this CTA's row half of X_mn, and the staging buffer, which the copier then
  // sends to the partner's X_mn (completing on the partner's exchange barrier).
  auto convert_x = [&](float scale) {
    if (tma) {
      mbar_arrive_expect_tx(sm.bar_xin(), kMnRows);   // the partner's copy into this CTA's X_mn
      ++xin_armed;
    }
    if (f16) pair_row_to_op<0, true>(tX, tX, Xs, r, cb, scale, mn_dst);
    else pair_row_to_op<1, true>(tX, tX, Xs, r, cb, scale, mn_dst);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (stager && lane == 0) mbar_arrive(sm.bar_stage());
  };
  // The copier, after its warp's arrival on the ready barrier: the staging
  // buffer to the partner's X_mn once all staging warps have written it.
  auto send_stage = [&]() -> bool {
    bool ok = true;
    if (copier) {
      ok = pair_wait(sm.bar_stage(), xj & 1u, sm, peer, a.status);
      if (ok) {
        bulk_copy_to_peer(peer_mn, sm.stage(), kMnRows, peer_xin);
        ++sent;
      }
    }
    ++xj;
    return ok;
  };
  // The even CTA's issuing thread: wait for the job's operands, then issue it.
  auto issue = [&](int jobkind, const ResidentStep *stp, bool exchange) -> bool {
    bool ok = pair_wait(sm.bar_ready(), job & 1u, sm, peer, a.status);
    if (ok && exchange) {
      ok = pair_wait(sm.bar_xin(), xin_seen & 1u, sm, peer, a.status);
      if (ok) ++xin_seen;
    }
    if (ok) {
      if (jobkind == kJobGram) pair_issue<kJobGram>(sm, tmem, nullptr, f16);
      else if (jobkind == kJobSquare) pair_issue<kJobSquare>(sm, tmem, stp, f16);
      else pair_issue<kJobUpdate>(sm, tmem, stp, f16);
      ++mma_issued;
    }
    return ok;
  };

  for (int64_t tile = pair; tile < a.n_tiles && !bad; tile += n_pairs, ++it) {
    TileCoord *cur = sm.coord(it & 1u), *nxt = sm.coord((it + 1u) & 1u);
    if (tma) {
      bulk_wait_read0();   // the previous tile's stores have finished reading X_s / S_s
      mbar_arrive(sm.bar_sfree());
      if (!ld_issued) {
        mbar_arrive_expect_tx(sm.bar_ld(), ld_bytes);
        load_rows(a.tmaps + cur->tm[kRoleIn], Xs, *cur, c, sm.bar_ld());
        if (step_mode) load_rows(a.tmaps + cur->tm[kRoleG], Xmn, *cur, c, sm.bar_ld());
        ++ld_armed;
      }
    }
    ld_issued = false;
    __syncwarp();
    bad = !pair_wait(sm.bar_ld(), it & 1u, sm, peer, a.status);
    if (tma && !bad) ++ld_seen;
    if (step_mode && !bad) bad = !pair_wait(sm.bar_sfree(), it & 1u, sm, peer, a.status);
    if (__any_sync(0xffffffffu, bad)) break;

    // ---- prologue: M' = mu M + G (or the plain input): bf16 to S_s for the
    // TMA store, this CTA's ||.||_F^2, fp32 copy to D_X.  M lands in X_s, G in
    // X_mn (K-major boxes).
    float sumsq = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float v[32];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t off = kmaj_off(r, 8 * cb + 4 * i + k);
        float m[8];
        unpack8(*reinterpret_cast<const uint4 *>(Xs + off), m);
        if (step_mode) {
          float g[8];
          unpack8(*reinterpret_cast<const uint4 *>(Xmn + off), g);
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] = fmaf(a.mu, m[e], g[e]);
          *reinterpret_cast<uint4 *>(Ss + off) = pack8_bf16(m);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[8 * k + e] = m[e];
          sumsq = fmaf(m[e], m[e], sumsq);
        }
      }
      tmem_st32(tX + 64 * cb + 32 * i, v);
    }
    tmem_wait_st();
    if (step_mode) fence_proxy_async_smem();
    sumsq = warp_sum(sumsq);
    if (lane == 0) sm.red()[warp] = sumsq;
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.bar_pro());
    bad = !pair_wait(sm.bar_pro(), it & 1u, sm, peer, a.status);
    if (__any_sync(0xffffffffu, bad)) break;
    tc_fence_after();
    float own = 0.f;   // this CTA's ||rows||^2, summed in one order by every thread
#pragma unroll
    for (int w = 0; w < kWarps; ++w) own += sm.red()[w];
    if (tma) {
      st_cluster_f32(peer_norm_addr, own);   // the partner's half of the tile norm
      mbar_arrive_cluster(peer_norm_bar);
      if (step_mode) {   // M' from S_s to HBM (S_s is next written after MMA1)
        store_rows(a.tmaps + cur->tm[kRoleIn], Ss, *cur, c);
        bulk_commit();
      }
    }
    __syncwarp();
    bad = !pair_wait(sm.bar_norm(), it & 1u, sm, peer, a.status);
    if (__any_sync(0xffffffffu, bad)) break;
    const float total = own + *sm.peer_norm();      // the same value in both CTAs (a + b = b + a)
    const float nrm = sqrtf(total);
    const float rho = (nrm + a.eps) * a.safety;
    f16 = a.op_fmt == 0;
    if (!f16 && a.f16_small)
      f16 = min(cur->h, cur->w) <= 64 && !(total > 0.f && nrm < kTinyNorm * rho);

    // ---- operand g_0 X_0 = r(g_0 M' / rho).  X_s and X_mn were read by every
    // thread of this CTA before bar_pro, and the partner's copy into X_mn
    // follows its conversion, which follows this CTA's norm.
    convert_x(a.gamma0 / rho);
    // M' (and the previous tile's W' and O) must have left S_s / X_s before
    // MMA1 completes and the first conversion overwrites S_s
    if (tma) bulk_wait_read0();
    ready();
    bad = !send_stage();
    if (leader && !bad) bad = !issue(kJobGram, nullptr, false);
    if (tma) {   // next tile of this pair, while MMA1 runs
      *nxt = decode_tile(a, nullptr, tile + n_pairs, cur->blk);
      if (nxt->blk >= 0) {
        prefetch_rows(a.tmaps + nxt->tm[kRoleIn], *nxt, c);
        if (step_mode) prefetch_rows(a.tmaps + nxt->tm[kRoleG], *nxt, c);
        if (has_w) prefetch_rows(a.tmaps + nxt->tm[kRoleW], *nxt, c);
      }
    }
    if (__any_sync(0xffffffffu, bad)) break;

    bool stop = false;
    for (int t = 0; t < a.K && !stop; ++t) {
      const ResidentStep *stp = &a.step[t];
      const bool last = t + 1 == a.K;
      // after MMA1: S = r(s D_P) to S_s and (packed) to D_X
      bad = !pair_wait(sm.bar_mma(), job++ & 1u, sm, peer, a.status);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      tc_fence_after();
      if (last && prefetch && tma && nxt->blk >= 0) {   // X_s is free: the next tile's M
        mbar_arrive_expect_tx(sm.bar_ld(), ld_bytes);
        load_rows(a.tmaps + nxt->tm[kRoleIn], Xs, *nxt, c, sm.bar_ld());
        ++ld_armed;
        g_pending = step_mode;
        ld_issued = true;
      }
      if (f16) pair_row_to_op<0, false>(tP, tX, Ss, r, cb, stp->s, nullptr);
      else pair_row_to_op<1, false>(tP, tX, Ss, r, cb, stp->s, nullptr);
      fence_proxy_async_smem();
      tc_fence_before();
      ready();
      if (c == 1 && tma) bad = !relay();
      if (leader) bad = !issue(kJobSquare, stp, false);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      // after MMA2: Bop = r(beta D_P + a I), packed in D_P
      bad = !pair_wait(sm.bar_mma(), job++ & 1u, sm, peer, a.status);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      tc_fence_after();
      if (last && has_w && tma) {   // S_s is free for good: W lands there for the epilogue
        mbar_arrive_expect_tx(sm.bar_w(), 4u * kChunk);
        load_rows(a.tmaps + cur->tm[kRoleW], Ss, *cur, c, sm.bar_w());
        ++w_armed;
      }
      if (f16) pair_row_to_bop<0>(tP, grow, cb, stp->beta, stp->a);
      else pair_row_to_bop<1>(tP, grow, cb, stp->beta, stp->a);
      tc_fence_before();
      ready();
      if (leader) bad = !issue(kJobUpdate, stp, true);   // MMA3 reads X_mn: the exchange must have landed
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      // after MMA3: next operand r(xr D_X) = g_{t+1} X_{t+1}: X_s, packed in D_X, X_mn
      bad = !pair_wait(sm.bar_mma(), job++ & 1u, sm, peer, a.status);
      if ((stop = __any_sync(0xffffffffu, bad))) break;
      tc_fence_after();
      if (!last) {
        convert_x(stp->xr);
        ready();
        bad = !send_stage();
        if (leader && !bad) bad = !issue(kJobGram, nullptr, false);
        if ((stop = __any_sync(0xffffffffu, bad))) break;
      } else if (prefetch && step_mode && tma && nxt->blk >= 0) {   // X_mn is free: the next tile's G
        load_rows(a.tmaps + nxt->tm[kRoleG], Xmn, *nxt, c, sm.bar_ld());
        g_pending = false;
      }
    }
    if (stop) break;

    // ---- epilogue: O = D_X / g;  W <- W - lr O   (this CTA's rows)
    if (has_w) {
      bad = !pair_wait(sm.bar_w(), it & 1u, sm, peer, a.status);
      if (tma && !bad) ++w_seen;
      if (__any_sync(0xffffffffu, bad)) break;
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float v[32];
      tmem_ld32(tX + 64 * cb + 32 * i, v);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t off = kmaj_off(r, 8 * cb + 4 * i + k);
        const float *o = v + 8 * k;   // gamma_{K-1} O
        if (a.has_o) {
          float ov[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) ov[e] = a.oscale * o[e];
          *reinterpret_cast<uint4 *>(Xs + off) = pack8_bf16(ov);
        }
        if (has_w) {
          const float lro = -a.lr * a.oscale;
          float w[8];
          unpack8(*reinterpret_cast<const uint4 *>(Ss + off), w);
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = fmaf(lro, o[e], w[e]);
          *reinterpret_cast<uint4 *>(Ss + off) = pack8_bf16(w);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(sm.bar_epi());
    if (tma) {
      bad = !pair_wait(sm.bar_epi(), it & 1u, sm, peer, a.status);
      if (!bad) {
        if (a.has_o) store_rows(a.tmaps + cur->tm[kRoleOut], Xs, *cur, c);
        if (has_w) store_rows(a.tmaps + cur->tm[kRoleW], Ss, *cur, c);
        bulk_commit();
      }
    }
    if (__any_sync(0xffffffffu, bad)) break;
  }
  if (tma) {
    // After an abort: wait (bounded) for this CTA's loads still in flight.  A
    // prefetched M whose G was not issued yet gets its G now, so that the
    // phase armed for both completes (X_mn's content no longer matters).
    if (g_pending) {   // the loop left tile `it` early: its successor's slot
      const TileCoord &nx = *sm.coord((it + 1u) & 1u);
      load_rows(a.tmaps + nx.tm[kRoleG], Xmn, nx, c, sm.bar_ld());
    }
    for (; ld_seen < ld_armed; ++ld_seen) mbar_wait(sm.bar_ld(), ld_seen & 1u, a.status);
    for (; w_seen < w_armed; ++w_seen) mbar_wait(sm.bar_w(), w_seen & 1u, a.status);
    bulk_wait0();
  }
  if (leader && mma_issued > 0) {
    // every pair MMA issued has finished before the pair releases its memory
    mbar_wait(sm.bar_mma(), (mma_issued - 1u) & 1u, a.status);
  }
  // Copies between the pair still in flight after an abort: each copier tells
  // the partner how many it sent, and after a cluster barrier each CTA waits
  // (bounded) until all of them have landed in its X_mn.
  if (copier) st_cluster_u32(mapa_shared(smem_u32(const_cast<uint32_t *>(sm.peer_sent())), peer), sent);
  // (the even CTA's exchange phases also count the odd CTA's relays: one for
  // every copy the odd CTA sent)
  if (c == 1 && tma)
    for (; relayed < sent; ++relayed) mbar_arrive_cluster(xin0_addr);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (tma) {
    const uint32_t n = *sm.peer_sent();
    for (; xin_seen < n; ++xin_seen) {
      if (xin_seen >= xin_armed) {
        mbar_arrive_expect_tx(sm.bar_xin(), kMnRows);
        ++xin_armed;
      }
      mbar_wait(sm.bar_xin(), xin_seen & 1u, a.status);
    }
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    ns_pair_kernel(const __grid_constant__ ResidentArgs args) {
  extern __shared__ uint8_t smem_raw[];
  PairSmem sm;
  sm.base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(sm.bar_ld(), 1);
    mbar_init(sm.bar_w(), 1);
    mbar_init(sm.bar_mma(), 1);
    mbar_init(sm.bar_ready(), 2 * kWarps);
    mbar_init(sm.bar_pro(), kWarps);
    mbar_init(sm.bar_norm(), 1);
    mbar_init(sm.bar_epi(), kWarps);
    mbar_init(sm.bar_never(), 1);
    mbar_init(sm.bar_stage(), kWarps / 2);
    mbar_init(sm.bar_xin(), cluster_ctarank() == 0 ? 2 : 1);   // even CTA: + the odd CTA's relay
    mbar_init(sm.bar_sfree(), 1);
    *sm.abort_flag() = 0;
    *sm.peer_norm() = 0.f;
    *sm.peer_sent() = 0u;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(sm.tmem_slot(), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();

  pair_main(args, sm, tmem);

  tc_fence_before();
  cluster_sync_all();   // neither CTA releases its memory while the partner may still use it
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace

int pair_smem_bytes() { return static_cast<int>(kSmemBytes); }

cudaError_t launch_ns_pair(const ResidentArgs &args, int pairs, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(ns_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  count_launch();
  ns_pair_kernel<<<2 * pairs, kThreads, kSmemBytes, stream>>>(args);
  return cudaGetLastError();
}

}  // namespace himuon
