// api.cu -- the C ABI of libhimuon: argument checks, the CMuon split, the tile
// planner (cross-layer batching and memory-bounded chunking), a small plan
// cache, and dispatch to the on-chip or the HBM-staged kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <list>
#include <map>
#include <mutex>
#include <memory>
#include <string>
#include <tuple>
#include <vector>

#include "himuon.h"
#include "layout.hpp"
#include "resident.hpp"
#include "staged.hpp"

namespace himuon {

// The device status word: kernels record the first device-side failure here
// (bounded waits that gave up, inconsistent descriptors) instead of trapping.
__device__ int g_device_status;

static std::atomic<long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

int *status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  static int *cache[64] = {};
  if (dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int *>(p);
  }
  return cache[dev];
}

bool log_enabled() {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("HIMUON_LOG");
    v = (e && e[0] == '1') ? 1 : 0;
  }
  return v == 1;
}

// HIMUON_FORCE_PATH=staged sends calls that would run on chip through the
// staged path instead (A/B comparisons of the two paths on the same call);
// read on every call and part of the plan key.
bool force_staged() {
  const char *e = getenv("HIMUON_FORCE_PATH");
  return e && strcmp(e, "staged") == 0;
}

// HIMUON_MAX_CTAS=n caps the CTAs of an on-chip launch (tests only: with a
// few CTAs every CTA, or CTA pair, runs many tiles in its loop, the way the
// large calls do); read on every call, 0 or unset = one per SM.
int max_ctas() {
  const char *e = getenv("HIMUON_MAX_CTAS");
  const int v = e ? atoi(e) : 0;
  return v > 0 ? v : 0;
}

size_t elem_size(int32_t dt) { return dt == HIMUON_FP32 ? 4 : 2; }
int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// ---------------------------------------------------------------- matrices and blocks
struct CallMats {
  int32_t n = 0;
  const himuon_mat *role[kNumRoles] = {nullptr, nullptr, nullptr, nullptr};  // arrays of n, or null
};

struct HostBlock {
  int32_t mat;
  int64_t row0, col0, rows, cols;
  int64_t T;            // tile edge
  int64_t tiles_r, tiles_c, tile_begin;
};

int check_mat(const himuon_mat &m) {
  if (!m.data || m.rows < 1 || m.cols < 1 || m.ld < m.cols) return HIMUON_ERR_INVALID;
  if (m.rows > (int64_t)1 << 30 || m.cols > (int64_t)1 << 30) return HIMUON_ERR_UNSUPPORTED;
  if (m.dtype < HIMUON_BF16 || m.dtype > HIMUON_FP32) return HIMUON_ERR_UNSUPPORTED;
  return HIMUON_OK;
}

int check_params(const himuon_ns_params *p) {
  if (!p || !p->coeffs) return HIMUON_ERR_INVALID;
  if (p->steps < 1 || p->steps > kMaxSteps) return HIMUON_ERR_UNSUPPORTED;
  if (p->compute < HIMUON_BF16 || p->compute > HIMUON_FP32) return HIMUON_ERR_UNSUPPORTED;
  if (!(p->eps >= 0.f) || !(p->safety >= 0.f)) return HIMUON_ERR_INVALID;
  for (int i = 0; i < 3 * p->steps; ++i)
    if (!isfinite(p->coeffs[i])) return HIMUON_ERR_INVALID;
  if (p->n_restart < 0 || (p->n_restart > 0 && !p->restart_at)) return HIMUON_ERR_INVALID;
  if (p->chunk_bytes < 0) return HIMUON_ERR_INVALID;
  return HIMUON_OK;
}

// CMuon split of every matrix into blocks, then the tile grid of each block.
int make_blocks(const CallMats &cm, const himuon_split *splits, int64_t tile, std::vector<HostBlock> &out,
                int64_t *n_tiles) {
  out.clear();
  const himuon_mat *base = nullptr;
  for (int r = 0; r < kNumRoles && !base; ++r) base = cm.role[r];
  int64_t next_tile = 0;
  for (int32_t i = 0; i < cm.n; ++i) {
    const himuon_mat &m = base[i];
    std::vector<std::pair<int64_t, int64_t>> spans;  // (offset, size) along the split dim
    int dim = 0;
    if (splits && splits[i].nblocks > 1) {
      const himuon_split &s = splits[i];
      if ((s.dim != 0 && s.dim != 1) || !s.sizes) return HIMUON_ERR_INVALID;
      dim = s.dim;
      int64_t off = 0;
      for (int b = 0; b < s.nblocks; ++b) {
        if (s.sizes[b] < 1) return HIMUON_ERR_INVALID;
        spans.push_back({off, s.sizes[b]});
        off += s.sizes[b];
      }
      if (off != (dim == 0 ? m.rows : m.cols)) return HIMUON_ERR_INVALID;
    } else {
      spans.push_back({0, dim == 0 ? m.rows : m.cols});
    }
    for (auto &sp : spans) {
      HostBlock b;
      b.mat = i;
      b.row0 = dim == 0 ? sp.first : 0;
      b.col0 = dim == 1 ? sp.first : 0;
      b.rows = dim == 0 ? sp.second : m.rows;
      b.cols = dim == 1 ? sp.second : m.cols;
      b.T = (tile <= 0) ? std::max(b.rows, b.cols) : tile;
      b.tiles_r = (b.rows + b.T - 1) / b.T;
      b.tiles_c = (b.cols + b.T - 1) / b.T;
      b.tile_begin = next_tile;
      next_tile += b.tiles_r * b.tiles_c;
      out.push_back(b);
    }
  }
  *n_tiles = next_tile;
  return HIMUON_OK;
}

int check_call(const CallMats &cm, const himuon_split *splits) {
  if (cm.n < 1) return HIMUON_ERR_INVALID;
  const himuon_mat *base = nullptr;
  for (int r = 0; r < kNumRoles && !base; ++r) base = cm.role[r];
  if (!base) return HIMUON_ERR_INVALID;
  for (int r = 0; r < kNumRoles; ++r) {
    if (!cm.role[r]) continue;
    for (int32_t i = 0; i < cm.n; ++i) {
      const int rc = check_mat(cm.role[r][i]);
      if (rc) return rc;
      if (cm.role[r][i].rows != base[i].rows || cm.role[r][i].cols != base[i].cols) return HIMUON_ERR_INVALID;
    }
  }
  (void)splits;
  return HIMUON_OK;
}

// ---------------------------------------------------------------- plans
enum PathKind { kPathResident = 0, kPathStaged = 1, kPathPair = 2 };

struct TileClass {
  int64_t n = 0, m = 0;      // padded iterate shape (n <= m)
  bool padded = false;       // some tile of the class is smaller than n x m
  bool thin = false;         // every tile of the class has a short side <= kThinSide
  std::vector<DevTile> tiles;
  int64_t dev_offset = 0;    // index of the class's first DevTile in the device table
};

struct Plan {
  int device = -1;
  PathKind path = kPathStaged;
  std::vector<HostBlock> blocks;
  int64_t n_tiles = 0;
  int pack = 1;                   // on-chip path: tiles per super-tile
  std::vector<TileClass> classes;
  void *dev = nullptr;            // [DevBlock...][CUtensorMap...][DevTile...]
  DevBlock *d_blocks = nullptr;
  CUtensorMap *d_tmaps = nullptr;
  DevTile *d_tiles = nullptr;
  ~Plan() {
    if (dev) cudaFree(dev);
  }
};

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

// 2-D map over a bf16 block for the on-chip kernel with `pack` tiles per
// 128 x 128 super-tile: pack 1 -> box 64 columns x 128 rows, 128-byte swizzle;
// pack 2 -> 64 x 64, 128-byte swizzle; pack 4 -> 32 x 32, 64-byte swizzle.
// Zero fill outside the block (the zero padding of ragged tiles).
bool make_block_map(CUtensorMap *map, void *ptr, int64_t rows, int64_t cols, int64_t ld, int pack) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  const cuuint32_t T = static_cast<cuuint32_t>(128 / pack);
  cuuint32_t box[2] = {pack == 1 ? 64u : T, pack == 1 ? 128u : T};
  cuuint32_t es[2] = {1, 1};
  const CUtensorMapSwizzle sw = pack == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void *block_ptr(const himuon_mat &m, const HostBlock &b) {
  return static_cast<char *>(m.data) + (b.row0 * m.ld + b.col0) * static_cast<int64_t>(elem_size(m.dtype));
}

// Tiles per super-tile of the on-chip kernel for this call (1, 2 or 4), or 0
// when the call needs the staged path: fp32 arithmetic, non-bf16 storage,
// misaligned rows, or tiles that are neither 128 x 128 (edge tiles smaller),
// 64 x 64, 32 x 32, nor a whole block of at most 128 x 128.
// The on-chip kernels read and write bf16 storage through 2-D tensor maps:
// every role bf16, row pitch and block origins 16-byte aligned, 16-bit arithmetic.
bool onchip_storage_ok(const CallMats &cm, const std::vector<HostBlock> &blocks, const himuon_ns_params &p) {
  if (p.compute == HIMUON_FP32) return false;
  for (int r = 0; r < kNumRoles; ++r) {
    if (!cm.role[r]) continue;
    for (int32_t i = 0; i < cm.n; ++i) {
      const himuon_mat &m = cm.role[r][i];
      if (m.dtype != HIMUON_BF16) return false;
      if ((m.ld * 2) % 16 != 0) return false;
    }
    for (const HostBlock &b : blocks)
      if (reinterpret_cast<uintptr_t>(block_ptr(cm.role[r][b.mat], b)) % 16 != 0) return false;
  }
  return true;
}

// T = 256 runs on chip on CTA pairs (every block tiled at 256).
bool pair_ok(const CallMats &cm, const std::vector<HostBlock> &blocks, const himuon_ns_params &p) {
  if (p.tile != 256 || !onchip_storage_ok(cm, blocks, p)) return false;
  for (const HostBlock &b : blocks)
    if (b.T != 256) return false;
  return true;
}

int resident_pack(const CallMats &cm, const std::vector<HostBlock> &blocks, const himuon_ns_params &p) {
  if (!onchip_storage_ok(cm, blocks, p)) return 0;
  const int pack = (p.tile == 64 || p.tile == 32) ? 128 / p.tile : 1;
  for (const HostBlock &b : blocks) {
    if (pack > 1) {
      if (b.T != p.tile) return 0;
    } else {
      const bool single = b.T >= std::max(b.rows, b.cols) && std::max(b.rows, b.cols) <= 128;
      if (!(b.T == 128 || single)) return 0;
    }
  }
  return pack;
}

std::string plan_key(int device, int op, const CallMats &cm, const himuon_split *splits, const himuon_ns_params &p) {
  std::string k;
  auto put = [&k](const void *d, size_t n) { k.append(static_cast<const char *>(d), n); };
  put(&device, sizeof device);
  put(&op, sizeof op);
  put(&cm.n, sizeof cm.n);
  put(&p.tile, sizeof p.tile);
  put(&p.compute, sizeof p.compute);
  const int staged = force_staged() ? 1 : 0;
  put(&staged, sizeof staged);
  for (int r = 0; r < kNumRoles; ++r) {
    const int present = cm.role[r] ? 1 : 0;
    put(&present, sizeof present);
    if (!present) continue;
    for (int32_t i = 0; i < cm.n; ++i) {
      const himuon_mat &m = cm.role[r][i];
      put(&m.data, sizeof m.data);
      put(&m.rows, sizeof m.rows);
      put(&m.cols, sizeof m.cols);
      put(&m.ld, sizeof m.ld);
      put(&m.dtype, sizeof m.dtype);
    }
  }
  for (int32_t i = 0; i < cm.n; ++i) {
    const int32_t nb = (splits && splits[i].nblocks > 1) ? splits[i].nblocks : 0;
    put(&nb, sizeof nb);
    if (nb) {
      put(&splits[i].dim, sizeof splits[i].dim);
      put(splits[i].sizes, sizeof(int64_t) * nb);
    }
  }
  return k;
}

struct PlanCache {
  std::mutex mu;   // lookups from several host threads do not corrupt the cache
  std::list<std::pair<std::string, std::shared_ptr<Plan>>> lru;
  std::map<std::string, std::list<std::pair<std::string, std::shared_ptr<Plan>>>::iterator> index;
  static constexpr size_t kCap = 64;   // a per-matrix-T call takes one entry per tile size
};
PlanCache &cache() {
  static PlanCache *c = new PlanCache();  // never destroyed: avoids freeing at exit after the context is gone
  return *c;
}

// Tiles whose short side is at most this are "thin": rounding their operands
// to bf16's 8 significant bits moves their output singular values by up to
// ~0.1 (a 16-bit operand type with 11 bits keeps them near 0.01).
constexpr int64_t kThinSide = 64;

// Staged tile classes: tiles grouped by padded iterate shape (n, m), n <= m
// (multiples of 128, tall tiles transposed), thin tiles in classes of their own.
void staged_classes(const std::vector<HostBlock> &blocks, std::vector<TileClass> &classes) {
  std::map<std::tuple<int64_t, int64_t, bool>, size_t> cls;
  for (size_t bi = 0; bi < blocks.size(); ++bi) {
    const HostBlock &b = blocks[bi];
    for (int64_t tr = 0; tr < b.tiles_r; ++tr)
      for (int64_t tc = 0; tc < b.tiles_c; ++tc) {
        DevTile t;
        t.block = static_cast<int32_t>(bi);
        t.r0 = static_cast<int32_t>(tr * b.T);
        t.c0 = static_cast<int32_t>(tc * b.T);
        t.h = static_cast<int32_t>(std::min(b.T, b.rows - t.r0));
        t.w = static_cast<int32_t>(std::min(b.T, b.cols - t.c0));
        t.transposed = t.h > t.w ? 1 : 0;
        const int64_t n = round_up(std::min(t.h, t.w), 128), m = round_up(std::max(t.h, t.w), 128);
        const bool thin = std::min(t.h, t.w) <= kThinSide;
        const auto key = std::make_tuple(n, m, thin);
        auto it = cls.find(key);
        if (it == cls.end()) {
          it = cls.emplace(key, classes.size()).first;
          TileClass c;
          c.n = n;
          c.m = m;
          c.padded = false;
          c.thin = thin;
          classes.push_back(c);
        }
        TileClass &c = classes[it->second];
        if (std::min(t.h, t.w) != n || std::max(t.h, t.w) != m) c.padded = true;
        c.tiles.push_back(t);
      }
  }
}

// Arithmetic of a staged class.  A bf16 call runs Gram NS with fp16 operands
// (the Gram Newton-Schulz page prescribes fp16 over bf16 for it), and thin
// tiles of standard NS in fp32 on the CUDA cores; otherwise as asked.
int class_compute(const TileClass &c, int op, int compute) {
  if (compute != HIMUON_BF16) return compute;
  if (op == HIMUON_OP_GRAM_NS) return HIMUON_FP16;
  return c.thin ? HIMUON_FP32 : HIMUON_BF16;
}

int build_plan(int device, int op, const CallMats &cm, const himuon_split *splits, const himuon_ns_params &p,
               std::shared_ptr<Plan> &out) {
  auto plan = std::make_shared<Plan>();
  plan->device = device;
  int rc = make_blocks(cm, splits, op == HIMUON_OP_NS_FULL ? 0 : p.tile, plan->blocks,
                       &plan->n_tiles);
  if (rc) return rc;
  const bool onchip_ok = op != HIMUON_OP_GRAM_NS && !force_staged();
  const bool pair = onchip_ok && pair_ok(cm, plan->blocks, p);
  const int pack = (onchip_ok && !pair) ? resident_pack(cm, plan->blocks, p) : 0;
  const bool resident = pack > 0 || pair;   // tiles on chip, read through tensor maps
  plan->path = pair ? kPathPair : (pack > 0 ? kPathResident : kPathStaged);
  plan->pack = pack > 0 ? pack : 1;

  std::vector<DevBlock> dblocks(plan->blocks.size());
  std::vector<CUtensorMap> tmaps;
  for (size_t bi = 0; bi < plan->blocks.size(); ++bi) {
    const HostBlock &b = plan->blocks[bi];
    DevBlock &d = dblocks[bi];
    memset(&d, 0, sizeof d);
    d.tile_begin = b.tile_begin;
    d.tiles_r = static_cast<int32_t>(b.tiles_r);
    d.tiles_c = static_cast<int32_t>(b.tiles_c);
    d.rows = static_cast<int32_t>(b.rows);
    d.cols = static_cast<int32_t>(b.cols);
    d.T = (resident && !pair) ? 128 / pack : static_cast<int32_t>(b.T);
    d.mat = b.mat;
    for (int r = 0; r < kNumRoles; ++r) {
      d.tmap[r] = -1;
      if (!cm.role[r]) continue;
      const himuon_mat &m = cm.role[r][b.mat];
      d.ptr[r] = block_ptr(m, b);
      d.ld[r] = m.ld;
      d.dtype[r] = m.dtype;
      if (resident) {
        CUtensorMap tm;
        if (!make_block_map(&tm, d.ptr[r], b.rows, b.cols, m.ld, pair ? 1 : pack)) return HIMUON_ERR_CUDA;
        d.tmap[r] = static_cast<int32_t>(tmaps.size());
        tmaps.push_back(tm);
      }
    }
  }
  std::vector<DevTile> dtiles;
  if (!resident) {
    staged_classes(plan->blocks, plan->classes);
    for (TileClass &c : plan->classes) {
      c.dev_offset = static_cast<int64_t>(dtiles.size());
      dtiles.insert(dtiles.end(), c.tiles.begin(), c.tiles.end());
    }
  }
  // one device buffer: blocks | tensor maps (64-byte aligned) | tiles
  const size_t sb = round_up(sizeof(DevBlock) * dblocks.size(), 128);
  const size_t st = round_up(sizeof(CUtensorMap) * tmaps.size(), 128);
  const size_t stl = sizeof(DevTile) * dtiles.size();
  const size_t total = sb + st + stl + 128;
  std::vector<char> host(total, 0);
  memcpy(host.data(), dblocks.data(), sizeof(DevBlock) * dblocks.size());
  if (!tmaps.empty()) memcpy(host.data() + sb, tmaps.data(), sizeof(CUtensorMap) * tmaps.size());
  if (!dtiles.empty()) memcpy(host.data() + sb + st, dtiles.data(), stl);
  if (cudaMalloc(&plan->dev, total) != cudaSuccess) return HIMUON_ERR_CUDA;
  if (cudaMemcpy(plan->dev, host.data(), total, cudaMemcpyHostToDevice) != cudaSuccess) return HIMUON_ERR_CUDA;
  plan->d_blocks = static_cast<DevBlock *>(plan->dev);
  plan->d_tmaps = reinterpret_cast<CUtensorMap *>(static_cast<char *>(plan->dev) + sb);
  plan->d_tiles = reinterpret_cast<DevTile *>(static_cast<char *>(plan->dev) + sb + st);
  if (log_enabled()) {
    fprintf(stderr, "[himuon] plan: op=%d path=%s blocks=%zu tiles=%lld classes=%zu tmaps=%zu\n", op,
            pair ? "pair" : (resident ? "resident" : "staged"), plan->blocks.size(), (long long)plan->n_tiles,
            plan->classes.size(), tmaps.size());
    for (const TileClass &c : plan->classes)
      fprintf(stderr, "[himuon]   class n=%lld m=%lld tiles=%zu padded=%d thin=%d compute=%d\n", (long long)c.n,
              (long long)c.m, c.tiles.size(), (int)c.padded, (int)c.thin, class_compute(c, op, p.compute));
  }
  out = plan;
  return HIMUON_OK;
}

int get_plan(int op, const CallMats &cm, const himuon_split *splits, const himuon_ns_params &p,
             std::shared_ptr<Plan> &out) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return HIMUON_ERR_NO_DEVICE;
  const std::string key = plan_key(device, op, cm, splits, p);
  PlanCache &c = cache();
  std::lock_guard<std::mutex> lock(c.mu);
  auto it = c.index.find(key);
  if (it != c.index.end()) {
    c.lru.splice(c.lru.begin(), c.lru, it->second);
    out = it->second->second;
    return HIMUON_OK;
  }
  std::shared_ptr<Plan> plan;
  const int rc = build_plan(device, op, cm, splits, p, plan);
  if (rc) return rc;
  c.lru.emplace_front(key, plan);
  c.index[key] = c.lru.begin();
  while (c.lru.size() > PlanCache::kCap) {
    c.index.erase(c.lru.back().first);
    c.lru.pop_back();
  }
  out = plan;
  return HIMUON_OK;
}

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return HIMUON_ERR_NO_DEVICE;
  }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return HIMUON_ERR_NO_DEVICE;
  return major == 10 ? HIMUON_OK : HIMUON_ERR_NO_DEVICE;
}

// ---------------------------------------------------------------- workspace layout
struct WsLayout {
  size_t x32a, x32b, x16a, x16b, a32, a16, b32, b16, q32, q16a, q16b, z32, z16, rz32, rz16, partial, scale, total;
};

// The 16-bit element paths of one call: bf16 NS packs the input unscaled and
// its first products apply 1/rho (prescale); other 16-bit calls without a
// momentum update (fp16 NS, Gram NS) sum squares in one pass over the input
// and write the scaled operand in a second (two_pass); the rest pack to fp32
// and normalise from there.
bool staged_prescale(int compute, int op) { return compute == HIMUON_BF16 && op != HIMUON_OP_GRAM_NS; }
bool staged_two_pass(int compute, int op) {
  return compute != HIMUON_FP32 && !staged_prescale(compute, op) && op != HIMUON_OP_MOMENTUM_STEP;
}

WsLayout ws_layout(int64_t n, int64_t m, int64_t count, int compute, int op) {
  const bool gram = op == HIMUON_OP_GRAM_NS;
  WsLayout L;
  memset(&L, 0, sizeof L);
  size_t off = 0;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off += round_up(static_cast<int64_t>(bytes), 256);
    return o;
  };
  const size_t nm = static_cast<size_t>(n * m * count), nn = static_cast<size_t>(n * n * count);
  const bool f32 = compute == HIMUON_FP32;
  // fp32 X: the fp32 path's iterate, and the input the normalisation pass
  // reads (the fp16 momentum step).  The other 16-bit paths pack straight to
  // 16 bits and their last product writes the caller's buffers.
  if (f32 || (!staged_prescale(compute, op) && !staged_two_pass(compute, op))) L.x32a = take(4 * nm);
  if (f32) L.x32b = take(4 * nm);
  else {
    L.x16a = take(2 * nm);
    L.x16b = take(2 * nm);
  }
  if (f32 || gram) L.a32 = take(4 * nn);   // (the 16-bit NS path keeps A in 16 bits only)
  if (!f32) L.a16 = take(2 * nn);
  if (!gram) {
    if (f32) L.b32 = take(4 * nn);
    else L.b16 = take(2 * nn);
  } else {
    // fp32 R (a32) and RZ in both arithmetics (C terms); Q and Z in fp32 only
    // when they are the operands
    L.rz32 = take(4 * nn);
    if (f32) {
      L.q32 = take(4 * nn);
      L.z32 = take(4 * nn);
      L.b32 = take(4 * nn);   // second Q buffer
    } else {
      L.q16a = take(2 * nn);
      L.q16b = take(2 * nn);
      L.z16 = take(2 * nn);
      L.rz16 = take(2 * nn);
    }
  }
  const int64_t parts = (std::max(n, m) + 31) / 32;
  L.partial = take(4 * parts * count);
  L.scale = take(8 * count);   // per-tile 1 / rho and 1 / rho^2 (the bf16 path)
  L.total = off;
  return L;
}

size_t chunk_limit(size_t ws_bytes, const himuon_ns_params &p) {
  size_t lim = ws_bytes;
  if (p.chunk_bytes > 0 && static_cast<size_t>(p.chunk_bytes) < lim) lim = static_cast<size_t>(p.chunk_bytes);
  return lim;
}

// Tiles per chunk of a class under the limit (0 if even one tile does not fit):
// the fewest chunks the limit allows, of equal size (a last chunk of a tile or
// two would run every product of the call once more at a tiny batch).
int64_t chunk_tiles(const TileClass &c, size_t limit, int compute, int op) {
  const int64_t tiles = static_cast<int64_t>(c.tiles.size());
  if (tiles < 1 || ws_layout(c.n, c.m, 1, compute, op).total > limit) return 0;
  int64_t lo = 1, hi = std::min<int64_t>(tiles, 65535);   // the workspace grows with the tile count
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (ws_layout(c.n, c.m, mid, compute, op).total <= limit) lo = mid;
    else hi = mid - 1;
  }
  const int64_t chunks = (tiles + lo - 1) / lo;
  return (tiles + chunks - 1) / chunks;
}

int64_t staged_ws_bytes(const Plan &plan, int op, int compute) {
  int64_t need = 0;
  for (const TileClass &c : plan.classes)
    need = std::max<int64_t>(need,
                             static_cast<int64_t>(ws_layout(c.n, c.m, 1, class_compute(c, op, compute), op).total));
  return need;
}

// ---------------------------------------------------------------- staged drivers
#define HIMUON_TRY(x)                      \
  do {                                     \
    cudaError_t e_ = (x);                  \
    if (e_ != cudaSuccess) return HIMUON_ERR_CUDA; \
  } while (0)

struct Ops {
  int compute;
  int32_t op16;   // operand dtype of the 16-bit copies
  int *status;
  cudaStream_t stream;
  // acc = A op(B), batched; A, B given by (pointer, rows, cols) of 16-bit or fp32 storage
  int mm(void *a, int64_t ar, int64_t ac, void *b, int64_t br, int64_t bc, int b_trans, int64_t M, int64_t N,
         int64_t K, int64_t batch, const Epilogue &ep) const {
    const int32_t dt = compute == HIMUON_FP32 ? HIMUON_FP32 : op16;
    Batch A{a, ar, ac, ar * ac, dt}, B{b, br, bc, br * bc, dt};
    cudaError_t e = compute == HIMUON_FP32 ? gemm_simt(A, B, b_trans, M, N, K, batch, ep, stream)
                                           : gemm_tc(A, B, b_trans, M, N, K, batch, ep, status, stream);
    return e == cudaSuccess ? HIMUON_OK : HIMUON_ERR_CUDA;
  }
};

Epilogue epi(float alpha, float beta, const float *c32, float *out32, void *out16, int32_t dt) {
  Epilogue e;
  e.alpha = alpha;
  e.beta = beta;
  e.c32 = c32;
  e.c16 = nullptr;
  e.alpha_batch = nullptr;
  e.out32 = out32;
  e.out16 = out16;
  e.out16_dtype = dt;
  e.diag = 0.f;
  e.out2_32 = nullptr;
  e.out2_16 = nullptr;
  e.diag2 = 0.f;
  e.sym = 0;
  e.lower32 = 0;
  e.sc_tiles = nullptr;
  e.sc_blocks = nullptr;
  e.sc_mode = 0;
  e.sc_lr = 0.f;
  return e;
}
Epilogue sym(Epilogue e) {
  e.sym = 1;
  return e;
}

int run_staged(const Plan &plan, int op, const himuon_ns_params &p, float mu, float lr, void *ws, size_t ws_bytes,
               cudaStream_t stream) {
  const bool gram = op == HIMUON_OP_GRAM_NS;
  const bool step = op == HIMUON_OP_MOMENTUM_STEP;
  const size_t limit = chunk_limit(ws_bytes, p);
  const float safety = p.safety > 0.f ? p.safety : 1.f;
  char *W = static_cast<char *>(ws);
  for (const TileClass &c : plan.classes) {
    const int compute = class_compute(c, op, p.compute);
    const bool f32 = compute == HIMUON_FP32;
    Ops ops{compute, compute == HIMUON_FP16 ? HIMUON_FP16 : HIMUON_BF16, status_ptr(), stream};
    const int32_t dt16 = ops.op16;
    const int64_t per = chunk_tiles(c, limit, compute, op);
    if (per < 1) return HIMUON_ERR_WORKSPACE;
    const int64_t n = c.n, m = c.m;
    for (int64_t t0 = 0; t0 < static_cast<int64_t>(c.tiles.size()); t0 += per) {
      const int64_t bc = std::min<int64_t>(per, static_cast<int64_t>(c.tiles.size()) - t0);
      const WsLayout L = ws_layout(n, m, bc, compute, op);
      float *x32[2] = {reinterpret_cast<float *>(W + L.x32a), f32 ? reinterpret_cast<float *>(W + L.x32b) : nullptr};
      void *x16[2] = {f32 ? nullptr : W + L.x16a, f32 ? nullptr : W + L.x16b};
      float *a32 = (f32 || gram) ? reinterpret_cast<float *>(W + L.a32) : nullptr;
      void *a16 = f32 ? nullptr : W + L.a16;
      const DevTile *tiles = plan.d_tiles + c.dev_offset + t0;
      // bf16 NS: the input goes to the bf16 operand as it is and the first
      // step's two products over X apply 1 / rho^2 and 1 / rho in their
      // epilogues (no normalisation pass, no fp32 copy of the input).  fp16
      // keeps the pass: an unnormalised input may not fit fp16's range.
      const bool prescale = staged_prescale(compute, op);
      const bool two_pass = staged_two_pass(compute, op);
      float *inv = reinterpret_cast<float *>(W + L.scale), *inv2 = inv + bc;
      if (c.padded) {   // the zero padding of ragged tiles (pack writes the valid part only)
        if (prescale || two_pass) HIMUON_TRY(cudaMemsetAsync(x16[0], 0, 2 * n * m * bc, stream));
        else HIMUON_TRY(cudaMemsetAsync(x32[0], 0, sizeof(float) * n * m * bc, stream));
      }
      PackArgs pk;
      pk.blocks = plan.d_blocks;
      pk.tiles = tiles;
      pk.n_tiles = bc;
      pk.n = n;
      pk.m = m;
      pk.x32 = (prescale || two_pass) ? nullptr : x32[0];
      pk.x16 = prescale ? x16[0] : nullptr;   // two_pass: sums of squares only, first
      pk.x16_dtype = dt16;
      pk.scale = nullptr;
      pk.partial = reinterpret_cast<float *>(W + L.partial);
      pk.parts = static_cast<int32_t>((std::max(n, m) + 31) / 32);
      pk.mode = step ? 1 : 0;
      pk.mu = mu;
      HIMUON_TRY(launch_pack(pk, stream));
      if (prescale || two_pass) {
        HIMUON_TRY(launch_tile_scales(pk.partial, pk.parts, bc, p.eps, safety, inv, inv2, stream));
        if (two_pass) {   // the scaled 16-bit operand from a second pass over the input
          pk.x16 = x16[0];
          pk.scale = inv;
          HIMUON_TRY(launch_pack(pk, stream));
        }
      } else {
        NormArgs na;
        na.n_tiles = bc;
        na.elems = n * m;
        na.x32 = x32[0];
        na.x16 = f32 ? nullptr : x16[0];
        na.x16_dtype = dt16;
        na.partial = pk.partial;
        na.parts = pk.parts;
        na.keep32 = f32 ? 1 : 0;   // the fp16 momentum step reads only the 16-bit copy
        na.eps = p.eps;
        na.safety = safety;
        HIMUON_TRY(launch_normalize(na, stream));
      }
      int cur = 0;  // which x buffer holds the current operand
      float *xfinal = x32[0];
      int rc = HIMUON_OK;
      // operand views: fp32 path reads the fp32 buffers directly
      auto xop = [&](int i) -> void * { return f32 ? static_cast<void *>(x32[i]) : x16[i]; };
      // the last product of the 16-bit paths writes the blocks' roles itself
      // (no fp32 copy of the result and no unpack pass)
      auto scatter = [&](Epilogue e) {
        e.out32 = nullptr;
        e.out16 = nullptr;
        e.sc_tiles = tiles;
        e.sc_blocks = plan.d_blocks;
        e.sc_mode = step ? 1 : 0;
        e.sc_lr = lr;
        return e;
      };
      if (!gram) {
        void *bop = f32 ? static_cast<void *>(W + L.b32) : W + L.b16;
        for (int t = 0; t < p.steps && rc == HIMUON_OK; ++t) {
          const float a = p.coeffs[3 * t], b = p.coeffs[3 * t + 1], cc = p.coeffs[3 * t + 2];
          // A = X X^T  (step 0 of the bf16 path: (X X^T) / rho^2)
          Epilogue e1 = sym(epi(1.f, 0.f, nullptr, f32 ? a32 : nullptr, a16, dt16));
          if (prescale && t == 0) e1.alpha_batch = inv2;
          rc = ops.mm(xop(cur), n, m, xop(cur), n, m, 1, n, n, m, bc, e1);
          if (rc) break;
          // 16-bit operands: Bop = r(b r(A) + c r(A) r(A) + a I), and X <- r(Bop X)
          // (fp32 accumulation, the whole update in one product, as on chip; the
          // b A term reads the same 16-bit A as the product's operands, whose
          // rounding is of the size of Bop's own).
          // fp32: B' = b A + c A A + (a - 1) I, and X <- X + B' X on the fp32 master.
          Epilogue e2 = epi(cc, b, f32 ? a32 : nullptr, f32 ? static_cast<float *>(bop) : nullptr, f32 ? nullptr : bop, dt16);
          if (!f32) e2.c16 = a16;
          e2.diag = f32 ? a - 1.f : a;
          e2.sym = 1;
          rc = ops.mm(f32 ? static_cast<void *>(a32) : a16, n, n, f32 ? static_cast<void *>(a32) : a16, n, n, 0, n, n,
                      n, bc, e2);
          if (rc) break;
          // X = a X + B X
          if (f32) {
            rc = ops.mm(bop, n, n, x32[cur], n, m, 0, n, m, n, bc, epi(1.f, 1.f, x32[cur], x32[1 - cur], nullptr, dt16));
            cur = 1 - cur;
            xfinal = x32[cur];
          } else {
            // the 16-bit operand for the next step, or the fp32 result after the last
            // (step 0 of the bf16 path: Bop (X / rho) = (Bop X) / rho)
            const bool last = t + 1 == p.steps;
            Epilogue e3 = epi(1.f, 0.f, nullptr, nullptr, x16[1 - cur], dt16);
            if (last) e3 = scatter(e3);
            if (prescale && t == 0) e3.alpha_batch = inv;
            rc = ops.mm(bop, n, n, x16[cur], n, m, 0, n, m, n, bc, e3);
            cur = 1 - cur;
          }
        }
      } else {
        // Gram NS (Algorithm 3): R = X X^T, Q = I; restarts X <- Q X.  The terms
        // a R, a RZ stay fp32 (C operands): folding a I into a 16-bit Z, or
        // reading R or RZ rounded to 16 bits, loses R's small eigen-directions,
        // which later steps feed back (fp16 R and RZ terms: 4.6% error on a
        // 256 x 1024 input without a restart).  It is fp16's precision, not its
        // range: the same copies scaled by 2^8 .. 2^14, all entries normal,
        // lose as much.  The
        // a Q term reads the 16-bit Q: Q's eigenvalues stay of the order of a
        // or above and Q is never fed back into R, so its rounding costs
        // nothing (equal or smaller errors under every restart pattern tried,
        // in an fp16 emulation against the fp64 map).  Between
        // restarts every n x n matrix here is a polynomial in one R, so all of
        // them commute and every n x n product is symmetric: computed as its
        // lower triangle.
        float *r32 = a32, *q32 = reinterpret_cast<float *>(W + L.q32), *z32 = reinterpret_cast<float *>(W + L.z32);
        float *rz32 = reinterpret_cast<float *>(W + L.rz32);
        float *q32b = f32 ? reinterpret_cast<float *>(W + L.b32) : nullptr;
        void *r16 = a16, *z16 = f32 ? nullptr : W + L.z16, *rz16 = f32 ? nullptr : W + L.rz16;
        void *q16[2] = {f32 ? nullptr : W + L.q16a, f32 ? nullptr : W + L.q16b};
        float *qf[2] = {f32 ? q32 : nullptr, q32b};   // fp32 Q: the fp32 path only
        int qc = 0;
        auto rop = [&]() -> void * { return f32 ? static_cast<void *>(r32) : r16; };
        auto zop = [&]() -> void * { return f32 ? static_cast<void *>(z32) : z16; };
        auto rzop = [&]() -> void * { return f32 ? static_cast<void *>(rz32) : rz16; };
        auto qop = [&](int i) -> void * { return f32 ? static_cast<void *>(qf[i]) : q16[i]; };
        bool q_identity = true;
        // every fp32 n x n matrix here is read only as the C term of another
        // symmetric product: its blocks above the diagonal are never written
        auto gsym = [f32](Epilogue e) {
          e.sym = 1;
          e.lower32 = f32 ? 0 : 1;
          return e;
        };
        auto restarts_at = [&p](int t) {
          for (int i = 0; i < p.n_restart; ++i)
            if (p.restart_at[i] == t) return true;
          return false;
        };
        rc = ops.mm(xop(cur), n, m, xop(cur), n, m, 1, n, n, m, bc, gsym(epi(1.f, 0.f, nullptr, r32, r16, dt16)));
        for (int t = 1; t <= p.steps && rc == HIMUON_OK; ++t) {
          const float a = p.coeffs[3 * (t - 1)], b = p.coeffs[3 * (t - 1) + 1], cc = p.coeffs[3 * (t - 1) + 2];
          const bool restart = restarts_at(t);
          // After the last step, or before a restart (which rebuilds R from the
          // new X and resets Q), this step's R, RZ and fp32 Q are never read:
          // those products and writes are skipped (the results are unchanged).
          const bool last_use = t == p.steps || restarts_at(t + 1);
          if (restart) {
            if (!q_identity) {  // X <- Q X
              if (f32) {
                rc = ops.mm(qop(qc), n, n, x32[cur], n, m, 0, n, m, n, bc, epi(1.f, 0.f, nullptr, x32[1 - cur], nullptr, dt16));
                cur = 1 - cur;
                xfinal = x32[cur];
              } else {
                // (the fp32 copy of X is written by the final product only)
                rc = ops.mm(qop(qc), n, n, x16[cur], n, m, 0, n, m, n, bc, epi(1.f, 0.f, nullptr, nullptr, x16[1 - cur], dt16));
                cur = 1 - cur;
              }
              if (rc) break;
              rc = ops.mm(xop(cur), n, m, xop(cur), n, m, 1, n, n, m, bc, gsym(epi(1.f, 0.f, nullptr, r32, r16, dt16)));
              if (rc) break;
            }
            q_identity = true;
          }
          // Z = b R + c R^2 (fp32 copy only when the operands are fp32).  Right
          // after Q = I the same epilogue also writes Q <- Q Z + a Q = Z + a I.
          Epilogue ez = gsym(epi(cc, b, r32, f32 ? z32 : nullptr, z16, dt16));
          if (q_identity) {
            ez.out2_32 = f32 ? qf[qc] : nullptr;
            ez.out2_16 = f32 ? nullptr : q16[qc];
            ez.diag2 = a;
          }
          rc = ops.mm(rop(), n, n, rop(), n, n, 0, n, n, n, bc, ez);
          if (rc) break;
          // Q <- Q Z + a Q
          if (q_identity) {
            q_identity = false;
          } else {
            Epilogue eq = f32 ? epi(1.f, a, qf[qc], qf[1 - qc], nullptr, dt16) : epi(1.f, a, nullptr, nullptr, q16[1 - qc], dt16);
            if (!f32) eq.c16 = q16[qc];
            rc = ops.mm(qop(qc), n, n, zop(), n, n, 0, n, n, n, bc, gsym(eq));
            qc = 1 - qc;
            if (rc) break;
          }
          if (last_use) continue;   // R_K, and R before a restart, are never used
          // RZ <- R Z + a R
          rc = ops.mm(rop(), n, n, zop(), n, n, 0, n, n, n, bc, gsym(epi(1.f, a, r32, rz32, rz16, dt16)));
          if (rc) break;
          // R <- Z RZ + a RZ
          rc = ops.mm(zop(), n, n, rzop(), n, n, 0, n, n, n, bc, gsym(epi(1.f, a, rz32, r32, r16, dt16)));
        }
        if (rc == HIMUON_OK) {
          // output Q X
          if (f32) {
            rc = ops.mm(qop(qc), n, n, x32[cur], n, m, 0, n, m, n, bc, epi(1.f, 0.f, nullptr, x32[1 - cur], nullptr, dt16));
            xfinal = x32[1 - cur];
          } else {
            rc = ops.mm(qop(qc), n, n, x16[cur], n, m, 0, n, m, n, bc, scatter(epi(1.f, 0.f, nullptr, nullptr, nullptr, dt16)));
          }
        }
      }
      if (rc) return rc;
      if (!f32) continue;   // written by the last product's epilogue
      UnpackArgs ua;
      ua.blocks = plan.d_blocks;
      ua.tiles = tiles;
      ua.n_tiles = bc;
      ua.n = n;
      ua.m = m;
      ua.x32 = xfinal;
      ua.mode = step ? 1 : 0;
      ua.lr = lr;
      HIMUON_TRY(launch_unpack(ua, stream));
    }
  }
  return HIMUON_OK;
}

int run_resident(const Plan &plan, int op, const himuon_ns_params &p, float mu, float lr, bool has_w, bool has_o,
                 cudaStream_t stream) {
  if (plan.n_tiles == 0) return HIMUON_OK;
  ResidentArgs a;
  memset(&a, 0, sizeof a);
  a.blocks = plan.d_blocks;
  a.tmaps = plan.d_tmaps;
  a.n_blocks = static_cast<int32_t>(plan.blocks.size());
  a.K = p.steps;
  a.n_tiles = plan.n_tiles;
  a.mode = op == HIMUON_OP_MOMENTUM_STEP ? 1 : 0;
  a.has_w = has_w ? 1 : 0;
  a.has_o = has_o ? 1 : 0;
  a.op_fmt = p.compute == HIMUON_FP16 ? 0 : 1;
  a.f16_small = p.compute == HIMUON_BF16 ? 1 : 0;
  a.mu = mu;
  a.lr = lr;
  a.eps = p.eps;
  a.safety = p.safety > 0.f ? p.safety : 1.f;
  a.status = status_ptr();
  // the kernel keeps a compact copy of the block table in shared memory when
  // it fits: 32-bit tile numbers, 16-bit tile counts and tensor-map indices
  bool fits = static_cast<int>(plan.blocks.size()) <= resident_max_smem_blocks() && plan.n_tiles < (int64_t(1) << 31);
  for (const HostBlock &b : plan.blocks) fits = fits && b.tiles_c < 65536 && b.cols < (int64_t(1) << 31);
  a.smem_blocks = fits ? 1 : 0;
  a.pack = plan.pack;
  // HIMUON_TEST_STALL=1 exercises the device timeout path (tests only): the
  // call then ends with HIMUON_ERR_TIMEOUT in the device status word.
  const char *stall = getenv("HIMUON_TEST_STALL");
  a.test_stall = (stall && stall[0] == '1') ? 1 : 0;
  make_resident_steps(a, p.coeffs, p.steps);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, plan.device);
  if (const int cap = max_ctas()) sms = std::max(2, std::min(sms, cap));
  if (plan.path == kPathPair) {   // one 256 x 256 tile per CTA pair at a time
    const int pairs = static_cast<int>(std::min<int64_t>(sms / 2, plan.n_tiles));
    return launch_ns_pair(a, pairs, stream) == cudaSuccess ? HIMUON_OK : HIMUON_ERR_CUDA;
  }
  const int64_t n_super = (plan.n_tiles + plan.pack - 1) / plan.pack;
  const int64_t want = (n_super + 1) / 2;
  const int grid = static_cast<int>(std::min<int64_t>(sms, want));
  return launch_ns_resident(a, grid, stream) == cudaSuccess ? HIMUON_OK : HIMUON_ERR_CUDA;
}

// One call's checks and plan, kept apart from its launch so that a call with
// per-matrix tile sizes can check every group before enqueuing the first.
struct Prepared {
  int op = 0;
  std::shared_ptr<Plan> plan;
  himuon_ns_params p{};
  bool has_w = false, has_o = false;
};

int prepare(int op, const CallMats &cm, const himuon_split *splits, const himuon_ns_params *p, void *ws,
            size_t ws_bytes, Prepared &pr) {
  int rc = check_params(p);
  if (rc) return rc;
  rc = check_call(cm, splits);
  if (rc) return rc;
  rc = check_device();
  if (rc) return rc;
  rc = get_plan(op, cm, splits, *p, pr.plan);
  if (rc) return rc;
  pr.op = op;
  pr.p = *p;
  pr.has_w = op == HIMUON_OP_MOMENTUM_STEP && cm.role[kRoleW];
  pr.has_o = cm.role[kRoleOut] != nullptr;
  if (pr.plan->path != kPathStaged) return HIMUON_OK;
  const int64_t need = staged_ws_bytes(*pr.plan, op, p->compute);
  if (!ws || static_cast<int64_t>(ws_bytes) < need) return HIMUON_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return HIMUON_ERR_ALIGNMENT;
  return HIMUON_OK;
}

int launch(const Prepared &pr, float mu, float lr, void *ws, size_t ws_bytes, void *stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pr.plan->path != kPathStaged) return run_resident(*pr.plan, pr.op, pr.p, mu, lr, pr.has_w, pr.has_o, s);
  return run_staged(*pr.plan, pr.op, pr.p, mu, lr, ws, ws_bytes, s);
}

// Matrices of a call regrouped by their tile size (p->tiles): per group, the
// role arrays and splits of its matrices in call order, and the params with
// `tile` set to the group's T.
struct TileGroup {
  int32_t T = 0;
  std::vector<int32_t> idx;
  std::vector<himuon_mat> role[kNumRoles];
  std::vector<himuon_split> splits;
  CallMats cm;
  himuon_ns_params p{};
};

int group_by_tile(const CallMats &cm, const himuon_split *splits, const himuon_ns_params *p,
                  std::vector<TileGroup> &groups) {
  if (cm.n < 1) return HIMUON_ERR_INVALID;
  groups.clear();
  for (int32_t i = 0; i < cm.n; ++i) {
    const int32_t T = p->tiles[i] <= 0 ? 0 : p->tiles[i];
    size_t g = 0;
    while (g < groups.size() && groups[g].T != T) ++g;
    if (g == groups.size()) {
      groups.emplace_back();
      groups.back().T = T;
    }
    groups[g].idx.push_back(i);
  }
  for (TileGroup &g : groups) {
    g.cm.n = static_cast<int32_t>(g.idx.size());
    for (int r = 0; r < kNumRoles; ++r) {
      if (!cm.role[r]) continue;
      for (int32_t i : g.idx) g.role[r].push_back(cm.role[r][i]);
      g.cm.role[r] = g.role[r].data();
    }
    if (splits)
      for (int32_t i : g.idx) g.splits.push_back(splits[i]);
    g.p = *p;
    g.p.tile = g.T;
    g.p.tiles = nullptr;
  }
  return HIMUON_OK;
}

// Tiled NS picks full-matrix NS for T <= 0; the other ops take T as given.
int group_op(int op, int32_t T) {
  if (op == HIMUON_OP_NS_TILED || op == HIMUON_OP_NS_FULL) return T <= 0 ? HIMUON_OP_NS_FULL : HIMUON_OP_NS_TILED;
  return op;
}

int dispatch(int op, const CallMats &cm, const himuon_split *splits, const himuon_ns_params *p, float mu, float lr,
             void *ws, size_t ws_bytes, void *stream) {
  if (p && p->tiles) {
    int rc = check_params(p);   // the whole call first: same error precedence as one group
    if (rc) return rc;
    rc = check_call(cm, splits);
    if (rc) return rc;
    std::vector<TileGroup> groups;
    rc = group_by_tile(cm, splits, p, groups);
    if (rc) return rc;
    std::vector<Prepared> prep(groups.size());
    for (size_t g = 0; g < groups.size(); ++g) {
      rc = prepare(group_op(op, groups[g].T), groups[g].cm, splits ? groups[g].splits.data() : nullptr, &groups[g].p,
                   ws, ws_bytes, prep[g]);
      if (rc) return rc;
    }
    for (const Prepared &pr : prep) {
      rc = launch(pr, mu, lr, ws, ws_bytes, stream);
      if (rc) return rc;
    }
    return HIMUON_OK;
  }
  Prepared pr;
  const int rc = prepare(op, cm, splits, p, ws, ws_bytes, pr);
  if (rc) return rc;
  return launch(pr, mu, lr, ws, ws_bytes, stream);
}

// Device scratch of one call with a single tile size (arguments checked).
int64_t workspace_one(const CallMats &cm, const himuon_split *splits, const himuon_ns_params &p, int op) {
  std::vector<HostBlock> blocks;
  int64_t n_tiles = 0;
  const int64_t tile = op == HIMUON_OP_NS_FULL ? 0 : p.tile;
  int rc = make_blocks(cm, splits, tile, blocks, &n_tiles);
  if (rc) return rc;
  if (op != HIMUON_OP_GRAM_NS && !force_staged() && (pair_ok(cm, blocks, p) || resident_pack(cm, blocks, p) > 0))
    return 0;
  // staged: one tile of the largest class is the minimum; a full chunk of every
  // class makes the call run in one chunk per class.
  int64_t need = 0;
  std::vector<TileClass> classes;
  staged_classes(blocks, classes);
  for (const TileClass &c : classes) {
    const int compute = class_compute(c, op, p.compute);
    int64_t k = std::min<int64_t>(static_cast<int64_t>(c.tiles.size()), 65535);
    int64_t bytes = static_cast<int64_t>(ws_layout(c.n, c.m, k, compute, op).total);
    if (p.chunk_bytes > 0 && bytes > p.chunk_bytes)
      bytes = std::max<int64_t>(p.chunk_bytes, static_cast<int64_t>(ws_layout(c.n, c.m, 1, compute, op).total));
    need = std::max(need, bytes);
  }
  return need;
}

}  // namespace

// Staged NS (in -> out) with every device byte it needs taken from one
// caller-supplied region `scratch` of `scratch_bytes` (256-byte aligned): the
// block and tile tables first, the per-chunk workspace after them.  Builds the
// plan on the host and uploads the tables with cudaMemcpyAsync on `stream`;
// allocates no device memory and does not touch the plan cache.
int run_staged_into(int op, const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                    const himuon_ns_params *p, void *scratch, size_t scratch_bytes, cudaStream_t stream) {
  if (!in || !out || !p || !scratch) return HIMUON_ERR_INVALID;
  if (op != HIMUON_OP_NS_TILED && op != HIMUON_OP_NS_FULL) return HIMUON_ERR_INVALID;
  int rc = check_params(p);
  if (rc) return rc;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = in;
  cm.role[kRoleOut] = out;
  rc = check_call(cm, splits);
  if (rc) return rc;
  rc = check_device();
  if (rc) return rc;
  Plan plan;
  cudaGetDevice(&plan.device);
  rc = make_blocks(cm, splits, op == HIMUON_OP_NS_FULL || p->tile <= 0 ? 0 : p->tile, plan.blocks, &plan.n_tiles);
  if (rc) return rc;
  std::vector<DevBlock> dblocks(plan.blocks.size());
  for (size_t bi = 0; bi < plan.blocks.size(); ++bi) {
    const HostBlock &b = plan.blocks[bi];
    DevBlock &d = dblocks[bi];
    memset(&d, 0, sizeof d);
    d.tile_begin = b.tile_begin;
    d.tiles_r = static_cast<int32_t>(b.tiles_r);
    d.tiles_c = static_cast<int32_t>(b.tiles_c);
    d.rows = static_cast<int32_t>(b.rows);
    d.cols = static_cast<int32_t>(b.cols);
    d.T = static_cast<int32_t>(b.T);
    d.mat = b.mat;
    for (int r = 0; r < kNumRoles; ++r) {
      d.tmap[r] = -1;
      if (!cm.role[r]) continue;
      const himuon_mat &m = cm.role[r][b.mat];
      d.ptr[r] = block_ptr(m, b);
      d.ld[r] = m.ld;
      d.dtype[r] = m.dtype;
    }
  }
  staged_classes(plan.blocks, plan.classes);
  std::vector<DevTile> dtiles;
  for (TileClass &c : plan.classes) {
    c.dev_offset = static_cast<int64_t>(dtiles.size());
    dtiles.insert(dtiles.end(), c.tiles.begin(), c.tiles.end());
  }
  const size_t sb = round_up(sizeof(DevBlock) * dblocks.size(), 256);
  const size_t st = round_up(sizeof(DevTile) * dtiles.size(), 256);
  if (sb + st >= scratch_bytes) return HIMUON_ERR_TOO_LARGE;
  const size_t ws_bytes = scratch_bytes - sb - st;
  if (static_cast<int64_t>(ws_bytes) < staged_ws_bytes(plan, op, p->compute)) return HIMUON_ERR_TOO_LARGE;
  char *base = static_cast<char *>(scratch);
  if (cudaMemcpyAsync(base, dblocks.data(), sizeof(DevBlock) * dblocks.size(), cudaMemcpyHostToDevice, stream) !=
          cudaSuccess ||
      cudaMemcpyAsync(base + sb, dtiles.data(), sizeof(DevTile) * dtiles.size(), cudaMemcpyHostToDevice, stream) !=
          cudaSuccess)
    return HIMUON_ERR_CUDA;
  plan.d_blocks = reinterpret_cast<DevBlock *>(base);
  plan.d_tiles = reinterpret_cast<DevTile *>(base + sb);
  himuon_ns_params q = *p;
  q.chunk_bytes = 0;
  return run_staged(plan, op, q, 0.f, 0.f, base + sb + st, ws_bytes, stream);
}

}  // namespace himuon

using namespace himuon;

extern "C" {

int himuon_ns_tiled(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                    const himuon_ns_params *p, void *ws, size_t ws_bytes, void *stream) {
  if (!in || !out || !p) return HIMUON_ERR_INVALID;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = in;
  cm.role[kRoleOut] = out;
  // with per-matrix tile sizes each group picks tiled or full NS by its own T
  const int op = (p->tiles || p->tile > 0) ? HIMUON_OP_NS_TILED : HIMUON_OP_NS_FULL;
  return dispatch(op, cm, splits, p, 0.f, 0.f, ws, ws_bytes, stream);
}

int himuon_ns_full(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                   const himuon_ns_params *p, void *ws, size_t ws_bytes, void *stream) {
  if (!in || !out || !p) return HIMUON_ERR_INVALID;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = in;
  cm.role[kRoleOut] = out;
  himuon_ns_params q = *p;   // every matrix is one tile: a per-matrix T does not apply
  q.tiles = nullptr;
  return dispatch(HIMUON_OP_NS_FULL, cm, splits, &q, 0.f, 0.f, ws, ws_bytes, stream);
}

int himuon_gram_ns(const himuon_mat *in, const himuon_mat *out, int32_t n, const himuon_split *splits,
                   const himuon_ns_params *p, void *ws, size_t ws_bytes, void *stream) {
  if (!in || !out || !p) return HIMUON_ERR_INVALID;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = in;
  cm.role[kRoleOut] = out;
  return dispatch(HIMUON_OP_GRAM_NS, cm, splits, p, 0.f, 0.f, ws, ws_bytes, stream);
}

int himuon_momentum_step(const himuon_mat *W, const himuon_mat *M, const himuon_mat *G, int32_t n, float mu,
                         float lr, const himuon_split *splits, const himuon_ns_params *p, const himuon_mat *update_out,
                         void *ws, size_t ws_bytes, void *stream) {
  if (!M || !G || !p || (!W && !update_out)) return HIMUON_ERR_INVALID;
  if (!isfinite(mu) || !isfinite(lr)) return HIMUON_ERR_INVALID;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = M;
  cm.role[kRoleG] = G;
  cm.role[kRoleW] = W;
  cm.role[kRoleOut] = update_out;
  return dispatch(HIMUON_OP_MOMENTUM_STEP, cm, splits, p, mu, lr, ws, ws_bytes, stream);
}

int64_t himuon_workspace_size(const himuon_mat *mats, int32_t n, const himuon_split *splits,
                              const himuon_ns_params *p, int32_t op) {
  int rc = check_params(p);
  if (rc) return rc;
  if (!mats || op < HIMUON_OP_NS_TILED || op > HIMUON_OP_MOMENTUM_STEP) return HIMUON_ERR_INVALID;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = mats;
  cm.role[kRoleOut] = mats;
  if (op == HIMUON_OP_MOMENTUM_STEP) cm.role[kRoleOut] = nullptr;
  rc = check_call(cm, splits);
  if (rc) return rc;
  if (!p->tiles || op == HIMUON_OP_NS_FULL) return workspace_one(cm, splits, *p, op);
  std::vector<TileGroup> groups;
  rc = group_by_tile(cm, splits, p, groups);
  if (rc) return rc;
  int64_t need = 0;
  for (const TileGroup &g : groups) {
    const int64_t b = workspace_one(g.cm, splits ? g.splits.data() : nullptr, g.p, group_op(op, g.T));
    if (b < 0) return b;
    need = std::max(need, b);
  }
  return need;
}

int himuon_get_device_status(void *stream) {
  if (check_device() != HIMUON_OK) return HIMUON_ERR_NO_DEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return HIMUON_ERR_CUDA;
  int *p = status_ptr();
  if (!p) return HIMUON_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return HIMUON_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return HIMUON_ERR_CUDA;
  return v;
}

const char *himuon_status_string(int code) {
  switch (code) {
    case HIMUON_OK: return "ok";
    case HIMUON_ERR_INVALID: return "invalid argument";
    case HIMUON_ERR_UNSUPPORTED: return "unsupported dtype, tile size or step count";
    case HIMUON_ERR_WORKSPACE: return "workspace too small";
    case HIMUON_ERR_ALIGNMENT: return "pointer or row pitch not 16-byte aligned";
    case HIMUON_ERR_CUDA: return "CUDA call failed";
    case HIMUON_ERR_TIMEOUT: return "device wait timed out";
    case HIMUON_ERR_DEVICE: return "inconsistent descriptor seen on the device";
    case HIMUON_ERR_NO_DEVICE: return "no usable sm_100 device";
    case HIMUON_ERR_TOO_LARGE: return "problem needs more scratch than himuon_ns_static's fixed device array";
    default: return "unknown status";
  }
}

int himuon_version(void) { return HIMUON_VERSION; }

int64_t himuon_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int64_t himuon_plan_tiles(const himuon_mat *mats, int32_t n, const himuon_split *splits, int32_t tile,
                          int64_t *records, int64_t cap) {
  if (!mats) return HIMUON_ERR_INVALID;
  CallMats cm;
  cm.n = n;
  cm.role[kRoleIn] = mats;
  int rc = check_call(cm, splits);
  if (rc) return rc;
  std::vector<HostBlock> blocks;
  int64_t n_tiles = 0;
  rc = make_blocks(cm, splits, tile, blocks, &n_tiles);
  if (rc) return rc;
  int64_t k = 0;
  for (const HostBlock &b : blocks)
    for (int64_t tr = 0; tr < b.tiles_r; ++tr)
      for (int64_t tc = 0; tc < b.tiles_c; ++tc, ++k) {
        if (!records || k >= cap) continue;
        int64_t *r = records + 5 * k;
        r[0] = b.mat;
        r[1] = b.row0 + tr * b.T;
        r[2] = b.col0 + tc * b.T;
        r[3] = std::min(b.T, b.rows - tr * b.T);
        r[4] = std::min(b.T, b.cols - tc * b.T);
      }
  return n_tiles;
}

}  // extern "C"
