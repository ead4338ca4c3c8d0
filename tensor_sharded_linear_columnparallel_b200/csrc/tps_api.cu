// tps_api.cu -- the C ABI (include/tps.h): argument validation, the head map and
// packed layouts, GEMM planning (tile orientation, tile width, stream-K), TMA
// tensor-map encoding and kernel launches. Host code only; every step of the
// block's arithmetic runs in the kernels of tps_kernels.cu.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tps.h"
#include "tps_internal.h"

namespace {

using tps::GemmArgs;

constexpr unsigned long long kTimeoutNs = 4000000000ull;  // bounded device waits: 4 s

std::atomic<int> g_plan_override{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------------ head map
struct HeadMap {
  int qs, kvs;          // query / KV heads per shard
  int kv_num, kv_den;   // first KV head of shard s = s*kv_num/kv_den
};

int head_map_calc(int hq, int hkv, int tp, HeadMap* hm) {
  if (hq <= 0 || hkv <= 0 || tp <= 0) return TPS_ERR_ARG;
  if (hq % tp != 0 || hq % hkv != 0) return TPS_ERR_DIVISIBILITY;
  HeadMap h{};
  h.qs = hq / tp;
  if (hkv % tp == 0) {
    h.kvs = hkv / tp;
    h.kv_num = hkv / tp;  // s * (hkv/tp)
    h.kv_den = 1;
  } else if (tp % hkv == 0) {
    h.kvs = 1;
    h.kv_num = hkv;       // floor(s*hkv/tp)
    h.kv_den = tp;
  } else {
    return TPS_ERR_DIVISIBILITY;
  }
  *hm = h;
  return TPS_OK;
}

// ------------------------------------------------------------------ packed layouts
struct PackGeom {
  int R;      // packed rows per shard (before padding to 128-row blocks)
  int Kp;     // packed row length (before padding to 64-element K blocks)
  int per_shard;  // valid output columns per shard
  int out_cols;   // output width of the column layer
  HeadMap hm;
  int RB() const { return (R + 127) / 128; }
  int KB() const { return (Kp + 63) / 64; }
  size_t bytes(int tp) const { return static_cast<size_t>(tp) * RB() * 128 * KB() * 64 * 2; }
};

int pack_geom(int kind, int64_t k, int64_t n, int tp, const tps_heads* heads, PackGeom* g) {
  if (k <= 0 || n <= 0 || tp <= 0) return TPS_ERR_ARG;
  if (k > (1LL << 30) || n > (1LL << 30)) return TPS_ERR_ARG;
  PackGeom o{};
  switch (kind) {
    case TPS_KIND_COLUMN:
      if (n % tp) return TPS_ERR_DIVISIBILITY;
      if (k % 8 || (n / tp) % 8) return TPS_ERR_ALIGN;
      o.R = static_cast<int>(n / tp);
      o.Kp = static_cast<int>(k);
      o.per_shard = o.R;
      o.out_cols = static_cast<int>(n);
      break;
    case TPS_KIND_ROW:
      if (k % tp) return TPS_ERR_DIVISIBILITY;
      if ((k / tp) % 8 || n % 8) return TPS_ERR_ALIGN;
      o.R = static_cast<int>(n);
      o.Kp = static_cast<int>(k / tp);
      o.per_shard = o.R;
      o.out_cols = static_cast<int>(n);
      break;
    case TPS_KIND_QKV: {
      if (heads == nullptr) return TPS_ERR_ARG;
      const int rc = head_map_calc(heads->hq, heads->hkv, tp, &o.hm);
      if (rc) return rc;
      if (heads->head_dim <= 0) return TPS_ERR_ARG;
      if (static_cast<int64_t>(heads->hq + 2 * heads->hkv) * heads->head_dim != n) return TPS_ERR_ARG;
      if (k % 8 || heads->head_dim % 8) return TPS_ERR_ALIGN;
      o.R = (o.hm.qs + 2 * o.hm.kvs) * heads->head_dim;
      o.Kp = static_cast<int>(k);
      o.per_shard = o.R;
      o.out_cols = tp * o.R;
      break;
    }
    case TPS_KIND_GATE_UP: {
      if (n % 2) return TPS_ERR_ARG;
      const int64_t I = n / 2;
      if (I % tp) return TPS_ERR_DIVISIBILITY;
      const int64_t Is = I / tp;
      if (k % 8 || Is % 8) return TPS_ERR_ALIGN;
      o.R = static_cast<int>((Is + 127) / 128 * 256);
      o.Kp = static_cast<int>(k);
      o.per_shard = static_cast<int>(Is);
      o.out_cols = static_cast<int>(I);
      break;
    }
    default:
      return TPS_ERR_ARG;
  }
  *g = o;
  return TPS_OK;
}

// ------------------------------------------------------------------ device info
int num_sms_current() {
  int dev = 0;
  int sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
  return sms;
}

int check_device() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TPS_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return TPS_ERR_CUDA;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return TPS_ERR_CUDA;
  if (major != 10 || minor != 0) return TPS_ERR_DEVICE;
  return TPS_OK;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load();
  if (f == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    f = reinterpret_cast<EncodeTiledFn>(p);
    fn.store(f);
  }
  return f;
}

// bf16 3-D tensor map; dims innermost first, strides of dims 1 and 2 in bytes,
// box {64, b1, b2} with the 128-byte swizzle; out-of-range elements read as 0.
int make_map(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
             uint32_t b1, uint32_t b2) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return TPS_ERR_CUDA;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {64, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TPS_OK : TPS_ERR_CUDA;
}

// bf16 4-D tensor map of a packed weight [shard][row block][K block][128][64]
// (shard and row block merged into the outermost dim), box {64, rows, 1, 1},
// 128-byte swizzle. Every box is one contiguous run of rows x 128 B.
int make_wmap(CUtensorMap* m, const void* ptr, int RB, int KB, int tp, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return TPS_ERR_CUDA;
  cuuint64_t dims[4] = {64, 128, static_cast<cuuint64_t>(KB), static_cast<cuuint64_t>(RB) * tp};
  cuuint64_t strides[3] = {128, 128 * 128, static_cast<cuuint64_t>(KB) * 128 * 128};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TPS_OK : TPS_ERR_CUDA;
}

// ------------------------------------------------------------------ planning
struct Problem {
  int static_ws;     // workspace is the static scratch: slots first, counters in its last kStaticCounterBytes
  int kind;          // tps::K_*
  int M, tp;
  int64_t k_inner;   // K extent per shard (column: k, row: k/tp)
  int w_rows;        // packed weight rows per shard (row: n)
  int per_shard;
  bool row, partials;
  int act;
  bool argmax;       // greedy argmax epilogue: whole tiles on one SM each (no pairs, no split)
  bool bf16;         // row-parallel bf16 exchange (TPS_REDUCE_BF16): tp = 1, a cluster split with cs = tp, or a shard chain
  int q_rows;        // QKV: query rows per shard (the shard's KV rows follow them)
  int kv_rep;        // QKV: shards sharing each KV head (tp / hkv when tp > hkv, else 1)
};

struct Plan {
  int swap, bn, dual, sk, grid, gm;
  int pair;           // token-major tile of 256 tokens on a CTA pair (tcgen05 cta_group::2)
  int nh;             // pair tiles: MMA halves of bn weight rows per tile (2 = wide tile of 2*bn rows)
  int cs;             // cluster split-K: cs CTAs share each tile's K range (row-parallel)
  int chain;          // bf16 exchange as a shard chain: one CTA walks a tile's shards in order
  int S_tiles, WT, MT, tiles, KBs, KI;
  int kv_rep, qt;     // QKV with replicated KV heads: KV tiles computed once per group of kv_rep shards
  int wcols;          // weight tiles in the tile space
  int dp_tiles;
  long long T;        // stream-K iterations (tiles past dp_tiles)
  double est;         // modelled cycles per SM
};

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

constexpr size_t kSlotStride = 128 * 256 * 4;  // largest stream-K segment slot (fp32 128 x 256)

size_t slot_region_bytes(int sms) { return 2 * static_cast<size_t>(sms) * kSlotStride; }

constexpr size_t kHdr = tps::kWsHeaderBytes;

// Raster group height: consecutive tiles of the tile space walk gm token tiles
// before the next weight tile, so a wave shares gm token tiles' X and its weight
// tiles in L2. Plan-override bits 24-26 (v = 1..7) force gm = 2^(v-1).
int raster_gm(int MT) {
  const int v = (g_plan_override.load() >> 24) & 7;
  const int gm = v ? (1 << (v - 1)) : 16;
  return std::max(1, std::min(MT, gm));
}   // status word header at the start of a caller workspace

// The status word of a call's workspace: its first int, when the workspace is
// at least as large as its header.
int* ws_status(void* ws, size_t ws_bytes) { return (ws != nullptr && ws_bytes >= kHdr) ? static_cast<int*>(ws) : nullptr; }

size_t slot_bytes(const Plan& p) { return static_cast<size_t>(tps::gemm_slot_elems(p.swap, p.bn, p.dual)) * 4; }

void fill_tiles(const Problem& pr, Plan& p) {
  const int WR = p.swap ? (p.dual ? 256 : 128) : p.bn * (p.pair && p.nh > 1 ? p.nh : 1);
  const int XR = p.pair ? 256 : p.swap ? p.bn : 128;
  p.WT = (pr.w_rows + WR - 1) / WR;
  p.MT = (pr.M + XR - 1) / XR;
  p.KBs = static_cast<int>((pr.k_inner + 63) / 64);
  if (pr.row && !pr.partials) {
    p.S_tiles = 1;
    p.KI = pr.tp * p.KBs;
  } else {
    p.S_tiles = pr.tp;
    p.KI = p.KBs;
  }
  p.wcols = p.S_tiles * p.WT;
  p.kv_rep = 1;
  p.qt = 0;
  // QKV with KV heads replicated over kv_rep shards: the replicas' KV rows equal the
  // first shard's of the group, so their tiles are computed once (by that shard)
  // and stored to every replica's columns -- when the KV rows start on a tile
  // boundary.
  if (pr.kind == tps::K_QKV && pr.kv_rep > 1 && pr.q_rows % WR == 0 && pr.tp % pr.kv_rep == 0) {
    p.kv_rep = pr.kv_rep;
    p.qt = pr.q_rows / WR;
    p.wcols = (pr.tp / pr.kv_rep) * (pr.kv_rep * p.qt + (p.WT - p.qt));
  }
  p.tiles = p.wcols * p.MT;
}

// Modelled SM cycles of one 64-wide K block, from B200 measurements of this
// kernel: token-major tiles are bound by feeding shared memory (every 128-byte
// tile row costs ~2.2 SM cycles of L2-to-SM transfer), measured at ~575 / ~610 /
// ~840 cycles for 64 / 128 / 256 weight rows; weight-major (decode) tiles stream
// weights from HBM at the per-SM share of its bandwidth (~24 B/cycle).
double kblock_cycles(const Plan& p) {
  if (p.pair && p.nh > 1) return 1020.0;   // 0.85 x two 256-wide pair K blocks (70B down: 1585 vs 2 x 935 cycles)
  if (p.pair) return p.bn <= 128 ? 460.0 : 600.0;
  if (!p.swap) return p.bn <= 64 ? 575.0 : p.bn <= 128 ? 610.0 : 840.0;
  const double rows = (p.dual ? 256.0 : 128.0) + p.bn;
  return std::max(rows * 2.3, (p.dual ? 256.0 : 128.0) * 128.0 / 24.0);
}

// Modelled epilogue cycles of one tile (16-column chunks, ~700 cycles each per
// epilogue warp); exposed once per CTA (the last tile's epilogue overlaps no
// main loop).
double epilogue_cycles(const Plan& p, const Problem& pr) {
  const int ncols = (!p.swap && pr.kind == tps::K_GATE_UP) ? p.bn / 2 : p.bn;
  return (ncols / 16) * 700.0;
}

// Modelled cost of the stream-K fix-up of a split tile: every segment writes its
// fp32 partial (chunks x 300 cycles), the last CTA loads the segments (rounds of
// four, ~1800 cycles of L2 latency per chunk and round) and finishes the tile.
double fixup_cycles(const Plan& p, const Problem& pr, int tiles_sk, int C) {
  if (tiles_sk <= 0) return 0.0;
  const double segs = 1.0 + static_cast<double>(C) / tiles_sk;
  const int acc_chunks = (p.bn * (p.dual ? 2 : 1)) / 16;
  const int out_chunks = ((!p.swap && pr.kind == tps::K_GATE_UP) ? p.bn / 2 : p.bn) / 16;
  const int parts = (pr.kind == tps::K_GATE_UP) ? 2 : 1;
  return acc_chunks * 300.0 + out_chunks * parts * std::ceil(segs / 4.0) * 1800.0 + epilogue_cycles(p, pr);
}

// Completes a plan whose orientation and tile width are set: data-parallel, or
// data-parallel for all full waves but the last plus stream-K for the remainder.
void finish_plan(const Problem& pr, Plan& p, int sms, size_t ws_bytes, int ov) {
  fill_tiles(pr, p);
  p.gm = raster_gm(p.MT);
  const int C = sms;
  const long long waves = (p.tiles + C - 1) / C;
  const double kb = kblock_cycles(p);
  p.sk = 0;
  p.dp_tiles = p.tiles;
  p.T = 0;
  p.grid = std::max(1, std::min(p.tiles, C));
  p.est = static_cast<double>(waves) * p.KI * kb + epilogue_cycles(p, pr);
  const bool fits =
      pr.static_ws
          ? (static_cast<size_t>(p.tiles) * 4 <= tps::kStaticCounterBytes &&
             2 * static_cast<size_t>(std::min<long long>(C, static_cast<long long>(p.tiles) * p.KI)) * slot_bytes(p) <=
                 ws_bytes - tps::kStaticCounterBytes)
          : (ws_bytes >= kHdr + slot_region_bytes(sms) + static_cast<size_t>(p.tiles) * 4 &&
             slot_bytes(p) <= kSlotStride);
  const bool allow = !pr.partials && !pr.argmax && p.KI >= 2 && !(ov & 32) && fits;
  if (!allow) return;
  if (ov & 16) {  // forced: pure stream-K over every tile
    const long long T = static_cast<long long>(p.tiles) * p.KI;
    const int g = static_cast<int>(std::min<long long>(C, T));
    if (g >= 2) {
      p.sk = 1;
      p.dp_tiles = 0;
      p.T = T;
      p.grid = g;
    }
    return;
  }
  const int dp_tiles = static_cast<int>((waves - 1) * C);
  const int rem = p.tiles - dp_tiles;
  const long long T = static_cast<long long>(rem) * p.KI;
  const int g = dp_tiles > 0 ? C : static_cast<int>(std::min<long long>(C, T));
  if (g < 2 || T < g) return;
  const double sk_est = static_cast<double>(waves - 1) * p.KI * kb + std::ceil(static_cast<double>(T) / g) * kb +
                        fixup_cycles(p, pr, rem, g);
  if (sk_est < 0.95 * p.est) {
    p.sk = 1;
    p.dp_tiles = dp_tiles;
    p.T = T;
    p.grid = g;
    p.est = sk_est;
  }
}

// Pair plans are considered for token-major tiles with more than 128 tokens;
// plan-override bit 64 forces them (when the device can host a pair), bit 128
// forbids them.
constexpr int kOvForceWide = 1 << 20;
constexpr int kOvNoWide = 1 << 21;
void finish_pair_plan(const Problem& pr, Plan& p, int max_pairs);
void consider_pairs(const Problem& pr, int ov, int forced_bn, Plan& best) {
  if ((ov & 128) || pr.M <= 128 || pr.partials || pr.argmax) return;
  const int maxp = tps::max_pair_clusters();
  if (maxp < 1) return;
  const bool gated = (pr.kind == tps::K_GATE_UP);
  for (int bn : {256, 128}) {
    if (gated && bn != 256) continue;
    if (forced_bn >= 64 && forced_bn != bn) continue;
    Plan q{};
    q.pair = 1;
    q.nh = 1;
    q.bn = bn;
    finish_pair_plan(pr, q, maxp);
    if ((ov & 64) ? (!best.pair || q.est < best.est) : (q.est < best.est * 0.98)) best = q;
  }
  // wide pair tiles: 256 tokens x 512 weight rows (two MMA halves), when the
  // shard's weight rows are a whole number of them (plan-override bit 20 prefers
  // them, bit 21 forbids them)
  if ((ov & kOvNoWide) || (forced_bn >= 64 && forced_bn != 256) || pr.w_rows % 512 != 0) return;
  Plan w{};
  w.pair = 1;
  w.nh = 2;
  w.bn = 256;
  finish_pair_plan(pr, w, maxp);
  if ((ov & kOvForceWide) ? true : (w.est < best.est * 0.98)) best = w;
}

// Cluster split-K plans for row-parallel GEMMs with few tiles and long K: the cs
// CTAs of a cluster each take a K share of one tile and reduce over distributed
// shared memory. Plan-override bit 16 forces them (when they fit), bit 17
// forbids them; bits 12-13 restrict the cluster size (1 = 2, 2 = 4, 3 = 8 CTAs).
constexpr int kOvForceCsplit = 1 << 16;
constexpr int kOvNoCsplit = 1 << 17;
void consider_csplit(const Problem& pr, int ov, int forced_bn, int sms, Plan& best) {
  if ((ov & kOvNoCsplit) || !pr.row || pr.partials || pr.bf16) return;
  // a CTA-pair plan that fills every pair stays; one that leaves pairs idle (few
  // token tiles, long K) competes with splitting each tile's K over a cluster
  if (best.pair && !(ov & kOvForceCsplit) && best.tiles >= tps::max_pair_clusters()) return;
  static const int kClusterCode[4] = {0, 2, 4, 8};
  const int forced_cs = kClusterCode[(ov >> 12) & 3];
  const bool swap = best.swap != 0;
  const int widths_tok[2] = {128, 64};
  for (int wi = 0; wi < (swap ? 1 : 2); ++wi) {
    const int bn = swap ? best.bn : widths_tok[wi];
    if (forced_bn >= 16 && forced_bn != bn) continue;
    for (int cs : {2, 4, 8}) {
      if (forced_cs != 0 && cs != forced_cs) continue;
      Plan q{};
      q.swap = swap ? 1 : 0;
      q.bn = bn;
      q.cs = cs;
      fill_tiles(pr, q);
      if (q.KI < 2 * cs) continue;
      const int maxc = tps::max_csplit_clusters(q.swap, bn, cs);
      if (maxc < 1) continue;
      q.gm = raster_gm(q.MT);
      q.sk = 0;
      q.dp_tiles = q.tiles;
      q.T = 0;
      q.grid = cs * std::min(q.tiles, maxc);
      const long long waves = (q.tiles + maxc - 1) / maxc;
      const double per_tile = std::ceil(static_cast<double>(q.KI) / cs) * kblock_cycles(q) + 2500.0 +
                              epilogue_cycles(q, pr) / cs;
      q.est = static_cast<double>(waves) * per_tile;
      (void)sms;
      if ((ov & kOvForceCsplit) ? (best.cs <= 1 || q.est < best.est) : (q.est < best.est * 0.95)) best = q;
    }
  }
}

// Completes a CTA-pair plan (data-parallel over pairs only).
void finish_pair_plan(const Problem& pr, Plan& p, int max_pairs) {
  fill_tiles(pr, p);
  p.gm = raster_gm(p.MT);
  const long long waves = (p.tiles + max_pairs - 1) / max_pairs;
  p.sk = 0;
  p.dp_tiles = p.tiles;
  p.T = 0;
  p.grid = 2 * std::max(1, std::min(p.tiles, max_pairs));
  // one accumulator buffer in a wide tile: every tile's epilogue (two halves on
  // eight epilogue warps, about one single-CTA tile's worth) is exposed
  const double epi = epilogue_cycles(p, pr) * (p.nh > 1 ? static_cast<double>(waves) : 1.0);
  p.est = static_cast<double>(waves) * p.KI * kblock_cycles(p) + epi;
}

// The bf16 exchange over tp = 2, 4 or 8 shards: a cluster of tp CTAs per tile,
// CTA r taking exactly shard r's K range, so every slot of the cluster reduce is
// one shard's whole fp32 partial; the owner rounds each to bf16 and sums them in
// shard order with a rounding after every addition. Orientation and width as the
// other plans of this size (weight-major up to 128 tokens). False when the
// cluster cannot be resident.
bool plan_bf16_exchange(const Problem& pr, int ov, Plan* out) {
  static const int kWidthCode[6] = {0, 16, 32, 64, 128, 256};
  const int wcode = (ov >> 8) & 15;
  const int forced_bn = (wcode >= 1 && wcode <= 5) ? kWidthCode[wcode] : 0;
  int orient = ov & 3;
  if (orient == 0) orient = (pr.M <= 128) ? 2 : 1;
  Plan q{};
  q.swap = orient == 2 ? 1 : 0;
  if (q.swap)
    q.bn = (forced_bn >= 16 && forced_bn <= 128) ? forced_bn : pr.M <= 16 ? 16 : pr.M <= 32 ? 32 : pr.M <= 64 ? 64 : 128;
  else
    q.bn = (forced_bn == 64) ? 64 : 128;
  q.cs = pr.tp;
  fill_tiles(pr, q);
  const int maxc = tps::max_csplit_clusters(q.swap, q.bn, q.cs);
  if (maxc < 1) return false;
  q.gm = raster_gm(q.MT);
  q.dp_tiles = q.tiles;
  q.grid = q.cs * std::min(q.tiles, maxc);
  *out = q;
  return true;
}

// The bf16 exchange as a shard chain: single-CTA data-parallel tiles (at most 128
// columns), each tile's K range walked shard by shard with a fresh accumulator per
// shard while the epilogue folds the previous shard into the running bf16 sum.
void plan_bf16_chain(const Problem& pr, int ov, int sms, Plan* out) {
  static const int kWidthCode[6] = {0, 16, 32, 64, 128, 256};
  const int wcode = (ov >> 8) & 15;
  const int forced_bn = (wcode >= 1 && wcode <= 5) ? kWidthCode[wcode] : 0;
  int orient = ov & 3;
  if (orient == 0) orient = (pr.M <= 128) ? 2 : 1;
  Plan q{};
  q.swap = orient == 2 ? 1 : 0;
  if (q.swap)
    q.bn = (forced_bn >= 16 && forced_bn <= 128) ? forced_bn : pr.M <= 16 ? 16 : pr.M <= 32 ? 32 : pr.M <= 64 ? 64 : 128;
  else
    q.bn = (forced_bn == 64) ? 64 : 128;
  q.cs = 1;
  q.chain = 1;
  fill_tiles(pr, q);
  q.gm = raster_gm(q.MT);
  q.dp_tiles = q.tiles;
  q.grid = std::max(1, std::min(q.tiles, sms));
  *out = q;
}

int plan_gemm(const Problem& pr, size_t ws_bytes, int sms, Plan* out) {
  const int ov = g_plan_override.load();
  if (pr.bf16 && pr.tp > 1) {
    // A cluster of tp CTAs per tile (tp = 2, 4, 8; plan-override bit 14 forces it) or
    // the shard chain (any tp; bit 30 forces it). Weight-major tiles (decode sizes)
    // take the cluster; token-major tiles the cheaper by a model of B200 runs: the
    // chain walks all tp*KBs K blocks of a tile on one SM and folds each shard
    // (~1500 cycles), the cluster walks KBs per CTA for tp times the tiles and pays
    // ~12000 cycles of exchange per tile (measured: m = 1024, n = 1024, tp = 8 chain
    // 38.9 us against 59.4; m = 512 both ~39 us; m = 2048, n = 4096 the chain).
    Plan chain{};
    plan_bf16_chain(pr, ov, sms, &chain);
    const bool cluster_ok = (pr.tp == 2 || pr.tp == 4 || pr.tp == 8);
    bool use_cluster = cluster_ok && !(ov & (1 << 30));
    if (use_cluster && !chain.swap && !(ov & (1 << 14))) {
      const double kb = 610.0;   // SM cycles per 64-wide K block of a 128 x 128 tile
      const double t_chain = std::ceil(static_cast<double>(chain.tiles) / sms) * pr.tp * (chain.KBs * kb + 1500.0);
      const double t_cluster =
          std::ceil(static_cast<double>(chain.tiles) * pr.tp / sms) * (chain.KBs * kb + 12000.0);
      use_cluster = t_cluster < t_chain;
    }
    if (use_cluster && !plan_bf16_exchange(pr, ov, out)) return TPS_ERR_UNIMPLEMENTED;
    if (!use_cluster) *out = chain;
    if (std::getenv("TPS_DEBUG_PLAN") != nullptr)
      std::fprintf(stderr, "tps plan: bf16 exchange M=%d tp=%d rows=%d | chain=%d swap=%d bn=%d tiles=%d cs=%d grid=%d\n",
                   pr.M, pr.tp, pr.w_rows, out->chain, out->swap, out->bn, out->tiles, out->cs, out->grid);
    return TPS_OK;
  }
  const bool gated = (pr.kind == tps::K_GATE_UP);
  int orient = ov & 3;
  if (orient == 0) orient = (pr.M <= 128) ? 2 : 1;
  static const int kWidthCode[6] = {0, 16, 32, 64, 128, 256};
  const int wcode = (ov >> 8) & 15;
  const int forced_bn = (wcode >= 1 && wcode <= 5) ? kWidthCode[wcode] : 0;
  Plan best{};
  if (orient == 2) {
    best.swap = 1;
    best.bn = pr.M <= 16 ? 16 : pr.M <= 32 ? 32 : pr.M <= 64 ? 64 : 128;
    if (forced_bn >= 16 && forced_bn <= 128) best.bn = forced_bn;
    best.dual = gated ? 1 : 0;
    finish_plan(pr, best, sms, ws_bytes, ov);
  } else if (gated) {
    best.swap = 0;
    best.bn = 256;  // [128 gate rows | 128 up rows] of one packed block
    best.dual = 0;
    finish_plan(pr, best, sms, ws_bytes, ov);
    consider_pairs(pr, ov, forced_bn, best);
  } else {
    bool have = false;
    for (int bn : {256, 128, 64}) {
      if (forced_bn >= 64 && bn != forced_bn) continue;
      Plan q{};
      q.swap = 0;
      q.bn = bn;
      q.dual = 0;
      finish_plan(pr, q, sms, ws_bytes, ov);
      if (!have || q.est < best.est * 0.98) {
        best = q;
        have = true;
      }
    }
    consider_pairs(pr, ov, forced_bn, best);
  }
  consider_csplit(pr, ov, forced_bn, sms, best);
  if (std::getenv("TPS_DEBUG_PLAN") != nullptr)
    std::fprintf(stderr,
                 "tps plan: kind=%d M=%d tp=%d k_inner=%lld rows=%d | pair=%d nh=%d swap=%d bn=%d dual=%d tiles=%d KI=%d "
                 "sk=%d dp_tiles=%d grid=%d cs=%d est=%.0f maxpairs=%d static_ws=%d\n",
                 pr.kind, pr.M, pr.tp, static_cast<long long>(pr.k_inner), pr.w_rows, best.pair, best.nh, best.swap, best.bn,
                 best.dual, best.tiles, best.KI, best.sk, best.dp_tiles, best.grid, best.cs, best.est,
                 tps::max_pair_clusters(), pr.static_ws);
  *out = best;
  return TPS_OK;
}

// Builds the tensor maps and kernel arguments of one GEMM and launches it.
struct GemmCall {
  Problem pr;
  const void* X;
  int64_t ldx;          // X row length (elements)
  const void* Wpk;
  int64_t w_rows_total; // rows per shard in the packed buffer (R)
  void* Y;
  int ldy;
  int y_f32;
  float* partials;
  const void* bias;
  int gate_off;
  HeadMap hm;
  int head_dim, hq, hkv;
  void* ws;
  size_t ws_bytes;
};

// Fused GELU MLP (one launch: fc1 tiles, then cluster split-K fc2 tiles that
// start per shard as fc1 finishes it). Plan-override bit 18 forces it (an error
// when it cannot run), bit 19 forbids it.
constexpr int kOvFusedMlp = 1 << 18;
constexpr int kOvNoFusedMlp = 1 << 19;

// GELU (prefill-sized m): fc1 as 128 x 128 token-major whole tiles, fc2 as 128 x
// 128 cluster split-K tiles. SiLU(gate)*up (m <= 64): gate/up as weight-major
// pairs of 128 gate + 128 up rows x 64 tokens, down as weight-major 128-row x
// 64-token cluster split-K tiles. Column tiles in token-block-major order, one
// resident cluster per row tile. False when the shape or the workspace (flags
// after the stream-K slots) does not fit.
bool plan_mlp_fused(const Problem& pr1, const Problem& pr2, size_t ws_bytes, int sms, int ov, Plan* p1, Plan* p2) {
  if (ov & kOvNoFusedMlp) return false;
  if (pr1.static_ws) return false;
  const bool gelu = (pr1.act == TPS_ACT_GELU && pr1.kind == tps::K_COLUMN);
  const bool gated = (pr1.act == TPS_ACT_SILU_MUL && pr1.kind == tps::K_GATE_UP);
  if (!gelu && !gated) return false;
  if (gelu && pr1.M <= 64 && !(ov & kOvFusedMlp)) return false;   // decode-shaped GELU: the two-kernel path
  if (gated && pr1.M > 64) return false;                          // prefill-shaped gate/up: the two-kernel path
  const int swap = gated ? 1 : 0;
  const int bn = gated ? 64 : 128;
  Plan q1{};
  q1.swap = swap;
  q1.bn = bn;
  q1.dual = gated ? 1 : 0;
  fill_tiles(pr1, q1);
  q1.gm = 1;
  q1.dp_tiles = q1.tiles;
  const size_t flags = (static_cast<size_t>(q1.MT) * pr1.tp + 1) * 4;
  if (ws_bytes < kHdr + slot_region_bytes(sms) + flags) return false;
  Plan best{};
  bool have = false;
  for (int cs : {4, 2, 8}) {
    Plan q{};
    q.swap = swap;
    q.bn = bn;
    q.cs = cs;
    fill_tiles(pr2, q);
    if (q.KI < 2 * cs) continue;
    if (tps::max_csplit_clusters(swap, bn, cs) < q.tiles) continue;   // every cluster resident at once
    q.gm = 1;
    q.dp_tiles = q.tiles;
    q.grid = cs * q.tiles;
    const long long waves1 = (q1.tiles + q.grid - 1) / q.grid;
    q.est = static_cast<double>(waves1) * (q1.KI * kblock_cycles(q1) + epilogue_cycles(q1, pr1)) +
            std::ceil(static_cast<double>(q.KI) / cs) * kblock_cycles(q) + 2500.0 + epilogue_cycles(q, pr2) / cs;
    if (!have || q.est < best.est) {
      best = q;
      have = true;
    }
  }
  if (!have) return false;
  *p1 = q1;
  p1->grid = best.grid;
  *p2 = best;
  return true;
}

// The gated MLP at decode sizes as one launch with stream-K over both layers
// (tps_mlp_sk_kernel): every CTA, one per SM, takes an equal share of the gate/up
// (tile, K block) iterations and then of the down iterations, so the weight stream
// covers all SMs in both layers. Plan-override bit 22 selects it (bit 18 then
// requires it), bit 23 forbids it; by default the cluster form runs. Workspace after the header: the gate/up segment
// slots (two per CTA), the down segment slots, then the tile counters of both
// layers and the readiness flags. False when it does not apply or does not fit.
constexpr int kOvSkMlp = 1 << 22;
constexpr int kOvNoSkMlp = 1 << 23;
struct SkMlpLayout {
  size_t slots2, cnt1, cnt2, ready;   // byte offsets from the workspace start
};
bool plan_mlp_sk(const Problem& pr1, const Problem& pr2, size_t ws_bytes, int sms, int ov, Plan* p1, Plan* p2,
                 SkMlpLayout* lay) {
  if (ov & kOvNoSkMlp) return false;
  if (pr1.static_ws || pr1.act != TPS_ACT_SILU_MUL || pr1.kind != tps::K_GATE_UP || pr1.M > 64) return false;
  const int resident = tps::mlp_sk_resident_ctas();
  if (resident < 1) return false;
  Plan q1{}, q2{};
  q1.swap = 1;
  q1.bn = 64;
  q1.dual = 1;
  fill_tiles(pr1, q1);
  q2.swap = 1;
  q2.bn = 64;
  fill_tiles(pr2, q2);
  const long long T1 = static_cast<long long>(q1.tiles) * q1.KI;
  const long long T2 = static_cast<long long>(q2.tiles) * q2.KI;
  // by default only when both layers have at least one K block per SM (the decode
  // shapes the form is for); forced, on any shape, with a grid no larger than either
  // layer's iterations
  if (!(ov & kOvSkMlp) && (T1 < sms || T2 < sms)) return false;
  const int grid = static_cast<int>(std::min<long long>(std::min(sms, resident), std::min(T1, T2)));
  for (Plan* q : {&q1, &q2}) {
    q->gm = 1;
    q->sk = 1;
    q->dp_tiles = 0;
    q->T = static_cast<long long>(q->tiles) * q->KI;
    q->grid = grid;
  }
  SkMlpLayout L{};
  L.slots2 = kHdr + 2 * static_cast<size_t>(grid) * tps::mlp_sk_slot_bytes(0);
  const size_t slots_end = L.slots2 + 2 * static_cast<size_t>(grid) * tps::mlp_sk_slot_bytes(1);
  L.cnt1 = std::max(slots_end, kHdr + slot_region_bytes(sms));
  L.cnt2 = L.cnt1 + static_cast<size_t>(q1.tiles) * 4;
  L.ready = L.cnt2 + static_cast<size_t>(q2.tiles) * 4;
  const size_t need = L.ready + (static_cast<size_t>(q1.MT) * pr1.tp + 1) * 4;
  if (ws_bytes < need) return false;
  *p1 = q1;
  *p2 = q2;
  *lay = L;
  return true;
}

// Tensor maps and kernel arguments of one planned GEMM (may enqueue the counter
// clear of the static scratch on `st`).
int build_gemm(const GemmCall& c, const Plan& p, int sms, cudaStream_t st, CUtensorMap* txp, CUtensorMap* twp,
               GemmArgs* ap) {
  int rc = 0;
  CUtensorMap& tx = *txp;
  CUtensorMap& tw = *twp;
  const int XR = p.swap ? p.bn : 128;                     // token rows per CTA tile
  const int WR = p.pair ? p.bn / 2 : p.swap ? (p.dual ? 256 : 128) : p.bn;  // weight rows per CTA tile
  const uint64_t M = static_cast<uint64_t>(c.pr.M);
  // Row problems whose shard K range is a whole number of 64-wide K blocks read X
  // through the plain 2-D map (shard ks's block kk is column ks*k_s + 64*kk);
  // otherwise X is viewed as [M][tp][k_s], so that every shard's K tail reads zeros.
  const bool x3d = c.pr.row && (c.pr.k_inner % 64 != 0);
  if (x3d) {
    // X viewed as [M][tp][k_s]: dims {k_s, tp, M}
    const uint64_t ks = static_cast<uint64_t>(c.pr.k_inner);
    rc = make_map(&tx, c.X, ks, static_cast<uint64_t>(c.pr.tp), M, ks * 2, static_cast<uint64_t>(c.ldx) * 2, 1, XR);
  } else if (c.pr.row) {
    const uint64_t k = static_cast<uint64_t>(c.pr.k_inner) * static_cast<uint64_t>(c.pr.tp);
    rc = make_map(&tx, c.X, k, M, 1, static_cast<uint64_t>(c.ldx) * 2, static_cast<uint64_t>(c.ldx) * 2 * M, XR, 1);
  } else {
    const uint64_t k = static_cast<uint64_t>(c.pr.k_inner);
    rc = make_map(&tx, c.X, k, M, 1, static_cast<uint64_t>(c.ldx) * 2, static_cast<uint64_t>(c.ldx) * 2 * M, XR, 1);
  }
  if (rc) return rc;
  const int RB = static_cast<int>((c.w_rows_total + 127) / 128);
  const int KB = static_cast<int>((c.pr.k_inner + 63) / 64);
  rc = make_wmap(&tw, c.Wpk, RB, KB, c.pr.tp, static_cast<uint32_t>(WR < 128 ? WR : 128));
  if (rc) return rc;

  GemmArgs& a = *ap;
  a = GemmArgs{};
  a.M = c.pr.M;
  a.tp = c.pr.tp;
  a.KBs = p.KBs;
  a.KI = p.KI;
  a.k_spans_shards = (c.pr.row && !c.pr.partials) ? 1 : 0;
  a.x_sharded = x3d ? 1 : 0;
  a.x_shard_cols = (c.pr.row && !x3d) ? static_cast<int>(c.pr.k_inner) : 0;
  a.S_tiles = p.S_tiles;
  a.WT = p.WT;
  a.wcols = p.wcols;
  a.kv_rep = p.kv_rep;
  a.qt = p.qt;
  a.MT = p.MT;
  a.tiles = p.tiles;
  a.gm = p.gm;
  a.RB = RB;
  a.sk = p.sk;
  a.dp_tiles = p.dp_tiles;
  a.cs = p.cs > 1 ? p.cs : 1;
  a.total_iters = p.T;
  if (p.sk && c.pr.static_ws) {
    // static scratch: counters in its last kStaticCounterBytes, cleared on every call
    a.ws_part = static_cast<float*>(c.ws);
    a.ws_cnt = reinterpret_cast<int*>(static_cast<char*>(c.ws) + c.ws_bytes - tps::kStaticCounterBytes);
    if (cudaMemsetAsync(a.ws_cnt, 0, static_cast<size_t>(p.tiles) * 4, st) != cudaSuccess) return TPS_ERR_CUDA;
  } else if (p.sk) {
    a.ws_part = reinterpret_cast<float*>(static_cast<char*>(c.ws) + kHdr);
    a.ws_cnt = reinterpret_cast<int*>(static_cast<char*>(c.ws) + kHdr + slot_region_bytes(sms));
  }
  // the static scratch has no status header: its calls report through the device-wide word only
  a.status = c.pr.static_ws ? nullptr : ws_status(c.ws, c.ws_bytes);
  a.out_mode = c.pr.partials ? tps::OUT_PARTIALS : tps::OUT_FINAL;
  a.kind = c.pr.kind;
  a.act = c.pr.act;
  a.per_shard = c.pr.per_shard;
  a.ldy = c.ldy;
  a.y_f32 = c.y_f32;
  a.Y = c.Y;
  a.partials = c.partials;
  a.bias = c.bias;
  a.gate_off = c.gate_off;
  a.q_cols = c.hm.qs * c.head_dim;
  a.kv_cols = c.hm.kvs * c.head_dim;
  a.hq_d = c.hq * c.head_dim;
  a.hkv_d = c.hkv * c.head_dim;
  a.kv_first_num = c.hm.kv_num;
  a.kv_first_den = c.hm.kv_den > 0 ? c.hm.kv_den : 1;
  a.head_dim = c.head_dim;
  a.timeout_ns = kTimeoutNs;
  a.bf16_chain = c.pr.bf16 ? 1 : 0;
  a.chain = p.chain;
  // CTA-pair tiles: the token rows of a raster group (gm token tiles of 256 rows, every
  // K block) are read by every weight tile of the group's sweep; when they take at most
  // half of L2 they are loaded with the evict-last policy. Plan-override bit 28 drops
  // that policy, bit 29 loads the weights with evict-first.
  if (p.pair) {
    const int ov = g_plan_override.load();
    const double kx = c.pr.row ? static_cast<double>(c.pr.k_inner) * c.pr.tp : static_cast<double>(c.pr.k_inner);
    const double group_x = static_cast<double>(std::min(p.gm, p.MT)) * 256.0 * kx * 2.0;
    if (!(ov & (1 << 28)) && group_x <= 64.0 * 1024 * 1024) a.l2_hint |= 1;
    if (ov & (1 << 29)) a.l2_hint |= 2;
  }
  return TPS_OK;
}

// ------------------------------------------------------------------ launch cache
// A serving loop calls the block with the same buffers and sizes every step. The
// plan, tensor maps and kernel arguments of a call are kept, keyed by every
// argument that shapes them, the plan override and the device, so a repeated
// call only launches. Small, round-robin replaced, one mutex.
struct LaunchKey {
  uint64_t v[40];
  int n;
  void add(uint64_t x) { v[n++] = x; }
  void addp(const void* p) { add(reinterpret_cast<uintptr_t>(p)); }
  bool operator==(const LaunchKey& o) const { return n == o.n && std::memcmp(v, o.v, sizeof(uint64_t) * n) == 0; }
};

template <class V>
struct LaunchCache {
  static constexpr int kSlots = 16;
  std::mutex mu;
  LaunchKey keys[kSlots];
  V vals[kSlots];
  bool used[kSlots] = {};
  int next = 0;
  bool get(const LaunchKey& k, V* out) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < kSlots; ++i)
      if (used[i] && keys[i] == k) {
        *out = vals[i];
        return true;
      }
    return false;
  }
  void put(const LaunchKey& k, const V& v) {
    std::lock_guard<std::mutex> lock(mu);
    keys[next] = k;
    vals[next] = v;
    used[next] = true;
    next = (next + 1) % kSlots;
  }
};

LaunchKey gemm_key(const GemmCall& c, int ov) {
  LaunchKey k{};
  int dev = -1;
  (void)cudaGetDevice(&dev);
  k.add(static_cast<uint64_t>(dev));
  k.add(static_cast<uint64_t>(static_cast<uint32_t>(ov)));
  k.add(static_cast<uint64_t>(c.pr.kind));
  k.add(static_cast<uint64_t>(c.pr.M));
  k.add(static_cast<uint64_t>(c.pr.tp));
  k.add(static_cast<uint64_t>(c.pr.k_inner));
  k.add(static_cast<uint64_t>(c.pr.w_rows));
  k.add(static_cast<uint64_t>(c.pr.per_shard));
  k.add(static_cast<uint64_t>((c.pr.row ? 1 : 0) | (c.pr.partials ? 2 : 0) | (c.pr.bf16 ? 4 : 0)));
  k.add(static_cast<uint64_t>(c.pr.act));
  k.addp(c.X);
  k.add(static_cast<uint64_t>(c.ldx));
  k.addp(c.Wpk);
  k.add(static_cast<uint64_t>(c.w_rows_total));
  k.addp(c.Y);
  k.add(static_cast<uint64_t>(c.ldy));
  k.add(static_cast<uint64_t>(c.y_f32));
  k.addp(c.partials);
  k.addp(c.bias);
  k.add(static_cast<uint64_t>(c.gate_off));
  k.add(static_cast<uint64_t>(c.hm.qs));
  k.add(static_cast<uint64_t>(c.hm.kvs));
  k.add(static_cast<uint64_t>(c.hm.kv_num));
  k.add(static_cast<uint64_t>(c.hm.kv_den));
  k.add(static_cast<uint64_t>(c.head_dim));
  k.add(static_cast<uint64_t>(c.hq));
  k.add(static_cast<uint64_t>(c.hkv));
  k.add(static_cast<uint64_t>(c.pr.kv_rep));
  k.addp(c.ws);
  k.add(static_cast<uint64_t>(c.ws_bytes));
  return k;
}

struct GemmLaunch {
  Plan p;
  CUtensorMap tx, tw;
  GemmArgs a;
};
LaunchCache<GemmLaunch> g_gemm_cache;

int launch_planned(const GemmLaunch& L, cudaStream_t st) {
  const Plan& p = L.p;
  const int rc = p.pair    ? tps::launch_gemm_pair(p.bn, p.nh, L.tx, L.tw, L.a, p.grid, st)
                 : p.cs > 1 ? tps::launch_gemm_csplit(p.swap, p.bn, p.cs, L.tx, L.tw, L.a, p.grid, st)
                            : tps::launch_gemm(p.swap, p.bn, p.dual, L.tx, L.tw, L.a, p.grid, st);
  return rc == 0 ? TPS_OK : (rc == -8 ? TPS_ERR_UNIMPLEMENTED : TPS_ERR_CUDA);
}

int run_gemm(const GemmCall& c, cudaStream_t st) {
  // the static scratch needs its counters cleared on every call: not cached
  const bool cacheable = !c.pr.static_ws;
  const int ov = g_plan_override.load();
  LaunchKey key{};
  GemmLaunch L{};
  if (cacheable) {
    key = gemm_key(c, ov);
    if (g_gemm_cache.get(key, &L)) return launch_planned(L, st);
  }
  const int sms = num_sms_current();
  Plan p{};
  int rc = plan_gemm(c.pr, c.ws_bytes, sms, &p);
  if (rc) return rc;
  CUtensorMap tx, tw;
  GemmArgs a{};
  rc = build_gemm(c, p, sms, st, &tx, &tw, &a);
  if (rc) return rc;
  if (cacheable) {
    L.p = p;
    L.tx = tx;
    L.tw = tw;
    L.a = a;
    g_gemm_cache.put(key, L);
  }
  rc = p.pair    ? tps::launch_gemm_pair(p.bn, p.nh, tx, tw, a, p.grid, st)
       : p.cs > 1 ? tps::launch_gemm_csplit(p.swap, p.bn, p.cs, tx, tw, a, p.grid, st)
                  : tps::launch_gemm(p.swap, p.bn, p.dual, tx, tw, a, p.grid, st);
  return rc == 0 ? TPS_OK : (rc == -8 ? TPS_ERR_UNIMPLEMENTED : TPS_ERR_CUDA);
}

size_t ws_bound(int64_t m, int64_t n, int64_t k, int tp, int sms) {
  // counters for the largest tile count any plan of these sizes can have
  const int64_t wide = std::max<int64_t>(n, k);
  const int64_t tiles = ((m + 15) / 16) * ((2 * wide + 63) / 64 + tp);
  return kHdr + slot_region_bytes(sms) + round256(static_cast<size_t>(tiles) * 4);
}

bool valid_dtype(int d) { return d == TPS_DTYPE_BF16 || d == TPS_DTYPE_F32; }

// The fused GELU MLP when it applies: TPS_OK or an error status, or
// kFusedNotApplicable (nothing enqueued) when the two-GEMM path must run.
constexpr int kFusedNotApplicable = 1;

struct MlpLaunch {
  int status;   // TPS_OK: launch these; else the status to return
  int swap;     // kernel form (0 token-major GELU, 1 weight-major gate/up)
  int sk;       // 1: the stream-K form (tps_mlp_sk_kernel)
  CUtensorMap tx, tw1, th, tw2;
  GemmArgs a1, a2;
  tps::MlpSync sy;
  int grid;
};
LaunchCache<MlpLaunch> g_mlp_cache;

int run_mlp_fused(const void* X, int64_t m, int64_t H, int64_t I, int tp, int act, const PackGeom& g1,
                  const void* pw1, const void* pw2, void* h, void* Y, int y_f32, void* ws, size_t ws_bytes,
                  cudaStream_t st) {
  const int ov = g_plan_override.load();
  LaunchKey key{};
  {
    int dev = -1;
    (void)cudaGetDevice(&dev);
    key.add(static_cast<uint64_t>(dev));
    key.add(static_cast<uint64_t>(static_cast<uint32_t>(ov)));
    key.addp(X);
    key.add(static_cast<uint64_t>(m));
    key.add(static_cast<uint64_t>(H));
    key.add(static_cast<uint64_t>(I));
    key.add(static_cast<uint64_t>(tp));
    key.add(static_cast<uint64_t>(act));
    key.addp(pw1);
    key.addp(pw2);
    key.addp(h);
    key.addp(Y);
    key.add(static_cast<uint64_t>(y_f32));
    key.addp(ws);
    key.add(static_cast<uint64_t>(ws ? ws_bytes : 0));
  }
  MlpLaunch L{};
  if (g_mlp_cache.get(key, &L)) {
    if (L.status != TPS_OK) return L.status;
    const int lrc = L.sk ? tps::launch_mlp_sk(L.tx, L.tw1, L.th, L.tw2, L.a1, L.a2, L.sy, L.grid, st)
                         : tps::launch_mlp_fused(L.swap, L.tx, L.tw1, L.th, L.tw2, L.a1, L.a2, L.sy, L.grid, st);
    return lrc == 0 ? TPS_OK : TPS_ERR_CUDA;
  }
  const int sms = num_sms_current();
  const bool gated = (act == TPS_ACT_SILU_MUL);
  GemmCall c1{};
  c1.pr.kind = gated ? tps::K_GATE_UP : tps::K_COLUMN;
  c1.pr.M = static_cast<int>(m);
  c1.pr.tp = tp;
  c1.pr.k_inner = H;
  c1.pr.w_rows = g1.R;
  c1.pr.per_shard = g1.per_shard;
  c1.pr.act = act;
  c1.X = X;
  c1.ldx = H;
  c1.Wpk = pw1;
  c1.w_rows_total = g1.R;
  c1.Y = h;
  c1.ldy = g1.out_cols;
  c1.gate_off = gated ? static_cast<int>(I) : 0;
  c1.hm.kv_den = 1;
  c1.ws = ws;   // the status header (the one-launch plan uses no stream-K slots)
  c1.ws_bytes = ws ? ws_bytes : 0;
  GemmCall c2{};
  c2.pr.kind = tps::K_ROW;
  c2.pr.M = static_cast<int>(m);
  c2.pr.tp = tp;
  c2.pr.k_inner = I / tp;
  c2.pr.w_rows = static_cast<int>(H);
  c2.pr.per_shard = static_cast<int>(H);
  c2.pr.row = true;
  c2.pr.act = TPS_ACT_NONE;
  c2.X = h;
  c2.ldx = I;
  c2.Wpk = pw2;
  c2.w_rows_total = H;
  c2.Y = Y;
  c2.ldy = static_cast<int>(H);
  c2.y_f32 = y_f32;
  c2.hm.kv_den = 1;
  c2.ws = ws;
  c2.ws_bytes = ws ? ws_bytes : 0;
  Plan p1{}, p2{};
  SkMlpLayout lay{};
  // the stream-K form when asked for (measured slower than the cluster form at the
  // decode shapes, see the kernel's notes); the cluster form otherwise
  if ((ov & kOvSkMlp) && plan_mlp_sk(c1.pr, c2.pr, ws ? ws_bytes : 0, sms, ov, &p1, &p2, &lay)) {
    CUtensorMap tx, tw1, th, tw2;
    GemmArgs a1{}, a2{};
    int rc = build_gemm(c1, p1, sms, st, &tx, &tw1, &a1);
    if (rc) return rc;
    rc = build_gemm(c2, p2, sms, st, &th, &tw2, &a2);
    if (rc) return rc;
    char* w = static_cast<char*>(ws);
    a1.ws_part = reinterpret_cast<float*>(w + kHdr);
    a2.ws_part = reinterpret_cast<float*>(w + lay.slots2);
    a1.ws_cnt = reinterpret_cast<int*>(w + lay.cnt1);
    a2.ws_cnt = reinterpret_cast<int*>(w + lay.cnt2);
    tps::MlpSync sy{};
    sy.ready = reinterpret_cast<int*>(w + lay.ready);
    sy.n_ready = p1.MT * tp;
    sy.done = sy.ready + sy.n_ready;
    sy.need = p1.WT;
    if (std::getenv("TPS_DEBUG_PLAN") != nullptr)
      std::fprintf(stderr, "tps plan: stream-K MLP act=%d M=%d tp=%d col tiles=%d KI=%d | row tiles=%d KI=%d grid=%d\n",
                   act, c1.pr.M, tp, p1.tiles, p1.KI, p2.tiles, p2.KI, p1.grid);
    L.status = TPS_OK;
    L.swap = 1;
    L.sk = 1;
    L.tx = tx;
    L.tw1 = tw1;
    L.th = th;
    L.tw2 = tw2;
    L.a1 = a1;
    L.a2 = a2;
    L.sy = sy;
    L.grid = p1.grid;
    g_mlp_cache.put(key, L);
    return tps::launch_mlp_sk(tx, tw1, th, tw2, a1, a2, sy, p1.grid, st) == 0 ? TPS_OK : TPS_ERR_CUDA;
  }
  if ((ov & kOvSkMlp) && (ov & kOvFusedMlp)) {   // the stream-K form was required
    L.status = TPS_ERR_UNIMPLEMENTED;
    g_mlp_cache.put(key, L);
    return L.status;
  }
  if (!plan_mlp_fused(c1.pr, c2.pr, ws ? ws_bytes : 0, sms, ov, &p1, &p2)) {
    L.status = (ov & kOvFusedMlp) ? TPS_ERR_UNIMPLEMENTED : kFusedNotApplicable;
    g_mlp_cache.put(key, L);
    return L.status;
  }
  CUtensorMap tx, tw1, th, tw2;
  GemmArgs a1{}, a2{};
  int rc = build_gemm(c1, p1, sms, st, &tx, &tw1, &a1);
  if (rc) return rc;
  rc = build_gemm(c2, p2, sms, st, &th, &tw2, &a2);
  if (rc) return rc;
  tps::MlpSync sy{};
  sy.ready = reinterpret_cast<int*>(static_cast<char*>(ws) + kHdr + slot_region_bytes(sms));
  sy.n_ready = p1.MT * tp;
  sy.done = sy.ready + sy.n_ready;
  sy.need = p1.WT;
  // The row layer's weights start streaming into L2 while the column layer finishes
  // (its last loads, epilogue and readiness flags leave HBM idle): every CTA prefetches
  // its whole row-layer range when the grid's ranges total at most 48 MB (about 40% of
  // L2). Measured: 1.5% faster for the GELU MLP at m = 512 (8 MB of fc2 weights); at
  // decode sizes (117 MB of down weights) a partial prefetch made the block 3% slower,
  // as the prefetch competes with the column layer's own weight stream.
  {
    const double box = 128.0 * 64.0 * 2.0;                  // one weight box (128 rows x 64 K, bf16)
    const int per_cta = (p2.KI + p2.cs - 1) / p2.cs;          // K blocks of a CTA's row-layer range
    const double total = box * per_cta * static_cast<double>(p2.grid);
    sy.prefetch2 = (total <= 48.0 * 1024 * 1024) ? per_cta : 0;
  }
  if (std::getenv("TPS_DEBUG_PLAN") != nullptr)
    std::fprintf(stderr, "tps plan: fused MLP act=%d M=%d tp=%d col tiles=%d KI=%d | row tiles=%d KI=%d cs=%d grid=%d\n",
                 act, c1.pr.M, tp, p1.tiles, p1.KI, p2.tiles, p2.KI, p2.cs, p2.grid);
  L.status = TPS_OK;
  L.swap = p1.swap;
  L.sk = 0;
  L.tx = tx;
  L.tw1 = tw1;
  L.th = th;
  L.tw2 = tw2;
  L.a1 = a1;
  L.a2 = a2;
  L.sy = sy;
  L.grid = p2.grid;
  g_mlp_cache.put(key, L);
  rc = tps::launch_mlp_fused(p1.swap, tx, tw1, th, tw2, a1, a2, sy, p2.grid, st);
  return rc == 0 ? TPS_OK : TPS_ERR_CUDA;
}

// The standalone reduction over the shards (fp32, or the bf16 exchange).
int reduce_common(const float* partials, int tp, int64_t m, int64_t n, const void* bias, void* Y, int y_dtype,
                  int bf16_chain, void* stream) {
  if (tp <= 0 || m < 0 || n <= 0) return TPS_ERR_ARG;
  if (!valid_dtype(y_dtype)) return TPS_ERR_DTYPE;
  if (n % 4) return TPS_ERR_ALIGN;
  if (m == 0) return TPS_OK;
  if (partials == nullptr || Y == nullptr) return TPS_ERR_ARG;
  if (!aligned16(partials) || !aligned16(Y) || (bias && !aligned16(bias))) return TPS_ERR_ALIGN;
  const int rc = check_device();
  if (rc) return rc;
  return tps::launch_reduce(partials, tp, m, n, bias, Y, y_dtype == TPS_DTYPE_F32, bf16_chain, num_sms_current(),
                            static_cast<cudaStream_t>(stream)) == 0
             ? TPS_OK
             : TPS_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* tps_status_string(int s) {
  switch (s) {
    case TPS_OK: return "TPS_OK";
    case TPS_ERR_ARG: return "TPS_ERR_ARG: invalid argument";
    case TPS_ERR_DIVISIBILITY: return "TPS_ERR_DIVISIBILITY: tp does not divide the split dimension";
    case TPS_ERR_ALIGN: return "TPS_ERR_ALIGN: pointer not 16-byte aligned or row length not a multiple of 8";
    case TPS_ERR_DTYPE: return "TPS_ERR_DTYPE: unsupported dtype";
    case TPS_ERR_WORKSPACE: return "TPS_ERR_WORKSPACE: buffer too small";
    case TPS_ERR_CUDA: return "TPS_ERR_CUDA: CUDA call failed";
    case TPS_ERR_TIMEOUT: return "TPS_ERR_TIMEOUT: bounded device wait expired";
    case TPS_ERR_UNIMPLEMENTED: return "TPS_ERR_UNIMPLEMENTED: not supported by this library";
    case TPS_ERR_DEVICE: return "TPS_ERR_DEVICE: not an sm_100 device";
    default: return "TPS_ERR_UNKNOWN";
  }
}

int tps_set_plan_override(int plan) { return g_plan_override.exchange(plan); }

int tp_head_map(int hq, int hkv, int tp, int32_t* q_first, int32_t* q_count, int32_t* kv_first,
                int32_t* kv_count) {
  HeadMap hm{};
  const int rc = head_map_calc(hq, hkv, tp, &hm);
  if (rc) return rc;
  for (int r = 0; r < tp; ++r) {
    if (q_first) q_first[r] = r * hm.qs;
    if (q_count) q_count[r] = hm.qs;
    if (kv_first) kv_first[r] = (r * hm.kv_num) / hm.kv_den;
    if (kv_count) kv_count[r] = hm.kvs;
  }
  return TPS_OK;
}

size_t tp_packed_bytes(int kind, int64_t k, int64_t n, int tp, const tps_heads* heads) {
  PackGeom g{};
  if (pack_geom(kind, k, n, tp, heads, &g) != TPS_OK) return 0;
  return g.bytes(tp);
}

int tp_shard_weights(int kind, const void* W, int transposed, int64_t k, int64_t n, int tp, const tps_heads* heads,
                     void* packed, size_t packed_bytes, void* stream) {
  if (W == nullptr || packed == nullptr || (transposed != 0 && transposed != 1)) return TPS_ERR_ARG;
  PackGeom g{};
  int rc = pack_geom(kind, k, n, tp, heads, &g);
  if (rc) return rc;
  if (!aligned16(W) || !aligned16(packed)) return TPS_ERR_ALIGN;
  if (packed_bytes < g.bytes(tp)) return TPS_ERR_WORKSPACE;
  rc = check_device();
  if (rc) return rc;
  tps::PackHost h{};
  h.W = W;
  h.out = packed;
  h.transposed = transposed;
  h.k = k;
  h.n = n;
  h.tp = tp;
  h.kind = kind;
  h.R = g.R;
  h.Kp = g.Kp;
  h.ns = (kind == TPS_KIND_COLUMN) ? static_cast<int>(n / tp) : 0;
  if (kind == TPS_KIND_QKV) {
    h.q_cols = g.hm.qs * heads->head_dim;
    h.kv_cols = g.hm.kvs * heads->head_dim;
    h.hq_d = heads->hq * heads->head_dim;
    h.hkv_d = heads->hkv * heads->head_dim;
    h.kv_first_num = g.hm.kv_num;
    h.kv_first_den = g.hm.kv_den;
    h.head_dim = heads->head_dim;
  } else {
    h.kv_first_den = 1;
  }
  if (kind == TPS_KIND_GATE_UP) {
    h.Is = g.per_shard;
    h.I = static_cast<int>(n / 2);
  }
  return tps::launch_pack(h, static_cast<cudaStream_t>(stream)) == 0 ? TPS_OK : TPS_ERR_CUDA;
}

int column_parallel_forward(const void* X, int64_t m, int64_t k, const void* packed_w, int kind, int64_t n, int tp,
                            const tps_heads* heads, const void* bias, int act, void* Y, int y_dtype, void* ws,
                            size_t ws_bytes, void* stream) {
  if (kind != TPS_KIND_COLUMN && kind != TPS_KIND_QKV && kind != TPS_KIND_GATE_UP) return TPS_ERR_ARG;
  if (m < 0 || m > (1LL << 30)) return TPS_ERR_ARG;
  if (!valid_dtype(y_dtype)) return TPS_ERR_DTYPE;
  if (kind == TPS_KIND_GATE_UP && act != TPS_ACT_SILU_MUL) return TPS_ERR_ARG;
  if (kind == TPS_KIND_QKV && act != TPS_ACT_NONE) return TPS_ERR_ARG;
  if (kind == TPS_KIND_COLUMN && act != TPS_ACT_NONE && act != TPS_ACT_GELU) return TPS_ERR_ARG;
  PackGeom g{};
  int rc = pack_geom(kind, k, n, tp, heads, &g);
  if (rc) return rc;
  if (m == 0) return TPS_OK;  // empty problem: no pointer is dereferenced
  if (X == nullptr || packed_w == nullptr || Y == nullptr) return TPS_ERR_ARG;
  if (!aligned16(X) || !aligned16(packed_w) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (ws && !aligned16(ws)))
    return TPS_ERR_ALIGN;
  rc = check_device();
  if (rc) return rc;
  GemmCall c{};
  c.pr.kind = kind;
  c.pr.M = static_cast<int>(m);
  c.pr.tp = tp;
  c.pr.k_inner = k;
  c.pr.w_rows = g.R;
  c.pr.per_shard = g.per_shard;
  c.pr.row = false;
  c.pr.partials = false;
  c.pr.act = act;
  c.X = X;
  c.ldx = k;
  c.Wpk = packed_w;
  c.w_rows_total = g.R;
  c.Y = Y;
  c.ldy = g.out_cols;
  c.y_f32 = (y_dtype == TPS_DTYPE_F32);
  c.bias = bias;
  c.gate_off = (kind == TPS_KIND_GATE_UP) ? static_cast<int>(n / 2) : 0;
  c.hm = g.hm;
  if (kind == TPS_KIND_QKV) {
    c.head_dim = heads->head_dim;
    c.hq = heads->hq;
    c.hkv = heads->hkv;
    c.pr.q_rows = g.hm.qs * heads->head_dim;
    c.pr.kv_rep = (g.hm.kv_den > 1) ? tp / heads->hkv : 1;
  } else {
    c.hm.kv_den = 1;
  }
  c.ws = ws;
  c.ws_bytes = ws ? ws_bytes : 0;
  return run_gemm(c, static_cast<cudaStream_t>(stream));
}

int row_parallel_forward(const void* X, int64_t m, int64_t k, const void* packed_v, int64_t n, int tp,
                         const void* bias, int reduce_mode, float* partials, void* Y, int y_dtype, void* ws,
                         size_t ws_bytes, void* stream) {
  if (m < 0 || m > (1LL << 30)) return TPS_ERR_ARG;
  if (!valid_dtype(y_dtype)) return TPS_ERR_DTYPE;
  if (reduce_mode != TPS_REDUCE_FUSED && reduce_mode != TPS_REDUCE_PARTIALS && reduce_mode != TPS_REDUCE_BF16)
    return TPS_ERR_ARG;
  PackGeom g{};
  int rc = pack_geom(TPS_KIND_ROW, k, n, tp, nullptr, &g);
  if (rc) return rc;
  if (m == 0) return TPS_OK;  // empty problem: no pointer is dereferenced
  if (X == nullptr || packed_v == nullptr || Y == nullptr) return TPS_ERR_ARG;
  if (reduce_mode == TPS_REDUCE_PARTIALS && partials == nullptr) return TPS_ERR_ARG;
  // the bf16 exchange runs inside the GEMM without a partials buffer (any tp), and
  // as the GEMM writing fp32 partials plus the bf16 reduce with one
  const bool bf16_two_kernels = (reduce_mode == TPS_REDUCE_BF16) && (partials != nullptr);
  if (!aligned16(X) || !aligned16(packed_v) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (ws && !aligned16(ws)) || (partials && !aligned16(partials)))
    return TPS_ERR_ALIGN;
  rc = check_device();
  if (rc) return rc;
  GemmCall c{};
  c.pr.kind = tps::K_ROW;
  c.pr.M = static_cast<int>(m);
  c.pr.tp = tp;
  c.pr.k_inner = k / tp;
  c.pr.w_rows = static_cast<int>(n);
  c.pr.per_shard = static_cast<int>(n);
  c.pr.row = true;
  c.pr.partials = (reduce_mode == TPS_REDUCE_PARTIALS) || bf16_two_kernels;
  c.pr.bf16 = (reduce_mode == TPS_REDUCE_BF16) && !bf16_two_kernels;
  c.pr.act = TPS_ACT_NONE;
  c.X = X;
  c.ldx = k;
  c.Wpk = packed_v;
  c.w_rows_total = n;
  c.Y = Y;
  c.ldy = static_cast<int>(n);
  c.y_f32 = (y_dtype == TPS_DTYPE_F32);
  c.partials = partials;
  c.bias = c.pr.partials ? nullptr : bias;
  c.hm.kv_den = 1;
  c.ws = ws;
  c.ws_bytes = ws ? ws_bytes : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = run_gemm(c, st);
  if (rc || !c.pr.partials) return rc;
  if (bf16_two_kernels) return shard_partial_reduce_bf16(partials, tp, m, n, bias, Y, y_dtype, stream);
  return shard_partial_reduce(partials, tp, m, n, bias, Y, y_dtype, stream);
}


int shard_partial_reduce(const float* partials, int tp, int64_t m, int64_t n, const void* bias, void* Y, int y_dtype,
                         void* stream) {
  return reduce_common(partials, tp, m, n, bias, Y, y_dtype, 0, stream);
}

int shard_partial_reduce_bf16(const float* partials, int tp, int64_t m, int64_t n, const void* bias, void* Y,
                              int y_dtype, void* stream) {
  return reduce_common(partials, tp, m, n, bias, Y, y_dtype, 1, stream);
}

// Argmax partial entries (value, index) per token and shard for a column problem
// with `per_shard` vocab columns per shard: weight-major tiles of 128 rows give
// four per tile, token-major tiles of >= 64 columns one.
int64_t argmax_entries_bound(int64_t per_shard) {
  return std::max<int64_t>(4 * ((per_shard + 127) / 128), (per_shard + 63) / 64);
}

int vocab_parallel_argmax(const void* X, int64_t m, int64_t H, const void* packed_w, int64_t V, int tp,
                          int32_t* out_idx, float* out_val, void* ws, size_t ws_bytes, void* stream) {
  if (m < 0 || m > (1LL << 30)) return TPS_ERR_ARG;
  PackGeom g{};
  int rc = pack_geom(TPS_KIND_COLUMN, H, V, tp, nullptr, &g);
  if (rc) return rc;
  if (m == 0) return TPS_OK;
  if (X == nullptr || packed_w == nullptr || out_idx == nullptr || ws == nullptr) return TPS_ERR_ARG;
  if (!aligned16(X) || !aligned16(packed_w) || !aligned16(ws) || (reinterpret_cast<uintptr_t>(out_idx) & 3) ||
      (reinterpret_cast<uintptr_t>(out_val) & 3))
    return TPS_ERR_ALIGN;
  if (ws_bytes < kHdr + static_cast<size_t>(m) * tp * argmax_entries_bound(g.per_shard) * 8) return TPS_ERR_WORKSPACE;
  rc = check_device();
  if (rc) return rc;
  GemmCall c{};
  c.pr.kind = tps::K_COLUMN;
  c.pr.M = static_cast<int>(m);
  c.pr.tp = tp;
  c.pr.k_inner = H;
  c.pr.w_rows = g.R;
  c.pr.per_shard = g.per_shard;
  c.pr.act = TPS_ACT_NONE;
  c.pr.argmax = true;
  c.X = X;
  c.ldx = H;
  c.Wpk = packed_w;
  c.w_rows_total = g.R;
  c.ldy = g.out_cols;
  c.hm.kv_den = 1;
  c.ws = ws;   // status header only: the argmax plans use no split
  c.ws_bytes = ws_bytes;
  const int sms = num_sms_current();
  Plan p{};
  rc = plan_gemm(c.pr, 0, sms, &p);
  if (rc) return rc;
  CUtensorMap tx, tw;
  GemmArgs a{};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = build_gemm(c, p, sms, st, &tx, &tw, &a);
  if (rc) return rc;
  const int parts = p.swap ? 4 : 1;
  const int entries = p.WT * parts;   // per token and shard
  a.amax = static_cast<char*>(ws) + kHdr;
  a.amax_stride = tp * entries;
  rc = tps::launch_gemm_argmax(p.swap, p.bn, tx, tw, a, p.grid, st);
  if (rc) return rc == -8 ? TPS_ERR_UNIMPLEMENTED : TPS_ERR_CUDA;
  return tps::launch_argmax_reduce(a.amax, static_cast<int>(m), tp, entries, out_idx, out_val, st) == 0 ? TPS_OK
                                                                                                     : TPS_ERR_CUDA;
}

int sharded_mlp_forward(const void* X, int64_t m, int64_t H, int64_t I, int tp, int act, const void* packed_up,
                        const void* packed_down, void* h_ws, void* Y, int y_dtype, void* ws, size_t ws_bytes,
                        void* stream) {
  if (act != TPS_ACT_GELU && act != TPS_ACT_SILU_MUL) return TPS_ERR_ARG;
  if (h_ws == nullptr) return TPS_ERR_ARG;
  const int kind = (act == TPS_ACT_GELU) ? TPS_KIND_COLUMN : TPS_KIND_GATE_UP;
  const int64_t n_up = (act == TPS_ACT_GELU) ? I : 2 * I;
  // validate both halves before enqueuing anything
  PackGeom g1{}, g2{};
  int rc = pack_geom(kind, H, n_up, tp, nullptr, &g1);
  if (rc) return rc;
  rc = pack_geom(TPS_KIND_ROW, I, H, tp, nullptr, &g2);
  if (rc) return rc;
  if (!valid_dtype(y_dtype)) return TPS_ERR_DTYPE;
  if (m < 0) return TPS_ERR_ARG;
  if (m == 0) return TPS_OK;
  if (X == nullptr || packed_up == nullptr || packed_down == nullptr || Y == nullptr) return TPS_ERR_ARG;
  if (!aligned16(X) || !aligned16(packed_up) || !aligned16(packed_down) || !aligned16(h_ws) || !aligned16(Y) ||
      (ws && !aligned16(ws)))
    return TPS_ERR_ALIGN;
  rc = check_device();
  if (rc) return rc;
  rc = run_mlp_fused(X, m, H, I, tp, act, g1, packed_up, packed_down, h_ws, Y, y_dtype == TPS_DTYPE_F32, ws,
                     ws_bytes, static_cast<cudaStream_t>(stream));
  if (rc != kFusedNotApplicable) return rc;
  rc = column_parallel_forward(X, m, H, packed_up, kind, n_up, tp, nullptr, nullptr, act, h_ws, TPS_DTYPE_BF16, ws,
                               ws_bytes, stream);
  if (rc) return rc;
  return row_parallel_forward(h_ws, m, I, packed_down, H, tp, nullptr, TPS_REDUCE_FUSED, nullptr, Y, y_dtype, ws,
                              ws_bytes, stream);
}

int sharded_attn_proj_forward(const void* X, const void* attn_out, int64_t m, int64_t H, const tps_heads* heads,
                              int tp, const void* packed_qkv, const void* packed_o, void* qkv_out, void* Y,
                              int y_dtype, void* ws, size_t ws_bytes, void* stream) {
  if (heads == nullptr) return TPS_ERR_ARG;
  const int64_t nq = static_cast<int64_t>(heads->hq + 2 * heads->hkv) * heads->head_dim;
  const int64_t ko = static_cast<int64_t>(heads->hq) * heads->head_dim;
  PackGeom g1{}, g2{};
  int rc = pack_geom(TPS_KIND_QKV, H, nq, tp, heads, &g1);
  if (rc) return rc;
  rc = pack_geom(TPS_KIND_ROW, ko, H, tp, nullptr, &g2);
  if (rc) return rc;
  if (!valid_dtype(y_dtype)) return TPS_ERR_DTYPE;
  if (m < 0) return TPS_ERR_ARG;
  if (m == 0) return TPS_OK;
  if (X == nullptr || attn_out == nullptr || packed_qkv == nullptr || packed_o == nullptr || qkv_out == nullptr ||
      Y == nullptr)
    return TPS_ERR_ARG;
  if (!aligned16(X) || !aligned16(attn_out) || !aligned16(packed_qkv) || !aligned16(packed_o) ||
      !aligned16(qkv_out) || !aligned16(Y) || (ws && !aligned16(ws)))
    return TPS_ERR_ALIGN;
  rc = column_parallel_forward(X, m, H, packed_qkv, TPS_KIND_QKV, nq, tp, heads, nullptr, TPS_ACT_NONE, qkv_out,
                               TPS_DTYPE_BF16, ws, ws_bytes, stream);
  if (rc) return rc;
  return row_parallel_forward(attn_out, m, ko, packed_o, H, tp, nullptr, TPS_REDUCE_FUSED, nullptr, Y, y_dtype, ws,
                              ws_bytes, stream);
}

int sharded_gqa_attention(const void* qkv, int64_t nseq, int64_t seqlen, const tps_heads* heads, int tp,
                          int causal, void* attn_out, void* stream) {
  if (heads == nullptr || nseq < 0 || seqlen < 0 || (causal != 0 && causal != 1)) return TPS_ERR_ARG;
  HeadMap hm{};
  int rc = head_map_calc(heads->hq, heads->hkv, tp, &hm);
  if (rc) return rc;
  if (heads->head_dim != tps::kAttnHeadDim) return TPS_ERR_UNIMPLEMENTED;
  const int64_t m = nseq * seqlen;
  if (nseq > (1LL << 30) || seqlen > (1LL << 30) || m > (1LL << 30)) return TPS_ERR_ARG;
  if (m == 0) return TPS_OK;
  if (qkv == nullptr || attn_out == nullptr) return TPS_ERR_ARG;
  if (!aligned16(qkv) || !aligned16(attn_out)) return TPS_ERR_ALIGN;
  rc = check_device();
  if (rc) return rc;
  const int d = heads->head_dim;
  tps::AttnArgs a{};
  a.nseq = static_cast<int>(nseq);
  a.S = static_cast<int>(seqlen);
  a.hq = heads->hq;
  a.qs = hm.qs;
  a.grp = heads->hq / heads->hkv;
  a.kvs = hm.kvs;
  a.kv_first_num = hm.kv_num;
  a.kv_first_den = hm.kv_den;
  a.shard_cols = (hm.qs + 2 * hm.kvs) * d;
  a.nqb = static_cast<int>((seqlen + 127) / 128);
  a.nkb = a.nqb;
  // plan-override bit 27: one query block per work item instead of two
  const int two_tiles = (g_plan_override.load() & (1 << 27)) ? 0 : 1;
  const int64_t items = nseq * static_cast<int64_t>(heads->hq) * (two_tiles ? (a.nqb + 1) / 2 : a.nqb);
  if (items > (1LL << 30)) return TPS_ERR_ARG;
  a.items = static_cast<int>(items);
  a.causal = causal;
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  a.out = attn_out;
  a.ldo = heads->hq * d;
  a.timeout_ns = kTimeoutNs;
  const int64_t cols = static_cast<int64_t>(tp) * a.shard_cols;
  CUtensorMap tm;
  rc = make_map(&tm, qkv, static_cast<uint64_t>(cols), static_cast<uint64_t>(m), 1, static_cast<uint64_t>(cols) * 2,
                static_cast<uint64_t>(cols) * 2 * static_cast<uint64_t>(m), 128, 1);
  if (rc) return rc;
  const int sms = num_sms_current();
  const int grid = a.items < sms ? a.items : sms;
  return tps::launch_attention(tm, a, two_tiles, grid, static_cast<cudaStream_t>(stream)) == 0 ? TPS_OK
                                                                                                : TPS_ERR_CUDA;
}

int row_parallel_forward_noalloc(const void* X, int64_t m, int64_t k, const void* packed_v, int64_t n, int tp,
                                 const void* bias, void* Y, int y_dtype, void* stream) {
  if (m < 0 || m > (1LL << 30)) return TPS_ERR_ARG;
  if (!valid_dtype(y_dtype)) return TPS_ERR_DTYPE;
  PackGeom g{};
  int rc = pack_geom(TPS_KIND_ROW, k, n, tp, nullptr, &g);
  if (rc) return rc;
  if (m > tps::kStaticMaxTokens) return TPS_ERR_WORKSPACE;  // beyond what the static scratch is sized for
  if (m == 0) return TPS_OK;
  if (X == nullptr || packed_v == nullptr || Y == nullptr) return TPS_ERR_ARG;
  if (!aligned16(X) || !aligned16(packed_v) || !aligned16(Y) || (bias && !aligned16(bias))) return TPS_ERR_ALIGN;
  rc = check_device();
  if (rc) return rc;
  void* scratch = nullptr;
  if (tps::static_scratch(&scratch) != 0) return TPS_ERR_CUDA;
  GemmCall c{};
  c.pr.static_ws = 1;
  c.pr.kind = tps::K_ROW;
  c.pr.M = static_cast<int>(m);
  c.pr.tp = tp;
  c.pr.k_inner = k / tp;
  c.pr.w_rows = static_cast<int>(n);
  c.pr.per_shard = static_cast<int>(n);
  c.pr.row = true;
  c.pr.partials = false;
  c.pr.act = TPS_ACT_NONE;
  c.X = X;
  c.ldx = k;
  c.Wpk = packed_v;
  c.w_rows_total = n;
  c.Y = Y;
  c.ldy = static_cast<int>(n);
  c.y_f32 = (y_dtype == TPS_DTYPE_F32);
  c.bias = bias;
  c.hm.kv_den = 1;
  c.ws = scratch;
  c.ws_bytes = tps::kStaticScratchBytes;
  return run_gemm(c, static_cast<cudaStream_t>(stream));
}

size_t tps_workspace_bytes(int fn, int64_t m, int64_t n, int64_t k, int tp) {
  if (m < 0 || n <= 0 || k <= 0 || tp <= 0) return 0;
  if (fn == TPS_FN_ARGMAX)
    return kHdr + round256(static_cast<size_t>(m) * tp * argmax_entries_bound((n + tp - 1) / tp) * 8);
  if (fn < TPS_FN_COLUMN || fn > TPS_FN_ATTN) return 0;
  return ws_bound(m, n, k, tp, num_sms_current());
}

int tps_sync_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned16(ws)) return TPS_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return TPS_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return TPS_ERR_CUDA;
  if (v == 0) return TPS_OK;
  if (cudaMemsetAsync(ws, 0, sizeof(int), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
    return TPS_ERR_CUDA;
  return v == TPS_ERR_DEVICE ? TPS_ERR_DEVICE : TPS_ERR_TIMEOUT;
}

int tps_device_error(void* stream) {
  int v = 0;
  if (tps::read_and_clear_device_error(static_cast<cudaStream_t>(stream), &v) != 0) return TPS_ERR_CUDA;
  if (v == 0) return TPS_OK;
  return v == TPS_ERR_DEVICE ? TPS_ERR_DEVICE : TPS_ERR_TIMEOUT;
}

int tps_debug_wait_timeout(int timeout_us, void* ws, size_t ws_bytes, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000) return TPS_ERR_ARG;
  if (ws != nullptr && ws_bytes < kHdr) return TPS_ERR_WORKSPACE;
  if (ws != nullptr && !aligned16(ws)) return TPS_ERR_ALIGN;
  const int rc = check_device();
  if (rc) return rc;
  return tps::launch_wait_timeout(static_cast<unsigned long long>(timeout_us) * 1000ull, ws_status(ws, ws_bytes),
                                  static_cast<cudaStream_t>(stream)) == 0
             ? TPS_OK
             : TPS_ERR_CUDA;
}

}  // extern "C"
