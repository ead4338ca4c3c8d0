// tps_internal.h -- declarations shared by the host API and the kernel
// translation unit (plain structs, no device code).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace tps {

enum : int { OUT_FINAL = 0, OUT_PARTIALS = 1 };
enum : int { K_COLUMN = 0, K_ROW = 1, K_QKV = 2, K_GATE_UP = 3 };
enum : int { A_NONE = 0, A_GELU = 1, A_SILU_MUL = 2 };

// Parameters of one sharded GEMM launch (see tps_gemm.cuh for the tile space).
struct GemmArgs {
  int M;                // tokens
  int tp;               // shards
  int KBs;              // 64-wide K blocks per shard K range
  int KI;               // K iterations per tile (KBs, or tp*KBs when k_spans_shards)
  int k_spans_shards;   // row FUSED: a tile's K loop runs over every shard
  int x_sharded;        // X tensor map is {k_s, tp, M} (row problems whose k_s is not a multiple of 64)
  int x_shard_cols;     // 2-D X map: column offset of shard ks's K range (row problems: k_s; column: 0)
  int S_tiles;          // shard groups in the tile space (column: tp, row fused: 1, partials: tp)
  int WT;               // weight tiles per shard group
  int wcols;            // weight tiles in the tile space (S_tiles * WT, fewer with kv_rep > 1)
  int kv_rep;           // QKV: shards sharing a KV head whose KV tiles the group's first shard computes once
  int qt;               // QKV with kv_rep > 1: query tiles per shard (the KV tiles follow them)
  int MT;               // token tiles
  int tiles;            // S_tiles * WT * MT
  int gm;               // raster group height (token tiles)
  int RB;               // 128-row blocks per shard in the packed weight
  // stream-K: tiles [0, dp_tiles) are data-parallel (dp_tiles is a multiple of the
  // grid), tiles [dp_tiles, tiles) are split by a stream-K partition of their
  // total_iters = (tiles - dp_tiles) * KI iterations over the grid
  int sk;
  int dp_tiles;
  int cs;               // cluster split: a cluster of cs CTAs shares each tile's K range (1 = off)
  long long total_iters;
  float* ws_part;
  int* ws_cnt;
  // epilogue
  int out_mode;
  int kind;
  int act;
  int per_shard;        // valid output columns per shard (column: n/tp, QKV: rows/shard, gate-up: I/tp, row: n)
  int ldy;              // output row length (elements)
  int y_f32;
  void* Y;
  float* partials;      // OUT_PARTIALS: [tp][M][per_shard] fp32
  void* amax;           // argmax epilogue: [M][amax_stride] (max logit, vocab index) per column tile
  int amax_stride;      // entries per token: tp * WT * (4 per-warp parts weight-major, 1 token-major)
  const void* bias;     // bf16, logical column order, or null
  int gate_off;         // gate-up: I (logical offset of the up bias)
  // QKV logical column map
  int q_cols;           // (hq/tp)*d
  int kv_cols;          // kv heads per shard * d
  int hq_d;             // hq*d
  int hkv_d;            // hkv*d
  int kv_first_num;     // first KV head of shard s = (s*kv_first_num)/kv_first_den
  int kv_first_den;
  int head_dim;
  unsigned long long timeout_ns;
  int* status;          // the caller's workspace status word (first word of ws), or null
  int bf16_chain;       // row-parallel bf16 exchange: partials rounded to bf16, summed in shard order,
                        // rounded after every addition (cluster split with cs = tp, a shard chain,
                        // or tp = 1)
  int chain;            // with bf16_chain: each tile's K range walked shard by shard by one CTA, a
                        // fresh accumulator per shard, the running bf16 sum kept in tensor memory
  int l2_hint;          // CTA-pair tiles: bit 0 loads X with the L2 evict-last policy, bit 1 loads W
                        // with evict-first (otherwise evict-normal)
};

// Readiness flags of the fused MLP kernel (global memory, zero between calls).
struct MlpSync {
  int* ready;   // [token blocks][tp]: fc1 tiles finished per (token block, shard)
  int* done;    // CTAs finished; the last one re-zeroes ready[] and done
  int n_ready;  // token blocks * tp
  int need;     // fc1 tiles per (token block, shard)
  int prefetch2;  // K blocks of its row-layer range whose weight boxes a CTA prefetches into L2
                  // once its column-layer loads are issued (0: none)
};

// One launch of the attention on local heads (tps_attn.cuh).
constexpr int kAttnHeadDim = 128;
struct AttnArgs {
  int nseq, S;                     // sequences; tokens per sequence (row of token t of sequence b: b*S + t)
  int hq, qs, grp;                 // query heads; query heads per shard; query heads per KV head
  int kvs;                         // KV heads per shard (replicas included)
  int kv_first_num, kv_first_den;  // first KV head of shard r = r*num/den
  int shard_cols;                  // columns of one shard's [q | k | v] block in a qkv row
  int nqb, nkb;                    // 128-row query blocks and key blocks per sequence
  int items;                       // work items (see launch_attention)
  int causal;
  float scale_log2;                // log2(e) / sqrt(d)
  void* out;                       // bf16 [nseq*S][ldo]
  int ldo;                         // hq * d
  unsigned long long timeout_ns;
  int* status;                     // launch status word, or null (device-wide word only)
};

struct PackHost {
  const void* W;
  void* out;
  int transposed;
  long long k, n;
  int tp, kind, R, Kp, ns;
  int q_cols, kv_cols, hq_d, hkv_d, kv_first_num, kv_first_den, head_dim;
  int Is, I;
};

// A caller workspace starts with a header of kWsHeaderBytes: its first int is the
// status word that kernels of calls given that workspace set on a device-side
// failure (read and cleared by tps_sync_status); the regions the kernels use
// (stream-K slots, tile counters, readiness flags, argmax entries) follow it.
constexpr size_t kWsHeaderBytes = 256;

// Allocation-free row-parallel entry point: size of the static scratch array,
// of its tile-counter region (at its end) and the largest token count served.
constexpr size_t kStaticScratchBytes = 12u << 20;
constexpr size_t kStaticCounterBytes = 64u << 10;
constexpr int kStaticMaxTokens = 64;
int static_scratch(void** ptr);

int gemm_smem_bytes(int swap, int bn, int dual);
int gemm_slot_elems(int swap, int bn, int dual);
// Column GEMM whose epilogue keeps, per token and tile, the largest logit and its
// vocab index instead of storing logits (a.amax); whole tiles only.
int launch_gemm_argmax(int swap, int bn, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid,
                       cudaStream_t st);
// Per token: the shard-local argmax over each shard's tile entries, then the max
// over shards (ties to the lowest index). part: [M][tp * per_shard_entries].
int launch_argmax_reduce(const void* part, int M, int tp, int per_shard_entries, int32_t* out_idx, float* out_val,
                         cudaStream_t st);
int launch_gemm(int swap, int bn, int dual, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a,
                int grid, cudaStream_t st);
int launch_gemm_csplit(int swap, int bn, int cs, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a,
                       int grid, cudaStream_t st);
int max_csplit_clusters(int swap, int bn, int cs);
// One-launch MLP: column tiles, then cluster-split row tiles, one launch of `grid`
// CTAs in clusters of a2.cs (the grid must fit the resident clusters). swap = 0:
// token-major 128-wide tiles (GELU); swap = 1: weight-major 64-token tiles with
// gate/up pairs (SiLU(gate)*up). Returns 0 or -6 (CUDA error).
int launch_mlp_fused(int swap, const CUtensorMap& tx, const CUtensorMap& tw1, const CUtensorMap& th,
                     const CUtensorMap& tw2, const GemmArgs& a1, const GemmArgs& a2, const MlpSync& sy, int grid,
                     cudaStream_t st);
// Token-major GEMM on CTA pairs: 256 tokens x (nh * bn) weight rows per tile.
// One-launch gated MLP at decode sizes (m <= 64) with stream-K over both layers on
// `grid` CTAs (at most mlp_sk_resident_ctas()); a1/a2 carry the stream-K
// partitions (sk = 1, dp_tiles = 0), their slots and tile counters.
int launch_mlp_sk(const CUtensorMap& tx, const CUtensorMap& tw1, const CUtensorMap& th, const CUtensorMap& tw2,
                  const GemmArgs& a1, const GemmArgs& a2, const MlpSync& sy, int grid, cudaStream_t st);
int mlp_sk_resident_ctas();
int mlp_sk_slot_bytes(int phase);   // bytes of one stream-K segment slot of phase 0 (gate/up) or 1 (down)
int launch_gemm_pair(int bn, int nh, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid,
                     cudaStream_t st);
int max_pair_clusters();
int launch_pack(const PackHost& h, cudaStream_t st);
// Attention on local heads over a qkv tensor map (box {64, 128}); grid CTAs,
// persistent. Returns 0 or -6 (CUDA error).
// two_tiles = 1: two 128-query blocks per work item sharing their K/V stream
// (items = nseq * hq * ceil(nqb / 2)); 0: one block per item (items = nseq * hq * nqb).
int launch_attention(const CUtensorMap& tqkv, const AttnArgs& a, int two_tiles, int grid, cudaStream_t st);
int attention_smem_bytes(int two_tiles);
// bf16_chain = 0: Y = P_0 + ... + P_{tp-1} (+ bias) in fp32; 1: every P_s rounded to
// bf16, summed in shard order with a bf16 rounding after each addition, bias added
// once with one more rounding.
int launch_reduce(const float* P, int tp, long long m, long long n, const void* bias, void* Y, int y_f32,
                  int bf16_chain, int num_sms, cudaStream_t st);
int launch_wait_timeout(unsigned long long timeout_ns, int* status, cudaStream_t st);
int read_and_clear_device_error(cudaStream_t st, int* out);

}  // namespace tps
