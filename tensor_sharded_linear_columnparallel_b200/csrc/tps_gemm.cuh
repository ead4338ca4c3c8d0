// tps_gemm.cuh -- the sharded linear-block GEMM for sm_100a.
//
// One kernel template serves every GEMM of the block:
//   * column-parallel (fc1 / gate-up / QKV): Y_s = X W_s for every shard s, the
//     tiles of all shards in one persistent launch; output columns of shard s are
//     written at its offset, so the output buffer is concat(Y_s).
//   * row-parallel (fc2 / down / o_proj): Y = sum_s X_s V_s. With the FUSED
//     reduction the K loop of a tile walks shard 0's K range, then shard 1's, ...,
//     all into ONE fp32 tensor-memory accumulator (split-K over shards folded into
//     the accumulator). When a stream-K partition splits a tile's K range over
//     several CTAs, each CTA writes its fp32 segment partial to the workspace and
//     the last CTA to finish the tile sums the segments in K order (fixed, so
//     the result is deterministic) and runs the epilogue. With cluster split-K
//     (CSPLIT) the cs CTAs of a thread-block cluster each take a contiguous share
//     of the tile's K range and the partial sums meet in distributed shared
//     memory (csplit_tile). With the PARTIALS reduction every tile is one
//     (shard, output tile) pair and P_s is stored to `partials[s]` for the
//     standalone reduce kernel.
//
// Hardware mapping (one CTA per SM, 6 warps):
//   warp 0   TMA producer: 128B-swizzled K-major tiles of X and W into a ring of
//            shared-memory stages, completion tracked by mbarriers (no multicast).
//   warp 1   tcgen05 MMA issuer (one thread), cta_group::1, M = 128, N = BN,
//            K = 16 per instruction, fp32 accumulators in tensor memory, two
//            accumulator buffers so the epilogue of one tile overlaps the main
//            loop of the next; warp 1 also allocates / frees tensor memory.
//   warps 2-5 epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//            32*(w%4) .. +31), then bias, activation (GELU, or SiLU(gate)*up) and
//            16-byte bf16 / fp32 stores straight from registers, 16 independent
//            elements per lane.
// Two tile orientations:
//   SWAP = false  tokens on the MMA M side (128 tokens x BN weight rows), for
//                 prefill-sized m.
//   SWAP = true   weight rows on the MMA M side (128 weight rows x BN tokens), for
//                 decode-sized m: the weight stream fills the 128-row MMA.
//   DUAL          (SWAP only) gate/up: two A tiles (128 gate rows and the matching
//                 128 up rows of one packed block) and two accumulators.
//   Token-major gate/up uses BN = 256 = [128 gate rows | 128 up rows] of a block.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "tps_internal.h"
#include "tps_ptx.cuh"

namespace tps {

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
// x rounded to bf16 (round to nearest, ties to even) and back to fp32.
__device__ __forceinline__ float bf16r(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// GELU(x) = 0.5 x (1 + erf(x / sqrt(2))) with erf from Abramowitz & Stegun,
// Handbook of Mathematical Functions, formula 7.1.28: for z >= 0,
//   erf(z) = 1 - (1 + a1 z + a2 z^2 + a3 z^3 + a4 z^4 + a5 z^5 + a6 z^6)^-16 + e(z),
//   |e(z)| <= 3e-7.
// With q = P(z)^-16 = 1 - erf(|z|): GELU(x) = x (1 - q/2) for x >= 0 and x q / 2
// for x < 0 (no cancellation in the negative tail). Two elements at a time on
// the packed fp32x2 pipe; one reciprocal per element on the special-function unit
// (P^16 overflows to +inf for |z| > ~17, where q = 0 is the correct limit).
__device__ __forceinline__ float2 gelu2(float2 x) {
  const float2 z = __fmul2_rn(f2(fabsf(x.x), fabsf(x.y)), f2(0.70710678118654752f, 0.70710678118654752f));
  float2 p = __ffma2_rn(f2(0.0000430638f, 0.0000430638f), z, f2(0.0002765672f, 0.0002765672f));
  p = __ffma2_rn(p, z, f2(0.0001520143f, 0.0001520143f));
  p = __ffma2_rn(p, z, f2(0.0092705272f, 0.0092705272f));
  p = __ffma2_rn(p, z, f2(0.0422820123f, 0.0422820123f));
  p = __ffma2_rn(p, z, f2(0.0705230784f, 0.0705230784f));
  p = __ffma2_rn(p, z, f2(1.0f, 1.0f));
  p = __fmul2_rn(p, p);   // P^2
  p = __fmul2_rn(p, p);   // P^4
  p = __fmul2_rn(p, p);   // P^8
  p = __fmul2_rn(p, p);   // P^16
  const float2 q = f2(rcp_approx(p.x), rcp_approx(p.y));
  const float2 pos = __fmul2_rn(x, __ffma2_rn(f2(-0.5f, -0.5f), q, f2(1.0f, 1.0f)));
  const float2 neg = __fmul2_rn(__fmul2_rn(x, f2(0.5f, 0.5f)), q);
  return f2(x.x < 0.0f ? (q.x > 0.0f ? neg.x : -0.0f) : pos.x, x.y < 0.0f ? (q.y > 0.0f ? neg.y : -0.0f) : pos.y);
}

// SiLU(g) * u = g u / (1 + exp(-g)), two elements at a time.
__device__ __forceinline__ float2 silu_mul2(float2 g, float2 u) {
  const float2 e = __fmul2_rn(g, f2(-1.4426950408889634f, -1.4426950408889634f));
  const float2 den = __fadd2_rn(f2(ex2_approx(e.x), ex2_approx(e.y)), f2(1.0f, 1.0f));
  return __fmul2_rn(__fmul2_rn(g, u), f2(rcp_approx(den.x), rcp_approx(den.y)));
}

// Logical (unsharded) column of output column `w` of shard `s`, used for bias.
__device__ __forceinline__ int logical_col(const GemmArgs& a, int s, int w) {
  if (a.kind == K_QKV) {
    const int kvf = (s * a.kv_first_num) / a.kv_first_den;
    if (w < a.q_cols) return s * a.q_cols + w;
    if (w < a.q_cols + a.kv_cols) return a.hq_d + kvf * a.head_dim + (w - a.q_cols);
    return a.hq_d + a.hkv_d + kvf * a.head_dim + (w - a.q_cols - a.kv_cols);
  }
  if (a.kind == K_ROW) return w;
  return s * a.per_shard + w;
}

__device__ __forceinline__ void tile_coords(const GemmArgs& a, int t, int& s, int& wt, int& mt) {
  const int span = a.gm * a.wcols;
  const int g = t / span;
  const int r = t - g * span;
  const int m_first = g * a.gm;
  const int gsz = min(a.gm, a.MT - m_first);
  mt = m_first + r % gsz;
  const int wc = r / gsz;
  if (a.kv_rep > 1) {
    // a group of kv_rep shards sharing one KV head: every shard's query tiles, then
    // the KV tiles once (the group's first shard; the epilogue stores the replicas)
    const int per = a.kv_rep * a.qt + (a.WT - a.qt);
    const int grp = wc / per;
    const int r2 = wc - grp * per;
    if (r2 < a.kv_rep * a.qt) {
      s = grp * a.kv_rep + r2 / a.qt;
      wt = r2 % a.qt;
    } else {
      s = grp * a.kv_rep;
      wt = a.qt + (r2 - a.kv_rep * a.qt);
    }
  } else {
    s = wc / a.WT;
    wt = wc - s * a.WT;
  }
}

// CTA that owns K iteration i of the flattened (tile, k) space under a stream-K
// partition of T iterations over C CTAs (CTA c owns [c*T/C, (c+1)*T/C)).
__device__ __forceinline__ int sk_owner(long long i, long long T, int C) {
  return static_cast<int>(((i + 1) * C + T - 1) / T) - 1;
}

// Workspace slot of CTA c's segment on the tile whose K iterations start at
// `tbeg`. A CTA's K range is contiguous, so it has at most two partial-tile
// segments: the one on the tile where its range begins (slot 2c) and the one on
// the tile where it ends (slot 2c+1); all tiles in between are whole.
__device__ __forceinline__ int sk_slot(int c, long long tbeg, long long T, int C) {
  const long long start = (static_cast<long long>(c) * T) / C;
  return start >= tbeg ? 2 * c : 2 * c + 1;
}

// Iterates the (tile, k_begin, k_end) segments of this CTA, identically in every
// role: first the data-parallel tiles t = blockIdx.x + i*gridDim.x < dp_tiles
// (whole K range), then, with stream-K, this CTA's contiguous share of the
// flattened (tile, k) iterations of the remaining tiles [dp_tiles, tiles).
struct SegIter {
  long long it, it_end;  // stream-K
  int t;                 // data-parallel
  int sub;               // shard chain: the next shard of tile t
  __device__ __forceinline__ void init(const GemmArgs& a) {
    sub = 0;
    t = (a.cs > 1) ? static_cast<int>(blockIdx.x) / a.cs : static_cast<int>(blockIdx.x);
    if (a.sk) {
      const long long T = a.total_iters;
      const int C = gridDim.x;
      it = (static_cast<long long>(blockIdx.x) * T) / C;
      it_end = (static_cast<long long>(blockIdx.x + 1) * T) / C;
    } else {
      it = it_end = 0;
    }
  }
  __device__ __forceinline__ bool next(const GemmArgs& a, int& tile, int& kb0, int& kb1) {
    if (a.chain) {
      // bf16 shard chain: a tile's shards in order 0, 1, ..., tp-1, one segment each
      if (t >= a.tiles) return false;
      tile = t;
      kb0 = sub * a.KBs;
      kb1 = kb0 + a.KBs;
      if (++sub == a.tp) {
        sub = 0;
        t += gridDim.x;
      }
      return true;
    }
    if (a.cs > 1) {
      // cluster split: every CTA of the cluster takes its contiguous share of the tile's K range
      if (t >= a.tiles) return false;
      const int r = static_cast<int>(blockIdx.x) % a.cs;
      tile = t;
      kb0 = (r * a.KI) / a.cs;
      kb1 = ((r + 1) * a.KI) / a.cs;
      t += static_cast<int>(gridDim.x) / a.cs;
      return true;
    }
    if (t < a.dp_tiles) {
      tile = t;
      kb0 = 0;
      kb1 = a.KI;
      t += gridDim.x;
      return true;
    }
    if (it >= it_end) return false;
    const int rel = static_cast<int>(it / a.KI);
    tile = a.dp_tiles + rel;
    kb0 = static_cast<int>(it - static_cast<long long>(rel) * a.KI);
    const long long rem = it_end - it;
    kb1 = static_cast<int>(min(static_cast<long long>(a.KI), kb0 + rem));
    it += kb1 - kb0;
    return true;
  }
};

constexpr int kEpiWarps = 4;                 // epilogue warps (1 per TMEM lane sub-partition)
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer warp + MMA warp + epilogue warps

// OR of `v` over the NT epilogue threads (named barrier 1).
template <int NT = 32 * kEpiWarps>
__device__ __forceinline__ bool epi_bar_or(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(v)), "n"(NT)
      : "memory");
  return out != 0;
}

// Barrier over the NT epilogue threads (named barrier 1).
template <int NT = 32 * kEpiWarps>
__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}

template <bool SWAP, int BN, bool DUAL, bool CSPLIT = false>
struct GemmCfg {
  static constexpr int XR = SWAP ? BN : 128;                   // token rows per tile
  static constexpr int WR = SWAP ? (DUAL ? 256 : 128) : BN;    // weight rows per tile
  static constexpr int WBOX = WR < 128 ? WR : 128;             // weight rows per TMA box
  static constexpr int NWB = WR / WBOX;                        // weight boxes per stage
  static constexpr int X_BYTES = XR * 128;
  static constexpr int W_BYTES = WR * 128;
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  static constexpr int STG_BYTES = 0;                           // the epilogue works from registers
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_LIMIT = 232448;                    // opt-in shared memory per CTA on sm_100
  static constexpr int P_BYTES = CSPLIT ? 128 * BN * 4 : 0;     // cluster split: cs slots of 128/cs fp32 rows
  static constexpr int STAGES_RAW = (SMEM_LIMIT - 1024 - BAR_BYTES - STG_BYTES - P_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr int ACC_COLS = BN * (DUAL ? 2 : 1);
  // the bf16 shard chain's running sum (fp32 cells holding bf16 values) after the two
  // accumulator buffers: single-accumulator tiles of at most 128 columns
  static constexpr int SUM_COLS = (!DUAL && !CSPLIT && BN <= 128) ? BN : 0;
  static constexpr int TMEM_NEED = 2 * ACC_COLS + SUM_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                                                : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(TMEM_NEED <= TMEM_COLS, "tensor memory columns");
  static constexpr int SLOT_ELEMS = 128 * ACC_COLS;            // fp32 per stream-K segment slot
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STG_BYTES + P_BYTES + 1024 + BAR_BYTES;
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, BN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
  static_assert(!CSPLIT || (!DUAL && BN <= 128 && (SWAP || BN >= 32)), "cluster split: single accumulator, BN <= 128");
  static_assert(!DUAL || SWAP, "dual A tiles only in weight-major tiles");
  static_assert(X_BYTES % 1024 == 0 && W_BYTES % 1024 == 0, "SW128 tiles are 1024-B aligned");
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
};

// ---------------------------------------------------------------- epilogue
// Finishes 16 accumulator columns [c0, c0+16) of the accumulator row `row` held
// by this thread (v; u = the up accumulator for gate/up): bias, activation,
// conversion and the stores, straight from registers.
//  token-major: the row is a token, the 16 columns are consecutive output
//    columns -> two 16-byte (bf16) or four 16-byte (fp32) stores.
//  weight-major: the row is a weight row (one output column), the 16 columns are
//    tokens; consecutive lanes write consecutive output columns.
// FULL = false compiles only what the one-launch MLP kernels need (no fp32 partials
// output, no bf16 exchange, no replicated KV columns, plain column-parallel bias
// indexing), which keeps their code small.
template <bool SWAP, int BN, bool FULL = true>
__device__ __forceinline__ void finish_row16(const GemmArgs& a, float (&v)[16], float (&u)[16], int s, int wt,
                                             int mt, int row, int c0, bool dry = false) {
  const bool gated = (a.act == A_SILU_MUL);
  const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(a.bias);
  int tok0, w0;
  if (!SWAP) {
    tok0 = mt * 128 + row;
    w0 = (gated ? wt * 128 : wt * BN) + c0;
    if (tok0 >= a.M) return;
  } else {
    tok0 = mt * BN + c0;
    w0 = wt * 128 + row;
    if (w0 >= a.per_shard) return;
  }
  // ---- partial sums of one shard (row-parallel PARTIALS): raw fp32, no bias
  if (FULL && a.out_mode == OUT_PARTIALS) {
    float* P = a.partials + static_cast<size_t>(s) * a.M * a.per_shard;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = SWAP ? tok0 + j : tok0;
      const int w = SWAP ? w0 : w0 + j;
      if (t < a.M && w < a.per_shard) P[static_cast<size_t>(t) * a.per_shard + w] = v[j];
    }
    return;
  }
  // ---- bf16 exchange of a single shard's partial (row-parallel, tp = 1): the
  // partial rounded to bf16, then the bias added once with one more rounding
  if (FULL && a.bf16_chain) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int w = SWAP ? w0 : w0 + j;
      v[j] = bf16r(v[j]);
      if (bias != nullptr && w < a.per_shard) v[j] = bf16r(v[j] + __bfloat162float(bias[w]));
    }
    bias = nullptr;
  }
  // ---- bias
  if (bias != nullptr) {
    if (!SWAP) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int w = w0 + j;
        if (w < a.per_shard) {
          if (gated) {
            v[j] += __bfloat162float(bias[s * a.per_shard + w]);
            u[j] += __bfloat162float(bias[a.gate_off + s * a.per_shard + w]);
          } else {
            v[j] += __bfloat162float(bias[FULL ? logical_col(a, s, w) : s * a.per_shard + w]);
          }
        }
      }
    } else {
      const float bx = gated ? __bfloat162float(bias[s * a.per_shard + w0])
                             : __bfloat162float(bias[FULL ? logical_col(a, s, w0) : s * a.per_shard + w0]);
      const float by = gated ? __bfloat162float(bias[a.gate_off + s * a.per_shard + w0]) : 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[j] += bx;
        if (gated) u[j] += by;
      }
    }
  }
  // ---- activation (uniform branch)
  if (gated) {
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float2 h = silu_mul2(f2(v[j], v[j + 1]), f2(u[j], u[j + 1]));
      v[j] = h.x;
      v[j + 1] = h.y;
    }
  } else if (a.act == A_GELU) {
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float2 h = gelu2(f2(v[j], v[j + 1]));
      v[j] = h.x;
      v[j + 1] = h.y;
    }
  }
  // ---- store (a KV tile computed once for kv_rep shards goes to every replica's columns)
  const int nrep = (FULL && a.kv_rep > 1 && w0 >= a.q_cols) ? a.kv_rep : 1;
  if (!SWAP) {
    const bool full = (w0 + 16 <= a.per_shard);
    uint32_t pk[8];
    if (!a.y_f32) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        pk[j] = *reinterpret_cast<uint32_t*>(&b);
      }
    }
#pragma unroll 1
    for (int rr = 0; rr < nrep; ++rr) {
      const int col0 = (a.kind == K_ROW) ? w0 : (s + rr) * a.per_shard + w0;
      const size_t o = static_cast<size_t>(tok0) * a.ldy + col0;
      if (a.y_f32) {
        float* Y = reinterpret_cast<float*>(a.Y) + o;
        if (full && ((o & 3) == 0)) {
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            if (!dry) *reinterpret_cast<float4*>(Y + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (!dry && w0 + j < a.per_shard) Y[j] = v[j];
        }
      } else {
        __nv_bfloat16* Y = reinterpret_cast<__nv_bfloat16*>(a.Y) + o;
        if (full && ((o & 7) == 0)) {
          if (!dry) {
            *reinterpret_cast<uint4*>(Y) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(Y + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (!dry && w0 + j < a.per_shard) Y[j] = __float2bfloat16_rn(v[j]);
        }
      }
    }
  } else {
#pragma unroll 1
    for (int rr = 0; rr < nrep; ++rr) {
      const int col = (a.kind == K_ROW) ? w0 : (s + rr) * a.per_shard + w0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = tok0 + j;
        if (t >= a.M) break;
        const size_t o = static_cast<size_t>(t) * a.ldy + col;
        if (dry) continue;
        if (a.y_f32)
          reinterpret_cast<float*>(a.Y)[o] = v[j];
        else
          reinterpret_cast<__nv_bfloat16*>(a.Y)[o] = __float2bfloat16_rn(v[j]);
      }
    }
  }
}

// ---------------------------------------------------------------- stream-K fix-up
// Sums, for this thread's accumulator row, the 16 columns [cb, cb+16) of the
// fp32 segment partials of a tile in K order (CTA first, first+1, ..., last). Loads of up to four segments are in flight before they are
// added. Slot layout: float4 groups [col/4][row][4].
template <int SLOT_ELEMS>
__device__ __forceinline__ void sk_sum16(const GemmArgs& a, float (&v)[16], int row, int cb, long long tbeg, int first,
                                         int nseg) {
  constexpr int G = 4;
  float4 acc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
  for (int g0 = 0; g0 < nseg; g0 += G) {
    float4 x[G][4];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (g0 + g < nseg) {
        const float4* sl = reinterpret_cast<const float4*>(
            a.ws_part + static_cast<size_t>(sk_slot(first + g0 + g, tbeg, a.total_iters, gridDim.x)) * SLOT_ELEMS);
#pragma unroll
        for (int q = 0; q < 4; ++q) x[g][q] = __ldcg(sl + ((cb >> 2) + q) * 128 + row);
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (g0 + g < nseg) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[q].x += x[g][q].x;
          acc[q].y += x[g][q].y;
          acc[q].z += x[g][q].z;
          acc[q].w += x[g][q].w;
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[4 * q] = acc[q].x;
    v[4 * q + 1] = acc[q].y;
    v[4 * q + 2] = acc[q].z;
    v[4 * q + 3] = acc[q].w;
  }
}

// Bias and store of four consecutive output columns w0..w0+3 of token `tok`
// (one 8-byte bf16 or 16-byte fp32 store when all four are in range and aligned).
__device__ __forceinline__ void store4(const GemmArgs& a, const float (&o)[4], int s, int tok, int w0,
                                       const __nv_bfloat16* bias) {
  float x[4] = {o[0], o[1], o[2], o[3]};
  if (bias != nullptr) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (w0 + j < a.per_shard) x[j] += __bfloat162float(bias[logical_col(a, s, w0 + j)]);
  }
  const size_t base = static_cast<size_t>(tok) * a.ldy + ((a.kind == K_ROW) ? w0 : s * a.per_shard + w0);
  const size_t esz = a.y_f32 ? 4 : 2;
  if (w0 + 4 <= a.per_shard && ((reinterpret_cast<uintptr_t>(a.Y) + base * esz) & (4 * esz - 1)) == 0) {
    if (a.y_f32) {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.Y) + base) = make_float4(x[0], x[1], x[2], x[3]);
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]);
      __nv_bfloat162 hi = __floats2bfloat162_rn(x[2], x[3]);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.Y) + base) =
          make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (w0 + j >= a.per_shard) break;
    if (a.y_f32)
      reinterpret_cast<float*>(a.Y)[base + j] = x[j];
    else
      reinterpret_cast<__nv_bfloat16*>(a.Y)[base + j] = __float2bfloat16_rn(x[j]);
  }
}

// Bias and store of output column `w` of the four consecutive tokens tok0..tok0+3.
__device__ __forceinline__ void store_tok4(const GemmArgs& a, const float (&o)[4], int s, int tok0, int w,
                                           const __nv_bfloat16* bias) {
  if (w >= a.per_shard) return;
  const float bv = (bias != nullptr) ? __bfloat162float(bias[logical_col(a, s, w)]) : 0.0f;
  const size_t col = static_cast<size_t>((a.kind == K_ROW) ? w : s * a.per_shard + w);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int t = tok0 + j;
    if (t >= a.M) break;
    const size_t off = static_cast<size_t>(t) * a.ldy + col;
    if (a.y_f32)
      reinterpret_cast<float*>(a.Y)[off] = o[j] + bv;
    else
      reinterpret_cast<__nv_bfloat16*>(a.Y)[off] = __float2bfloat16_rn(o[j] + bv);
  }
}

// ---------------------------------------------------------------- cluster split-K
// One tile of a cluster-split GEMM, for the epilogue thread holding accumulator
// row `row`. CTA rank o of the cluster owns rows [o*rs, (o+1)*rs), rs = 128/cs
// (tokens, or weight rows in the weight-major orientation), and finishes them.
// Every CTA's partial buffer holds cs slots, one per source rank, each with the
// owned rows of that rank's fp32 partial.
// (1) wait until every owner has finished reading the previous tile (this CTA's
// `consumed`); (2) store the accumulator row (this CTA's K share) into the
// owner's slot for this rank -- remote stores into its shared memory -- release
// tensor memory and release-arrive on the owner's `ready`; (3) wait for this
// CTA's own `ready`: all cs partials of its rows are in place; (4) sum them in
// rank order 0, 1, ..., cs-1 (K order, deterministic) from local shared memory,
// add the bias and store; (5) arrive on every CTA's `consumed` -- except after
// the cluster's last tile: then every remote access to a CTA's shared memory has
// completed by its own `ready` wait and the CTAs may exit. Every wait is
// bounded. Slot layout, both orientations: [rs rows][BN columns] fp32 with the
// float4 group index XOR'd with the row (conflict-free 16-byte stores and loads).
// EPW epilogue warps: 4 (one thread per accumulator row) or 8 (two threads per row,
// each pushing half of the row's columns; `ready` then counts 256 arrivals and
// `consumed` 256 * cs).
// (2) of csplit_tile: this thread's accumulator row (or its half, EPW = 8) into the
// owner's slot for this CTA's rank. Not inlined, so that a dry call (no stores) made
// while the main loop runs fetches the very instructions the real call executes.
template <bool SWAP, int BN, int EPW>
__device__ __noinline__ void csplit_push(int cs, float* gP, uint32_t sP, uint32_t tacc, bool has_k, int row,
                                         int ep_tid, bool dry) {
  static_assert(EPW == 4 || EPW == 8, "one or two epilogue threads per accumulator row");
  constexpr int kCols = BN * 4 / EPW;                               // columns this thread pushes
  constexpr int kCw = kCols >= 32 ? 32 : 16;                        // columns per tensor-memory load
  static_assert(kCols % kCw == 0, "whole loads");
  constexpr int kSwz = (BN / 4 < 8 ? BN / 4 : 8) - 1;              // float4-group swizzle mask
  // cs is 2, 4 or 8: every index below is a shift or a mask
  const int lrs = 7 - (__ffs(cs) - 1);                            // rs = 128 / cs = 1 << lrs
  const int slot_floats = (1 << lrs) * BN;
  const uint32_t rank = static_cast<uint32_t>(blockIdx.x) & static_cast<uint32_t>(cs - 1);
  const uint32_t owner = static_cast<uint32_t>(row >> lrs);
  const int rr = row & ((1 << lrs) - 1);                        // row within the owned slice
  const bool local = (owner == rank);
  float* lslot = gP + static_cast<size_t>(rank) * slot_floats;
  const uint32_t rslot = mapa_shared(sP + static_cast<uint32_t>(rank) * slot_floats * 4u, owner);
  const int cbeg = (EPW == 8) ? (ep_tid >> 7) * kCols : 0;      // this thread's half of the row (EPW = 8)
#pragma unroll 1
  for (int c0 = cbeg; c0 < cbeg + kCols; c0 += kCw) {
    float v[kCw];
    if constexpr (kCw == 32)
      tmem_ld32(tacc + c0, v);
    else
      tmem_ld16(tacc + c0, v);
    if (!has_k) {
#pragma unroll
      for (int j = 0; j < kCw; ++j) v[j] = 0.0f;
    }
#pragma unroll
    for (int g = 0; g < kCw / 4; ++g) {
      const int f = rr * BN + ((((c0 >> 2) + g) ^ (rr & kSwz)) << 2);
      if (dry) continue;
      if (local)
        *reinterpret_cast<float4*>(lslot + f) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      else
        st_dsmem_f4(rslot + 4u * f, v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
    }
  }
}

// What the cluster reduce of a row-parallel tile reads from the launch arguments,
// passed by value to the non-inlined reduce (a reference to the launch arguments
// would turn every field read into a generic load from the parameter space).
struct RowOut {
  void* Y;
  const __nv_bfloat16* bias;
  int M, ldy, n, y_f32, cs, bf16_chain;
};
__device__ __forceinline__ RowOut row_out(const GemmArgs& a) {
  return RowOut{a.Y, static_cast<const __nv_bfloat16*>(a.bias), a.M, a.ldy, a.per_shard, a.y_f32, a.cs, a.bf16_chain};
}

// (4) of csplit_tile: reduce from local shared memory in rank order. Work item = 4
// consecutive values of one slot row: token-major, 4 output columns of one token
// (lanes along the columns); weight-major, one output column of 4 tokens (lanes along
// the output columns). Either way a warp's stores are contiguous. The bias is added
// once (column w of a row-parallel output is logical column w). Not inlined, and
// callable dry (no stores), for the same reason as csplit_push.
template <bool SWAP, int BN, int EPW, bool CHAIN>
__device__ __noinline__ void csplit_reduce(const RowOut o, const float* gP, int wt, int mt, int ep_tid, bool dry) {
  constexpr int kSwz = (BN / 4 < 8 ? BN / 4 : 8) - 1;
  constexpr int kLg = (BN >= 128) ? 5 : (BN >= 64) ? 4 : (BN >= 32) ? 3 : 2;   // log2(BN / 4)
  const int cs = o.cs;
  const int lrs = 7 - (__ffs(cs) - 1);
  const int rs = 1 << lrs;
  const int slot_floats = rs * BN;
  const uint32_t rank = static_cast<uint32_t>(blockIdx.x) & static_cast<uint32_t>(cs - 1);
  const int rbase = static_cast<int>(rank) << lrs;
  const bool chain = CHAIN && o.bf16_chain;
  const int nitems = rs * (BN / 4);
  constexpr int NB = 4;
  constexpr int CSMAX = 8;
#pragma unroll 1
  for (int i0 = ep_tid; i0 < nitems; i0 += NB * 32 * EPW) {
    float4 acc[NB];
    int lo[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      acc[b] = make_float4(0.f, 0.f, 0.f, 0.f);
      const int it = min(i0 + b * 32 * EPW, nitems - 1);
      const int r = SWAP ? (it & (rs - 1)) : (it >> kLg);
      const int g = SWAP ? (it >> lrs) : (it & (BN / 4 - 1));
      lo[b] = r * BN + ((g ^ (r & kSwz)) << 2);
    }
    if (!chain) {
#pragma unroll
      for (int q = 0; q < CSMAX; ++q) {
        if (q < cs) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float4 x = *reinterpret_cast<const float4*>(gP + static_cast<size_t>(q) * slot_floats + lo[b]);
            acc[b].x += x.x; acc[b].y += x.y; acc[b].z += x.z; acc[b].w += x.w;
          }
        }
      }
    } else {
      // bf16 exchange (cs = tp: slot q holds shard q's whole partial): every partial
      // rounded to bf16, summed in shard order with a rounding after each addition
#pragma unroll
      for (int q = 0; q < CSMAX; ++q) {
        if (q < cs) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float4 x = *reinterpret_cast<const float4*>(gP + static_cast<size_t>(q) * slot_floats + lo[b]);
            acc[b].x = bf16r(acc[b].x + bf16r(x.x));
            acc[b].y = bf16r(acc[b].y + bf16r(x.y));
            acc[b].z = bf16r(acc[b].z + bf16r(x.z));
            acc[b].w = bf16r(acc[b].w + bf16r(x.w));
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const int it = i0 + b * 32 * EPW;
      if (it >= nitems) break;
      float x[4] = {acc[b].x, acc[b].y, acc[b].z, acc[b].w};
      if (!SWAP) {
        // four output columns w0..w0+3 of token tok
        const int tok = mt * 128 + rbase + (it >> kLg);
        const int w0 = wt * BN + ((it & (BN / 4 - 1)) << 2);
        if (o.bias != nullptr) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (w0 + j < o.n) x[j] = chain ? bf16r(x[j] + __bfloat162float(o.bias[w0 + j]))   // once, rounded again
                                           : x[j] + __bfloat162float(o.bias[w0 + j]);
        }
        if (dry || tok >= o.M) continue;
        const size_t base = static_cast<size_t>(tok) * o.ldy + w0;
        const size_t esz = o.y_f32 ? 4 : 2;
        if (w0 + 4 <= o.n && ((reinterpret_cast<uintptr_t>(o.Y) + base * esz) & (4 * esz - 1)) == 0) {
          if (o.y_f32) {
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(o.Y) + base) = make_float4(x[0], x[1], x[2], x[3]);
          } else {
            __nv_bfloat162 l2 = __floats2bfloat162_rn(x[0], x[1]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2], x[3]);
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(o.Y) + base) =
                make_uint2(*reinterpret_cast<uint32_t*>(&l2), *reinterpret_cast<uint32_t*>(&h2));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (w0 + j >= o.n) break;
            if (o.y_f32)
              reinterpret_cast<float*>(o.Y)[base + j] = x[j];
            else
              reinterpret_cast<__nv_bfloat16*>(o.Y)[base + j] = __float2bfloat16_rn(x[j]);
          }
        }
      } else {
        // output column w of the four consecutive tokens tok0..tok0+3
        const int w = wt * 128 + rbase + (it & (rs - 1));
        const int tok0 = mt * BN + ((it >> lrs) << 2);
        if (w >= o.n) continue;
        const float bw = (o.bias != nullptr) ? __bfloat162float(o.bias[w]) : 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = tok0 + j;
          if (dry || t >= o.M) break;
          const float y = chain ? bf16r(x[j] + bw) : x[j] + bw;
          const size_t off = static_cast<size_t>(t) * o.ldy + w;
          if (o.y_f32)
            reinterpret_cast<float*>(o.Y)[off] = y;
          else
            reinterpret_cast<__nv_bfloat16*>(o.Y)[off] = __float2bfloat16_rn(y);
        }
      }
    }
  }
}

template <bool SWAP, int BN, int EPW = kEpiWarps, bool CHAIN = true>
__device__ __forceinline__ bool csplit_tile(const GemmArgs& a, float* gP, uint32_t sP, uint32_t ready_bar,
                                            uint32_t consumed_bar, uint32_t tempty, volatile int* abort_flag,
                                            uint64_t tmo, uint32_t tacc, bool has_k, int s, int wt, int mt, int row,
                                            int lane, int ep_tid, int nloc, bool last) {
  const int cs = a.cs;
  const int lrs = 7 - (__ffs(cs) - 1);
  const uint32_t owner = static_cast<uint32_t>(row >> lrs);
  if (nloc > 0 && !mbar_wait_cluster(consumed_bar, static_cast<uint32_t>((nloc - 1) & 1), abort_flag, tmo, a.status))
    return false;
  // (2) accumulator row -> the owner's slot for this rank (same offset in every CTA)
  csplit_push<SWAP, BN, EPW>(cs, gP, sP, tacc, has_k, row, ep_tid, false);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(tempty);
  // publish: the release arrive orders this thread's stores before it
  mbar_arrive_cluster(mapa_shared(ready_bar, owner));
  // (3) every rank's partial of this CTA's rows is in place
  if (!mbar_wait_cluster(ready_bar, static_cast<uint32_t>(nloc & 1), abort_flag, tmo, a.status)) return false;
  // (4) the sum in rank order, bias, stores
  csplit_reduce<SWAP, BN, EPW, CHAIN>(row_out(a), gP, wt, mt, ep_tid, false);
  // (5) this CTA has read every slot of this tile
  if (!last)
    for (int r = 0; r < cs; ++r) mbar_arrive_cluster(mapa_shared(consumed_bar, static_cast<uint32_t>(r)));
  return true;
}

// A dry pass through csplit_tile's two non-inlined parts (no stores, no barriers), made
// while the main loop runs so that their instructions are already fetched when the
// accumulator is ready. `tacc_spare` must be tensor memory no MMA is writing yet; gP is
// only read.
template <bool SWAP, int BN, int EPW = kEpiWarps, bool CHAIN = true>
__device__ __forceinline__ void csplit_warm(const GemmArgs& a, float* gP, uint32_t sP, uint32_t tacc_spare, int row,
                                            int ep_tid) {
  csplit_push<SWAP, BN, EPW>(a.cs, gP, sP, tacc_spare, true, row, ep_tid, true);
  csplit_reduce<SWAP, BN, EPW, CHAIN>(row_out(a), gP, 0, 0, ep_tid, true);
}

// ---------------------------------------------------------------- greedy argmax epilogue
// Greedy decoding over a vocab-parallel lm_head ("Tensor Parallel：当一张 GPU 放不下一个
// 大模型", section "lm_head 怎么处理": each shard finds its largest logit, then the
// largest over shards is taken). Instead of storing the tile's logits, the tile
// writes, per token, its largest logit and that logit's vocab index (the lowest
// index on ties) to a.amax[token][entry], entry = (s * WT + wt) * parts + part:
// token-major tiles have one part (a thread owns a token row and scans the tile's
// columns in increasing order); weight-major tiles have one part per epilogue
// warp (32 vocab rows, reduced across lanes by shuffles).
struct AmaxEntry {
  float v;
  int i;
};

__device__ __forceinline__ void amax_take(float& bv, int& bi, float v, int i) {
  if (v > bv || (v == bv && i < bi)) {
    bv = v;
    bi = i;
  }
}

template <bool SWAP, int BN>
__device__ __forceinline__ void argmax_tile(const GemmArgs& a, uint32_t tacc, int s, int wt, int mt, int row, int q,
                                            int lane) {
  AmaxEntry* out = static_cast<AmaxEntry*>(a.amax);
  const int tcol = s * a.WT + wt;
  constexpr int kNone = 0x7fffffff;
  if (!SWAP) {
    const int tok = mt * 128 + row;
    float bv = -INFINITY;
    int bi = kNone;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float v[16];
      tmem_ld16(tacc + c0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int w = wt * BN + c0 + j;
        if (w < a.per_shard && v[j] > bv) {   // increasing column order: strict > keeps the first
          bv = v[j];
          bi = s * a.per_shard + w;
        }
      }
    }
    if (tok < a.M) out[static_cast<size_t>(tok) * a.amax_stride + tcol] = AmaxEntry{bv, bi};
  } else {
    const int w = wt * 128 + row;   // this thread's vocab row within the shard
    const bool valid = w < a.per_shard;
    const int idx = s * a.per_shard + w;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      float v[16];
      tmem_ld16(tacc + c0, v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {   // unrolled: v[] stays in registers
        float bv = valid ? v[j] : -INFINITY;
        int bi = valid ? idx : kNone;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
          amax_take(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
        const int tok = mt * BN + c0 + j;
        if (lane == 0 && tok < a.M) out[static_cast<size_t>(tok) * a.amax_stride + tcol * 4 + q] = AmaxEntry{bv, bi};
      }
    }
  }
}

// ---------------------------------------------------------------- the kernel
template <bool SWAP, int BN, bool DUAL, bool CSPLIT = false, bool ARGMAX = false>
__global__ void __launch_bounds__(kThreads, 1)
    tps_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const GemmArgs a) {
  using C = GemmCfg<SWAP, BN, DUAL, CSPLIT>;
  constexpr int STAGES = C::STAGES;
  if (CSPLIT && !cluster_size_is(static_cast<uint32_t>(a.cs), a.status)) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sX = base;                               // STAGES x X tiles
  const uint32_t sW = base + STAGES * C::X_BYTES;         // STAGES x W tiles
  const uint32_t sP = base + STAGES * C::STAGE_BYTES + C::STG_BYTES;        // cluster-split partial tile
  float* gP = reinterpret_cast<float*>(gbase + STAGES * C::STAGE_BYTES + C::STG_BYTES);
  const uint32_t sBar = sP + C::P_BYTES;                                     // barriers
  uint8_t* gBar = gbase + STAGES * C::STAGE_BYTES + C::STG_BYTES + C::P_BYTES;
  // barrier map: full[STAGES], empty[STAGES], tfull[2], tempty[2], done, epi_done
  auto full_bar = [&](int i) { return sBar + 8u * i; };
  auto empty_bar = [&](int i) { return sBar + 8u * (STAGES + i); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * STAGES + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * STAGES + 2 + i); };
  const uint32_t done_bar = sBar + 8u * (2 * STAGES + 4);
  const uint32_t epi_done_bar = sBar + 8u * (2 * STAGES + 5);
  const uint32_t ready_bar = sBar + 8u * (2 * STAGES + 6);      // cluster split: all partials of a tile written
  const uint32_t consumed_bar = sBar + 8u * (2 * STAGES + 7);   // cluster split: all slices of a tile read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 8));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 8) + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 8) + 8);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 8) + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), kEpiWarps);
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_done_bar, kEpiWarps);
    if (CSPLIT) {
      mbar_init(ready_bar, 32 * kEpiWarps);          // one arrive per accumulator row of the owned slice, all ranks
      mbar_init(consumed_bar, 32 * kEpiWarps * a.cs);  // every epilogue thread of every rank
    }
    *abort_flag = 0;
    *last_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  if (CSPLIT)
    cluster_sync_all();   // every CTA's barriers are initialised before any remote arrive
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;
  (void)sP;
  (void)gP;
  // Programmatic dependent launch: the next kernel of the stream may be scheduled
  // now (its CTAs take SMs as this grid's CTAs exit). This grid's own wait for
  // the previous kernel (griddepcontrol.wait) is in the producer, before its
  // first load; every global access of the other roles follows that load.
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      SegIter seg;
      seg.init(a);
      int tile, kb0, kb1;
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      griddep_wait();
      while (ok && seg.next(a, tile, kb0, kb1)) {
        int s, wt, mt;
        tile_coords(a, tile, s, wt, mt);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
          const int ks = a.k_spans_shards ? kb / a.KBs : s;      // shard of this K block
          const int kk = a.k_spans_shards ? kb - ks * a.KBs : kb;
          mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
          const int xrow = mt * C::XR;
          if (a.x_sharded)
            tma_load_3d(sX + stage * C::X_BYTES, &tmX, full_bar(stage), kk * 64, ks, xrow);
          else
            tma_load_3d(sX + stage * C::X_BYTES, &tmX, full_bar(stage), ks * a.x_shard_cols + kk * 64, xrow, 0);
          // packed weights are [shard][row block of 128][K block of 64][128][64]: each box
          // is one contiguous run of WBOX rows x 128 B
#pragma unroll
          for (int j = 0; j < C::NWB; ++j) {
            const int row0 = wt * C::WR + j * C::WBOX;
            tma_load_4d(sW + stage * C::W_BYTES + j * C::WBOX * 128, &tmW, full_bar(stage), 0, row0 & 127, kk,
                        ks * a.RB + (row0 >> 7));
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // wait (bounded) for the copies still in flight before the CTA may exit
      const long long first = issued > STAGES ? issued - STAGES : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait(full_bar(static_cast<int>(i % STAGES)), static_cast<uint32_t>((i / STAGES) & 1), never_flag,
                  200000000ull, a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      SegIter seg;
      seg.init(a);
      int tile, kb0, kb1;
      int stage = 0;
      uint32_t phase = 0;
      int nloc = 0;
      bool ok = true;
      bool any = false;
      while (ok && seg.next(a, tile, kb0, kb1)) {
        const int buf = nloc & 1;
        const uint32_t use = static_cast<uint32_t>(nloc >> 1);
        if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * C::ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, tmo, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xa = sX + stage * C::X_BYTES;
          const uint32_t wa = sW + stage * C::W_BYTES;
          const uint64_t dx = smem_desc_sw128(xa);
          const uint64_t dw = smem_desc_sw128(wa);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
            const uint64_t koff = static_cast<uint64_t>(kk * 2);   // 32 B along K, in 16-B units
            if (SWAP) {
              umma_bf16(d0, dw + koff, dx + koff, C::IDESC, acc);
              if (DUAL) {
                const uint64_t dw2 = smem_desc_sw128(wa + 128 * 128);  // up rows 128..255 of the block
                umma_bf16(d0 + BN, dw2 + koff, dx + koff, C::IDESC, acc);
              }
            } else {
              umma_bf16(d0, dx + koff, dw + koff, C::IDESC, acc);
            }
          }
          umma_commit(empty_bar(stage));
          any = true;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tfull_bar(buf));
        ++nloc;
      }
      // every issued MMA must be complete before tensor memory is released
      if (any) {
        umma_commit(done_bar);
        mbar_wait(done_bar, 0, never_flag, 200000000ull, a.status);
      }
      // ... and every epilogue warp must be done reading it
      mbar_wait(epi_done_bar, 0, never_flag, tmo, a.status);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane sub-partition of this warp
    const int half = (warp - 2) >> 2;       // with 8 epilogue warps, warps w and w+4 alternate chunks (0 here)
    const int row = q * 32 + lane;          // accumulator row (TMEM lane)
    const int ep_tid = threadIdx.x - 64;
    const bool gated = (a.act == A_SILU_MUL);
    const int ncols = (!SWAP && gated) ? BN / 2 : BN;
    const int uoff = DUAL ? BN : BN / 2;
    SegIter seg;
    seg.init(a);
    int tile, kb0, kb1;
    int nloc = 0;
    while (seg.next(a, tile, kb0, kb1)) {
      const int buf = nloc & 1;
      const uint32_t use = static_cast<uint32_t>(nloc >> 1);
      const bool ok = mbar_wait(tfull_bar(buf), use & 1u, abort_flag, tmo, a.status);
      if (epi_bar_or(!ok)) break;            // all epilogue threads leave together
      tc_fence_after();
      int s, wt, mt;
      tile_coords(a, tile, s, wt, mt);
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * C::ACC_COLS);
      if constexpr (CSPLIT) {
        if (!csplit_tile<SWAP, BN>(a, gP, sP, ready_bar, consumed_bar, tempty_bar(buf), abort_flag, tmo, tacc,
                                   kb0 < kb1, s, wt, mt, row, lane, ep_tid, nloc, seg.t >= a.tiles))
          break;
        ++nloc;
        continue;
      }
      if constexpr (C::SUM_COLS > 0) {
        if (a.chain) {
          // bf16 shard chain: this segment is shard sh's whole partial P_sh. The running
          // sum S (bf16 values, kept in tensor memory after the accumulator buffers)
          // becomes S = bf16(S + bf16(P_sh)), S = bf16(P_0) for the first shard; after the
          // last shard the bias is added once with one more rounding and Y is stored.
          const int sh = kb0 / a.KBs;
          const bool last = (sh == a.tp - 1);
          const uint32_t tsum =
              tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(2 * C::ACC_COLS);
          static_assert(kEpiWarps == 4, "one epilogue thread per accumulator row");
          if (!last && C::ACC_COLS % 32 == 0) {
            // 32 columns per step, the stores' completion awaited once
#pragma unroll 1
            for (int c0 = 0; c0 < C::ACC_COLS; c0 += 32) {
              float v[32], sum[32];
              tmem_ld32(tacc + c0, v);
              if (sh > 0) {
                tmem_ld32(tsum + c0, sum);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) sum[j] = 0.0f;
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) sum[j] = bf16r(sum[j] + bf16r(v[j]));
              tmem_st32_nowait(tsum + c0, sum);
            }
            tmem_wait_st_all();
          } else {
#pragma unroll 1
            for (int c0 = 0; c0 < C::ACC_COLS; c0 += 16) {
              float v[16], sum[16];
              tmem_ld16(tacc + c0, v);
              if (sh > 0) {
                tmem_ld16(tsum + c0, sum);
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) sum[j] = 0.0f;
              }
#pragma unroll
              for (int j = 0; j < 16; ++j) sum[j] = bf16r(sum[j] + bf16r(v[j]));
              if (last)
                finish_row16<SWAP, BN>(a, sum, v, s, wt, mt, row, c0);   // bias once, rounded; stores
              else
                tmem_st16_wait(tsum + c0, sum);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(buf));
          ++nloc;
          continue;
        }
      }
      if constexpr (ARGMAX) {   // whole tiles only: the planner gives argmax plans no split
        argmax_tile<SWAP, BN>(a, tacc, s, wt, mt, row, q, lane);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(buf));
        ++nloc;
        continue;
      }
      const bool whole = (kb0 == 0 && kb1 == a.KI);
      bool finish = whole;
      long long tbeg = 0;
      int first = 0, nseg = 1;
      if (!whole) {
        // stream-K segment: park the fp32 partial, the last CTA of the tile reduces
        tbeg = static_cast<long long>(tile - a.dp_tiles) * a.KI;   // within the stream-K region
        first = sk_owner(tbeg, a.total_iters, gridDim.x);
        nseg = sk_owner(tbeg + a.KI - 1, a.total_iters, gridDim.x) - first + 1;
        float4* slot = reinterpret_cast<float4*>(
            a.ws_part + static_cast<size_t>(sk_slot(blockIdx.x, tbeg, a.total_iters, gridDim.x)) * C::SLOT_ELEMS);
        // slot layout: float4 groups [col/4][row][4] -> every float4 store / load of a
        // warp touches 512 contiguous bytes
#pragma unroll 1
        for (int c0 = 16 * half; c0 < C::ACC_COLS; c0 += 16 * (kEpiWarps / 4)) {
          float v[16];
          tmem_ld16(tacc + c0, v);
#pragma unroll
          for (int g = 0; g < 4; ++g)
            __stcg(slot + ((c0 >> 2) + g) * 128 + row, make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(buf));
        __threadfence();
        epi_bar();
        if (ep_tid == 0) {
          const int prev = atomicAdd(a.ws_cnt + tile, 1);
          *last_flag = (prev == nseg - 1) ? 1 : 0;
        }
        epi_bar();
        finish = (*last_flag != 0);
        if (finish) __threadfence();
      }
      if (finish) {
        // one pass over this warp's 16-column chunks: fetch (TMEM, or the sum of the
        // stream-K partials in K order), then bias, activation and stores from registers
#pragma unroll 1
        for (int c0 = 16 * half; c0 < ncols; c0 += 16 * (kEpiWarps / 4)) {
          float v[16], u[16];
          if (whole) {
            tmem_ld16(tacc + c0, v);
            if (gated) tmem_ld16(tacc + uoff + c0, u);
          } else {
            sk_sum16<C::SLOT_ELEMS>(a, v, row, c0, tbeg, first, nseg);
            if (gated) sk_sum16<C::SLOT_ELEMS>(a, u, row, c0 + uoff, tbeg, first, nseg);
          }
          finish_row16<SWAP, BN>(a, v, u, s, wt, mt, row, c0);
        }
      }
      if (whole) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(buf));
      } else {
        if (finish && ep_tid == 0) a.ws_cnt[tile] = 0;   // leave the counter zeroed for the next call
        epi_bar();   // last_flag is rewritten by the next segment
      }
      ++nloc;
    }
    // this warp no longer touches tensor memory: let warp 1 release it
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_done_bar);
  }
  // No CTA-wide barrier here: the roles ran on single lanes, and tensor memory
  // is released by warp 1 only after the epilogue warps signalled epi_done.
}

}  // namespace tps
