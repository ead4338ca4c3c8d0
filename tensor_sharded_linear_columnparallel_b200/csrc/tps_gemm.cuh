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
//     the result is deterministic) and runs the epilogue. With the PARTIALS
//     reduction every tile is one (shard, output tile) pair and P_s is stored to
//     `partials[s]` for the standalone reduce kernel.
//
// Hardware mapping (one CTA per SM, 6 warps):
//   warp 0   TMA producer: 128B-swizzled K-major tiles of X and W into a ring of
//            shared-memory stages, completion tracked by mbarriers (no multicast).
//   warp 1   tcgen05 MMA issuer (one thread), cta_group::1, M = 128, N = BN,
//            K = 16 per instruction, fp32 accumulators in tensor memory, two
//            accumulator buffers so the epilogue of one tile overlaps the main
//            loop of the next; warp 1 also allocates / frees tensor memory.
//   warps 2-5 epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//            32*(w%4) .. +31), bias, activation (GELU, or SiLU(gate)*up), bf16 or
//            fp32 stores, stream-K fix-up.
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

__device__ __forceinline__ float gelu_erf(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }
__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }

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
  const int wtt = a.S_tiles * a.WT;
  const int span = a.gm * wtt;
  const int g = t / span;
  const int r = t - g * span;
  const int m_first = g * a.gm;
  const int gsz = min(a.gm, a.MT - m_first);
  mt = m_first + r % gsz;
  const int wc = r / gsz;
  s = wc / a.WT;
  wt = wc - s * a.WT;
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

// Iterates the (tile, k_begin, k_end) segments of this CTA, identically in every role.
struct SegIter {
  long long it, it_end;  // stream-K
  int t;                 // data-parallel
  __device__ __forceinline__ void init(const GemmArgs& a) {
    if (a.sk) {
      const long long T = a.total_iters;
      const int C = gridDim.x;
      it = (static_cast<long long>(blockIdx.x) * T) / C;
      it_end = (static_cast<long long>(blockIdx.x + 1) * T) / C;
    } else {
      t = blockIdx.x;
    }
  }
  __device__ __forceinline__ bool next(const GemmArgs& a, int& tile, int& kb0, int& kb1) {
    if (a.sk) {
      if (it >= it_end) return false;
      tile = static_cast<int>(it / a.KI);
      kb0 = static_cast<int>(it - static_cast<long long>(tile) * a.KI);
      const long long rem = it_end - it;
      kb1 = static_cast<int>(min(static_cast<long long>(a.KI), kb0 + rem));
      it += kb1 - kb0;
      return true;
    }
    if (t >= a.tiles) return false;
    tile = t;
    kb0 = 0;
    kb1 = a.KI;
    t += gridDim.x;
    return true;
  }
};

__device__ __forceinline__ bool epi_bar_or(bool v) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return out != 0;
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <bool SWAP, int BN, bool DUAL>
struct GemmCfg {
  static constexpr int XR = SWAP ? BN : 128;                   // token rows per tile
  static constexpr int WR = SWAP ? (DUAL ? 256 : 128) : BN;    // weight rows per tile
  static constexpr int X_BYTES = XR * 128;
  static constexpr int W_BYTES = WR * 128;
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  static constexpr int STAGES_RAW = (220 * 1024) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr int ACC_COLS = BN * (DUAL ? 2 : 1);
  static constexpr int TMEM_NEED = 2 * ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                                                : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int CH = BN >= 32 ? 32 : 16;                // epilogue column chunk
  static constexpr int SLOT_ELEMS = 128 * ACC_COLS;            // fp32 per stream-K segment slot
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + BAR_BYTES;
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, BN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
  static_assert(!DUAL || SWAP, "dual A tiles only in weight-major tiles");
  static_assert(X_BYTES % 1024 == 0 && W_BYTES % 1024 == 0, "SW128 tiles are 1024-B aligned");
  static_assert(STAGES >= 2, "pipeline depth");
};

// ---------------------------------------------------------------- epilogue store
// Writes CH consecutive accumulator columns of one accumulator row. `v` holds the
// (first) accumulator, `u` the up accumulator for gate-up (token-major: columns
// +128 of the same tile; weight-major DUAL: the second accumulator).
template <bool SWAP, int BN, bool DUAL, int CH>
__device__ __forceinline__ void store_chunk(const GemmArgs& a, int s, int wt, int mt, int row, int c0,
                                            const float* v, const float* u) {
  const bool gated = (a.act == A_SILU_MUL);
  if (a.out_mode == OUT_PARTIALS) {
    // P_s of a row-parallel tile, fp32, no bias: partials[s][token][w]
    float* P = a.partials + static_cast<size_t>(s) * a.M * a.per_shard;
    if (!SWAP) {
      const int tok = mt * 128 + row;
      if (tok >= a.M) return;
      const int w0 = wt * BN + c0;
      float* dst = P + static_cast<size_t>(tok) * a.per_shard + w0;
      if (w0 + CH <= a.per_shard && (a.per_shard % 4) == 0) {
#pragma unroll
        for (int j = 0; j < CH; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < CH; ++j)
          if (w0 + j < a.per_shard) dst[j] = v[j];
      }
    } else {
      const int w = wt * 128 + row;
      if (w >= a.per_shard) return;
#pragma unroll
      for (int j = 0; j < CH; ++j) {
        const int tok = mt * BN + c0 + j;
        if (tok < a.M) P[static_cast<size_t>(tok) * a.per_shard + w] = v[j];
      }
    }
    return;
  }

  if (!SWAP) {
    const int tok = mt * 128 + row;
    if (tok >= a.M) return;
    // weight-row (or gate-up feature) index of column c0 within the shard
    const int w0 = gated ? (wt * 128 + c0) : (wt * BN + c0);
    float o[CH];
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      float x = v[j];
      const int w = w0 + j;
      if (gated) {
        float y = u[j];
        if (a.bias != nullptr && w < a.per_shard) {
          x += __bfloat162float(static_cast<const __nv_bfloat16*>(a.bias)[s * a.per_shard + w]);
          y += __bfloat162float(static_cast<const __nv_bfloat16*>(a.bias)[a.gate_off + s * a.per_shard + w]);
        }
        x = silu_f(x) * y;
      } else {
        if (a.bias != nullptr && w < a.per_shard) x += __bfloat162float(static_cast<const __nv_bfloat16*>(a.bias)[logical_col(a, s, w)]);
        if (a.act == A_GELU) x = gelu_erf(x);
      }
      o[j] = x;
    }
    const int col0 = (a.kind == K_ROW) ? w0 : s * a.per_shard + w0;
    const bool full = (w0 + CH <= a.per_shard);
    if (a.y_f32) {
      float* dst = reinterpret_cast<float*>(a.Y) + static_cast<size_t>(tok) * a.ldy + col0;
      if (full && (col0 % 4) == 0 && (a.ldy % 4) == 0) {
#pragma unroll
        for (int j = 0; j < CH; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
      } else {
#pragma unroll
        for (int j = 0; j < CH; ++j)
          if (w0 + j < a.per_shard) dst[j] = o[j];
      }
    } else {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(a.Y) + static_cast<size_t>(tok) * a.ldy + col0;
      if (full && (col0 % 8) == 0 && (a.ldy % 8) == 0) {
#pragma unroll
        for (int j = 0; j < CH; j += 8) {
          uint4 pk;
          __nv_bfloat162 b0 = __floats2bfloat162_rn(o[j + 0], o[j + 1]);
          __nv_bfloat162 b1 = __floats2bfloat162_rn(o[j + 2], o[j + 3]);
          __nv_bfloat162 b2 = __floats2bfloat162_rn(o[j + 4], o[j + 5]);
          __nv_bfloat162 b3 = __floats2bfloat162_rn(o[j + 6], o[j + 7]);
          pk.x = *reinterpret_cast<uint32_t*>(&b0);
          pk.y = *reinterpret_cast<uint32_t*>(&b1);
          pk.z = *reinterpret_cast<uint32_t*>(&b2);
          pk.w = *reinterpret_cast<uint32_t*>(&b3);
          *reinterpret_cast<uint4*>(dst + j) = pk;
        }
      } else {
#pragma unroll
        for (int j = 0; j < CH; ++j)
          if (w0 + j < a.per_shard) dst[j] = __float2bfloat16_rn(o[j]);
      }
    }
  } else {
    // weight-major tile: this thread owns one weight row (or gate-up feature) and
    // CH consecutive tokens; consecutive lanes write consecutive output columns.
    const int w = wt * 128 + row;
    if (w >= a.per_shard) return;
    float bx = 0.f, by = 0.f;
    if (a.bias != nullptr) {
      if (gated) {
        bx = __bfloat162float(static_cast<const __nv_bfloat16*>(a.bias)[s * a.per_shard + w]);
        by = __bfloat162float(static_cast<const __nv_bfloat16*>(a.bias)[a.gate_off + s * a.per_shard + w]);
      } else {
        bx = __bfloat162float(static_cast<const __nv_bfloat16*>(a.bias)[logical_col(a, s, w)]);
      }
    }
    const int col = (a.kind == K_ROW) ? w : s * a.per_shard + w;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
      const int tok = mt * BN + c0 + j;
      if (tok >= a.M) break;
      float x = v[j] + bx;
      if (gated) {
        x = silu_f(x) * (u[j] + by);
      } else if (a.act == A_GELU) {
        x = gelu_erf(x);
      }
      if (a.y_f32)
        reinterpret_cast<float*>(a.Y)[static_cast<size_t>(tok) * a.ldy + col] = x;
      else
        reinterpret_cast<__nv_bfloat16*>(a.Y)[static_cast<size_t>(tok) * a.ldy + col] = __float2bfloat16_rn(x);
    }
  }
}

template <int CH>
__device__ __forceinline__ void tmem_ld_chunk(uint32_t taddr, float (&v)[CH]) {
  if constexpr (CH == 32) tmem_ld32(taddr, v);
  else tmem_ld16(taddr, v);
}

// ---------------------------------------------------------------- the kernel
template <bool SWAP, int BN, bool DUAL>
__global__ void __launch_bounds__(192, 1)
    tps_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const GemmArgs a) {
  using C = GemmCfg<SWAP, BN, DUAL>;
  constexpr int STAGES = C::STAGES;
  constexpr int CH = C::CH;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sX = base;                               // STAGES x X tiles
  const uint32_t sW = base + STAGES * C::X_BYTES;         // STAGES x W tiles
  const uint32_t sBar = base + STAGES * C::STAGE_BYTES;   // barriers
  uint8_t* gBar = gbase + STAGES * C::STAGE_BYTES;
  // barrier map: full[STAGES], empty[STAGES], tfull[2], tempty[2], done
  auto full_bar = [&](int i) { return sBar + 8u * i; };
  auto empty_bar = [&](int i) { return sBar + 8u * (STAGES + i); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * STAGES + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * STAGES + 2 + i); };
  const uint32_t done_bar = sBar + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 5) + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 5) + 8);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 5) + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 4);
    }
    mbar_init(done_bar, 1);
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
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;

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
      while (ok && seg.next(a, tile, kb0, kb1)) {
        int s, wt, mt;
        tile_coords(a, tile, s, wt, mt);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const int ks = a.k_spans_shards ? kb / a.KBs : s;      // shard of this K block
          const int kk = a.k_spans_shards ? kb - ks * a.KBs : kb;
          mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
          const int xrow = mt * C::XR;
          if (a.x_sharded)
            tma_load_3d(sX + stage * C::X_BYTES, &tmX, full_bar(stage), kk * 64, ks, xrow);
          else
            tma_load_3d(sX + stage * C::X_BYTES, &tmX, full_bar(stage), kk * 64, xrow, 0);
          tma_load_3d(sW + stage * C::W_BYTES, &tmW, full_bar(stage), kk * 64, wt * C::WR, ks);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // wait (bounded) for the copies still in flight before the CTA may exit
      const long long first = issued > STAGES ? issued - STAGES : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait(full_bar(static_cast<int>(i % STAGES)), static_cast<uint32_t>((i / STAGES) & 1), never_flag,
                  200000000ull);
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
        if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * C::ACC_COLS);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, tmo)) { ok = false; break; }
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
        mbar_wait(done_bar, 0, never_flag, 200000000ull);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane sub-partition of this warp
    const int row = q * 32 + lane;          // accumulator row (TMEM lane)
    const int ep_tid = threadIdx.x - 64;
    SegIter seg;
    seg.init(a);
    int tile, kb0, kb1;
    int nloc = 0;
    while (seg.next(a, tile, kb0, kb1)) {
      const int buf = nloc & 1;
      const uint32_t use = static_cast<uint32_t>(nloc >> 1);
      const bool ok = mbar_wait(tfull_bar(buf), use & 1u, abort_flag, tmo);
      if (epi_bar_or(!ok)) break;            // all 128 epilogue threads leave together
      tc_fence_after();
      int s, wt, mt;
      tile_coords(a, tile, s, wt, mt);
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * C::ACC_COLS);
      const bool whole = !a.sk || (kb0 == 0 && kb1 == a.KI);
      if (whole) {
        const bool gated_tm = (!SWAP && a.act == A_SILU_MUL);
        const int ncols = gated_tm ? BN / 2 : BN;
#pragma unroll 1
        for (int c0 = 0; c0 < ncols; c0 += CH) {
          float v[CH];
          float u[CH];
          tmem_ld_chunk<CH>(tacc + c0, v);
          if (gated_tm) tmem_ld_chunk<CH>(tacc + BN / 2 + c0, u);
          if (DUAL) tmem_ld_chunk<CH>(tacc + BN + c0, u);
          store_chunk<SWAP, BN, DUAL, CH>(a, s, wt, mt, row, c0, v, u);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(buf));
      } else {
        // stream-K segment: park the fp32 partial, the last CTA of the tile reduces
        const long long tbeg = static_cast<long long>(tile) * a.KI;
        const int first = sk_owner(tbeg, a.total_iters, gridDim.x);
        const int last = sk_owner(tbeg + a.KI - 1, a.total_iters, gridDim.x);
        const int nseg = last - first + 1;
        float* slot = a.ws_part + static_cast<size_t>(sk_slot(blockIdx.x, tbeg, a.total_iters, gridDim.x)) * C::SLOT_ELEMS;
#pragma unroll 1
        for (int c0 = 0; c0 < C::ACC_COLS; c0 += CH) {
          float v[CH];
          tmem_ld_chunk<CH>(tacc + c0, v);
#pragma unroll
          for (int j = 0; j < CH; ++j) __stcg(slot + static_cast<size_t>(c0 + j) * 128 + row, v[j]);
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
        if (*last_flag) {
          __threadfence();
          const bool gated_tm = (!SWAP && a.act == A_SILU_MUL);
          const int ncols = gated_tm ? BN / 2 : BN;
#pragma unroll 1
          for (int c0 = 0; c0 < ncols; c0 += CH) {
            float v[CH];
            float u[CH];
#pragma unroll
            for (int j = 0; j < CH; ++j) { v[j] = 0.f; u[j] = 0.f; }
            for (int g = 0; g < nseg; ++g) {   // K order: CTA first, first+1, ..., last
              const float* sl =
                  a.ws_part + static_cast<size_t>(sk_slot(first + g, tbeg, a.total_iters, gridDim.x)) * C::SLOT_ELEMS;
#pragma unroll
              for (int j = 0; j < CH; ++j) {
                v[j] += __ldcg(sl + static_cast<size_t>(c0 + j) * 128 + row);
                if (gated_tm) u[j] += __ldcg(sl + static_cast<size_t>(BN / 2 + c0 + j) * 128 + row);
                if (DUAL) u[j] += __ldcg(sl + static_cast<size_t>(BN + c0 + j) * 128 + row);
              }
            }
            store_chunk<SWAP, BN, DUAL, CH>(a, s, wt, mt, row, c0, v, u);
          }
          if (ep_tid == 0) a.ws_cnt[tile] = 0;   // leave the counter zeroed for the next call
        }
        epi_bar();   // last_flag is rewritten by the next segment
      }
      ++nloc;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace tps
