// tps_mlp_sk.cuh -- the gated MLP block at decode-sized m (at most 64 tokens) in ONE
// persistent launch that streams the weights on every SM in both layers.
//
// Same mathematics and the same readiness argument as tps_mlp_kernel ("张量并行
// （Tensor Parallelism）推理部署实战", §二; "Tensor Parallel：当一张 GPU 放不下一个大模型",
// section "MLP 里的 tensor parallel": the row layer's shard s reads only the column
// layer's shard s), but the work is split by stream-K instead of by tiles, so the
// weight stream is spread evenly over all CTAs (one per SM): at decode sizes the
// block reads its weights once and nothing else, and a layer whose tiles cover
// only some of the SMs (112 gate/up tile pairs at I = 14336, tp = 8) leaves the
// rest of the HBM bandwidth unused.
//
// Phase 1 (column layer, gate/up): the (tile, K block) iterations of all gate/up
//   tile pairs (weight-major: 128 gate + 128 up rows x 64 tokens, two
//   accumulators) are cut into one contiguous range per CTA. A tile whose K range
//   spans several CTAs is finished by the last of them to arrive (an atomic
//   counter per tile): each earlier CTA parks its fp32 partials in the workspace,
//   the last one sums them in K order (deterministic), applies SiLU(gate)*up,
//   stores h and makes a release increment of ready[token block][shard].
// Phase 2 (row layer, down): the same partition over the down tiles (128 weight
//   rows x 64 tokens, K over every shard's range in shard order); before loading a
//   K block of shard s the producer waits (bounded, acquire) until
//   ready[token block][s] counts every gate/up tile of that shard, then orders
//   its TMA reads after those stores with a proxy fence. The last CTA of a tile
//   sums the partials in K order -- the cross-shard reduction -- and stores Y.
// Phase 1 has no cross-CTA wait, so every gate/up tile is finished once every CTA
// has run its phase 1; the launch never has more CTAs than can be resident at
// once (one per SM), so a phase-2 wait never holds an SM another CTA's phase 1
// needs. Every wait is bounded all the same. The tile counters are left zero by
// their finishing CTA and the last CTA to finish re-zeroes ready[], so the
// workspace is zero between calls.
#pragma once

#include "tps_mlp.cuh"   // tps_gemm.cuh and the MLP kernels' wait limit

namespace tps {

constexpr int kSkBN = 64;                                 // tokens per tile (the MMA's N)
using SkC1 = GemmCfg<true, kSkBN, true, false>;           // gate/up tile pair: 256 weight rows
using SkC2 = GemmCfg<true, kSkBN, false, false>;          // down tile: 128 weight rows

struct MlpSkCfg {
  static constexpr int X_BYTES = SkC1::X_BYTES;           // 64 token rows x 64 K
  static constexpr int W_BYTES = SkC1::W_BYTES;           // the larger (phase 1) weight tile
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES_RAW = (SMEM_LIMIT - 1024 - BAR_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr int ACC_COLS = SkC1::ACC_COLS;         // gate + up accumulators (>= phase 2's)
  static constexpr int TMEM_COLS = 2 * ACC_COLS <= 128 ? 128 : 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + BAR_BYTES;
  static constexpr uint32_t IDESC = SkC1::IDESC;
  static_assert(SkC1::IDESC == SkC2::IDESC, "same MMA shape in both phases");
  static_assert(SkC1::X_BYTES == SkC2::X_BYTES, "same token tile in both phases");
  static_assert(2 * ACC_COLS <= 256, "two accumulator buffers");
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
};

// One stream-K segment of a phase in the epilogue (warps 2-5, thread = weight row):
// park the partial, or finish the tile (whole, or as the last CTA to arrive).
// Returns true when this CTA finished the tile (the caller publishes it).
template <bool DUAL>
__device__ __forceinline__ bool mlp_sk_segment(const GemmArgs& a, uint32_t tacc, uint32_t tempty, int tile, int kb0,
                                               int kb1, int row, int lane, int ep_tid, volatile int* last_flag) {
  using C = GemmCfg<true, kSkBN, DUAL, false>;
  int s, wt, mt;
  tile_coords(a, tile, s, wt, mt);
  const bool whole = (kb0 == 0 && kb1 == a.KI);
  bool finish = whole;
  long long tbeg = 0;
  int first = 0, nseg = 1;
  if (!whole) {
    tbeg = static_cast<long long>(tile - a.dp_tiles) * a.KI;
    first = sk_owner(tbeg, a.total_iters, gridDim.x);
    nseg = sk_owner(tbeg + a.KI - 1, a.total_iters, gridDim.x) - first + 1;
    float4* slot = reinterpret_cast<float4*>(
        a.ws_part + static_cast<size_t>(sk_slot(blockIdx.x, tbeg, a.total_iters, gridDim.x)) * C::SLOT_ELEMS);
#pragma unroll 1
    for (int c0 = 0; c0 < C::ACC_COLS; c0 += 16) {
      float v[16];
      tmem_ld16(tacc + c0, v);
#pragma unroll
      for (int g = 0; g < 4; ++g)
        __stcg(slot + ((c0 >> 2) + g) * 128 + row, make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]));
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tempty);
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
#pragma unroll 1
    for (int c0 = 0; c0 < kSkBN; c0 += 16) {
      float v[16], u[16];
      if (whole) {
        tmem_ld16(tacc + c0, v);
        if (DUAL) tmem_ld16(tacc + kSkBN + c0, u);
      } else {
        sk_sum16<C::SLOT_ELEMS>(a, v, row, c0, tbeg, first, nseg);
        if (DUAL) sk_sum16<C::SLOT_ELEMS>(a, u, row, c0 + kSkBN, tbeg, first, nseg);
      }
      finish_row16<true, kSkBN, false>(a, v, u, s, wt, mt, row, c0);
    }
  }
  if (whole) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(tempty);
  } else {
    if (finish && ep_tid == 0) a.ws_cnt[tile] = 0;   // leave the counter zeroed for the next call
    epi_bar();                                       // last_flag is rewritten by the next segment
  }
  return finish;
}

__global__ void __launch_bounds__(kThreads, 1)
    tps_mlp_sk_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                      const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW2,
                      const GemmArgs a1, const GemmArgs a2, const MlpSync sy) {
  using M = MlpSkCfg;
  constexpr int STAGES = M::STAGES;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sX = base;
  const uint32_t sW = base + STAGES * M::X_BYTES;
  const uint32_t sBar = base + STAGES * M::STAGE_BYTES;
  uint8_t* gBar = gbase + STAGES * M::STAGE_BYTES;
  auto full_bar = [&](int i) { return sBar + 8u * i; };
  auto empty_bar = [&](int i) { return sBar + 8u * (STAGES + i); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * STAGES + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * STAGES + 2 + i); };
  const uint32_t done_bar = sBar + 8u * (2 * STAGES + 4);
  const uint32_t epi_done_bar = sBar + 8u * (2 * STAGES + 5);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 6));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 6) + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 6) + 8);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 6) + 12);

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
    *abort_flag = 0;
    *last_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), M::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = a1.timeout_ns;
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      griddep_wait();
      SegIter seg;
      int tile, kb0, kb1;
      seg.init(a1);
      while (ok && seg.next(a1, tile, kb0, kb1)) {
        int s, wt, mt;
        tile_coords(a1, tile, s, wt, mt);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait<kMlpSuspendNs>(empty_bar(stage), phase ^ 1u, abort_flag, tmo, a1.status)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), SkC1::STAGE_BYTES);
          tma_load_3d(sX + stage * M::X_BYTES, &tmX, full_bar(stage), kb * 64, mt * kSkBN, 0);
#pragma unroll
          for (int j = 0; j < SkC1::NWB; ++j) {
            const int row0 = wt * SkC1::WR + j * SkC1::WBOX;
            tma_load_4d(sW + stage * M::W_BYTES + j * SkC1::WBOX * 128, &tmW1, full_bar(stage), 0, row0 & 127, kb,
                        s * a1.RB + (row0 >> 7));
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      seg.init(a2);
      while (ok && seg.next(a2, tile, kb0, kb1)) {
        int s2, wt2, mt2;
        tile_coords(a2, tile, s2, wt2, mt2);
        int ready_shard = -1;
        for (int kb = kb0; kb < kb1; ++kb) {
          const int ks = kb / a2.KBs;   // shard of this K block
          const int kk = kb - ks * a2.KBs;
          if (ks != ready_shard) {
            // every gate/up tile of (token block mt2, shard ks) has stored its h columns
            if (!wait_count_geq(sy.ready + mt2 * a2.tp + ks, sy.need, abort_flag, tmo, a1.status)) {
              ok = false;
              break;
            }
            fence_proxy_async_global();
            ready_shard = ks;
          }
          if (!mbar_wait<kMlpSuspendNs>(empty_bar(stage), phase ^ 1u, abort_flag, tmo, a1.status)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), SkC2::STAGE_BYTES);
          if (a2.x_sharded)
            tma_load_3d(sX + stage * M::X_BYTES, &tmH, full_bar(stage), kk * 64, ks, mt2 * kSkBN);
          else
            tma_load_3d(sX + stage * M::X_BYTES, &tmH, full_bar(stage), ks * a2.x_shard_cols + kk * 64, mt2 * kSkBN,
                        0);
          tma_load_4d(sW + stage * M::W_BYTES, &tmW2, full_bar(stage), 0, 0, kk, ks * a2.RB + wt2);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // wait (bounded) for the copies still in flight before the CTA may exit
      const long long first = issued > STAGES ? issued - STAGES : 0;
      for (long long i = first; i < issued; ++i)
        mbar_wait<kMlpSuspendNs>(full_bar(static_cast<int>(i % STAGES)), static_cast<uint32_t>((i / STAGES) & 1), never_flag,
                  200000000ull, a1.status);
      // This CTA reads no flag any more. The last CTA to get here re-zeroes them:
      // each was read at its full count by some CTA, so all increments are done.
      if (ok) {
        __threadfence();
        if (atomicAdd(sy.done, 1) == static_cast<int>(gridDim.x) - 1) {
          for (int i = 0; i < sy.n_ready; ++i) sy.ready[i] = 0;
          *sy.done = 0;
          __threadfence();
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int nloc = 0;
      bool ok = true;
      bool any = false;
#pragma unroll 1
      for (int ph = 0; ok && ph < 2; ++ph) {
        const GemmArgs& a = ph == 0 ? a1 : a2;
        const bool dual = (ph == 0);
        SegIter seg;
        seg.init(a);
        int tile, kb0, kb1;
        while (ok && seg.next(a, tile, kb0, kb1)) {
          const int buf = nloc & 1;
          const uint32_t use = static_cast<uint32_t>(nloc >> 1);
          if (!mbar_wait<kMlpSuspendNs>(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag, tmo, a1.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * M::ACC_COLS);
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait<kMlpSuspendNs>(full_bar(stage), phase, abort_flag, tmo, a1.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t wa = sW + stage * M::W_BYTES;
            const uint64_t dx = smem_desc_sw128(sX + stage * M::X_BYTES);
            const uint64_t dw = smem_desc_sw128(wa);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
              const uint64_t koff = static_cast<uint64_t>(kk * 2);
              umma_bf16(d0, dw + koff, dx + koff, M::IDESC, acc);
              if (dual) {
                const uint64_t dw2 = smem_desc_sw128(wa + 128 * 128);   // up rows 128..255 of the pair
                umma_bf16(d0 + kSkBN, dw2 + koff, dx + koff, M::IDESC, acc);
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
      }
      if (any) {
        umma_commit(done_bar);
        mbar_wait<kMlpSuspendNs>(done_bar, 0, never_flag, 200000000ull, a1.status);
      }
      mbar_wait<kMlpSuspendNs>(epi_done_bar, 0, never_flag, tmo, a1.status);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, M::TMEM_COLS);
  } else {
    // -------------------------------------------------------------- epilogue (warps 2-5)
    const int q = warp & 3;
    const int row = q * 32 + lane;          // accumulator row = weight row of the tile
    const int ep_tid = threadIdx.x - 64;
    int nloc = 0;
    bool failed = false;
#pragma unroll 1
    for (int ph = 0; !failed && ph < 2; ++ph) {
      const GemmArgs& a = ph == 0 ? a1 : a2;
      SegIter seg;
      seg.init(a);
      int tile, kb0, kb1;
      while (seg.next(a, tile, kb0, kb1)) {
        const int buf = nloc & 1;
        const uint32_t use = static_cast<uint32_t>(nloc >> 1);
        const bool ok = mbar_wait<kMlpSuspendNs>(tfull_bar(buf), use & 1u, abort_flag, tmo, a1.status);
        if (epi_bar_or(!ok)) { failed = true; break; }   // all epilogue threads leave together
        tc_fence_after();
        const uint32_t tacc =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * M::ACC_COLS);
        if (ph == 0) {
          if (mlp_sk_segment<true>(a, tacc, tempty_bar(buf), tile, kb0, kb1, row, lane, ep_tid, last_flag)) {
            // publish the finished gate/up tile: every epilogue thread's h stores, then
            // one release increment of its (token block, shard) flag
            int s, wt, mt;
            tile_coords(a, tile, s, wt, mt);
            epi_bar();
            if (ep_tid == 0) {
              fence_proxy_async_global();
              red_release_gpu_add(sy.ready + mt * a.tp + s, 1);
            }
          }
        } else {
          mlp_sk_segment<false>(a, tacc, tempty_bar(buf), tile, kb0, kb1, row, lane, ep_tid, last_flag);
        }
        ++nloc;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_done_bar);
  }
}

}  // namespace tps
