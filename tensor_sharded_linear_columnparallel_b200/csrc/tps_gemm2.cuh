// tps_gemm2.cuh -- token-major sharded GEMM on CTA pairs (tcgen05 cta_group::2).
//
// Same tile space, K walk (over the shards for row-parallel) and epilogue as
// tps_gemm_kernel, but a tile is 256 tokens x BN weight rows computed by a pair
// of CTAs on two SMs of one cluster: each CTA loads its own 128 token rows of X
// and its own BN/2 weight rows into its shared memory (plain TMA loads, no
// multicast), the pair leader issues one M=256 tcgen05.mma.cta_group::2 per K
// step that reads both CTAs' shared memory, and each CTA's tensor memory holds
// its 128 accumulator rows. Per SM and 64-wide K block this moves 128 + BN/2 tile
// rows instead of 128 + BN, which is what limits the single-CTA tile.
//
// Wide tiles (NH = 2): a tile is 256 tokens x 2*BN weight rows, two MMAs of N = BN
// per K step on the same token tile, so per SM and K block the tile moves 128 +
// BN rows for twice the MMA work of an NH = 1 tile (a quarter fewer bytes per
// FLOP at BN = 256). The two accumulators fill the 512 tensor-memory columns, so
// there is one accumulator buffer: the next tile's MMAs wait for the epilogue.
//
// Barriers: full[s] lives in the leader (both CTAs' copies count bytes on it);
// empty[s] and tmem_full[b] live in both CTAs and are signalled by the leader's
// multicast commit; tmem_empty[b] lives in the leader and both CTAs' epilogue
// warps arrive on it. Data-parallel tiles only (no stream-K).
#pragma once

#include "tps_gemm.cuh"

namespace tps {

// Two epilogue warps per tensor-memory lane sub-partition: warps w and w+4 read
// the same 32 accumulator rows and take alternate 16-column chunks, so two warps
// per SM sub-partition hide each other's load and activation latency.
constexpr int kEpi2Warps = 8;
constexpr int kThreads2 = 64 + 32 * kEpi2Warps;

template <int BN, int NH = 1>
struct Gemm2Cfg {
  static constexpr int BH = BN / 2;                            // weight rows of one MMA half held by each CTA
  static constexpr int WBOX = BH < 128 ? BH : 128;
  static constexpr int NWB = BH / WBOX;
  static constexpr int A_BYTES = 128 * 128;                    // 128 token rows x 64 K
  static constexpr int BH_BYTES = BH * 128;                    // one N half's weight rows of this CTA
  static constexpr int B_BYTES = NH * BH_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STG_BYTES = 0;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES_RAW = (SMEM_LIMIT - 1024 - BAR_BYTES - STG_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr int ACC_COLS = NH * BN;                     // one tile's accumulators
  static constexpr int NBUF = NH == 1 ? 2 : 1;                 // accumulator buffers
  static constexpr int TMEM_NEED = NBUF * ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STG_BYTES + 1024 + BAR_BYTES;
  static constexpr uint32_t IDESC = idesc_bf16_f32(256, BN);
  static_assert(BN == 128 || BN == 256, "pair tiles are 256 x 128 or 256 x 256 per MMA");
  static_assert(NH == 1 || NH == 2, "one or two MMA halves per tile");
  static_assert(TMEM_NEED <= 512, "tensor memory columns");
  static_assert(BH_BYTES % 1024 == 0, "SW128 tiles are 1024-B aligned");
  static_assert(STAGES >= 3, "pipeline depth");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
};

template <int BN, int NH = 1>
__global__ void __launch_bounds__(kThreads2, 1)
    tps_gemm2_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const GemmArgs a) {
  using C = Gemm2Cfg<BN, NH>;
  constexpr int STAGES = C::STAGES;
  if (!cluster_size_is(2u, a.status)) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sA = base;
  const uint32_t sB = base + STAGES * C::A_BYTES;
  const uint32_t sBar = base + STAGES * C::STAGE_BYTES + C::STG_BYTES;
  uint8_t* gBar = gbase + STAGES * C::STAGE_BYTES + C::STG_BYTES;
  auto full_bar = [&](int i) { return sBar + 8u * i; };
  auto empty_bar = [&](int i) { return sBar + 8u * (STAGES + i); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * STAGES + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * STAGES + 2 + i); };
  const uint32_t done_bar = sBar + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 6));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 6) + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 6) + 12);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0 = leader (issues the MMA), 1 = peer
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 2 * kEpi2Warps);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  cluster_sync_all();          // both CTAs' barriers initialised and tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;
  // Programmatic dependent launch: as in tps_gemm_kernel, the wait for the
  // previous kernel is in the producer, before its first load.
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // L2 policies: the token rows of a raster group are read again by every weight
      // tile of the group's sweep, a weight tile only by the group's token tiles in
      // the same wave (GemmArgs::l2_hint)
      const uint64_t pol_x = (a.l2_hint & 1) ? l2_policy_evict_last() : l2_policy_evict_normal();
      const uint64_t pol_w = (a.l2_hint & 2) ? l2_policy_evict_first() : l2_policy_evict_normal();
      griddep_wait();
      for (int tile = pair; ok && tile < a.tiles; tile += npairs) {
        int s, wt, mt;
        tile_coords(a, tile, s, wt, mt);
        for (int kb = 0; kb < a.KI; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
          const int ks = a.k_spans_shards ? kb / a.KBs : s;
          const int kk = a.k_spans_shards ? kb - ks * a.KBs : kb;
          const uint32_t fb = mapa_shared(full_bar(stage), 0);
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
          const int xrow = mt * 256 + static_cast<int>(rank) * 128;
          if (a.x_sharded)
            tma2_load_3d_hint(sA + stage * C::A_BYTES, &tmX, fb, kk * 64, ks, xrow, pol_x);
          else
            tma2_load_3d_hint(sA + stage * C::A_BYTES, &tmX, fb, ks * a.x_shard_cols + kk * 64, xrow, 0, pol_x);
#pragma unroll
          for (int h = 0; h < NH; ++h) {
#pragma unroll
            for (int j = 0; j < C::NWB; ++j) {
              const int row0 = (wt * NH + h) * BN + static_cast<int>(rank) * C::BH + j * C::WBOX;
              tma2_load_4d_hint(sB + stage * C::B_BYTES + h * C::BH_BYTES + j * C::WBOX * 128, &tmW, fb, 0,
                                row0 & 127, kk, ks * a.RB + (row0 >> 7), pol_w);
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader only)
      int stage = 0;
      uint32_t phase = 0;
      int nloc = 0;
      bool ok = true;
      bool any = false;
      for (int tile = pair; ok && tile < a.tiles; tile += npairs) {
        const int buf = nloc % C::NBUF;
        const uint32_t use = static_cast<uint32_t>(nloc / C::NBUF);
        if (!mbar_wait(tempty_bar(buf), (use & 1u) ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + static_cast<uint32_t>(buf * C::ACC_COLS);
        for (int kb = 0; kb < a.KI; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, tmo, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(sA + stage * C::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t koff = static_cast<uint64_t>(kk * 2);
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              const uint64_t db = smem_desc_sw128(sB + stage * C::B_BYTES + h * C::BH_BYTES);
              umma2_bf16(d0 + h * BN, da + koff, db + koff, C::IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma2_commit_mc(empty_bar(stage), 0x3);
          any = true;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_mc(tfull_bar(buf), 0x3);
        ++nloc;
      }
      if (any) {
        umma2_commit_mc(done_bar, 0x1);
        mbar_wait(done_bar, 0, never_flag, 200000000ull, a.status);
      }
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;                 // tensor-memory lane sub-partition of this warp
    const int half = (warp - 2) >> 2;       // chunks c0 = 16 * (2k + half)
    const int row = q * 32 + lane;
    const bool gated = (a.act == A_SILU_MUL);
    const int ncols = gated ? BN / 2 : BN;
    int nloc = 0;
    for (int tile = pair; tile < a.tiles; tile += npairs) {
      const int buf = nloc % C::NBUF;
      const uint32_t use = static_cast<uint32_t>(nloc / C::NBUF);
      const bool ok = mbar_wait(tfull_bar(buf), use & 1u, abort_flag, tmo, a.status);
      if (epi_bar_or<32 * kEpi2Warps>(!ok)) break;
      tc_fence_after();
      int s, wt, mt;
      tile_coords(a, tile, s, wt, mt);
      const int mt128 = mt * 2 + static_cast<int>(rank);   // this CTA's 128 token rows
#pragma unroll 1
      for (int h = 0; h < NH; ++h) {
        // MMA half h is the BN-row weight tile wt * NH + h
        const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                              static_cast<uint32_t>(buf * C::ACC_COLS + h * BN);
#pragma unroll 1
        for (int c0 = 16 * half; c0 < ncols; c0 += 32) {
          float v[16], u[16];
          tmem_ld16(tacc + c0, v);
          if (gated) tmem_ld16(tacc + BN / 2 + c0, u);
          finish_row16<false, BN>(a, v, u, s, wt * NH + h, mt128, row, c0);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(buf), 0));
      ++nloc;
    }
  }

  // Every role has finished (all MMAs completed before the last tmem_full), so no
  // CTA touches the other's shared or tensor memory any more.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace tps
