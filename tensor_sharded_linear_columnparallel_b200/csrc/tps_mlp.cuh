// tps_mlp.cuh -- an MLP block (column-parallel fc1 or gate/up with its fused
// activation, row-parallel fc2 / down with the cross-shard reduction) in ONE
// persistent launch.
//
// "张量并行（Tensor Parallelism）推理部署实战", §二 (Megatron MLP) and "Tensor
// Parallel：当一张 GPU 放不下一个大模型", section "MLP 里的 tensor parallel": the
// column layer's shard s produces h_s = act(X W_s) and the row layer's shard s
// consumes only h_s, so no exchange is needed between the two GEMMs -- only the
// row layer's partial sums meet. That is what lets the row GEMM start on a shard
// as soon as that shard's column tiles are written, without waiting for the
// whole layer.
//
// Phase 1 (every CTA): column tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
//   (whole K); the epilogue applies the activation (GELU, or SiLU(gate)*up with
//   the gate and up accumulators of a DUAL weight-major tile), stores h (bf16)
//   and, after a barrier over the epilogue warps, one thread makes a release
//   increment of ready[token block][shard].
// Phase 2 (a cluster of cs CTAs per row tile): the cluster split-K of
//   tps_gemm_kernel<SWAP, BN, false, true>. Before the producer loads a K block
//   of shard s it waits (bounded, acquire) until ready[token block][s] counts
//   every column tile of that shard, then orders its TMA reads after those
//   stores with a proxy fence.
// Both phases share the stage ring (sized for the larger stage), the barriers
//   and the two tensor-memory accumulators (phase 2 uses the buffer after phase
//   1's last one, so its main loop overlaps phase 1's epilogue). The grid never
//   exceeds the clusters the occupancy API reports resident at once (one CTA per
//   SM), so every CTA whose column tile a wait needs is running; every wait is
//   bounded all the same. The last CTA to finish re-zeroes ready[] -- every
//   increment and every read of it is done by then -- so the flags are zero
//   between calls.
//
// Orientations: SWAP = false (tokens on the MMA M side; prefill-sized m, GELU)
// and SWAP = true with DUAL1 (weight rows on the M side, gate and up blocks of
// 128 rows each; decode-sized m, SiLU(gate)*up).
#pragma once

#include "tps_gemm.cuh"

namespace tps {

// Eight epilogue warps: two per tensor-memory lane quarter. In phase 1 warps w
// and w+4 take the two 64-column halves of a token-major tile (alternate
// 16-column chunks of a weight-major one); the cluster split of phase 2 runs on
// all eight (two threads per accumulator row, each pushing half of its columns).
constexpr int kEpiMWarps = 8;
// Suspend limit of the one-launch MLP kernels' mbarrier waits: their producer and
// MMA threads wait long (on readiness flags, on the other layer) next to the
// epilogue warps of their sub-partitions. Measured with the L2 flushed: GELU MLP
// 36.7 -> 35.8 us, gated decode 73.7 -> 72.6 us (the same limit made the attention
// and the greedy lm_head GEMM about 1% slower, so those keep the system's own).
constexpr uint32_t kMlpSuspendNs = 20000;
constexpr int kThreadsM = 64 + 32 * kEpiMWarps;

template <bool SWAP, int BN, bool DUAL1>
struct MlpCfg {
  using C1 = GemmCfg<SWAP, BN, DUAL1, false>;   // phase 1 tile shapes
  using C2 = GemmCfg<SWAP, BN, false, true>;    // phase 2 tile shapes and partial buffer
  static constexpr int X_BYTES = C1::X_BYTES;   // same token rows in both phases
  static_assert(C1::X_BYTES == C2::X_BYTES, "token tile");
  static constexpr int W_BYTES = C1::W_BYTES > C2::W_BYTES ? C1::W_BYTES : C2::W_BYTES;
  static constexpr int STAGE_BYTES = X_BYTES + W_BYTES;
  static constexpr int P_BYTES = C2::P_BYTES;
  // token-major phase-1 epilogue staging: 4 KB per epilogue warp (32 rows x 128 B)
  static constexpr int STG_BYTES = SWAP ? 0 : kEpiMWarps * 4096;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int STAGES_RAW = (SMEM_LIMIT - 1024 - BAR_BYTES - P_BYTES - STG_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 12 ? 12 : STAGES_RAW;
  static constexpr int ACC_COLS = C1::ACC_COLS;   // >= phase 2's BN
  static constexpr int TMEM_NEED = 2 * ACC_COLS;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                                                : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + P_BYTES + STG_BYTES + 1024 + BAR_BYTES;
  static constexpr uint32_t IDESC = C1::IDESC;
  static_assert(C1::IDESC == C2::IDESC, "same MMA shape in both phases");
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
};

// Phase-1 epilogue of a token-major tile without the gate (GELU, or no activation):
// warp (q, half) owns accumulator lanes 32q .. 32q+31 (tokens) and columns
// [64 half, 64 half + 64) of the tile. Two 32-column tensor-memory loads, the bias and
// the activation on 32 independent values each, bf16 packing; then the warp's 32 x 64 block
// passes through its own 4 KB of shared memory (16-byte chunk c of row r at
// r * 128 + ((c ^ (r & 7)) * 16), conflict-free both ways) so that every global store
// instruction writes whole 128-byte row segments (8 lanes per row, 4 rows) instead of
// 16 bytes of 32 different rows. Not inlined: a dry call (dry = true: no global
// stores) made while the main loop runs fetches the instructions the real call then
// finds in the instruction cache -- the epilogue runs once per CTA, right after the
// L2 has been flushed of everything, code included, in the measured setting.
struct TokEpi {   // the launch arguments the token-major epilogue reads, passed by value
  __nv_bfloat16* Y;
  const __nv_bfloat16* bias;
  int M, ldy, per_shard, act;
};
template <int BN>
__device__ __noinline__ void mlp_epi_tok64(const TokEpi a, uint32_t tacc_q, uint32_t stg, int s, int wt, int mt,
                                           int q, int half, int lane, bool dry) {
  static_assert(BN == 128, "two 64-column halves per tile");
  const int wc0 = wt * BN + 64 * half;   // shard column of the warp's first column
  const __nv_bfloat16* bias = a.bias;
  // not unrolled: the epilogue runs once per CTA, so after the L2 flush its code is
  // fetched cold, and half the code is worth more than the second half's overlap
  // (A/B: GELU MLP 35.8 -> 33.7 us)
#pragma unroll 1
  for (int sub = 0; sub < 2; ++sub) {    // 32 columns at a time
    float v[32];
    tmem_ld32(tacc_q + static_cast<uint32_t>(64 * half + 32 * sub), v);
    if (bias != nullptr) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int w = wc0 + 32 * sub + j;
        if (w < a.per_shard) v[j] += __bfloat162float(bias[s * a.per_shard + w]);   // column-parallel
      }
    }
    if (a.act == A_GELU) {
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float2 h = gelu2(f2(v[j], v[j + 1]));
        v[j] = h.x;
        v[j + 1] = h.y;
      }
    }
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const int c = 4 * sub + c4;        // 16-byte chunk of the row's 128 bytes
      uint32_t pk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[8 * c4 + 2 * k], v[8 * c4 + 2 * k + 1]);
        pk[k] = *reinterpret_cast<uint32_t*>(&b);
      }
      st_shared_v4(stg + static_cast<uint32_t>(lane * 128 + ((c ^ (lane & 7)) << 4)), pk[0], pk[1], pk[2], pk[3]);
    }
  }
  __syncwarp();
  const int cc = lane & 7;
  const int w = wc0 + 8 * cc;
  __nv_bfloat16* Y = a.Y;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 4 * i + (lane >> 3);
    const uint4 d = ld_shared_v4(stg + static_cast<uint32_t>(r * 128 + ((cc ^ (r & 7)) << 4)));
    const int tok = mt * 128 + q * 32 + r;
    if (!dry && tok < a.M && w < a.per_shard)
      *reinterpret_cast<uint4*>(Y + static_cast<size_t>(tok) * a.ldy + static_cast<size_t>(s) * a.per_shard + w) = d;
  }
  __syncwarp();   // the staging block may be rewritten by this warp's next tile
}

// Phase-1 epilogue of a weight-major gate/up tile pair (decode sizes): thread = one
// weight row w0 of the shard (accumulator lane), warp half `half` takes every other
// 16-token chunk; SiLU(gate + bias) * (up + bias), stored as h[token][shard column].
// Not inlined, arguments by value, callable dry: see mlp_epi_tok64.
struct GateEpi {
  __nv_bfloat16* Y;
  const __nv_bfloat16* bias;
  int M, ldy, per_shard, gate_off;
};
template <int BN>
__device__ __noinline__ void mlp_epi_gate(const GateEpi a, uint32_t tacc_q, int s, int wt, int mt, int row, int half,
                                          int uoff, bool dry) {
  const int w0 = wt * 128 + row;
  // rows past the shard's end still take part in the tensor-memory loads, which are
  // warp-wide (.sync.aligned): only their bias reads and stores are skipped
  const bool live = w0 < a.per_shard;
  const int col = s * a.per_shard + w0;
  const float bx = (live && a.bias != nullptr) ? __bfloat162float(a.bias[col]) : 0.0f;
  const float by = (live && a.bias != nullptr) ? __bfloat162float(a.bias[a.gate_off + col]) : 0.0f;
#pragma unroll 1
  for (int c0 = 16 * half; c0 < BN; c0 += 32) {
    float v[16], u[16];
    tmem_ld16(tacc_q + c0, v);
    tmem_ld16(tacc_q + uoff + c0, u);
    const int tok0 = mt * BN + c0;
    if (a.bias != nullptr) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v[j] += bx;
        u[j] += by;
      }
    }
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      const float2 h = silu_mul2(f2(v[j], v[j + 1]), f2(u[j], u[j + 1]));
      v[j] = h.x;
      v[j + 1] = h.y;
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int t = tok0 + j;
      if (t >= a.M) break;
      if (!dry && live) a.Y[static_cast<size_t>(t) * a.ldy + col] = __float2bfloat16_rn(v[j]);
    }
  }
}
__device__ __forceinline__ GateEpi gate_epi(const GemmArgs& a) {
  return GateEpi{static_cast<__nv_bfloat16*>(a.Y), static_cast<const __nv_bfloat16*>(a.bias), a.M, a.ldy, a.per_shard,
                 a.gate_off};
}

__device__ __forceinline__ TokEpi tok_epi(const GemmArgs& a) {
  return TokEpi{static_cast<__nv_bfloat16*>(a.Y), static_cast<const __nv_bfloat16*>(a.bias), a.M, a.ldy, a.per_shard,
                a.act};
}

template <bool SWAP, int BN, bool DUAL1>
__global__ void __launch_bounds__(kThreadsM, 1)
    tps_mlp_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                   const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW2,
                   const GemmArgs a1, const GemmArgs a2, const MlpSync sy) {
  using M = MlpCfg<SWAP, BN, DUAL1>;
  using C1 = typename M::C1;
  using C2 = typename M::C2;
  constexpr int STAGES = M::STAGES;
  if (!cluster_size_is(static_cast<uint32_t>(a2.cs), a1.status)) return;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sX = base;
  const uint32_t sW = base + STAGES * M::X_BYTES;
  const uint32_t sP = base + STAGES * M::STAGE_BYTES;
  float* gP = reinterpret_cast<float*>(gbase + STAGES * M::STAGE_BYTES);
  const uint32_t sStg = sP + M::P_BYTES;   // phase-1 epilogue staging (token-major)
  const uint32_t sBar = sStg + M::STG_BYTES;
  uint8_t* gBar = gbase + STAGES * M::STAGE_BYTES + M::P_BYTES + M::STG_BYTES;
  auto full_bar = [&](int i) { return sBar + 8u * i; };
  auto empty_bar = [&](int i) { return sBar + 8u * (STAGES + i); };
  auto tfull_bar = [&](int i) { return sBar + 8u * (2 * STAGES + i); };
  auto tempty_bar = [&](int i) { return sBar + 8u * (2 * STAGES + 2 + i); };
  const uint32_t done_bar = sBar + 8u * (2 * STAGES + 4);
  const uint32_t epi_done_bar = sBar + 8u * (2 * STAGES + 5);
  const uint32_t ready_bar = sBar + 8u * (2 * STAGES + 6);
  const uint32_t consumed_bar = sBar + 8u * (2 * STAGES + 7);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 8));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gBar + 8 * (2 * STAGES + 8) + 4);
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
      mbar_init(tempty_bar(i), kEpiMWarps);
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_done_bar, kEpiMWarps);
    mbar_init(ready_bar, 32 * kEpiMWarps);   // both threads of a row push half of it
    mbar_init(consumed_bar, 32 * kEpiMWarps * a2.cs);
    *abort_flag = 0;
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
  cluster_sync_all();   // every CTA's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = a1.timeout_ns;
  griddep_launch_dependents();

  // phase 2: one row tile per cluster, this CTA's contiguous share of its K range
  const int cs = a2.cs;
  const int cl = static_cast<int>(blockIdx.x) / cs;
  const int crank = static_cast<int>(blockIdx.x) % cs;
  const int kb0_2 = (crank * a2.KI) / cs;
  const int kb1_2 = ((crank + 1) * a2.KI) / cs;
  const bool has2 = cl < a2.tiles;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      griddep_wait();
      for (int t = blockIdx.x; ok && t < a1.tiles; t += gridDim.x) {
        int s, wt, mt;
        tile_coords(a1, t, s, wt, mt);
        for (int kb = 0; kb < a1.KI; ++kb) {
          if (!mbar_wait<kMlpSuspendNs>(empty_bar(stage), phase ^ 1u, abort_flag, tmo, a1.status)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), C1::STAGE_BYTES);
          tma_load_3d(sX + stage * M::X_BYTES, &tmX, full_bar(stage), kb * 64, mt * C1::XR, 0);
#pragma unroll
          for (int j = 0; j < C1::NWB; ++j) {
            const int row0 = wt * C1::WR + j * C1::WBOX;
            tma_load_4d(sW + stage * M::W_BYTES + j * C1::WBOX * 128, &tmW1, full_bar(stage), 0, row0 & 127, kb,
                        s * a1.RB + (row0 >> 7));
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (ok && has2) {
        int s2, wt2, mt2;
        tile_coords(a2, cl, s2, wt2, mt2);
        if (sy.prefetch2 > 0) {
          // the leading row-layer weight boxes of this CTA: into L2 while the column layer finishes
          for (int kb = kb0_2; kb < min(kb1_2, kb0_2 + sy.prefetch2); ++kb) {
            const int ks = kb / a2.KBs;
            const int kk = kb - ks * a2.KBs;
#pragma unroll
            for (int j = 0; j < C2::NWB; ++j) {
              const int row0 = wt2 * C2::WR + j * C2::WBOX;
              tma_prefetch_4d(&tmW2, 0, row0 & 127, kk, ks * a2.RB + (row0 >> 7));
            }
          }
        }
        int ready_shard = -1;
        for (int kb = kb0_2; kb < kb1_2; ++kb) {
          const int ks = kb / a2.KBs;   // shard of this K block
          const int kk = kb - ks * a2.KBs;
          if (ks != ready_shard) {
            // every column tile of (token block mt2, shard ks) has stored its h columns
            if (!wait_count_geq(sy.ready + mt2 * a2.tp + ks, sy.need, abort_flag, tmo, a1.status)) { ok = false; break; }
            fence_proxy_async_global();
            ready_shard = ks;
          }
          if (!mbar_wait<kMlpSuspendNs>(empty_bar(stage), phase ^ 1u, abort_flag, tmo, a1.status)) { ok = false; break; }
          mbar_arrive_expect_tx(full_bar(stage), C2::STAGE_BYTES);
          if (a2.x_sharded)
            tma_load_3d(sX + stage * M::X_BYTES, &tmH, full_bar(stage), kk * 64, ks, mt2 * C2::XR);
          else
            tma_load_3d(sX + stage * M::X_BYTES, &tmH, full_bar(stage), ks * a2.x_shard_cols + kk * 64, mt2 * C2::XR,
                        0);
#pragma unroll
          for (int j = 0; j < C2::NWB; ++j) {
            const int row0 = wt2 * C2::WR + j * C2::WBOX;
            tma_load_4d(sW + stage * M::W_BYTES + j * C2::WBOX * 128, &tmW2, full_bar(stage), 0, row0 & 127, kk,
                        ks * a2.RB + (row0 >> 7));
          }
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
      const int ntiles1 = (a1.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                          static_cast<int>(gridDim.x);
      const int njobs = max(ntiles1, 0) + (has2 ? 1 : 0);
      for (int j = 0; ok && j < njobs; ++j) {
        const bool p2 = (j == njobs - 1) && has2;
        const bool dual = DUAL1 && !p2;
        const int kb0 = p2 ? kb0_2 : 0;
        const int kb1 = p2 ? kb1_2 : a1.KI;
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
            if (SWAP) {
              umma_bf16(d0, dw + koff, dx + koff, M::IDESC, acc);
              if (dual) {
                const uint64_t dw2 = smem_desc_sw128(wa + 128 * 128);   // up rows 128..255 of the block
                umma_bf16(d0 + BN, dw2 + koff, dx + koff, M::IDESC, acc);
              }
            } else {
              umma_bf16(d0, dx + koff, dw + koff, M::IDESC, acc);
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
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;      // which half of a tile's columns this warp takes
    const int row = q * 32 + lane;
    const int ep_tid = threadIdx.x - 64;   // 0..255 on warps 2-9
    const int uoff = DUAL1 ? BN : BN / 2;   // the up accumulator's columns after the gate's
    int nloc = 0;
    bool failed = false;
    {
      // Dry passes through both phases' epilogue code while the column layer's MMAs run
      // (see mlp_epi_tok64): they read the second accumulator buffer, which the row
      // layer's MMAs write only after the readiness flags, and this CTA's partial-sum
      // slots, and store nothing.
      const uint32_t spare =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(M::ACC_COLS);
      if constexpr (!SWAP)
        mlp_epi_tok64<BN>(tok_epi(a1), spare, sStg + static_cast<uint32_t>(warp - 2) * 4096u, 0, 0, 0, q, half, lane,
                          true);
      else
        mlp_epi_gate<BN>(gate_epi(a1), spare, 0, 0, 0, row, half, uoff, true);
      csplit_warm<SWAP, BN, kEpiMWarps, false>(a2, gP, sP, spare, row, ep_tid);
    }
    for (int t = blockIdx.x; t < a1.tiles; t += gridDim.x) {
      const int buf = nloc & 1;
      const uint32_t use = static_cast<uint32_t>(nloc >> 1);
      const bool ok = mbar_wait<kMlpSuspendNs>(tfull_bar(buf), use & 1u, abort_flag, tmo, a1.status);
      if (epi_bar_or<32 * kEpiMWarps>(!ok)) { failed = true; break; }
      tc_fence_after();
      int s, wt, mt;
      tile_coords(a1, t, s, wt, mt);
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * M::ACC_COLS);
      if constexpr (!SWAP) {
        // the token-major form runs only the GELU MLP (the gated MLP is fused at decode
        // sizes only, weight-major), and h is bf16
        mlp_epi_tok64<BN>(tok_epi(a1), tacc, sStg + static_cast<uint32_t>(warp - 2) * 4096u, s, wt, mt, q, half, lane,
                          false);
      } else {
        // the weight-major form runs only the gated MLP (gate and up accumulators, DUAL1)
        mlp_epi_gate<BN>(gate_epi(a1), tacc, s, wt, mt, row, half, uoff, false);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
      // publish the tile: all epilogue threads' h stores, then one release increment
      epi_bar<32 * kEpiMWarps>();
      if (ep_tid == 0) {
        fence_proxy_async_global();
        red_release_gpu_add(sy.ready + mt * a1.tp + s, 1);
      }
      ++nloc;
    }
    if (!failed && has2) {
      const int buf = nloc & 1;
      const uint32_t use = static_cast<uint32_t>(nloc >> 1);
      const bool ok = mbar_wait<kMlpSuspendNs>(tfull_bar(buf), use & 1u, abort_flag, tmo, a1.status);
      if (!epi_bar_or<32 * kEpiMWarps>(!ok)) {
        tc_fence_after();
        int s2, wt2, mt2;
        tile_coords(a2, cl, s2, wt2, mt2);
        const uint32_t tacc =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * M::ACC_COLS);
        // the only cluster-split tile of this CTA: barrier phase 0, nothing to wait for after it
        csplit_tile<SWAP, BN, kEpiMWarps, false>(a2, gP, sP, ready_bar, consumed_bar, tempty_bar(buf), abort_flag, tmo,
                                          tacc, kb0_2 < kb1_2, s2, wt2, mt2, row, lane, ep_tid, 0, true);
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_done_bar);
  }
}

}  // namespace tps
