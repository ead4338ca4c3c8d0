// tps_kernels.cu -- every device kernel of the library and its host-side
// launcher: the sharded GEMM instantiations, the weight packer, the standalone
// cross-shard reduction and the bounded-wait self-test. All device code lives in
// this one translation unit (so the device error word needs no relocatable code).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <cstdio>
#include <atomic>
#include <mutex>

#include "tps_gemm.cuh"
#include "tps_gemm2.cuh"
#include "tps_mlp.cuh"
#include "tps_mlp_sk.cuh"
#include "tps_attn.cuh"
#include "tps_internal.h"

namespace tps {

// ============================================================================
// Weight packer: a bit copy of the logical weight into the packed layout
//   out[s][rb][kb][r][c] = W[col_off(s) + 64*kb + c][row_src(s, 128*rb + r)]
// (source W[k][n], or W^T[n][k] when transposed), zero where the packed row or
// K index falls in the padding. Each [128][64] block is 16 KB contiguous.
// ============================================================================
struct PackArgs {
  const uint16_t* W;
  uint16_t* out;
  int transposed;
  long long k, n;      // logical W[k, n]
  int tp;
  int kind;
  int R;               // valid packed rows per shard
  int Kp;              // valid packed row length (k, or k/tp for ROW)
  int RB, KB;          // 128-row blocks and 64-wide K blocks per shard
  // COLUMN
  int ns;
  // QKV
  int q_cols, kv_cols, hq_d, hkv_d, kv_first_num, kv_first_den, head_dim;
  // GATE_UP
  int Is, I;
};

__device__ __forceinline__ long long pack_row_src(const PackArgs& p, int s, int r) {
  if (r >= p.R) return -1;
  switch (p.kind) {
    case K_COLUMN:
      return static_cast<long long>(s) * p.ns + r;
    case K_ROW:
      return r;
    case K_QKV: {
      const int kvf = (s * p.kv_first_num) / p.kv_first_den;
      if (r < p.q_cols) return static_cast<long long>(s) * p.q_cols + r;
      if (r < p.q_cols + p.kv_cols) return p.hq_d + kvf * p.head_dim + (r - p.q_cols);
      return p.hq_d + p.hkv_d + kvf * p.head_dim + (r - p.q_cols - p.kv_cols);
    }
    default: {  // K_GATE_UP: packed rows [256b, 256b+128) gate, [256b+128, 256b+256) up
      const int blk = r >> 8;
      const int half = (r >> 7) & 1;
      const int f = blk * 128 + (r & 127);
      if (f >= p.Is) return -1;
      return static_cast<long long>(half) * p.I + static_cast<long long>(s) * p.Is + f;
    }
  }
}

// One block fills one 64 (rows) x 64 (K) half of a packed [128][64] block through
// shared memory, so the read (along whichever source dimension is contiguous)
// and the write (along K) are both coalesced.
__global__ void __launch_bounds__(256) tps_pack_kernel(const PackArgs p) {
  __shared__ uint16_t tile[64][65];
  const int s = blockIdx.z;
  const int r0 = blockIdx.y * 64;            // packed row (within the shard, padded)
  const int c0 = blockIdx.x * 64;            // packed K index (padded)
  const long long coff = (p.kind == K_ROW) ? static_cast<long long>(s) * p.Kp : 0;
  const int tid = threadIdx.x;
  if (p.transposed) {
    // source W^T[n][k]: contiguous along K
    for (int i = tid; i < 64 * 64; i += 256) {
      const int rr = i >> 6, cc = i & 63;
      const int c = c0 + cc;
      uint16_t v = 0;
      const long long j = pack_row_src(p, s, r0 + rr);
      if (j >= 0 && c < p.Kp) v = p.W[j * p.k + coff + c];
      tile[rr][cc] = v;
    }
  } else {
    // source W[k][n]: contiguous along the output-feature index j
    for (int i = tid; i < 64 * 64; i += 256) {
      const int cc = i >> 6, rr = i & 63;
      const int c = c0 + cc;
      uint16_t v = 0;
      const long long j = pack_row_src(p, s, r0 + rr);
      if (j >= 0 && c < p.Kp) v = p.W[(coff + c) * p.n + j];
      tile[rr][cc] = v;
    }
  }
  __syncthreads();
  const int rb = r0 >> 7, kb = c0 >> 6;
  uint16_t* blk = p.out + ((static_cast<long long>(s) * p.RB + rb) * p.KB + kb) * (128 * 64);
  for (int i = tid; i < 64 * 64; i += 256) {
    const int rr = i >> 6, cc = i & 63;
    blk[((r0 & 127) + rr) * 64 + cc] = tile[rr][cc];
  }
}

// ============================================================================
// Standalone cross-shard reduction: Y = ((P_0 + P_1) + ...) + P_{tp-1} (+ bias),
// 16-byte vector loads, shard order fixed. BF16 = true is the exchange of bf16
// partials: every P_s rounded to bf16, a bf16 rounding after every addition and
// after the bias.
// ============================================================================
template <bool BF16>
__global__ void __launch_bounds__(256) tps_reduce_kernel(const float* __restrict__ P, int tp, long long mn,
                                                         int n, const __nv_bfloat16* __restrict__ bias, void* Y,
                                                         int y_f32) {
  const long long nvec = mn >> 2;
  for (long long v = blockIdx.x * 256LL + threadIdx.x; v < nvec; v += static_cast<long long>(gridDim.x) * 256) {
    const float4* p4 = reinterpret_cast<const float4*>(P) + v;
    float4 acc = __ldcs(p4);
    if (BF16) acc = make_float4(bf16r(acc.x), bf16r(acc.y), bf16r(acc.z), bf16r(acc.w));
    for (int s = 1; s < tp; ++s) {
      const float4 x = __ldcs(p4 + static_cast<long long>(s) * nvec);
      if (BF16) {
        acc.x = bf16r(acc.x + bf16r(x.x));
        acc.y = bf16r(acc.y + bf16r(x.y));
        acc.z = bf16r(acc.z + bf16r(x.z));
        acc.w = bf16r(acc.w + bf16r(x.w));
      } else {
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
      }
    }
    if (bias != nullptr) {
      const int c = static_cast<int>((v * 4) % n);
      acc.x += __bfloat162float(bias[c + 0]);
      acc.y += __bfloat162float(bias[c + 1]);
      acc.z += __bfloat162float(bias[c + 2]);
      acc.w += __bfloat162float(bias[c + 3]);
      if (BF16) acc = make_float4(bf16r(acc.x), bf16r(acc.y), bf16r(acc.z), bf16r(acc.w));
    }
    if (y_f32) {
      reinterpret_cast<float4*>(Y)[v] = acc;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      reinterpret_cast<uint2*>(Y)[v] = pk;
    }
  }
}

// ============================================================================
// Bounded-wait self-test: one thread waits on a barrier that nothing completes.
// ============================================================================
__global__ void tps_wait_timeout_kernel(unsigned long long timeout_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    mbar_wait(smem_u32(&bar), 0, &abort_flag, timeout_ns, status);
  }
}

// ============================================================================
// Host launchers
// ============================================================================
// Token-major GEMM launches carry programmatic stream serialization: the kernel
// may be scheduled while the previous kernel of the stream drains, runs its
// prologue (barrier init, tensor-memory allocation, descriptor prefetch), and
// waits in griddepcontrol.wait for that kernel's completion before touching
// global memory. Weight-major (decode-shaped, HBM-bound) launches do not: there
// the early start measured ~3 us slower per gate/up -> down step (the kernels
// still call griddepcontrol, which is then a no-op). A cluster launch adds the
// cluster dimension.
struct LaunchCfg {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  LaunchCfg(int grid, int smem, cudaStream_t st, int cluster, int threads = kThreads, bool pdl = true) {
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = st;
    int n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    ++n;
    if (cluster > 1) {
      attr[n].id = cudaLaunchAttributeClusterDimension;
      attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
      attr[n].val.clusterDim.y = 1;
      attr[n].val.clusterDim.z = 1;
      ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = static_cast<unsigned>(n);
  }
};

template <bool SWAP, int BN, bool DUAL, bool ARGMAX = false>
static int launch_one(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid,
                      cudaStream_t st) {
  using Cfg = GemmCfg<SWAP, BN, DUAL>;
  auto kfn = tps_gemm_kernel<SWAP, BN, DUAL, false, ARGMAX>;
  // the shared-memory opt-in is per device: remember it per device ordinal
  static unsigned long long attr_done = 0ull;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -6;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
      return -6;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  LaunchCfg lc(grid, Cfg::SMEM_BYTES, st, 1, kThreads, !SWAP);
  if (cudaLaunchKernelEx(&lc.cfg, kfn, tx, tw, a) != cudaSuccess) return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

template <bool SWAP, int BN>
static int launch_csplit(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid, cudaStream_t st) {
  using Cfg = GemmCfg<SWAP, BN, false, true>;
  auto kfn = tps_gemm_kernel<SWAP, BN, false, true>;
  static unsigned long long attr_done = 0ull;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -6;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
      return -6;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  LaunchCfg lc(grid, Cfg::SMEM_BYTES, st, a.cs, kThreads, !SWAP);
  if (cudaLaunchKernelEx(&lc.cfg, kfn, tx, tw, a) != cudaSuccess) return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

template <bool SWAP, int BN>
static int csplit_clusters(int cs) {
  using Cfg = GemmCfg<SWAP, BN, false, true>;
  auto kfn = tps_gemm_kernel<SWAP, BN, false, true>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cs), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess) return 0;
  return n;
}

int launch_gemm_csplit(int swap, int bn, int cs, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a,
                       int grid, cudaStream_t st) {
  (void)cs;
#define TPS_C(S, B) \
  if (swap == S && bn == B) return launch_csplit<S, B>(tx, tw, a, grid, st);
  TPS_C(false, 128) TPS_C(false, 64) TPS_C(true, 16) TPS_C(true, 32) TPS_C(true, 64) TPS_C(true, 128)
#undef TPS_C
  return -8;
}

// Largest number of resident clusters of `cs` CTAs of a cluster-split kernel on
// the current device (cached per device, orientation, width and cluster size).
int max_csplit_clusters(int swap, int bn, int cs) {
  static std::mutex mu;
  static int cache[64][2][8][9] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || cs < 2 || cs > 8) return 0;
  const int bi = bn == 16 ? 0 : bn == 32 ? 1 : bn == 64 ? 2 : bn == 128 ? 3 : 7;
  if (bi == 7) return 0;
  std::lock_guard<std::mutex> lock(mu);
  int& c = cache[dev][swap ? 1 : 0][bi][cs];
  if (c == 0) {
    int n = 0;
    if (!swap && bn == 128) n = csplit_clusters<false, 128>(cs);
    else if (!swap && bn == 64) n = csplit_clusters<false, 64>(cs);
    else if (swap && bn == 16) n = csplit_clusters<true, 16>(cs);
    else if (swap && bn == 32) n = csplit_clusters<true, 32>(cs);
    else if (swap && bn == 64) n = csplit_clusters<true, 64>(cs);
    else if (swap && bn == 128) n = csplit_clusters<true, 128>(cs);
    c = n > 0 ? n : -1;
  }
  return c > 0 ? c : 0;
}

// One-launch MLP: a cluster launch like the cluster-split GEMM. The CTAs of
// phase 2 wait for phase-1 tiles of other CTAs; the planner keeps the grid within
// the clusters that are resident at once (one CTA per SM), and the waits are
// bounded. Instantiations: token-major 128-wide (GELU, prefill) and weight-major
// 64-token gate/up (SiLU(gate)*up, decode).
template <bool SWAP, int BN, bool DUAL1>
static int launch_mlp_t(const CUtensorMap& tx, const CUtensorMap& tw1, const CUtensorMap& th, const CUtensorMap& tw2,
                        const GemmArgs& a1, const GemmArgs& a2, const MlpSync& sy, int grid, cudaStream_t st) {
  using Cfg = MlpCfg<SWAP, BN, DUAL1>;
  auto kfn = tps_mlp_kernel<SWAP, BN, DUAL1>;
  static unsigned long long attr_done = 0ull;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -6;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
      return -6;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  // programmatic serialization for the token-major form only (as for the GEMMs)
  LaunchCfg lc(grid, Cfg::SMEM_BYTES, st, a2.cs, kThreadsM, !SWAP);
  if (cudaLaunchKernelEx(&lc.cfg, kfn, tx, tw1, th, tw2, a1, a2, sy) != cudaSuccess) return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_mlp_fused(int swap, const CUtensorMap& tx, const CUtensorMap& tw1, const CUtensorMap& th,
                     const CUtensorMap& tw2, const GemmArgs& a1, const GemmArgs& a2, const MlpSync& sy, int grid,
                     cudaStream_t st) {
  if (!swap) return launch_mlp_t<false, 128, false>(tx, tw1, th, tw2, a1, a2, sy, grid, st);
  return launch_mlp_t<true, 64, true>(tx, tw1, th, tw2, a1, a2, sy, grid, st);
}

// Stream-K one-launch gated MLP (decode sizes): a plain launch of `grid` CTAs, one
// per SM; the planner keeps the grid within the CTAs that are resident at once.
int launch_mlp_sk(const CUtensorMap& tx, const CUtensorMap& tw1, const CUtensorMap& th, const CUtensorMap& tw2,
                  const GemmArgs& a1, const GemmArgs& a2, const MlpSync& sy, int grid, cudaStream_t st) {
  static unsigned long long attr_done = 0ull;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -6;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(tps_mlp_sk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, MlpSkCfg::SMEM_BYTES) !=
        cudaSuccess)
      return -6;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  LaunchCfg lc(grid, MlpSkCfg::SMEM_BYTES, st, 1, kThreads, false);
  if (cudaLaunchKernelEx(&lc.cfg, tps_mlp_sk_kernel, tx, tw1, th, tw2, a1, a2, sy) != cudaSuccess) return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

// CTAs of the stream-K MLP kernel resident at once on the current device (SMs x
// blocks per SM; cached per device), 0 on error.
int mlp_sk_resident_ctas() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] > 0) return cache[dev];
  if (cudaFuncSetAttribute(tps_mlp_sk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, MlpSkCfg::SMEM_BYTES) !=
      cudaSuccess)
    return 0;
  int per_sm = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tps_mlp_sk_kernel, kThreads, MlpSkCfg::SMEM_BYTES) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  cache[dev] = per_sm * sms;
  return cache[dev];
}

int mlp_sk_slot_bytes(int phase) {
  return (phase == 0 ? SkC1::SLOT_ELEMS : SkC2::SLOT_ELEMS) * 4;
}

int gemm_smem_bytes(int swap, int bn, int dual) {
#define TPS_SM(S, B, D) \
  if (swap == S && bn == B && dual == D) return GemmCfg<S, B, D>::SMEM_BYTES;
  TPS_SM(false, 256, false) TPS_SM(false, 128, false) TPS_SM(false, 64, false)
  TPS_SM(true, 16, false) TPS_SM(true, 32, false) TPS_SM(true, 64, false) TPS_SM(true, 128, false)
  TPS_SM(true, 16, true) TPS_SM(true, 32, true) TPS_SM(true, 64, true) TPS_SM(true, 128, true)
#undef TPS_SM
  return -1;
}

int gemm_slot_elems(int swap, int bn, int dual) {
  (void)swap;
  return 128 * bn * (dual ? 2 : 1);
}

int launch_gemm_argmax(int swap, int bn, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid,
                       cudaStream_t st) {
#define TPS_A(S, B) \
  if (swap == S && bn == B) return launch_one<S, B, false, true>(tx, tw, a, grid, st);
  TPS_A(false, 256) TPS_A(false, 128) TPS_A(false, 64) TPS_A(true, 16) TPS_A(true, 32) TPS_A(true, 64)
  TPS_A(true, 128)
#undef TPS_A
  return -8;
}

// One CTA per token over its tp x per_shard_entries tile results. The selection
// (larger logit, then lower vocab index) is a total order, so reducing all the
// entries at once gives exactly the shard-local argmaxes followed by the max over
// shards in shard order. Launched as a programmatic dependent of the GEMM: the
// block is resident before the GEMM ends and waits for its results in hardware.
constexpr int kAmaxThreads = 256;

__global__ void __launch_bounds__(kAmaxThreads) tps_argmax_reduce_kernel(const AmaxEntry* __restrict__ part, int M,
                                                                         int entries, int32_t* __restrict__ out_idx,
                                                                         float* __restrict__ out_val) {
  __shared__ AmaxEntry red[kAmaxThreads / 32];
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int tok = blockIdx.x; tok < M; tok += gridDim.x) {
    const AmaxEntry* p = part + static_cast<size_t>(tok) * entries;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll 8
    for (int e = threadIdx.x; e < entries; e += kAmaxThreads) {
      const AmaxEntry x = p[e];
      amax_take(bv, bi, x.v, x.i);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
      amax_take(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
    if (lane == 0) red[warp] = AmaxEntry{bv, bi};
    __syncthreads();
    if (warp == 0) {
      bv = lane < kAmaxThreads / 32 ? red[lane].v : -INFINITY;
      bi = lane < kAmaxThreads / 32 ? red[lane].i : 0x7fffffff;
#pragma unroll
      for (int o = 4; o > 0; o >>= 1)
        amax_take(bv, bi, __shfl_xor_sync(0xffffffffu, bv, o), __shfl_xor_sync(0xffffffffu, bi, o));
      if (lane == 0) {
        out_idx[tok] = bi;
        if (out_val != nullptr) out_val[tok] = bv;
      }
    }
    __syncthreads();
  }
}

int launch_argmax_reduce(const void* part, int M, int tp, int per_shard_entries, int32_t* out_idx, float* out_val,
                         cudaStream_t st) {
  const int grid = M < 4 * 148 ? M : 4 * 148;
  LaunchCfg lc(grid, 0, st, 1, kAmaxThreads, true);
  if (cudaLaunchKernelEx(&lc.cfg, tps_argmax_reduce_kernel, static_cast<const AmaxEntry*>(part), M,
                         tp * per_shard_entries, out_idx, out_val) != cudaSuccess)
    return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int attention_smem_bytes(int two_tiles) { return two_tiles ? kAttn2SmemBytes : kAttnSmemBytes; }

int launch_attention(const CUtensorMap& tqkv, const AttnArgs& a, int two_tiles, int grid, cudaStream_t st) {
  static unsigned long long attr_done[2] = {0ull, 0ull};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -6;
  const unsigned long long bit = 1ull << (dev & 63);
  const int v = two_tiles ? 1 : 0;
  const int smem = attention_smem_bytes(v);
  auto* fn = v ? tps_attn2_kernel : tps_attn_kernel;
  if (!(__atomic_load_n(&attr_done[v], __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -6;
    __atomic_fetch_or(&attr_done[v], bit, __ATOMIC_ACQ_REL);
  }
  LaunchCfg lc(grid, smem, st, 1, v ? kAttn2Threads : kAttnThreads, true);
  if (cudaLaunchKernelEx(&lc.cfg, fn, tqkv, a) != cudaSuccess) return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_gemm(int swap, int bn, int dual, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a,
                int grid, cudaStream_t st) {
#define TPS_L(S, B, D) \
  if (swap == S && bn == B && dual == D) return launch_one<S, B, D>(tx, tw, a, grid, st);
  TPS_L(false, 256, false) TPS_L(false, 128, false) TPS_L(false, 64, false)
  TPS_L(true, 16, false) TPS_L(true, 32, false) TPS_L(true, 64, false) TPS_L(true, 128, false)
  TPS_L(true, 16, true) TPS_L(true, 32, true) TPS_L(true, 64, true) TPS_L(true, 128, true)
#undef TPS_L
  return -8;
}

template <int BN, int NH>
static int launch_pair(const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid, cudaStream_t st) {
  using Cfg = Gemm2Cfg<BN, NH>;
  auto kfn = tps_gemm2_kernel<BN, NH>;
  static unsigned long long attr_done = 0ull;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -6;
  const unsigned long long bit = 1ull << (dev & 63);
  if (!(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & bit)) {
    if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES) != cudaSuccess)
      return -6;
    __atomic_fetch_or(&attr_done, bit, __ATOMIC_ACQ_REL);
  }
  LaunchCfg lc(grid, Cfg::SMEM_BYTES, st, 2, kThreads2);
  if (cudaLaunchKernelEx(&lc.cfg, kfn, tx, tw, a) != cudaSuccess) return -6;
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_gemm_pair(int bn, int nh, const CUtensorMap& tx, const CUtensorMap& tw, const GemmArgs& a, int grid,
                     cudaStream_t st) {
  if (bn == 256 && nh == 2) return launch_pair<256, 2>(tx, tw, a, grid, st);
  if (bn == 256 && nh == 1) return launch_pair<256, 1>(tx, tw, a, grid, st);
  if (bn == 128 && nh == 1) return launch_pair<128, 1>(tx, tw, a, grid, st);
  return -8;
}

// Largest number of CTA pairs of the pair kernel that can be resident at once on
// the current device (cached per device ordinal; the kernel's shared memory keeps
// it to one CTA per SM in every form).
int max_pair_clusters() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  auto kfn = tps_gemm2_kernel<256, 1>;
  if (cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, Gemm2Cfg<256, 1>::SMEM_BYTES) !=
      cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads2, 1, 1);
  cfg.dynamicSmemBytes = Gemm2Cfg<256, 1>::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) != cudaSuccess) return 0;
  if (dev < 64) cache[dev] = n;
  return n;
}

// ============================================================================
// Static scratch of the allocation-free row-parallel entry point: stream-K
// segment slots and tile counters for callers that cannot provide a workspace.
// Every device that loads the library holds it until the process exits.
// ============================================================================
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The CUDA context current on the calling thread (driver entry point, looked up
// once), or null when it cannot be read.
static CUcontext current_context() {
  typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
  static std::atomic<CtxGetCurrentFn> fn{nullptr};
  CtxGetCurrentFn f = fn.load();
  if (f == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr)
      return nullptr;
    f = reinterpret_cast<CtxGetCurrentFn>(p);
    fn.store(f);
  }
  CUcontext c = nullptr;
  return f(&c) == CUDA_SUCCESS ? c : nullptr;
}

int static_scratch(void** ptr) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  static CUcontext ctx[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -6;
  std::lock_guard<std::mutex> lock(mu);
  // The address is looked up once per device and context: a context that was torn
  // down and created again (cudaDeviceReset) loads the module again, and the array
  // may then sit at another address.
  const CUcontext cur = current_context();
  if (addr[dev] == nullptr || cur == nullptr || cur != ctx[dev]) {
    // a symbol's host-side name is not a device address: ask the runtime, with
    // the device current (this also makes its primary context current)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return -6;
    addr[dev] = p;
    ctx[dev] = current_context();
  }
  *ptr = addr[dev];
  return 0;
}

int launch_pack(const PackHost& h, cudaStream_t st) {
  PackArgs p{};
  p.W = static_cast<const uint16_t*>(h.W);
  p.out = static_cast<uint16_t*>(h.out);
  p.transposed = h.transposed;
  p.k = h.k;
  p.n = h.n;
  p.tp = h.tp;
  p.kind = h.kind;
  p.R = h.R;
  p.Kp = h.Kp;
  p.RB = (h.R + 127) / 128;
  p.KB = (h.Kp + 63) / 64;
  p.ns = h.ns;
  p.q_cols = h.q_cols;
  p.kv_cols = h.kv_cols;
  p.hq_d = h.hq_d;
  p.hkv_d = h.hkv_d;
  p.kv_first_num = h.kv_first_num;
  p.kv_first_den = h.kv_first_den;
  p.head_dim = h.head_dim;
  p.Is = h.Is;
  p.I = h.I;
  dim3 grid(p.KB, p.RB * 2, h.tp);
  tps_pack_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_reduce(const float* P, int tp, long long m, long long n, const void* bias, void* Y, int y_f32,
                  int bf16_chain, int num_sms, cudaStream_t st) {
  const long long nvec = (m * n) >> 2;
  long long blocks = (nvec + 255) / 256;
  const long long cap = static_cast<long long>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (bf16_chain)
    tps_reduce_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        P, tp, m * n, static_cast<int>(n), static_cast<const __nv_bfloat16*>(bias), Y, y_f32);
  else
    tps_reduce_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        P, tp, m * n, static_cast<int>(n), static_cast<const __nv_bfloat16*>(bias), Y, y_f32);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int launch_wait_timeout(unsigned long long timeout_ns, int* status, cudaStream_t st) {
  tps_wait_timeout_kernel<<<1, 32, 0, st>>>(timeout_ns, status);
  return cudaGetLastError() == cudaSuccess ? 0 : -6;
}

int read_and_clear_device_error(cudaStream_t st, int* out) {
  int v = 0;
  if (cudaStreamSynchronize(st) != cudaSuccess) return -6;
  if (cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(int)) != cudaSuccess) return -6;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(int)) != cudaSuccess) return -6;
  *out = v;
  return 0;
}

}  // namespace tps
