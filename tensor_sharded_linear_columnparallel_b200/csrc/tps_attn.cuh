// tps_attn.cuh -- attention on local heads, between the column-parallel QKV and
// the row-parallel o_proj ("Tensor Parallel：当一张 GPU 放不下一个大模型", section
// "Attention 里的 tensor parallel": every shard keeps the q/k/v of its own heads,
// computes their attention locally, and its output stays split by head for the
// row-parallel o_proj). Head dimension 128.
//
// A work item is (sequence, query head, block of 128 queries); persistent CTAs
// take items heaviest first (with a causal mask the late query blocks see the most
// keys). For every 128-key block j of an item the tensor core computes
// S_j = Q K_j^T into tensor memory; four softmax warps (one query row per thread)
// take the running row max, write P_j = exp(S_j / sqrt(d) - max) as bf16 into
// shared memory in the 128-byte-swizzled K-major layout, and the tensor core
// computes P_j V_j into a second tensor-memory buffer, reading V MN-major straight
// from its TMA tile. The softmax warps rescale and add those block products in
// registers, so the running output never leaves the SM; the row sum of the
// weights divides it at the end.
//
// Roles (7 warps): 0 = Q and K loads, 1 = MMA issue, 2 = V loads, 3..6 = softmax
// and output. K and V rings of two 128-key stages each, two P buffers, tensor
// memory S[2] and PV[2] (512 columns): S_{j+1} runs on the tensor core while the
// softmax of S_j runs, and P_j V_j while the softmax of S_{j+1} runs.
#pragma once

#include "tps_gemm.cuh"

namespace tps {

constexpr int kAttnD = kAttnHeadDim;           // head dimension
constexpr int kAttnBlk = 128;                  // queries per item, keys per block
constexpr int kAttnThreads = 7 * 32;
constexpr int kAttnTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 operand (two 64-wide boxes)
constexpr int kAttnHalf = kAttnTileBytes / 2;  // one 128-row x 64-column box
constexpr int kAttnOffQ = 0;
constexpr int kAttnOffK = kAttnOffQ + kAttnTileBytes;
constexpr int kAttnOffV = kAttnOffK + 2 * kAttnTileBytes;
constexpr int kAttnOffP = kAttnOffV + 2 * kAttnTileBytes;
constexpr int kAttnOffBar = kAttnOffP + 2 * kAttnTileBytes;
constexpr int kAttnSmemBytes = kAttnOffBar + 256 + 1024;
constexpr uint32_t kAttnIdescS = idesc_bf16_f32(128, 128);
constexpr uint32_t kAttnIdescPV = idesc_bf16_f32(128, 128) | (1u << 16);   // B (= V) MN-major
static_assert(kAttnSmemBytes <= 232448, "shared memory budget");

// Shared-memory descriptor of an MN-major operand written by TMA with the 128-byte
// swizzle: rows of 64 bf16 along N (128 B), one row per K index, 8-row atoms
// 1024 B apart along K (stride byte offset); the next 64 N indices start
// `n_step` bytes further (leading byte offset).
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr, uint32_t n_step) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(n_step >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Orders this thread's generic-proxy shared-memory stores before later reads of
// the same bytes by the tensor core (async proxy).
__device__ __forceinline__ void fence_proxy_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

struct AttnItem {
  int seq, h, qb, nblk;
  int qcol, kcol, vcol;   // first column of the head's q / k / v in a qkv row
};

__device__ __forceinline__ AttnItem attn_item(const AttnArgs& a, int item) {
  AttnItem t;
  const int per = a.nseq * a.hq;
  const int band = item / per;
  const int rem = item - band * per;
  t.qb = a.nqb - 1 - band;                 // heaviest (latest) query blocks first
  t.seq = rem / a.hq;
  t.h = rem - t.seq * a.hq;                // neighbouring CTAs share KV heads in L2
  t.nblk = a.causal ? t.qb + 1 : a.nkb;
  const int r = t.h / a.qs;
  const int lk = t.h / a.grp - (r * a.kv_first_num) / a.kv_first_den;   // KV head within shard r
  t.qcol = r * a.shard_cols + (t.h - r * a.qs) * kAttnD;
  t.kcol = r * a.shard_cols + (a.qs + lk) * kAttnD;
  t.vcol = t.kcol + a.kvs * kAttnD;
  return t;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    tps_attn_kernel(const __grid_constant__ CUtensorMap tmQKV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kAttnOffQ;
  const uint32_t sK = base + kAttnOffK;
  const uint32_t sV = base + kAttnOffV;
  const uint32_t sP = base + kAttnOffP;
  const uint32_t sBar = base + kAttnOffBar;
  const uint32_t q_full = sBar, q_empty = sBar + 8;
  auto k_full = [&](int i) { return sBar + 16u + 8u * i; };
  auto k_empty = [&](int i) { return sBar + 32u + 8u * i; };
  auto v_full = [&](int i) { return sBar + 48u + 8u * i; };
  auto v_empty = [&](int i) { return sBar + 64u + 8u * i; };
  auto s_full = [&](int i) { return sBar + 80u + 8u * i; };
  auto s_empty = [&](int i) { return sBar + 96u + 8u * i; };
  auto p_full = [&](int i) { return sBar + 112u + 8u * i; };
  auto p_empty = [&](int i) { return sBar + 128u + 8u * i; };
  auto o_full = [&](int i) { return sBar + 144u + 8u * i; };
  auto o_empty = [&](int i) { return sBar + 160u + 8u * i; };
  const uint32_t done_bar = sBar + 176u, epi_done_bar = sBar + 184u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kAttnOffBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kAttnOffBar + 196);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gbase + kAttnOffBar + 200);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(s_empty(i), 4);
      mbar_init(p_full(i), 4);
      mbar_init(p_empty(i), 1);
      mbar_init(o_full(i), 1);
      mbar_init(o_empty(i), 4);
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_done_bar, 4);
    *abort_flag = 0;
    *never_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQKV);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t tmo = a.timeout_ns;
  griddep_launch_dependents();

  if (warp == 0 || warp == 2) {
    if (lane == 0) {
      // ------------------------------------------------ loads: warp 0 Q and K, warp 2 V
      const bool is_k = (warp == 0);
      long long n = 0;          // K (or V) blocks issued
      long long nq = 0;         // Q tiles issued
      int it = 0;
      bool ok = true;
      griddep_wait();
      for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++it) {
        const AttnItem t = attn_item(a, item);
        const int row0 = t.seq * a.S;
        if (is_k) {
          if (!mbar_wait(q_empty, static_cast<uint32_t>(it & 1) ^ 1u, abort_flag, tmo)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full, kAttnTileBytes);
          tma_load_3d(sQ, &tmQKV, q_full, t.qcol, row0 + t.qb * kAttnBlk, 0);
          tma_load_3d(sQ + kAttnHalf, &tmQKV, q_full, t.qcol + 64, row0 + t.qb * kAttnBlk, 0);
          ++nq;
        }
        for (int j = 0; j < t.nblk; ++j, ++n) {
          const int st = static_cast<int>(n & 1);
          const uint32_t u = static_cast<uint32_t>((n >> 1) & 1);
          const uint32_t emp = is_k ? k_empty(st) : v_empty(st);
          const uint32_t ful = is_k ? k_full(st) : v_full(st);
          if (!mbar_wait(emp, u ^ 1u, abort_flag, tmo)) { ok = false; break; }
          const uint32_t dst = (is_k ? sK : sV) + st * kAttnTileBytes;
          const int col = is_k ? t.kcol : t.vcol;
          mbar_arrive_expect_tx(ful, kAttnTileBytes);
          tma_load_3d(dst, &tmQKV, ful, col, row0 + j * kAttnBlk, 0);
          tma_load_3d(dst + kAttnHalf, &tmQKV, ful, col + 64, row0 + j * kAttnBlk, 0);
        }
      }
      // wait (bounded) for the copies still in flight before the CTA may exit
      if (nq > 0) mbar_wait(q_full, static_cast<uint32_t>((nq - 1) & 1), never_flag, 200000000ull);
      for (long long i = n > 2 ? n - 2 : 0; i < n; ++i)
        mbar_wait(is_k ? k_full(static_cast<int>(i & 1)) : v_full(static_cast<int>(i & 1)),
                  static_cast<uint32_t>((i >> 1) & 1), never_flag, 200000000ull);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      long long g = 0;          // blocks of earlier items
      int it = 0;
      bool ok = true, any = false;
      const uint64_t dq0 = smem_desc_sw128(sQ), dq1 = smem_desc_sw128(sQ + kAttnHalf);
      for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x, ++it) {
        const AttnItem t = attn_item(a, item);
        if (!mbar_wait(q_full, static_cast<uint32_t>(it & 1), abort_flag, tmo)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; j <= t.nblk; ++j) {
          if (j < t.nblk) {
            const long long gj = g + j;
            const int b = static_cast<int>(gj & 1);
            const uint32_t u = static_cast<uint32_t>((gj >> 1) & 1);
            if (!mbar_wait(k_full(b), u, abort_flag, tmo)) { ok = false; break; }
            if (!mbar_wait(s_empty(b), u ^ 1u, abort_flag, tmo)) { ok = false; break; }
            tc_fence_after();
            const uint32_t kb = sK + b * kAttnTileBytes;
            const uint64_t dk0 = smem_desc_sw128(kb), dk1 = smem_desc_sw128(kb + kAttnHalf);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t off = static_cast<uint64_t>((kk & 3) * 2);   // 16 d = 32 B along K
              umma_bf16(tmem_base + b * 128, (kk < 4 ? dq0 : dq1) + off, (kk < 4 ? dk0 : dk1) + off, kAttnIdescS,
                        kk > 0 ? 1u : 0u);
            }
            umma_commit(k_empty(b));
            umma_commit(s_full(b));
            if (j == t.nblk - 1) umma_commit(q_empty);
            any = true;
          }
          if (j >= 1) {
            const long long gp = g + j - 1;
            const int b = static_cast<int>(gp & 1);
            const uint32_t u = static_cast<uint32_t>((gp >> 1) & 1);
            if (!mbar_wait(p_full(b), u, abort_flag, tmo)) { ok = false; break; }
            if (!mbar_wait(v_full(b), u, abort_flag, tmo)) { ok = false; break; }
            if (!mbar_wait(o_empty(b), u ^ 1u, abort_flag, tmo)) { ok = false; break; }
            tc_fence_after();
            const uint32_t pb = sP + b * kAttnTileBytes;
            const uint32_t vb = sV + b * kAttnTileBytes;
            const uint64_t dp0 = smem_desc_sw128(pb), dp1 = smem_desc_sw128(pb + kAttnHalf);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {   // 16 keys per MMA: 32 B along K in P, 2048 B (16 rows) in V
              const uint64_t off = static_cast<uint64_t>((kk & 3) * 2);
              umma_bf16(tmem_base + 256 + b * 128, (kk < 4 ? dp0 : dp1) + off,
                        smem_desc_sw128_mn(vb + kk * 2048, kAttnHalf), kAttnIdescPV, kk > 0 ? 1u : 0u);
            }
            umma_commit(v_empty(b));
            umma_commit(p_empty(b));
            umma_commit(o_full(b));
          }
        }
        if (!ok) break;
        g += t.nblk;
      }
      // every issued MMA must be complete before tensor memory is released
      if (any) {
        umma_commit(done_bar);
        mbar_wait(done_bar, 0, never_flag, 200000000ull);
      }
      // ... and every softmax warp must be done reading it
      mbar_wait(epi_done_bar, 0, never_flag, tmo);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  } else {
    // -------------------------------------------------- softmax and output (warps 3..6)
    const int q = warp & 3;                       // tensor-memory lane quarter
    const int row = q * 32 + lane;                // query row within the item
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float c = a.scale_log2;
    long long g = 0;
    bool ok = true;
    float o[kAttnD];
    for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x) {
      const AttnItem t = attn_item(a, item);
      const int qidx = t.qb * kAttnBlk + row;     // query position within the sequence
      float m_run = -INFINITY, l_run = 0.f, alpha_prev = 0.f;
#pragma unroll
      for (int i = 0; i < kAttnD; ++i) o[i] = 0.f;
      for (int j = 0; j <= t.nblk; ++j) {
        float alpha_cur = 0.f;
        if (j < t.nblk) {
          const long long gj = g + j;
          const int b = static_cast<int>(gj & 1);
          const uint32_t u = static_cast<uint32_t>((gj >> 1) & 1);
          if (!__all_sync(0xffffffffu, mbar_wait(s_full(b), u, abort_flag, tmo))) { ok = false; break; }
          tc_fence_after();
          const uint32_t ts = tmem_base + lane_off + static_cast<uint32_t>(b * 128);
          const int kbase = j * kAttnBlk;
          const bool masked = (kbase + kAttnBlk > a.S) || (a.causal && j == t.qb);
          const int last = (a.causal ? min(qidx, a.S - 1) : a.S - 1) - kbase;   // last visible key in the block
          float mx = -INFINITY;
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            float v[16];
            tmem_ld16(ts + cc * 16, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) mx = fmaxf(mx, (masked && cc * 16 + i > last) ? -INFINITY : v[i]);
          }
          const float m_new = fmaxf(m_run, mx);
          const float mc = (m_new == -INFINITY ? 0.f : m_new) * c;
          alpha_cur = ex2_approx(fmaf(m_run, c, -mc));     // exp((m_old - m_new) / sqrt(d)); 0 for the first block
          if (!__all_sync(0xffffffffu, mbar_wait(p_empty(b), u ^ 1u, abort_flag, tmo))) { ok = false; break; }
          const uint32_t prow = sP + static_cast<uint32_t>(b * kAttnTileBytes + row * 128);
          float rs = 0.f;
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            float v[16];
            tmem_ld16(ts + cc * 16, v);
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float s0 = (masked && cc * 16 + 2 * i > last) ? -INFINITY : v[2 * i];
              const float s1 = (masked && cc * 16 + 2 * i + 1 > last) ? -INFINITY : v[2 * i + 1];
              const float p0 = ex2_approx(fmaf(s0, c, -mc));
              const float p1 = ex2_approx(fmaf(s1, c, -mc));
              rs += p0 + p1;
              w[i] = pack_bf16(p0, p1);
            }
            // keys [16cc, 16cc+16) = 16-byte chunks 2cc, 2cc+1 of the row; chunk ci sits in
            // key box ci/8 at swizzled position (ci%8) ^ (row%8)
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int ci = cc * 2 + k2;
              st_shared_v4(prow + (ci >> 3) * kAttnHalf + (((ci & 7) ^ (row & 7)) << 4), w[4 * k2], w[4 * k2 + 1],
                           w[4 * k2 + 2], w[4 * k2 + 3]);
            }
          }
          l_run = fmaf(l_run, alpha_cur, rs);
          m_run = m_new;
          fence_proxy_async_shared();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(p_full(b));
            mbar_arrive(s_empty(b));
          }
        }
        if (j >= 1) {
          const long long gp = g + j - 1;
          const int b = static_cast<int>(gp & 1);
          const uint32_t u = static_cast<uint32_t>((gp >> 1) & 1);
          if (!__all_sync(0xffffffffu, mbar_wait(o_full(b), u, abort_flag, tmo))) { ok = false; break; }
          tc_fence_after();
          const uint32_t to = tmem_base + lane_off + static_cast<uint32_t>(256 + b * 128);
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            float v[16];
            tmem_ld16(to + cc * 16, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[cc * 16 + i] = fmaf(o[cc * 16 + i], alpha_prev, v[i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_empty(b));
        }
        alpha_prev = alpha_cur;
      }
      if (!ok) break;
      g += t.nblk;
      if (qidx < a.S) {
        const float inv = 1.0f / l_run;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) +
                                              (static_cast<size_t>(t.seq) * a.S + qidx) * a.ldo + t.h * kAttnD);
#pragma unroll
        for (int k8 = 0; k8 < kAttnD / 8; ++k8) {
          uint4 pk;
          pk.x = pack_bf16(o[8 * k8] * inv, o[8 * k8 + 1] * inv);
          pk.y = pack_bf16(o[8 * k8 + 2] * inv, o[8 * k8 + 3] * inv);
          pk.z = pack_bf16(o[8 * k8 + 4] * inv, o[8 * k8 + 5] * inv);
          pk.w = pack_bf16(o[8 * k8 + 6] * inv, o[8 * k8 + 7] * inv);
          dst[k8] = pk;
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_done_bar);
  }
}

}  // namespace tps
