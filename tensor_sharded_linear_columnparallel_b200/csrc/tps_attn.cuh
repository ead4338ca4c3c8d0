// tps_attn.cuh -- attention on local heads, between the column-parallel QKV and
// the row-parallel o_proj ("Tensor Parallel：当一张 GPU 放不下一个大模型", section
// "Attention 里的 tensor parallel": every shard keeps the q/k/v of its own heads,
// computes their attention locally, and its output stays split by head for the
// row-parallel o_proj). Head dimension 128.
//
// A work item is (sequence, query head, block of 128 queries); persistent CTAs
// take items heaviest first (with a causal mask the late query blocks see the most
// keys), in snake order over the CTAs (attn_item_of). For every 128-key block j
// of an item the tensor core computes S_j = Q K_j^T into tensor memory; the softmax
// warps take the running row max and write P_j = exp(S_j / sqrt(d) - max) as packed
// bf16 pairs back into the first 64 columns of S_j's own tensor-memory buffer, and
// the tensor core adds P_j V_j into the output accumulator O in tensor memory with
// A = P_j read from tensor memory and V read MN-major straight from its TMA tile. The reference max behind P moves only when a
// block's max exceeds it by more than 8 / (log2(e) / sqrt(d)) (weights up to
// 2^8 are exact enough in bf16 and harmless in fp32); only then do the softmax
// warps rescale O in tensor memory, after the previous block's product has
// landed. The row sum of the weights, kept against the same reference, divides O
// at the end -- the result is the same softmax, whatever the reference.
//
// Roles (11 warps): 0 = Q and K loads, 1 = MMA issue, 2 = V loads, 3..10 =
// softmax and output, two warps per query row: warps w and w+4 read the same
// tensor-memory lanes and take 64 of the 128 keys of each block (and 64 of the
// 128 output columns) each, exchanging their partial row max through shared
// memory. K and V rings of three 128-key stages each, tensor memory S/P[2] and O
// (384 of 512 columns): S_{j+1} runs on the tensor core while the softmax of S_j
// runs, and P_j V_j while the softmax of S_{j+1} runs. The tcgen05.mma operations
// one thread issues form one in-order pipeline, so S_{j+2}, issued after P_j V_j,
// overwrites buffer j mod 2 only after P_j has been read.
#pragma once

#include "tps_gemm.cuh"

namespace tps {

constexpr int kAttnD = kAttnHeadDim;           // head dimension
constexpr int kAttnBlk = 128;                  // queries per item, keys per block
constexpr int kAttnSoftWarps = 8;
constexpr int kAttnThreads = (3 + kAttnSoftWarps) * 32;
constexpr int kAttnTileBytes = 128 * 128 * 2;  // one 128 x 128 bf16 operand (two 64-wide boxes)
constexpr int kAttnHalf = kAttnTileBytes / 2;  // one 128-row x 64-column box
constexpr int kAttnStages = 3;                 // K and V ring stages
constexpr int kAttnOffQ = 0;
constexpr int kAttnOffK = kAttnOffQ + kAttnTileBytes;
constexpr int kAttnOffV = kAttnOffK + kAttnStages * kAttnTileBytes;
constexpr int kAttnOffBar = kAttnOffV + kAttnStages * kAttnTileBytes;
constexpr int kAttnOffRed = kAttnOffBar + 256;                  // [2 halves][128 rows] fp32
constexpr int kAttnOffFlag = kAttnOffRed + 2 * 128 * 4;         // [2 halves][128 rows] u8
constexpr int kAttnSmemBytes = kAttnOffFlag + 2 * 128 + 1024;
constexpr uint32_t kAttnIdescS = idesc_bf16_f32(128, 128);
constexpr uint32_t kAttnIdescPV = idesc_bf16_f32(128, 128) | (1u << 16);   // A (= P) in TMEM, B (= V) MN-major
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

// D[tmem] (+)= A[tmem] * B[smem desc], bf16 x bf16 -> fp32, one CTA: A is M = 128
// lanes (rows) by K = 16 elements held as 8 columns of packed bf16 pairs.
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

// registers -> TMEM, 32 lanes x 32 columns, and the wait for its completion.
__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Barrier over the two softmax warps of one tensor-memory lane quarter (ids 1..4).
__device__ __forceinline__ void pair_sync(int q) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// 2^x for a pair, x <= 8, on the FMA pipe instead of the special-function unit:
// 2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f from a cubic
// whose coefficients are a minimax fit on that interval (Lawson's iteratively
// reweighted least squares), relative error below 7.5e-5 -- far inside the bf16
// rounding P gets next. j is read from the low mantissa bits of x + 1.5 * 2^23 and
// added to the exponent field. x is clamped to -126 so the exponent cannot wrap: a
// masked score (x = -inf) gives 2^-126 * p (about 1e-38) instead of 0.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x = f2(fmaxf(x.x, -126.0f), fmaxf(x.y, -126.0f));
  const float2 t = __fadd2_rn(x, f2(12582912.0f, 12582912.0f));
  const float2 jf = __fadd2_rn(t, f2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(jf, f2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(f2(0.0551716648f, 0.0551716648f), f, f2(0.2426111251f, 0.2426111251f));
  p = __ffma2_rn(p, f, f2(0.6932609677f, 0.6932609677f));
  p = __ffma2_rn(p, f, f2(0.9999280572f, 0.9999280572f));
  return f2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
            __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// max(a, b, c) in one instruction (the three-input form of max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

struct AttnItem {
  int seq, h, qb, nblk;
  int qcol, kcol, vcol;   // first column of the head's q / k / v in a qkv row
};

// First column of query head h's q, and of its KV head's k and v, in a qkv row: the
// head lives on shard r = h / qs, whose [q | k | v] block starts at r * shard_cols.
__device__ __forceinline__ void attn_head_cols(const AttnArgs& a, int h, int& qcol, int& kcol, int& vcol) {
  const int r = h / a.qs;
  const int lk = h / a.grp - (r * a.kv_first_num) / a.kv_first_den;   // KV head within shard r
  qcol = r * a.shard_cols + (h - r * a.qs) * kAttnD;
  kcol = r * a.shard_cols + (a.qs + lk) * kAttnD;
  vcol = kcol + a.kvs * kAttnD;
}

__device__ __forceinline__ AttnItem attn_item(const AttnArgs& a, int item) {
  AttnItem t;
  const int per = a.nseq * a.hq;
  const int band = item / per;
  const int rem = item - band * per;
  t.qb = a.nqb - 1 - band;                 // heaviest (latest) query blocks first
  t.seq = rem / a.hq;
  t.h = rem - t.seq * a.hq;                // neighbouring CTAs share KV heads in L2
  t.nblk = a.causal ? t.qb + 1 : a.nkb;
  attn_head_cols(a, t.h, t.qcol, t.kcol, t.vcol);
  return t;
}

// Item of this CTA in round r of the persistent loop. Items are numbered heaviest
// first; the CTAs take them in snake order (round 0 left to right, round 1 right to
// left, ...), so the CTA that takes the heaviest item of one round takes the
// lightest of the next (at S = 2048 with 32 heads over 148 SMs the most loaded
// CTA has 31 key blocks of work instead of 38 with a plain stride).
__device__ __forceinline__ int attn_item_of(int r) {
  const int g = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  return r * g + ((r & 1) ? (g - 1 - c) : c);
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
  const uint32_t sBar = base + kAttnOffBar;
  const uint32_t q_full = sBar, q_empty = sBar + 8;
  auto k_full = [&](int i) { return sBar + 16u + 8u * i; };    // [kAttnStages]
  auto k_empty = [&](int i) { return sBar + 40u + 8u * i; };
  auto v_full = [&](int i) { return sBar + 64u + 8u * i; };
  auto v_empty = [&](int i) { return sBar + 88u + 8u * i; };
  auto s_full = [&](int i) { return sBar + 112u + 8u * i; };   // [2]
  auto s_empty = [&](int i) { return sBar + 128u + 8u * i; };
  auto p_full = [&](int i) { return sBar + 144u + 8u * i; };
  auto o_full = [&](int i) { return sBar + 160u + 8u * i; };
  auto o_empty = [&](int i) { return sBar + 176u + 8u * i; };
  const uint32_t pv_done = o_full(0);   // one phase per P V product (every block)
  const uint32_t o_ready = o_full(1);   // one phase per item: its last product is in O
  const uint32_t o_free = o_empty(0);   // one phase per item: the softmax warps have read O
  const uint32_t done_bar = sBar + 192u, epi_done_bar = sBar + 200u;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kAttnOffBar + 208);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kAttnOffBar + 212);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gbase + kAttnOffBar + 216);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kAttnStages; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_empty(i), kAttnSoftWarps);
      mbar_init(p_full(i), kAttnSoftWarps);
      mbar_init(o_full(i), 1);
      mbar_init(o_empty(i), kAttnSoftWarps);
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_done_bar, kAttnSoftWarps);
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
      for (int item = attn_item_of(0); ok && item < a.items; ++it, item = attn_item_of(it)) {
        const AttnItem t = attn_item(a, item);
        const int row0 = t.seq * a.S;
        if (is_k) {
          if (!mbar_wait(q_empty, static_cast<uint32_t>(it & 1) ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full, kAttnTileBytes);
          tma_load_3d(sQ, &tmQKV, q_full, t.qcol, row0 + t.qb * kAttnBlk, 0);
          tma_load_3d(sQ + kAttnHalf, &tmQKV, q_full, t.qcol + 64, row0 + t.qb * kAttnBlk, 0);
          ++nq;
        }
        for (int j = 0; j < t.nblk; ++j, ++n) {
          const int st = static_cast<int>(n % kAttnStages);
          const uint32_t u = static_cast<uint32_t>((n / kAttnStages) & 1);
          const uint32_t emp = is_k ? k_empty(st) : v_empty(st);
          const uint32_t ful = is_k ? k_full(st) : v_full(st);
          if (!mbar_wait(emp, u ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
          const uint32_t dst = (is_k ? sK : sV) + st * kAttnTileBytes;
          const int col = is_k ? t.kcol : t.vcol;
          mbar_arrive_expect_tx(ful, kAttnTileBytes);
          tma_load_3d(dst, &tmQKV, ful, col, row0 + j * kAttnBlk, 0);
          tma_load_3d(dst + kAttnHalf, &tmQKV, ful, col + 64, row0 + j * kAttnBlk, 0);
        }
      }
      // wait (bounded) for the copies still in flight before the CTA may exit
      if (nq > 0) mbar_wait(q_full, static_cast<uint32_t>((nq - 1) & 1), never_flag, 200000000ull, a.status);
      for (long long i = n > kAttnStages ? n - kAttnStages : 0; i < n; ++i)
        mbar_wait(is_k ? k_full(static_cast<int>(i % kAttnStages)) : v_full(static_cast<int>(i % kAttnStages)),
                  static_cast<uint32_t>((i / kAttnStages) & 1), never_flag, 200000000ull, a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      long long g = 0;          // blocks of earlier items
      int it = 0;
      bool ok = true, any = false;
      const uint64_t dq0 = smem_desc_sw128(sQ), dq1 = smem_desc_sw128(sQ + kAttnHalf);
      for (int item = attn_item_of(0); ok && item < a.items; ++it, item = attn_item_of(it)) {
        const AttnItem t = attn_item(a, item);
        if (!mbar_wait(q_full, static_cast<uint32_t>(it & 1), abort_flag, tmo, a.status)) { ok = false; break; }
        tc_fence_after();
        for (int j = 0; j <= t.nblk; ++j) {
          if (j < t.nblk) {
            const long long gj = g + j;
            const int b = static_cast<int>(gj & 1);                      // S / P buffer
            const uint32_t u = static_cast<uint32_t>((gj >> 1) & 1);
            const int r = static_cast<int>(gj % kAttnStages);           // K ring stage
            const uint32_t ur = static_cast<uint32_t>((gj / kAttnStages) & 1);
            if (!mbar_wait(k_full(r), ur, abort_flag, tmo, a.status)) { ok = false; break; }
            // S_j overwrites buffer b: its previous S was read by the softmax warps (s_empty),
            // and the P written there was read by the P V product issued before this MMA
            if (!mbar_wait(s_empty(b), u ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t kb = sK + r * kAttnTileBytes;
            const uint64_t dk0 = smem_desc_sw128(kb), dk1 = smem_desc_sw128(kb + kAttnHalf);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t off = static_cast<uint64_t>((kk & 3) * 2);   // 16 d = 32 B along K
              umma_bf16(tmem_base + b * 128, (kk < 4 ? dq0 : dq1) + off, (kk < 4 ? dk0 : dk1) + off, kAttnIdescS,
                        kk > 0 ? 1u : 0u);
            }
            umma_commit(k_empty(r));
            umma_commit(s_full(b));
            if (j == t.nblk - 1) umma_commit(q_empty);
            any = true;
          }
          if (j >= 1) {
            const int jp = j - 1;
            const long long gp = g + jp;
            const int b = static_cast<int>(gp & 1);
            const uint32_t u = static_cast<uint32_t>((gp >> 1) & 1);
            const int r = static_cast<int>(gp % kAttnStages);           // V ring stage
            const uint32_t ur = static_cast<uint32_t>((gp / kAttnStages) & 1);
            // the first product of an item overwrites O: the previous item's O must have been read
            if (jp == 0 && !mbar_wait(o_free, static_cast<uint32_t>(it & 1) ^ 1u, abort_flag, tmo, a.status)) {
              ok = false;
              break;
            }
            if (!mbar_wait(p_full(b), u, abort_flag, tmo, a.status)) { ok = false; break; }
            if (!mbar_wait(v_full(r), ur, abort_flag, tmo, a.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t vb = sV + r * kAttnTileBytes;
            // A = P_j from tensor memory: 128 query lanes, keys packed two per column in
            // the first 64 columns of S buffer b (8 columns = 16 keys per MMA)
            const uint32_t pa = tmem_base + static_cast<uint32_t>(b * 128);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // 16 keys per MMA: 2048 B (16 rows) of V
              umma_bf16_tmem_a(tmem_base + 256, pa + kk * 8, smem_desc_sw128_mn(vb + kk * 2048, kAttnHalf),
                               kAttnIdescPV, (jp > 0 || kk > 0) ? 1u : 0u);
            umma_commit(v_empty(r));
            umma_commit(pv_done);
            if (jp == t.nblk - 1) umma_commit(o_ready);
          }
        }
        if (!ok) break;
        g += t.nblk;
      }
      // every issued MMA must be complete before tensor memory is released
      if (any) {
        umma_commit(done_bar);
        mbar_wait(done_bar, 0, never_flag, 200000000ull, a.status);
      }
      // ... and every softmax warp must be done reading it
      mbar_wait(epi_done_bar, 0, never_flag, tmo, a.status);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  } else {
    // -------------------------------------------------- softmax and output (warps 3..10)
    // The two warps of a row pair meet only in `exchange` (a 64-thread named
    // barrier, which cannot time out). So that neither ever waits there for a
    // partner that left, a warp whose bounded wait failed does not leave at once:
    // it skips its work up to the next exchange, reports the failure there, and
    // both warps leave together.
    const int q = warp & 3;                       // tensor-memory lane quarter
    const int half = (warp - 3) >> 2;             // keys / output columns [64 half, 64 half + 64)
    const int row = q * 32 + lane;                // query row within the item
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    float* red = reinterpret_cast<float*>(gbase + kAttnOffRed);
    volatile uint8_t* flg = gbase + kAttnOffFlag;
    const int mine = half * 128 + row, other = (half ^ 1) * 128 + row;
    // returns the partner's value; ok becomes false when either warp has failed
    // (the tensor-memory fences order this warp's reads of S before its partner's
    // writes of P into the same columns, after the barrier)
    auto exchange = [&](float v, bool& okp) -> float {
      red[mine] = v;
      flg[mine] = okp ? 1 : 0;
      tc_fence_before();
      pair_sync(q);
      tc_fence_after();
      const float ov = red[other];
      const bool ook = flg[other] != 0;
      pair_sync(q);                               // the slots are free again
      okp = okp && ook;
      return ov;
    };
    const float c = a.scale_log2;
    const uint32_t to = tmem_base + lane_off + static_cast<uint32_t>(256 + half * 64);   // this warp's O columns
    long long g = 0;
    int it = 0;
    bool ok = true;
    for (int item = attn_item_of(0); ok && item < a.items; ++it, item = attn_item_of(it)) {
      const AttnItem t = attn_item(a, item);
      const int qidx = t.qb * kAttnBlk + row;     // query position within the sequence
      float m_ref = -INFINITY;                    // reference max behind P (score units)
      float l_run = 0.f;                          // this half's row sum against m_ref
      for (int j = 0; j < t.nblk; ++j) {
        const long long gj = g + j;
        const int b = static_cast<int>(gj & 1);
        const uint32_t u = static_cast<uint32_t>((gj >> 1) & 1);
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(s_full(b), u, abort_flag, tmo, a.status));
        const int kbase = j * kAttnBlk + half * 64;
        const bool masked = (kbase + 64 > a.S) || (a.causal && j == t.qb);
        const int last = (a.causal ? min(qidx, a.S - 1) : a.S - 1) - kbase;   // last visible key of this half
        float sv[64];
        float mx = -INFINITY;
        if (ok) {
          tc_fence_after();
          const uint32_t ts = tmem_base + lane_off + static_cast<uint32_t>(b * 128 + half * 64);
          tmem_ld64(ts, sv);
          if (masked) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (i > last) sv[i] = -INFINITY;
          }
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent max chains
#pragma unroll
          for (int i = 0; i < 64; i += 2) m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], sv[i], sv[i + 1]);
          mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_empty(b));   // S_j is in registers: its buffer may be refilled
        }
        mx = fmaxf(mx, exchange(mx, ok));          // the block's row max over both halves
        if (!ok) break;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0 || (mx - m_ref) * c > 8.0f) {
          const float m_new = fmaxf(m_ref, mx);
          if (j > 0) {
            alpha = ex2_approx((m_ref - m_new) * c);
            rescale = true;
          }
          m_ref = m_new;
        }
        const float mc = (m_ref == -INFINITY ? 0.f : m_ref) * c;
        if (ok) {
          // P_j as packed bf16 pairs into the first 64 columns of S buffer b (both halves'
          // S are in registers by now): this half's 64 keys are columns [32 half, 32 half + 32)
          uint32_t w[32];
          const float2 c2 = f2(c, c), nmc2 = f2(-mc, -mc);
          float2 r2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};   // row sum: two chains of packed pairs
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 e = __ffma2_rn(f2(sv[2 * i], sv[2 * i + 1]), c2, nmc2);
            // one pair in four on the FMA pipe, the rest on the special-function unit
            const float2 pp = (i & 3) == 3 ? exp2_poly2(e) : f2(ex2_approx(e.x), ex2_approx(e.y));
            r2[i & 1] = __fadd2_rn(r2[i & 1], pp);
            w[i] = pack_bf16(pp.x, pp.y);
          }
          tmem_st32_wait(tmem_base + lane_off + static_cast<uint32_t>(b * 128 + half * 32), w);
          const float rs = (r2[0].x + r2[1].x) + (r2[0].y + r2[1].y);
          l_run = fmaf(l_run, alpha, rs);
        }
        if (ok && __any_sync(0xffffffffu, rescale)) {
          // O must hold the products of every earlier block before it is rescaled. The
          // parity wait on pv_done is exact here: the product of block j-2 is complete
          // (S_j was issued after it) and that of block j cannot start before p_full.
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done, static_cast<uint32_t>((gj - 1) & 1), abort_flag, tmo, a.status));
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              float v[16];
              tmem_ld16(to + cc * 16, v);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] *= alpha;
              tmem_st16_wait(to + cc * 16, v);
            }
          }
        }
        if (ok) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full(b));
        }
      }
      // the item's last product is in O; then agree with the partner
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_ready, static_cast<uint32_t>(it & 1), abort_flag, tmo, a.status));
      const float l_row = l_run + exchange(l_run, ok);
      if (!ok) break;
      g += t.nblk;
      tc_fence_after();
      const float inv = 1.0f / l_row;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) +
                           (static_cast<size_t>(t.seq) * a.S + qidx) * a.ldo + t.h * kAttnD + half * 64;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float v[16];
        tmem_ld16(to + cc * 16, v);
        if (qidx < a.S) {
          uint4 pk0, pk1;
          pk0.x = pack_bf16(v[0] * inv, v[1] * inv);
          pk0.y = pack_bf16(v[2] * inv, v[3] * inv);
          pk0.z = pack_bf16(v[4] * inv, v[5] * inv);
          pk0.w = pack_bf16(v[6] * inv, v[7] * inv);
          pk1.x = pack_bf16(v[8] * inv, v[9] * inv);
          pk1.y = pack_bf16(v[10] * inv, v[11] * inv);
          pk1.z = pack_bf16(v[12] * inv, v[13] * inv);
          pk1.w = pack_bf16(v[14] * inv, v[15] * inv);
          reinterpret_cast<uint4*>(dst + cc * 16)[0] = pk0;
          reinterpret_cast<uint4*>(dst + cc * 16)[1] = pk1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);        // the next item's first product may overwrite O
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_done_bar);
  }
}

// ---------------------------------------------------------------- two query tiles per CTA
// The same attention with a work item of two consecutive 128-query blocks of one
// (sequence, head): tiles A (block 2p) and B (block 2p + 1) share every K and V
// block the CTA streams, and the tensor core alternates between them so that the
// softmax of one tile runs while the products of the other are computed. Tensor
// memory holds S_A, S_B, O_A and O_B (4 x 128 of the 512 columns); each tile has one
// S buffer, into whose first 64 columns its softmax writes P (packed bf16 pairs).
// Per key block j the MMA thread issues, in order,
//   P_A(j-1) V_{j-1} -> O_A,  S_A(j) = Q_A K_j^T,  P_B(j-1) V_{j-1} -> O_B,  S_B(j)
// (shifted by one block: S_A(j+1) follows P_A(j) V_j), so S_X(j) overwrites the P of
// tile X only after the product that reads it, and when the softmax warps of tile X
// see S_X(j) complete, every earlier product into O_X is complete as well: a
// rescale of O_X needs no further wait. Warp 0 loads Q, K and V, warp 1 issues the
// MMAs, softmax warps 2-5 take tile A and 6-9 tile B, one thread per query row and
// all 128 keys of a block, so a row's max and sum need no exchange between warps.
// With a causal mask tile A sees one key block less than tile B (its last block is
// B's diagonal) and skips it; when the query blocks are odd in number the last item
// has tile A only.
constexpr int kAttn2Stages = 2;                                        // K and V ring stages
constexpr int kAttnPolyEvery = 4;                                      // exp2 pairs per FMA-polynomial pair
constexpr int kAttn2Threads = (2 + kAttnSoftWarps) * 32;               // loads, MMA, 2 x 4 softmax warps
constexpr int kAttn2OffQ = 0;                                          // Q_A, Q_B
constexpr int kAttn2OffK = kAttn2OffQ + 2 * kAttnTileBytes;
constexpr int kAttn2OffV = kAttn2OffK + kAttn2Stages * kAttnTileBytes;
constexpr int kAttn2OffBar = kAttn2OffV + kAttn2Stages * kAttnTileBytes;
constexpr int kAttn2SmemBytes = kAttn2OffBar + 256 + 1024;
constexpr uint32_t kA2KF = 16, kA2KE = kA2KF + 8 * kAttn2Stages, kA2VF = kA2KE + 8 * kAttn2Stages,
                   kA2VE = kA2VF + 8 * kAttn2Stages, kA2SF = kA2VE + 8 * kAttn2Stages, kA2PF = kA2SF + 16,
                   kA2OR = kA2PF + 16, kA2OF = kA2OR + 16, kA2Done = kA2OF + 16, kA2Epi = kA2Done + 8,
                   kA2Slot = kA2Epi + 8;
static_assert(kA2Slot + 12 <= 256, "barrier block");
static_assert(kAttn2SmemBytes <= 232448, "shared memory budget");

struct AttnPair {
  int seq, h, qa;          // query tiles A = block qa, B = block qa + 1
  int nA, nB, nblk;        // key blocks of tile A, of tile B (0: no tile B), of the item
  int qcol, kcol, vcol;
};

// Items are numbered heaviest first: band 0 holds the last pair of query blocks of
// every (sequence, head).
__device__ __forceinline__ AttnPair attn_pair(const AttnArgs& a, int item) {
  AttnPair t;
  const int npairs = (a.nqb + 1) >> 1;
  const int per = a.nseq * a.hq;
  const int band = item / per;
  const int rem = item - band * per;
  t.qa = 2 * (npairs - 1 - band);
  t.seq = rem / a.hq;
  t.h = rem - t.seq * a.hq;
  const bool has_b = t.qa + 1 < a.nqb;
  t.nA = a.causal ? t.qa + 1 : a.nkb;
  t.nB = has_b ? (a.causal ? t.qa + 2 : a.nkb) : 0;
  t.nblk = t.nA > t.nB ? t.nA : t.nB;
  attn_head_cols(a, t.h, t.qcol, t.kcol, t.vcol);
  return t;
}

// TMEM -> registers, 32 lanes x 128 columns (two loads, one wait).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float (&v)[128]) {
  uint32_t r[128];
#define TPS_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                  "=r"(r[i + 6]), "=r"(r[i + 7])
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : TPS_R8(0), TPS_R8(8), TPS_R8(16), TPS_R8(24), TPS_R8(32), TPS_R8(40), TPS_R8(48), TPS_R8(56)
      : "r"(taddr)
      : "memory");
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : TPS_R8(64), TPS_R8(72), TPS_R8(80), TPS_R8(88), TPS_R8(96), TPS_R8(104), TPS_R8(112), TPS_R8(120)
      : "r"(taddr + 64u)
      : "memory");
#undef TPS_R8
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// registers -> TMEM, 32 lanes x 8 columns, without the wait (tmem_wait_st).
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t (&w)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(kAttn2Threads, 1)
    tps_attn2_kernel(const __grid_constant__ CUtensorMap tmQKV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kAttn2OffQ;
  const uint32_t sK = base + kAttn2OffK;
  const uint32_t sV = base + kAttn2OffV;
  const uint32_t sBar = base + kAttn2OffBar;
  const uint32_t q_full = sBar, q_empty = sBar + 8;
  auto k_full = [&](int i) { return sBar + kA2KF + 8u * i; };   // [kAttn2Stages]
  auto k_empty = [&](int i) { return sBar + kA2KE + 8u * i; };
  auto v_full = [&](int i) { return sBar + kA2VF + 8u * i; };
  auto v_empty = [&](int i) { return sBar + kA2VE + 8u * i; };
  auto s_full = [&](int x) { return sBar + kA2SF + 8u * x; };   // [tile]: S_X(j) is in tensor memory
  auto p_full = [&](int x) { return sBar + kA2PF + 8u * x; };   // [tile]: P_X(j) is in tensor memory
  auto o_ready = [&](int x) { return sBar + kA2OR + 8u * x; };  // [tile]: the item's last product is in O_X
  auto o_free = [&](int x) { return sBar + kA2OF + 8u * x; };   // [tile]: O_X has been read out
  const uint32_t done_bar = sBar + kA2Done, epi_done_bar = sBar + kA2Epi;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kAttn2OffBar + kA2Slot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kAttn2OffBar + kA2Slot + 4);
  volatile int* never_flag = reinterpret_cast<volatile int*>(gbase + kAttn2OffBar + kA2Slot + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < kAttn2Stages; ++i) {
      mbar_init(k_full(i), 1);
      mbar_init(k_empty(i), 1);
      mbar_init(v_full(i), 1);
      mbar_init(v_empty(i), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), kAttnSoftWarps / 2);
      mbar_init(o_ready(x), 1);
      mbar_init(o_free(x), kAttnSoftWarps / 2);
    }
    mbar_init(done_bar, 1);
    mbar_init(epi_done_bar, kAttnSoftWarps);
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

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ loads: Q, then K_j and V_j in turn.
      // V_j waits for the product P_B(j-2) V_{j-2}, which the tensor core completes before
      // S_B(j-1), the product K_{j+1} waits for: the shared order delays no K load.
      long long n = 0;          // K/V blocks issued
      long long nq = 0;         // Q loads issued
      int it = 0;
      bool ok = true;
      griddep_wait();
      for (int item = attn_item_of(0); ok && item < a.items; ++it, item = attn_item_of(it)) {
        const AttnPair t = attn_pair(a, item);
        const int row0 = t.seq * a.S;
        if (!mbar_wait(q_empty, static_cast<uint32_t>(it & 1) ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
        const int ntiles = t.nB > 0 ? 2 : 1;
        mbar_arrive_expect_tx(q_full, ntiles * kAttnTileBytes);
        for (int x = 0; x < ntiles; ++x) {
          const int r = row0 + (t.qa + x) * kAttnBlk;
          tma_load_3d(sQ + x * kAttnTileBytes, &tmQKV, q_full, t.qcol, r, 0);
          tma_load_3d(sQ + x * kAttnTileBytes + kAttnHalf, &tmQKV, q_full, t.qcol + 64, r, 0);
        }
        ++nq;
        for (int j = 0; ok && j < t.nblk; ++j, ++n) {
          const int st = static_cast<int>(n % kAttn2Stages);
          const uint32_t u = static_cast<uint32_t>((n / kAttn2Stages) & 1);
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const uint32_t emp = kv ? v_empty(st) : k_empty(st);
            const uint32_t ful = kv ? v_full(st) : k_full(st);
            if (!mbar_wait(emp, u ^ 1u, abort_flag, tmo, a.status)) { ok = false; break; }
            const uint32_t dst = (kv ? sV : sK) + st * kAttnTileBytes;
            const int col = kv ? t.vcol : t.kcol;
            mbar_arrive_expect_tx(ful, kAttnTileBytes);
            tma_load_3d(dst, &tmQKV, ful, col, row0 + j * kAttnBlk, 0);
            tma_load_3d(dst + kAttnHalf, &tmQKV, ful, col + 64, row0 + j * kAttnBlk, 0);
          }
          if (!ok) {   // K of this block may be in flight: count the block
            ++n;
            break;
          }
        }
      }
      // wait (bounded) for the copies still in flight before the CTA may exit
      if (nq > 0) mbar_wait(q_full, static_cast<uint32_t>((nq - 1) & 1), never_flag, 200000000ull, a.status);
      for (long long i = n > kAttn2Stages ? n - kAttn2Stages : 0; i < n; ++i) {
        mbar_wait(k_full(static_cast<int>(i % kAttn2Stages)), static_cast<uint32_t>((i / kAttn2Stages) & 1),
                  never_flag, 200000000ull, a.status);
        mbar_wait(v_full(static_cast<int>(i % kAttn2Stages)), static_cast<uint32_t>((i / kAttn2Stages) & 1),
                  never_flag, 200000000ull, a.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      long long n = 0;            // K/V blocks of earlier items
      long long cnt[2] = {0, 0};  // S (and P) blocks of earlier items, per tile
      int its[2] = {0, 0};        // earlier items that had the tile
      int it = 0;
      bool ok = true, any = false;
      auto slot = [&](int j) { return static_cast<int>((n + j) % kAttn2Stages); };
      auto sph = [&](int j) { return static_cast<uint32_t>(((n + j) / kAttn2Stages) & 1); };
      // S_X(j) = Q_X K_j^T into S buffer x (K block j already waited for)
      auto issue_s = [&](int x, int j) {
        const uint32_t kb = sK + slot(j) * kAttnTileBytes;
        const uint32_t qb = sQ + x * kAttnTileBytes;
        const uint64_t dk0 = smem_desc_sw128(kb), dk1 = smem_desc_sw128(kb + kAttnHalf);
        const uint64_t dq0 = smem_desc_sw128(qb), dq1 = smem_desc_sw128(qb + kAttnHalf);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t off = static_cast<uint64_t>((kk & 3) * 2);   // 16 d = 32 B along K
          umma_bf16(tmem_base + x * 128, (kk < 4 ? dq0 : dq1) + off, (kk < 4 ? dk0 : dk1) + off, kAttnIdescS,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full(x));
      };
      for (int item = attn_item_of(0); ok && item < a.items; ++it, item = attn_item_of(it)) {
        const AttnPair t = attn_pair(a, item);
        const int nx[2] = {t.nA, t.nB};
        if (!mbar_wait(q_full, static_cast<uint32_t>(it & 1), abort_flag, tmo, a.status)) { ok = false; break; }
        if (!mbar_wait(k_full(slot(0)), sph(0), abort_flag, tmo, a.status)) { ok = false; break; }
        tc_fence_after();
        if (t.nA > 0) issue_s(0, 0);
        if (t.nB > 0) issue_s(1, 0);
        umma_commit(k_empty(slot(0)));
        if (t.nblk == 1) umma_commit(q_empty);
        any = true;
        for (int j = 0; ok && j < t.nblk; ++j) {
          bool k_next = false;   // K block j + 1 waited for
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (j >= nx[x]) continue;
            // the first product of an item overwrites O_X: the previous item's O_X must be read out
            if (j == 0 && its[x] > 0 &&
                !mbar_wait(o_free(x), static_cast<uint32_t>((its[x] - 1) & 1), abort_flag, tmo, a.status)) {
              ok = false;
              break;
            }
            if (!mbar_wait(p_full(x), static_cast<uint32_t>((cnt[x] + j) & 1), abort_flag, tmo, a.status) ||
                !mbar_wait(v_full(slot(j)), sph(j), abort_flag, tmo, a.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // O_X += P_X(j) V_j: A = P from the first 64 columns of S buffer x (16 keys, 8
            // columns per MMA), B = V read MN-major from its TMA tile (2048 B = 16 keys)
            const uint32_t vb = sV + slot(j) * kAttnTileBytes;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_bf16_tmem_a(tmem_base + 256 + x * 128, tmem_base + x * 128 + kk * 8,
                               smem_desc_sw128_mn(vb + kk * 2048, kAttnHalf), kAttnIdescPV,
                               (j > 0 || kk > 0) ? 1u : 0u);
            if (j == nx[x] - 1) umma_commit(o_ready(x));
            if (j + 1 < nx[x]) {
              if (!k_next) {
                if (!mbar_wait(k_full(slot(j + 1)), sph(j + 1), abort_flag, tmo, a.status)) { ok = false; break; }
                tc_fence_after();
                k_next = true;
              }
              issue_s(x, j + 1);
            }
          }
          if (!ok) break;
          umma_commit(v_empty(slot(j)));
          if (j + 1 < t.nblk) {
            umma_commit(k_empty(slot(j + 1)));
            if (j + 2 == t.nblk) umma_commit(q_empty);   // the item's last S products are issued
          }
        }
        if (!ok) break;
        n += t.nblk;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          cnt[x] += nx[x];
          if (nx[x] > 0) ++its[x];
        }
      }
      // every issued MMA must be complete before tensor memory is released
      if (any) {
        umma_commit(done_bar);
        mbar_wait(done_bar, 0, never_flag, 200000000ull, a.status);
      }
      // ... and every softmax warp must be done reading it
      mbar_wait(epi_done_bar, 0, never_flag, tmo, a.status);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  } else {
    // -------------------------------------------------- softmax and output (warps 2..9)
    const int x = (warp - 2) >> 2;                // query tile: 0 = A (warps 2-5), 1 = B (warps 6-9)
    const int q = warp & 3;                       // tensor-memory lane quarter
    const int row = q * 32 + lane;                // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t ts = tmem_base + lane_off + static_cast<uint32_t>(x * 128);         // S_X / P_X
    const uint32_t to = tmem_base + lane_off + static_cast<uint32_t>(256 + x * 128);   // O_X
    const float c = a.scale_log2;
    long long cnt = 0;   // S blocks of this tile in earlier items
    int its = 0;         // earlier items with this tile
    int it = 0;
    bool ok = true;
    for (int item = attn_item_of(0); ok && item < a.items; ++it, item = attn_item_of(it)) {
      const AttnPair t = attn_pair(a, item);
      const int nb = x ? t.nB : t.nA;
      if (nb == 0) continue;                      // no tile B in this item
      const int qblk = t.qa + x;
      const int qidx = qblk * kAttnBlk + row;     // query position within the sequence
      const int lastq = a.causal ? min(qidx, a.S - 1) : a.S - 1;
      float m_ref = -INFINITY;                    // reference max behind P (score units)
      float l_run = 0.f;                          // row sum of the weights against m_ref
      for (int j = 0; j < nb; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(x), static_cast<uint32_t>((cnt + j) & 1), abort_flag, tmo,
                                               a.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kbase = j * kAttnBlk;
        const bool masked = (kbase + kAttnBlk > a.S) || (a.causal && j == qblk);
        const int last = lastq - kbase;           // last visible key of the block
        // pass 1: the block's row max
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent max chains
        {
          float sv[128];
          tmem_ld128(ts, sv);   // both halves in flight, one wait
          if (masked) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i > last) sv[i] = -INFINITY;
          }
#pragma unroll
          for (int i = 0; i < 128; i += 2) m4[(i >> 1) & 3] = fmax3(m4[(i >> 1) & 3], sv[i], sv[i + 1]);
        }
        const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0 || (mx - m_ref) * c > 8.0f) {
          const float m_new = fmaxf(m_ref, mx);
          if (j > 0) {
            alpha = ex2_approx((m_ref - m_new) * c);
            rescale = true;
          }
          m_ref = m_new;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          // O_X holds every earlier product of the item (they completed before S_X(j))
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            float v[16];
            tmem_ld16(to + cc * 16, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= alpha;
            tmem_st16_wait(to + cc * 16, v);
          }
        }
        // pass 2: P_X(j) as packed bf16 pairs into the first 64 columns of S buffer x (the
        // scores of keys 64-127 sit in columns 64-127, read before any P is written there)
        const float mc = (m_ref == -INFINITY ? 0.f : m_ref) * c;
        const float2 c2 = f2(c, c), nmc2 = f2(-mc, -mc);
        float2 r2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};   // row sum: two chains of packed pairs
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float sv[64];
          tmem_ld64(ts + hh * 64, sv);
          if (masked) {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (hh * 64 + i > last) sv[i] = -INFINITY;
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 e = __ffma2_rn(f2(sv[16 * cc + 2 * i], sv[16 * cc + 2 * i + 1]), c2, nmc2);
              // one pair in kAttnPolyEvery on the FMA pipe: the special-function unit is
              // the busiest unit of the softmax
              const float2 pp = (i % kAttnPolyEvery) == kAttnPolyEvery - 1 ? exp2_poly2(e)
                                                                            : f2(ex2_approx(e.x), ex2_approx(e.y));
              r2[i & 1] = __fadd2_rn(r2[i & 1], pp);
              w[i] = pack_bf16(pp.x, pp.y);
            }
            tmem_st8u(ts + hh * 32 + cc * 8, w);
          }
        }
        tmem_wait_st();
        l_run = fmaf(l_run, alpha, (r2[0].x + r2[1].x) + (r2[0].y + r2[1].y));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(x));
      }
      if (!ok) break;
      // the item's last product is in O_X
      if (!__all_sync(0xffffffffu, mbar_wait(o_ready(x), static_cast<uint32_t>(its & 1), abort_flag, tmo, a.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = 1.0f / l_run;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) +
                           (static_cast<size_t>(t.seq) * a.S + qidx) * a.ldo + t.h * kAttnD;
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        float v[16];
        tmem_ld16(to + cc * 16, v);
        if (qidx < a.S) {
          uint4 pk0, pk1;
          pk0.x = pack_bf16(v[0] * inv, v[1] * inv);
          pk0.y = pack_bf16(v[2] * inv, v[3] * inv);
          pk0.z = pack_bf16(v[4] * inv, v[5] * inv);
          pk0.w = pack_bf16(v[6] * inv, v[7] * inv);
          pk1.x = pack_bf16(v[8] * inv, v[9] * inv);
          pk1.y = pack_bf16(v[10] * inv, v[11] * inv);
          pk1.z = pack_bf16(v[12] * inv, v[13] * inv);
          pk1.w = pack_bf16(v[14] * inv, v[15] * inv);
          reinterpret_cast<uint4*>(dst + cc * 16)[0] = pk0;
          reinterpret_cast<uint4*>(dst + cc * 16)[1] = pk1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free(x));     // the next item's first product may overwrite O_X
      cnt += nb;
      ++its;
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(epi_done_bar);
  }
}

}  // namespace tps
