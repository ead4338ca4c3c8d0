/*
 * tps.h -- C ABI of the tensor-sharded (column/row-parallel) linear block for
 * one NVIDIA B200 (sm_100a).
 *
 * What the library computes (all shards of one tensor-parallel group emulated as
 * separate weight partitions on ONE GPU; the cross-shard "all-reduce" is an
 * on-device reduction, nothing crosses GPUs):
 *
 *   column-parallel  Y = X W,  W = [W_0, ..., W_{tp-1}] split by output columns,
 *                    Y_i = X W_i, Y = concat(Y_i)
 *       -- "Tensor Parallel：当一张 GPU 放不下一个大模型", section "Column Parallel
 *          Linear：按输出维度切"; "张量并行（Tensor Parallelism）推理部署实战", §1.1.
 *   row-parallel     Y = X V,  V = [V_0; ...; V_{tp-1}] split by input rows,
 *                    X = [X_0, ..., X_{tp-1}], P_i = X_i V_i, Y = sum_i P_i
 *       -- same pages, section "Row Parallel Linear：按输入维度切" and §1.2; the sum
 *          (not a concat) is the all-reduce of "Tensor Parallel 深入解析：多加 GPU，
 *          推理为什么可能更慢", section "两张卡如何共同算出一层" (39 + 131 = 170).
 *   MLP              h = act(X W1) column-parallel, Y = h W2 row-parallel, one
 *                    reduction ("张量并行…推理部署实战" §二, Megatron MLP; act = GELU),
 *                    or h = SiLU(X Wg) * (X Wu) ("Tensor Parallel：当一张 GPU 放不下
 *                    一个大模型", section "MLP 里的 tensor parallel").
 *   attention proj.  QKV column-parallel by head, o_proj row-parallel by head
 *                    (section "Attention 里的 tensor parallel"); with GQA, KV heads
 *                    are replicated when tp exceeds the KV-head count ("Tensor
 *                    Parallel 深入解析", section "权重变小，不代表所有显存都按比例变小").
 *   attention        on each shard's own heads between QKV and o_proj: causal GQA
 *                    softmax(Q K^T / sqrt(d)) V per head (section "Attention 里的
 *                    tensor parallel": attention per GPU on its local heads).
 *   greedy lm_head   vocab split column-parallel; each shard's argmax over its vocab
 *                    slice, then the max over shards (section "lm_head 怎么处理").
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Element types: activations and weights are bf16 (IEEE bfloat16, passed as
 *    raw 16-bit storage); products accumulate in fp32 on the tensor cores.
 *    Outputs are bf16 (TPS_DTYPE_BF16, round-to-nearest-even) or fp32.
 *  - All matrices are dense row-major with the leading dimension equal to the
 *    row length (no padding between rows).
 *  - Weights use the math orientation W[k, n] (rows = input features, columns =
 *    output features, Y = X W) unless `transposed` = 1 says the buffer holds
 *    the nn.Linear orientation W^T[n, k].
 *  - Every device pointer must be 16-byte aligned; every per-shard row length
 *    (k, k/tp, n/tp, n, head_dim, I/tp) must be a multiple of 8 elements.
 *  - Ownership: the caller allocates and frees every buffer (inputs, outputs,
 *    packed weights, workspace). The library never allocates device memory.
 *  - Asynchrony: every call enqueues its kernels on `stream` (a cudaStream_t
 *    passed as void*, NULL = legacy default stream) and returns at once. The
 *    returned status covers host-side validation and launch errors only; a
 *    device-side stall is reported later: for a call given a workspace, in the
 *    status word at the start of that workspace (read by tps_sync_status), and
 *    for every call in the library's device-wide word (tps_device_error).
 *  - Workspaces (`ws`, `ws_bytes`): caller-owned device memory, zero-filled
 *    before first use. Its first 256 bytes are a header whose first int is the
 *    status word of the calls given that workspace (TPS_OK, or the
 *    TPS_ERR_TIMEOUT / TPS_ERR_DEVICE of a failed call); the split-K slots,
 *    tile counters, readiness flags and argmax entries follow the header. A
 *    workspace smaller than its header carries no status word.
 *  - Overlap with the previous kernel: the GEMM kernels are launched with
 *    programmatic stream serialization. A GEMM's CTAs may be scheduled while the
 *    previous kernel of the stream drains and set up their shared and tensor
 *    memory; they read or write global memory only after that kernel has
 *    completed, so stream order is kept for every buffer.
 *  - Errors: no exception crosses the ABI. Invalid arguments are rejected
 *    before any CUDA call and nothing is enqueued.
 *  - m = 0 is a valid empty problem: the call validates and returns TPS_OK
 *    without launching anything.
 */
#ifndef TPS_H
#define TPS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TPS_API __attribute__((visibility("default")))
#else
#define TPS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TPS_OK = 0,
  TPS_ERR_ARG = -1,           /* null pointer, bad enum, negative size, bad combination */
  TPS_ERR_DIVISIBILITY = -2,  /* tp does not divide the split dimension / head counts */
  TPS_ERR_ALIGN = -3,         /* pointer not 16-B aligned or row length not a multiple of 8 */
  TPS_ERR_DTYPE = -4,         /* unsupported output dtype */
  TPS_ERR_WORKSPACE = -5,     /* workspace or packed buffer too small */
  TPS_ERR_CUDA = -6,          /* a CUDA runtime/driver call failed (launch, tensor map) */
  TPS_ERR_TIMEOUT = -7,       /* a bounded device-side wait expired (tps_device_error) */
  TPS_ERR_UNIMPLEMENTED = -8, /* valid request outside what this library supports */
  TPS_ERR_DEVICE = -9         /* current device is not an sm_100 (B200-class) GPU */
} tps_status;

/* Weight kinds (how a logical weight is split into shards). */
enum {
  TPS_KIND_COLUMN = 0,  /* W[k, n] split by output columns: shard i = W[:, i*n/tp : (i+1)*n/tp] */
  TPS_KIND_ROW = 1,     /* V[k, n] split by input rows:     shard i = V[i*k/tp : (i+1)*k/tp, :] */
  TPS_KIND_QKV = 2,     /* W[k, (hq+2*hkv)*d] = [Wq | Wk | Wv], split by attention head */
  TPS_KIND_GATE_UP = 3  /* W[k, 2*I] = [Wg | Wu], both split by output columns */
};

/* Epilogue activations of the column-parallel layer. */
enum {
  TPS_ACT_NONE = 0,
  TPS_ACT_GELU = 1,      /* exact form 0.5*y*(1+erf(y/sqrt(2))), kinds COLUMN */
  TPS_ACT_SILU_MUL = 2   /* h = SiLU(gate) * up, kind GATE_UP only (and required there) */
};

enum { TPS_DTYPE_BF16 = 0, TPS_DTYPE_F32 = 1 };

/* Row-parallel reduction modes. */
enum {
  TPS_REDUCE_FUSED = 0,    /* partial sums reduced inside the GEMM (accumulator / split-K fix-up) */
  TPS_REDUCE_PARTIALS = 1, /* write every P_i to `partials` [tp][m][n] fp32, then shard_partial_reduce */
  TPS_REDUCE_BF16 = 2      /* the partials exchanged in bf16 (see row_parallel_forward) */
};

/* Function ids for tps_workspace_bytes(). */
enum { TPS_FN_COLUMN = 0, TPS_FN_ROW = 1, TPS_FN_MLP = 2, TPS_FN_ATTN = 3, TPS_FN_ARGMAX = 4 };

/* Attention head geometry (QKV kind and the attention composite). */
typedef struct {
  int32_t hq;        /* query heads */
  int32_t hkv;       /* KV heads (GQA); hq % hkv == 0 */
  int32_t head_dim;  /* d, multiple of 8 */
} tps_heads;

/*
 * tp_head_map -- query/KV head to shard assignment.
 *   Shard r holds query heads [q_first[r], q_first[r] + q_count[r]) with
 *   q_count = hq/tp (contiguous blocks: 32 heads over tp=4 -> heads 0-7, 8-15, ...,
 *   "Tensor Parallel：当一张 GPU 放不下一个大模型", section "Attention 里的 tensor
 *   parallel"). KV heads: [kv_first[r], kv_first[r] + kv_count[r]); when tp divides
 *   hkv, kv_count = hkv/tp; when tp > hkv (hkv divides tp) every shard holds the one
 *   head floor(r*hkv/tp), i.e. each KV head is replicated tp/hkv times ("Tensor
 *   Parallel 深入解析", section "权重变小，不代表所有显存都按比例变小").
 *   Output arrays are HOST arrays of length tp, owned by the caller; any may be NULL.
 *   Errors: TPS_ERR_ARG for non-positive sizes, TPS_ERR_DIVISIBILITY when tp does
 *   not divide hq ("张量并行…推理部署实战" §6.3), hkv does not divide hq, or neither of
 *   tp, hkv divides the other. Host-only; no GPU needed.
 */
TPS_API int tp_head_map(int hq, int hkv, int tp, int32_t* q_first, int32_t* q_count,
                int32_t* kv_first, int32_t* kv_count);

/*
 * tp_packed_bytes -- size in bytes of the packed (sharded) form of a weight.
 *   Every shard s is one contiguous partition holding R packed rows of Kp
 *   elements (one packed row = one output feature's input weights, K-major):
 *     kind COLUMN : W[k, n]            -> R = n/tp, Kp = k; row r = column s*n/tp + r of W
 *     kind ROW    : V[k, n]            -> R = n,    Kp = k/tp; row r = column r of
 *                                         V[s*k/tp : (s+1)*k/tp, :]
 *     kind QKV    : W[k, (hq+2hkv)*d]  -> R = (hq/tp + 2*kvs)*d, Kp = k; shard s's rows are
 *                                         [its q heads | its k heads | its v heads],
 *                                         kvs = KV heads per shard (tp_head_map), replicas included
 *     kind GATE_UP: W[k, 2*I]          -> Is = I/tp, R = 256*ceil(Is/128), Kp = k; rows
 *                                         [256j, 256j+128) are gate columns s*Is + 128j + (0..127),
 *                                         rows [256j+128, 256j+256) the same up columns
 *   The rows and K are stored in tiles: shard s is [RB][KB][128][64] bf16 with
 *   RB = ceil(R/128) and KB = ceil(Kp/64), i.e. element (r, c) of shard s sits at
 *   ((s*RB + r/128)*KB + c/64)*8192 + (r%128)*64 + c%64. Rows and K indices in the
 *   padding are zero. Total bytes = tp * RB*128 * KB*64 * 2.
 *   `heads` is read for kind QKV only. Returns 0 on invalid arguments. Host-only.
 */
TPS_API size_t tp_packed_bytes(int kind, int64_t k, int64_t n, int tp, const tps_heads* heads);

/*
 * tp_shard_weights -- one-time split of a full weight into its tp shards, in the
 *   packed layout above (weights are static and are split once at start-up,
 *   "张量并行…推理部署实战" §三, 差异二).
 *   W: device, bf16, W[k, n] (transposed = 0) or W^T[n, k] (transposed = 1).
 *   packed: device, caller-owned, at least tp_packed_bytes(...) bytes.
 *   A pure bit copy (no arithmetic). Errors: TPS_ERR_ARG, TPS_ERR_DIVISIBILITY,
 *   TPS_ERR_ALIGN, TPS_ERR_WORKSPACE (packed_bytes too small), TPS_ERR_CUDA.
 */
TPS_API int tp_shard_weights(int kind, const void* W, int transposed, int64_t k, int64_t n, int tp,
                     const tps_heads* heads, void* packed, size_t packed_bytes, void* stream);

/*
 * column_parallel_forward -- Y_i = act(X W_i + b_i) for every shard, written
 *   side by side so that the output buffer IS concat(Y_i) (no communication).
 *   X: device bf16 [m, k], replicated input of every shard.
 *   packed_w: packed weight of `kind` (COLUMN, QKV or GATE_UP); n is the logical
 *     column count (COLUMN: n, QKV: (hq+2hkv)*d, GATE_UP: 2*I).
 *   bias: device bf16 in logical column order ([n]; QKV [(hq+2hkv)*d]; GATE_UP
 *     [2*I] = [b_gate | b_up]) or NULL.
 *   act: NONE or GELU for COLUMN; NONE for QKV; SILU_MUL for GATE_UP.
 *   Y: device [m, n_out] of y_dtype, n_out = n (COLUMN), tp*(hq/tp+2*kvs)*d (QKV,
 *     shard-major [q|k|v] blocks, replicated KV heads appear once per shard), I
 *     (GATE_UP, h = SiLU(gate)*up; shard r at columns [r*I/tp, (r+1)*I/tp)).
 *   ws/ws_bytes: optional workspace (may be NULL/0) used by split-K plans for
 *     small m and for the call's status word; see tps_workspace_bytes. It must be
 *     zero-filled before its first use; every call that completes leaves its
 *     status word, tile counters and flags zero again (its split-K segment slots
 *     keep partial sums that every call writes before it reads them).
 */
TPS_API int column_parallel_forward(const void* X, int64_t m, int64_t k, const void* packed_w, int kind,
                            int64_t n, int tp, const tps_heads* heads, const void* bias, int act,
                            void* Y, int y_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * row_parallel_forward -- Y = sum_{i=0}^{tp-1} X_i V_i (+ bias, added once after
 *   the sum).
 *   X: device bf16 [m, k]; shard i consumes columns [i*k/tp, (i+1)*k/tp).
 *   packed_v: packed ROW weight of V[k, n].
 *   bias: device bf16 [n] or NULL.
 *   reduce_mode FUSED: the cross-shard sum happens inside the GEMM (one fp32
 *     accumulator walks all shards' K ranges; when the tile count is too small for
 *     the GPU, shard/K segments are split across CTAs and the last CTA of a tile
 *     sums the fp32 segment partials from `ws` in fixed K order -- deterministic).
 *   reduce_mode PARTIALS: every P_i is written to `partials` (device fp32
 *     [tp][m][n], caller-owned) and then reduced by shard_partial_reduce.
 *   reduce_mode BF16: the numerics of an all-reduce of bf16 activations ("张量并行
 *     …推理部署实战" §5.1: the deployment's all-reduce runs on the bf16 outputs of
 *     the row-parallel layer; the pages fix no order, so shard order is taken):
 *     every P_i (fp32 accumulation) is rounded to bf16, the rounded partials are
 *     added in shard order 0, 1, ..., tp-1 with a bf16 rounding after every
 *     addition, and the bias is added once at the end with one more rounding
 *     (Y holds bf16 values also when y_dtype is fp32). With partials = NULL it
 *     runs inside one GEMM, for any tp: tp = 2, 4, 8 with weight-major tiles or a
 *     small token-major problem (a cost model decides) as a thread-block cluster of
 *     tp CTAs per tile (CTA r computes shard r's partial, the partials meet in
 *     distributed shared memory); otherwise as a shard chain
 *     (one CTA per tile walks the shards in order, a fresh accumulator per shard,
 *     and folds each partial into the running bf16 sum held in tensor memory).
 *     With a `partials` buffer (fp32 [tp][m][n]) it runs as the GEMM writing P_i
 *     followed by shard_partial_reduce_bf16.
 *   Y: device [m, n] of y_dtype.
 */
TPS_API int row_parallel_forward(const void* X, int64_t m, int64_t k, const void* packed_v, int64_t n,
                         int tp, const void* bias, int reduce_mode, float* partials, void* Y,
                         int y_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * shard_partial_reduce -- the standalone on-device all-reduce of tp partial sums:
 *   Y[r, c] = ((P_0[r,c] + P_1[r,c]) + ...) + P_{tp-1}[r,c] (+ bias[c]), fp32, in shard
 *   order. partials: device fp32 [tp][m][n]; bias: device bf16 [n] or NULL;
 *   Y: device [m, n] of y_dtype. n must be a multiple of 4.
 */
TPS_API int shard_partial_reduce(const float* partials, int tp, int64_t m, int64_t n, const void* bias,
                         void* Y, int y_dtype, void* stream);

/*
 * shard_partial_reduce_bf16 -- the standalone exchange of bf16 partials: every
 *   P_s[r, c] is rounded to bf16 (round to nearest, ties to even), then
 *   Y[r, c] = bf16(...bf16(bf16(P_0) + bf16(P_1)) + ... + bf16(P_{tp-1})), and with
 *   a bias, Y = bf16(Y + bias[c]) -- the numerics of an all-reduce of bf16
 *   activations in shard order ("张量并行…推理部署实战" §5.1). Arguments, layouts and
 *   errors as shard_partial_reduce.
 */
TPS_API int shard_partial_reduce_bf16(const float* partials, int tp, int64_t m, int64_t n, const void* bias,
                                      void* Y, int y_dtype, void* stream);

/*
 * sharded_mlp_forward -- the MLP block: h = act(column(X)), Y = row(h), one
 *   reduction. act = GELU: packed_up is a COLUMN pack of W1[H, I] (fc1). act =
 *   SILU_MUL: packed_up is a GATE_UP pack of [Wg | Wu] ([H, 2I]). packed_down is a
 *   ROW pack of W2[I, H]. h_ws: device bf16 [m, I], caller-owned, receives the
 *   intermediate (shard r at columns [r*I/tp, (r+1)*I/tp)). Y: device [m, H].
 *   No bias (the pages' MLP blocks are bias-free; zero bias in every workload).
 *   Equivalent to column_parallel_forward followed by row_parallel_forward (FUSED).
 *   Given a workspace (tps_workspace_bytes with TPS_FN_MLP), the block runs as
 *   ONE kernel when every cluster of its row phase can be resident at once --
 *   act = GELU with more than 64 tokens (token-major tiles), act = SILU_MUL with
 *   at most 64 tokens (weight-major gate/up pairs): column tiles first, then the
 *   row GEMM's tiles, each starting on a shard as soon as all of that shard's
 *   column tiles are in h (the row layer's shard r reads only the column layer's
 *   shard r), with flags in the workspace that the kernel leaves zero. Otherwise
 *   it launches the two GEMMs.
 */
TPS_API int sharded_mlp_forward(const void* X, int64_t m, int64_t H, int64_t I, int tp, int act,
                        const void* packed_up, const void* packed_down, void* h_ws, void* Y,
                        int y_dtype, void* ws, size_t ws_bytes, void* stream);

/*
 * vocab_parallel_argmax -- greedy decoding over a vocab-parallel lm_head
 *   ("Tensor Parallel：当一张 GPU 放不下一个大模型", section "lm_head 怎么处理": the
 *   lm_head is split by vocab = column parallel, each rank finds the largest logit
 *   of its vocab slice, then the largest over ranks is taken). logits = X W with
 *   W[H, V] given as a COLUMN pack (shard r = vocab [r*V/tp, (r+1)*V/tp)); for
 *   every token: each shard's local argmax, then the max over shards, ties going
 *   to the lowest vocab index. No logits are written. X: device bf16 [m, H];
 *   out_idx: device int32 [m] (vocab index); out_val: device fp32 [m] (the
 *   largest logit) or NULL; ws: device workspace of at least
 *   tps_workspace_bytes(TPS_FN_ARGMAX, m, V, H, tp) bytes (required), no
 *   initial contents needed. Errors: TPS_ERR_WORKSPACE when ws is smaller.
 */
TPS_API int vocab_parallel_argmax(const void* X, int64_t m, int64_t H, const void* packed_w, int64_t V, int tp,
                                  int32_t* out_idx, float* out_val, void* ws, size_t ws_bytes, void* stream);

/*
 * sharded_attn_proj_forward -- the attention block's two projections.
 *   qkv_out = column-parallel QKV of X (kind QKV, layout as column_parallel_forward,
 *   bf16) and Y = row-parallel o_proj of attn_out [m, hq*d] (shard r owns the
 *   columns of its query heads), reduced across shards. packed_o is a ROW pack of
 *   Wo[hq*d, H]. Y: device [m, H] of y_dtype.
 */
TPS_API int sharded_attn_proj_forward(const void* X, const void* attn_out, int64_t m, int64_t H,
                              const tps_heads* heads, int tp, const void* packed_qkv,
                              const void* packed_o, void* qkv_out, void* Y, int y_dtype,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * sharded_gqa_attention -- attention on local heads, the step between the
 *   column-parallel QKV and the row-parallel o_proj ("Tensor Parallel：当一张 GPU
 *   放不下一个大模型", section "Attention 里的 tensor parallel": each shard holds the
 *   q/k/v of its own heads and computes their attention locally; the output stays
 *   split by head). For every query head h (shard r = h / (hq/tp)) and sequence:
 *   O_h = softmax(Q_h K_g^T / sqrt(d)) V_g with g = h / (hq/hkv) the head's KV
 *   group, read from shard r's own [q | k | v] block (a replicated KV head is read
 *   from the copy in r's block). causal = 1: query t sees keys 0..t of its own
 *   sequence; 0: all keys of its sequence. Softmax in fp32; the weights are
 *   rounded to bf16 for the weights-times-V product (fp32 accumulation).
 *   qkv: device bf16 [nseq*seqlen, tp*(hq/tp + 2*kvs)*d], the QKV layout that
 *     column_parallel_forward writes for kind QKV (row b*seqlen + t = token t of
 *     sequence b). attn_out: device bf16 [nseq*seqlen, hq*d], caller-owned; query
 *     head h at columns [h*d, (h+1)*d) -- the input layout of the o_proj row pack.
 *   head_dim must be 128 (TPS_ERR_UNIMPLEMENTED otherwise). Errors: TPS_ERR_ARG,
 *   TPS_ERR_DIVISIBILITY (head map), TPS_ERR_ALIGN (16-byte pointers),
 *   TPS_ERR_DEVICE, TPS_ERR_CUDA. Asynchronous on `stream`; bounded device waits
 *   (tps_device_error reports a timeout).
 */
TPS_API int sharded_gqa_attention(const void* qkv, int64_t nseq, int64_t seqlen, const tps_heads* heads,
                                  int tp, int causal, void* attn_out, void* stream);

/*
 * row_parallel_forward_noalloc -- row_parallel_forward (FUSED reduction) for
 *   callers that cannot allocate device memory and cannot hand in a workspace:
 *   for example an inference engine that has reserved all device memory up
 *   front under a fixed memory plan, or code running inside a region where it
 *   must not call the allocator. The pages have no counterpart of this call; it
 *   exists only for such callers.
 *   Instead of a caller workspace it uses a scratch array that lives in the
 *   library itself (a file-scope device array of 12 MiB, held by every GPU that
 *   loads the library until the process exits) for the split-K segment partials
 *   and tile counters. It allocates nothing (no cudaMalloc, cudaFree or
 *   allocating library call). Limit: m <= 64 tokens (the decode sizes the scratch
 *   is sized for); larger m returns TPS_ERR_WORKSPACE without launching anything.
 *   Arguments, layouts and the other errors are those of row_parallel_forward.
 *   The first call on a device looks up the scratch array's device address (once
 *   per device, with that device current), so make the first call before any
 *   stream capture. Every call clears the counters it needs on `stream` and
 *   shares the one scratch array: calls that overlap on the GPU (different
 *   streams, or host threads, without ordering between them) race on it and
 *   must be serialised by the caller.
 */
TPS_API int row_parallel_forward_noalloc(const void* X, int64_t m, int64_t k, const void* packed_v, int64_t n,
                                         int tp, const void* bias, void* Y, int y_dtype, void* stream);

/*
 * tps_workspace_bytes -- workspace size that lets every plan of `fn` use its
 *   preferred split. fn = TPS_FN_COLUMN (n = packed rows, i.e. the logical n for
 *   COLUMN, 2*I for GATE_UP), TPS_FN_ROW (n = output width, k = input width),
 *   TPS_FN_MLP (n = H, k = I; gated MLP needs the same or less),
 *   TPS_FN_ATTN (n = H, k = hq*d), TPS_FN_ARGMAX (n = V, k = H: the per-tile
 *   maxima of vocab_parallel_argmax, required). Plans given a smaller workspace fall back to
 *   fewer splits (never to an error). Uses the current device's SM count when a
 *   GPU is present, else 148. Returns 0 for invalid arguments.
 */
TPS_API size_t tps_workspace_bytes(int fn, int64_t m, int64_t n, int64_t k, int tp);

/* Human-readable name of a tps_status value (static string). */
TPS_API const char* tps_status_string(int status);

/*
 * tps_sync_status -- the status of the calls given workspace `ws`
 *   ("Asynchrony" above): synchronizes `stream` (the stream those calls were
 *   enqueued on), reads the status word at the start of `ws`, clears it and
 *   returns it: TPS_OK, TPS_ERR_TIMEOUT (a bounded wait inside one of those
 *   calls' kernels expired) or TPS_ERR_DEVICE (a cluster kernel found itself
 *   launched without its cluster shape). Calls on other workspaces -- e.g. on
 *   another stream -- do not touch this word, so a failure is reported to the
 *   caller whose call failed. After a failure, outputs of that call are
 *   undefined and the rest of `ws` must be zeroed again before reuse.
 *   ws: device, 16-byte aligned, at least 256 bytes. Errors: TPS_ERR_ARG (null
 *   or unaligned ws), TPS_ERR_CUDA.
 */
TPS_API int tps_sync_status(void* ws, void* stream);

/*
 * tps_device_error -- synchronizes `stream`, then returns and clears the
 *   library's device-wide error word for the current device (set by a failed
 *   kernel of any call, with or without a workspace): TPS_OK, or
 *   TPS_ERR_TIMEOUT when a bounded wait inside a kernel expired (the kernel then
 *   skipped the rest of its work, released its tensor memory and returned), or
 *   TPS_ERR_DEVICE when a kernel that exchanges data inside a thread-block
 *   cluster found itself launched without that cluster shape (it then returned
 *   at entry without doing its work). After either, outputs are undefined and a
 *   workspace given to the failed call must be zeroed again before reuse.
 */
TPS_API int tps_device_error(void* stream);

/*
 * tps_set_plan_override -- testing/benchmark hook, process-wide, that forces
 *   the GEMM plan of subsequent calls: 0 = automatic; low bits 1 = token-major
 *   tiles (tokens on the MMA M side), 2 = weight-major tiles (weight rows on the
 *   MMA M side); +16 forces split-K (stream-K) whenever a workspace is given,
 *   +32 forbids it; bits 8-11 force the tile width on the non-M side
 *   (1 = 16, 2 = 32, 3 = 64, 4 = 128, 5 = 256 columns; token-major tiles take
 *   64/128/256, weight-major 16..128; gate/up token-major tiles are always 256);
 *   +64 prefers token-major tiles of 256 tokens on a CTA pair (two SMs, one
 *   cluster) whenever the problem has more than 128 tokens, +128 forbids them;
 *   bit 16 (65536) prefers cluster split-K for row-parallel GEMMs (the CTAs of
 *   a cluster each take a share of K of one tile and reduce through distributed
 *   shared memory) whenever it fits, bit 17 forbids it; bits 12-13 restrict its
 *   cluster size (1 = 2, 2 = 4, 3 = 8 CTAs); bit 18 requires the one-launch form
 *   of sharded_mlp_forward (TPS_ERR_UNIMPLEMENTED when it cannot run), bit 19
 *   forbids it; bit 20 prefers wide CTA-pair tiles (256 tokens x 512 weight rows)
 *   where the shard's weight rows are a whole number of them, bit 21 forbids
 *   them; bit 22 selects the stream-K form of the one-launch gated MLP (every CTA
 *   streams both layers), bit 23 the cluster form; bits 24-26 (v = 1..7) set
 *   the tile raster's token-tile group to 2^(v-1) (0 = 16); bit 27 runs
 *   sharded_gqa_attention with one 128-query block per work item instead of two;
 *   bit 28 drops the L2 evict-last policy of CTA-pair tiles' token rows, bit 29
 *   loads their weights with evict-first; bit 30 runs the fused bf16 exchange
 *   (TPS_REDUCE_BF16 without a partials buffer) as the shard chain, bit 14 as a
 *   cluster of tp CTAs per tile (tp = 2, 4, 8), whichever the planner would
 *   choose. Returns the previous value.
 */
TPS_API int tps_set_plan_override(int plan);

/*
 * tps_debug_wait_timeout -- self-test of the bounded device wait: launches one
 *   CTA that waits on a shared-memory barrier nothing will ever complete, with a
 *   limit of `timeout_us` microseconds (1..1000000). The kernel records
 *   TPS_ERR_TIMEOUT in the device-wide word and, when `ws` is given (device,
 *   16-byte aligned, ws_bytes >= 256), in that workspace's status word, then
 *   returns; read them with tps_device_error() and tps_sync_status(). Nothing
 *   faults, traps or hangs. Errors: TPS_ERR_ARG, TPS_ERR_WORKSPACE (ws_bytes <
 *   256), TPS_ERR_ALIGN.
 */
TPS_API int tps_debug_wait_timeout(int timeout_us, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TPS_H */
