/*
 * mla_decode.h — C ABI of the B200 (sm_100a) MLA latent-cache decode library.
 *
 * One call of mla_decode_run performs one decode step of Multi-Head Latent
 * Attention in its absorbed form over a paged latent KV cache:
 *
 *   q_lat[b,t,h,:] = q_nope[b,t,h,:] . W_UK[h]                      (absorb)
 *   s[j]   = scale * (q_lat . cKV[b,j] + q_rope[b,t,h] . k_rope[b,j]),  j <= L_b - Lq + t
 *   o_lat  = softmax(s) . cKV[b, :]                                  (latent accumulation)
 *   out[b,t,h,:] = o_lat . W_UV[h]                                   (up-projection)
 *
 * Sources: the TPLA abstract (latent cKV cache; partition of the latent and of
 * each head's input dimension, independent attention per shard, summed
 * results), "TransMLA: Multi-Head Latent Attention Is All You Need" abstract
 * (the Absorb operation keeps the cache compressed), the pith.science verdict
 * record for 2502.07864 (key_machinery: absorbed form is exact; core_discovery:
 * one RoPE key per token common to all heads; referee report on Eq. 26: the
 * MQA form).
 *
 * Layouts (row-major, last dimension contiguous, element type = dims.dtype):
 *   q_nope   [B, Lq, H, d_nope]
 *   q_rope   [B, Lq, H, d_rope]   query after RoPE (decode applies no rotation)
 *   kv_cache [num_blocks, page_size, r + d_rope]; columns [0, r) are cKV,
 *            columns [r, r + d_rope) the decoupled RoPE key (after RoPE)
 *   block_table int32 [B, block_table_stride]; entry (b, i) is the block that
 *            holds tokens [i*page_size, (i+1)*page_size) of sequence b. The
 *            slots of a sequence's last block past L_b are read (whole pages
 *            move) and their cKV weighted by exactly 0: their cKV columns must
 *            hold finite values (any; 0 * NaN would still be NaN).
 *   seq_lens int32 [B], L_b counts the Lq query tokens (they are the newest
 *            Lq cache rows; query t sees keys j <= L_b - Lq + t)
 *   w_uk     [H, d_nope, r]     w_uv [H, r, d_v]
 *   out      [B, Lq, H, d_v]
 * TPLA (latent_shards = S > 1): shard s owns latent columns
 * [s*r/S, (s+1)*r/S) of cKV, of W_UK[h] and of W_UV[h]; every shard adds the
 * full RoPE score and has its own softmax; the shard outputs are summed.
 *
 * Ownership: the caller owns every device buffer, including the workspace;
 * the library owns only the plan (host memory). mla_decode_run does not
 * allocate, synchronise or read device memory on the host, so a stream may be
 * captured into a CUDA graph around it.
 *
 * Errors: every call returns an mla_status_t; nothing aborts the process and
 * no exception crosses the ABI. Errors found on the device (a block-table
 * entry outside [0, num_blocks), a sequence length outside
 * [Lq, block_table_stride * page_size], a bounded wait that ran out) are
 * recorded in a status word inside the workspace; the affected work is
 * skipped (never read out of bounds) and mla_decode_read_status returns the
 * first recorded code.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 1

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,         /* null pointer, non-positive size, bad length */
  MLA_ERR_UNSUPPORTED = 2,         /* dims outside what the kernels implement */
  MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes below the plan's size */
  MLA_ERR_CUDA = 4,                /* a CUDA runtime call failed */
  MLA_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait ran out */
  MLA_ERR_BOUNDS = 6,              /* block id or sequence length out of range */
  MLA_ERR_NO_DEVICE = 7            /* no usable sm_100 device */
} mla_status_t;

/* MLA_FP8_CACHE: activations, weights and output bf16; the cache holds per
 * token r E4M3 codes of cKV, one fp32 scale s_t and the RoPE key in bf16
 * divided by s_t (see mla_decode_run_fp8). Tensor-core path, one latent shard. */
typedef enum { MLA_BF16 = 0, MLA_FP32 = 1, MLA_FP8_CACHE = 2 } mla_dtype_t;

/* Kernel family selection (mla_plan_options_t.kernel). */
typedef enum {
  MLA_KERNEL_AUTO = 0,    /* tcgen05 path where supported, else SIMT */
  MLA_KERNEL_SIMT = 1,    /* CUDA-core fp32 path (all dims; the fp32 path) */
  MLA_KERNEL_TCGEN05 = 2  /* tensor-core path: d_rope = 64, d_nope = d_v = 128, H*Lq <= 128;
                             bf16 with r = 512 (1 or 2 latent shards) or r = 256 (1 shard:
                             one TPLA shard per GPU), or the FP8 cache with r = 512 */
} mla_kernel_t;

typedef struct {
  int32_t num_heads;      /* H */
  int32_t latent_rank;    /* r (cKV width) */
  int32_t rope_dim;       /* d_rope */
  int32_t nope_dim;       /* d_nope (W_UK rows per head) */
  int32_t v_dim;          /* d_v (W_UV columns per head) */
  int32_t q_len;          /* Lq query tokens per sequence (1, or 2 for MTP) */
  int32_t page_size;      /* tokens per cache block; 64 */
  int32_t latent_shards;  /* 1 = MLA, 2 = TPLA two-shard form */
  float softmax_scale;    /* multiplies q.k; usually 1/sqrt(d_nope + d_rope) */
  int32_t dtype;          /* mla_dtype_t of every tensor argument */
} mla_dims_t;

typedef struct {
  int32_t num_sms;        /* SMs to plan for; 0 = query the current device */
  int32_t kernel;         /* mla_kernel_t */
  int32_t num_workers;    /* 0 = automatic; else the number of page ranges */
} mla_plan_options_t;

typedef struct {
  int32_t batch;
  int32_t rows;             /* H * Lq rows per sequence */
  int32_t kernel;           /* mla_kernel_t that mla_decode_run launches */
  int32_t num_workers;      /* page ranges (one CTA pair each on tcgen05) */
  int32_t num_split_slots;  /* partial-result slots = num_workers + batch - 1 */
  int32_t launches_per_run; /* kernels one mla_decode_run launches */
  int64_t total_pages;      /* sum over b of ceil(L_b / page_size) at plan time */
  uint64_t workspace_bytes;
} mla_plan_info_t;

typedef struct mla_plan* mla_plan_t; /* opaque, library-owned host object */

/* Supported-dims check and workspace sizing for a batch.
 * seq_lens_host [batch] (host memory) gives the lengths the plan balances;
 * the device lengths passed to run may differ as long as each stays in
 * [Lq, block_table_stride * page_size]: the split partition is recomputed
 * on the device every run, so only balance (not correctness) depends on the
 * plan-time lengths. batch >= 1: an empty batch has nothing to decode and is
 * refused with MLA_ERR_INVALID_ARG. On success *plan_out receives a new plan
 * (free it with mla_plan_destroy) and *workspace_bytes the workspace size run
 * needs. */
mla_status_t mla_decode_plan(const mla_dims_t* dims, int32_t batch,
                             const int32_t* seq_lens_host, int32_t num_sms,
                             mla_plan_t* plan_out, size_t* workspace_bytes);

/* mla_decode_plan with explicit options (kernel family, worker count);
 * opts may be NULL for the defaults. */
mla_status_t mla_decode_plan_ex(const mla_dims_t* dims, int32_t batch,
                                const int32_t* seq_lens_host,
                                const mla_plan_options_t* opts,
                                mla_plan_t* plan_out, size_t* workspace_bytes);

/* One decode step, enqueued on `stream` (a cudaStream_t; NULL = legacy default
 * stream). All pointers are device pointers except `plan`. The workspace must
 * hold at least the plan's workspace_bytes and may not be shared by two runs
 * in flight at once. Returns MLA_OK once the kernels are enqueued. */
mla_status_t mla_decode_run(mla_plan_t plan,
                            const void* q_nope, const void* q_rope,
                            const void* kv_cache, int64_t num_blocks,
                            const int32_t* block_table, int32_t block_table_stride,
                            const int32_t* seq_lens_dev,
                            const void* w_uk, const void* w_uv,
                            void* out, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Options of mla_decode_run_ex. */
typedef struct {
  /* cudaEvent_t handles recorded on `stream` immediately before and after the
   * split-KV decode kernel (the dominant kernel of a run), for timing it
   * inside a full step; NULL to record nothing. The events are caller-owned. */
  void* decode_start_event;
  void* decode_stop_event;
} mla_run_options_t;

/* mla_decode_run with options; opts may be NULL (then identical to run). */
mla_status_t mla_decode_run_ex(mla_plan_t plan,
                               const void* q_nope, const void* q_rope,
                               const void* kv_cache, int64_t num_blocks,
                               const int32_t* block_table, int32_t block_table_stride,
                               const int32_t* seq_lens_dev,
                               const void* w_uk, const void* w_uv,
                               void* out, void* workspace, size_t workspace_bytes,
                               void* stream, const mla_run_options_t* opts);

/* One decode step over an FP8 latent cache (plan made with dims.dtype =
 * MLA_FP8_CACHE; mla_decode_run / _ex refuse such a plan with
 * MLA_ERR_INVALID_ARG). The operation is the one above on the dequantised
 * cache; the TransMLA abstract names DeepSeek's FP8 quantisation among the
 * optimisations a converted model can use, and this per-token-scale layout is
 * this library's reading of it. The cache is three device tensors over the
 * same blocks:
 *   kv_codes uint8 [num_blocks, page_size, r]   E4M3 ("e4m3fn") codes of cKV
 *   kv_rope  bf16  [num_blocks, page_size, d_rope] RoPE key divided by s_t
 *   kv_scale fp32  [num_blocks, page_size]      s_t, so that cKV_t = s_t * code_t
 *                                               and k_rope_t = s_t * kv_rope_t
 * (kv_scale 16-byte aligned). As for the bf16 cache, the codes of slots past
 * L_b must be finite (no 0x7F or 0xFF); their RoPE keys and scales may hold
 * anything. Every other argument, the workspace and the errors are as for
 * mla_decode_run_ex. The tensor-core MMAs take e4m3 / e5m2 operands: the
 * absorbed query as an e4m3 value plus an e5m2 correction, and P * s_t, scaled
 * per group of 256 keys by a power of two toward the top of e4m3's range, as
 * two e4m3 terms; by the rounding steps alone the expected relative error
 * against the dequantised cache (2.8e-3 rms) is below the bf16 path's
 * (3.3e-3). s_t must be positive and finite for every visible key
 * (any magnitude). The absorbed query q_nope . W_UK[h] must stay below 448 in
 * magnitude (e4m3's largest finite value): larger entries saturate. */
mla_status_t mla_decode_run_fp8(mla_plan_t plan,
                                const void* q_nope, const void* q_rope,
                                const void* kv_codes, const void* kv_rope, const float* kv_scale,
                                int64_t num_blocks,
                                const int32_t* block_table, int32_t block_table_stride,
                                const int32_t* seq_lens_dev,
                                const void* w_uk, const void* w_uv,
                                void* out, void* workspace, size_t workspace_bytes,
                                void* stream, const mla_run_options_t* opts);

/* Decode step without a caller workspace, for callers that cannot allocate
 * device memory where they run decode steps (an engine whose memory pool owns
 * the whole device and forbids side allocations, or a latency-critical loop
 * that cannot afford the implicit device synchronisation of cudaMalloc and
 * cudaFree). The source pages have no counterpart to this entry point; it is a
 * deployment convenience of this library.
 *
 * Arguments are those of mla_decode_run minus the workspace: the caller still
 * passes every input and the output. The scratch the step needs comes from a
 * fixed 32 MiB array in this library's device image (every GPU that loads the
 * library holds it until the process exits). Plans whose workspace_bytes
 * exceed 32 MiB are rejected with MLA_ERR_WORKSPACE_TOO_SMALL before any device
 * work. On a 148-SM device the tensor-core plans of these batches fit: 16 x 8K
 * tokens with 32 heads (~6.5 MB), 32 x 32K tokens with 128 heads, one or two
 * latent shards (~32.3 MB); 64 sequences x 2 query tokens x 64 heads (~45 MB)
 * do not. Plans over the FP8 cache are refused with MLA_ERR_UNSUPPORTED (this
 * entry point wraps mla_decode_run only). No cudaMalloc, cudaFree or other
 * allocating call is made.
 *
 * The first call on a device sets up that device: it resolves the array's
 * device address and clears its header (a synchronous memset followed by a
 * device synchronisation). Make that first call before any stream capture.
 * The address is kept per device index for the life of the process: calls
 * must run in the device's primary context (the CUDA runtime's), with no
 * cudaDeviceReset in between.
 * All calls in the process share the one array per device and it keeps the
 * last call's contents; two calls whose work overlaps on the GPU (different
 * streams, or different threads) race on it and must be serialised by the
 * caller. Errors detected on the device are recorded in the array's status
 * word, which this entry point does not report; use mla_decode_run with a
 * workspace and mla_decode_read_status to diagnose them. */
mla_status_t mla_decode_run_no_alloc(mla_plan_t plan,
                                     const void* q_nope, const void* q_rope,
                                     const void* kv_cache, int64_t num_blocks,
                                     const int32_t* block_table, int32_t block_table_stride,
                                     const int32_t* seq_lens_dev,
                                     const void* w_uk, const void* w_uv,
                                     void* out, void* stream);

/* One decode step with threshold skipping of negligible key groups. The BLASST
 * abstract (on the kk6lht.com "GQA-to-MLA" search listing) compares a fixed
 * threshold with the running maximum the online softmax already keeps and
 * skips, for blocks of scores found negligible, their exponentials, the value
 * loads and the P.V products. Here the block is a group of 256 keys (4 pages)
 * of one split segment, for all H * Lq query rows of the sequence together:
 * the group is skipped when, for every row, its largest score in log2 units
 * (score * softmax_scale * log2 e, over the keys the row may see) is below
 * the row's running maximum over the segment's earlier groups plus skip_log2
 * (a finite threshold <= 0, or -inf to skip nothing). A row's first group with
 * a visible key in a segment is always kept. Groups start at each segment's
 * first page, so which groups exist depends on the plan's split partition
 * (mla_plan_segments); a plan gives the same result every run. The result is
 * the attention over the kept keys (an approximation of the full step by
 * design), merged across segments as in mla_decode_run. Plans: bf16 on the
 * tensor-core kernel, r = 512, one latent shard (else MLA_ERR_UNSUPPORTED).
 * The call also writes two int32 counters into the workspace header: the
 * number of skipped groups (byte offset 8) and of all groups (offset 12).
 * opts (may be NULL): timing events around the decode kernel, as for
 * mla_decode_run_ex. */
mla_status_t mla_decode_run_blasst(mla_plan_t plan,
                                   const void* q_nope, const void* q_rope,
                                   const void* kv_cache, int64_t num_blocks,
                                   const int32_t* block_table, int32_t block_table_stride,
                                   const int32_t* seq_lens_dev,
                                   const void* w_uk, const void* w_uv,
                                   void* out, void* workspace, size_t workspace_bytes,
                                   float skip_log2, void* stream, const mla_run_options_t* opts);

/* Self-test of the device-side timeout path (diagnostics; not a decode).
 * Runs one step of mla_decode_run on the same arguments, except that in the
 * split-KV decode kernel every bounded wait gives up after wait_limit_ns
 * (1 us .. 2 s) instead of 2 s, and the softmax warps withhold the release of
 * their score buffers in tensor memory. A worker with three or more groups of
 * 256 keys then reaches a wait that nothing completes: that wait runs out, the
 * kernel records MLA_ERR_DEVICE_TIMEOUT in the workspace status word, its
 * other roles stop at their next wait, the tensor memory is released and the
 * kernel returns; no trap, fault or hang, and the context stays usable. The
 * output is undefined. Read the status with mla_decode_read_status. Plans for
 * the bf16 cache on the tensor-core kernel only (else MLA_ERR_UNSUPPORTED). */
mla_status_t mla_decode_selftest_timeout(mla_plan_t plan,
                                         const void* q_nope, const void* q_rope,
                                         const void* kv_cache, int64_t num_blocks,
                                         const int32_t* block_table, int32_t block_table_stride,
                                         const int32_t* seq_lens_dev,
                                         const void* w_uk, const void* w_uv,
                                         void* out, void* workspace, size_t workspace_bytes,
                                         uint64_t wait_limit_ns, void* stream);

/* ---- Prefill in the MLA (non-absorbed) form -------------------------------
 * TPLA's abstract keeps the MLA form for the compute-bound prefill and the
 * absorbed / TPLA form for the memory-bound decode. mla_prefill_run computes,
 * for a batch of prompts, causal attention of every prompt token over the
 * prompt's own tokens with per-head keys and values recovered from the latent
 * rows:
 *   K[h,t] = [cKV[t] . W_UK[h]^T || k_rope[t]],   V[h,t] = cKV[t] . W_UV[h]
 *   out[t,h,:] = softmax_{j <= t}(scale q[t,h] . K[h,j]) . V[h, :]
 * with q = [q_nope || q_rope] (TransMLA abstract: keys and values come from the
 * latent by up-projection). The tokens of all prompts are concatenated:
 * sequence b owns rows [cu[b], cu[b+1]) of
 *   q_nope [T, H, d_nope], q_rope [T, H, d_rope], out [T, H, d_v] and
 *   kv_rows [T, r + d_rope] (the prompt tokens' latent rows, the same rows the
 *   caller writes into the paged cache; columns [0, r) cKV, [r, r + d_rope)
 *   the RoPE key after RoPE).
 * cu_seqlens_dev int32 [B + 1] (device) must hold the plan's lengths' prefix
 * sums. The workspace (caller-owned) holds the up-projected K_nope and V,
 * 2 T H (d_nope + d_v) bytes, plus a 1 KB header whose status word reports
 * device-side errors (read it with mla_decode_read_status).
 * Supported: bf16, r = 512, d_rope = 64, d_nope = d_v = 128, one latent shard
 * (else MLA_ERR_UNSUPPORTED); dims.q_len and dims.page_size are not used. */
typedef struct mla_prefill_plan* mla_prefill_plan_t;

mla_status_t mla_prefill_plan(const mla_dims_t* dims, int32_t batch, const int32_t* seq_lens_host,
                              mla_prefill_plan_t* plan_out, size_t* workspace_bytes);

/* Enqueues the prefill on `stream` (two kernels: the up-projection, then the
 * causal attention); all pointers but `plan` are device pointers. */
mla_status_t mla_prefill_run(mla_prefill_plan_t plan, const void* q_nope, const void* q_rope,
                             const void* kv_rows, const int32_t* cu_seqlens_dev,
                             const void* w_uk, const void* w_uv, void* out,
                             void* workspace, size_t workspace_bytes, void* stream);

/* mla_prefill_run with options; opts may be NULL. The two events of
 * mla_run_options_t are recorded around the attention kernel (the dominant
 * kernel of a prefill). */
mla_status_t mla_prefill_run_ex(mla_prefill_plan_t plan, const void* q_nope, const void* q_rope,
                                const void* kv_rows, const int32_t* cu_seqlens_dev,
                                const void* w_uk, const void* w_uv, void* out,
                                void* workspace, size_t workspace_bytes, void* stream,
                                const mla_run_options_t* opts);

void mla_prefill_plan_destroy(mla_prefill_plan_t plan);

/* Clears the workspace header (status word) with an async memset on `stream`.
 * Call once after allocating a workspace, before its first run. */
mla_status_t mla_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, copies the workspace status word to *device_status
 * (an mla_status_t value; MLA_OK if nothing was recorded) and clears it. */
mla_status_t mla_decode_read_status(const void* workspace, void* stream,
                                    int32_t* device_status);

/* Plan facts for callers and tests. */
mla_status_t mla_plan_get_info(mla_plan_t plan, mla_plan_info_t* info);

/* The plan-time split partition, computed on the host by the same function the
 * kernels evaluate on the device. Each segment is 5 int32 values:
 * (worker, sequence, first page, end page (exclusive), partial slot).
 * Writes min(capacity, count) segments to `out` (may be NULL when capacity is
 * 0) and the total number to *count. */
mla_status_t mla_plan_segments(mla_plan_t plan, int32_t* out, int64_t capacity,
                               int64_t* count);

void mla_plan_destroy(mla_plan_t plan);
const char* mla_status_string(mla_status_t status);
int32_t mla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
