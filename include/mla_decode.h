/*
 * mla_decode.h - C ABI of libmla_decode.so: Multi-head Latent Attention (MLA)
 * decode attention over a paged latent KV cache, for NVIDIA B200 (sm_100a).
 *
 * What it computes. The pages this library follows name the operation - an
 * MLA decode kernel used under speculative decoding (evermx.com, "TokenSpeed:
 * speed-of-light LLM inference engine for agentic workloads", section
 * "Pluggable Kernel Registry") over KV pages reached through index indirection
 * rather than copies, with the whole decode step CUDA-graph captured
 * (zubnet.ai, "LightSeek TokenSpeed 580 TPS Qwen3.5-397B-A17B B200", second
 * paragraph) - without giving a formula. The library computes the absorbed
 * MLA decode definition:
 *
 *   K_b[j]  = latent row of token j of sequence b, 576 wide (512 compressed
 *             latent + 64 RoPE), stored at cache page block_table[b][j / 64],
 *             slot j % 64;  V_b[j] = K_b[j][0:512]
 *   query t of the q_len tokens of a step sees tokens j <= L_b - q_len + t
 *   z_j     = scale * <q[b][t][h], K_b[j]>          (scale usually 1/sqrt(192))
 *   lse     = ln sum_j exp(z_j)
 *   out     = sum_j exp(z_j - lse) * V_b[j]
 *
 * Conventions for every call:
 *   - Pointers marked DEVICE are CUDA device (or managed) memory on the current
 *     device; they must be 16-byte aligned unless stated otherwise. The caller
 *     allocates and owns every buffer, including the workspace; the library
 *     allocates no device memory and keeps no pointer after a call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is only
 *     enqueued; nothing is synchronised with the host, so plan + run can be
 *     captured in a CUDA graph. For fixed (batch, max_pages_per_seq, q_len,
 *     heads, kv_dtype) the launches and workspace size are fixed; the
 *     *contents* of seqlens and block_table may change between graph replays.
 *   - Return value: MLA_OK or a negative mla_status. Argument problems are
 *     found on the host before anything is enqueued; the message is kept per
 *     thread and read with mla_get_last_error(). Problems only the device can
 *     see (a bad sequence length or page id, a wait that timed out) never trap:
 *     they set bits of a flag word in the workspace, read with
 *     mla_read_device_flag().
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,         /* a null/misaligned pointer, a bad size or value */
  MLA_ERR_UNSUPPORTED = -2,         /* a shape/dtype/device this build does not handle */
  MLA_ERR_WORKSPACE_TOO_SMALL = -3, /* workspace_bytes below what mla_decode_plan reported */
  MLA_ERR_CUDA = -4,                /* a CUDA runtime/driver call failed (message has the code) */
  MLA_ERR_DEVICE_FLAG = -5          /* mla_read_device_flag: the device reported a problem */
} mla_status;

typedef enum {
  MLA_KV_BF16 = 0,     /* cache page = 64 tokens x 576 bf16 (73,728 bytes) */
  MLA_KV_FP8_E4M3 = 1  /* cache page = 64 x 576 e4m3 codes then 64 fp32 per-token scales (37,120 bytes) */
} mla_kv_dtype;

/* Device flag bits (mla_read_device_flag). */
#define MLA_FLAG_TIMEOUT 1     /* a bounded on-device wait gave up; outputs are not valid */
#define MLA_FLAG_BAD_SEQLEN 2  /* some seqlens[b] < q_len or > 64 * max_pages_per_seq; its rows are NaN */
#define MLA_FLAG_BAD_PAGE 4    /* a referenced block_table entry is outside [0, num_pages) */
#define MLA_FLAG_BAD_PREFIX 8  /* mla_decode_cascade: a sequence's prefix pages are not sequence 0's */
#define MLA_FLAG_PLAN_MISMATCH 16 /* a run's plan is not the one the last mla_decode_plan on its workspace wrote */

/*
 * mla_decode_plan - size the workspace and (optionally) plan one decode step.
 *
 * seqlens            DEVICE int32 [batch]: L_b, tokens of sequence b including
 *                    the q_len new ones (4-byte aligned). Read only when
 *                    workspace != NULL, by a planner kernel on `stream`.
 * block_table        DEVICE int32 [batch][max_pages_per_seq] (4-byte aligned),
 *                    or NULL. When given (and workspace != NULL), the planner
 *                    also range-checks the entries the step will read (the
 *                    first ceil(L_b / 64) of row b) against [0, num_pages); the
 *                    decode kernel reports a bad entry as MLA_FLAG_BAD_PAGE
 *                    (and also checks every entry where it reads it).
 * num_pages          pages in the pool mla_decode_run will read (1 .. 2^31-1);
 *                    ignored when block_table is NULL.
 * batch              >= 0 (0 plans an empty step).
 * max_pages_per_seq  >= 1: columns of block_table (the most pages any L_b may use).
 * q_len              1..4 query tokens per sequence (1 verified + up to 3 drafts).
 * heads              1..128 query heads; q_len * heads <= 512.
 * kv_dtype           mla_kv_dtype of the cache that mla_decode_run will read.
 * sm_budget          SMs the step may use, 0 = all. Work is spread over
 *                    clusters of 2 SMs; fewer SMs means fewer KV splits. (An
 *                    extension to the plain plan call: scheduling and tests.)
 * workspace          DEVICE, 256-byte aligned, or NULL to only query the size.
 * workspace_bytes    in: capacity of `workspace` (ignored when it is NULL);
 *                    out: bytes this (batch, max_pages_per_seq, q_len, heads,
 *                    kv_dtype) needs. The size does not depend on seqlens.
 * num_splits         out (may be NULL): the most partial results the workspace
 *                    can hold, i.e. the upper bound on split-KV pieces.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE_TOO_SMALL,
 * MLA_ERR_CUDA. The planner clears the device flag word.
 */
MLA_API int mla_decode_plan(const int32_t* seqlens, const int32_t* block_table, int64_t num_pages, int batch,
                            int max_pages_per_seq, int q_len, int heads, int kv_dtype, int sm_budget,
                            void* workspace, size_t* workspace_bytes, int* num_splits, void* stream);

/*
 * mla_decode_run - enqueue the decode attention of one planned step.
 *
 * q             DEVICE bf16 [batch][q_len][heads][576]: absorbed queries
 *               [W_UK^T q_nope (512) | q_rope (64)], RoPE already applied.
 * kv_cache      DEVICE page pool, num_pages pages of the layout kv_dtype names.
 * num_pages     pages in the pool (1 .. 2^31-1); every referenced block_table
 *               entry must be in [0, num_pages).
 * block_table   DEVICE int32 [batch][max_pages_per_seq] (4-byte aligned);
 *               entries past ceil(L_b / 64) are never read.
 * seqlens       DEVICE int32 [batch], the same buffer/contents given to plan.
 * out           DEVICE bf16 [batch][q_len][heads][512] (written).
 * lse           DEVICE fp32 [batch][q_len][heads], natural log (written;
 *               4-byte aligned).
 * scale         softmax scale > 0 applied to q.k (1/sqrt(192) for the
 *               128 + 64 per-head QK width of DeepSeek-style MLA).
 * workspace     the planned workspace, workspace_bytes its capacity.
 * All shape arguments must equal those given to mla_decode_plan.
 * Plan used: the one the planner kernel wrote, except for a batch of at most
 * 32 sequences on a workspace this process planned, whose decode kernel
 * derives the same plan from seqlens itself (with the SM budget of the last
 * mla_decode_plan call on the workspace) and so starts without waiting for the
 * planner kernel. If the two differ (for example a captured plan replayed after
 * a later plan call with another budget) the device flag gets
 * MLA_FLAG_PLAN_MISMATCH and the outputs are not valid.
 * Slots past L_b in a sequence's last page may hold anything (even NaN).
 */
MLA_API int mla_decode_run(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                   const int32_t* block_table, const int32_t* seqlens, void* out, float* lse, int batch,
                   int max_pages_per_seq, int q_len, int heads, float scale, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Phases of a run, for callers that schedule (or time) them separately. */
#define MLA_PHASE_ATTEND 1   /* the main kernel: per-piece attention, unsplit rows finished */
#define MLA_PHASE_COMBINE 2  /* the split combine: merges pieces of split sequences */

/*
 * mla_decode_run_phases - mla_decode_run restricted to the phases in `phases`
 * (a non-empty OR of MLA_PHASE_*). Running MLA_PHASE_ATTEND and then
 * MLA_PHASE_COMBINE on the same stream with the same arguments is exactly
 * mla_decode_run. Same arguments, ownership and errors as mla_decode_run.
 */
MLA_API int mla_decode_run_phases(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                                  const int32_t* block_table, const int32_t* seqlens, void* out, float* lse,
                                  int batch, int max_pages_per_seq, int q_len, int heads, float scale,
                                  void* workspace, size_t workspace_bytes, int phases, void* stream);

/*
 * mla_decode_noalloc - one whole decode step (plan + run) that needs no
 * workspace from the caller and allocates nothing.
 *
 * The pages this library follows have no counterpart to this call. It exists
 * for callers that cannot provide a device buffer of their own: code reaching
 * the library through a foreign-function layer without a CUDA allocator,
 * processes whose device memory belongs to a pool they cannot draw from, or
 * loops that must not allocate at all. The workspace is instead a fixed array
 * of MLA_NOALLOC_SCRATCH_BYTES built into the library: every GPU that loads the
 * library keeps that much device memory until the process exits.
 *
 * Arguments, layouts and errors are those of mla_decode_plan + mla_decode_run
 * (with sm_budget 0). A shape whose workspace would not fit in the array fails
 * with MLA_ERR_WORKSPACE_TOO_SMALL and a message giving both sizes.
 * All calls share the one array and it keeps the last call's contents (nothing
 * in it has to start at zero; each call rewrites what it reads). Calls whose
 * work overlaps on the GPU - on different streams, or from racing host threads -
 * corrupt each other's results, so order them (e.g. one stream). The first call
 * on a device looks up the array's device address (cudaGetSymbolAddress), and
 * so does the first call after the device's context changed (for example after
 * cudaDeviceReset, which reloads the library's device code); make those calls
 * before starting any stream capture.
 */
#define MLA_NOALLOC_SCRATCH_BYTES (48u << 20)
MLA_API int mla_decode_noalloc(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                               const int32_t* block_table, const int32_t* seqlens, void* out, float* lse, int batch,
                               int max_pages_per_seq, int q_len, int heads, float scale, void* stream);

/*
 * mla_decode_cascade - one decode step for a batch whose sequences share the
 * KV pages of a common prefix (multi-turn agentic serving with prefix reuse:
 * zubnet.ai, "LightSeek TokenSpeed 580 TPS Qwen3.5-397B-A17B B200", second
 * paragraph; 24-ai.news, "TokenSpeed ... 580 token/s", optimisations list).
 *
 * Same result as mla_decode_plan + mla_decode_run (up to rounding), computed
 * as a cascade: the first prefix_len tokens (block-table entries 0 ..
 * prefix_len/64 - 1, which must be the same page ids in every sequence) are
 * attended by the union of the batch's batch * q_len * heads query rows as
 * one sequence - a 128-row tile then holds the rows of several sequences and
 * loads each prefix page once for all of them - and each sequence's remaining
 * tokens by an ordinary step; the two are merged by their log-sum-exp weights.
 *
 * prefix_len  a multiple of 64 in [0, 64 * max_pages_per_seq]; every sequence
 *             needs L_b >= prefix_len + q_len (its new tokens are not in the
 *             prefix). 0 runs an ordinary step.
 * workspace / workspace_bytes  as for mla_decode_plan: NULL workspace queries
 *             the size (in: capacity, out: bytes needed), which depends on
 *             (batch, max_pages_per_seq, q_len, heads, kv_dtype) only.
 * batch * q_len * heads <= 8192. Other arguments, layouts and errors: those of
 * mla_decode_plan + mla_decode_run. Device-detected problems go to the
 * workspace's flag word (mla_read_device_flag): MLA_FLAG_BAD_SEQLEN for a
 * sequence too short for the prefix (its rows are NaN), MLA_FLAG_BAD_PREFIX
 * when a sequence's first prefix_len/64 block-table entries differ from
 * sequence 0's (its results are then not valid), and the decode flags.
 */
MLA_API int mla_decode_cascade(const void* q, const void* kv_cache, int64_t num_pages, int kv_dtype,
                               const int32_t* block_table, const int32_t* seqlens, int prefix_len, void* out,
                               float* lse, int batch, int max_pages_per_seq, int q_len, int heads, float scale,
                               void* workspace, size_t* workspace_bytes, void* stream);

/*
 * mla_cache_append - write the q_len new tokens of each sequence into the
 * paged latent cache (the step that precedes mla_decode_plan/run).
 *
 * The pages keep the KV cache in pages reached through index indirection
 * instead of copies (zubnet.ai, "LightSeek TokenSpeed 580 TPS Qwen3.5-397B-A17B
 * B200", second paragraph). The new tokens are the last q_len positions of
 * each sequence, already counted in seqlens: token t of sequence b goes to
 * position j = L_b - q_len + t, i.e. page block_table[b][j / 64], slot j % 64.
 *
 * kv_new       DEVICE bf16 [batch][q_len][576] (16-byte aligned): the new
 *              tokens' latent rows [512 latent | 64 rope].
 * kv_cache     DEVICE page pool of num_pages pages (written in place), the
 *              layout kv_dtype names. MLA_KV_BF16: the row is copied.
 *              MLA_KV_FP8_E4M3: sigma = amax_d |x_d| / 448 (1.0 for an all-zero
 *              row) goes to the page's scale slot and e4m3(x_d / sigma),
 *              rounded to nearest-even and saturated to +-448, to its codes;
 *              both divisions are IEEE fp32. (The pages give no quantisation
 *              rule; this is the library's reading, the one its fp8 decode
 *              path assumes.) NaN inputs are stored as NaN codes.
 * block_table  DEVICE int32 [batch][max_pages_per_seq] (4-byte aligned).
 * seqlens      DEVICE int32 [batch] (4-byte aligned), counting the new tokens.
 * flag         DEVICE int32 word or NULL: MLA_FLAG_BAD_SEQLEN is OR-ed in for
 *              a sequence with L_b < q_len or L_b > 64 * max_pages_per_seq,
 *              MLA_FLAG_BAD_PAGE for a page id outside [0, num_pages); such
 *              rows are not written. (Not the workspace flag, which
 *              mla_decode_plan clears.)
 * Only the written slots change; the caller owns every buffer; nothing is
 * synchronised with the host (graph-capturable). Errors: MLA_ERR_INVALID_ARG,
 * MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA.
 */
MLA_API int mla_cache_append(const void* kv_new, void* kv_cache, int64_t num_pages, int kv_dtype,
                             const int32_t* block_table, const int32_t* seqlens, int batch, int max_pages_per_seq,
                             int q_len, int32_t* flag, void* stream);

/*
 * mla_absorb_q / mla_project_out - the per-head projections around the decode
 * attention in the absorbed MLA form.
 *
 * The pages name an MLA decode kernel (evermx.com, "TokenSpeed: speed-of-light
 * LLM inference engine for agentic workloads", section "Pluggable Kernel
 * Registry"); in the absorbed form the per-head up-projections W_UK[h] and
 * W_UV[h] (each [128][512], from the 512-wide latent to the 128-wide per-head
 * no-RoPE key / value) move out of the attention onto the query and the
 * output:
 *   mla_absorb_q   : q_out[n][h] = [ W_UK[h]^T q[n][h][0:128] | q[n][h][128:192] ]
 *                    (the 576-wide query row mla_decode_run reads)
 *   mla_project_out: y[n][h] = W_UV[h] o[n][h]   (o = the decode output)
 * for the n_tokens = batch * q_len query tokens of a step, in bf16 with fp32
 * accumulation on the tensor cores (outputs rounded to nearest-even bf16).
 *
 * q        DEVICE bf16 [n_tokens][heads][192]: per-head query [128 nope | 64 rope],
 *          RoPE already applied.
 * w_uk     DEVICE bf16 [heads][128][512];  w_uv  DEVICE bf16 [heads][128][512].
 * q_out    DEVICE bf16 [n_tokens][heads][576] (written).
 * o        DEVICE bf16 [n_tokens][heads][512];  y  DEVICE bf16 [n_tokens][heads][128] (written).
 * n_tokens 0 .. 1,048,576 (0 is a no-op); heads 1 .. 128.
 * flag     DEVICE int32 word or NULL: MLA_FLAG_TIMEOUT is OR-ed in if an
 *          on-device wait ran out (the outputs are then not valid).
 * All pointers 16-byte aligned. Nothing is synchronised with the host.
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA.
 */
MLA_API int mla_absorb_q(const void* q, const void* w_uk, void* q_out, int n_tokens, int heads, int32_t* flag,
                         void* stream);
MLA_API int mla_project_out(const void* o, const void* w_uv, void* y, int n_tokens, int heads, int32_t* flag,
                            void* stream);

/* Message for the last non-OK status returned on this thread ("" if none). */
MLA_API const char* mla_get_last_error(void);

/*
 * mla_read_device_flag - copy the workspace's device flag word to *flag.
 * Synchronises `stream` (this call is for checks and tests, not the hot path).
 * Returns MLA_OK when the flag is 0, MLA_ERR_DEVICE_FLAG when any MLA_FLAG_*
 * bit is set, MLA_ERR_CUDA / MLA_ERR_INVALID_ARG on failure.
 */
MLA_API int mla_read_device_flag(const void* workspace, int* flag, void* stream);

/* Test hook: bound, in nanoseconds, of every on-device wait of later runs on
 * this thread (default 1e9). A run whose wait expires returns early with
 * MLA_FLAG_TIMEOUT set, it does not hang. */
MLA_API int mla_set_wait_timeout_ns(uint64_t timeout_ns);

/* Library version string. */
MLA_API const char* mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
