/*
 * gqa_decode.h -- C ABI of libgqadecode.so: grouped-query decode attention
 * over a sequence-split KV cache, for NVIDIA B200 (sm_100a).
 *
 * The method (kernbench "_attention_mesh_mlo.py", decode kernel
 * attention_mesh_mlo_kernel and its module docstring): the single-token query
 * Q is replicated, the KV cache is cut along the sequence into contiguous
 * shards; each shard computes its partial attention as a triplet
 *     m = max_j s_j,   l = sum_j exp(s_j - m),   o = sum_j exp(s_j - m) v_j
 * ("One-shot local partial attention"), the triplets are combined with the
 * log-sum-exp rule (m_c = max(m, m'), l = l e^{m-m_c} + l' e^{m'-m_c},
 * o = o e^{m-m_c} + o' e^{m'-m_c}) and the result is O = o / l ("Final
 * normalize").  Here the shards are split-KV chunks on one GPU.
 *
 * Logits: s_j = scale * <q[b][h][:], k[row][g][:]> where query head h reads
 * kv head g = floor(h / (h_q / h_kv)) (contiguous groups, as in the tinygrad
 * "llama speed tracking" page's Attention.__call__, which shards q by
 * n_rep * head_dim beside k and v by head_dim).
 *
 * ---------------------------------------------------------------- layouts
 *   q        [B][h_q][d_head]            dtype (fp32 or bf16), contiguous
 *   k_cache  [sum_b S_b][h_kv][d_head]   dtype, packed: sequence b occupies
 *   v_cache  [sum_b S_b][h_kv][d_head]   rows S_0 + ... + S_{b-1} onwards
 *   seqlens  int32 [B]                   S_b (device memory)
 *   kv_rows  rows of k_cache and v_cache (host value), or -1 if not known
 *   out      fp32 [B][h_q][d_head]       O = o / l (0 where S_b == 0)
 *   m, l     fp32 [B][h_q][n_slots]      per-split triplets (m in natural
 *   o        fp32 [B][h_q][n_slots][d_head]   log units, o unnormalised)
 * With every S_b equal to S the packed cache is the dense [B][S][h_kv][d]
 * layout.
 *
 * Split policies (the page splits evenly, 1/n_ranks per rank):
 *   by count: split i of sequence b covers [i*L_b, min((i+1)*L_b, S_b)),
 *             L_b = ceil(S_b / n_splits); n_slots = n_splits;
 *   chunked:  split i covers [i*chunk_len, min((i+1)*chunk_len, S_b)),
 *             n_slots = max(1, ceil(max_seqlen / chunk_len)).
 * An empty split's triplet is (-inf, 0, 0).
 *
 * ------------------------------------------------------------ conventions
 * - Every pointer argument is a DEVICE pointer on the current CUDA device and
 *   is owned by the caller, except `workspace == NULL` (see below).
 * - q, k_cache, v_cache and every fp32 output must be 16-byte aligned.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *   stream).  Every call is asynchronous on that stream and never
 *   synchronises the host, except for workspace growth (below) and
 *   gqa_decode_get_status().
 * - Arguments are checked on the host; on any error the call returns a
 *   nonzero gqa_status and launches nothing.  Supported: d_head in {64, 128};
 *   h_q % h_kv == 0; 1 <= n_splits <= 1024 (n_slots <= 1024 when chunked);
 *   finite scale; dtype GQA_F32 or GQA_BF16 (q, k and v share it).
 *   n_splits = 0 on a fused call picks the count (gqa_decode_auto_splits).
 * - Errors that only the device can see (a negative S_b, S_b above
 *   max_seqlen in chunked mode, a bounded wait that ran out) set bits of a
 *   per-device status word, read and cleared by gqa_decode_get_status().
 * - No stray reads: a kernel reads only cache rows that belong to the batch
 *   (rows [0, sum_b S_b)); rows of a neighbouring sequence that fall inside a
 *   loaded tile are masked by index, so they must hold finite values (any
 *   packed cache does).  The one exception is the early L2 prefetch (see
 *   kv_rows): it brings rows into the L2 cache only, never into a result,
 *   and may touch any row below kv_rows.
 * - kv_rows (packed-cache calls): the number of rows the caller allocated
 *   for k_cache and v_cache (each is [kv_rows][h_kv][d_head]).  When it is
 *   given (>= 1), no cache row at or past it is read: rows past it read as
 *   zero, and sum_b S_b > kv_rows sets GQA_ERR_DEVICE_SEQLEN in the status
 *   word.  kv_rows = 0 is an empty cache (every S_b must be 0).  Knowing it
 *   also lets the bf16 kernels issue L2 prefetches of their first K/V tiles
 *   before the kernel that precedes them on the stream has finished (the
 *   lengths they read for that may not be final yet; every prefetched row is
 *   checked against kv_rows, and the result never depends on it).
 *   kv_rows = -1: not known -- no clipping, no early prefetch; values below
 *   -1 are GQA_ERR_INVALID_ARG, values above 2^31 - 1 GQA_ERR_UNSUPPORTED.
 */
#ifndef GQA_DECODE_H
#define GQA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GQA_API __attribute__((visibility("default")))
#else
#define GQA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_INVALID_ARG = 1,     /* bad pointer, size, alignment or value */
    GQA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. d_head 96) */
    GQA_ERR_CUDA = 3,            /* a CUDA runtime / driver call failed */
    GQA_ERR_WORKSPACE = 4,       /* caller workspace too small or misaligned */
    GQA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded wait in a kernel ran out */
    GQA_ERR_DEVICE_SEQLEN = 6,   /* a kernel saw S_b < 0 or S_b > max_seqlen */
    GQA_ERR_DEVICE_BOUNDS = 7    /* checked build: an index check failed (access skipped) */
} gqa_status;

typedef enum { GQA_F32 = 0, GQA_BF16 = 1 } gqa_dtype;

/* Version of this ABI (major * 10000 + minor * 100 + patch): 300 (0.3.0)
 * adds the kv_rows argument of the packed-cache calls; 0.2.0 added
 * gqa_decode_fused_plan. */
GQA_API int gqa_decode_version(void);

/* Human-readable name of a gqa_status value (static storage). */
GQA_API const char *gqa_decode_error_string(int status);

/* Bytes of workspace gqa_decode_attn needs: a fixed 256 KiB ticket area (one
 * int32 counter per (b, kv head, head block); at most 65536 of them) followed
 * by fp32 triplets for every (b, h, split).  Returns 0 for arguments
 * gqa_decode_attn would reject. */
GQA_API size_t gqa_decode_workspace_size(int B, int h_q, int h_kv, int d_head, int n_splits);

/* Same for gqa_decode_attn_chunked. */
GQA_API size_t gqa_decode_chunked_workspace_size(int B, int h_q, int h_kv, int d_head,
                                         int chunk_len, int max_seqlen);

/*
 * Fused decode attention, split by count: every split's triplet is computed
 * and the splits of each (b, kv head) are merged in split order into
 * out[b][h][:] for the group's query heads -- by the CTA that finishes the
 * group's last split, or by a second kernel over all rows (see
 * gqa_decode_fused_plan and gqa_decode_launches_per_call).  The result equals
 * gqa_decode_partial followed by mlo_merge up to fp32 rounding (bit for bit
 * on the fp32 path, which shares the per-split kernel).
 *
 * workspace: NULL, or caller device memory of at least
 *   gqa_decode_workspace_size(...) bytes, 256-byte aligned, whose first
 *   256 KiB (the ticket area) are ZERO-FILLED before its first use.  Every
 *   call that completes returns the tickets it used to zero and writes
 *   triplets only past the ticket area, so one workspace serves calls of any
 *   shape without clearing; after a device error (status word set) zero the
 *   ticket area again.  Calls that share a workspace must be ordered on one
 *   stream.  With NULL the library uses a
 *   grow-only workspace of its own per device (growing it synchronises the
 *   device); calls that use it must be ordered on one stream.
 */
GQA_API int gqa_decode_attn(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seqlens, long long kv_rows, float *out,
                    int B, int h_q, int h_kv, int d_head, int n_splits, float scale,
                    int dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * gqa_decode_attn without any allocation.  No passage of the method's pages
 * corresponds to this entry point; it exists for callers that cannot call
 * cudaMalloc -- for example a plugin inside a host program that owns every
 * device allocation through its own pool, or a latency-critical path that
 * cannot afford the device-wide synchronisation cudaMalloc may imply.
 *
 * Same arguments and result as gqa_decode_attn minus the workspace: the
 * scratch (ticket area + triplets) is a fixed 40 MiB array in the library's
 * own device memory, held by every device that loads the library until the
 * process exits.  A call whose scratch would exceed 40 MiB
 * (gqa_decode_workspace_size(...) > 40 MiB) returns GQA_ERR_WORKSPACE and
 * launches nothing.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  Every call clears the tickets it uses
 * (one cudaMemsetAsync on the stream) and then runs the fused kernels; a call
 * that merges in a second kernel (gqa_decode_launches_per_call == 2) reads no
 * ticket and skips the clearing.  Nothing is allocated or freed.  All calls
 * on a device share that device's one array,
 * which keeps the last call's contents: calls that overlap on the GPU (for
 * instance on two streams) race and corrupt each other's results, so order
 * them on one stream.
 */
GQA_API int gqa_decode_attn_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *seqlens, long long kv_rows, float *out,
                                    int B, int h_q, int h_kv, int d_head, int n_splits,
                                    float scale, int dtype, void *stream);

/*
 * Append-and-attend, the step just before decode attention in a decode loop
 * (the tt-metal "[Llama2] Perf burndown" page's `update_cache`), fused into
 * the attention call: the new token's k and v (k_new, v_new: [B][h_kv][d_head],
 * dtype) are written into the cache at row S_b of each sequence, and the query
 * attends over the S_b + 1 keys, the new one included.
 *
 * The cache is padded, not packed: k_cache, v_cache are [B][cache_capacity]
 * [h_kv][d_head] and sequence b's key j is row b * cache_capacity + j, so
 * there is room to append.  Requires S_b + 1 <= cache_capacity; a sequence
 * without room is attended over its cached rows only and reported as
 * GQA_ERR_DEVICE_SEQLEN in the status word.  seqlens is NOT advanced: the
 * caller adds 1 for the next step.  The split of the S_b + 1 keys, the
 * workspace and the result are as for gqa_decode_attn.  Only the new rows
 * are written; no other cache row is read or written outside [0, S_b + 1)
 * of each sequence, except that rows of the previous sequence's unused tail
 * may be read into a masked, zeroed tile.  The cache's B * cache_capacity
 * rows play the part of kv_rows (the early L2 prefetch of the bf16 kernels
 * stays inside them).
 */
GQA_API int gqa_decode_attn_append(const void *q, const void *k_new, const void *v_new,
                                   void *k_cache, void *v_cache, const int32_t *seqlens,
                                   float *out, int B, int h_q, int h_kv, int d_head,
                                   int cache_capacity, int n_splits, float scale, int dtype,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Fused decode attention with fixed-length chunks (ragged batches): split i
 * of sequence b covers [i*chunk_len, min((i+1)*chunk_len, S_b)); the last
 * chunk may be partial.  max_seqlen bounds every S_b (host-known, so no
 * device-to-host copy is needed); a larger S_b sets GQA_ERR_DEVICE_SEQLEN in
 * the status word and only its first n_slots chunks are used.
 */
GQA_API int gqa_decode_attn_chunked(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, long long kv_rows, float *out,
                            int B, int h_q, int h_kv, int d_head, int chunk_len, int max_seqlen,
                            float scale, int dtype, void *workspace, size_t workspace_bytes,
                            void *stream);

/*
 * Partial attention only ("One-shot local partial attention" of the page, one
 * split per shard): writes the (m, l, o) triplet of every (b, h, split) into
 * m, l [B][h_q][n_splits] and o [B][h_q][n_splits][d_head] (fp32, m in
 * natural-log units, o unnormalised, empty split = (-inf, 0, 0)).
 */
GQA_API int gqa_decode_partial(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seqlens, long long kv_rows, float *m, float *l, float *o,
                       int B, int h_q, int h_kv, int d_head, int n_splits, float scale,
                       int dtype, void *stream);

/* Partial attention with the chunked split policy (n_slots triplets per row,
 * n_slots = max(1, ceil(max_seqlen / chunk_len))). */
GQA_API int gqa_decode_partial_chunked(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *seqlens, long long kv_rows, float *m, float *l,
                               float *o,
                               int B, int h_q, int h_kv, int d_head, int chunk_len,
                               int max_seqlen, float scale, int dtype, void *stream);

/*
 * Log-sum-exp merge and normalisation of n_splits triplets per row (the
 * page's merge of received triplets, then "Final normalize"):
 *   M = max_i m_i,  l* = sum_i l_i e^{m_i - M},  o* = sum_i o_i e^{m_i - M},
 *   out = o* / l*   (0 when every triplet of the row is empty).
 * m, l: fp32 [rows][n_splits]; o: fp32 [rows][n_splits][d_head];
 * out: fp32 [rows][d_head].  Splits are summed in index order, so the result
 * is deterministic.  1 <= d_head <= 256, n_splits >= 1.
 */
GQA_API int mlo_merge(const float *m, const float *l, const float *o, float *out,
              int rows, int n_splits, int d_head, void *stream);

/*
 * The same merge for triplets gathered from n_ranks sequence shards -- the
 * page's multi-rank form (kernbench "_attention_mesh_mlo.py": replicated Q,
 * KV sharded along the sequence over ranks, each rank's triplet merged into
 * the others').  Rank r's triplets are m, l fp32 [rows][n_splits] starting
 * r * rank_stride_ml floats after m (and l), and o fp32
 * [rows][n_splits][d_head] starting r * rank_stride_o floats after o -- the
 * layout an all-gather of every rank's gqa_decode_partial output produces
 * (stride rows * n_splits and rows * n_splits * d_head when m, l and o are
 * gathered separately; one common stride when each rank's m, l, o are packed
 * in one buffer).  A row's splits are summed in rank-major order, so the
 * result equals mlo_merge over the rank-major concatenation.
 * 1 <= d_head <= 256, n_ranks * n_splits <= 2^20; with n_ranks > 1 the
 * strides must keep the ranks' blocks apart.
 */
GQA_API int mlo_merge_ranked(const float *m, const float *l, const float *o, float *out,
                             int rows, int n_ranks, int n_splits, int d_head,
                             long long rank_stride_ml, long long rank_stride_o, void *stream);

/*
 * Split count the library would choose: the largest n_splits whose grid
 * (n_splits x kv heads x head blocks x B CTAs) still fits on the current
 * device in one wave, capped so a split keeps at least 256 keys when
 * max_seqlen > 0 (0: unknown).  Passing n_splits = 0 to gqa_decode_attn,
 * gqa_decode_attn_noalloc, gqa_decode_attn_append or
 * gqa_decode_workspace_size makes that choice for the call (the append call
 * caps with its cache capacity).  Returns n >= 1, or a negative gqa_status.
 */
GQA_API int gqa_decode_auto_splits(int B, int h_q, int h_kv, int d_head, int max_seqlen);

/*
 * Number of kernels one fused call (gqa_decode_attn / _chunked / _noalloc)
 * launches on the current device for this shape (n_slots = n_splits, or
 * ceil(max_seqlen / chunk_len) when chunked): 1 when the CTA that finishes a
 * group's splits last merges them, or 2 when the splits' triplets are merged
 * by a second kernel -- the persistent decode kernel, and the one-wave grid
 * of groups of 8 or more query heads.  0 for B == 0; a negative gqa_status
 * on bad arguments.
 */
GQA_API int gqa_decode_launches_per_call(int B, int h_q, int h_kv, int d_head, int n_slots,
                                         int dtype);

/*
 * The launch plan one fused call takes on the current device for this shape
 * (arguments as for gqa_decode_launches_per_call):
 *   GQA_PLAN_SIMT        fp32: one CUDA-core kernel per (split, kv head, b);
 *   GQA_PLAN_ONE_WAVE    bf16, every split CTA resident at once: one
 *                        tensor-core kernel, merged by ticket (groups of
 *                        fewer than 8 query heads) or by a second kernel;
 *   GQA_PLAN_PERSISTENT  bf16, up to four times that many splits: persistent
 *                        CTAs over the splits, then the row-merge kernel;
 *   GQA_PLAN_MANY_WAVES  bf16, more: the per-split kernel with two stages per
 *                        warp, merged by ticket.
 * Returns the plan (>= 0), or a negative gqa_status on bad arguments
 * (-GQA_ERR_INVALID_ARG also for B == 0, which launches nothing).
 */
enum { GQA_PLAN_SIMT = 0, GQA_PLAN_ONE_WAVE = 1, GQA_PLAN_PERSISTENT = 2, GQA_PLAN_MANY_WAVES = 3 };
GQA_API int gqa_decode_fused_plan(int B, int h_q, int h_kv, int d_head, int n_slots, int dtype);

/*
 * Synchronises `stream`, then reads and clears this device's status word.
 * Returns GQA_OK, GQA_ERR_DEVICE_TIMEOUT, GQA_ERR_DEVICE_BOUNDS,
 * GQA_ERR_DEVICE_SEQLEN (in that order of precedence) or GQA_ERR_CUDA.
 */
GQA_API int gqa_decode_get_status(void *stream);

/*
 * The checked build.  libgqadecode_checked.so is this library compiled with
 * -DGQA_CHECKED: every global access whose element index the kernels derive
 * (query rows, split triplet slots, merged rows, tickets, the appended
 * token's source and cache row, prefill output rows) is first tested against
 * the extent the call's arguments give it.  A failed test sets
 * GQA_ERR_DEVICE_BOUNDS in the status word, records the first failure, and
 * skips the access, so a wrong index never reaches memory.  Same entry
 * points and results otherwise; the normal build compiles the tests away.
 *
 * gqa_decode_checked_build: 1 in the checked build, 0 otherwise.
 * gqa_decode_bounds_report: synchronises `stream`, returns and clears the
 *   first failed test since the last report as ((site << 56) | index) + 1,
 *   0 when none failed (always 0 in the normal build), ~0 on a CUDA error.
 *   Sites: 1 query row, 2 triplet slot, 3 merged row, 4 ticket, 5 appended
 *   row, 6 prefill output row, 7 the self-test.
 * gqa_decode_selftest_bounds: launches one test whose index equals its
 *   extent (the store it guards is skipped); afterwards the status word reads
 *   GQA_ERR_DEVICE_BOUNDS and the report names site 7.  GQA_ERR_UNSUPPORTED
 *   in the normal build.
 */
GQA_API int gqa_decode_checked_build(void);
GQA_API unsigned long long gqa_decode_bounds_report(void *stream);
GQA_API int gqa_decode_selftest_bounds(void *stream);

/* Upper bound, in nanoseconds, on every wait inside the kernels (default
 * 1e9).  A wait that runs out records GQA_ERR_DEVICE_TIMEOUT and the kernel
 * returns without hanging.  0 restores the default. */
GQA_API int gqa_decode_set_wait_timeout_ns(unsigned long long timeout_ns);

/*
 * Self-test of the bounded wait: launches one CTA that waits on a barrier no
 * thread ever signals, with a bound of `timeout_ns`.  The wait runs out, the
 * kernel records GQA_ERR_DEVICE_TIMEOUT in the status word and returns; the
 * next gqa_decode_get_status() reports it.  Nothing else is touched.
 */
GQA_API int gqa_decode_selftest_wait_timeout(unsigned long long timeout_ns, void *stream);

/* Frees this device's library-owned workspace (after synchronising it). */
GQA_API int gqa_decode_release(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_DECODE_H */
