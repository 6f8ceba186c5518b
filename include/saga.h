/*
 * saga.h - C ABI of the SAGA + Atop-N single-token decode attention library
 * (libsaga.so, hand-written CUDA for sm_100a).
 *
 * Method: "More Value per Key: Asymmetric Sparse Attention for Faster LLM
 * Decoding" (arXiv 2610.04753).  SAGA decouples the key-head count h_k from
 * the value-head count h_v (ai.info summary, Key Contributions #3); Atop-N
 * keeps, per (batch, query head), the cached positions whose logit is >= a
 * threshold that is the exact N-th largest logit, recomputed only every n
 * decode steps and reused in between, found by per-element comparison
 * instead of sorting (Key Contributions #2, Methodology in Plain English
 * ¶2); the probability-value product then touches only the kept value rows
 * (Main Findings, "Bottleneck shift").
 *
 * Shapes and layouts (all row-major, innermost last; bf16 = IEEE bfloat16):
 *   q      [batch, h_q, head_dim]            bf16   this step's queries
 *   k      [batch, l_cap, h_k, head_dim]     bf16   key cache
 *   v      [batch, l_cap, h_v, v_head_dim]   bf16   value cache
 *          positions 0 .. l_kv-1 of each batch element are valid; rows
 *          l_kv .. l_cap-1 are capacity and are never used.
 *   logits [batch, h_q, l_kv]                fp32   s = q.k / sqrt(head_dim)
 *   thresh [batch, h_q]                      fp32   Atop-N thresholds (tau)
 *   out    [batch, h_q, v_head_dim]          fp32
 *   sel_idx[batch, h_q, l_kv]                int32  kept positions, ascending,
 *                                                   first sel_cnt entries valid
 *   sel_cnt[batch, h_q]                      int32
 * Head maps: query head i reads key head i*h_k/h_q and value head i*h_v/h_q
 * (contiguous groups, as in grouped-query attention).
 *
 * Supported shapes: head_dim = v_head_dim in {64, 128}, or head_dim 32 with
 * v_head_dim 64 and h_k >= 2 (keys of half the value dim: the pages' Sigma-
 * style head layout, Main Findings "Head count beats head dimension");
 * h_k in {1, 2, 4, 8}; h_q a
 * multiple of h_k and of h_v with h_q/h_k <= 16 and h_q <= 128;
 * saga_decode_dense also needs h_v a multiple or a divisor of h_k, and a
 * stage (32 KB of keys and the value rows of the same positions) that fits
 * twice in shared memory; with more than two value heads per key head, or
 * a stage too large (e.g. SAGA's (h_k, h_v) = (1, 8), the Sigma-style 32-dim
 * keys with h_v = 8), the kernel treats every value head as a key head of
 * its own, each reading its key head's rows (h_v in {2, 4, 8} and
 * h_q/h_v <= 16 then);
 * 1 <= l_kv <= l_cap; batch*l_cap < 2^31.  Others return
 * SAGA_ERR_UNSUPPORTED.
 *
 * Conventions shared by every call:
 *   - Ownership: the caller allocates and owns every buffer (device memory,
 *     16-byte aligned), the thresholds and the workspace included.  The
 *     library allocates no device memory.
 *   - Asynchrony: every call only enqueues work on `stream` and returns; no
 *     call synchronises the host or reads device data back (except the two
 *     workspace readers, saga_workspace_error and saga_workspace_empty_rows,
 *     which say so).  All grids are
 *     sized from the shapes, never from data, so a sequence of calls can be
 *     captured in a CUDA graph (make one uncaptured call per shape first so
 *     device properties are cached outside the capture).
 *   - Validation: arguments are checked before anything is enqueued; on an
 *     error nothing is launched and no output is touched.
 *   - Workspace: `ws` must hold saga_workspace_bytes(dims, N) bytes and must
 *     be zeroed once after allocation (or passed to saga_workspace_reset).
 *     A workspace sized for dims with a larger l_kv (all else equal) serves
 *     every shorter length, so a growing cache needs one sized for l_cap.
 *     Calls that share a workspace must be ordered on one stream.
 *   - Device-side faults: kernels bound every wait; a wait that runs out
 *     sets a sticky flag in the workspace that saga_workspace_error reads.
 *   - Return value: SAGA_OK (0) or a negative saga_status.
 */
#ifndef SAGA_H
#define SAGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side state of the library (no device memory is allocated): per
 * device, the device's properties and the kernels whose shared-memory limit
 * has been raised on it (CUDA keeps that attribute per device); the launch
 * counter (saga_launch_count); per host thread, the measurement events of
 * saga_set_kernel_events; and, for saga_topn_refresh_noalloc, the device
 * address of its scratch array per device.  All of it is filled on first use
 * and guarded by mutexes.  It is not rebuilt after cudaDeviceReset: a process
 * that resets a device must not call this library on that device again (its
 * cached attributes and scratch address belong to the destroyed context). */

/* Same type as cudaStream_t; 0 is the legacy default stream. */
typedef struct CUstream_st* saga_stream_t;

typedef struct {
    int32_t batch;     /* b                                   */
    int32_t h_q;       /* query heads                          */
    int32_t h_k;       /* key heads   (SAGA: h_k < h_v allowed) */
    int32_t h_v;       /* value heads                          */
    int32_t head_dim;  /* d_k: key (and query) head dim        */
    int32_t l_kv;      /* valid cached positions               */
    int32_t l_cap;     /* cache capacity (row stride in positions) */
    int32_t v_head_dim; /* d_v: value head dim; 0 means d_k    */
} saga_dims;

typedef enum {
    SAGA_OK = 0,
    SAGA_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, non-positive size, l_kv > l_cap, N <= 0 */
    SAGA_ERR_UNSUPPORTED = -2,  /* shape outside the supported set above */
    SAGA_ERR_WORKSPACE = -3,    /* ws_bytes < saga_workspace_bytes(...) */
    SAGA_ERR_CUDA = -4,         /* a CUDA call or launch failed */
    SAGA_ERR_DEVICE = -5,       /* no device, or the device is not sm_100 */
    SAGA_ERR_TIMEOUT = -6,      /* saga_workspace_error: a bounded device wait ran out */
    SAGA_ERR_BOUNDS = -7        /* saga_workspace_error, debug builds (SAGA_DEBUG): a kernel read
                                   a position, count or slot out of range and skipped it */
} saga_status;

/* Bytes of workspace the calls below need for these dimensions.  Depends on
 * the shapes only (not on N, which is checked to be positive); returns 0 for
 * invalid or unsupported dimensions.  Host-only, no CUDA call. */
size_t saga_workspace_bytes(const saga_dims* dims, int32_t N);

/* Dense (full-attention) grouped-query decode: every cached position kept.
 * The speedup denominator (ai.info summary, Main Findings: the end-to-end
 * speedups are measured against full attention).  out[b,i,:] = softmax_j(s[b,i,j]) V[b,j,vh(i),:].
 * Split-K over l_kv (flash-decoding) followed by a log-sum-exp combine. */
int saga_decode_dense(const saga_dims* dims, const void* q, const void* k, const void* v,
                      float* out, void* ws, size_t ws_bytes, saga_stream_t stream);

/* Threshold refresh, run on steps with t mod n == 0 (the caller schedules).
 * thresh_out[b,i] = the exact N-th largest logit of row (b,i), counting
 * duplicates (Key Contributions #2: the exact threshold is found on every
 * n-th token only); N >= l_kv gives -inf (keep everything); a threshold of
 * -0.0 is written as +0.0.
 *   logits_in  != NULL: use these logits [b,h_q,l_kv]; q and k are ignored.
 *   logits_in  == NULL: compute the logits from q and k; if logits_out is
 *                       not NULL they are also written there, so the
 *                       following saga_atopn_decode can reuse them.
 * Exact radix select (three passes over 32-bit order-preserving keys). */
int saga_topn_refresh(const saga_dims* dims, int32_t N, const void* q, const void* k,
                      const float* logits_in, float* logits_out, float* thresh_out,
                      void* ws, size_t ws_bytes, saga_stream_t stream);

/* One Atop-N decode step with the thresholds `thresh` (fresh from
 * saga_topn_refresh on refresh steps, reused otherwise).  The kept set is
 * found by a per-element comparison with the stored threshold, not by a sort
 * (ai.info summary, Key Contributions #2; Methodology in Plain English ¶2),
 * and only the kept value rows of value head vh(i) are read (Main Findings,
 * "Bottleneck shift"; SAGA heads, Key Contributions #3):
 *   tau_eff = min(thresh[b,i], max_j s[b,i,j]);  keep j  <=>  s[b,i,j] >= tau_eff;
 *   out[b,i,:] = sum_kept softmax(s) V[b,j,vh(i),:].
 * The min() keeps the row's maximal entries when a stale threshold lies
 * above every logit (the pages are silent on that case).
 *   logits_in != NULL: the logits are read from there (q, k may be NULL);
 *                      the select/compact, gathered-PV and combine kernels
 *                      run.  Exception: with sel_idx == NULL, q and k given,
 *                      and few long rows (b*h_q <= 64 and l_kv >= 65536,
 *                      where one compare CTA per row would leave most of the
 *                      GPU idle), the fused path below runs instead; it
 *                      recomputes the same logits bit for bit with the same
 *                      tensor-core routine as saga_topn_refresh, so the kept
 *                      set is identical.
 *   logits_in == NULL: the fused kernel computes the logits on chip,
 *                      compares, and gathers only the kept value rows;
 *                      logits never reach device memory.  With sel_idx, one
 *                      more kernel writes the positions that on-chip compare
 *                      kept (the same kernels decide the output either way).
 * sel_idx (nullable): kept positions of each row, ascending; entries past
 *                     sel_cnt[b,i] are left as they were.
 * sel_cnt (nullable): number kept per row. */
int saga_atopn_decode(const saga_dims* dims, const void* q, const void* k, const void* v,
                      const float* thresh, const float* logits_in, float* out,
                      int32_t* sel_idx, int32_t* sel_cnt, void* ws, size_t ws_bytes,
                      saga_stream_t stream);

/* One refresh step in one call: the exact thresholds (as
 * saga_topn_refresh), then the decode with them (as saga_atopn_decode over
 * the step's logits) -- the step that Atop-N takes on every n-th token
 * (ai.info summary, Key Contributions #2: the exact top-N threshold is
 * recomputed, then entries are kept by a per-element comparison).  Results,
 * bit for bit: thresh_out as saga_topn_refresh writes it; out, sel_idx and
 * sel_cnt as saga_atopn_decode over those logits writes them.
 * The logits are written to the workspace once and read twice (the radix
 * passes of the threshold's first two digits): the second also copies out
 * every logit at or above the lower edge of the threshold's first-digit
 * bucket (every kept one among them), and one kernel then finds the last
 * digit and compacts the kept entries from those candidates alone.  Exceptions: N >= l_kv (thresh_out = -inf, full attention) and
 * rows longer than the compaction's on-chip bitmap allows (l_kv above about
 * 900K) compact from the stored logits; few long rows (b*h_q <= 64 and
 * l_kv >= 65536) take saga_atopn_decode's fused path after the refresh (the
 * same logits, recomputed bit for bit).
 * q, k, v, thresh_out [b,h_q], out [b,h_q,d_v]: required.
 * sel_idx, sel_cnt (nullable): as in saga_atopn_decode. */
int saga_atopn_refresh_step(const saga_dims* dims, int32_t N, const void* q, const void* k,
                            const void* v, float* thresh_out, float* out, int32_t* sel_idx,
                            int32_t* sel_cnt, void* ws, size_t ws_bytes, saga_stream_t stream);

/* ---- Sequence shards (the pages run one GPU; this is an extension) ----
 * A decode whose cached sequence is split into contiguous shards, one per
 * rank (each rank's dims: its own l_kv and l_cap; the same b, heads and q).
 * The threshold stays the exact N-th largest logit of the whole row: each
 * rank histograms a digit of its own logits, the caller sums the histograms
 * across ranks (an all-reduce), and every rank takes the same digit from the
 * sum (3 passes: 11, 11 and 10 bits of an order-preserving key, as
 * saga_topn_refresh).  Each rank then decodes its shard into a partial
 * record per row, the caller gathers the records of all ranks, and
 * saga_merge_partials merges them (log-sum-exp) into the output a single
 * GPU would give, empty-set rule included.  Callers order the calls of one
 * rank on one stream; the cross-rank exchange is the caller's (NCCL). */

/* Logits of this shard: logits_out[b,i,j] = q[b,i,:].k[b,j,kh(i),:]/sqrt(d),
 * fp32, j < l_kv (the same values saga_topn_refresh computes). */
int saga_qk_logits(const saga_dims* dims, const void* q, const void* k, float* logits_out,
                   void* ws, size_t ws_bytes, saga_stream_t stream);

/* Digit histogram of radix pass `pass` (0, 1, 2) over this shard's logits
 * [b,h_q,l_kv]: hist[b*h_q][2048] (overwritten) counts, per row, the keys
 * that carry the prefix in state[row] (ignored for pass 0) by their digit.
 * state [b*h_q][2] uint32 is the one saga_topn_select_digit keeps. */
int saga_topn_histogram(const saga_dims* dims, int32_t pass, const float* logits,
                        const uint32_t* state, uint32_t* hist, saga_stream_t stream);

/* Digit choice of pass `pass` from the histograms summed over every shard:
 * updates state [b*h_q][2] (prefix, remaining rank; rank 0 once the row's
 * threshold is known) and, once known, thresh_out[b*h_q]: the N-th largest
 * logit of the whole row, or -inf when N is at least the row's total
 * length (decided in pass 0).  Identical sums give identical results on
 * every rank. */
int saga_topn_select_digit(const saga_dims* dims, int32_t N, int32_t pass, const uint32_t* hist,
                           uint32_t* state, float* thresh_out, saga_stream_t stream);

/* saga_atopn_decode over this shard, without normalising: part[b*h_q] gets
 * records of d_v + 4 floats (m, l, count, row max, o[d_v]):
 *   count > 0: m = the shard's largest logit (kept), l = sum exp(s - m) and
 *              o = sum exp(s - m) V over the shard's kept entries;
 *   count = 0: m = -inf, l = number of the shard's positions at its row max,
 *              o = the sum of their value rows (the empty-set rule's data).
 * count is stored as int32 bits.  q and k are required even with logits_in
 * (a shard that keeps nothing recomputes its maxima from them). */
int saga_atopn_decode_partial(const saga_dims* dims, const void* q, const void* k, const void* v,
                              const float* thresh, const float* logits_in, float* part, void* ws,
                              size_t ws_bytes, saga_stream_t stream);

/* out[b*h_q][d_v] from the R shards' records parts[R][b*h_q][d_v + 4]:
 * with M the largest m over records that kept something,
 * out = sum_r exp(m_r - M) o_r / sum_r exp(m_r - M) l_r; when no shard kept
 * anything, the mean of the value rows at the row's maximum over the shards
 * holding it.  sel_cnt (nullable): kept entries per row (or the number at
 * the maximum).  Only b, h_q and the value head dim of dims are used. */
int saga_merge_partials(const saga_dims* dims, const float* parts, int32_t R, float* out,
                        int32_t* sel_cnt, saga_stream_t stream);

/* Allocation-free threshold refresh (the paper has no counterpart; this is
 * a convenience of this library).  Computes exactly what saga_topn_refresh
 * computes with logits_in != NULL -- thresh_out[b,i] = the N-th largest of
 * logits_in[b,i,:] (-inf if N >= l_kv) -- but takes no workspace, for callers
 * that cannot allocate device memory on the decode path (a plugin inside a
 * host engine that owns all device memory and gives its plugins no
 * allocator; a loop that must not call cudaMalloc after start-up because it
 * can synchronise the device or fail under memory pressure).  Only head_dim-
 * independent fields of dims are used (batch, h_q, l_kv).
 *   - Scratch: a 16 MiB file-scope device array inside libsaga.so, held by
 *     every GPU that loads the library until the process exits; it covers
 *     batch*h_q <= 682 rows.  More rows return SAGA_ERR_WORKSPACE and
 *     enqueue nothing.  Nothing is allocated: no cudaMalloc/cudaFree, no
 *     allocating library call.
 *   - First call per device: looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current) and caches it; make
 *     that first call before any stream capture.
 *   - Every call clears the array's histograms on `stream` and then reuses
 *     it, so calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on the shared scratch: order them on one stream.
 * Errors: SAGA_ERR_INVALID_ARG (null/misaligned pointer, N <= 0, bad dims),
 * SAGA_ERR_WORKSPACE (too many rows), SAGA_ERR_DEVICE, SAGA_ERR_CUDA. */
int saga_topn_refresh_noalloc(const saga_dims* dims, int32_t N, const float* logits_in,
                              float* thresh_out, saga_stream_t stream);

/* Cache growth (real decode: each generated token appends its own key and
 * value rows before it attends; "More Value per Key" measures latency over
 * 32 generated tokens, ai.info summary, Main Findings).  Writes
 *   k_new [batch, h_k, head_dim] bf16 -> k[b, l_kv, :, :]
 *   v_new [batch, h_v, v_head_dim] bf16 -> v[b, l_kv, :, :]
 * i.e. at the first free row of each batch element's cache; the caller then
 * decodes with l_kv + 1.  The thresholds of the last refresh stay valid for
 * the grown cache (the new position is compared like any other).
 * Errors: SAGA_ERR_INVALID_ARG (l_kv >= l_cap: no free row; null or
 * misaligned pointer; bad dims), SAGA_ERR_UNSUPPORTED, SAGA_ERR_DEVICE,
 * SAGA_ERR_CUDA. */
int saga_cache_append(const saga_dims* dims, const void* k_new, const void* v_new, void* k,
                      void* v, saga_stream_t stream);

/* Failure-path self-test (the paper has no counterpart): one CTA waits, with
 * the bounded wait every pipelined kernel uses, on a barrier that nothing
 * completes; after limit_us microseconds (1 .. 1000000) it gives up, sets the
 * workspace's sticky timeout flag and returns.  Lets a test check that a
 * wait which runs out surfaces as SAGA_ERR_TIMEOUT from saga_workspace_error
 * and leaves the context usable.  Only the first 256 bytes of ws are used. */
int saga_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us, saga_stream_t stream);

/* Enqueue a zeroing of the workspace (sticky flags included). */
int saga_workspace_reset(void* ws, size_t ws_bytes, saga_stream_t stream);

/* Synchronise `stream`, read and clear the workspace's sticky device flag:
 * SAGA_OK, SAGA_ERR_TIMEOUT, SAGA_ERR_BOUNDS (debug builds only: the
 * library compiled with SAGA_DEBUG checks every position, count and slot a
 * kernel takes from another kernel's output, and skips the access instead
 * of trapping), or SAGA_ERR_CUDA if the read itself failed. */
int saga_workspace_error(void* ws, size_t ws_bytes, saga_stream_t stream);

/* Synchronise `stream`, then read and clear the workspace's count of rows
 * that kept nothing and took the empty-set rule (tau_eff = min(tau, row
 * max): a stale threshold above every logit of the row keeps its maximal
 * entries; the pages leave that case open) in the decode calls since the
 * last read, into *count_out.  Rows of saga_atopn_decode_partial are not
 * counted (the merge of the shards decides their rule). */
int saga_workspace_empty_rows(void* ws, size_t ws_bytes, uint64_t* count_out, saga_stream_t stream);

/* Static description of a status code. */
const char* saga_status_string(int status);

/* Number of kernels this library has launched in this process (host counter,
 * incremented per launch; graph replays are not counted). */
uint64_t saga_launch_count(void);

/* Measurement hook for the calling host thread: while set, the dominant
 * kernel of each call (the fused decode kernel, the dense kernel, the logits
 * kernel) is bracketed by cudaEventRecord(start) / cudaEventRecord(stop) on
 * the call's stream.  Pass NULL, NULL to clear.  Events are cudaEvent_t. */
void saga_set_kernel_events(void* start_event, void* stop_event);

/* ABI version (major * 100 + minor). */
int saga_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAGA_H */
