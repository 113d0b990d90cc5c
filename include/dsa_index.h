/*
 * dsa_index.h — C ABI of the B200 (sm_100a) lightning-indexer library.
 *
 * The DeepSeek Sparse Attention (DSA) lightning indexer selects, for every
 * query, the k keys of its causal prefix that sparse attention will read.
 * In the pages this library follows, the indexer has to score each key that
 * precedes a query and it retains the k = 2048 best positions (PIVOT:
 * Efficient Query-Group Indexing for Token-Level Sparse Attention — Abstract;
 * MLI Restructures DeepSeek Sparse Attention — Core Idea); the pages do not
 * print the score itself.
 * This library uses the standard DSA indexer score
 *
 *     I[t, s] = sum_h  w[t, h] * ReLU( q[t, h, :] . k[s, :] )
 *
 * with fp32 accumulation, no extra scale, and (fp8 keys) k[s, :] =
 * e4m3(bytes[s, :]) * K_scale[s].  Query row t sits at key position
 * p_t = q_pos0 + t and sees keys 0..p_t (causal prefix; AttentionIndex
 * Architecture — Key findings: causality is a hard constraint).
 *
 * Selection: the k largest I[t, s] over s <= p_t, ties broken toward the
 * lower key index.  Each output row is a SET: its min(k, p_t + 1) entries
 * (index, score) come in no particular order; the remaining slots hold
 * index -1 and score -inf.
 *
 * Conventions for every call below
 *   - All tensor pointers are DEVICE pointers on the current CUDA device
 *     (except the *_host calls, whose tensors are in host memory),
 *     row-major and contiguous, 16-byte aligned.  Offsets arrays of the decode
 *     call are device pointers too.
 *   - The caller owns every buffer, including `workspace`; the library never
 *     allocates, never frees and never synchronises `stream` (a cudaStream_t;
 *     NULL is the legacy default stream).  Calls are asynchronous.
 *   - Size the workspace with the matching *_workspace_size call; its first
 *     bytes hold a device status word that kernels set on a device-side
 *     failure (a bounded wait that gave up); read it with dsa_check_status.
 *     Zero the workspace's first 8 bytes before its first use;
 *     dsa_check_status clears the word again after reading it.
 *   - Return value: DSA_OK or a negative DSA_ERR_* code; on an error nothing
 *     has been launched.
 *   - Empty calls are valid: no query rows (prefill T = 0; decode B = 0,
 *     then total_q = total_keys = 0).  They check the shape arguments,
 *     launch nothing, may pass NULL tensor pointers and return DSA_OK; their
 *     workspace (or staging) size is 256 bytes.
 *   - Supported shapes: bf16 Q/K with H = 64, d = 128 run on the tcgen05
 *     tensor-core kernel; fp32 Q/K (any H <= 128, d <= 256, H*d <= 8192) and
 *     other bf16 / fp8-key shapes run on an exact fp32 CUDA-core kernel.
 *   - Inputs must be finite.
 */
#ifndef DSA_INDEX_H
#define DSA_INDEX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types */
#define DSA_DTYPE_BF16 0
#define DSA_DTYPE_FP32 1
#define DSA_DTYPE_FP8_E4M3 2 /* keys only; needs K_scale */

/* status codes */
#define DSA_OK 0
#define DSA_ERR_INVALID_ARG (-1) /* null pointer, bad size, misaligned pointer */
#define DSA_ERR_UNSUPPORTED (-2) /* valid but not implemented shape / dtype */
#define DSA_ERR_WORKSPACE (-3)   /* workspace too small */
#define DSA_ERR_CUDA (-4)        /* a CUDA runtime call or launch failed */
#define DSA_ERR_TIMEOUT (-5)     /* a device-side bounded wait gave up */
#define DSA_ERR_DEVICE (-6)      /* current device is not sm_100 */
#define DSA_ERR_INTERNAL (-7)    /* a device-side consistency check failed */

/* group modes (PIVOT abstract: the Refine and Reuse variants; ADIndex —
 * Inference: refinement that also adds query-specific tokens) */
#define DSA_GROUP_REFINE 0
#define DSA_GROUP_REUSE 1
#define DSA_GROUP_REFINE_LOCAL 2

/* Human-readable text for a status code (static storage). */
const char* dsa_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int dsa_version(void);

/* Failure-path control, for tests of the bounded waits (ADIndex — Deployment
 * Guidance: a fallback path is only trustworthy once it has been exercised).
 * Every wait of the tensor-core kernel is bounded: when it runs out, the
 * kernel records DSA_ERR_TIMEOUT in the status word, lets the copies and MMAs
 * it already issued land, frees its tensor memory and returns, so the device
 * stays usable.  `budget_us` sets the time budget, in microseconds, of the
 * waits between the kernel's roles for the tensor-core launches that follow
 * (0 restores the default of 2 s; the final drain of issued work always
 * keeps the default).
 * With `hold_first_tile` nonzero, the first CTA of the following dense-kind
 * launches never loads its first key tile, so the wait for it runs out and
 * that launch reports DSA_ERR_TIMEOUT (its outputs are then unspecified).
 * Process-wide, read at each launch; call it between calls, never while
 * another thread launches.  Returns DSA_OK. */
int dsa_debug_set_wait(unsigned int budget_us, int hold_first_tile);

/* Synchronises `stream`, then reads and clears the device status word kept
 * in `workspace`.  Returns DSA_OK, the recorded DSA_ERR_TIMEOUT,
 * DSA_ERR_INTERNAL or DSA_ERR_INVALID_ARG (decode offsets that failed their
 * device check), or DSA_ERR_CUDA if the stream reported an error. */
int dsa_check_status(void* workspace, void* stream);

/* ------------------------------------------------------------------------
 * Dense prefill indexer.
 *   Q   [T, H, d]  bf16 or fp32 (q_dtype)
 *   w   [T, H]     fp32 head weights
 *   K   [N, d]     bf16, fp32 or fp8 e4m3 bytes (k_dtype)
 *   K_scale [N]    fp32 per-key scale (> 0), fp8 keys only, else NULL
 *   q_pos0         key position of query row 0; needs 0 <= q_pos0 and
 *                  q_pos0 + T <= N
 *   k              keys kept per query, 1 <= k <= 65536
 *   idx [T, k] int32, val [T, k] fp32 — outputs (see selection above)
 * Cost: O(sum_t (p_t + 1) * H * d) multiply-adds; the [T, N] score matrix
 * is never written to memory.
 * ---------------------------------------------------------------------- */
int dsa_index_dense_workspace_size(int T, int N, int H, int d, int k,
                                   int q_dtype, int k_dtype, size_t* bytes);
int dsa_index_dense(const void* Q, const float* w, const void* K,
                    const float* K_scale, int T, int N, int H, int d,
                    int64_t q_pos0, int k, int q_dtype, int k_dtype,
                    int32_t* idx, float* val, void* workspace,
                    size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Group-shared prefill indexer (PIVOT abstract): the queries of a group are
 * merged into one proxy query, one scan of the whole prefix by that proxy
 * yields a candidate bank, and each query's top-k is then taken from the
 * bank.
 *   group  G >= 1: rows gG .. min(T,(g+1)G)-1 form group g; ng = ceil(T/G)
 *   bank   B >= k: candidate-bank size of the proxy scan
 *   mode   DSA_GROUP_REFINE: member t re-scores the bank keys <= p_t with
 *          its own q, w and keeps its top-k.
 *          DSA_GROUP_REUSE: member t keeps the first k bank keys <= p_t in
 *          the proxy's ranking, valued by the proxy score.
 *          DSA_GROUP_REFINE_LOCAL: Refine whose candidates also hold the
 *          member's own stretch of the group, positions p_first .. p_t
 *          (p_first = the group's first member): the query-specific tokens
 *          the ADIndex page keeps in refinement, read as the recent keys a
 *          shared proxy may rank low.  Needs G <= 4096.
 *   Proxy: qbar[g] = mean of the members' q (fp32 mean, rounded to q_dtype),
 *          wbar[g] = mean of the members' w (fp32).  The proxy scans keys
 *          0..L_g, L_g = position of the group's last member.
 *   bank_idx [ng, B] int32, bank_val [ng, B] fp32: optional outputs (NULL to
 *          skip) — the bank in the proxy's ranking order (score descending,
 *          lower key first).  Unused slots: -1 / -inf.  Asking for them
 *          costs a sort of every group's bank; without them Refine does not
 *          rank the bank (it re-scores it as a set) and Reuse ranks only the
 *          bank's top k + G - 1 entries, the only ones a member can take.
 *   proxy_q [ng, H, d] (q_dtype), proxy_w [ng, H] fp32: optional outputs.
 * ---------------------------------------------------------------------- */
int dsa_index_group_workspace_size(int T, int N, int H, int d, int k,
                                   int group, int bank, int q_dtype,
                                   int k_dtype, size_t* bytes);
int dsa_index_group(const void* Q, const float* w, const void* K,
                    const float* K_scale, int T, int N, int H, int d,
                    int64_t q_pos0, int k, int group, int bank, int mode,
                    int q_dtype, int k_dtype, int32_t* idx, float* val,
                    int32_t* bank_idx, float* bank_val, void* proxy_q,
                    float* proxy_w, void* workspace, size_t workspace_bytes,
                    void* stream);

/* ------------------------------------------------------------------------
 * Decode indexer over a batch of key caches (ADIndex — Why the Indexer
 * Becomes the Bottleneck: each decode query rescans the historical keys;
 * PIVOT abstract: the queries of one multi-token-prediction step).
 *   K [sum N_b, d]: sequence b owns rows k_offsets[b] .. k_offsets[b+1]-1
 *   Q [sum m_b, H, d], w [sum m_b, H]: sequence b owns query rows
 *          q_offsets[b] .. q_offsets[b+1]-1 (1 <= m_b <= min(4, N_b))
 *   New query j of sequence b sits at position N_b - m_b + j and sees its
 *   sequence's keys 0 .. N_b - m_b + j.  Output indices are local to the
 *   sequence (0 .. N_b - 1).
 *   k_offsets [B+1] int64, q_offsets [B+1] int32: DEVICE arrays, read on
 *          the device only (no synchronisation).  The kernels check every
 *          sequence they read: 0 <= k_offsets[b], 1 <= N_b <= max_keys,
 *          k_offsets[b+1] <= total_keys, 0 <= q_offsets[b], q_offsets[b+1]
 *          <= total_q, 1 <= m_b <= min(4, N_b).  A sequence that fails is
 *          skipped and DSA_ERR_INVALID_ARG is recorded in the status word
 *          (dsa_check_status); the outputs of such a call are unspecified,
 *          but no kernel reads or writes outside the buffers the sizes
 *          describe.
 *   total_keys: k_offsets[B] (host value: rows of K; tensor copies never
 *          read beyond it).
 *   max_keys: an upper bound on every N_b (host value; sizes the split of
 *          each cache over the GPU's multiprocessors and the workspace);
 *          max_keys <= total_keys.
 *   On the tensor-core path (bf16 q, bf16 or fp8 k, H = 64, d = 128) K
 *   rows are addressed with 32-bit coordinates: total_keys above
 *   2^31 - 256 returns DSA_ERR_UNSUPPORTED.
 * ---------------------------------------------------------------------- */
int dsa_index_decode_workspace_size(int B, int total_q, int max_keys, int H,
                                    int d, int k, int q_dtype, int k_dtype,
                                    size_t* bytes);
int dsa_index_decode(const void* Q, const float* w, const void* K,
                     const float* K_scale, const int64_t* k_offsets,
                     const int32_t* q_offsets, int B, int total_q,
                     int64_t total_keys, int max_keys, int H, int d, int k,
                     int q_dtype,
                     int k_dtype, int32_t* idx, float* val, void* workspace,
                     size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * PIVOT in decode (PIVOT abstract: the queries decoded together in one
 * multi-token-prediction step form a natural group).  Sequence b's m_b new
 * queries are one group:
 *   proxy   qbar[b] = mean of its queries' q (fp32 mean, rounded to q_dtype),
 *           wbar[b] = mean of their w (fp32); the proxy sits at the last
 *           query's position N_b - 1 and scans keys 0..N_b - 1;
 *   bank    the proxy's top-`bank` keys (indices local to the sequence);
 *   mode    DSA_GROUP_REFINE: query j (position N_b - m_b + j) re-scores the
 *           bank keys <= its position with its own q, w and keeps its top-k;
 *           DSA_GROUP_REUSE: it keeps the first k bank keys <= its position
 *           in the proxy's ranking, valued by the proxy score;
 *           DSA_GROUP_REFINE_LOCAL: Refine whose candidates also hold the
 *           sequence's new keys N_b - m_b .. its own position.
 *   Arguments as for dsa_index_decode (1 <= m_b <= min(4, N_b), device
 *   offsets, local output indices; a first kernel checks the offsets as
 *   listed there plus q_offsets[B] = total_q, and when they fail no later
 *   kernel of the call does any work), plus bank (k <= bank <= 16384), mode and
 *   the optional outputs bank_idx/bank_val [B, bank] (ranked, -1 / -inf
 *   padded; asking for them costs a sort of every bank) and proxy_q
 *   [B, H, d] (q_dtype) / proxy_w [B, H] fp32.  Tensor-core shape only (bf16
 *   q, bf16 or fp8 k, H = 64, d = 128); other shapes DSA_ERR_UNSUPPORTED.
 * ---------------------------------------------------------------------- */
int dsa_index_decode_group_workspace_size(int B, int total_q, int max_keys,
                                          int H, int d, int k, int bank,
                                          int q_dtype, int k_dtype,
                                          size_t* bytes);
int dsa_index_decode_group(const void* Q, const float* w, const void* K,
                           const float* K_scale, const int64_t* k_offsets,
                           const int32_t* q_offsets, int B, int total_q,
                           int64_t total_keys, int max_keys, int H, int d,
                           int k, int bank, int mode, int q_dtype,
                           int k_dtype, int32_t* idx, float* val,
                           int32_t* bank_idx, float* bank_val, void* proxy_q,
                           float* proxy_w, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Two-stage selection over contiguous key blocks (block routing; the
 * AttentionIndex page, Why Positional Blocks Lose Recall): a comparator for
 * the dense and group-shared forms.  Keys form blocks of 128 (the last one
 * may be shorter); a block's representative is its mean key (fp32 mean of
 * the keys times their scale, rounded to bf16).  Query t at p_t:
 *   route   score the representatives of the complete blocks before it
 *           (blocks 0 .. (p_t+1)/128 - 1: no key beyond p_t reaches routing)
 *           with the indexer formula and keep the best n_blocks (ties to the
 *           lower block);
 *   refine  the candidates are those blocks' keys plus its own partial block
 *           (keys (p_t+1)/128*128 .. p_t); keep the top-k by the native
 *           score.
 *   Arguments as for dsa_index_dense, plus n_blocks (1 .. 65536) and the
 *   optional outputs block_idx [T, n_blocks] int32 (routed blocks, -1
 *   padded, in no particular order) and reps [ceil(N/128), d] bf16.
 *   Tensor-core shape only (bf16 q, bf16 or fp8 k, H = 64, d = 128).
 * ---------------------------------------------------------------------- */
int dsa_index_block_routed_workspace_size(int T, int N, int H, int d, int k,
                                          int n_blocks, int q_dtype,
                                          int k_dtype, size_t* bytes);
int dsa_index_block_routed(const void* Q, const float* w, const void* K,
                           const float* K_scale, int T, int N, int H, int d,
                           int64_t q_pos0, int k, int n_blocks, int q_dtype,
                           int k_dtype, int32_t* idx, float* val,
                           int32_t* block_idx, void* reps, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Inverted-file routing (AttentionIndex page: keys grouped by similarity
 * rather than position, each query routed over the cluster centres, the
 * candidates refined with the native indexer score), a comparator in its
 * plain form: no learned encoder, no causal index versions (causality by
 * masking: a query's candidates are cluster members with key <= p_t).
 *
 * dsa_ivf_build: Lloyd k-means over the keys (Euclidean; centroid i starts
 *   at key floor(i N / C); nearest centroid, ties to the lower one; means;
 *   an empty cluster keeps its centroid), `iters` >= 1 iterations, then the
 *   keys are laid out cluster after cluster in `index` (size from
 *   dsa_ivf_index_size; the caller owns it).  fp8 keys are clustered by
 *   their scaled values.  Centroid sums use atomics, so the low bits of the
 *   centroids (and, at near-ties, assignments) may differ between runs.
 *   Layout of `index` (256-byte aligned parts): off [C+1] int32, perm [N]
 *   int32 (clustered row -> key), assign [N] int32, keys [N, d] bf16,
 *   centroids [C, d] bf16, centroids [C, d] fp32.
 * dsa_index_ivf_routed: query t scores the bf16 centroids with the indexer
 *   formula, keeps the best n_probe clusters (ties to the lower cluster),
 *   and keeps the top-k of the native score over their members with key
 *   <= p_t.  max_tiles bounds the 128-row tiles of one query's probed
 *   clusters (sum of ceil(size/128)); a query above it is cut there and
 *   DSA_ERR_INTERNAL is recorded.  cluster_idx [T, n_probe]: optional
 *   output.  Tensor-core shape only (bf16 q, bf16 or fp8 k, H = 64,
 *   d = 128).
 * ---------------------------------------------------------------------- */
int dsa_ivf_index_size(int N, int d, int C, size_t* bytes);
int dsa_ivf_build_workspace_size(int N, int H, int d, int C, int q_dtype,
                                 int k_dtype, size_t* bytes);
int dsa_ivf_build(const void* K, const float* K_scale, int N, int H, int d,
                  int C, int iters, int q_dtype, int k_dtype, void* index,
                  size_t index_bytes, void* workspace, size_t workspace_bytes,
                  void* stream);
int dsa_index_ivf_routed_workspace_size(int T, int N, int H, int d, int k,
                                        int C, int n_probe, int max_tiles,
                                        int q_dtype, int k_dtype,
                                        size_t* bytes);
int dsa_index_ivf_routed(const void* Q, const float* w, const void* index,
                         const float* K_scale, int T, int N, int H, int d,
                         int64_t q_pos0, int k, int C, int n_probe,
                         int max_tiles, int q_dtype, int k_dtype,
                         int32_t* idx, float* val, int32_t* cluster_idx,
                         void* workspace, size_t workspace_bytes,
                         void* stream);

/* ------------------------------------------------------------------------
 * Dense indexer that allocates nothing (the pages have no counterpart: this
 * is an integration aid).  For callers that cannot hand the library a
 * workspace — code running inside a host application that reserved all
 * device memory up front (a serving engine sizing its KV cache to the whole
 * GPU, say), or a loop where a late cudaMalloc may fail under memory pressure
 * or stall the device.
 *   Same inputs, outputs and results as dsa_index_dense with bf16 Q/K,
 *   H = 64 and d = 128 (other shapes: DSA_ERR_UNSUPPORTED).  No workspace:
 *   the scratch (a status word and per-CTA candidate lists) lives in a fixed
 *   32 MiB array in device memory that every GPU loading this library holds
 *   until the process exits.  Each CTA needs 4 * round_up(N, 512) * 8 bytes
 *   of it; the grid shrinks to fit, and N above about 1.04 million keys
 *   returns DSA_ERR_WORKSPACE.
 *   The first call on a device looks up that device's copy of the array
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   The call is synchronous: it waits for `stream` and returns the device
 *   status of this call (DSA_OK, DSA_ERR_TIMEOUT, DSA_ERR_INTERNAL).
 *   Every call on a device shares the one array: calls that overlap on the
 *   GPU (other streams, other host threads) race; serialise them.
 *   It calls no allocation routine (no cudaMalloc, no cudaFree).
 * ---------------------------------------------------------------------- */
int dsa_index_dense_static(const void* Q, const float* w, const void* K, int T,
                           int N, int H, int d, int64_t q_pos0, int k,
                           int32_t* idx, float* val, void* stream);

/* ------------------------------------------------------------------------
 * Host-buffer entry points (an integration aid; the pages have none): the
 * dense, group and decode indexers above with every tensor argument in HOST
 * memory — inputs, outputs and, for decode, the offsets arrays.  Same
 * operation, argument meaning, layouts and results as the device calls.
 *   staging: a DEVICE buffer of at least *_host_staging_size bytes, 16-byte
 *          aligned, owned by the caller; the call stages the inputs, the
 *          outputs and the indexer's workspace in it (no zeroing needed).
 *   chunk_rows (dense, group): rows per pipeline chunk, 0 for the library's
 *          choice (about 16 chunks of at least 1024 rows, at most 64
 *          chunks), rounded up to a multiple of 4 (dense) or of `group`, so
 *          that every group lies inside one chunk and the results equal one
 *          call over all rows.  The keys are copied first; then, chunk by
 *          chunk, the copy in of chunk c+1, the indexer on chunk c and the
 *          copy out of chunk c-1 overlap: the copies run on two streams the
 *          call creates and destroys, the indexer on `stream`, ordered by
 *          events.  The group staging size depends on chunk_rows: pass the
 *          same value to both calls.
 *   Decode is one chunk (the cache copy dwarfs the scan); its copies and
 *          the indexer run on `stream`.
 *   Synchronous: returns once the outputs are in host memory (or an error
 *   has stopped the call and every copy it queued has drained), with
 *   DSA_OK, a DSA_ERR_* of the arguments or of a CUDA call, or the device
 *   status of the call (DSA_ERR_TIMEOUT, DSA_ERR_INTERNAL).
 *   Host buffers should be page-locked (cudaHostAlloc, cudaHostRegister):
 *   then the copies overlap the indexer; pageable memory gives the same
 *   results with the copies serialised by the driver.
 * ---------------------------------------------------------------------- */
int dsa_index_dense_host_staging_size(int T, int N, int H, int d, int k,
                                      int q_dtype, int k_dtype,
                                      size_t* bytes);
int dsa_index_dense_host(const void* Q, const float* w, const void* K,
                         const float* K_scale, int T, int N, int H, int d,
                         int64_t q_pos0, int k, int q_dtype, int k_dtype,
                         int chunk_rows, int32_t* idx, float* val,
                         void* staging, size_t staging_bytes, void* stream);
int dsa_index_group_host_staging_size(int T, int N, int H, int d, int k,
                                      int group, int bank, int q_dtype,
                                      int k_dtype, int chunk_rows,
                                      size_t* bytes);
int dsa_index_group_host(const void* Q, const float* w, const void* K,
                         const float* K_scale, int T, int N, int H, int d,
                         int64_t q_pos0, int k, int group, int bank, int mode,
                         int q_dtype, int k_dtype, int chunk_rows,
                         int32_t* idx, float* val, void* staging,
                         size_t staging_bytes, void* stream);
int dsa_index_decode_host_staging_size(int B, int total_q,
                                       int64_t total_keys, int max_keys,
                                       int H, int d, int k, int q_dtype,
                                       int k_dtype, size_t* bytes);
int dsa_index_decode_host(const void* Q, const float* w, const void* K,
                          const float* K_scale, const int64_t* k_offsets,
                          const int32_t* q_offsets, int B, int total_q,
                          int64_t total_keys, int max_keys, int H, int d,
                          int k, int q_dtype, int k_dtype, int32_t* idx,
                          float* val, void* staging, size_t staging_bytes,
                          void* stream);

/* ------------------------------------------------------------------------
 * Test aid: the full score matrix S [T, N] fp32 of the dense call (the same
 * kernel and epilogue arithmetic; entries with s > p_t hold -inf).
 * Needs T * N <= 2^26.  Uses the dense workspace.
 * ---------------------------------------------------------------------- */
int dsa_debug_scores(const void* Q, const float* w, const void* K,
                     const float* K_scale, int T, int N, int H, int d,
                     int64_t q_pos0, int q_dtype, int k_dtype, float* S,
                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Kernel timer (instrumentation; the pages describe no counterpart).
 *
 * dsa_kernel_timer_start arms a process-wide timer: each later launch of the
 * scoring kernel (tensor-core or fp32 CUDA-core; made by dsa_index_dense,
 * dsa_index_group, dsa_index_decode, dsa_index_dense_static or
 * dsa_debug_scores) records a CUDA event pair around itself on the caller's
 * stream, for the first max_launches launches; later ones are not timed.
 * The proxy, gather, rank, merge and widening kernels are never timed.  The
 * events are created here, so arm the timer outside a timed region and
 * outside CUDA graph capture.
 *
 * dsa_kernel_timer_stop disarms it, waits for the recorded events, writes the
 * summed duration of the timed launches in milliseconds to *total_ms and
 * their number to *launches, and destroys the events.
 *
 * Both return DSA_OK; DSA_ERR_INVALID_ARG for max_launches outside
 * [1, 2^20], a start while armed, a stop while disarmed or a null pointer;
 * DSA_ERR_CUDA if creating or reading an event fails.  Launches from several
 * host threads are counted in the order they take a slot.
 * ---------------------------------------------------------------------- */
int dsa_kernel_timer_start(int max_launches);
int dsa_kernel_timer_stop(float* total_ms, int* launches);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEX_H */
