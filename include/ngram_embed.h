/*
 * ngram_embed.h — C ABI of libngram_embed.so: the forward hot path of the hashed
 * N-gram embedding layer ("Over-Encoding") on one NVIDIA B200 (sm_100a).
 *
 * The operation is defined in "Scaling Embeddings Outperforms Scaling Experts in
 * Language Models" (LongCat team), section 2 "N-gram Embedding":
 *   Eq. 2  H_{n,k}(t_{i-n+1..i}) = (sum_{j=0}^{n-1} t_{i-j} * V0^j) mod V_{n,k}
 *   Eq. 3  e_i = ( E_0(t_i) + sum_{n=2..N} sum_{k=1..K} W_{n,k} E_{n,k}(H_{n,k}(...)) )
 *                / ((N-1)K + 1)
 * with E_0 in R^{V0 x D}, E_{n,k} in R^{V_{n,k} x d}, W_{n,k} in R^{D x d}, d = D/((N-1)K);
 * and in section 4.2 "N-gram Cache": n-gram context ids kept per sequence on the
 * device, updated as speculative tokens are accepted or rejected.
 *
 * Conventions (the paper is silent on them):
 *   - S = (N-1)K sub-tables in the order s = (n-2)K + (k-1), n = 2..N, k = 1..K.
 *   - W_stacked is [D x D] row-major with W_stacked[o][s*d + c] = W_{n,k}[o][c], so the
 *     projection is G * W_stacked^T, G[i] = concat_s E_s[idx[i][s]].
 *   - A position before the start of a sequence reads the pad id 0 (prefill), or the
 *     sequence's committed history in the N-gram cache (decode).
 *   - Eq. 2 is evaluated exactly (Horner's rule, every step reduced mod V_{n,k} in
 *     64-bit integers; no wrap-around).
 *
 * Memory and ownership: every device buffer (tables, W, tokens, offsets, outputs, cache
 * arrays, workspace) is allocated and owned by the caller. The library owns only the
 * host-side plan. No call allocates device memory or synchronises, except
 * ngram_embed_get_status (which synchronises its stream). Calls are asynchronous and
 * ordered by `stream` (a cudaStream_t passed as void*; NULL = the legacy default stream).
 * A plan may be used from one host thread at a time.
 *
 * Layouts: all tables are dense row-major. bf16 tables hold raw bf16 bit patterns.
 * Device pointers to tables, W, outputs and the workspace must be 16-byte aligned;
 * for the tensor-core path (bf16, D % 128 == 0, d % 64 == 0) table rows are d*2 bytes,
 * a multiple of 16, and the base pointers 16-byte aligned.
 *
 * Errors: functions return NGRAM_OK (0) or a negative NGRAM_ERR_* code for bad
 * arguments found on the host; nothing is launched then. Errors that only the device
 * can see (a token id outside [0, V0), decreasing offsets, a bad cache slot, an invalid
 * rollback, an evicted context position, a bounded wait that ran out) set bits of a
 * sticky status word in the workspace (NGRAM_STATUS_*); the kernels then substitute a
 * safe value (row 0, the pad id, or leave the cache slot unchanged) and never trap.
 * Read the word with ngram_embed_get_status; clear it with ngram_embed_clear_status.
 */
#ifndef NGRAM_EMBED_H
#define NGRAM_EMBED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes (host-side checks) ---- */
#define NGRAM_OK 0
#define NGRAM_ERR_INVALID_ARG -1   /* NULL pointer, negative size, bad config value */
#define NGRAM_ERR_UNSUPPORTED -2   /* config outside the supported limits */
#define NGRAM_ERR_MISALIGNED -3    /* a pointer is not 16-byte aligned */
#define NGRAM_ERR_WORKSPACE -4     /* workspace smaller than ngram_embed_workspace_bytes */
#define NGRAM_ERR_CUDA -5          /* a CUDA runtime/driver call or a launch failed */

/* ---- sticky device status bits (in the workspace) ---- */
#define NGRAM_STATUS_BAD_TOKEN 0x1       /* token id outside [0, V0); row 0 / pad used */
#define NGRAM_STATUS_BAD_OFFSETS 0x2     /* seq/tok offsets not non-decreasing from 0 to T */
#define NGRAM_STATUS_BAD_SLOT 0x4        /* cache slot outside [0, max_seqs) */
#define NGRAM_STATUS_BAD_APPEND 0x8      /* append of more than `capacity` ids */
#define NGRAM_STATUS_BAD_ROLLBACK 0x10   /* rollback < 0, > committed, or past the ring */
#define NGRAM_STATUS_EVICTED 0x20        /* context position no longer held by the ring */
#define NGRAM_STATUS_TIMEOUT 0x40        /* a bounded device wait ran out (kernel returned) */

/* ---- element types ---- */
#define NGRAM_BF16 0
#define NGRAM_F32 1

/* ---- limits ---- */
#define NGRAM_MAX_N 8          /* largest n-gram order */
#define NGRAM_MAX_SUBTABLES 32 /* largest S = (N-1)K */

typedef struct ngram_embed_plan ngram_embed_plan; /* opaque, host-side */

/* Shape of one N-gram embedding layer (section 2, Eq. 3). */
typedef struct {
  int64_t V0;          /* base vocabulary size, 1 <= V0 < 2^31 */
  int32_t D;           /* hidden size; D % S == 0 */
  int32_t N;           /* largest n-gram order, 1 <= N <= NGRAM_MAX_N (N = 1: e_i = E_0(t_i)) */
  int32_t K;           /* sub-tables per order, K >= 1, S = (N-1)K <= NGRAM_MAX_SUBTABLES */
  const int64_t* V_nk; /* host array of S sub-table sizes in order s, 1 <= V_nk < 2^31 */
  int32_t dtype;       /* NGRAM_BF16 or NGRAM_F32 (tables, W and output) */
} ngram_embed_config;

/* The decode-side N-gram cache (section 4.2): per slot, a ring of the newest ids.
 * All arrays are caller-owned device memory.
 *   ring[slot * capacity + (pos % capacity)] = committed id at position pos,
 *   len[slot]        = number of committed ids (positions 0 .. len-1),
 *   valid_from[slot] = oldest position the ring still holds.
 * capacity must be >= N-1 (a decode step of P ids per sequence needs >= N-1+P to roll
 * back a whole step). ngram_cache_reset zeroes len and valid_from. */
typedef struct {
  int32_t* ring;
  int64_t* len;
  int64_t* valid_from;
  int32_t capacity;
  int32_t max_seqs;
} ngram_cache;

/* Validate a config and build a plan on the current CUDA device.
 * Returns NGRAM_ERR_INVALID_ARG / NGRAM_ERR_UNSUPPORTED on a bad config. */
int ngram_embed_plan_create(const ngram_embed_config* cfg, ngram_embed_plan** out);
int ngram_embed_plan_destroy(ngram_embed_plan* plan);

/* Device workspace bytes for calls of up to max_tokens tokens: a 33,024-byte head (the
 * status word, then the stream-K arrival counters), the [max_tokens x S] int32 index
 * buffer, then, for plans that use the tensor-core kernel, 2 x (SM count) x 128 x W fp32
 * stream-K partial tiles, W = 512 where the 512-column pair tiles apply (D % 512 == 0, tile
 * width 256), else 256 (the plan's SM count: see ngram_embed_plan_set_sm_count), then,
 * while the dense-A form is on (ngram_embed_plan_set_dense_a), the [max_tokens x D] bf16
 * G buffer, each region rounded up to 256 bytes. A workspace without
 * the partials or G (head + index buffer) is accepted too; the projection then takes the
 * forms that fit. The head must be zeroed once before first use (ngram_embed_clear_status
 * does it); the rest needs no init. The kernels leave the counters zero after every call
 * that did not set NGRAM_STATUS_TIMEOUT. */
size_t ngram_embed_workspace_bytes(const ngram_embed_plan* plan, int64_t max_tokens);

/* The whole layer (section 2, Eq. 2 + Eq. 3) for num_tokens tokens in num_seqs sequences.
 *   tokens       [num_tokens] int32 device ids in [0, V0)
 *   seq_offsets  [num_seqs + 1] int32 device CSR offsets, 0 = off[0] <= ... <= off[B] = T
 *   E0           [V0 x D] device table; E_nk: HOST array of S device pointers, table s
 *                is [V_nk[s] x d]; W_stacked [D x D] device
 *   cache        NULL: positions before a sequence start read pad 0 (prefill).
 *                non-NULL: they read the committed history of cache slot
 *                cache_slots[b] (or b if cache_slots is NULL), as the ring holds it
 *                when the kernel runs.
 *   out          [num_tokens x D] device, dtype of the plan
 *   workspace    device, >= ngram_embed_workspace_bytes(plan, num_tokens) bytes
 * num_tokens may be 0 (nothing is launched). */
int ngram_embed_fwd(const ngram_embed_plan* plan, const int32_t* tokens,
                    const int32_t* seq_offsets, int32_t num_seqs, int64_t num_tokens,
                    const void* E0, const void* const* E_nk, const void* W_stacked,
                    const ngram_cache* cache, const int32_t* cache_slots, void* out,
                    void* workspace, size_t workspace_bytes, void* stream);

/* One speculative-decode step in two launches instead of three: the commit of the previous
 * step's accepted ids (exactly ngram_cache_commit(commit_tokens, commit_stride,
 * commit_counts), skipped if commit_counts is NULL) fused with this step's context hashing,
 * then the projection — the same results as ngram_cache_commit followed by ngram_embed_fwd
 * with the cache. Sequence b's slot is cache_slots[b] (or b) for both parts. */
int ngram_embed_fwd_step(const ngram_embed_plan* plan, const int32_t* commit_tokens,
                         int32_t commit_stride, const int32_t* commit_counts, const int32_t* tokens,
                         const int32_t* seq_offsets, int32_t num_seqs, int64_t num_tokens,
                         const void* E0, const void* const* E_nk, const void* W_stacked,
                         const ngram_cache* cache, const int32_t* cache_slots, void* out,
                         void* workspace, size_t workspace_bytes, void* stream);

/* Eq. 2 alone (context assembly + hash): idx_out[i * S + s] = H_{n,k}(...) as int32,
 * bit-exact. Arguments as for ngram_embed_fwd; idx_out is [num_tokens x S] device. */
int ngram_hash_indices(const ngram_embed_plan* plan, const int32_t* tokens,
                       const int32_t* seq_offsets, int32_t num_seqs, int64_t num_tokens,
                       const ngram_cache* cache, const int32_t* cache_slots, int32_t* idx_out,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Eq. 3 given indices from ngram_hash_indices: sub-row lookup, projection, E_0 add and
 * the 1/((N-1)K+1) scale. idx is [num_tokens x S] int32 device. */
int ngram_embed_project(const ngram_embed_plan* plan, const int32_t* tokens,
                        const int32_t* idx, int64_t num_tokens, const void* E0,
                        const void* const* E_nk, const void* W_stacked, void* out,
                        void* workspace, size_t workspace_bytes, void* stream);

/* The table lookups of Eq. 3 alone (the HBM-bound stage of a step, for callers that run
 * their own projection): G_out[i][s*d + c] = E_s[idx[i][s]][c], [T x D] device, plan dtype
 * (the concatenated sub-rows the projection multiplies). If E0_out is not NULL, also
 * E0_out[i] = E_0[tokens[i]] ([T x D], plan dtype); tokens and E0 are then required and
 * tokens outside [0, V0) read row 0 and set NGRAM_STATUS_BAD_TOKEN. Calls that copy 2^32
 * 16-byte vectors or more (about 500k tokens at D = 4096) return NGRAM_ERR_UNSUPPORTED. */
int ngram_embed_gather(const ngram_embed_plan* plan, const int32_t* idx, int64_t num_tokens,
                       const void* const* E_nk, void* G_out, const int32_t* tokens, const void* E0,
                       void* E0_out, void* workspace, size_t workspace_bytes, void* stream);

/* ---- N-gram cache (section 4.2) ----
 * slots: [n] int32 device cache slots, distinct within one call (NULL: slot i for entry i).
 * Invalid entries set a status bit and leave their slot unchanged. */

/* Forget the history of the listed slots (len = valid_from = 0). */
int ngram_cache_reset(const ngram_embed_plan* plan, const ngram_cache* cache,
                      const int32_t* slots, int32_t n, void* workspace, size_t workspace_bytes,
                      void* stream);

/* Commit ids: entry i appends tokens[tok_offsets[i] .. tok_offsets[i+1]) (device CSR,
 * at most `capacity` ids) to slot slots[i]. */
int ngram_cache_append(const ngram_embed_plan* plan, const ngram_cache* cache,
                       const int32_t* slots, const int32_t* tokens, const int32_t* tok_offsets,
                       int32_t n, void* workspace, size_t workspace_bytes, void* stream);

/* Commit the accepted prefix of a speculative step in one launch: entry i appends
 * tokens[i*stride .. i*stride + counts[i]) (device int32; 0 <= counts[i] <= min(stride,
 * capacity)) to slot slots[i]. Equivalent to ngram_cache_append of all `stride` ids followed
 * by ngram_cache_rollback of stride - counts[i]. */
int ngram_cache_commit(const ngram_embed_plan* plan, const ngram_cache* cache,
                       const int32_t* slots, const int32_t* tokens, int32_t stride,
                       const int32_t* counts, int32_t n, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Un-commit ids: entry i drops the newest counts[i] ids (device int32) of slot slots[i].
 * Rejected (status bit, slot unchanged) if counts[i] < 0, counts[i] > len, or the newest
 * N-1 remaining positions are no longer all held by the ring. */
int ngram_cache_rollback(const ngram_embed_plan* plan, const ngram_cache* cache,
                         const int32_t* slots, const int32_t* counts, int32_t n,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ngram_embed_fwd for callers that cannot allocate device memory (plugin hosts that pass a
 * layer only its inputs and outputs; latency-critical loops where cudaMalloc's implicit
 * device-wide synchronisation is not allowed). The paper has no counterpart: this is an
 * interface convenience. Same arguments and results as ngram_embed_fwd, but the workspace
 * is a fixed 4 MiB array inside the library (every GPU that loads the library holds it
 * until exit). A call needs the workspace head and its index buffer to fit:
 * 33,024 + num_tokens * S * 4 bytes (rounded up to 256) <= 4 MiB, about 131,000 tokens at
 * S = 8; larger calls return NGRAM_ERR_WORKSPACE and launch nothing. The stream-K schedule
 * runs only when its partial tiles fit too (2 x SMs x 128 x 256 x 4 bytes: a plan limited
 * to a few SMs by ngram_embed_plan_set_sm_count). Allocates nothing. The first call on a
 * device looks up the array's device address (once per device; a failed lookup returns
 * NGRAM_ERR_CUDA and is retried by the next call); make that first call before any stream
 * capture. Each call zeroes the array's whole head (the status word and the stream-K
 * arrival counters) on `stream`, then, if status_out (a device int32) is not NULL, copies
 * the call's device status bits there on `stream`. All calls share the one array and it
 * keeps the last call's contents: calls that overlap on the GPU (for example on two
 * streams) race and must be avoided. */
int ngram_embed_fwd_static_ws(const ngram_embed_plan* plan, const int32_t* tokens,
                              const int32_t* seq_offsets, int32_t num_seqs, int64_t num_tokens,
                              const void* E0, const void* const* E_nk, const void* W_stacked,
                              const ngram_cache* cache, const int32_t* cache_slots, void* out,
                              int32_t* status_out, void* stream);

/* ---- draft-phase embedding cache (section 4.2, optimisations for speculative decoding) ----
 * Embeddings computed while drafting are kept so that verification does not compute them
 * again. Entry (slot, j) holds the embedding of the token at in-step position j of the
 * sequence in cache slot `slot`, with the N ids of its window as the key. A token's output
 * depends only on its window, so a token whose window equals its entry's key takes the
 * stored row (bit-identical to what was computed), and nothing needs invalidating when
 * drafts are rejected or the history moves on. Caller-owned device arrays:
 *   keys [max_seqs x positions x N] int32 (reset before first use), emb [max_seqs x
 *   positions x D] in the plan dtype, 16-byte aligned. */
typedef struct {
  int32_t* keys;
  void* emb;
  int32_t positions;  /* entries per slot: the in-step positions (e.g. 1 + drafts) */
  int32_t max_seqs;   /* slots; must be >= the N-gram cache's max_seqs */
} ngram_draft_cache;

/* Empty the entries of slots[0..n) (of slots 0..n-1 if slots is NULL). */
int ngram_draft_cache_reset(const ngram_embed_plan* plan, const ngram_draft_cache* dc,
                            const int32_t* slots, int32_t n, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ngram_embed_fwd through the N-gram cache ring (cache required) and the draft cache: hits
 * are copied, misses computed (projection over the misses only, their count read on the
 * device) and stored. In-step positions beyond dc->positions are computed, not cached.
 *   hits_out   device int32 (may be NULL): incremented by the number of hits
 *   workspace  >= ngram_embed_draft_workspace_bytes(plan, num_tokens) */
size_t ngram_embed_draft_workspace_bytes(const ngram_embed_plan* plan, int64_t max_tokens);
int ngram_embed_fwd_draft(const ngram_embed_plan* plan, const int32_t* tokens,
                          const int32_t* seq_offsets, int32_t num_seqs, int64_t num_tokens,
                          const void* E0, const void* const* E_nk, const void* W_stacked,
                          const ngram_cache* cache, const int32_t* cache_slots,
                          const ngram_draft_cache* dc, void* out, int32_t* hits_out,
                          void* workspace, size_t workspace_bytes, void* stream);

/* ---- backward (training; the pages train the layer from scratch, section 6) ----
 * Gradients of Eq. 3 given g = dL/de (bf16 [num_tokens x D]) and the forward's indices
 * (idx from ngram_hash_indices, [num_tokens x S]); c = output scale / ((N-1)K+1):
 *   dE0[t_i]            += c g_i
 *   dE_nk[s][idx[i][s]] += (c g W_stacked)[i][s d .. s d + d)     (rows that collide add up)
 *   dW                  += c g^T G,  G[i] = the concatenated sub-rows of token i
 * All gradients are fp32 device arrays of their parameter's shape (dE0 [V0 x D], dE_nk[s]
 * [V_nk[s] x d], dW [D x D]), accumulated with atomic adds (the summation order varies
 * between runs; the terms do not). Any of dE0, dE_nk (HOST array of S device pointers) and
 * dW may be NULL to skip that gradient; W_stacked is needed for dE_nk, E_nk for dW.
 * bf16 tensor-core plans only (else NGRAM_ERR_UNSUPPORTED). Index values outside
 * [0, V_nk) read/write row 0 and set NGRAM_STATUS_BAD_TOKEN.
 *   workspace  >= ngram_embed_bwd_workspace_bytes(plan, num_tokens): G, the gathered
 *              sub-rows [num_tokens x D] bf16, and the dE0 sort buffers (about
 *              2 D num_tokens + 4 V0 + 8 num_tokens bytes); its head is the status word.
 * The GEMMs read g and W_stacked where they lie (the tensor cores take the operands that are
 * not K-major in memory as MN-major tiles): nothing is transposed. */
size_t ngram_embed_bwd_workspace_bytes(const ngram_embed_plan* plan, int64_t max_tokens);
int ngram_embed_bwd(const ngram_embed_plan* plan, const int32_t* tokens, const int32_t* idx,
                    int64_t num_tokens, const void* const* E_nk, const void* W_stacked,
                    const void* grad_out, float* dE0, float* const* dE_nk, float* dW,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ---- hash statistics (section 3.2.2, Fig. 3): choosing table sizes ----
 * For the n-gram hash H = X_n mod V (Eq. 2, the layer's context rule: pad 0 before a
 * sequence start) over a token stream:
 *   rows_hit[j]       number of distinct rows (X_n mod moduli[j]) hit by the stream
 *                     (hit rate = rows_hit[j] / moduli[j]);
 *   *distinct_ngrams  number of distinct n-gram windows in the stream (exact: windows
 *                     compared as integers X_n when V0^n < 2^64, else id by id);
 *   collisions at moduli[j] = *distinct_ngrams - rows_hit[j].
 * tokens / seq_offsets as for ngram_embed_fwd (device); moduli, rows_hit, distinct_ngrams
 * are HOST arrays. Analysis, not the hot path: the call synchronises `stream`.
 *   workspace  >= ngram_hash_stats_workspace_bytes(num_tokens, max modulus, num_moduli) */
size_t ngram_hash_stats_workspace_bytes(int64_t max_tokens, int64_t max_modulus, int num_moduli);
int ngram_hash_stats(int64_t V0, int n, const int32_t* tokens, const int32_t* seq_offsets,
                     int32_t num_seqs, int64_t num_tokens, const int64_t* moduli, int num_moduli,
                     int64_t* rows_hit, int64_t* distinct_ngrams, void* workspace,
                     size_t workspace_bytes, void* stream);

/* ---- embedding amplification (section 3.2.4) ----
 * The pages amplify the N-gram embedding output early in training, either by a constant
 * factor or by a LayerNorm before it joins the residual stream (the factor is garbled in
 * the text: a sqrt(D)-like constant; the caller chooses it).
 *
 * Multiply every output of ngram_embed_fwd / ngram_embed_project by `scale` (folded into
 * the 1/((N-1)K+1) factor of the epilogue: no extra pass). Default 1. Rejects 0 and
 * non-finite values. */
int ngram_embed_plan_set_output_scale(ngram_embed_plan* plan, float scale);

/* y[i] = (x[i] - mean(x[i])) / sqrt(var(x[i]) + eps) * gamma + beta over each row of D
 * values (population variance; fp32 arithmetic; plan dtype in and out).
 *   x, y   [num_tokens x D] device, 16-byte aligned; y may equal x (in place)
 *   gamma, beta  [D] fp32 device, or NULL for 1 and 0
 *   eps    in [0, 1] */
int ngram_embed_layernorm(const ngram_embed_plan* plan, const void* x, int64_t num_tokens,
                          const float* gamma, const float* beta, float eps, void* y,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream` and copy the sticky status word to *status_out. */
int ngram_embed_get_status(const void* workspace, void* stream, int32_t* status_out);
/* Zero the workspace head: status word and stream-K counters (asynchronous on `stream`). */
int ngram_embed_clear_status(void* workspace, void* stream);

/* Self-test of the device-side bounded wait used by every pipeline barrier of the
 * tensor-core kernel: launches one warp that waits on a barrier nothing completes.
 * The wait must give up after limit_ns (<= 2 s), set NGRAM_STATUS_TIMEOUT in the
 * workspace status word and return; the context stays usable. */
int ngram_embed_selftest_wait_timeout(void* workspace, int64_t limit_ns, void* stream);

/* Static description of a return code. */
const char* ngram_embed_error_string(int code);

/* Which projection kernel a plan uses: 1 = tcgen05 tensor-core kernel, 0 = CUDA-core kernel. */
int ngram_embed_plan_uses_tensor_cores(const ngram_embed_plan* plan);

/* Choose the projection kernel of a plan (for testing one implementation against another):
 *   0 = automatic (tensor cores when the shape allows: bf16, D % 128 == 0, d % 64 == 0, N >= 2),
 *   1 = tensor cores, every gathered A row brought in by TMA (tile::gather4),
 *   2 = tensor cores, A rows split between TMA gather4 and 16-byte cp.async (default),
 *   3 = CUDA cores.
 * Returns NGRAM_ERR_UNSUPPORTED if the shape does not admit the chosen kernel. */
int ngram_embed_plan_set_variant(ngram_embed_plan* plan, int variant);

/* Variant 2: how many of the 128 rows of each gathered tile TMA brings in (0, 32, 64, 96
 * or 128; -1 = default: 128 in the pair form, 0 in the one-CTA form); cp.async brings in the
 * rest. A tuning knob: results do not change. */
int ngram_embed_plan_set_tma_rows(ngram_embed_plan* plan, int rows);

/* Tensor-core kernel form: 1 = pairs of CTAs on neighbouring SMs share each 256-token tile
 * (tcgen05 cta_group::2; each CTA loads half of the W tile; A rows by cp.async when tma_rows
 * is 0, else all by TMA gather4), 0 = one CTA per 128-token tile, -1 (default) = automatic:
 * the pair form, except where the one-CTA form's stream-K schedule applies (see
 * ngram_embed_plan_set_stream_k). A tuning knob: results agree within the stated tolerance
 * (the k-block order differs). */
int ngram_embed_plan_set_cta_pair(ngram_embed_plan* plan, int on);

/* How many SMs the plan's kernels use: 0 = all of the device's (default), else 2 ..
 * the device's count. Grids, stream-K shares and the workspace's partial tiles follow it
 * (ngram_embed_workspace_bytes shrinks with it), so other work can keep the remaining SMs.
 * Without a device any count >= 2 is accepted, which lets ngram_embed_plan_kernel_form
 * report the choice a device of that size would make. NGRAM_ERR_INVALID_ARG otherwise. */
int ngram_embed_plan_set_sm_count(ngram_embed_plan* plan, int sms);

/* CTA-pair form with 512-column tiles: each pair gathers a 256-row A block once per k-block
 * and issues two tcgen05 MMAs of N = 256 on it (half the gathered rows per FLOP of the
 * 256-column tiles); the accumulator fills all 512 TMEM columns and each half is drained and
 * freed separately. Applies when the tile width is 256 and D % 512 == 0, with A rows by TMA
 * gather4. 1 = on (with the stream-K schedule if ngram_embed_plan_set_stream_k(plan, 1)),
 * 0 = off, -1 (default) = automatic. A tuning knob: results agree within the stated
 * tolerance. NGRAM_ERR_INVALID_ARG for other values. */
int ngram_embed_plan_set_pair_wide(ngram_embed_plan* plan, int on);

/* The projection kernel a call of num_tokens tokens would run, given a workspace of
 * ngram_embed_workspace_bytes(plan, num_tokens): 0 = CUDA cores, 1 = one CTA per tile,
 * 2 = one CTA per SM with the stream-K schedule, 3 = CTA pairs, 4 = CTA pairs with
 * 512-column tiles, 5 = CTA pairs with the stream-K schedule, 9 = CTA pairs with 512-column
 * tiles and the stream-K schedule (these gather the A rows from the sub-tables inside the
 * projection); 6 = the call's sub-rows gathered into G first by a stand-alone gather kernel,
 * then CTA pairs reading A as dense TMA boxes of G, 7 = the same with the pairs' stream-K
 * schedule, 8 = the same with 512-column tiles (see ngram_embed_plan_set_dense_a); 10 = CTA
 * pairs over column ranges (see ngram_embed_plan_set_pair_columns), 11 = the same reading A
 * as dense TMA boxes of G; negative on bad arguments. */
int ngram_embed_plan_kernel_form(const ngram_embed_plan* plan, int64_t num_tokens);

/* ngram_embed_fwd_step in one launch (on request): where the step's projection runs the
 * one-CTA tensor-core form and S <= 8, two otherwise idle warps of every CTA of that
 * projection commit the previous step's ids and hash this step's (Eq. 2 of "Scaling
 * Embeddings Outperforms Scaling Experts in Language Models", section 2, over the N-gram
 * cache of section 4.2) for a share of the sequences, with the same code as the separate
 * commit + hash launch, and the gather warps start once every sequence is done. The launch is
 * cooperative (all CTAs resident, one per SM); the wait is bounded (TIMEOUT status). Outputs,
 * indices (in the workspace), ring and status bits are those of the two-launch step. It
 * counts sequences and CTAs in the workspace's status header (zero between calls;
 * ngram_embed_clear_status re-arms them after a TIMEOUT). 1 = on; 0 = the separate commit +
 * hash launch (default: measured on B200 at the 1280-token decode step, D = 4096, in graphs
 * of 200 steps: 64.4 us in one launch against 62.6 us in two; the hash's latency then sits
 * at the head of every CTA's main loop). NGRAM_ERR_INVALID_ARG for other values. */
int ngram_embed_plan_set_fused_step(ngram_embed_plan* plan, int on);

/* Form of the backward pass's two dense GEMMs (dG = c g W_stacked and dW = c g^T G, the
 * gradients of Eq. 3 of "Scaling Embeddings Outperforms Scaling Experts in Language Models",
 * section 2): 1 = CTA pairs (tcgen05.mma.cta_group::2, 256-row x 256-column tiles, 128 when
 * D % 256 != 0; each CTA of a pair loads its 128 rows of A and half of B per k-block;
 * default); 2 = CTA pairs with 256 x 512 tiles where D % 512 == 0 (two N = 256 accumulator
 * halves filling TMEM, drained half by half; measured on B200 at D = 2048, T = 32768: 0.58 ms
 * for the whole backward against 0.55 ms with 256-column tiles, the drain of the single
 * accumulator stalling the MMAs); 0 = one CTA per 128-row tile (0.62 ms). Pairs need a plan
 * SM budget of at least 2 (otherwise the one-CTA form runs). A tuning knob: results agree
 * within the stated tolerance (the fp32 atomic-add order differs). NGRAM_ERR_INVALID_ARG for
 * other values or a null plan. */
int ngram_embed_plan_set_backward_pair(ngram_embed_plan* plan, int on);

/* Streams of ngram_embed_bwd. 1 (default): the memory-bound kernels (the gather of G for dW,
 * the dE0 counting sort and sums) run on an auxiliary stream that the plan owns, forked from
 * the caller's stream with an event after everything queued there and joined back before the
 * call returns (the caller's stream waits for all of the call's work; dW's GEMM waits for G
 * only), so they overlap the dG GEMM. The first backward call that forks creates the stream
 * and three events on the plan's device (do it once outside CUDA-graph capture); calls on one
 * plan share them, so a plan's backward calls must be issued from one host thread at a time;
 * ngram_embed_plan_destroy releases them. 0: every kernel on the caller's stream, in order.
 * Results agree within the stated tolerance either way (the fp32 atomic-add order differs).
 * NGRAM_ERR_INVALID_ARG for other values or a null plan. */
int ngram_embed_plan_set_backward_streams(ngram_embed_plan* plan, int on);

/* CTA-pair form over column ranges (Eq. 3 of "Scaling Embeddings Outperforms Scaling Experts
 * in Language Models", section 2, partitioned by output columns): the pairs are spread evenly
 * over the 256-token row blocks and each pair computes the full sum over K for a contiguous
 * range of columns (a multiple of 64; two MMAs of N = half the range per k-step), so a call
 * whose 256 x 512 tiles are fewer than the pairs keeps every pair busy without stream-K's
 * partial sums. Ranges wider than 512 columns run as several passes over K. With the dense-A
 * form on (ngram_embed_plan_set_dense_a) it reads A as dense boxes of G. 1 = whenever the
 * plan's tile width is 256, the pair form is allowed and the token count is known on the
 * host; 0 = never (default: measured on B200 at a 1280-token decode step at D = 4096, 61 us
 * for the projection, 57 us reading G, against 55 us for the one-CTA form's stream-K; -1 is
 * accepted as 0). A tuning knob: results agree within the stated tolerance (the k-block order
 * differs). NGRAM_ERR_INVALID_ARG for other values. */
int ngram_embed_plan_set_pair_columns(ngram_embed_plan* plan, int mode);

/* Dense-A form of the tensor-core projection: the call's sub-rows are first copied into a
 * G buffer [num_tokens x D] (bf16) in the workspace by a gather kernel that keeps every
 * resident thread's loads in flight, then the CTA-pair kernel reads its A tiles as dense
 * 2-D TMA boxes of G instead of gathering rows itself; in ngram_embed_fwd_step the commit,
 * the hash and this gather are one launch. 1 = on (whenever the workspace holds G and the
 * plan allows the pair form with 256-column tiles), 0 = off (default: measured on B200 at a
 * 1280-token decode step, 78 us against 70 us for the fused forms, whose limit there is the
 * rate at which shared memory fills from L2, not the row gather). ngram_embed_workspace_bytes
 * includes G while it is on. The stream-K schedule applies to it where whole tiles would
 * leave a thin last wave of pairs, 512-column tiles where they fill their waves. A tuning
 * knob: results agree within the stated tolerance (the k-block order differs).
 * NGRAM_ERR_INVALID_ARG for other values. */
int ngram_embed_plan_set_dense_a(ngram_embed_plan* plan, int mode);

/* Tensor-core tile width in output columns: 256 (default when D % 256 == 0) or 128. */
int ngram_embed_plan_set_tile_n(ngram_embed_plan* plan, int tile_n);

/* Depth of the one-CTA tensor-core kernel's ring of gathered A stages (16 KB each); the rest
 * of its 224 KB of shared memory holds the ring of W tiles and the epilogue's output tile.
 * Tile width 256: 2, 4 or 6 (W ring 4, 3 or 2 deep); width 128: 6, 8 or 10 (W 6, 4 or 2).
 * Any other even depth up to 12 selects the default (4 at width 256, 8 at 128), as does 0.
 * The CTA-pair form keeps one ring of combined (A, W) stages. A tuning knob: results do not
 * change. */
int ngram_embed_plan_set_a_stages(ngram_embed_plan* plan, int stages);

/* Schedule of the tensor-core kernels: 0 = automatic, 1 = stream-K whenever possible (for
 * the pairs' 256-column tiles only when ngram_embed_plan_set_cta_pair(plan, 1) also fixes
 * the pair form and 512-column tiles are off), 2 = never. Stream-K gives every worker (a
 * CTA, or a CTA pair) an equal run of (tile, k-block) units; a tile split between workers is
 * summed in fp32, in worker order, by whichever finishes its piece last, so no worker waits
 * for another. Automatic: the one-CTA form with stream-K when its grid takes two or more
 * waves of one tile per CTA and the last wave leaves many SMs idle (a 1280-token decode step
 * at D = 4096). The pairs' 512-column tiles take it only when both are asked for
 * (ngram_embed_plan_set_pair_wide(plan, 1) too; measured slower at the decode step: a
 * piece's epilogue cannot overlap the next piece's MMAs with one 512-column accumulator).
 * It needs the workspace's partial tiles, at most 2048 one-CTA tiles (1024 pair tiles, 512
 * 512-column tiles) and at least one k-block per worker (half a tile per pair for the
 * 512-column tiles), and is not used when the token count is read on the device; otherwise
 * the kernel takes one tile per worker. A tuning knob: results agree within the stated
 * tolerance (the summation order differs). */
int ngram_embed_plan_set_stream_k(ngram_embed_plan* plan, int mode);

/* 1 = launch every kernel of the plan as a programmatic dependent launch: it may be
 * scheduled while the kernel before it on the stream finishes, and runs only its setup
 * (barriers, tensor-memory allocation) until that kernel has completed and its writes are
 * visible. 0 (default) = plain launches: measured on B200 inside CUDA graphs, the gap
 * between launches is already about 1 us, and early-scheduled grids slowed the decode
 * step's hash -> projection pair down. Results do not change. */
int ngram_embed_plan_set_pdl(ngram_embed_plan* plan, int on);

#ifdef __cplusplus
}
#endif
#endif /* NGRAM_EMBED_H */
