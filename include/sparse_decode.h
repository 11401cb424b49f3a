/*
 * sparse_decode.h -- C ABI of the head-wise sparse decode attention library
 * (libsparsedecode.so, sm_100a).
 *
 * One decode step of one attention layer, for a batch of sequences whose
 * keys and values live in a paged bf16 cache:
 *
 *   retrieval heads  score every cached token in an r = 16 dimensional index
 *                    space built from pre-RoPE keys, keep a per-(sequence,
 *                    head) token set by dynamic top-p or fixed top-k, and run
 *                    exact softmax attention over the kept rows only;
 *   local heads      attend to a few sink tokens plus a recent window.
 *
 * Sources (gist.science summary pages):
 *   RTPurbo page  "Full attention strikes back: moving full attention to sparse
 *                 attention within hundreds of training steps",
 *                 gist.science/ar/paper/2605.16928, Methodology 1 (retrieval vs
 *                 local heads; local heads use a sliding window with attention
 *                 sinks, retrieval heads keep the full KV and select sparsely at
 *                 decode), 2 (r << d, r = 16, projection of pre-RoPE q and k),
 *                 3 (dynamic top-p: accumulate low-dimensional attention mass to
 *                 the cumulative threshold p, e.g. 0.9; fixed top-k as the
 *                 alternative), 5 (histogram-based, sort-free threshold and a
 *                 bandwidth-optimised sparse decode kernel).
 *   ICS page      "Inference-time context sparsity: illusion or opportunity?",
 *                 gist.science/ar/paper/2605.24168, 2 (Oracle Top-K), 3a (50x
 *                 sparsity = ~2% of tokens), 3c (decode traffic O(N d) -> O(k d)).
 *   AoH page      "Autonomy-of-Heads: Data-Free Sparse Attention from Frozen
 *                 Query-Key Geometry", gist.science/ar/paper/2608.06849,
 *                 Methodology 4 (streaming heads keep sinks + recent window;
 *                 head roles pooled per GQA group).
 *
 * Conventions for every call:
 *   - Pointers named "device" must point to memory of the device that was
 *     current when sparse_decode_init ran.  The caller owns all of them; the
 *     library never frees caller memory.
 *   - bf16 tensors are raw IEEE bfloat16 bit patterns (uint16), row-major and
 *     densely packed in the order of their stated shapes.  The caches, k_pre,
 *     q and q_pre must start on a 16-byte boundary (they are read with 16-byte
 *     vector and asynchronous copies); a misaligned one is rejected with
 *     SD_ERR_INVALID_ARG.
 *   - Hot calls (index_keys, local_append, select, attend and their joined
 *     and split forms) allocate nothing, never synchronise the host, and
 *     enqueue their work on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are
 *     detected on the host before any launch and nothing is enqueued.
 *   - Data-dependent errors found on the device (a page id outside
 *     [0, num_pages), a sequence length above max_pages_per_seq * page_size,
 *     a selected position out of range) never fault: the kernel skips the bad
 *     access, sets a bit in a device error word and carries on; results are
 *     then unspecified.  sparse_decode_error_word reads and clears the word.
 *   - The context is not thread-safe: one host thread at a time per context.
 *     Calls on the same context and stream are ordered; calls that share a
 *     workspace must not overlap on the device.
 *
 * Shapes: B = batch, Hq = query heads, Hkv = KV heads, G = Hq / Hkv (GQA
 * group), d = head_dim (64 or 128), r = index_dim (16), P = page_size (16),
 * H_ret = number of retrieval heads, MAXP = max_pages_per_seq,
 * L = MAXP * P (longest supported context).
 *
 * Caches (caller-owned, device):
 *   k_cache, v_cache  bf16 [num_pages, Hkv, P, d]; token j of sequence b, KV
 *                     head g lives at [page_table[b][j / P], g, j % P, :].
 *   index_cache       bf16 [num_pages, Hkv, P, r]; same addressing.
 *   page_table        int32 [B, MAXP]; entries at and past ceil(N_b / P) are
 *                     never read.
 *   seq_lens          int32 [B]; N_b, 0 <= N_b <= L.  The current token is
 *                     position N_b - 1 and is already in the caches.
 */
#ifndef SPARSE_DECODE_H
#define SPARSE_DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SD_API __attribute__((visibility("default")))
#else
#define SD_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sd_ctx sd_ctx;          /* opaque, host-side */
typedef void *sd_stream;               /* a cudaStream_t */

typedef enum {
  SD_OK = 0,
  SD_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size or an inconsistent shape */
  SD_ERR_UNSUPPORTED = 2,   /* a valid request the library does not implement */
  SD_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the size query */
  SD_ERR_CUDA = 4,          /* a CUDA runtime call or a kernel launch failed */
  SD_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up */
  SD_ERR_DEVICE_DATA = 6,   /* a device-side check rejected input data */
  SD_ERR_HOST_MEMORY = 7    /* a host allocation failed inside the call (no C++ exception ever
                               leaves a call); work the call enqueued before it stays enqueued */
} sd_status;

/* Selection mode of retrieval heads (RTPurbo page, Methodology 3). */
enum { SD_TOP_P = 0, SD_TOP_K = 1 };

/* Bits of the device error word. */
enum {
  SD_EBIT_PAGE = 1u,       /* page id outside [0, num_pages) */
  SD_EBIT_SEQLEN = 2u,     /* N_b < 0 or N_b > L */
  SD_EBIT_SEL = 4u,        /* sel_idx entry outside [0, N_b), not ascending, or sel_count > sel_stride */
  SD_EBIT_SLOT = 8u,       /* index_keys slot outside [0, num_pages * P) */
  SD_EBIT_TIMEOUT = 16u    /* a bounded device-side wait gave up */
};

/*
 * Layer configuration, copied by sparse_decode_init.
 *
 *   num_q_heads, num_kv_heads  Hq and Hkv; Hkv divides Hq; G = Hq/Hkv <= 16.
 *   head_dim                   d, 64 or 128.
 *   index_dim                  r, must be 16 (RTPurbo page, Methodology 2).
 *   page_size                  P, must be 16.
 *   num_pages                  pages in the caller's cache pool (bounds checks).
 *   head_is_retrieval          host int32 [Hq]: 1 = retrieval head, 0 = local
 *                              head (RTPurbo page, Methodology 1).  Copied.
 *   window, num_sinks          local heads attend to positions
 *                              [0, num_sinks) U [N_b - window, N_b), clamped to
 *                              [0, N_b) (RTPurbo Methodology 1; AoH Methodology 4).
 *   mode                       SD_TOP_P or SD_TOP_K.
 *   top_p                      in (0, 1]; keeps the smallest set of highest index
 *                              scores whose softmax mass reaches top_p; every
 *                              token tied with the threshold score is kept;
 *                              top_p = 1 keeps every token.
 *   top_k, top_k_frac          top-k budget k_b = top_k if top_k > 0, else
 *                              max(1, floor(top_k_frac * N_b)) (frac in (0, 1]),
 *                              capped at N_b; ties go to the lower position.
 *   attn_scale                 logit scale of the attention; <= 0 selects 1/sqrt(d).
 *   index_scale                c in s_j = c * <P^T q, k~_j>; <= 0 selects
 *                              sqrt(d) / r, which makes the index score an
 *                              unbiased estimate of q.k/sqrt(d) for a projection
 *                              with i.i.d. N(0, 1/d) entries.
 *   max_batch                  largest B of any later call.
 *   max_pages_per_seq          MAXP, the page-table row length; MAXP * P (the
 *                              longest context) must not exceed 2^25 tokens.
 */
typedef struct {
  int num_q_heads;
  int num_kv_heads;
  int head_dim;
  int index_dim;
  int page_size;
  int num_pages;
  const int32_t *head_is_retrieval;
  int window;
  int num_sinks;
  int mode;
  float top_p;
  int top_k;
  float top_k_frac;
  float attn_scale;
  float index_scale;
  int max_batch;
  int max_pages_per_seq;
} sd_config;

/*
 * sparse_decode_init -- validate `cfg`, copy it and the index projection, and
 * create a context bound to the current CUDA device.
 *
 *   proj  device bf16 [Hkv, d, r]: one r x d projection per KV head, applied
 *         to pre-RoPE keys of that head and to pre-RoPE queries of its GQA
 *         group (RTPurbo page, Methodology 2).  Copied; the caller may free
 *         it after the call.
 *   out   receives the context; NULL on failure.
 *
 * Allocates the device copy of the projection, a head table and a 4-byte
 * device error word.  Returns SD_ERR_INVALID_ARG or SD_ERR_UNSUPPORTED for a
 * bad or unsupported configuration (among them a pool whose
 * num_pages * Hkv * P cache rows do not fit 32-bit row numbers),
 * SD_ERR_CUDA if a device allocation fails, SD_ERR_HOST_MEMORY if a host one
 * does.
 */
SD_API sd_status sparse_decode_init(const sd_config *cfg, const void *proj, sd_ctx **out);

/*
 * sparse_decode_workspace_size -- bytes of device workspace that select and
 * attend need for a batch of `batch` sequences (batch <= max_batch).  The
 * same workspace serves both calls.  `bytes` receives the size.
 */
SD_API sd_status sparse_decode_workspace_size(const sd_ctx *ctx, int batch, size_t *bytes);

/*
 * sparse_decode_index_keys -- write index entries for `num_tokens` keys
 * (RTPurbo page, Methodology 2):
 *
 *   index_cache[slot_t / P, g, slot_t % P, :] = bf16_rne( P_g^T k_pre[t, g, :] )
 *
 * with the dot products accumulated in float64 and rounded once to bf16,
 * round to nearest even.
 *
 *   k_pre        device bf16 [num_tokens, Hkv, d], pre-RoPE keys.
 *   slots        device int32 [num_tokens], page * P + offset of each token.
 *   index_cache  device bf16 [num_pages, Hkv, P, r], written in place.
 *
 * num_tokens == 0 is a no-op.  A slot outside [0, num_pages * P) sets
 * SD_EBIT_SLOT and is skipped.
 */
SD_API sd_status sparse_decode_index_keys(sd_ctx *ctx, const void *k_pre, const int32_t *slots,
                                   int num_tokens, void *index_cache, sd_stream stream);

/*
 * sparse_decode_select -- per (sequence b, retrieval head h) token sets
 * (RTPurbo page, Methodology 2-3 and 5; ICS page, 2):
 *
 *   q~_h = P_g^T q_pre[b, h]                    (float64, then float32)
 *   s_j  = index_scale * <q~_h, k~_j>           j < N_b, float32
 *   top-p: S = { j : s_j >= tau }, tau the largest score whose
 *          upper set {s >= tau} holds softmax(s) mass >= top_p
 *   top-k: the k_b highest s_j, ties to the lower position
 *
 *   q_pre       device bf16 [B, Hq, d], pre-RoPE queries (only retrieval
 *               heads are read).
 *   index_cache device bf16, filled by sparse_decode_index_keys.
 *   sel_idx     device int32 [B, H_ret, sel_stride]: row (b, i) receives the
 *               positions of the i-th retrieval head (retrieval heads in
 *               ascending q-head order), ascending.
 *   sel_count   device int32 [B, H_ret]: set sizes.
 *   sel_stride  row capacity: >= L for SD_TOP_P; >= the largest k_b for
 *               SD_TOP_K (min(top_k, L), or max(1, floor(top_k_frac * L))).
 *   workspace   device memory of at least sparse_decode_workspace_size bytes.
 *
 * N_b == 0 yields an empty set.  Returns SD_ERR_WORKSPACE if ws_bytes is too
 * small.  A configuration without retrieval heads is a no-op.
 */
SD_API sd_status sparse_decode_select(sd_ctx *ctx, const void *q_pre, const void *index_cache,
                               const int32_t *page_table, const int32_t *seq_lens, int batch,
                               int32_t *sel_idx, int32_t *sel_count, int sel_stride,
                               void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * sparse_decode_select_exact -- per (sequence b, retrieval head h) token sets
 * chosen by the exact attention logits instead of the index (ICS page, 2: the
 * "Oracle Top-K" reference selector, applied here with top-k or top-p alike):
 *
 *   s_j = attn_scale * <q[b, h], k_j>           j < N_b, float32 accumulation
 *   top-p / top-k over s_j exactly as for sparse_decode_select
 *
 *   q           device bf16 [B, Hq, d], post-RoPE queries (only retrieval
 *               heads are read).
 *   k_cache     device bf16 [num_pages, Hkv, P, d]; page_table, seq_lens as
 *               described above.
 *   sel_idx, sel_count, sel_stride, workspace, ws_bytes   as for
 *               sparse_decode_select (the same workspace size).
 *
 * Every cached key of every retrieval KV group is read once per call
 * (2 d bytes per token, against 2 r for the index): a ground truth for the
 * index selection, not a substitute for it.  Errors as for
 * sparse_decode_select.
 */
SD_API sd_status sparse_decode_select_exact(sd_ctx *ctx, const void *q, const void *k_cache,
                                     const int32_t *page_table, const int32_t *seq_lens, int batch,
                                     int32_t *sel_idx, int32_t *sel_count, int sel_stride,
                                     void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * sparse_decode_attend -- attention output of every head (ICS page, 3c;
 * RTPurbo Methodology 1):
 *
 *   out[b, h] = sum_{j in S} e^{l_j - max l} v_j / sum_{j in S} e^{l_j - max l},
 *   l_j = attn_scale * <q[b, h], k_j>
 *
 * with S the selected set of a retrieval head (from sel_idx / sel_count, as
 * written by sparse_decode_select or by the caller) and the sinks + window of a
 * local head.  One softmax over the whole set; fp32 accumulation; an empty
 * set gives zeros.  Each KV row of a GQA group is read once per call even
 * when several heads of the group selected it.
 *
 *   q          device bf16 [B, Hq, d], post-RoPE queries.
 *   k_cache, v_cache, page_table, seq_lens   as described above.
 *   sel_idx, sel_count, sel_stride           as for select (ascending rows);
 *              may be NULL when there are no retrieval heads.
 *   out        device float32 [B, Hq, d].
 *   workspace  device memory of at least sparse_decode_workspace_size bytes.
 */
SD_API sd_status sparse_decode_attend(sd_ctx *ctx, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *page_table,
                               const int32_t *seq_lens, int batch, const int32_t *sel_idx,
                               const int32_t *sel_count, int sel_stride, float *out,
                               void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * sparse_decode_select_attend -- sparse_decode_select followed by
 * sparse_decode_attend on the same sets, in one call: the decode step of the
 * layer (RTPurbo page, Methodology 1-3 and 5; ICS page, 3c).  The arguments
 * are the union of theirs (q_pre and index_cache for the selection, q and the
 * K/V caches for the attention; sel_idx / sel_count receive the sets as
 * sparse_decode_select writes them); the results are identical to the two
 * calls in a row.
 *
 * Joined, the last selection pass writes each (sequence, retrieval KV group)'s
 * union of selected rows straight into the workspace instead of attend
 * rebuilding it from sel_idx (when a group has at most four retrieval heads and
 * their context bitmaps fit one CTA's shared memory; otherwise the two calls
 * run as they are).  Errors as for the two calls.
 */
SD_API sd_status sparse_decode_select_attend(sd_ctx *ctx, const void *q_pre, const void *q,
                                      const void *index_cache, const void *k_cache, const void *v_cache,
                                      const int32_t *page_table, const int32_t *seq_lens, int batch,
                                      int32_t *sel_idx, int32_t *sel_count, int sel_stride, float *out,
                                      void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * Split cache layout (RTPurbo page, Methodology 1: local heads only ever see
 * the sinks and the recent window; AoH page, Methodology 4: the KV memory of
 * streaming heads is the saving).  The paged caches then hold only the
 * retrieval KV groups, and each local KV group keeps a compacted cache of
 * num_sinks + window rows per sequence instead of the whole context:
 *
 *   k_ret, v_ret      bf16 [num_pages, R, P, d], R = number of retrieval KV
 *                     groups (KV heads with at least one retrieval query head,
 *                     in ascending KV-head order); token j of sequence b,
 *                     i-th retrieval group, at [page_table[b][j / P], i, j % P, :].
 *   local_k, local_v  bf16 [max_batch, Lg, num_sinks + window, d], Lg = number
 *                     of local KV groups (KV heads with at least one local
 *                     query head, ascending); position j of sequence b,
 *                     i-th local group, at [b, i, slot(j), :] with
 *                     slot(j) = j for j < num_sinks, else
 *                     num_sinks + j % window.  Row b is sequence b of a call's
 *                     batch, like row b of page_table.
 *
 * A KV group with both kinds of query heads is kept in both.  The index cache
 * keeps its layout.  Every position in [0, num_sinks) U [N_b - window, N_b)
 * has its own slot, so after the tokens of a sequence are appended in
 * position order the compacted rows hold exactly the rows its local heads
 * attend to at length N_b; the outputs equal those of the full layout.
 */

/* R and Lg of the split layout (0 on a NULL context). */
SD_API int sparse_decode_num_retrieval_groups(const sd_ctx *ctx);
SD_API int sparse_decode_num_local_groups(const sd_ctx *ctx);

/*
 * sparse_decode_local_append -- copy the keys and values of `num_tokens` new
 * tokens into the compacted local caches:
 *
 *   local_k[s_t, i, slot(p_t), :] = k_new[t, g_i, :]   (and likewise v)
 *
 * for every local KV group i (KV head g_i), s_t = seq_ids[t], p_t = positions[t].
 *
 *   k_new, v_new      device bf16 [num_tokens, Hkv, d], post-RoPE keys and the
 *                     values of the new tokens (the rows of every KV head; only
 *                     local groups are read).
 *   seq_ids           device int32 [num_tokens], in [0, max_batch).
 *   positions         device int32 [num_tokens], in [0, L).
 *   local_k, local_v  device bf16, the split layout's compacted caches.
 *
 * A token whose sequence or position is out of range sets SD_EBIT_SLOT and is
 * skipped.  Positions >= num_sinks with window == 0 are kept nowhere (no
 * error).  Tokens of one call that land on the same slot of the same
 * sequence (more than `window` positions past the sinks of one sequence in a
 * call) race: which one stays is unspecified; append at most the last
 * `window` such positions of a sequence per call.  num_tokens == 0, or no
 * local group, is a no-op.
 */
SD_API sd_status sparse_decode_local_append(sd_ctx *ctx, const void *k_new, const void *v_new,
                                     const int32_t *seq_ids, const int32_t *positions, int num_tokens,
                                     void *local_k, void *local_v, sd_stream stream);

/*
 * sparse_decode_attend_split -- sparse_decode_attend on the split layout:
 * retrieval heads read k_ret / v_ret, local heads their compacted caches.
 * Same arguments otherwise; the outputs equal those of sparse_decode_attend
 * on the full caches holding the same data.  k_ret / v_ret may be NULL
 * without retrieval heads, local_k / local_v without local heads (or with
 * num_sinks + window == 0).  Returns SD_ERR_UNSUPPORTED when
 * batch * Lg * (num_sinks + window) reaches 2^32 rows.
 */
SD_API sd_status sparse_decode_attend_split(sd_ctx *ctx, const void *q, const void *k_ret, const void *v_ret,
                                     const void *local_k, const void *local_v, const int32_t *page_table,
                                     const int32_t *seq_lens, int batch, const int32_t *sel_idx,
                                     const int32_t *sel_count, int sel_stride, float *out,
                                     void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * sparse_decode_select_attend_split -- sparse_decode_select_attend on the split
 * layout (the index cache keeps its layout).  Arguments, results and errors as
 * for sparse_decode_select_attend and sparse_decode_attend_split.
 */
SD_API sd_status sparse_decode_select_attend_split(sd_ctx *ctx, const void *q_pre, const void *q,
                                            const void *index_cache, const void *k_ret, const void *v_ret,
                                            const void *local_k, const void *local_v,
                                            const int32_t *page_table, const int32_t *seq_lens, int batch,
                                            int32_t *sel_idx, int32_t *sel_count, int sel_stride, float *out,
                                            void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * sparse_decode_prefill -- attention outputs of the queries of a prefill
 * chunk (RTPurbo page, Methodology 1: retrieval heads keep their full KV
 * through prefill, local heads use the sliding window with sinks; AoH page,
 * Methodology 4: streaming heads keep sinks + a recent window, with chunked
 * prefill).  Sequence b's chunk is its last T_b = q_starts[b+1] - q_starts[b]
 * positions, N_b - T_b .. N_b - 1, whose keys and values are already in the
 * caches (written by the caller, like every earlier position).  The query at
 * position i of head h attends to
 *
 *   retrieval head  keys 0 .. i                              (dense causal)
 *   local head      keys [0, num_sinks) U [i - window + 1, i], within [0, i]
 *
 * with one softmax over those keys (scale attn_scale, float32 accumulation;
 * an empty set gives zeros).
 *
 *   q          device bf16 [total_q, Hq, d], post-RoPE queries packed by
 *              sequence: sequence b's chunk at rows q_starts[b] ..
 *              q_starts[b+1] - 1.
 *   q_starts   device int32 [batch + 1], nondecreasing, q_starts[0] = 0,
 *              q_starts[batch] = total_q, T_b <= N_b.
 *   k_cache, v_cache, page_table, seq_lens   as described above (N_b =
 *              seq_lens[b] includes the chunk).
 *   out        device float32 [total_q, Hq, d], 16-byte aligned.
 *
 * No workspace.  A sequence whose q_starts or length is inconsistent sets
 * SD_EBIT_SEQLEN and is skipped; page ids as for attend.
 */
SD_API sd_status sparse_decode_prefill(sd_ctx *ctx, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts,
                                int batch, int total_q, float *out, sd_stream stream);

/*
 * sparse_decode_attend_noalloc -- sparse_decode_attend without a workspace
 * argument: the call uses a fixed scratch area compiled into the library
 * (64 MiB per device) and allocates nothing.  An addition of this library;
 * the pages describe no such call.
 *
 * For callers that cannot hand over device memory on the decode path: an
 * engine whose device memory is all planned before it starts serving, where
 * an allocation in the middle of a step could synchronise the device or fail
 * under memory pressure, or a host program without a device allocator of its
 * own.
 *
 * Arguments, layouts and results are those of sparse_decode_attend.
 *   - Returns SD_ERR_WORKSPACE, with the sizes in sparse_decode_last_error,
 *     when this batch needs more than the built-in scratch (the amount
 *     sparse_decode_workspace_size reports for attend grows with the batch,
 *     the retrieval groups and max_pages_per_seq); nothing is launched then.
 *   - Nothing in the scratch has to start at zero: the call's own kernels
 *     clear the counters they use, in stream order, before reading them.
 *   - The scratch is one area per device, shared by every context and stream
 *     of the process: two of these calls on the same device that are not
 *     ordered on one stream (other streams, threads or contexts) race and may
 *     give wrong outputs.  Order them, or use sparse_decode_attend with
 *     separate workspaces.
 *   - Every call looks up the scratch address of the current device with
 *     cudaGetSymbolAddress (a cheap lookup; nothing is cached, so a device
 *     reset between calls leaves no stale address).  The first call on a
 *     device may load the library's device code there: make that first call
 *     outside any stream capture.
 */
SD_API sd_status sparse_decode_attend_noalloc(sd_ctx *ctx, const void *q, const void *k_cache,
                                      const void *v_cache, const int32_t *page_table,
                                      const int32_t *seq_lens, int batch, const int32_t *sel_idx,
                                      const int32_t *sel_count, int sel_stride, float *out,
                                      sd_stream stream);

/*
 * sparse_decode_error_word -- wait for `stream`, copy the device error word
 * into *word (may be NULL) and clear it.  Returns SD_OK when the word was 0,
 * SD_ERR_TIMEOUT when SD_EBIT_TIMEOUT was set, SD_ERR_DEVICE_DATA otherwise.
 * This call synchronises the stream.
 */
SD_API sd_status sparse_decode_error_word(sd_ctx *ctx, sd_stream stream, uint32_t *word);

/*
 * sparse_decode_testing_stall_prefill -- testing only, off by default.  While
 * on != 0, every CTA of the d = 128 prefill kernel first waits on an mbarrier
 * that nothing arrives at: a device-side wait that cannot end.  Its bound (2 s
 * of the global timer) runs out, the CTA's other roles stop at their next wait,
 * its MMAs and copies are drained, its outputs are written as zeros and the
 * error word gets SD_EBIT_TIMEOUT; the context stays usable.  The tests use it
 * to check that the bounded waits end and are reported.  Process-wide; set it
 * back to 0 before production calls.
 */
SD_API void sparse_decode_testing_stall_prefill(int on);

/* Number of retrieval heads (rows per sequence in sel_idx / sel_count). */
SD_API int sparse_decode_num_retrieval_heads(const sd_ctx *ctx);

/* Message describing the last failure on this context ("" if none). */
SD_API const char *sparse_decode_last_error(const sd_ctx *ctx);

/* Static description of a status code. */
SD_API const char *sparse_decode_status_string(sd_status status);

/* Release the context and its device allocations.  NULL is a no-op. */
SD_API void sparse_decode_destroy(sd_ctx *ctx);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_DECODE_H */
