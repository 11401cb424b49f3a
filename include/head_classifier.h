/*
 * head_classifier.h -- C ABI of the data-free head classifier in
 * libsparsedecode.so: which attention heads are retrieval heads, from the
 * frozen query and key projections alone.  Its output is the
 * head_is_retrieval table of sparse_decode_init.
 *
 * Source: AoH page "Autonomy-of-Heads: Data-Free Sparse Attention from Frozen
 * Query-Key Geometry", gist.science/ar/paper/2608.06849, Methodology:
 *   1  head h's kernel attention operator M_h = W_K^T W_Q (d_model x d_model);
 *   2  its effective rank ER(h) = exp(-sum_k s_k log s_k), s_k the nonzero
 *      singular values of M_h divided by their sum; low ER = concentrated
 *      spectrum = retrieval head, high ER = streaming (local) head;
 *   3  the nonzero singular values follow from d_head x d_head matrices
 *      built from W_Q W_Q^T and W_K W_K^T;
 *   4  heads ranked by ER, the lowest become retrieval heads; under GQA the
 *      head scores are mean-pooled to the group.
 *
 * Weights: W_Q^h is the d_head x d_model block of rows h*d_head ..
 * (h+1)*d_head - 1 of the query projection [Hq*d_head, d_model] (q = W x),
 * W_K^g likewise of the key projection [Hkv*d_head, d_model]; query head h
 * pairs with KV head h / (Hq / Hkv).
 */
#ifndef HEAD_CLASSIFIER_H
#define HEAD_CLASSIFIER_H

#include "sparse_decode.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * sparse_decode_head_er_workspace_size -- device workspace bytes of
 * sparse_decode_head_effective_rank for these sizes (float64 Gram matrices:
 * num_layers * (Hq + Hkv) * head_dim^2 * 8 bytes).
 */
SD_API sd_status sparse_decode_head_er_workspace_size(int num_layers, int num_q_heads, int num_kv_heads,
                                               int head_dim, size_t *bytes);

/*
 * sparse_decode_head_effective_rank -- ER(h) of every query head of
 * `num_layers` layers (Methodology 1-3).
 *
 *   w_q        device bf16 [num_layers, Hq * head_dim, d_model], row-major.
 *   w_k        device bf16 [num_layers, Hkv * head_dim, d_model].
 *   eff_rank   device float64 [num_layers, Hq], written.
 *   workspace  device memory of sparse_decode_head_er_workspace_size bytes.
 *
 * head_dim must be 64 or 128, d_model a positive multiple of 32, Hkv a
 * divisor of Hq; w_q and w_k 16-byte aligned.  All arithmetic is float64:
 * Gram matrices of the bf16 blocks, their Cholesky factors L (a pivot at or
 * below head_dim * eps * the largest diagonal entry zeroes its column), and
 * the singular values of L_k^T L_q by one-sided Jacobi rotations.  A
 * singular value counts as nonzero above head_dim * eps * the largest; a head
 * without one gets ER 1 (the empty sum); a head whose rotations have not
 * converged after 60 sweeps gets NaN.  num_layers == 0 is a no-op.  Returns
 * SD_ERR_INVALID_ARG or SD_ERR_UNSUPPORTED for bad sizes or pointers,
 * SD_ERR_WORKSPACE for a short workspace, SD_ERR_CUDA if a launch fails.
 * Enqueued on `stream`; never synchronises the host.
 */
SD_API sd_status sparse_decode_head_effective_rank(const void *w_q, const void *w_k, int num_layers, int d_model,
                                            int num_q_heads, int num_kv_heads, int head_dim, double *eff_rank,
                                            void *workspace, size_t ws_bytes, sd_stream stream);

/*
 * sparse_decode_classify_heads -- Methodology 4 on the host: mean-pool the
 * ER of each GQA group's query heads (summed in head order, then divided by
 * the group size), rank the groups by pooled ER (equal values: the lower KV
 * head first), and mark every query head of the `num_retrieval_groups`
 * lowest as retrieval (1), the others 0.
 *
 *   eff_rank           host float64 [Hq] (one layer).
 *   head_is_retrieval  host int32 [Hq], written.
 *
 * 0 <= num_retrieval_groups <= Hkv.  A NaN ER ranks after every number.
 */
SD_API sd_status sparse_decode_classify_heads(const double *eff_rank, int num_q_heads, int num_kv_heads,
                                       int num_retrieval_groups, int32_t *head_is_retrieval);

#ifdef __cplusplus
}
#endif

#endif /* HEAD_CLASSIFIER_H */
