/*
 * gqa_prefill.h -- causal prefill attention (S_q = T > 1) in libgqadecode.so,
 * the compute-bound counterpart of the decode entry points of gqa_decode.h.
 *
 * What it computes: for every sequence b of a packed batch and every query
 * position i < S_b, query head h attends the keys 0..i of the same sequence,
 *     s_ij = scale * <q_i, k_j>,  O_i = sum_{j<=i} e^{s_ij - m_i} v_j
 *                                     / sum_{j<=i} e^{s_ij - m_i},
 * with kv head g = floor(h / (h_q / h_kv)) as in decode.  This is the
 * "Optimized SDPA, flash-attention style" item of the tt-metal "[Llama2]
 * Perf burndown" page's "Prefill 2k" list; the scaling-book "All About
 * Transformer Inference" page explains why it is compute-bound (its
 * arithmetic intensity grows with T) where decode is bandwidth-bound.
 *
 * ---------------------------------------------------------------- layouts
 *   q        [total_rows][h_q][d_head]   bf16, packed by sequence: sequence b
 *   k, v     [total_rows][h_kv][d_head]  occupies rows S_0 + ... + S_{b-1}
 *                                        onwards (S_b rows), q, k, v alike
 *   seqlens  int32 [B]                   S_b (device memory)
 *   out      fp32 [total_rows][h_q][d_head]
 * total_rows = sum_b S_b (host-known); max_seqlen >= every S_b (host-known:
 * it sizes the grid, so no device-to-host copy is needed).
 *
 * Conventions are those of gqa_decode.h: device pointers owned by the caller,
 * q, k, v and out 16-byte aligned, asynchronous on `stream`, host-side
 * argument checks (nonzero gqa_status and nothing launched on error).
 * Supported: d_head == 128, dtype == GQA_BF16 (GQA_F32 and other head sizes
 * return GQA_ERR_UNSUPPORTED), h_q % h_kv == 0, finite scale, B, h_q and
 * ceil(max_seqlen / 128) at most 65535, total_rows < 2^31.  B == 0 or
 * total_rows == 0 is a no-op.
 *
 * Device-side errors go to the status word (gqa_decode_get_status): a
 * negative S_b (treated as 0), an S_b above max_seqlen (rows past the first
 * ceil(max_seqlen/128)*128 are not written), lengths that sum past
 * total_rows (clipped to the rows that exist), a bounded wait that ran out.
 * Rows of out that belong to no sequence are not written.
 *
 * Numerics: fp32 logits and softmax; P enters the P.V product as bf16, and a
 * block of 128 query rows x 64 keys also adds the rounding remainder of P
 * (a second bf16 part, so P is exact to ~2^-17 there) whenever some row of
 * the block holds more than a third of its running softmax mass in those
 * keys -- every row's first keys, and any tile that carries a row's dominant
 * keys; fp32 accumulation and output.  Tested against the fp64 oracle with
 * |e| <= 2e-3 + 1e-2 |ref| on bf16 inputs.
 */
#ifndef GQA_PREFILL_H
#define GQA_PREFILL_H

#include "gqa_decode.h"

#ifdef __cplusplus
extern "C" {
#endif

GQA_API int gqa_prefill_attn(const void *q, const void *k, const void *v, const int32_t *seqlens,
                             float *out, int B, int total_rows, int max_seqlen, int h_q, int h_kv,
                             int d_head, float scale, int dtype, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GQA_PREFILL_H */
