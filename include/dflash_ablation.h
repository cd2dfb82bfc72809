/*
 * dflash_ablation.h — the input-fusion drafter that KV injection is compared
 * against (DFlash-ja, gist.science technical summary: section 3, contribution 2,
 * and section 4, KV-injection ablation bullet: conditioning every draft layer
 * through its K/V cache is compared with feeding the context feature at the
 * drafter's input only).  The pages give no equations for it; the reading here:
 * each context row's feature is that row's input hidden state; the row passes
 * through every draft layer like a token (pre-norm, RoPE at the row's position,
 * attention causal over the context, O-projection, MLP), and each layer caches
 * the K/V of its own normed state instead of projecting the feature directly.
 * The context rows carry no token ids here, so no embedding is added.  Drafting
 * over a cache filled this way is dflash_draft_block, unchanged.
 */
#ifndef DFLASH_ABLATION_H_
#define DFLASH_ABLATION_H_

#include "dflash.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Append `rows` context rows per request through the draft layers (bf16
 * handles).  ctx: device bf16 [batch * rows, H], row b * rows + j is request b's
 * row at position len[b] + j (16-byte aligned); in practice the output of
 * dflash_fuse_context.  For every layer l, with x the rows' hidden states
 * (initially ctx):
 *   h = R(RMSNorm(x) g_in_l); K_l[p] = R(RoPE_p(h Wk_l^T)), V_l[p] = R(h Wv_l^T)
 *   written to cache position p = len[b] + j; for l < n_layers - 1 also
 *   q = R(RoPE_p(h Wq_l^T)); o = R(softmax over cache rows [0, p]) V (causal,
 *   bf16 P as in the draft step); x = R(x + o Wo_l^T); then the SwiGLU MLP as in
 *   the draft step.  The last layer's attention and MLP change no cached value
 *   and are not run.
 * Then len[b] += row_count[b] (row_count: device int32[batch], each in
 * [0, rows], or NULL for `rows`); committed is not changed.  Rows past
 * row_count[b] are computed and written past the new len as scratch.
 * 1 <= rows <= max_gamma.  Appending rows in calls of any sizes gives the same
 * cache as one call up to fp32 summation order (each row sees only rows at or
 * before its position).
 * Errors: DFLASH_INVALID_ARG, DFLASH_UNSUPPORTED (fp32 handles); device:
 * DFLASH_CAPACITY when len[b] + rows > capacity (the request is skipped),
 * DFLASH_INVALID_ARG when a row_count is outside [0, rows]. */
int dflash_ingest_fused_input(dflash_handle* h, dflash_cache* c, const void* ctx, int rows,
                              const int32_t* row_count, dflash_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_ABLATION_H_ */
