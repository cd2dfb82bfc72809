/*
 * dflash.h — C ABI of a B200 (sm_100a) implementation of the DFlash draft step.
 *
 * DFlash ("DFlash: Block Diffusion for Flash Speculative Decoding", technical
 * summaries on gist.science, ja/nl pages) drafts a block of tokens for
 * speculative decoding with a small block-diffusion model that is conditioned
 * on the target model's hidden features.  The four calls below are its draft
 * step:
 *
 *   dflash_fuse_context  §2.2 (inference design), context-feature bullet:
 *                        hidden states of a fixed, uniformly spaced set of
 *                        target layers are concatenated and projected into one
 *                        compact context feature (here followed by RMSNorm).
 *   dflash_inject_kv     §2.2, KV-injection bullet: the feature goes through
 *                        every draft layer's own key/value projection and is
 *                        kept in the draft model's KV cache, so every layer is
 *                        conditioned on it.
 *   dflash_draft_block   §2.2, parallel block diffusion bullet: one forward pass
 *                        over a block of gamma positions (the clean anchor token
 *                        of the target, §2.3 random-anchor bullet, followed by
 *                        gamma-1 mask tokens) predicts gamma-1 tokens; the
 *                        embedding and LM head are the target's (§2.3
 *                        architecture bullet).
 *   dflash_accept        §5 (claims), lossless: only the longest prefix of
 *                        drafts equal to the target's own greedy tokens is kept.
 *
 * The summaries give no layer equations.  This library implements the plain
 * reading of a pre-norm decoder layer, and the CPU test oracle implements the
 * same reading independently.  With R() = round-to-nearest-even to the storage
 * type (bf16; identity for fp32 storage) and all accumulation in fp32:
 *
 *   fuse:    ctx_r = R( RMSNorm( R( concat_i h_i[r] . W_fc^T ) ) * g_fc )
 *   inject:  for layer l, row r at position p = len + r:
 *            K_l[p] = R( RoPE_p( ctx_r . Wk_l^T ) ),  V_l[p] = R( ctx_r . Wv_l^T )
 *   draft:   x_0 = E[anchor], x_j = E[mask_id] (j = 1..gamma-1), position len + j;
 *            per layer: h = R(RMSNorm(x) g_in); q,k = R(RoPE(h Wq^T)), R(RoPE(h Wk^T));
 *            v = R(h Wv^T); o = R(softmax(q K^T / sqrt(d)) V) over all cached
 *            rows [0, len) and all gamma block rows (no mask; query head hq
 *            reads kv head hq / (n_q_heads / n_kv_heads); P is rounded to bf16
 *            before it weights V: with t_i = q.k_i log2(e) / sqrt(d),
 *            P_i = R(2^(t_i - b)) for an integer b, divided by the sum of the
 *            unrounded 2^(t_i - b); every integer b below the row maximum gives
 *            the same o, as the values differ by one exact power of two);
 *            x = R(x + o Wo^T); h2 = R(RMSNorm(x) g_post);
 *            m = R(silu(h2 Wg^T) * (h2 Wu^T)); x = R(x + m Wd^T).
 *            Then hf_j = R(RMSNorm(x_j) g_final) for j = 1..gamma-1, logits =
 *            hf_j . lm_head^T (fp32), draft_j = argmax (ties to the lowest id).
 *   accept:  a = largest k <= gamma-1 with drafts[i] == target[i] for all i < k;
 *            next_anchor = target[a]; committed += a + 1; len = min(len, committed).
 *   RMSNorm(x) = x / sqrt(mean(x^2) + eps).  RoPE rotates pairs (i, i + d/2) by
 *   p * theta^(-2i/d) (cos/sin tabulated in fp64, stored as fp32).
 *
 * Conventions for every entry point
 *   - Pointers to tensors are DEVICE pointers unless stated otherwise; the
 *     caller owns all memory.  Matrices are row-major [out, in] (PyTorch
 *     nn.Linear layout).  Storage type is bf16 or fp32 per dflash_config.dtype.
 *   - Calls are asynchronous on the given CUDA stream (NULL = legacy default
 *     stream) and never synchronise the host, except dflash_create,
 *     dflash_cache_init's host checks and dflash_cache_status.
 *   - A handle or cache must be used from one stream at a time.
 *   - Return value: DFLASH_OK (0) or a negative dflash_status.  Host-detected
 *     errors return before anything is enqueued.  Errors that only the device
 *     can see (capacity, state, token range) are recorded in the cache's sticky
 *     first-error-wins status word; the affected requests are skipped (their
 *     cache rows and lengths are left unchanged, their drafts / accept length
 *     / next anchor are written as -1) and the other requests proceed.  Read
 *     and clear the word with dflash_cache_status.
 */
#ifndef DFLASH_H_
#define DFLASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dflash_stream; /* a cudaStream_t */

#define DFLASH_MAX_LAYERS 16

enum dflash_dtype { DFLASH_F32 = 0, DFLASH_BF16 = 1 };

enum dflash_status {
    DFLASH_OK = 0,
    DFLASH_INVALID_ARG = -1,   /* null pointer, size out of range, mismatched handle/cache */
    DFLASH_UNSUPPORTED = -2,   /* shape the kernels do not implement (see dflash_create) */
    DFLASH_CUDA = -3,          /* a CUDA runtime or driver call failed */
    DFLASH_WORKSPACE = -4,     /* workspace or cache memory smaller than required */
    DFLASH_CAPACITY = -5,      /* device: len + rows > capacity (inject) or len + gamma > capacity (draft) */
    DFLASH_STATE = -6,         /* device: len != committed when drafting */
    DFLASH_TOKEN_RANGE = -7,   /* device: anchor or target token outside [0, vocab) */
    DFLASH_TIMEOUT = -8        /* device: a bounded pipeline wait ran out (library fault) */
};

typedef struct {
    int hidden;          /* H: draft hidden size */
    int n_layers;        /* L: draft layers (<= DFLASH_MAX_LAYERS) */
    int n_q_heads;       /* query heads */
    int n_kv_heads;      /* key/value heads; n_q_heads % n_kv_heads == 0 */
    int head_dim;        /* d: 64 or 128 */
    int intermediate;    /* SwiGLU intermediate size */
    int vocab;           /* V: shared vocabulary */
    int n_sel;           /* selected target layers (<= 8) */
    int target_hidden;   /* H_t: target hidden size */
    int mask_id;         /* token id of the mask token, in [0, vocab) */
    int max_gamma;       /* largest block size a call may use (1..32) */
    int dtype;           /* DFLASH_BF16 or DFLASH_F32 */
    int max_batch;       /* most requests per cache / call */
    int max_rows;        /* most rows per dflash_fuse_context / dflash_inject_kv call */
    int max_position;    /* positions (cache capacity) stay below this */
    int reserved;
    double rope_theta;   /* RoPE base */
    double rms_eps;      /* RMSNorm epsilon */
} dflash_config;

/* Weight table.  The handle BORROWS these device pointers: they must stay valid
 * and unchanged for the handle's lifetime.  lm_head may equal embed (tied). */
typedef struct {
    const void* w_fc;     /* [H, n_sel*H_t]: columns ordered layer-major, ascending layer */
    const void* g_fc;     /* [H] */
    const void* embed;    /* [V, H] */
    const void* lm_head;  /* [V, H] */
    const void* g_final;  /* [H] */
    const void* g_in[DFLASH_MAX_LAYERS];    /* [H] */
    const void* wq[DFLASH_MAX_LAYERS];      /* [n_q_heads*d, H] */
    const void* wk[DFLASH_MAX_LAYERS];      /* [n_kv_heads*d, H] */
    const void* wv[DFLASH_MAX_LAYERS];      /* [n_kv_heads*d, H] */
    const void* wo[DFLASH_MAX_LAYERS];      /* [H, n_q_heads*d] */
    const void* g_post[DFLASH_MAX_LAYERS];  /* [H] */
    const void* w_gate[DFLASH_MAX_LAYERS];  /* [I, H] */
    const void* w_up[DFLASH_MAX_LAYERS];    /* [I, H] */
    const void* w_down[DFLASH_MAX_LAYERS];  /* [H, I] */
} dflash_weights;

typedef struct dflash_handle dflash_handle;
typedef struct dflash_cache dflash_cache;

/* Bytes of device workspace a handle for cfg needs.  No CUDA call. */
int dflash_workspace_bytes(const dflash_config* cfg, size_t* bytes);

/* Create a handle.  Validates cfg (DFLASH_INVALID_ARG / DFLASH_UNSUPPORTED),
 * checks ws_bytes (DFLASH_WORKSPACE), builds the RoPE table and tensor maps,
 * and initialises the workspace (synchronously, on the legacy stream).
 * workspace: device memory, 1024-byte aligned, borrowed for the handle's life.
 * bf16 needs: H, I, H_t multiples of 64; head_dim 64 or 128;
 * (n_q_heads/n_kv_heads) * max_gamma <= 128.  Requires an sm_100 device. */
int dflash_create(const dflash_config* cfg, const dflash_weights* w, void* workspace,
                  size_t ws_bytes, dflash_handle** out);
void dflash_destroy(dflash_handle* h);

/* Cache memory for `batch` requests of `capacity` positions each.  Layout of
 * that memory (all offsets from its base, which must be 1024-byte aligned):
 *   [0, 256)            int32 status word (sticky, first error wins) + padding
 *   [256, ...)          int32 len[batch], padded to a multiple of 256 bytes
 *   next                int32 committed[batch], padded to a multiple of 256 bytes
 *   next (1024-aligned) K/V slab, storage type, [batch][L][2 (K, V)][n_kv_heads][capacity][d]
 * dflash_cache_info reports these offsets. */
int dflash_cache_bytes(const dflash_handle* h, int batch, int capacity, size_t* bytes);

/* Bind caller memory as a cache and zero its status word, len and committed
 * (enqueued on stream).  The cache BORROWS mem.  capacity <= max_position. */
int dflash_cache_init(const dflash_handle* h, void* mem, size_t bytes, int batch, int capacity,
                      dflash_cache** out, dflash_stream stream);
void dflash_cache_release(dflash_cache* c);

typedef struct {
    int batch, capacity;
    int32_t* status;      /* device */
    int32_t* len;         /* device [batch] */
    int32_t* committed;   /* device [batch] */
    void* slab;           /* device */
    int64_t stride_kv;    /* elements between consecutive kv heads (= capacity*d) */
    int64_t stride_kind;  /* elements between K and V of one layer */
    int64_t stride_layer; /* elements between layers */
    int64_t stride_request; /* elements between requests */
} dflash_cache_info;
int dflash_cache_get_info(const dflash_cache* c, dflash_cache_info* info);

/* Set len[b] = committed[b] = lens[b] for every request (lens: device
 * int32[batch]).  For callers that filled the slab themselves. */
int dflash_cache_set_len(dflash_cache* c, const int32_t* lens, dflash_stream stream);

/* Synchronise `stream`, then return and clear the cache's sticky status word
 * (DFLASH_OK if no device error was recorded), or DFLASH_TIMEOUT if any
 * kernel of the handle reported a timeout. */
int dflash_cache_status(dflash_handle* h, dflash_cache* c, dflash_stream stream);

/* a1. ctx_out[r] = fused context feature of row r, r < total_rows.
 * hiddens: HOST array of n_sel DEVICE pointers, hiddens[i] -> [total_rows, H_t]
 * with row stride row_stride elements (>= H_t; row_stride*elem a multiple of 16 bytes).
 * ctx_out: device [total_rows, H] in the storage type.  total_rows <= max_rows;
 * total_rows == 0 is a no-op. */
int dflash_fuse_context(dflash_handle* h, const void* const* hiddens, int64_t row_stride,
                        int total_rows, void* ctx_out, dflash_stream stream);

/* a2. Append context rows to the cache.  ctx: device [total_rows, H].
 * Request b owns rows ctx[row_start[b] .. row_start[b] + row_count[b]) (device
 * int32 arrays of length batch; ranges inside [0, total_rows)); row r of request
 * b is written at position len[b] + r, then len[b] += row_count[b].  committed
 * is not changed.  row_count may be computed on the device (e.g. accept_len+1).
 * Device errors: CAPACITY when len[b] + row_count[b] > capacity. */
int dflash_inject_kv(dflash_handle* h, dflash_cache* c, const void* ctx, const int32_t* row_start,
                     const int32_t* row_count, int total_rows, dflash_stream stream);

/* a1 + a2 in one call: the verify-side pre-step.  DFlash-ja §2.2, context-feature
 * bullet (the verified rows' hidden states of the selected target layers are
 * concatenated and projected) and KV-injection bullet (the feature goes into every
 * draft layer's K/V cache), taken straight from the target's verification output.
 * Computes exactly dflash_fuse_context followed by dflash_inject_kv of the same
 * rows (the same rounding points: ctx = R(RMSNorm(R(y)) * g_fc) is what the K/V
 * projections read), but with small batches of rows (at most 16 per call) the
 * RMSNorm is folded into the injection GEMM: the W_fc GEMM also writes its rows'
 * partial sums of squares, and the injection GEMM normalises its token tiles in
 * shared memory, so no separate normalisation kernel runs and the feature is not
 * re-read from memory.  Larger calls (prefill) run the two calls one after the other.
 * hiddens, row_stride: as dflash_fuse_context; row_start, row_count (device),
 * total_rows: as dflash_inject_kv (rows index the hidden-state rows).
 * ctx_out: NULL, or device [total_rows, H] storage type receiving the context
 * feature as dflash_fuse_context would write it.  Errors: as the two calls. */
int dflash_fuse_inject(dflash_handle* h, dflash_cache* c, const void* const* hiddens, int64_t row_stride,
                       const int32_t* row_start, const int32_t* row_count, int total_rows, void* ctx_out,
                       dflash_stream stream);

/* a3..a7. Draft one block per request.  anchor: device int32[batch].
 * 1 <= gamma <= max_gamma.  drafts: device int32[batch, gamma-1].
 * logits_opt: NULL or device fp32[batch, gamma-1, V]; margin_opt: NULL or device
 * fp32[batch, gamma-1] (top-1 minus top-2 logit).  The block's own K/V are
 * written to cache positions [len, len+gamma) as scratch; len is unchanged.
 * Device errors: STATE (len != committed), CAPACITY (len+gamma > capacity),
 * TOKEN_RANGE (anchor). */
int dflash_draft_block(dflash_handle* h, dflash_cache* c, const int32_t* anchor, int gamma,
                       int32_t* drafts, float* logits_opt, float* margin_opt, dflash_stream stream);

/* a8. Accept the longest matching prefix.  drafts: device int32[batch, gamma-1];
 * target: device int32[batch, gamma] (the target's greedy token after each of the
 * block's positions); accept_len, next_anchor: device int32[batch].  Works in both
 * cycle orders: after injecting the gamma verified rows (rolls len back to the
 * new committed length) or before injecting accept_len+1 rows (len unchanged).
 * Device errors: TOKEN_RANGE (target). */
int dflash_accept(dflash_handle* h, dflash_cache* c, const int32_t* drafts, const int32_t* target,
                  int gamma, int32_t* accept_len, int32_t* next_anchor, dflash_stream stream);

const char* dflash_status_string(int status);

/* Number of kernel launches the calls above enqueued since the handle was
 * created (host-side counter). */
int64_t dflash_launch_count(const dflash_handle* h);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_H_ */
