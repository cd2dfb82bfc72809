/*
 * dflash_diag.h — diagnostic entry points of libdflash.
 *
 * These are not part of the DFlash draft step.  They expose single kernels of
 * the library (for kernel-level tests), the host-side work partition of the
 * tensor-core GEMM (for CPU tests), and a stand-in for the target model's
 * verification pass that benchmarks and chained tests use to drive the
 * draft/accept cycle with planned acceptance lengths.
 */
#ifndef DFLASH_DIAG_H_
#define DFLASH_DIAG_H_

#include "dflash.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Scratch bytes (device) that dflash_diag_gemm_bf16 needs for these sizes. */
int dflash_diag_gemm_scratch_bytes(int M, int N, int K, size_t* bytes);

/* Y[m, n] = sum_k X[m, k] * W[n, k] with the sm_100a tcgen05 GEMM (fp32
 * accumulation, fp32 output).  X: device bf16 [M, K], W: device bf16 [N, K],
 * Y: device fp32 [M, N]; K % 8 == 0, 1 <= M <= 4096.  scratch: device memory of
 * dflash_diag_gemm_scratch_bytes, 256-byte aligned; it must be zero on the first
 * call (the kernel leaves it zeroed again).  grid: persistent CTAs to use (0 = one
 * per SM); a small grid forces the split-K fix-up path. */
int dflash_diag_gemm_bf16(const void* X, const void* W, float* Y, int M, int N, int K,
                          void* scratch, size_t scratch_bytes, int grid, dflash_stream stream);

/* Same, recording a per-CTA timeline into trace (device int64[grid * 8]):
 * globaltimer stamps (ns) at entry, producer past the dependency wait, first
 * stage landed, last MMA issued, accumulators drained, epilogue done, exit;
 * then the CTA's clock64 span. */
int dflash_diag_gemm_bf16_traced(const void* X, const void* W, float* Y, int M, int N, int K, void* scratch,
                                 size_t scratch_bytes, int grid, int64_t* trace, dflash_stream stream);

/* Size of the static device array that dflash_diag_gemm_bf16_noalloc keeps its
 * scratch in (6 MiB per device, reserved when the library's module loads). */
#define DFLASH_NOALLOC_SCRATCH_BYTES (6u << 20)

/* dflash_diag_gemm_bf16 without caller scratch and without any device
 * allocation.  This is a library utility with no counterpart in the DFlash
 * method; it serves callers that cannot allocate device memory (a host that
 * owns all memory through its own pool, a serving loop that forbids allocator
 * calls).  The split-tile partials and tile counters live in a static device
 * array of DFLASH_NOALLOC_SCRATCH_BYTES; nothing is allocated, by this call or
 * any library it uses.
 *
 * Same operands, layout and result as dflash_diag_gemm_bf16: X device bf16
 * [M, K], W device bf16 [N, K], Y device fp32 [M, N] (all owned by the caller),
 * K % 8 == 0, 1 <= M <= 4096; grid = persistent CTAs (0 = one per SM).
 *
 * Size limit: the scratch needed is a 256-byte status word, the tile counters
 * (4 bytes per 128 x nt output tile, nt = 16/32/64/128/256 from M, rounded up
 * to 256 bytes) and 2 * CTAs * nt * 512 bytes of partials.  At the largest grid
 * (160 CTAs), M <= 32 fits for N up to 33.5 million and M <= 16 for N up to 117
 * million; a larger M fits only with a smaller grid.  A call whose need exceeds
 * the array returns DFLASH_WORKSPACE and launches nothing.  Other returns: DFLASH_INVALID_ARG (bad sizes, pointers or
 * alignment), DFLASH_CUDA (the symbol lookup, the counter clear or the launch
 * failed).
 *
 * The first call on each device looks up the array's address with that device
 * current (this may load the module); make that first call before any stream
 * capture begins.  The address is kept together with the CUDA context it was
 * looked up in and looked up again when the current context differs (after a
 * device reset).  Each call clears the status word and the counters on `stream`
 * before the launch; a wait that runs out is reported by
 * dflash_diag_gemm_bf16_noalloc_status, not by this call's return value.
 * One array serves every caller on a device: calls that may overlap on the same
 * device (other streams, other host threads) race on it and must be serialised
 * by the caller. */
int dflash_diag_gemm_bf16_noalloc(const void* X, const void* W, float* Y, int M, int N, int K, int grid,
                                  dflash_stream stream);

/* Status of the last dflash_diag_gemm_bf16_noalloc on this device: synchronises
 * `stream` (the stream of that call) and writes to *status (host) DFLASH_OK, or
 * DFLASH_TIMEOUT when a bounded wait inside the kernel ran out, in which case Y
 * is incomplete.  The word lives in the same static array and is cleared by the
 * next dflash_diag_gemm_bf16_noalloc.  Allocates nothing.  Returns DFLASH_OK,
 * DFLASH_INVALID_ARG (status NULL) or DFLASH_CUDA. */
int dflash_diag_gemm_bf16_noalloc_status(int32_t* status, dflash_stream stream);

/* Work partition of the persistent split-K GEMM (host only, no CUDA call).
 * `units` k-blocks in total, `kb` k-blocks per output tile, `ctas` CTAs.  For
 * output tile `tile`: first_cta = first CTA contributing to it, n_contrib = the
 * number of CTAs contributing.  Returns DFLASH_INVALID_ARG on bad sizes. */
int dflash_diag_partition(int64_t units, int kb, int ctas, int64_t tile, int* first_cta, int* n_contrib);

/* Stand-in for the target's greedy verification of one block per request:
 * target[b, i] = drafts[b, i] for i < a_plan[b]; target[b, a_plan[b]] differs from
 * drafts[b, a_plan[b]] when a_plan[b] < gamma-1; other entries are rand_tokens[b, i].
 * All pointers are device int32: drafts [batch, gamma-1], a_plan [batch] (values
 * in [0, gamma-1]), rand_tokens and target [batch, gamma].  A draft of -1 (skipped
 * request) is treated like any other token. */
int dflash_diag_synth_target(const int32_t* drafts, const int32_t* a_plan, const int32_t* rand_tokens,
                             int batch, int gamma, int vocab, int32_t* target, dflash_stream stream);

/* Diagnostic timer.  While enabled, the handle brackets each launch group of
 * the four calls (a GEMM, an attention split + combine pair, a norm, ...) with
 * two CUDA events recorded on the launch stream, up to max_launches groups.
 * Not for use under CUDA-graph capture.  dflash_diag_timing_read synchronises
 * `stream`, writes up to max_entries (kind, milliseconds) pairs in launch order,
 * and restarts the log.  dflash_diag_timed_name names a kind. */
int dflash_diag_timing_enable(dflash_handle* h, int max_launches);
int dflash_diag_timing_read(dflash_handle* h, dflash_stream stream, int* kinds, float* ms, int max_entries,
                            int* n_entries);
int dflash_diag_timing_disable(dflash_handle* h);
const char* dflash_diag_timed_name(int kind);

/* The block-attention kernel alone (bf16 handles): for every request b and
 * layer `layer`, q (device bf16 [batch*gamma, n_q_heads*head_dim], rows b*gamma+j)
 * attends over cache rows [0, len[b] + gamma) of that layer (the caller writes
 * the block's own K/V rows at [len, len+gamma) and keeps len + gamma <= capacity);
 * out: device bf16, same layout as q.  q must be 16-byte aligned (DFLASH_INVALID_ARG
 * otherwise).  Synchronises the stream. */
int dflash_diag_attention(dflash_handle* h, dflash_cache* c, const void* q, void* out, int layer, int gamma,
                          dflash_stream stream);

/* Same, recording per-CTA timestamps into trace (device int64[batch * n_kv_heads
 * * splits * 8]: entry, past the dependency wait, Q in tensor memory, first tile landed,
 * key loop done, partial ready, past the cluster barrier, merge done) and the
 * split count used into *splits_out (host int, may be NULL). */
int dflash_diag_attention_traced(dflash_handle* h, dflash_cache* c, const void* q, void* out, int layer, int gamma,
                                 int64_t* trace, int* splits_out, dflash_stream stream);

/* Step trace: per-block %globaltimer stamps (ns) of every kernel the handle's
 * bf16 calls launch while it is set, for attributing a captured step's time to
 * its kernels.  buf: device int64[words], zero-filled by the caller; each traced
 * launch takes the next blocks * words_per_block words (a launch that does not fit
 * is not traced).  Block b of a launch stamps word b * words_per_block + wait_idx
 * once past its dependency wait and word b * words_per_block + exit_idx when it is
 * done; blocks a launch does not use stay zero.  The pointers are fixed at launch
 * time, so a step captured in a CUDA graph with tracing set writes the same words
 * on every replay.  dflash_diag_step_trace(h, NULL, 0) stops tracing; setting a
 * buffer restarts the record list.  Launches outside the handle's calls (the
 * verification stand-in) are not traced. */
int dflash_diag_step_trace(dflash_handle* h, int64_t* buf, int64_t words);

/* The launches traced since dflash_diag_step_trace was set, in launch order:
 * recs (host int32[max_records][5]) = (kind, blocks, words_per_block, wait_idx,
 * exit_idx), offsets (host int64[max_records]) = first word of the launch in buf;
 * kind names come from dflash_diag_timed_name.  *n_records = the number traced
 * (may exceed max_records; only max_records are written). */
int dflash_diag_step_trace_records(const dflash_handle* h, int32_t* recs, int64_t* offsets, int max_records,
                                   int* n_records);

/* Capture of the draft step's intermediate states, for call-local parity checks
 * (each stage compared with the oracle run on the GPU's own input to it).  While
 * set, every dflash_draft_block on the handle also copies (on its stream):
 *   x_layers: device [(n_layers+1)][batch*gamma][hidden], storage type: the
 *             residual stream after the embedding (slot 0) and after each layer l
 *             (slot l+1), rows b*gamma + j;
 *   hf:       device [batch*(gamma-1)][hidden], storage type: the final-norm rows
 *             that the LM head reads, rows b*(gamma-1) + j-1.
 * Either may be NULL; dflash_diag_draft_capture(h, NULL, NULL) stops capturing.
 * The buffers are borrowed and must hold the largest batch*gamma drafted while set.
 * Not for use under CUDA-graph capture of a timed step (the copies are extra work). */
int dflash_diag_draft_capture(dflash_handle* h, void* x_layers, void* hf);

/* Capture of every layer's intermediate states (bf16 handles), for per-stage
 * parity checks.  While set, every dflash_draft_block also writes, for each layer
 * l, slot l (rows b*gamma + j, storage type) of:
 *   h_in:  [n_layers][batch*gamma][hidden]       the normalised layer input R(RMSNorm(x) g_in)
 *   q:     [n_layers][batch*gamma][n_q_heads*d]  the queries after RoPE
 *   o:     [n_layers][batch*gamma][n_q_heads*d]  the attention output
 *   x_mid: [n_layers][batch*gamma][hidden]       the residual stream after the O-projection
 *   h2:    [n_layers][batch*gamma][hidden]       the normalised MLP input R(RMSNorm(x_mid) g_post)
 *   act:   [n_layers][batch*gamma][intermediate] the SwiGLU output
 * The block's own K/V of each layer stay in the cache rows [len, len + gamma).
 * With the norms folded into the GEMMs, h_in and h2 are written by the GEMMs'
 * normalising warp from the tiles the MMAs read.  Any pointer may be NULL;
 * dflash_diag_draft_capture_stages(h, NULL, ...) stops.  Not for timed steps. */
int dflash_diag_draft_capture_stages(dflash_handle* h, void* h_in, void* q, void* o, void* x_mid, void* h2,
                                     void* act);

/* Self-test of the device-side bounded wait used by the pipelined kernels: a
 * one-warp kernel waits on a shared-memory barrier that nothing arrives at.  The
 * wait gives up after its limit (about 2 s), records DFLASH_TIMEOUT in the
 * handle's status word and the kernel returns, leaving the context usable.
 * out: device int32, set to 0 when the wait ran out (1 would mean it completed).
 * dflash_cache_status then reports DFLASH_TIMEOUT once. */
int dflash_diag_wait_selftest(dflash_handle* h, int32_t* out, dflash_stream stream);

/* Launch mode of every kernel of the library (process-wide, default 1):
 * 1 = programmatic dependent launch (a kernel may be scheduled while the
 * previous kernel of the stream drains; each kernel waits for its predecessor's
 * results in-kernel, and the GEMM streams its first weight tiles before that
 * wait), 0 = plain stream-ordered launches. */
int dflash_diag_set_launch_mode(int programmatic);

/* Weight tiles (128 x 64 bf16 each) that every CTA of the tensor-core GEMM
 * prefetches into L2, beyond the tiles it loads into its shared-memory ring,
 * before waiting for the previous kernel of the stream (process-wide, 0..256;
 * applies to launches enqueued afterwards).  The weights never depend on the
 * previous kernel, so this keeps HBM streaming across kernel boundaries. */
int dflash_diag_set_gemm_prefetch(int tiles);
/* The current setting of dflash_diag_set_gemm_prefetch. */
int dflash_diag_gemm_prefetch(void);

/* Shared-memory ring stages each CTA of the tensor-core GEMM fills with weight
 * tiles before waiting for the previous kernel (process-wide, 0..64; 0 = the whole
 * ring; default 6).  A shallower pre-wait burst leaves the previous kernel's
 * finishing memory round trips less contended. */
int dflash_diag_set_gemm_pre_stages(int stages);

/* Largest thread-block cluster the tensor-core GEMM may use for 16-token tiles
 * (process-wide, 0..4; default 0 = never, as measured faster on B200 for the
 * drafter shapes here; 1 = never).  In cluster mode each cluster
 * owns whole output tiles and its CTAs split their k-blocks; a split tile's
 * partial accumulators travel to the CTA that finishes it through distributed
 * shared memory instead of global memory.  The launcher takes the cluster size
 * (2..max) whose partition is shorter than the whole-grid partition plus its
 * global-memory fix-up, if any. */
int dflash_diag_set_gemm_max_cluster(int max_cluster);

/* How many clusters of `cluster_size` CTAs (2..8) of the cluster-mode GEMM kernel
 * can be resident at once on the current device (a cluster must fit one GPC);
 * 0 if none or out of range.  The launcher's choice of cluster size uses this. */
int dflash_diag_gemm_max_active_clusters(int cluster_size);

/* How the tensor-core GEMM finishes an output tile whose k-blocks are split
 * over several CTAs (process-wide; applies to launches enqueued afterwards).
 * 0 (the default): the CTA holding the tile's first k-blocks finishes it; it
 * waits (bounded) for the other contributors' published partials and adds them
 * in contributor order.  1: every contributor publishes its partial and counts
 * it with an atomic, and the one that counts last finishes.  Both add the
 * partials in the same order, so the results are bit-identical. */
int dflash_diag_set_split_finisher(int last_arriver);

/* The last `ctas` CTAs (0..64) of the draft step's other whole-grid GEMMs take
 * `units` (0..64) fewer k-block units each (process-wide; default 24, 3; 0, 0 for
 * equal shares).  They land on the SMs the previous kernel's last CTAs held and
 * start after them; the shift also moves every tile's split points, which is the
 * larger effect and depends on the shapes. */
int dflash_diag_set_gemm_tail(int ctas, int units);

/* k-block units (0..64, default 9) fewer for each O-projection CTA that lands on
 * an SM the attention still holds (process-wide; applies to calls enqueued
 * afterwards).  Those CTAs start when the attention ends, without the weight
 * stages the others loaded during it; 0 gives every CTA an equal share. */
int dflash_diag_set_o_late_deficit(int units);

/* Whether the draft step folds each RMSNorm into the GEMM that consumes its
 * output (process-wide, default 1; applies to calls enqueued afterwards).  When
 * on and the token tile is at most 16 wide (batch 1 at gamma 16), the producer
 * of the residual stream (the embedding, the O-projection and the
 * down-projection) also writes per-tile partial sums of squares of its rows, and
 * the QKV and gate/up GEMMs read x itself and normalise each token tile in shared
 * memory.  The final norm before the LM head stays a kernel of its own (the LM
 * head streams its weights at the HBM roofline, where the folded form measured
 * slower) unless on = 2, which folds it too.  0 = one RMSNorm kernel before each
 * of them. */
int dflash_diag_set_norm_fold(int on);

/* Placement of the O-projection GEMM of each draft layer (process-wide, default 1):
 * 1 = on the SMs the preceding attention kernel does not occupy (when it occupies
 * at most three quarters of them), with those CTAs prefetching their whole weight
 * range into L2 while the attention runs; 0 = on every SM like the other GEMMs. */
int dflash_diag_set_o_beside_attention(int on);

/* Work partition of dflash_inject_kv's GEMM (process-wide, applies to calls
 * enqueued afterwards).  1 (default): whole output tiles in one launch (no tile is
 * split across CTAs; the fast choice for many rows, e.g. prefill); 0: split-K with
 * one launch per slab of token-tile rows.  Either way the fp32 summation order of
 * every K/V element does not depend on the number of rows injected, so chunked
 * injection writes the same bits as one call.  dflash_fuse_inject always uses the
 * split-K slabs (its few rows per call stream the weights on every SM). */
int dflash_diag_set_inject_partition(int whole_tiles);

/* "sm_100a" for this build. */
const char* dflash_diag_arch(void);

#ifdef __cplusplus
}
#endif
#endif /* DFLASH_DIAG_H_ */
