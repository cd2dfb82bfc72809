// Persistent split-K tensor-core GEMM of libdflash: parameters, the work
// partition (shared by host and device), and the launcher's interface.
//
// Every projection of the draft step is Y[m, n] = sum_k X[m, k] W[n, k] with
// the weights W streamed from HBM once and the tokens X few (16 rows at batch
// 1).  The kernel computes it "swap-AB": a 128-row weight tile is the tcgen05 A
// operand (M = 128), NT tokens are the B operand (N = NT), the fp32 tile lives
// in TMEM.  Work units are k-blocks of 64 along K of every output tile; the
// grid's CTAs take equal contiguous ranges of units (a range may start or end
// inside a tile), so all SMs stream the same number of weight bytes whatever
// the shape.  A tile split across CTAs is finished by its first contributor
// (the CTA holding its k-block 0, for which the tile is the last segment): it
// waits, bounded, for the others' published fp32 partials and adds them in
// contributor order, so the result does not depend on arrival order (optionally
// the last contributor to arrive finishes instead, adding in the same order).
// Only a tile's first contributor ever waits, and only for CTAs that publish
// before waiting on anything, so the waits form no cycle.
#pragma once
#include "common.cuh"

namespace df {

enum EpiKind : int {
    EPI_F32 = 0,     // out fp32[m, n] = acc
    EPI_BF16 = 1,    // out bf16[m, n] = R(acc)
    EPI_RESID = 2,   // out bf16[m, n] = R(out + acc)            (O-proj, down-proj)
    EPI_QKV = 3,     // q = R(RoPE(acc)) -> q buffer; k = R(RoPE(acc)), v = R(acc) -> cache scratch
    EPI_SWIGLU = 4,  // out bf16[m, f] = R(silu(gate) * up)     (A tile = 64 gate rows + 64 up rows)
    EPI_INJECT = 5,  // K = R(RoPE(acc)), V = R(acc) -> cache rows of the owning request
    EPI_LMHEAD = 6,  // per 128-vocab tile and token: top-1 (value, id) and top-2 value; optional fp32 logits
};

constexpr int kMaxAMats = 10;   // weight matrices stacked in one A operand
constexpr int kMaxBMaps = 8;    // activation tensor maps concatenated along K

struct GemmAMat {
    int rows;    // rows of this weight matrix
    int tile0;   // first n-tile of this matrix
    int ntiles;  // n-tiles of this matrix
    int feat0;   // unused by the kernel; global feature offset for callers
};

struct GemmParams {
    CUtensorMap ta[kMaxAMats];   // weight maps, box {64, 128} (SwiGLU: {64, 64})
    CUtensorMap tb[kMaxBMaps];   // activation maps, box {64, NT}
    CUtensorMap tx;              // EPI_RESID, NT >= 64: the residual rows out[M][ldo], box {128, 32}, no
                                 //    swizzle (set by the launcher; has_tx says whether it is valid)
    int has_tx;
    GemmAMat amat[kMaxAMats];
    int n_amat;
    int swiglu;                  // A = rows [64t, 64t+64) of ta[0] then of ta[1]
    int kb_per_b;                // k-blocks served by one activation map
    int M, K, KB;                // tokens, reduction length, k-blocks per tile
    int n_tiles, m_tiles;
    long long units;             // n_tiles * m_tiles * KB
    int ctas;
    int whole_tiles;             // 1: CTAs take whole output tiles (no split-K): every output is one
                                 //    in-order accumulation over all of K, whatever M and the grid
    int l2_prefetch;             // weight tiles past the shared-memory ring prefetched into L2 before the wait
    int pre_stages;              // ring stages filled with weights before the wait (0: the whole ring)
    int late_from, late_deficit; // whole-grid partition: CTAs [late_from, ctas) start late (their SMs
                                 //    are held by the previous kernel) and take late_deficit fewer
                                 //    k-block units each (0: equal shares)
    int grouped;                 // 1: CTAs in groups of m_tiles, one per token tile, splitting the
                                 //    (weight tile, k-block) units between groups (set by the launcher)
    int cluster;                 // >= 2: CTAs in thread-block clusters of this size, each cluster owning
                                 //    whole tiles, split tiles reduced through distributed shared
                                 //    memory (set by the launcher for 16-token tiles when it pays)
    int last_arriver;            // split tiles: 1 = finished by whichever contributor counts in last;
                                 //    0 = by the contributor holding the tile's first k-blocks, which
                                 //    waits for the others' partials and stores none of its own
    float* partial;              // [2 * ctas][NT][128] fp32 split-tile partials
    int* counters;               // [n_tiles * m_tiles], zero between launches
    int* status;                 // handle status word (DFLASH_TIMEOUT)
    int epi;
    void* out;                   // EPI_F32 / BF16 / RESID / SWIGLU output, EPI_QKV q buffer
    int ldo;                     // its row stride in elements
    // EPI_QKV / EPI_INJECT
    int d, gamma, cap, layer, batch;
    const int* len;
    const int* req_ok;
    const float2* rope;          // [max_position][d/2] (cos, sin)
    __nv_bfloat16* slab;
    long long s_req, s_layer, s_kind, s_kv;
    const int* row_start;
    const int* row_count;
    int row0;                    // EPI_INJECT: global index of this launch's first token row
    // EPI_LMHEAD
    int vocab;
    float* logits;               // [M, vocab] or null (with lm_gamma: [M / lm_gamma * (lm_gamma - 1), vocab])
    float4* records;             // [M][n_tiles]: (top1, id bits, top2, 0)
    int lm_gamma;                // > 0: token rows are whole blocks of lm_gamma; logits skip each block's row 0
    // RMSNorm folded into the GEMM that consumes the normalised rows: the B operand
    // is the residual stream x, and every B stage is rewritten in shared memory as
    // R(x * inv_rms(row) * gain[k]) before the MMA reads it.  inv_rms comes from
    // per-tile partial sums of squares written by the producer of x.
    const float* ssq_in;         // [ssq_tiles][ssq_ld] (null: plain B operand)
    int ssq_tiles;
    int ssq_ld;
    const __nv_bfloat16* gain;   // [K]
    float eps;
    int norm_h;                  // features of a row (the mean's divisor)
    __nv_bfloat16* norm_out;     // optional copy of the normalised rows [M][norm_out_ld] (written from n-tile 0)
    int norm_out_ld;
    // EPI_RESID / EPI_BF16: partial sums of squares of the written rows, per output n-tile
    float* ssq_out;              // [n_tiles][ssq_ld] or null
    // Diagnostic trace (null in normal use): per CTA 8 globaltimer stamps (ns):
    // entry, producer past the dependency wait, first stage landed, last MMA
    // issued, accumulators drained, epilogue done, exit, clock64 span of the CTA.
    long long* trace;
};

// ---------------------------------------------------------------------------
// Work partition.  CTA p owns units [begin(p), begin(p+1)), begin(p) = p*U/P.
// Requires U >= P so that no CTA is empty.
// ---------------------------------------------------------------------------
__host__ __device__ inline long long sk_begin(int p, long long U, int P) {
    return (long long)p * U / P;
}
// The CTA that owns unit u: the largest p with begin(p) <= u, i.e.
// p = ceil((u+1) P / U) - 1.
__host__ __device__ inline int sk_owner(long long u, long long U, int P) {
    return (int)(((u + 1) * (long long)P - 1) / U);
}
__host__ __device__ inline int sk_first_cta(long long tile, int KB, long long U, int P) {
    return sk_owner(tile * KB, U, P);
}
__host__ __device__ inline int sk_n_contrib(long long tile, int KB, long long U, int P) {
    return sk_owner((tile + 1) * KB - 1, U, P) - sk_owner(tile * KB, U, P) + 1;
}
// Tokens per MMA tile for M rows.
inline int pick_nt(int M) {
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

// Row-major bf16 tensor map without swizzle (box {box_inner, box_rows}); false when the
// driver's encoder is unavailable or the layout is not 16-byte aligned.
bool encode_bf16_rows(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride,
                      uint32_t box_inner, uint32_t box_rows);

// Weight tiles each CTA prefetches into L2 (beyond its shared-memory ring)
// before its dependency wait; process-wide, set by dflash_diag_set_gemm_prefetch.
int gemm_l2_prefetch();
void set_gemm_l2_prefetch(int tiles);
// Ring stages each CTA fills with weight tiles before its dependency wait (0 = all).
int gemm_pre_stages();
void set_gemm_pre_stages(int stages);
int gemm_last_arriver();
void set_gemm_last_arriver(int on);
int gemm_max_cluster();
void set_gemm_max_cluster(int c);
int gemm_max_active_clusters(int c);   // resident clusters of c CTAs of the cluster-mode 16-token kernel

// Host launcher (gemm_tc.cu).  Fills the derived fields (KB, tiles, units,
// ctas) and launches on `stream`.  Returns a cudaError_t; cudaErrorInvalidValue
// when units * 160 reaches 2^32 (the kernel's split-tile bookkeeping is 32-bit).
int launch_gemm_tc(GemmParams& p, int nt, int num_sms, cudaStream_t stream);

// 2-D bf16 tensor map (abi.cu): `inner` contiguous elements per row, `rows`
// rows of `stride` elements, box {64, box_rows}, 128-byte swizzle, zero fill
// out of bounds.  False when the driver's encoder rejects it.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride,
                    uint32_t box_rows);

// Bytes of split-tile partial scratch for ctas CTAs at tile width nt.
inline size_t gemm_partial_bytes(int ctas, int nt) { return (size_t)2 * ctas * nt * 128 * sizeof(float); }

}  // namespace df
