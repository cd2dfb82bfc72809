// C ABI of libdflash (include/dflash.h): argument validation, workspace and
// cache layout, tensor-map encoding, and the launch sequence of each call.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/dflash.h"
#include "../../include/dflash_ablation.h"
#include "../../include/dflash_diag.h"
#include "attn.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "kernels.cuh"

using namespace df;

namespace df {
static bool g_pdl = true;
// RMSNorm folded into the GEMMs that consume the normalised rows (draft step,
// token tiles up to kFoldMaxNT wide; wider tiles give the two normalising warps
// more work per stage than the weight stream leaves them, measured slower than a
// separate norm kernel); dflash_diag_set_norm_fold switches it.
static bool g_fold = true;
// Partition of dflash_inject_kv's GEMM: whole output tiles (every K/V element one
// in-order sum over all of K), or split-K per slab of tile rows.  Whole tiles are
// faster for wide token tiles (prefill); the fused per-cycle call
// dflash_fuse_inject always uses split-K slabs (all SMs stream at batch 1).
static bool g_inject_whole = true;
// Whether the final norm is folded into the LM-head GEMM too (see draft_bf16).
static bool g_fold_head = false;
// O-projection on the SMs the attention does not hold (see layers_bf16).
static bool g_o_beside_attention = false;
static int g_o_late_deficit = 9;   // units fewer for the O-projection CTAs that start after the attention (measured: 0, 3, 9)
constexpr int kFoldMaxNT = 16;
void set_pdl(bool on) { g_pdl = on; }
bool pdl_enabled() { return g_pdl; }
void ensure_carveout(const void* fn) {
    static std::vector<const void*> done;
    for (const void* f : done)
        if (f == fn) return;
    cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    done.push_back(fn);
}

typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static PFN_encodeTiled_t get_encode() {
    static PFN_encodeTiled_t fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_encodeTiled_t)p;
    }
    return fn;
}

// 2-D bf16 tensor map: `inner` contiguous elements per row, `rows` rows of
// `stride` elements, box {64, box_rows}, 128-byte swizzle, zero fill out of bounds.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride,
                    uint32_t box_rows) {
    PFN_encodeTiled_t enc = get_encode();
    if (!enc || rows == 0 || inner == 0) return false;
    if (((uintptr_t)base & 15) || ((stride * 2) & 15)) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {stride * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor map of row-major rows (no swizzle): `inner` elements per row, `rows`
// rows of `stride` elements, box {box_inner, box_rows}, zero fill out of bounds.
bool encode_bf16_rows(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride,
                      uint32_t box_inner, uint32_t box_rows) {
    PFN_encodeTiled_t enc = get_encode();
    if (!enc || rows == 0 || inner == 0) return false;
    if (((uintptr_t)base & 15) || ((stride * 2) & 15) || ((box_inner * 2) & 15)) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {stride * 2};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace df

namespace {

inline size_t al(size_t v, size_t a = 1024) { return (v + a - 1) / a * a; }
inline int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

constexpr int kMaxCtas = 160;   // >= SMs of any B200 part

struct WsLayout {
    size_t status, rope, x, h, q, o, act, hf, y, y32, lgs, req_ok, gpart, gcnt, rec, ssq, ssq_ctx, total;
    int nt_max;
    long long n_counters;
};

int m_tiles_for(int M) { return M <= 0 ? 0 : cdiv(M, pick_nt(M)); }

void make_layout(const dflash_config& c, WsLayout& L) {
    const bool bf = c.dtype == DFLASH_BF16;
    const size_t es = bf ? 2 : 4;
    const long long H = c.hidden, d = c.head_dim, Nq = (long long)c.n_q_heads * d, Nkv = (long long)c.n_kv_heads * d;
    const long long I = c.intermediate, V = c.vocab;
    const long long Mmax = (long long)c.max_batch * c.max_gamma;
    const long long Mlm = std::max(1LL, (long long)c.max_batch * (c.max_gamma - 1));
    const long long R = std::max(1, c.max_rows);
    size_t off = 0;
    L.status = off; off += 1024;
    L.rope = off; off = al(off + (size_t)c.max_position * (d / 2) * sizeof(float2));
    L.x = off; off = al(off + Mmax * H * es);
    L.h = off; off = al(off + Mmax * H * es);
    L.q = off; off = al(off + Mmax * Nq * es);
    L.o = off; off = al(off + Mmax * Nq * es);
    L.act = off; off = al(off + Mmax * I * es);
    L.hf = off; off = al(off + Mlm * H * es);
    L.y = off; off = al(off + R * H * es);
    L.req_ok = off; off = al(off + (size_t)c.max_batch * 4);
    L.y32 = L.lgs = L.gpart = L.gcnt = L.rec = L.ssq = L.ssq_ctx = off;
    L.nt_max = 0;
    L.n_counters = 0;
    if (!bf) {
        long long y32 = std::max(std::max(Mmax * (Nq + 2 * Nkv), Mmax * 2 * I), std::max(Mmax * H, R * 2 * Nkv));
        L.y32 = off; off = al(off + (size_t)y32 * 4);
        L.lgs = off; off = al(off + (size_t)Mlm * V * 4);
    } else {
        L.nt_max = pick_nt((int)std::max(std::max(Mmax, Mlm), R));
        L.gpart = off; off = al(off + gemm_partial_bytes(kMaxCtas, L.nt_max));
        const long long t_layer = std::max(std::max((long long)cdiv(Nq, 128) + 2 * cdiv(Nkv, 128), (long long)cdiv(H, 128)),
                                           I / 64);
        const long long t_big = std::max((long long)cdiv(H, 128), 10LL * cdiv(Nkv, 128));
        L.n_counters = std::max(std::max(t_layer * m_tiles_for((int)Mmax),
                                         (long long)cdiv(V, 128) * m_tiles_for((int)std::max(Mlm, Mmax))),
                                t_big * m_tiles_for((int)R));
        L.gcnt = off; off = al(off + (size_t)L.n_counters * 4);
        // LM-head records for whole blocks (the folded final norm runs the head on all gamma rows)
        L.rec = off; off = al(off + (size_t)cdiv(V, 128) * std::max(Mlm, Mmax) * sizeof(float4));
        // per-(128-feature tile, token row) partial sums of squares of the residual stream
        L.ssq = off; off = al(off + (size_t)cdiv(H, 128) * Mmax * sizeof(float));
        // the same for the projected context rows of dflash_fuse_inject
        L.ssq_ctx = off; off = al(off + (size_t)cdiv(H, 128) * R * sizeof(float));
    }
    L.total = off;
}

int validate_config(const dflash_config* c) {
    if (!c) return DFLASH_INVALID_ARG;
    if (c->hidden <= 0 || c->n_layers < 0 || c->n_layers > DFLASH_MAX_LAYERS || c->n_q_heads <= 0 ||
        c->n_kv_heads <= 0 || c->head_dim <= 0 || c->intermediate <= 0 || c->vocab <= 0 || c->n_sel <= 0 ||
        c->target_hidden <= 0 || c->max_gamma < 1 || c->max_batch < 1 || c->max_rows < 0 || c->max_position < 2 ||
        !(c->rope_theta > 0) || !(c->rms_eps >= 0))
        return DFLASH_INVALID_ARG;
    if (c->mask_id < 0 || c->mask_id >= c->vocab) return DFLASH_INVALID_ARG;
    if (c->n_q_heads % c->n_kv_heads) return DFLASH_INVALID_ARG;
    if (c->dtype != DFLASH_BF16 && c->dtype != DFLASH_F32) return DFLASH_INVALID_ARG;
    if (c->max_gamma > 32 || c->n_sel > 8 || (c->head_dim & 1)) return DFLASH_UNSUPPORTED;
    if (c->hidden % 8 || c->target_hidden % 8) return DFLASH_UNSUPPORTED;
    if (c->dtype == DFLASH_BF16) {
        if (c->head_dim != 64 && c->head_dim != 128) return DFLASH_UNSUPPORTED;
        if (c->hidden % 64 || c->intermediate % 64 || c->target_hidden % 64) return DFLASH_UNSUPPORTED;
        if ((c->n_q_heads / c->n_kv_heads) * c->max_gamma > 128) return DFLASH_UNSUPPORTED;
    } else {
        if (c->max_position > 12000) return DFLASH_UNSUPPORTED;   // fp32 attention keeps a row of scores in smem
    }
    return DFLASH_OK;
}

}  // namespace

struct dflash_handle {
    dflash_config cfg;
    dflash_weights w;
    int num_sms;
    uint8_t* ws;
    size_t ws_bytes;
    WsLayout L;
    int* status;
    float2* rope;
    void *x, *h, *q, *o, *act, *hf, *y;
    float *y32, *lgs, *gpart, *ssq, *ssq_ctx;
    int *req_ok, *gcnt;
    float4* rec;
    CUtensorMap tm_wfc, tm_lm;
    CUtensorMap tm_wq[DFLASH_MAX_LAYERS], tm_wk[DFLASH_MAX_LAYERS], tm_wv[DFLASH_MAX_LAYERS], tm_wo[DFLASH_MAX_LAYERS];
    CUtensorMap tm_wg[DFLASH_MAX_LAYERS], tm_wu[DFLASH_MAX_LAYERS], tm_wd[DFLASH_MAX_LAYERS];
    long long launches;
    // Diagnostic capture (dflash_diag_draft_capture): residual stream after the
    // embedding and after every layer, and the final-norm rows.
    void* cap_x = nullptr;
    void* cap_hf = nullptr;
    // per-layer stage captures (dflash_diag_draft_capture_stages), each [L][M][width]
    void* cap_h = nullptr;     // normalised layer input (width H)
    void* cap_q = nullptr;     // q (n_q_heads * d)
    void* cap_o = nullptr;     // attention output (n_q_heads * d)
    void* cap_xm = nullptr;    // residual stream after the O-projection (H)
    void* cap_h2 = nullptr;    // normalised MLP input (H)
    void* cap_act = nullptr;   // SwiGLU output (intermediate)
    // Diagnostic step trace (dflash_diag_step_trace): per-block %globaltimer
    // stamps of every traced launch, laid out one launch after the other.
    long long* tr_buf = nullptr;
    long long tr_cap = 0, tr_used = 0;
    struct TraceRec { int kind, blocks, words, wait_idx, exit_idx; long long offset; };
    std::vector<TraceRec> tr_recs;
    // Diagnostic timing (dflash_diag_timing_*): event pairs around launches.
    std::vector<cudaEvent_t> ev;
    std::vector<int> ev_kind;
    int ev_used = 0;
    bool timing = false;
};

struct dflash_cache {
    const dflash_handle* h;
    uint8_t* mem;
    size_t bytes;
    int batch, capacity;
    int* status;
    int* len;
    int* committed;
    void* slab;
    long long s_kv, s_kind, s_layer, s_req;
    CUtensorMap tm_slab;
};

namespace {

struct CacheLayout {
    size_t len, committed, slab, total;
};
void cache_layout(const dflash_config& c, int batch, int capacity, CacheLayout& L) {
    const size_t es = c.dtype == DFLASH_BF16 ? 2 : 4;
    L.len = 256;
    L.committed = L.len + al((size_t)batch * 4, 256);
    L.slab = al(L.committed + al((size_t)batch * 4, 256), 1024);
    L.total = L.slab + (size_t)batch * c.n_layers * 2 * c.n_kv_heads * (size_t)capacity * c.head_dim * es;
}

inline cudaStream_t S(dflash_stream s) { return (cudaStream_t)s; }
inline cudaStream_t st_of(dflash_stream s) { return (cudaStream_t)s; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? DFLASH_OK : DFLASH_CUDA; }

bool aligned16(const void* p) { return p && (((uintptr_t)p) & 15) == 0; }

// Launch groups reported by the diagnostic timer.
enum TimedKind {
    TK_EMBED = 0, TK_RMSNORM, TK_GEMM_QKV, TK_ATTENTION, TK_GEMM_O, TK_GEMM_SWIGLU, TK_GEMM_DOWN, TK_GEMM_LMHEAD,
    TK_LM_REDUCE, TK_GEMM_FUSE, TK_GEMM_INJECT, TK_INJECT_FINALIZE, TK_ACCEPT, TK_SET_LEN, TK_SIMT_F32, TK_COUNT
};
const char* kTimedNames[TK_COUNT] = {"embed", "rmsnorm", "gemm_qkv", "attention", "gemm_o", "gemm_swiglu",
                                     "gemm_down", "gemm_lmhead", "lm_reduce", "gemm_fuse", "gemm_inject",
                                     "inject_finalize", "accept", "set_len", "simt_f32"};

// Records a CUDA event before and after the launches in its scope when the
// handle's diagnostic timer is on (events on the launch stream).
struct Timed {
    dflash_handle* h;
    cudaStream_t st;
    int slot = -1;
    Timed(dflash_handle* h_, int kind, cudaStream_t st_) : h(h_), st(st_) {
        if (h->timing && h->ev_used + 2 <= (int)h->ev.size()) {
            slot = h->ev_used;
            h->ev_used += 2;
            h->ev_kind[slot / 2] = kind;
            cudaEventRecord(h->ev[slot], st);
        }
    }
    ~Timed() {
        if (slot >= 0) cudaEventRecord(h->ev[slot + 1], st);
    }
};

// Room for one launch's step trace: `blocks` x `words` int64 stamps, the
// stamp past the dependency wait at word wait_idx and the exit stamp at word
// exit_idx of each block.  Null when tracing is off or the buffer is full.
long long* trace_slot(dflash_handle* h, int kind, int blocks, int words, int wait_idx, int exit_idx) {
    if (!h->tr_buf || blocks <= 0) return nullptr;
    const long long need = (long long)blocks * words;
    if (h->tr_used + need > h->tr_cap) return nullptr;
    long long* p = h->tr_buf + h->tr_used;
    h->tr_recs.push_back({kind, blocks, words, wait_idx, exit_idx, h->tr_used});
    h->tr_used += need;
    return p;
}
// Small kernels: two stamps per block (past the wait, exit).
long long* trace_small(dflash_handle* h, int kind, int blocks) { return trace_slot(h, kind, blocks, 2, 0, 1); }

// Diagnostic capture of the residual stream x ([B*gamma][H]) into slot `slot`
// of the caller's [(L+1)][B*gamma][H] buffer.
void capture_x(dflash_handle* h, int slot, int M, cudaStream_t st) {
    if (!h->cap_x) return;
    const size_t es = h->cfg.dtype == DFLASH_BF16 ? 2 : 4;
    const size_t row = (size_t)M * h->cfg.hidden * es;
    cudaMemcpyAsync((uint8_t*)h->cap_x + (size_t)slot * row, h->x, row, cudaMemcpyDeviceToDevice, st);
}
// Diagnostic stage capture: rows x width elements of `src` into slot `layer` of dst.
void capture_stage(dflash_handle* h, void* dst, const void* src, int layer, int M, int width, cudaStream_t st) {
    if (!dst) return;
    const size_t es = h->cfg.dtype == DFLASH_BF16 ? 2 : 4;
    const size_t bytes = (size_t)M * width * es;
    cudaMemcpyAsync((uint8_t*)dst + (size_t)layer * bytes, src, bytes, cudaMemcpyDeviceToDevice, st);
}
void capture_hf(dflash_handle* h, int Mlm, cudaStream_t st) {
    if (!h->cap_hf) return;
    const size_t es = h->cfg.dtype == DFLASH_BF16 ? 2 : 4;
    cudaMemcpyAsync(h->cap_hf, h->hf, (size_t)Mlm * h->cfg.hidden * es, cudaMemcpyDeviceToDevice, st);
}

// Common GEMM plumbing.
void gemm_common(dflash_handle* h, GemmParams& p) {
    p.l2_prefetch = gemm_l2_prefetch();
    p.pre_stages = gemm_pre_stages();
    p.last_arriver = gemm_last_arriver();
    p.partial = h->gpart;
    p.counters = h->gcnt;
    p.status = h->status;
    p.ctas = 0;
}

// The last CTAs of a launch land on the SMs the previous kernel's last CTAs held and
// start after them: the last g_tail_ctas CTAs of the step's other whole-grid GEMMs
// take g_tail_deficit fewer k-block units.  The shift also moves the split points
// of every tile, and that dominates: 24 CTAs x 3 units measured best on the
// Qwen3-8B-shaped drafter (neighbouring settings were slower, and the
// Qwen3-4B-shaped one is slower with it).
static int g_tail_ctas = 24, g_tail_deficit = 3;

int run_gemm(dflash_handle* h, GemmParams& p, int nt, cudaStream_t st, int kind, int ctas = 0, int l2_prefetch = -1) {
    gemm_common(h, p);
    if (p.late_deficit == 0 && g_tail_ctas > 0 && g_tail_deficit > 0 && ctas == 0 && kind != TK_SIMT_F32) {
        p.late_from = std::min(h->num_sms, kMaxCtas) - g_tail_ctas;
        p.late_deficit = g_tail_deficit;
    }
    if (ctas > 0) p.ctas = ctas;
    if (l2_prefetch >= 0) p.l2_prefetch = l2_prefetch;
    // GEMM trace: 8 stamps per CTA (gemm.cuh), past the wait at 1, exit at 6;
    // room for the largest grid, CTAs the launch does not use stay zero.
    p.trace = trace_slot(h, kind, kMaxCtas, 8, 1, 6);
    int e = launch_gemm_tc(p, nt, std::min(h->num_sms, kMaxCtas), st);
    h->launches += p.units > 0 ? 1 : 0;
    return e == 0 ? DFLASH_OK : DFLASH_CUDA;
}

// Activation operand map: rows x K bf16 with row stride `stride`, box rows nt.
bool act_map(CUtensorMap* m, const void* base, int rows, int K, long long stride, int nt) {
    return encode_bf16_2d(m, base, (uint64_t)K, (uint64_t)rows, (uint64_t)stride, (uint32_t)nt);
}


}  // namespace

// The injection GEMMs of rows [0, total_rows) of `src` ([total_rows, H] bf16):
// all layers' Wk/Wv stacked as one A operand (up to kMaxAMats matrices per
// launch), RoPE and the cache write in the epilogue.  Either partition keeps the
// fp32 summation order of every K/V element independent of the number of rows,
// so injecting rows in chunks writes the same bits as injecting them at once:
//  - whole: one launch, CTAs take whole output tiles (each element one in-order
//    sum over all of K); at batch 1 only n-tiles CTAs stream the weights, but
//    wide token tiles (prefill) run without split-K partials;
//  - split: one launch per slab of nt rows, each with a single m-tile, so the
//    split-K partition over n_tiles x k-blocks is the same for every slab; all
//    SMs stream the weights (the per-cycle injection of a few rows).
// With ssq (the projected rows' per-tile sums of squares, [cdiv(H,128)][max_rows]),
// src holds the un-normalised rows and each launch applies RMSNorm * g_fc to its
// token tiles in shared memory (and copies the normalised rows to ctx_out when it
// is not null).
static int inject_gemms(dflash_handle* h, dflash_cache* cc, const void* src, const int32_t* row_start,
                 const int32_t* row_count, int total_rows, const float* ssq, void* ctx_out, bool whole,
                 cudaStream_t st) {
    const dflash_config& c = h->cfg;
    const int H = c.hidden, d = c.head_dim, Nkv = c.n_kv_heads * d;
    const int nt = pick_nt(total_rows);
    const int slab = whole ? total_rows : nt;   // whole tiles: one launch over all rows
    for (int row0 = 0; row0 < total_rows; row0 += slab) {
        const int rows = std::min(slab, total_rows - row0);
        CUtensorMap tb;
        if (!act_map(&tb, (const uint8_t*)src + (size_t)row0 * H * 2, rows, H, H, nt)) return DFLASH_INVALID_ARG;
        for (int l0 = 0; l0 < c.n_layers; l0 += kMaxAMats / 2) {
            const int nl = std::min(kMaxAMats / 2, c.n_layers - l0);
            GemmParams p;
            std::memset(&p, 0, sizeof(p));
            for (int i = 0; i < nl; ++i) {
                p.ta[2 * i] = h->tm_wk[l0 + i];
                p.ta[2 * i + 1] = h->tm_wv[l0 + i];
                p.amat[2 * i].rows = Nkv;
                p.amat[2 * i + 1].rows = Nkv;
            }
            p.n_amat = 2 * nl;
            p.tb[0] = tb;
            p.kb_per_b = cdiv(H, 64);
            p.M = rows;
            p.row0 = row0;
            p.whole_tiles = whole ? 1 : 0;
            p.K = H;
            p.epi = EPI_INJECT;
            p.d = d;
            p.cap = cc->capacity;
            p.layer = l0;
            p.batch = cc->batch;
            p.len = cc->len;
            p.rope = h->rope;
            p.slab = (__nv_bfloat16*)cc->slab;
            p.s_req = cc->s_req;
            p.s_layer = cc->s_layer;
            p.s_kind = cc->s_kind;
            p.s_kv = cc->s_kv;
            p.row_start = row_start;
            p.row_count = row_count;
            if (ssq) {
                p.ssq_in = ssq + row0;
                p.ssq_tiles = cdiv(H, 128);
                p.ssq_ld = std::max(1, c.max_rows);
                p.gain = (const __nv_bfloat16*)h->w.g_fc;
                p.eps = (float)c.rms_eps;
                p.norm_h = H;
                if (ctx_out && l0 == 0) {
                    p.norm_out = (__nv_bfloat16*)ctx_out + (size_t)row0 * H;
                    p.norm_out_ld = H;
                }
            }
            Timed t(h, TK_GEMM_INJECT, st);
            int r = run_gemm(h, p, nt, st, TK_GEMM_INJECT);
            if (r) return r;
        }
    }
    return DFLASH_OK;
}

// a1's projection: y = R(concat_i hiddens[i] . W_fc^T) into the workspace's y
// ([total_rows, H] bf16), with ssq (or null) receiving the rows' per-tile sums
// of squares ([cdiv(H,128)][max_rows]).
static int fuse_gemm(dflash_handle* h, const void* const* hiddens, int64_t row_stride, int total_rows, float* ssq,
                     cudaStream_t st) {
    const dflash_config& c = h->cfg;
    if ((row_stride * 2) % 16) return DFLASH_INVALID_ARG;
    for (int i = 0; i < c.n_sel; ++i)
        if (!aligned16(hiddens[i])) return DFLASH_INVALID_ARG;
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    const int nt = pick_nt(total_rows);
    p.ta[0] = h->tm_wfc;
    p.n_amat = 1;
    p.amat[0].rows = c.hidden;
    for (int i = 0; i < c.n_sel; ++i)
        if (!act_map(&p.tb[i], hiddens[i], total_rows, c.target_hidden, row_stride, nt)) return DFLASH_INVALID_ARG;
    p.kb_per_b = c.target_hidden / 64;
    p.M = total_rows;
    p.K = c.n_sel * c.target_hidden;
    p.epi = EPI_BF16;
    p.out = h->y;
    p.ldo = c.hidden;
    if (ssq) {
        p.ssq_out = ssq;
        p.ssq_ld = std::max(1, c.max_rows);
    }
    Timed t(h, TK_GEMM_FUSE, st);
    return run_gemm(h, p, nt, st, TK_GEMM_FUSE);
}

extern "C" {

const char* dflash_status_string(int s) {
    switch (s) {
    case DFLASH_OK: return "ok";
    case DFLASH_INVALID_ARG: return "invalid argument";
    case DFLASH_UNSUPPORTED: return "unsupported shape";
    case DFLASH_CUDA: return "CUDA error";
    case DFLASH_WORKSPACE: return "workspace or cache memory too small";
    case DFLASH_CAPACITY: return "cache capacity exceeded";
    case DFLASH_STATE: return "cache state: len != committed";
    case DFLASH_TOKEN_RANGE: return "token id out of range";
    case DFLASH_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
    }
}

int dflash_workspace_bytes(const dflash_config* cfg, size_t* bytes) {
    int v = validate_config(cfg);
    if (v) return v;
    if (!bytes) return DFLASH_INVALID_ARG;
    WsLayout L;
    make_layout(*cfg, L);
    *bytes = L.total;
    return DFLASH_OK;
}

int dflash_create(const dflash_config* cfg, const dflash_weights* w, void* workspace, size_t ws_bytes,
                  dflash_handle** out) {
    int v = validate_config(cfg);
    if (v) return v;
    if (!w || !workspace || !out) return DFLASH_INVALID_ARG;
    if ((uintptr_t)workspace & 1023) return DFLASH_INVALID_ARG;
    const dflash_config& c = *cfg;
    if (!w->w_fc || !w->g_fc || !w->embed || !w->lm_head || !w->g_final) return DFLASH_INVALID_ARG;
    for (int l = 0; l < c.n_layers; ++l)
        if (!w->g_in[l] || !w->wq[l] || !w->wk[l] || !w->wv[l] || !w->wo[l] || !w->g_post[l] || !w->w_gate[l] ||
            !w->w_up[l] || !w->w_down[l])
            return DFLASH_INVALID_ARG;
    WsLayout L;
    make_layout(c, L);
    if (ws_bytes < L.total) return DFLASH_WORKSPACE;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DFLASH_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return DFLASH_CUDA;
    if (prop.major != 10) return DFLASH_UNSUPPORTED;   // built for sm_100a only

    dflash_handle* h = new (std::nothrow) dflash_handle();
    if (!h) return DFLASH_CUDA;
    h->cfg = c;
    h->w = *w;
    h->num_sms = prop.multiProcessorCount;
    h->ws = (uint8_t*)workspace;
    h->ws_bytes = ws_bytes;
    h->L = L;
    uint8_t* b = h->ws;
    h->status = (int*)(b + L.status);
    h->rope = (float2*)(b + L.rope);
    h->x = b + L.x;
    h->h = b + L.h;
    h->q = b + L.q;
    h->o = b + L.o;
    h->act = b + L.act;
    h->hf = b + L.hf;
    h->y = b + L.y;
    h->y32 = (float*)(b + L.y32);
    h->lgs = (float*)(b + L.lgs);
    h->req_ok = (int*)(b + L.req_ok);
    h->gpart = (float*)(b + L.gpart);
    h->gcnt = (int*)(b + L.gcnt);
    h->rec = (float4*)(b + L.rec);
    h->ssq = (float*)(b + L.ssq);
    h->ssq_ctx = (float*)(b + L.ssq_ctx);
    h->launches = 0;

    // RoPE table: angle p * theta^(-2i/d) in fp64, stored as fp32 (cos, sin).
    const int half = c.head_dim / 2;
    std::vector<float2> tab((size_t)c.max_position * half);
    for (int i = 0; i < half; ++i) {
        const double inv_freq = std::pow(c.rope_theta, -2.0 * i / c.head_dim);
        for (long long pos = 0; pos < c.max_position; ++pos) {
            const double ang = (double)pos * inv_freq;
            tab[(size_t)pos * half + i] = make_float2((float)std::cos(ang), (float)std::sin(ang));
        }
    }
    cudaError_t e = cudaMemcpy(h->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemset(h->status, 0, 1024);
    if (e == cudaSuccess) e = cudaMemset(h->req_ok, 0, (size_t)c.max_batch * 4);
    if (e == cudaSuccess && L.n_counters > 0) e = cudaMemset(h->gcnt, 0, (size_t)L.n_counters * 4);
    if (e == cudaSuccess) e = cudaStreamSynchronize(0);
    if (e != cudaSuccess) {
        delete h;
        return DFLASH_CUDA;
    }
    if (c.dtype == DFLASH_BF16) {
        const int H = c.hidden, d = c.head_dim, Nq = c.n_q_heads * d, Nkv = c.n_kv_heads * d, I = c.intermediate;
        bool ok = encode_bf16_2d(&h->tm_wfc, w->w_fc, (uint64_t)c.n_sel * c.target_hidden, H,
                                 (uint64_t)c.n_sel * c.target_hidden, 128) &&
                  encode_bf16_2d(&h->tm_lm, w->lm_head, H, c.vocab, H, 128);
        for (int l = 0; ok && l < c.n_layers; ++l) {
            ok = encode_bf16_2d(&h->tm_wq[l], w->wq[l], H, Nq, H, 128) &&
                 encode_bf16_2d(&h->tm_wk[l], w->wk[l], H, Nkv, H, 128) &&
                 encode_bf16_2d(&h->tm_wv[l], w->wv[l], H, Nkv, H, 128) &&
                 encode_bf16_2d(&h->tm_wo[l], w->wo[l], Nq, H, Nq, 128) &&
                 encode_bf16_2d(&h->tm_wg[l], w->w_gate[l], H, I, H, 64) &&
                 encode_bf16_2d(&h->tm_wu[l], w->w_up[l], H, I, H, 64) &&
                 encode_bf16_2d(&h->tm_wd[l], w->w_down[l], I, H, I, 128);
        }
        if (!ok) {
            delete h;
            return get_encode() ? DFLASH_INVALID_ARG : DFLASH_CUDA;
        }
    }
    *out = h;
    return DFLASH_OK;
}

void dflash_destroy(dflash_handle* h) {
    if (!h) return;
    for (auto e : h->ev) cudaEventDestroy(e);
    delete h;
}

int64_t dflash_launch_count(const dflash_handle* h) { return h ? h->launches : 0; }

int dflash_cache_bytes(const dflash_handle* h, int batch, int capacity, size_t* bytes) {
    if (!h || !bytes || batch < 1 || batch > h->cfg.max_batch || capacity < 1 || capacity > h->cfg.max_position)
        return DFLASH_INVALID_ARG;
    CacheLayout L;
    cache_layout(h->cfg, batch, capacity, L);
    *bytes = L.total;
    return DFLASH_OK;
}

int dflash_cache_init(const dflash_handle* h, void* mem, size_t bytes, int batch, int capacity, dflash_cache** out,
                      dflash_stream stream) {
    if (!h || !mem || !out || batch < 1 || batch > h->cfg.max_batch || capacity < 1 ||
        capacity > h->cfg.max_position)
        return DFLASH_INVALID_ARG;
    if ((uintptr_t)mem & 1023) return DFLASH_INVALID_ARG;
    CacheLayout L;
    cache_layout(h->cfg, batch, capacity, L);
    if (bytes < L.total) return DFLASH_WORKSPACE;
    const dflash_config& c = h->cfg;
    dflash_cache* cc = new (std::nothrow) dflash_cache();
    if (!cc) return DFLASH_CUDA;
    cc->h = h;
    cc->mem = (uint8_t*)mem;
    cc->bytes = bytes;
    cc->batch = batch;
    cc->capacity = capacity;
    cc->status = (int*)mem;
    cc->len = (int*)((uint8_t*)mem + L.len);
    cc->committed = (int*)((uint8_t*)mem + L.committed);
    cc->slab = (uint8_t*)mem + L.slab;
    cc->s_kv = (long long)capacity * c.head_dim;
    cc->s_kind = cc->s_kv * c.n_kv_heads;
    cc->s_layer = cc->s_kind * 2;
    cc->s_req = cc->s_layer * c.n_layers;
    if (c.dtype == DFLASH_BF16 && c.n_layers > 0) {
        const uint64_t rows = (uint64_t)batch * cc->s_req / c.head_dim;
        if (!encode_bf16_2d(&cc->tm_slab, cc->slab, c.head_dim, rows, c.head_dim, 64)) {
            delete cc;
            return DFLASH_CUDA;
        }
    }
    if (cudaMemsetAsync(mem, 0, L.slab, S(stream)) != cudaSuccess) {
        delete cc;
        return DFLASH_CUDA;
    }
    *out = cc;
    return DFLASH_OK;
}

void dflash_cache_release(dflash_cache* c) { delete c; }

int dflash_cache_get_info(const dflash_cache* c, dflash_cache_info* info) {
    if (!c || !info) return DFLASH_INVALID_ARG;
    info->batch = c->batch;
    info->capacity = c->capacity;
    info->status = c->status;
    info->len = c->len;
    info->committed = c->committed;
    info->slab = c->slab;
    info->stride_kv = c->s_kv;
    info->stride_kind = c->s_kind;
    info->stride_layer = c->s_layer;
    info->stride_request = c->s_req;
    return DFLASH_OK;
}

int dflash_cache_set_len(dflash_cache* c, const int32_t* lens, dflash_stream stream) {
    if (!c || !lens) return DFLASH_INVALID_ARG;
    launch_set_len(lens, c->batch, c->capacity, c->len, c->committed, c->status, S(stream),
                   trace_small(const_cast<dflash_handle*>(c->h), TK_SET_LEN, cdiv(c->batch, 128)));
    const_cast<dflash_handle*>(c->h)->launches += 1;
    return cuda_status(cudaGetLastError());
}

int dflash_cache_status(dflash_handle* h, dflash_cache* c, dflash_stream stream) {
    if (!h || !c || c->h != h) return DFLASH_INVALID_ARG;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return DFLASH_CUDA;
    int hs = 0, cs = 0;
    if (cudaMemcpy(&hs, h->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DFLASH_CUDA;
    if (cudaMemcpy(&cs, c->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DFLASH_CUDA;
    if (cudaMemset(c->status, 0, 4) != cudaSuccess) return DFLASH_CUDA;
    if (hs && cudaMemset(h->status, 0, 4) != cudaSuccess) return DFLASH_CUDA;
    if (cudaStreamSynchronize(0) != cudaSuccess) return DFLASH_CUDA;
    return hs ? hs : cs;
}

// ---------------------------------------------------------------------------
// a1: fuse context
// ---------------------------------------------------------------------------
int dflash_fuse_context(dflash_handle* h, const void* const* hiddens, int64_t row_stride, int total_rows,
                        void* ctx_out, dflash_stream stream) {
    if (!h || !hiddens || !ctx_out || total_rows < 0 || total_rows > h->cfg.max_rows) return DFLASH_INVALID_ARG;
    const dflash_config& c = h->cfg;
    if (row_stride < c.target_hidden) return DFLASH_INVALID_ARG;
    for (int i = 0; i < c.n_sel; ++i)
        if (!hiddens[i]) return DFLASH_INVALID_ARG;
    if (total_rows == 0) return DFLASH_OK;
    cudaStream_t st = S(stream);
    const int H = c.hidden;
    if (c.dtype == DFLASH_BF16) {
        if (!aligned16(ctx_out)) return DFLASH_INVALID_ARG;
        int r = fuse_gemm(h, hiddens, row_stride, total_rows, nullptr, st);
        if (r) return r;
        Timed t(h, TK_RMSNORM, st);
        launch_rmsnorm<__nv_bfloat16>((const __nv_bfloat16*)h->y, (const __nv_bfloat16*)h->w.g_fc,
                                      (__nv_bfloat16*)ctx_out, total_rows, H, (float)c.rms_eps, total_rows, 0, 0, st,
                                      trace_small(h, TK_RMSNORM, total_rows));
    } else {
        Timed t(h, TK_SIMT_F32, st);
        XSegs xs;
        std::memset(&xs, 0, sizeof(xs));
        for (int i = 0; i < c.n_sel; ++i) xs.ptr[i] = (const float*)hiddens[i];
        xs.stride = row_stride;
        xs.width = c.target_hidden;
        launch_gemm_f32(xs, (const float*)h->w.w_fc, (float*)h->y, total_rows, H, c.n_sel * c.target_hidden, H, 0, st);
        launch_rmsnorm<float>((const float*)h->y, (const float*)h->w.g_fc, (float*)ctx_out, total_rows, H,
                              (float)c.rms_eps, total_rows, 0, 0, st);
        h->launches += 1;
    }
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// a2: inject KV
// ---------------------------------------------------------------------------
int dflash_inject_kv(dflash_handle* h, dflash_cache* cc, const void* ctx, const int32_t* row_start,
                     const int32_t* row_count, int total_rows, dflash_stream stream) {
    if (!h || !cc || cc->h != h || !ctx || !row_start || !row_count || total_rows < 0 ||
        total_rows > h->cfg.max_rows)
        return DFLASH_INVALID_ARG;
    if (total_rows == 0) return DFLASH_OK;
    const dflash_config& c = h->cfg;
    cudaStream_t st = S(stream);
    const int H = c.hidden, d = c.head_dim, Nkv = c.n_kv_heads * d;
    if (c.dtype == DFLASH_BF16) {
        if (!aligned16(ctx)) return DFLASH_INVALID_ARG;
        int r = inject_gemms(h, cc, ctx, row_start, row_count, total_rows, nullptr, nullptr, g_inject_whole, st);
        if (r) return r;
    } else {
        Timed t(h, TK_SIMT_F32, st);
        XSegs xs;
        std::memset(&xs, 0, sizeof(xs));
        xs.ptr[0] = (const float*)ctx;
        xs.stride = H;
        xs.width = H;
        for (int l = 0; l < c.n_layers; ++l) {
            launch_gemm_f32(xs, (const float*)h->w.wk[l], h->y32, total_rows, Nkv, H, 2 * Nkv, 0, st);
            launch_gemm_f32(xs, (const float*)h->w.wv[l], h->y32, total_rows, Nkv, H, 2 * Nkv, Nkv, st);
            launch_epi_inject_f32(h->y32, total_rows, Nkv, d, row_start, row_count, cc->batch, cc->len, cc->capacity,
                                  h->rope, (float*)cc->slab, cc->s_req, cc->s_layer, cc->s_kind, cc->s_kv, l, st);
            h->launches += 3;
        }
    }
    Timed t(h, TK_INJECT_FINALIZE, st);
    launch_inject_finalize(row_count, cc->batch, cc->capacity, cc->len, cc->status, st,
                           c.dtype == DFLASH_BF16 ? trace_small(h, TK_INJECT_FINALIZE, cdiv(cc->batch, 128)) : nullptr);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// a1 + a2 in one call: the verify-side pre-step
// ---------------------------------------------------------------------------
int dflash_fuse_inject(dflash_handle* h, dflash_cache* cc, const void* const* hiddens, int64_t row_stride,
                       const int32_t* row_start, const int32_t* row_count, int total_rows, void* ctx_out,
                       dflash_stream stream) {
    if (!h || !cc || cc->h != h || !hiddens || !row_start || !row_count || total_rows < 0 ||
        total_rows > h->cfg.max_rows)
        return DFLASH_INVALID_ARG;
    const dflash_config& c = h->cfg;
    if (row_stride < c.target_hidden) return DFLASH_INVALID_ARG;
    for (int i = 0; i < c.n_sel; ++i)
        if (!hiddens[i]) return DFLASH_INVALID_ARG;
    if (total_rows == 0) return DFLASH_OK;
    cudaStream_t st = S(stream);
    if (c.dtype == DFLASH_BF16 && g_fold && pick_nt(total_rows) <= kFoldMaxNT) {
        if (ctx_out && !aligned16(ctx_out)) return DFLASH_INVALID_ARG;
        // W_fc GEMM writing y and its rows' partial sums of squares, then the
        // injection GEMMs normalising y (RMSNorm * g_fc) tile by tile in shared
        // memory: the context feature never goes through a separate kernel.
        int r = fuse_gemm(h, hiddens, row_stride, total_rows, h->ssq_ctx, st);
        if (r) return r;
        r = inject_gemms(h, cc, h->y, row_start, row_count, total_rows, h->ssq_ctx, ctx_out, false, st);
        if (r) return r;
        Timed t(h, TK_INJECT_FINALIZE, st);
        launch_inject_finalize(row_count, cc->batch, cc->capacity, cc->len, cc->status, st,
                               trace_small(h, TK_INJECT_FINALIZE, cdiv(cc->batch, 128)));
        h->launches += 1;
        return cuda_status(cudaGetLastError());
    }
    // wide token tiles (prefill) and fp32 storage: the two calls one after the other
    // (the normalised rows go to ctx_out, or in place over y)
    void* ctx = ctx_out ? ctx_out : h->y;
    int r = dflash_fuse_context(h, hiddens, row_stride, total_rows, ctx, stream);
    if (r) return r;
    return dflash_inject_kv(h, cc, ctx, row_start, row_count, total_rows, stream);
}

// ---------------------------------------------------------------------------
// a3..a7: draft block
// ---------------------------------------------------------------------------
// The draft step folds each RMSNorm into the GEMM that consumes its output when
// the token tile is at most kFoldMaxNT wide (see GemmParams::ssq_in).
static bool fold_norms(const dflash_handle* h, int M) {
    return g_fold && h->cfg.dtype == DFLASH_BF16 && pick_nt(M) <= kFoldMaxNT;
}

// Consume the residual stream x normalised by `gain` (RMSNorm folded into the GEMM).
static void fold_in(dflash_handle* h, GemmParams& p, const void* gain, int ssq_tiles) {
    p.ssq_in = h->ssq;
    p.ssq_tiles = ssq_tiles;
    p.ssq_ld = h->cfg.max_batch * h->cfg.max_gamma;
    p.gain = (const __nv_bfloat16*)gain;
    p.eps = (float)h->cfg.rms_eps;
    p.norm_h = h->cfg.hidden;
}

// The draft layers over the block rows in h->x ([B * gamma][H], rows b * gamma +
// j at positions len[b] + j), every request validated in h->req_ok.  Each layer
// writes the rows' own K/V at cache rows [len, len + gamma).  draft: attention
// without a mask (the block is bidirectional) and the rows' K/V are scratch.
// ingest (input fusion): causal attention (row j sees positions <= len + j), and
// the last layer stops once its K/V are written (its attention and MLP change no
// cached value); the caller then appends the rows to the cache.
static int layers_bf16(dflash_handle* h, dflash_cache* cc, int gamma, bool ingest, cudaStream_t st) {
    const dflash_config& c = h->cfg;
    const int B = cc->batch, M = B * gamma;
    const int H = c.hidden, d = c.head_dim, Nq = c.n_q_heads * d, Nkv = c.n_kv_heads * d, I = c.intermediate;
    typedef __nv_bfloat16 bf;
    const int nt = pick_nt(M);
    const bool fold = fold_norms(h, M);
    const int nH = cdiv(H, 128);                 // producer n-tiles of x: partial sums per row
    const int ssq_ld = c.max_batch * c.max_gamma;
    CUtensorMap tm_h, tm_o, tm_act, tm_x;
    if (!act_map(&tm_h, h->h, M, H, H, nt) || !act_map(&tm_o, h->o, M, Nq, Nq, nt) ||
        !act_map(&tm_act, h->act, M, I, I, nt) || !act_map(&tm_x, h->x, M, H, H, nt))
        return DFLASH_CUDA;
    int splits, chunk;
    attn_plan(B, c.n_kv_heads, cc->capacity, h->num_sms, attn_max_cluster(d), splits, chunk);
    AttnParams ap;
    std::memset(&ap, 0, sizeof(ap));
    ap.tmap = cc->tm_slab;
    ap.q = (const bf*)h->q;
    ap.out = (bf*)h->o;
    ap.len = cc->len;
    ap.req_ok = h->req_ok;
    ap.gamma = gamma;
    ap.G = c.n_q_heads / c.n_kv_heads;
    ap.nq = c.n_q_heads;
    ap.nkv = c.n_kv_heads;
    ap.splits = splits;
    ap.chunk = chunk;
    ap.rows_kv = cc->s_kv / d;
    ap.rows_kind = cc->s_kind / d;
    ap.rows_layer = cc->s_layer / d;
    ap.rows_req = cc->s_req / d;
    ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    ap.status = h->status;
    ap.causal = ingest ? 1 : 0;
    const int attn_blocks = splits * c.n_kv_heads * B;

    capture_x(h, 0, M, st);
    for (int l = 0; l < c.n_layers; ++l) {
        if (!fold) {
            Timed t(h, TK_RMSNORM, st);
            launch_rmsnorm<bf>((const bf*)h->x, (const bf*)h->w.g_in[l], (bf*)h->h, M, H, (float)c.rms_eps, M, 0, 0, st,
                               trace_small(h, TK_RMSNORM, M));
            h->launches += 1;
            capture_stage(h, h->cap_h, h->h, l, M, H, st);
        }
        {   // QKV + RoPE; block K/V to cache scratch rows [len, len + gamma)
            GemmParams p;
            std::memset(&p, 0, sizeof(p));
            p.ta[0] = h->tm_wq[l];
            p.ta[1] = h->tm_wk[l];
            p.ta[2] = h->tm_wv[l];
            p.amat[0].rows = Nq;
            p.amat[1].rows = Nkv;
            p.amat[2].rows = Nkv;
            p.n_amat = 3;
            p.tb[0] = fold ? tm_x : tm_h;
            if (fold) fold_in(h, p, h->w.g_in[l], l == 0 ? 1 : nH);   // layer 0: the embedding's row sums
            if (fold && h->cap_h) {   // diagnostic: the normaliser also writes the rows it normalised
                p.norm_out = (bf*)h->cap_h + (size_t)l * M * H;
                p.norm_out_ld = H;
            }
            p.kb_per_b = cdiv(H, 64);
            p.M = M;
            p.K = H;
            p.epi = EPI_QKV;
            p.out = h->q;
            p.ldo = Nq;
            p.d = d;
            p.gamma = gamma;
            p.cap = cc->capacity;
            p.layer = l;
            p.batch = B;
            p.len = cc->len;
            p.req_ok = h->req_ok;
            p.rope = h->rope;
            p.slab = (bf*)cc->slab;
            p.s_req = cc->s_req;
            p.s_layer = cc->s_layer;
            p.s_kind = cc->s_kind;
            p.s_kv = cc->s_kv;
            Timed t(h, TK_GEMM_QKV, st);
            int r = run_gemm(h, p, nt, st, TK_GEMM_QKV);
            if (r) return r;
        }
        capture_stage(h, h->cap_q, h->q, l, M, Nq, st);
        if (ingest && l == c.n_layers - 1) break;   // the last layer's K/V are written
        ap.layer = l;
        // attention trace: 8 stamps per CTA (attn.cuh), past the wait at 1, merge done at 7
        ap.trace = trace_slot(h, TK_ATTENTION, attn_blocks, 8, 1, 7);
        {
            Timed t(h, TK_ATTENTION, st);
            int e = launch_attention(ap, d, B, st, &h->launches);
            if (e) return DFLASH_CUDA;
        }
        capture_stage(h, h->cap_o, h->o, l, M, Nq, st);
        {   // O-proj + residual
            GemmParams p;
            std::memset(&p, 0, sizeof(p));
            p.ta[0] = h->tm_wo[l];
            p.amat[0].rows = H;
            p.n_amat = 1;
            p.tb[0] = tm_o;
            p.kb_per_b = cdiv(Nq, 64);
            p.M = M;
            p.K = Nq;
            p.epi = EPI_RESID;
            p.out = h->x;
            p.ldo = H;
            if (fold) {
                p.ssq_out = h->ssq;
                p.ssq_ld = ssq_ld;
            }
            Timed t(h, TK_GEMM_O, st);
            // The attention holds attn_blocks SMs until it ends: the O-projection's
            // CTAs that land there (the highest block indices: CTAs are dispatched in
            // order) start when it ends, without the weight stages the others loaded
            // during it, so they take g_o_late_deficit fewer k-block units.  (Optional:
            // run the O-projection on the other SMs only, prefetching into L2.)
            const bool beside = g_o_beside_attention && attn_blocks * 4 <= h->num_sms * 3;
            if (!beside && attn_blocks < h->num_sms) {
                p.late_from = h->num_sms - attn_blocks;
                p.late_deficit = g_o_late_deficit;
            }
            int r = beside ? run_gemm(h, p, nt, st, TK_GEMM_O, h->num_sms - attn_blocks, 64)
                           : run_gemm(h, p, nt, st, TK_GEMM_O);
            if (r) return r;
        }
        capture_stage(h, h->cap_xm, h->x, l, M, H, st);
        if (!fold) {
            Timed t(h, TK_RMSNORM, st);
            launch_rmsnorm<bf>((const bf*)h->x, (const bf*)h->w.g_post[l], (bf*)h->h, M, H, (float)c.rms_eps, M, 0, 0, st,
                               trace_small(h, TK_RMSNORM, M));
            h->launches += 1;
            capture_stage(h, h->cap_h2, h->h, l, M, H, st);
        }
        {   // gate/up + SwiGLU
            GemmParams p;
            std::memset(&p, 0, sizeof(p));
            p.ta[0] = h->tm_wg[l];
            p.ta[1] = h->tm_wu[l];
            p.n_amat = 2;
            p.swiglu = 1;
            p.n_tiles = I / 64;
            p.tb[0] = fold ? tm_x : tm_h;
            if (fold) fold_in(h, p, h->w.g_post[l], nH);
            if (fold && h->cap_h2) {
                p.norm_out = (bf*)h->cap_h2 + (size_t)l * M * H;
                p.norm_out_ld = H;
            }
            p.kb_per_b = cdiv(H, 64);
            p.M = M;
            p.K = H;
            p.epi = EPI_SWIGLU;
            p.out = h->act;
            p.ldo = I;
            Timed t(h, TK_GEMM_SWIGLU, st);
            int r = run_gemm(h, p, nt, st, TK_GEMM_SWIGLU);
            if (r) return r;
        }
        capture_stage(h, h->cap_act, h->act, l, M, I, st);
        {   // down + residual
            GemmParams p;
            std::memset(&p, 0, sizeof(p));
            p.ta[0] = h->tm_wd[l];
            p.amat[0].rows = H;
            p.n_amat = 1;
            p.tb[0] = tm_act;
            p.kb_per_b = cdiv(I, 64);
            p.M = M;
            p.K = I;
            p.epi = EPI_RESID;
            p.out = h->x;
            p.ldo = H;
            if (fold) {
                p.ssq_out = h->ssq;
                p.ssq_ld = ssq_ld;
            }
            Timed t(h, TK_GEMM_DOWN, st);
            int r = run_gemm(h, p, nt, st, TK_GEMM_DOWN);
            if (r) return r;
        }
        capture_x(h, l + 1, M, st);
    }
    return DFLASH_OK;
}

static int draft_bf16(dflash_handle* h, dflash_cache* cc, int gamma, int32_t* drafts, float* logits, float* margin,
                      cudaStream_t st) {
    const dflash_config& c = h->cfg;
    const int B = cc->batch, M = B * gamma, Mlm = B * (gamma - 1);
    const int H = c.hidden;
    typedef __nv_bfloat16 bf;
    const int nt = pick_nt(M);
    const bool fold = fold_norms(h, M);
    const int nH = cdiv(H, 128);
    int r = layers_bf16(h, cc, gamma, false, st);
    if (r) return r;
    CUtensorMap tm_hf, tm_x;
    if (!act_map(&tm_hf, h->hf, Mlm, H, H, pick_nt(Mlm)) || !act_map(&tm_x, h->x, M, H, H, nt)) return DFLASH_CUDA;
    // The LM head streams the largest weight at the HBM roofline, where the folded
    // normaliser's per-stage work measured slower than one final-norm kernel: the
    // final norm stays a kernel of its own unless g_fold_head is set.
    const bool fold_head = fold && g_fold_head;
    (void)nt;
    if (!fold_head) {
        Timed t(h, TK_RMSNORM, st);
        launch_rmsnorm<bf>((const bf*)h->x, (const bf*)h->w.g_final, (bf*)h->hf, Mlm, H, (float)c.rms_eps, gamma - 1,
                           gamma, 1, st, trace_small(h, TK_RMSNORM, Mlm));
        h->launches += 1;
        capture_hf(h, Mlm, st);
    } else if (h->cap_hf) {
        // diagnostic capture only: the folded head never materialises hf
        launch_rmsnorm<bf>((const bf*)h->x, (const bf*)h->w.g_final, (bf*)h->cap_hf, Mlm, H, (float)c.rms_eps,
                           gamma - 1, gamma, 1, st);
    }
    {   // shared LM head + per-tile top-2 (folded: over every block row, the final
        // norm applied to x on the fly; the anchor rows' results are not used)
        GemmParams p;
        std::memset(&p, 0, sizeof(p));
        p.ta[0] = h->tm_lm;
        p.amat[0].rows = c.vocab;
        p.n_amat = 1;
        p.tb[0] = fold_head ? tm_x : tm_hf;
        p.kb_per_b = cdiv(H, 64);
        p.M = fold_head ? M : Mlm;
        p.K = H;
        p.epi = EPI_LMHEAD;
        p.vocab = c.vocab;
        p.logits = logits;
        p.records = h->rec;
        if (fold_head) {
            fold_in(h, p, h->w.g_final, nH);
            p.lm_gamma = gamma;
        }
        Timed t(h, TK_GEMM_LMHEAD, st);
        int r = run_gemm(h, p, fold_head ? nt : pick_nt(Mlm), st, TK_GEMM_LMHEAD);
        if (r) return r;
    }
    Timed t(h, TK_LM_REDUCE, st);
    launch_lm_reduce(h->rec, cdiv(c.vocab, 128), Mlm, gamma - 1, h->req_ok, drafts, margin, st,
                     trace_small(h, TK_LM_REDUCE, Mlm), fold_head ? 1 : 0);
    h->launches += 1;
    return DFLASH_OK;
}

static int draft_f32(dflash_handle* h, dflash_cache* cc, int gamma, int32_t* drafts, float* logits, float* margin,
                     cudaStream_t st) {
    const dflash_config& c = h->cfg;
    const int B = cc->batch, M = B * gamma, Mlm = B * (gamma - 1);
    const int H = c.hidden, d = c.head_dim, Nq = c.n_q_heads * d, Nkv = c.n_kv_heads * d, I = c.intermediate;
    const int ldq = Nq + 2 * Nkv;
    Timed t(h, TK_SIMT_F32, st);
    float *x = (float*)h->x, *hh = (float*)h->h, *q = (float*)h->q, *o = (float*)h->o, *act = (float*)h->act;
    XSegs xh{}, xo{}, xa{}, xf{};
    xh.ptr[0] = hh; xh.stride = H; xh.width = H;
    xo.ptr[0] = o; xo.stride = Nq; xo.width = Nq;
    xa.ptr[0] = act; xa.stride = I; xa.width = I;
    xf.ptr[0] = (float*)h->hf; xf.stride = H; xf.width = H;
    capture_x(h, 0, M, st);
    for (int l = 0; l < c.n_layers; ++l) {
        launch_rmsnorm<float>(x, (const float*)h->w.g_in[l], hh, M, H, (float)c.rms_eps, M, 0, 0, st);
        launch_gemm_f32(xh, (const float*)h->w.wq[l], h->y32, M, Nq, H, ldq, 0, st);
        launch_gemm_f32(xh, (const float*)h->w.wk[l], h->y32, M, Nkv, H, ldq, Nq, st);
        launch_gemm_f32(xh, (const float*)h->w.wv[l], h->y32, M, Nkv, H, ldq, Nq + Nkv, st);
        launch_epi_qkv_f32(h->y32, M, Nq, Nkv, d, gamma, cc->len, h->req_ok, h->rope, q, (float*)cc->slab, cc->s_req,
                           cc->s_layer, cc->s_kind, cc->s_kv, l, st);
        int e = launch_attn_f32(q, (const float*)cc->slab, cc->len, h->req_ok, o, B, gamma, c.n_q_heads,
                                c.n_q_heads / c.n_kv_heads, d, cc->s_req, cc->s_layer, cc->s_kind, cc->s_kv, l,
                                cc->capacity, st);
        if (e) return DFLASH_CUDA;
        launch_gemm_f32(xo, (const float*)h->w.wo[l], h->y32, M, H, Nq, H, 0, st);
        launch_resid_f32(x, h->y32, (long long)M * H, st);
        launch_rmsnorm<float>(x, (const float*)h->w.g_post[l], hh, M, H, (float)c.rms_eps, M, 0, 0, st);
        launch_gemm_f32(xh, (const float*)h->w.w_gate[l], h->y32, M, I, H, 2 * I, 0, st);
        launch_gemm_f32(xh, (const float*)h->w.w_up[l], h->y32, M, I, H, 2 * I, I, st);
        launch_swiglu_f32(h->y32, act, M, I, st);
        launch_gemm_f32(xa, (const float*)h->w.w_down[l], h->y32, M, H, I, H, 0, st);
        launch_resid_f32(x, h->y32, (long long)M * H, st);
        h->launches += 14;
        capture_x(h, l + 1, M, st);
    }
    launch_rmsnorm<float>(x, (const float*)h->w.g_final, (float*)h->hf, Mlm, H, (float)c.rms_eps, gamma - 1, gamma, 1,
                          st);
    capture_hf(h, Mlm, st);
    float* lg = logits ? logits : h->lgs;
    launch_gemm_f32(xf, (const float*)h->w.lm_head, lg, Mlm, c.vocab, H, c.vocab, 0, st);
    launch_top2_rows(lg, Mlm, c.vocab, gamma - 1, h->req_ok, drafts, margin, st);
    h->launches += 3;
    return DFLASH_OK;
}

int dflash_draft_block(dflash_handle* h, dflash_cache* cc, const int32_t* anchor, int gamma, int32_t* drafts,
                       float* logits_opt, float* margin_opt, dflash_stream stream) {
    if (!h || !cc || cc->h != h || !anchor || gamma < 1 || gamma > h->cfg.max_gamma) return DFLASH_INVALID_ARG;
    if (gamma > 1 && !drafts) return DFLASH_INVALID_ARG;
    const dflash_config& c = h->cfg;
    cudaStream_t st = S(stream);
    {
    Timed t(h, TK_EMBED, st);
    if (c.dtype == DFLASH_BF16)
        launch_embed<__nv_bfloat16>((const __nv_bfloat16*)h->w.embed, anchor, c.mask_id, cc->batch, gamma, c.hidden,
                                    c.vocab, cc->len, cc->committed, cc->capacity, (__nv_bfloat16*)h->x, h->req_ok,
                                    cc->status, st, trace_small(h, TK_EMBED, cc->batch * gamma),
                                    gamma > 1 && fold_norms(h, cc->batch * gamma) ? h->ssq : nullptr);
    else
        launch_embed<float>((const float*)h->w.embed, anchor, c.mask_id, cc->batch, gamma, c.hidden, c.vocab, cc->len,
                            cc->committed, cc->capacity, (float*)h->x, h->req_ok, cc->status, st);
    h->launches += 1;
    }
    if (gamma == 1) return cuda_status(cudaGetLastError());
    int r = c.dtype == DFLASH_BF16 ? draft_bf16(h, cc, gamma, drafts, logits_opt, margin_opt, st)
                                   : draft_f32(h, cc, gamma, drafts, logits_opt, margin_opt, st);
    if (r) return r;
    return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Input-fusion ablation: the context rows through the draft layers
// ---------------------------------------------------------------------------
int dflash_ingest_fused_input(dflash_handle* h, dflash_cache* cc, const void* ctx, int rows,
                              const int32_t* row_count, dflash_stream stream) {
    if (!h || !cc || cc->h != h || !ctx || rows < 1 || rows > h->cfg.max_gamma) return DFLASH_INVALID_ARG;
    const dflash_config& c = h->cfg;
    if (c.dtype != DFLASH_BF16) return DFLASH_UNSUPPORTED;
    if (!aligned16(ctx)) return DFLASH_INVALID_ARG;
    cudaStream_t st = S(stream);
    const int B = cc->batch, M = B * rows;
    launch_ingest_begin((const __nv_bfloat16*)ctx, B, rows, c.hidden, cc->len, cc->capacity, (__nv_bfloat16*)h->x,
                        h->req_ok, cc->status, fold_norms(h, M) ? h->ssq : nullptr, st);
    h->launches += 1;
    int r = layers_bf16(h, cc, rows, true, st);
    if (r) return r;
    launch_ingest_end(row_count, rows, B, h->req_ok, cc->len, cc->status, st);
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// a8: accept
// ---------------------------------------------------------------------------
int dflash_accept(dflash_handle* h, dflash_cache* cc, const int32_t* drafts, const int32_t* target, int gamma,
                  int32_t* accept_len, int32_t* next_anchor, dflash_stream stream) {
    if (!h || !cc || cc->h != h || !target || !accept_len || !next_anchor || gamma < 1 || gamma > h->cfg.max_gamma)
        return DFLASH_INVALID_ARG;
    if (gamma > 1 && !drafts) return DFLASH_INVALID_ARG;
    Timed t(h, TK_ACCEPT, st_of(stream));
    launch_accept(drafts ? drafts : target, target, cc->batch, gamma, h->cfg.vocab, cc->len, cc->committed, accept_len,
                  next_anchor, cc->status, S(stream), trace_small(h, TK_ACCEPT, cdiv(cc->batch * 32, 128)));
    h->launches += 1;
    return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// Diagnostics
// ---------------------------------------------------------------------------
const char* dflash_diag_arch(void) { return "sm_100a"; }

int dflash_diag_partition(int64_t units, int kb, int ctas, int64_t tile, int* first_cta, int* n_contrib) {
    if (units <= 0 || kb <= 0 || units % kb || ctas <= 0 || ctas > units || tile < 0 || tile * kb >= units || !first_cta ||
        !n_contrib)
        return DFLASH_INVALID_ARG;
    *first_cta = sk_first_cta(tile, kb, units, ctas);
    *n_contrib = sk_n_contrib(tile, kb, units, ctas);
    return DFLASH_OK;
}

int dflash_diag_gemm_scratch_bytes(int M, int N, int K, size_t* bytes) {
    if (!bytes || M < 1 || M > 4096 || N < 1 || K < 8 || K % 8) return DFLASH_INVALID_ARG;
    const int nt = pick_nt(M);
    const size_t counters = (size_t)cdiv(N, 128) * cdiv(M, nt) * 4;
    *bytes = al(counters, 256) + gemm_partial_bytes(kMaxCtas, nt);
    return DFLASH_OK;
}

int dflash_diag_gemm_bf16_traced(const void* X, const void* W, float* Y, int M, int N, int K, void* scratch,
                                 size_t scratch_bytes, int grid, int64_t* trace, dflash_stream stream);
int dflash_diag_gemm_bf16(const void* X, const void* W, float* Y, int M, int N, int K, void* scratch,
                          size_t scratch_bytes, int grid, dflash_stream stream) {
    return dflash_diag_gemm_bf16_traced(X, W, Y, M, N, K, scratch, scratch_bytes, grid, nullptr, stream);
}

int dflash_diag_gemm_bf16_traced(const void* X, const void* W, float* Y, int M, int N, int K, void* scratch,
                                 size_t scratch_bytes, int grid, int64_t* trace, dflash_stream stream) {
    size_t need = 0;
    if (dflash_diag_gemm_scratch_bytes(M, N, K, &need) != DFLASH_OK) return DFLASH_INVALID_ARG;
    if (!X || !W || !Y || !scratch || ((uintptr_t)scratch & 255)) return DFLASH_INVALID_ARG;
    if (scratch_bytes < need) return DFLASH_WORKSPACE;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return DFLASH_CUDA;
    const int nt = pick_nt(M);
    GemmParams p;
    std::memset(&p, 0, sizeof(p));
    if (!encode_bf16_2d(&p.ta[0], W, K, N, K, 128) || !encode_bf16_2d(&p.tb[0], X, K, M, K, nt))
        return DFLASH_INVALID_ARG;
    p.amat[0].rows = N;
    p.n_amat = 1;
    p.kb_per_b = cdiv(K, 64);
    p.M = M;
    p.K = K;
    p.epi = EPI_F32;
    p.out = Y;
    p.ldo = N;
    const size_t counters = al((size_t)cdiv(N, 128) * cdiv(M, nt) * 4, 256);
    p.counters = (int*)scratch;
    p.partial = (float*)((uint8_t*)scratch + counters);
    p.status = nullptr;
    p.trace = (long long*)trace;
    p.last_arriver = gemm_last_arriver();
    p.ctas = grid > 0 ? std::min(grid, kMaxCtas) : 0;
    int e = launch_gemm_tc(p, nt, std::min(sms, kMaxCtas), S(stream));
    return e == 0 ? DFLASH_OK : DFLASH_CUDA;
}

int dflash_diag_synth_target(const int32_t* drafts, const int32_t* a_plan, const int32_t* rand_tokens, int batch,
                             int gamma, int vocab, int32_t* target, dflash_stream stream) {
    if (!a_plan || !rand_tokens || !target || batch < 1 || gamma < 1 || vocab < 2) return DFLASH_INVALID_ARG;
    if (gamma > 1 && !drafts) return DFLASH_INVALID_ARG;
    launch_synth_target(drafts ? drafts : a_plan, a_plan, rand_tokens, batch, gamma, vocab, target, S(stream));
    return cuda_status(cudaGetLastError());
}

int dflash_diag_timing_enable(dflash_handle* h, int max_launches) {
    if (!h || max_launches < 1 || max_launches > (1 << 20)) return DFLASH_INVALID_ARG;
    for (auto e : h->ev) cudaEventDestroy(e);
    h->ev.assign(2 * (size_t)max_launches, nullptr);
    h->ev_kind.assign(max_launches, -1);
    for (auto& e : h->ev)
        if (cudaEventCreate(&e) != cudaSuccess) return DFLASH_CUDA;
    h->ev_used = 0;
    h->timing = true;
    return DFLASH_OK;
}

int dflash_diag_timing_read(dflash_handle* h, dflash_stream stream, int* kinds, float* ms, int max_entries,
                            int* n_entries) {
    if (!h || !kinds || !ms || !n_entries || max_entries < 0) return DFLASH_INVALID_ARG;
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return DFLASH_CUDA;
    const int n = std::min(h->ev_used / 2, max_entries);
    for (int i = 0; i < n; ++i) {
        float t = 0.f;
        if (cudaEventElapsedTime(&t, h->ev[2 * i], h->ev[2 * i + 1]) != cudaSuccess) return DFLASH_CUDA;
        kinds[i] = h->ev_kind[i];
        ms[i] = t;
    }
    *n_entries = n;
    h->ev_used = 0;
    return DFLASH_OK;
}

int dflash_diag_timing_disable(dflash_handle* h) {
    if (!h) return DFLASH_INVALID_ARG;
    h->timing = false;
    for (auto e : h->ev) cudaEventDestroy(e);
    h->ev.clear();
    h->ev_kind.clear();
    h->ev_used = 0;
    return DFLASH_OK;
}

int dflash_diag_attention_traced(dflash_handle* h, dflash_cache* cc, const void* q, void* out, int layer, int gamma,
                                 int64_t* trace, int* splits_out, dflash_stream stream);
int dflash_diag_attention(dflash_handle* h, dflash_cache* cc, const void* q, void* out, int layer, int gamma,
                          dflash_stream stream) {
    return dflash_diag_attention_traced(h, cc, q, out, layer, gamma, nullptr, nullptr, stream);
}

int dflash_diag_attention_traced(dflash_handle* h, dflash_cache* cc, const void* q, void* out, int layer, int gamma,
                                 int64_t* trace, int* splits_out, dflash_stream stream) {
    if (!h || !cc || cc->h != h || !q || !out || layer < 0 || layer >= h->cfg.n_layers || gamma < 1 ||
        gamma > h->cfg.max_gamma || h->cfg.dtype != DFLASH_BF16)
        return DFLASH_INVALID_ARG;
    const dflash_config& c = h->cfg;
    const int d = c.head_dim;
    // all requests are attended (req_ok = 1): the caller keeps len + gamma <= capacity
    std::vector<int> ones(cc->batch, 1);
    if (cudaMemcpyAsync(h->req_ok, ones.data(), cc->batch * sizeof(int), cudaMemcpyHostToDevice, S(stream)) !=
        cudaSuccess)
        return DFLASH_CUDA;
    AttnParams ap;
    std::memset(&ap, 0, sizeof(ap));
    int splits, chunk;
    attn_plan(cc->batch, c.n_kv_heads, cc->capacity, h->num_sms, attn_max_cluster(d), splits, chunk);
    ap.tmap = cc->tm_slab;
    if ((uintptr_t)q & 15) return DFLASH_INVALID_ARG;   // q rows are read as 16-byte vectors
    ap.q = (const __nv_bfloat16*)q;
    ap.out = (__nv_bfloat16*)out;
    ap.len = cc->len;
    ap.req_ok = h->req_ok;
    ap.gamma = gamma;
    ap.G = c.n_q_heads / c.n_kv_heads;
    ap.nq = c.n_q_heads;
    ap.nkv = c.n_kv_heads;
    ap.layer = layer;
    ap.splits = splits;
    ap.chunk = chunk;
    ap.rows_kv = cc->s_kv / d;
    ap.rows_kind = cc->s_kind / d;
    ap.rows_layer = cc->s_layer / d;
    ap.rows_req = cc->s_req / d;
    ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)d));
    ap.status = h->status;
    ap.trace = (long long*)trace;
    if (splits_out) *splits_out = splits;
    const int e = launch_attention(ap, d, cc->batch, S(stream), &h->launches);
    if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return DFLASH_CUDA;
    return e == 0 ? DFLASH_OK : DFLASH_CUDA;
}

int dflash_diag_step_trace(dflash_handle* h, int64_t* buf, int64_t words) {
    if (!h || (buf && words <= 0)) return DFLASH_INVALID_ARG;
    h->tr_buf = (long long*)buf;
    h->tr_cap = buf ? words : 0;
    h->tr_used = 0;
    h->tr_recs.clear();
    return DFLASH_OK;
}

int dflash_diag_step_trace_records(const dflash_handle* h, int32_t* recs, int64_t* offsets, int max_records,
                                   int* n_records) {
    if (!h || !n_records || max_records < 0 || (max_records > 0 && (!recs || !offsets))) return DFLASH_INVALID_ARG;
    const int n = std::min((int)h->tr_recs.size(), max_records);
    for (int i = 0; i < n; ++i) {
        const auto& r = h->tr_recs[i];
        recs[5 * i + 0] = r.kind;
        recs[5 * i + 1] = r.blocks;
        recs[5 * i + 2] = r.words;
        recs[5 * i + 3] = r.wait_idx;
        recs[5 * i + 4] = r.exit_idx;
        offsets[i] = r.offset;
    }
    *n_records = (int)h->tr_recs.size();
    return DFLASH_OK;
}

int dflash_diag_draft_capture_stages(dflash_handle* h, void* h_in, void* q, void* o, void* x_mid, void* h2,
                                     void* act) {
    if (!h) return DFLASH_INVALID_ARG;
    h->cap_h = h_in;
    h->cap_q = q;
    h->cap_o = o;
    h->cap_xm = x_mid;
    h->cap_h2 = h2;
    h->cap_act = act;
    return DFLASH_OK;
}

int dflash_diag_draft_capture(dflash_handle* h, void* x_layers, void* hf) {
    if (!h) return DFLASH_INVALID_ARG;
    h->cap_x = x_layers;
    h->cap_hf = hf;
    return DFLASH_OK;
}

int dflash_diag_wait_selftest(dflash_handle* h, int32_t* out, dflash_stream stream) {
    if (!h || !out) return DFLASH_INVALID_ARG;
    const int e = launch_wait_selftest(h->status, out, S(stream));
    h->launches += 1;
    return e == 0 ? DFLASH_OK : DFLASH_CUDA;
}

int dflash_diag_set_gemm_prefetch(int tiles) {
    if (tiles < 0 || tiles > 256) return DFLASH_INVALID_ARG;
    set_gemm_l2_prefetch(tiles);
    return DFLASH_OK;
}

int dflash_diag_gemm_prefetch(void) { return gemm_l2_prefetch(); }

int dflash_diag_set_gemm_pre_stages(int stages) {
    if (stages < 0 || stages > 64) return DFLASH_INVALID_ARG;
    set_gemm_pre_stages(stages);
    return DFLASH_OK;
}

int dflash_diag_set_gemm_max_cluster(int max_cluster) {
    if (max_cluster < 0 || max_cluster > 4) return DFLASH_INVALID_ARG;
    set_gemm_max_cluster(max_cluster);
    return DFLASH_OK;
}

int dflash_diag_gemm_max_active_clusters(int cluster_size) {
    if (cluster_size < 2 || cluster_size > 8) return 0;
    return gemm_max_active_clusters(cluster_size);
}

int dflash_diag_set_split_finisher(int last_arriver) {
    set_gemm_last_arriver(last_arriver);
    return DFLASH_OK;
}

int dflash_diag_set_gemm_tail(int ctas, int units) {
    if (ctas < 0 || ctas > 64 || units < 0 || units > 64) return DFLASH_INVALID_ARG;
    g_tail_ctas = ctas;
    g_tail_deficit = units;
    return DFLASH_OK;
}

int dflash_diag_set_o_late_deficit(int units) {
    if (units < 0 || units > 64) return DFLASH_INVALID_ARG;
    g_o_late_deficit = units;
    return DFLASH_OK;
}

int dflash_diag_set_o_beside_attention(int on) {
    g_o_beside_attention = on != 0;
    return DFLASH_OK;
}

int dflash_diag_set_inject_partition(int whole_tiles) {
    g_inject_whole = whole_tiles != 0;
    return DFLASH_OK;
}

int dflash_diag_set_norm_fold(int on) {
    g_fold = on != 0;
    g_fold_head = on > 1;
    return DFLASH_OK;
}

int dflash_diag_set_launch_mode(int programmatic) {
    set_pdl(programmatic != 0);
    return DFLASH_OK;
}

const char* dflash_diag_timed_name(int kind) { return (kind >= 0 && kind < TK_COUNT) ? kTimedNames[kind] : "?"; }

}  // extern "C"
