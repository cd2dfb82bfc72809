// Memory-bound and latency-bound kernels of the draft step, and the fp32
// (SIMT) path used when the storage type is fp32.
#include "kernels.cuh"

namespace df {

// ---------------------------------------------------------------------------
// a3: embedding of [anchor, mask, ..., mask] + per-request validation.
// One CTA per block row m = b*gamma + j.  A request is drafted only when
// len == committed, len + gamma <= capacity and the anchor is a valid token;
// otherwise its rows are zero, req_ok[b] = 0 and the first error is recorded.
// ---------------------------------------------------------------------------
// With ssq non-null the block also writes its row's sum of squares ssq[m] (the
// statistic of the first layer's input RMSNorm, which the QKV GEMM applies).
template <typename T>
__global__ void k_embed(const T* __restrict__ embed, const int* __restrict__ anchor, int mask_id, int gamma, int H,
                        int V, const int* __restrict__ len, const int* __restrict__ committed, int cap,
                        T* __restrict__ x, int* __restrict__ req_ok, int* __restrict__ status, float* __restrict__ ssq,
                        long long* tr) {
    griddep_wait();
    griddep_launch();
    trace_mark(tr, 0);
    const int m = blockIdx.x, b = m / gamma, j = m % gamma;
    const int L0 = len[b], a = anchor[b];
    int err = 0;
    if (L0 != committed[b]) err = DFLASH_STATE;
    else if (L0 + gamma > cap) err = DFLASH_CAPACITY;
    else if (a < 0 || a >= V) err = DFLASH_TOKEN_RANGE;
    if (j == 0 && threadIdx.x == 0) {
        req_ok[b] = err == 0;
        if (err) set_error(status, err);
    }
    T* dst = x + (size_t)m * H;
    if (err) {
        for (int i = threadIdx.x; i < H; i += blockDim.x) stf(dst + i, 0.0f);
        if (ssq && threadIdx.x == 0) ssq[m] = 0.f;
        trace_mark(tr, 1);
        return;
    }
    const int tok = (j == 0) ? a : mask_id;
    const T* src = embed + (size_t)tok * H;
    constexpr int VEC = 16 / sizeof(T);
    float ss = 0.f;
    for (int i = threadIdx.x * VEC; i < H; i += blockDim.x * VEC) {
        const uint4 u = *reinterpret_cast<const uint4*>(src + i);
        *reinterpret_cast<uint4*>(dst + i) = u;
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
            const float v = ldf(e + k);
            ss += v * v;
        }
    }
    if (ssq) {   // fixed order: each thread's chunks, the warp butterfly, then the warps in order
        __shared__ float red[32];
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        if (threadIdx.x == 0) {
            float t = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
            ssq[m] = t;
        }
    }
    trace_mark(tr, 1);
}

// ---------------------------------------------------------------------------
// Input fusion, first step: the context rows become the block's input hidden
// states.  One CTA per row m = b * rows + j: x[m] = ctx[m], ssq[m] = its sum of
// squares (when ssq is set), req_ok[b] = (len[b] + rows <= capacity); a request
// that does not fit records DFLASH_CAPACITY and is skipped.
// ---------------------------------------------------------------------------
__global__ void k_ingest_begin(const __nv_bfloat16* __restrict__ ctx, int rows, int H, const int* __restrict__ len,
                               int cap, __nv_bfloat16* __restrict__ x, int* __restrict__ req_ok,
                               int* __restrict__ status, float* __restrict__ ssq) {
    griddep_wait();
    griddep_launch();
    const int m = blockIdx.x, b = m / rows, j = m % rows;
    const bool fits = len[b] >= 0 && len[b] + rows <= cap;
    if (j == 0 && threadIdx.x == 0) {
        req_ok[b] = fits ? 1 : 0;
        if (!fits) set_error(status, DFLASH_CAPACITY);
    }
    const __nv_bfloat16* src = ctx + (size_t)m * H;
    __nv_bfloat16* dst = x + (size_t)m * H;
    float ss = 0.f;
    for (int i = threadIdx.x * 8; i < H; i += blockDim.x * 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(src + i);
        *reinterpret_cast<uint4*>(dst + i) = u;
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&u);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float v = bf2f(e[k]);
            ss += v * v;
        }
    }
    if (ssq) {   // the same fixed order as the embedding's
        __shared__ float red[32];
        for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
        __syncthreads();
        if (threadIdx.x == 0) {
            float t = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
            ssq[m] = t;
        }
    }
}

// Input fusion, last step: append the ingested rows, len[b] += row_count[b]
// (all `rows` when row_count is null) for every request that was processed.
__global__ void k_ingest_end(const int* __restrict__ row_count, int rows, int B, const int* __restrict__ req_ok,
                             int* __restrict__ len, int* __restrict__ status) {
    griddep_wait();
    griddep_launch();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B || !req_ok[b]) return;
    const int n = row_count ? row_count[b] : rows;
    if (n < 0 || n > rows) {
        set_error(status, DFLASH_INVALID_ARG);
        return;
    }
    len[b] += n;
}

// ---------------------------------------------------------------------------
// RMSNorm: y[o] = R(x[in(o)] / sqrt(mean(x^2) + eps) * g), fp32 math.
// in(o) = (o / grp) * gstride + goff + o % grp selects the rows (grp = rows,
// gstride = 0, goff = 0 is the identity; grp = gamma-1, gstride = gamma,
// goff = 1 keeps the mask positions of every block).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void k_rmsnorm(const T* __restrict__ x, const T* __restrict__ g, T* __restrict__ y, int H, float eps,
                          int grp, int gstride, int goff, long long* tr) {
    constexpr int VEC = 16 / sizeof(T);          // elements per 16-byte access
    constexpr int KEEP = 4;                      // vectors of x and g a thread keeps in registers
    const int o = blockIdx.x;
    const int in = (o / grp) * gstride + goff + o % grp;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)in * H);
    const uint4* gr = reinterpret_cast<const uint4*>(g);
    uint4* yr = reinterpret_cast<uint4*>(y + (size_t)o * H);
    const int nv = H / VEC;
    // the gain is a weight: fetch it before waiting for the kernel that writes x
    uint4 gk[KEEP], xk[KEEP];
#pragma unroll
    for (int j = 0; j < KEEP; ++j) {
        const int i = threadIdx.x + j * blockDim.x;
        if (i < nv) gk[j] = gr[i];
    }
    griddep_wait();
    griddep_launch();
    trace_mark(tr, 0);
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < KEEP; ++j) {
        const int i = threadIdx.x + j * blockDim.x;
        if (i < nv) xk[j] = xr[i];
    }
#pragma unroll
    for (int j = 0; j < KEEP; ++j) {
        const int i = threadIdx.x + j * blockDim.x;
        if (i < nv) {
            const T* e = reinterpret_cast<const T*>(&xk[j]);
#pragma unroll
            for (int k = 0; k < VEC; ++k) {
                const float v = ldf(e + k);
                ss += v * v;
            }
        }
    }
    for (int i = threadIdx.x + KEEP * blockDim.x; i < nv; i += blockDim.x) {   // rows wider than the kept part
        const uint4 u = xr[i];
        const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
        for (int k = 0; k < VEC; ++k) {
            const float v = ldf(e + k);
            ss += v * v;
        }
    }
    __shared__ float red[32];
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
        for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    const float inv = 1.0f / sqrtf(red[0] / (float)H + eps);
    auto norm_store = [&](int i, const uint4& u, const uint4& gu) {
        const T* e = reinterpret_cast<const T*>(&u);
        const T* ge = reinterpret_cast<const T*>(&gu);
        uint4 out;
        T* oe = reinterpret_cast<T*>(&out);
#pragma unroll
        for (int k = 0; k < VEC; ++k) stf(oe + k, ldf(e + k) * inv * ldf(ge + k));
        yr[i] = out;
    };
#pragma unroll
    for (int j = 0; j < KEEP; ++j) {
        const int i = threadIdx.x + j * blockDim.x;
        if (i < nv) norm_store(i, xk[j], gk[j]);
    }
    for (int i = threadIdx.x + KEEP * blockDim.x; i < nv; i += blockDim.x) norm_store(i, xr[i], gr[i]);
    trace_mark(tr, 1);
}

// Top-2 merge with ties of the top value to the lower id.
DF_DEV void top2m(float& a1, int& ai, float& a2, float b1, int bi, float b2) {
    if (b1 > a1 || (b1 == a1 && bi < ai)) {
        a2 = fmaxf(a1, b2);
        a1 = b1;
        ai = bi;
    } else {
        a2 = fmaxf(a2, b1);
    }
}

// ---------------------------------------------------------------------------
// LM-head reduction (bf16 path): merge the per-vocab-tile top-2 records of
// every draft row.  One CTA per row m = b*(gamma-1) + j; the row's records are
// contiguous ([M][n_vt]), so the CTA reads them coalesced in one or two rounds.
// ---------------------------------------------------------------------------
constexpr int kLmReduceThreads = 512;

__global__ void __launch_bounds__(kLmReduceThreads) k_lm_reduce(const float4* __restrict__ rec, int n_vt, int M,
                                                                 int gm1, const int* __restrict__ req_ok,
                                                                 int* __restrict__ drafts, float* __restrict__ margin,
                                                                 int rec_blocks, long long* tr) {
    griddep_wait();
    griddep_launch();
    trace_mark(tr, 0);
    __shared__ float s1[kLmReduceThreads / 32], s2[kLmReduceThreads / 32];
    __shared__ int si[kLmReduceThreads / 32];
    const int m = blockIdx.x, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    // records of draft row m: row m, or with rec_blocks (records for whole blocks of
    // gamma = gm1 + 1 rows, anchor rows included) row m + m / gm1 + 1
    const float4* row = rec + (size_t)(rec_blocks ? m + m / gm1 + 1 : m) * n_vt;
    float a1 = -INFINITY, a2 = -INFINITY;
    int ai = 0x7fffffff;
    for (int t = threadIdx.x; t < n_vt; t += kLmReduceThreads) {
        const float4 r = row[t];
        top2m(a1, ai, a2, r.x, __float_as_int(r.y), r.z);
    }
    for (int off = 16; off > 0; off >>= 1) {
        const float b1 = __shfl_xor_sync(0xffffffffu, a1, off);
        const int bi = __shfl_xor_sync(0xffffffffu, ai, off);
        const float b2 = __shfl_xor_sync(0xffffffffu, a2, off);
        top2m(a1, ai, a2, b1, bi, b2);
    }
    if (lane == 0) { s1[w] = a1; si[w] = ai; s2[w] = a2; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 1; k < kLmReduceThreads / 32; ++k) top2m(a1, ai, a2, s1[k], si[k], s2[k]);
        const bool ok = req_ok[m / gm1] != 0;
        drafts[m] = ok ? ai : -1;
        if (margin) margin[m] = ok ? a1 - a2 : 0.f;
    }
    trace_mark(tr, 1);
}

// fp32 path: top-2 over the fp32 logits of each row; one CTA per row.
__global__ void k_top2_rows(const float* __restrict__ logits, int V, int gm1, const int* __restrict__ req_ok,
                            int* __restrict__ drafts, float* __restrict__ margin) {
    griddep_wait();
    griddep_launch();
    const int m = blockIdx.x;
    const float* row = logits + (size_t)m * V;
    float a1 = -INFINITY, a2 = -INFINITY;
    int ai = 0x7fffffff;
    for (int v = threadIdx.x; v < V; v += blockDim.x) top2m(a1, ai, a2, row[v], v, -INFINITY);
    for (int off = 16; off > 0; off >>= 1) {
        const float b1 = __shfl_xor_sync(0xffffffffu, a1, off);
        const int bi = __shfl_xor_sync(0xffffffffu, ai, off);
        const float b2 = __shfl_xor_sync(0xffffffffu, a2, off);
        top2m(a1, ai, a2, b1, bi, b2);
    }
    __shared__ float s1[32], s2[32];
    __shared__ int si[32];
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) { s1[w] = a1; si[w] = ai; s2[w] = a2; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int k = 1; k < (int)(blockDim.x >> 5); ++k) top2m(a1, ai, a2, s1[k], si[k], s2[k]);
        const bool ok = req_ok[m / gm1] != 0;
        drafts[m] = ok ? ai : -1;
        if (margin) margin[m] = ok ? a1 - a2 : 0.f;
    }
}

// ---------------------------------------------------------------------------
// a8: acceptance.  One warp per request: lane i compares draft i with target i;
// the accepted length is the number of leading matches.
// ---------------------------------------------------------------------------
__global__ void k_accept(const int* __restrict__ drafts, const int* __restrict__ target, int B, int gamma, int V,
                         int* __restrict__ len, int* __restrict__ committed, int* __restrict__ accept_len,
                         int* __restrict__ next_anchor, int* __restrict__ status, long long* tr) {
    griddep_wait();
    griddep_launch();
    trace_mark(tr, 0);
    const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (b >= B) return;
    const int tg = lane < gamma ? target[(size_t)b * gamma + lane] : 0;
    const bool bad = lane < gamma && (tg < 0 || tg >= V);
    const bool match = lane < gamma - 1 && drafts[(size_t)b * (gamma - 1) + lane] == tg;
    const unsigned bad_mask = __ballot_sync(0xffffffffu, bad);
    const unsigned match_mask = __ballot_sync(0xffffffffu, match);
    const int a = __ffs(~match_mask) - 1;       // leading matches; <= gamma-1
    const int tok_a = __shfl_sync(0xffffffffu, tg, a & 31);
    if (lane == 0) {
        if (bad_mask) {
            set_error(status, DFLASH_TOKEN_RANGE);
            accept_len[b] = -1;
            next_anchor[b] = -1;
        } else {
            accept_len[b] = a;
            next_anchor[b] = tok_a;
            const int c = committed[b] + a + 1;
            committed[b] = c;
            if (len[b] > c) len[b] = c;
        }
    }
    trace_mark(tr, 1);
}

// After an injection: len[b] += row_count[b] for every request that fitted.
__global__ void k_inject_finalize(const int* __restrict__ row_count, int B, int cap, int* __restrict__ len,
                                  int* __restrict__ status, long long* tr) {
    griddep_wait();
    griddep_launch();
    trace_mark(tr, 0);
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) {
        const int rc = row_count[b];
        if (rc < 0) set_error(status, DFLASH_INVALID_ARG);
        else if (len[b] + rc > cap) set_error(status, DFLASH_CAPACITY);
        else len[b] += rc;
    }
    trace_mark(tr, 1);
}

__global__ void k_set_len(const int* __restrict__ lens, int B, int cap, int* __restrict__ len,
                          int* __restrict__ committed, int* __restrict__ status, long long* tr) {
    griddep_wait();
    griddep_launch();
    trace_mark(tr, 0);
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) {
        const int v = lens[b];
        if (v < 0 || v > cap) {
            set_error(status, DFLASH_CAPACITY);
        } else {
            len[b] = v;
            committed[b] = v;
        }
    }
    trace_mark(tr, 1);
}

// Stand-in for the target's greedy verification (diagnostic).
__global__ void k_synth_target(const int* __restrict__ drafts, const int* __restrict__ a_plan,
                               const int* __restrict__ rnd, int B, int gamma, int V, int* __restrict__ target) {
    griddep_wait();
    griddep_launch();
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * gamma) return;
    const int b = idx / gamma, i = idx % gamma;
    const int a = a_plan[b];
    int t = rnd[idx];
    if (i < a) {
        t = drafts[(size_t)b * (gamma - 1) + i];
    } else if (i == a && i < gamma - 1) {
        const int d = drafts[(size_t)b * (gamma - 1) + i];
        if (t == d) t = (t + 1) % V;
    }
    target[idx] = t;
}

// Self-test of the bounded pipeline wait: one thread waits on an mbarrier that
// nothing ever arrives at; the wait gives up after its limit, records
// DFLASH_TIMEOUT in *status and the kernel returns normally.
__global__ void k_wait_selftest(int* status, int* out) {
    griddep_wait();
    griddep_launch();
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        const bool ok = mbar_wait(&bar, 0, (volatile int*)&abort_flag, status);
        *out = ok ? 1 : 0;
    }
}

// ---------------------------------------------------------------------------
// fp32 SIMT path
// ---------------------------------------------------------------------------

// Y[m, ycol0 + n] = sum_k X[m, k] W[n, k]; one warp per output, lanes over k.
// X is the concatenation along k of nseg segments, segment s at xs.ptr[s]
// with row stride xs.stride and xs.width columns.
__global__ void k_gemm_f32(XSegs xs, const float* __restrict__ W, float* __restrict__ Y, int M, int N, int K,
                           int ldy, int ycol0) {
    griddep_wait();
    griddep_launch();
    const long long wid = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= (long long)M * N) return;
    const int m = (int)(wid / N), n = (int)(wid % N);
    const float* wr = W + (size_t)n * K;
    float acc = 0.f;
    for (int k = lane; k < K; k += 32) {
        const int s = k / xs.width;
        const float xv = xs.ptr[s][(size_t)m * xs.stride + (k - s * xs.width)];
        acc += xv * wr[k];
    }
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) Y[(size_t)m * ldy + ycol0 + n] = acc;
}

// QKV epilogue: Y [M, Nq + 2*Nkv] = [q | k | v] -> q (RoPE), cache k (RoPE), v.
__global__ void k_epi_qkv_f32(const float* __restrict__ Y, int M, int Nq, int Nkv, int d, int gamma,
                              const int* __restrict__ len, const int* __restrict__ req_ok,
                              const float2* __restrict__ rope, float* __restrict__ q, float* __restrict__ slab,
                              long long s_req, long long s_layer, long long s_kind, long long s_kv, int layer) {
    griddep_wait();
    griddep_launch();
    const int ld = Nq + 2 * Nkv;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)M * ld) return;
    const int m = (int)(idx / ld), n = (int)(idx % ld);
    const int b = m / gamma, j = m % gamma;
    if (!req_ok[b]) return;
    const int pos = len[b] + j;
    const int sec = n < Nq ? 0 : (n < Nq + Nkv ? 1 : 2);
    const int lr = n - (sec == 0 ? 0 : (sec == 1 ? Nq : Nq + Nkv));
    const int i_in = lr % d, half = d / 2;
    float x = Y[idx];
    if (sec < 2) {
        const int pn = (i_in < half) ? n + half : n - half;
        const float pr = Y[(size_t)m * ld + pn];
        const float2 cs = rope[(size_t)pos * half + (i_in % half)];
        x = (i_in < half) ? (x * cs.x - pr * cs.y) : (x * cs.x + pr * cs.y);
    }
    if (sec == 0) {
        q[(size_t)m * Nq + lr] = x;
    } else {
        const int g = lr / d;
        slab[(size_t)b * s_req + (size_t)layer * s_layer + (size_t)(sec - 1) * s_kind + (size_t)g * s_kv +
             (size_t)pos * d + i_in] = x;
    }
}

// Inject epilogue for one layer: Y [rows, 2*Nkv] = [k | v] -> cache rows.
__global__ void k_epi_inject_f32(const float* __restrict__ Y, int rows, int Nkv, int d, const int* __restrict__ row_start,
                                 const int* __restrict__ row_count, int B, const int* __restrict__ len, int cap,
                                 const float2* __restrict__ rope, float* __restrict__ slab, long long s_req,
                                 long long s_layer, long long s_kind, long long s_kv, int layer) {
    griddep_wait();
    griddep_launch();
    const int ld = 2 * Nkv;
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)rows * ld) return;
    const int m = (int)(idx / ld), n = (int)(idx % ld);
    int b = -1, pos = -1;
    for (int bb = 0; bb < B; ++bb) {
        const int rs = row_start[bb], rc = row_count[bb];
        if (m >= rs && m < rs + rc) {
            if (len[bb] + rc <= cap) { b = bb; pos = len[bb] + (m - rs); }
            break;
        }
    }
    if (b < 0) return;
    const int kind = n < Nkv ? 0 : 1;
    const int lr = n - kind * Nkv;
    const int i_in = lr % d, half = d / 2;
    float x = Y[idx];
    if (kind == 0) {
        const int pn = (i_in < half) ? n + half : n - half;
        const float pr = Y[(size_t)m * ld + pn];
        const float2 cs = rope[(size_t)pos * half + (i_in % half)];
        x = (i_in < half) ? (x * cs.x - pr * cs.y) : (x * cs.x + pr * cs.y);
    }
    const int g = lr / d;
    slab[(size_t)b * s_req + (size_t)layer * s_layer + (size_t)kind * s_kind + (size_t)g * s_kv + (size_t)pos * d +
         i_in] = x;
}

// x += Y (fp32 residual), elementwise over [M, H].
__global__ void k_resid_f32(float* __restrict__ x, const float* __restrict__ Y, long long n) {
    griddep_wait();
    griddep_launch();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) x[i] += Y[i];
}

// act = silu(gate) * up with Y = [gate | up] of width 2I.
__global__ void k_swiglu_f32(const float* __restrict__ Y, float* __restrict__ act, int M, int I) {
    griddep_wait();
    griddep_launch();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)M * I) return;
    const int m = (int)(i / I), f = (int)(i % I);
    const float g = Y[(size_t)m * 2 * I + f], u = Y[(size_t)m * 2 * I + I + f];
    act[i] = g / (1.0f + expf(-g)) * u;
}

// fp32 attention: one CTA per (block position j, query head hq, request b);
// two-pass softmax over all len + gamma keys (no mask).
__global__ void k_attn_f32(const float* __restrict__ q, const float* __restrict__ slab, const int* __restrict__ len,
                           const int* __restrict__ req_ok, float* __restrict__ o, int gamma, int nq, int G, int d,
                           long long s_req, long long s_layer, long long s_kind, long long s_kv, int layer, float scale) {
    griddep_wait();
    griddep_launch();
    extern __shared__ float sh[];     // [n] scores, then [d] query
    const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
    const int m = b * gamma + j;
    float* out = o + (size_t)m * nq * d + (size_t)hq * d;
    if (!req_ok[b]) {
        for (int t = threadIdx.x; t < d; t += blockDim.x) out[t] = 0.f;
        return;
    }
    const int n = len[b] + gamma, g = hq / G;
    const float* K = slab + (size_t)b * s_req + (size_t)layer * s_layer + (size_t)g * s_kv;
    const float* Vv = K + s_kind;
    const float* qv = q + (size_t)m * nq * d + (size_t)hq * d;
    float* s = sh;
    __shared__ float red[32];
    float mx = -INFINITY;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        float acc = 0.f;
        for (int t = 0; t < d; ++t) acc += qv[t] * K[(size_t)i * d + t];
        s[i] = acc * scale;
        mx = fmaxf(mx, s[i]);
    }
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = red[0];
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) t = fmaxf(t, red[w]);
        red[0] = t;
    }
    __syncthreads();
    mx = red[0];
    __syncthreads();
    float z = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        s[i] = expf(s[i] - mx);
        z += s[i];
    }
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = z;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
        red[0] = t;
    }
    __syncthreads();
    const float inv = 1.0f / red[0];
    for (int t = threadIdx.x; t < d; t += blockDim.x) {
        float acc = 0.f;
        for (int i = 0; i < n; ++i) acc += s[i] * Vv[(size_t)i * d + t];
        out[t] = acc * inv;
    }
}

// ---------------------------------------------------------------------------
// Launch wrappers
// ---------------------------------------------------------------------------
template <typename T>
void launch_embed(const T* embed, const int* anchor, int mask_id, int B, int gamma, int H, int V, const int* len,
                  const int* committed, int cap, T* x, int* req_ok, int* status, cudaStream_t st, long long* tr,
                  float* ssq) {
    launch_k(k_embed<T>, dim3(B * gamma), dim3(128), 0, st, embed, anchor, mask_id, gamma, H, V, len, committed, cap, x,
             req_ok, status, ssq, tr);
}
template <typename T>
void launch_rmsnorm(const T* x, const T* g, T* y, int rows, int H, float eps, int grp, int gstride, int goff,
                    cudaStream_t st, long long* tr) {
    if (rows <= 0) return;
    launch_k(k_rmsnorm<T>, dim3(rows), dim3(H / (16 / (int)sizeof(T)) >= 256 ? 256 : 128), 0, st, x, g, y, H, eps,
             grp, gstride, goff, tr);
}
template void launch_embed<float>(const float*, const int*, int, int, int, int, int, const int*, const int*, int,
                                  float*, int*, int*, cudaStream_t, long long*, float*);
template void launch_embed<__nv_bfloat16>(const __nv_bfloat16*, const int*, int, int, int, int, int, const int*,
                                          const int*, int, __nv_bfloat16*, int*, int*, cudaStream_t, long long*,
                                          float*);
template void launch_rmsnorm<float>(const float*, const float*, float*, int, int, float, int, int, int, cudaStream_t,
                                    long long*);
template void launch_rmsnorm<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*, __nv_bfloat16*, int, int,
                                            float, int, int, int, cudaStream_t, long long*);

void launch_lm_reduce(const float4* rec, int n_vt, int M, int gm1, const int* req_ok, int* drafts, float* margin,
                      cudaStream_t st, long long* tr, int rec_blocks) {
    launch_k(k_lm_reduce, dim3(M), dim3(kLmReduceThreads), 0, st, rec, n_vt, M, gm1, req_ok, drafts, margin,
             rec_blocks, tr);
}
void launch_top2_rows(const float* logits, int M, int V, int gm1, const int* req_ok, int* drafts, float* margin,
                      cudaStream_t st) {
    launch_k(k_top2_rows, dim3(M), dim3(256), 0, st, logits, V, gm1, req_ok, drafts, margin);
}
void launch_accept(const int* drafts, const int* target, int B, int gamma, int V, int* len, int* committed,
                   int* accept_len, int* next_anchor, int* status, cudaStream_t st, long long* tr) {
    launch_k(k_accept, dim3((B * 32 + 127) / 128), dim3(128), 0, st, drafts, target, B, gamma, V, len, committed,
             accept_len, next_anchor, status, tr);
}
void launch_ingest_begin(const __nv_bfloat16* ctx, int B, int rows, int H, const int* len, int cap, __nv_bfloat16* x,
                         int* req_ok, int* status, float* ssq, cudaStream_t st) {
    launch_k(k_ingest_begin, dim3(B * rows), dim3(128), 0, st, ctx, rows, H, len, cap, x, req_ok, status, ssq);
}
void launch_ingest_end(const int* row_count, int rows, int B, const int* req_ok, int* len, int* status,
                       cudaStream_t st) {
    launch_k(k_ingest_end, dim3((B + 127) / 128), dim3(128), 0, st, row_count, rows, B, req_ok, len, status);
}
void launch_inject_finalize(const int* row_count, int B, int cap, int* len, int* status, cudaStream_t st,
                            long long* tr) {
    launch_k(k_inject_finalize, dim3((B + 127) / 128), dim3(128), 0, st, row_count, B, cap, len, status, tr);
}
void launch_set_len(const int* lens, int B, int cap, int* len, int* committed, int* status, cudaStream_t st,
                    long long* tr) {
    launch_k(k_set_len, dim3((B + 127) / 128), dim3(128), 0, st, lens, B, cap, len, committed, status, tr);
}
void launch_synth_target(const int* drafts, const int* a_plan, const int* rnd, int B, int gamma, int V, int* target,
                         cudaStream_t st) {
    launch_k(k_synth_target, dim3((B * gamma + 127) / 128), dim3(128), 0, st, drafts, a_plan, rnd, B, gamma, V, target);
}
int launch_wait_selftest(int* status, int* out, cudaStream_t st) {
    return (int)launch_k(k_wait_selftest, dim3(1), dim3(32), 0, st, status, out);
}
void launch_gemm_f32(const XSegs& xs, const float* W, float* Y, int M, int N, int K, int ldy, int ycol0,
                     cudaStream_t st) {
    const long long warps = (long long)M * N;
    if (warps == 0) return;
    launch_k(k_gemm_f32, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0, st, xs, W, Y, M, N, K, ldy, ycol0);
}
void launch_epi_qkv_f32(const float* Y, int M, int Nq, int Nkv, int d, int gamma, const int* len, const int* req_ok,
                        const float2* rope, float* q, float* slab, long long s_req, long long s_layer, long long s_kind,
                        long long s_kv, int layer, cudaStream_t st) {
    const long long n = (long long)M * (Nq + 2 * Nkv);
    launch_k(k_epi_qkv_f32, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, Y, M, Nq, Nkv, d, gamma, len, req_ok, rope, q, slab,
                                                               s_req, s_layer, s_kind, s_kv, layer);
}
void launch_epi_inject_f32(const float* Y, int rows, int Nkv, int d, const int* row_start, const int* row_count, int B,
                           const int* len, int cap, const float2* rope, float* slab, long long s_req, long long s_layer,
                           long long s_kind, long long s_kv, int layer, cudaStream_t st) {
    const long long n = (long long)rows * 2 * Nkv;
    if (n == 0) return;
    launch_k(k_epi_inject_f32, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, Y, rows, Nkv, d, row_start, row_count, B, len, cap,
                                                                  rope, slab, s_req, s_layer, s_kind, s_kv, layer);
}
void launch_resid_f32(float* x, const float* Y, long long n, cudaStream_t st) {
    launch_k(k_resid_f32, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, x, Y, n);
}
void launch_swiglu_f32(const float* Y, float* act, int M, int I, cudaStream_t st) {
    const long long n = (long long)M * I;
    launch_k(k_swiglu_f32, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, Y, act, M, I);
}
int launch_attn_f32(const float* q, const float* slab, const int* len, const int* req_ok, float* o, int B, int gamma,
                    int nq, int G, int d, long long s_req, long long s_layer, long long s_kind, long long s_kv,
                    int layer, int cap, cudaStream_t st) {
    const size_t smem = (size_t)cap * sizeof(float);
    static size_t set_to = 0;
    if (smem > 48 * 1024 && smem > set_to) {
        cudaError_t e = cudaFuncSetAttribute(k_attn_f32, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
        set_to = smem;
    }
    dim3 grid(gamma, nq, B);
    launch_k(k_attn_f32, dim3(grid), dim3(128), smem, st, q, slab, len, req_ok, o, gamma, nq, G, d, s_req, s_layer, s_kind, s_kv, layer,
                                        1.0f / sqrtf((float)d));
    return (int)cudaGetLastError();
}

}  // namespace df
