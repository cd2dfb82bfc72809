// DFlash draft-step oracle: a plain, slow, double-precision CPU implementation.
//
// TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
// GPU library is checked against.  Only the test suite, the package smoke
// check and the benchmark's CPU-baseline leg may load it.  It shares no code,
// header, table or constant generator with the CUDA library, and the CUDA
// library never calls it.
//
// What it computes follows the DFlash technical summaries ("DFlash – Block
// Diffusion for Flash Speculative Decoding", gist.science ja/nl pages):
//   * §2.2 (inference design), context-feature bullet: hidden states of a fixed,
//     uniformly spaced set of target layers are concatenated and projected into
//     one compact context feature                         -> oracle_fuse_context
//   * §2.2, KV-injection bullet: that feature enters the key/value projection of
//     every draft layer and is kept in the draft KV cache   -> oracle_inject_kv
//   * §2.2, parallel block diffusion bullet: one forward pass predicts a block of
//     masked positions; §2.3 random-anchor bullet: the block starts from the
//     target's clean token; §2.3 architecture bullet: embedding and LM head are
//     shared with the target                               -> oracle_draft_block
//   * §5 (claims), lossless verification: drafts are kept only while they equal
//     the target's own greedy tokens                      -> oracle_accept
//   * §2.3 loss-weighting bullet: w_k = exp(-(k-1)/gamma)  -> oracle_loss_weights
//   * §3 contribution 2 / §4 KV-injection ablation: the input-fusion drafter that
//     KV injection is compared against                  -> oracle_ingest_fused_input
//
// The summaries give no layer equations.  The layer internals used here
// (pre-norm RMSNorm, rotate-half RoPE, grouped-query attention without a mask,
// SwiGLU MLP, a final norm before the LM head) and the bf16 storage points R()
// are the plain reading of a standard decoder layer; the CUDA library states
// the same reading in its header.  R() is round-to-nearest-even to bf16 when
// storage is bf16 and the identity when storage is fp32.  Every accumulation is
// fp64.  No blocking, fusion or reordering is done beyond what the definitions
// state: plain loops, parallelised over independent outputs only.
//
// Pins (the test suite's CPU tests): R() against torch's bf16 cast and brute
// force; RMSNorm, RoPE and attention against library routines, closed forms
// and invariants; accept exhaustively against a brute-force scan; the loss
// weights against their closed form; fuse, inject and draft through invariants
// (concat order, chunked = one-shot injection, one bidirectional pass, zero
// layers = norm + shared head); the input-fusion ingest against a torch causal
// composition, chunked = one-shot, and one layer = injecting the normed feature.  The composition of oracle_fuse_context,
// oracle_inject_kv and oracle_draft_block as a DFlash drafter (norm placement,
// positions, mask id) follows the reading above and cannot be checked against
// a trained DFlash model here: parity unpinned against the paper's model.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#include <limits>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

struct oracle_config {
    int hidden, n_layers, n_q_heads, n_kv_heads, head_dim, intermediate, vocab;
    int n_sel, target_hidden, mask_id;
    int storage;            // 0: fp32 storage, R() is the identity. 1: bf16 storage.
    double rope_theta, rms_eps;
    int acc32;              // 1: accumulate dot products in fp32 instead of fp64
                            //    (a timing / sensitivity variant; parity uses 0)
};

// All matrices are [out, in] row-major in the storage type (uint16 bf16 bit
// patterns, or float).  lm_head may alias embed (tied embedding / LM head).
struct oracle_weights {
    const void* w_fc;      // [hidden, n_sel*target_hidden]
    const void* g_fc;      // [hidden]
    const void* embed;     // [vocab, hidden]
    const void* lm_head;   // [vocab, hidden]
    const void* g_final;   // [hidden]
    const void* g_in[16];
    const void* wq[16];    // [n_q_heads*head_dim, hidden]
    const void* wk[16];    // [n_kv_heads*head_dim, hidden]
    const void* wv[16];    // [n_kv_heads*head_dim, hidden]
    const void* wo[16];    // [hidden, n_q_heads*head_dim]
    const void* g_post[16];
    const void* w_gate[16];  // [intermediate, hidden]
    const void* w_up[16];    // [intermediate, hidden]
    const void* w_down[16];  // [hidden, intermediate]
};

// ---------------------------------------------------------------------------
// Storage-type helpers
// ---------------------------------------------------------------------------

static inline double bf16_bits_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return (double)f;
}

static inline double load(const void* p, long i, int storage) {
    if (storage == 1) return bf16_bits_to_double(((const uint16_t*)p)[i]);
    return (double)((const float*)p)[i];
}

// Round-to-nearest-even of a double to the nearest bf16 value (8 significant
// bits, exponent range of fp32, gradual underflow).  Direct rounding from the
// double, not via fp32, so there is no double rounding.
double oracle_round_bf16(double x) {
    if (std::isnan(x) || std::isinf(x) || x == 0.0) return x;
    int e;
    std::frexp(x, &e);                 // |x| = m * 2^e, m in [0.5, 1)
    int E = e - 1;                     // |x| in [2^E, 2^(E+1))
    if (E < -126) E = -126;            // subnormal range: fixed quantum 2^-133
    double quantum = std::ldexp(1.0, E - 7);
    double q = std::nearbyint(x / quantum);   // default FP env rounds half to even
    double r = q * quantum;
    if (std::fabs(r) >= std::ldexp(1.0, 128)) return x > 0 ? INFINITY : -INFINITY;
    return r;
}

void oracle_round_bf16_array(const double* x, double* y, long n) {
    for (long i = 0; i < n; ++i) y[i] = oracle_round_bf16(x[i]);
}

static inline double R(double x, int storage) {
    return storage == 1 ? oracle_round_bf16(x) : x;
}

// ---------------------------------------------------------------------------
// Building blocks (each exported so the tests can pin it on its own)
// ---------------------------------------------------------------------------

// y = x / sqrt(mean(x^2) + eps) * g      (no rounding)
void oracle_rmsnorm(const double* x, const double* g, int n, double eps, double* y) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double inv = 1.0 / std::sqrt(ss / n + eps);
    for (int i = 0; i < n; ++i) y[i] = x[i] * inv * g[i];
}

// Rotate-half rotary embedding of one head vector v[0..d) at position pos:
// pairs (i, i + d/2), angle pos * theta^(-2i/d).
void oracle_rope(double* v, int d, long pos, double theta) {
    int h = d / 2;
    for (int i = 0; i < h; ++i) {
        double inv_freq = std::pow(theta, -2.0 * i / d);
        double ang = (double)pos * inv_freq;
        double c = std::cos(ang), s = std::sin(ang);
        double a = v[i], b = v[i + h];
        v[i] = a * c - b * s;
        v[i + h] = b * c + a * s;
    }
}

// Multi-head attention without a mask, over one block of keys, unnormalised.
// q: [nrow][nq][d]; k, v: [nkv][n][d].  Query head hq reads key/value head
// hq / (nq/nkv).  Scores are scaled by 1/sqrt(d) and the softmax is written in
// base 2 with an integer shift: t_i = (q . k_i) * log2(e) / sqrt(d),
// B = floor(max_i t_i), e_i = 2^(t_i - B).  Outputs per (row, head):
//   num[r][hq][u] = sum_i P_i v_i[u] with P_i = e_i, or R(e_i) (bf16) when round_p,
//   z[r][hq]      = sum_i e_i        (the unrounded weights),
//   base[r][hq]   = B                (-inf when n == 0).
// Because B is an integer, the weights of a key are the same numbers times an
// exact power of two whatever block of keys it is in, so blocks with their own
// bases combine exactly: rescale each block's num and z by 2^(B_block - B_all).
void oracle_attention_block(const double* q, int nrow, int nq, const double* k, const double* v,
                            int n, int nkv, int d, int round_p, double* num, double* z, double* base) {
    int G = nq / nkv;
    const double scale = 1.4426950408889634 / std::sqrt((double)d);   // log2(e) / sqrt(d)
    #pragma omp parallel for collapse(2) schedule(static)
    for (int r = 0; r < nrow; ++r) {
        for (int hq = 0; hq < nq; ++hq) {
            int g = hq / G;
            const double* qv = q + ((long)r * nq + hq) * d;
            const double* kh = k + (long)g * n * d;
            const double* vh = v + (long)g * n * d;
            std::vector<double> t(n > 0 ? n : 1);
            double m = -INFINITY;
            for (int i = 0; i < n; ++i) {
                double acc = 0.0;
                for (int u = 0; u < d; ++u) acc += qv[u] * kh[(long)i * d + u];
                t[i] = acc * scale;
                if (t[i] > m) m = t[i];
            }
            const double B = std::floor(m);
            double Z = 0.0;
            for (int i = 0; i < n; ++i) { t[i] = std::exp2(t[i] - B); Z += t[i]; }
            double* ov = num + ((long)r * nq + hq) * d;
            for (int u = 0; u < d; ++u) ov[u] = 0.0;
            for (int i = 0; i < n; ++i) {
                double e = round_p ? oracle_round_bf16(t[i]) : t[i];
                for (int u = 0; u < d; ++u) ov[u] += e * vh[(long)i * d + u];
            }
            z[(long)r * nq + hq] = Z;
            base[(long)r * nq + hq] = B;
        }
    }
}

// Attention output: o = num / z of oracle_attention_block over all n keys,
// which is softmax(q K^T / sqrt(d)) V (with round_p: the bf16-rounded weights
// R(2^(t_i - B)) in the numerator, the unrounded ones in the denominator).  The
// output is not rounded here.
void oracle_attention(const double* q, int nrow, int nq, const double* k, const double* v,
                      int n, int nkv, int d, int round_p, double* o) {
    std::vector<double> z((size_t)nrow * nq), base((size_t)nrow * nq);
    oracle_attention_block(q, nrow, nq, k, v, n, nkv, d, round_p, o, z.data(), base.data());
    for (long rh = 0; rh < (long)nrow * nq; ++rh)
        for (int u = 0; u < d; ++u) o[rh * d + u] /= z[rh];
}

// y[m][n] = sum_k x[m][k] * W[n][k]; W in storage type, [N, K] row-major.
static int g_acc32 = 0;   // set from oracle_config.acc32 by each entry point

static void linear(const double* x, int M, int K, const void* W, int N, int storage, double* y) {
    #pragma omp parallel
    {
        std::vector<double> wrow(K);
        #pragma omp for schedule(static)
        for (int nn = 0; nn < N; ++nn) {
            for (int kk = 0; kk < K; ++kk) wrow[kk] = load(W, (long)nn * K + kk, storage);
            for (int mm = 0; mm < M; ++mm) {
                const double* xr = x + (long)mm * K;
                if (g_acc32) {
                    float acc = 0.0f;
                    for (int kk = 0; kk < K; ++kk) acc += (float)xr[kk] * (float)wrow[kk];
                    y[(long)mm * N + nn] = acc;
                    continue;
                }
                double acc = 0.0;
                // fp64 dot product; the simd reduction only changes the order
                // in which fp64 partial sums are added.
                #pragma omp simd reduction(+:acc)
                for (int kk = 0; kk < K; ++kk) acc += xr[kk] * wrow[kk];
                y[(long)mm * N + nn] = acc;
            }
        }
    }
}

static void load_vec(const void* p, int n, int storage, double* out) {
    for (int i = 0; i < n; ++i) out[i] = load(p, i, storage);
}

// Uniformly spaced target layers, shallow to deep (reading of §2.2's
// context-feature bullet; the pages name no indices): l_i = round(i*(L_t-1)/(n_sel-1)).
void oracle_layer_ids(int n_target_layers, int n_sel, int* ids) {
    for (int i = 0; i < n_sel; ++i) {
        if (n_sel == 1) { ids[i] = n_target_layers - 1; continue; }
        double t = (double)i * (n_target_layers - 1) / (n_sel - 1);
        ids[i] = (int)std::floor(t + 0.5);
    }
}

// §2.3 loss-weighting bullet: w_k = exp(-(k-1)/gamma), k = 1..gamma.
void oracle_loss_weights(int gamma, double* w) {
    for (int k = 1; k <= gamma; ++k) w[k - 1] = std::exp(-(double)(k - 1) / gamma);
}

// ---------------------------------------------------------------------------
// a1: fuse the context feature.
// ctx_r = R( RMSNorm( R( concat_i h_i[r] . W_fc^T ) ) * g_fc )
// hiddens[i] points at n_sel arrays of [rows, target_hidden] (row stride in
// elements), concatenated in ascending layer order along the feature axis.
// ---------------------------------------------------------------------------
void oracle_fuse_context(const oracle_config* c, const oracle_weights* w,
                         const void* const* hiddens, long row_stride, int rows, double* ctx_out) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, Ht = c->target_hidden, Kc = c->n_sel * Ht;
    std::vector<double> cat((size_t)rows * Kc);
    for (int r = 0; r < rows; ++r)
        for (int i = 0; i < c->n_sel; ++i)
            for (int t = 0; t < Ht; ++t)
                cat[(size_t)r * Kc + (size_t)i * Ht + t] = load(hiddens[i], (long)r * row_stride + t, S);
    std::vector<double> y((size_t)rows * H);
    linear(cat.data(), rows, Kc, w->w_fc, H, S, y.data());
    std::vector<double> g(H);
    load_vec(w->g_fc, H, S, g.data());
    std::vector<double> tmp(H);
    for (int r = 0; r < rows; ++r) {
        double* yr = y.data() + (size_t)r * H;
        for (int t = 0; t < H; ++t) yr[t] = R(yr[t], S);
        oracle_rmsnorm(yr, g.data(), H, c->rms_eps, tmp.data());
        for (int t = 0; t < H; ++t) ctx_out[(size_t)r * H + t] = R(tmp[t], S);
    }
}

// ---------------------------------------------------------------------------
// a2: inject the context feature into every draft layer's K/V cache.
// For layer l and row r at absolute position p = pos0 + r:
//   K_l[p] = R( RoPE_p( ctx_r . W_k,l^T ) ),  V_l[p] = R( ctx_r . W_v,l^T )
// Cache layout (this oracle's own): k_cache/v_cache [L][nkv][cap][d].
// ---------------------------------------------------------------------------
void oracle_inject_kv(const oracle_config* c, const oracle_weights* w, const double* ctx,
                      int rows, int pos0, double* k_cache, double* v_cache, int cap) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, d = c->head_dim, nkv = c->n_kv_heads, Nkv = nkv * d;
    std::vector<double> kk((size_t)rows * Nkv), vv((size_t)rows * Nkv);
    for (int l = 0; l < c->n_layers; ++l) {
        linear(ctx, rows, H, w->wk[l], Nkv, S, kk.data());
        linear(ctx, rows, H, w->wv[l], Nkv, S, vv.data());
        for (int r = 0; r < rows; ++r) {
            long p = (long)pos0 + r;
            for (int g = 0; g < nkv; ++g) {
                double* kh = kk.data() + (size_t)r * Nkv + (size_t)g * d;
                double* vh = vv.data() + (size_t)r * Nkv + (size_t)g * d;
                oracle_rope(kh, d, p, c->rope_theta);
                size_t base = (((size_t)l * nkv + g) * cap + p) * d;
                for (int t = 0; t < d; ++t) {
                    k_cache[base + t] = R(kh[t], S);
                    v_cache[base + t] = R(vh[t], S);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Input-fusion ablation (the conditioning DFlash is compared against: DFlash
// technical summary, §3 contribution 2 and the KV-injection ablation bullet of
// §4).  Instead of a2, context row r at absolute position p = pos0 + r enters
// the drafter as its input hidden state x = ctx_r and passes through the draft
// layers like a token; each layer caches the K/V of its own normed state:
//   h = R(RMSNorm(x) * g_in,l);  K_l[p] = R(RoPE_p(h . W_k,l^T));  V_l[p] = R(h . W_v,l^T)
//   q = R(RoPE_p(h . W_q,l^T));  o = R(attention over cached rows [0, p]) (causal)
//   x = R(x + o . W_o,l^T);  h2 = R(RMSNorm(x) * g_post,l);
//   m = R(silu(h2 . W_g,l^T) * (h2 . W_u,l^T));  x = R(x + m . W_d,l^T)
// The last layer's attention and MLP change no cached value and are skipped.
// Rows are appended in order and attend only to rows at or before their own
// position, so appending in chunks gives the same cache as appending at once.
// ---------------------------------------------------------------------------
void oracle_ingest_fused_input(const oracle_config* c, const oracle_weights* w, const double* ctx,
                               int rows, int pos0, double* k_cache, double* v_cache, int cap) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, d = c->head_dim, nq = c->n_q_heads, nkv = c->n_kv_heads;
    int Nq = nq * d, Nkv = nkv * d, I = c->intermediate;
    std::vector<double> x(ctx, ctx + (size_t)rows * H);
    std::vector<double> g(H), tmp(H), h((size_t)rows * H), y((size_t)rows * H);
    std::vector<double> q((size_t)rows * Nq), kk((size_t)rows * Nkv), vv((size_t)rows * Nkv), o((size_t)rows * Nq);
    std::vector<double> gt((size_t)rows * I), up((size_t)rows * I), mm((size_t)rows * I);
    for (int l = 0; l < c->n_layers; ++l) {
        load_vec(w->g_in[l], H, S, g.data());
        for (int r = 0; r < rows; ++r) {
            oracle_rmsnorm(x.data() + (size_t)r * H, g.data(), H, c->rms_eps, tmp.data());
            for (int t = 0; t < H; ++t) h[(size_t)r * H + t] = R(tmp[t], S);
        }
        linear(h.data(), rows, H, w->wk[l], Nkv, S, kk.data());
        linear(h.data(), rows, H, w->wv[l], Nkv, S, vv.data());
        for (int r = 0; r < rows; ++r) {
            long p = (long)pos0 + r;
            for (int g2 = 0; g2 < nkv; ++g2) {
                double* kh = kk.data() + (size_t)r * Nkv + (size_t)g2 * d;
                const double* vh = vv.data() + (size_t)r * Nkv + (size_t)g2 * d;
                oracle_rope(kh, d, p, c->rope_theta);
                size_t base = (((size_t)l * nkv + g2) * cap + p) * d;
                for (int t = 0; t < d; ++t) {
                    k_cache[base + t] = R(kh[t], S);
                    v_cache[base + t] = R(vh[t], S);
                }
            }
        }
        if (l == c->n_layers - 1) break;
        linear(h.data(), rows, H, w->wq[l], Nq, S, q.data());
        for (int r = 0; r < rows; ++r)
            for (int hq = 0; hq < nq; ++hq)
                oracle_rope(q.data() + (size_t)r * Nq + (size_t)hq * d, d, (long)pos0 + r, c->rope_theta);
        for (auto& e : q) e = R(e, S);
        // causal: row r reads cached rows [0, pos0 + r]
        for (int r = 0; r < rows; ++r) {
            int n = pos0 + r + 1;
            std::vector<double> K((size_t)nkv * n * d), Vv((size_t)nkv * n * d);
            for (int g2 = 0; g2 < nkv; ++g2)
                for (int i = 0; i < n; ++i)
                    for (int t = 0; t < d; ++t) {
                        size_t src = (((size_t)l * nkv + g2) * cap + i) * d + t;
                        K[((size_t)g2 * n + i) * d + t] = k_cache[src];
                        Vv[((size_t)g2 * n + i) * d + t] = v_cache[src];
                    }
            oracle_attention(q.data() + (size_t)r * Nq, 1, nq, K.data(), Vv.data(), n, nkv, d, S == 1,
                             o.data() + (size_t)r * Nq);
        }
        for (auto& e : o) e = R(e, S);
        linear(o.data(), rows, Nq, w->wo[l], H, S, y.data());
        for (size_t i = 0; i < x.size(); ++i) x[i] = R(x[i] + y[i], S);
        load_vec(w->g_post[l], H, S, g.data());
        for (int r = 0; r < rows; ++r) {
            oracle_rmsnorm(x.data() + (size_t)r * H, g.data(), H, c->rms_eps, tmp.data());
            for (int t = 0; t < H; ++t) h[(size_t)r * H + t] = R(tmp[t], S);
        }
        linear(h.data(), rows, H, w->w_gate[l], I, S, gt.data());
        linear(h.data(), rows, H, w->w_up[l], I, S, up.data());
        for (size_t i = 0; i < mm.size(); ++i) {
            double a = gt[i];
            mm[i] = R(a / (1.0 + std::exp(-a)) * up[i], S);
        }
        linear(mm.data(), rows, I, w->w_down[l], H, S, y.data());
        for (size_t i = 0; i < x.size(); ++i) x[i] = R(x[i] + y[i], S);
    }
}

// ---------------------------------------------------------------------------
// a4..a6, one stage at a time (each exported, so a test can feed a stage its
// input from elsewhere).  rows of the block: j = 0..gamma-1 at absolute
// position len + j.
// ---------------------------------------------------------------------------

// RMSNorm of `rows` rows of width H with gain g (storage type), rounded:
// out = R(RMSNorm(x) * g).
void oracle_norm_rows(const oracle_config* c, const void* g_w, const double* x, int rows, double* out) {
    int S = c->storage, H = c->hidden;
    std::vector<double> g(H), tmp(H);
    load_vec(g_w, H, S, g.data());
    for (int j = 0; j < rows; ++j) {
        oracle_rmsnorm(x + (size_t)j * H, g.data(), H, c->rms_eps, tmp.data());
        for (int t = 0; t < H; ++t) out[(size_t)j * H + t] = R(tmp[t], S);
    }
}

// a4: q = R(RoPE(h . Wq^T)), k = R(RoPE(h . Wk^T)), v = R(h . Wv^T) of layer l for
// the normalised rows h [gamma][H]; q [gamma][nq*d], k, v [gamma][nkv*d].
void oracle_layer_qkv(const oracle_config* c, const oracle_weights* w, int l, const double* h, int len,
                      int gamma, double* q, double* k, double* v) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, d = c->head_dim, nq = c->n_q_heads, nkv = c->n_kv_heads;
    int Nq = nq * d, Nkv = nkv * d;
    linear(h, gamma, H, w->wq[l], Nq, S, q);
    linear(h, gamma, H, w->wk[l], Nkv, S, k);
    linear(h, gamma, H, w->wv[l], Nkv, S, v);
    for (int j = 0; j < gamma; ++j) {
        long p = (long)len + j;
        for (int hq = 0; hq < nq; ++hq) oracle_rope(q + (size_t)j * Nq + (size_t)hq * d, d, p, c->rope_theta);
        for (int g2 = 0; g2 < nkv; ++g2) oracle_rope(k + (size_t)j * Nkv + (size_t)g2 * d, d, p, c->rope_theta);
    }
    for (long i = 0; i < (long)gamma * Nq; ++i) q[i] = R(q[i], S);
    for (long i = 0; i < (long)gamma * Nkv; ++i) { k[i] = R(k[i], S); v[i] = R(v[i], S); }
}

// a5: o = R(attention) of the block's queries q [gamma][nq*d] over layer l's
// committed context rows [0, len) (k_cache/v_cache, [L][nkv][cap][d]) followed by
// the block's own rows kb, vb [gamma][nkv*d] (no mask; bf16 P with bf16 storage).
void oracle_layer_attention(const oracle_config* c, int l, const double* q, const double* kb, const double* vb,
                            const double* k_cache, const double* v_cache, int cap, int len, int gamma, double* o) {
    int S = c->storage, d = c->head_dim, nq = c->n_q_heads, nkv = c->n_kv_heads;
    int Nkv = nkv * d, n = len + gamma;
    std::vector<double> K((size_t)nkv * n * d), Vv((size_t)nkv * n * d);
    for (int g2 = 0; g2 < nkv; ++g2) {
        for (int i = 0; i < len; ++i)
            for (int t = 0; t < d; ++t) {
                size_t src = (((size_t)l * nkv + g2) * cap + i) * d + t;
                K[((size_t)g2 * n + i) * d + t] = k_cache[src];
                Vv[((size_t)g2 * n + i) * d + t] = v_cache[src];
            }
        for (int j = 0; j < gamma; ++j)
            for (int t = 0; t < d; ++t) {
                K[((size_t)g2 * n + len + j) * d + t] = kb[(size_t)j * Nkv + (size_t)g2 * d + t];
                Vv[((size_t)g2 * n + len + j) * d + t] = vb[(size_t)j * Nkv + (size_t)g2 * d + t];
            }
    }
    oracle_attention(q, gamma, nq, K.data(), Vv.data(), n, nkv, d, S == 1, o);
    for (long i = 0; i < (long)gamma * nq * d; ++i) o[i] = R(o[i], S);
}

// a6, first half: x_out = R(x + o . Wo^T) for rows [gamma].
void oracle_layer_oproj(const oracle_config* c, const oracle_weights* w, int l, const double* o, const double* x,
                        int gamma, double* x_out) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, Nq = c->n_q_heads * c->head_dim;
    std::vector<double> y((size_t)gamma * H);
    linear(o, gamma, Nq, w->wo[l], H, S, y.data());
    for (size_t i = 0; i < y.size(); ++i) x_out[i] = R(x[i] + y[i], S);
}

// a6, second half: m = R(silu(h2 . Wg^T) * (h2 . Wu^T)) for the normalised rows
// h2 [gamma][H] (m [gamma][I] optional), then x_out = R(x + m . Wd^T).
// The down-projection and residual add of layer l from the SwiGLU output m
// [gamma][intermediate]: x_out = R(x + m . Wd^T).
void oracle_layer_down(const oracle_config* c, const oracle_weights* w, int l, const double* m, const double* x,
                       int gamma, double* x_out) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, I = c->intermediate;
    std::vector<double> y((size_t)gamma * H);
    linear(m, gamma, I, w->w_down[l], H, S, y.data());
    for (size_t i = 0; i < y.size(); ++i) x_out[i] = R(x[i] + y[i], S);
}

void oracle_layer_mlp(const oracle_config* c, const oracle_weights* w, int l, const double* h2, const double* x,
                      int gamma, double* m_out, double* x_out) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, I = c->intermediate;
    std::vector<double> gt((size_t)gamma * I), up((size_t)gamma * I), mm((size_t)gamma * I);
    linear(h2, gamma, H, w->w_gate[l], I, S, gt.data());
    linear(h2, gamma, H, w->w_up[l], I, S, up.data());
    for (size_t i = 0; i < mm.size(); ++i) {
        double a = gt[i];
        double silu = a / (1.0 + std::exp(-a));
        mm[i] = R(silu * up[i], S);
    }
    if (m_out) std::memcpy(m_out, mm.data(), sizeof(double) * mm.size());
    oracle_layer_down(c, w, l, mm.data(), x, gamma, x_out);
}

// ---------------------------------------------------------------------------
// a4..a6: one draft layer l on the block's hidden states x [gamma][H], in place:
//   h = R(RMSNorm(x) * g_in); q, k, v (oracle_layer_qkv); o (oracle_layer_attention);
//   x = R(x + o . Wo^T); h2 = R(RMSNorm(x) * g_post); x = R(x + m . Wd^T) with the
//   SwiGLU m (oracle_layer_mlp).  The block's own K/V are used for this pass only
//   and are not written to the cache.
// ---------------------------------------------------------------------------
void oracle_draft_layer(const oracle_config* c, const oracle_weights* w, int l,
                        const double* k_cache, const double* v_cache, int cap, int len,
                        int gamma, double* x) {
    int H = c->hidden, Nq = c->n_q_heads * c->head_dim, Nkv = c->n_kv_heads * c->head_dim;
    size_t xs = (size_t)gamma * H;
    std::vector<double> h(xs), q((size_t)gamma * Nq), kb((size_t)gamma * Nkv), vb((size_t)gamma * Nkv);
    std::vector<double> o((size_t)gamma * Nq), xm(xs);
    oracle_norm_rows(c, w->g_in[l], x, gamma, h.data());
    oracle_layer_qkv(c, w, l, h.data(), len, gamma, q.data(), kb.data(), vb.data());
    oracle_layer_attention(c, l, q.data(), kb.data(), vb.data(), k_cache, v_cache, cap, len, gamma, o.data());
    oracle_layer_oproj(c, w, l, o.data(), x, gamma, xm.data());
    oracle_norm_rows(c, w->g_post[l], xm.data(), gamma, h.data());
    oracle_layer_mlp(c, w, l, h.data(), xm.data(), gamma, nullptr, x);
}

// a7 (second half): the shared LM head and argmax on already-normalised rows
// hf [rows][H]: logits = hf . lm_head^T (not rounded), drafts[r] = argmax
// (ties to the lowest index), margin[r] = top-1 minus top-2 logit.
// logits (optional): [rows][vocab]; margin (optional).
void oracle_lm_head(const oracle_config* c, const oracle_weights* w, const double* hf, int rows,
                    int* drafts, double* logits, double* margin) {
    g_acc32 = c->acc32;
    int S = c->storage, H = c->hidden, V = c->vocab;
    if (rows <= 0) return;
    std::vector<double> lg((size_t)rows * V);
    linear(hf, rows, H, w->lm_head, V, S, lg.data());
    for (int r = 0; r < rows; ++r) {
        const double* row = lg.data() + (size_t)r * V;
        int best = 0;
        for (int vv = 1; vv < V; ++vv) if (row[vv] > row[best]) best = vv;
        double second = -INFINITY;
        for (int vv = 0; vv < V; ++vv) if (vv != best && row[vv] > second) second = row[vv];
        drafts[r] = best;
        if (margin) margin[r] = (V > 1) ? row[best] - second : INFINITY;
    }
    if (logits) std::memcpy(logits, lg.data(), sizeof(double) * lg.size());
}

// a7 (first half): the final norm of the mask positions j = 1..gamma-1 of the
// block's last hidden states x [gamma][H]: hf[j-1] = R(RMSNorm(x_j) * g_final).
void oracle_final_norm(const oracle_config* c, const oracle_weights* w, const double* x, int gamma,
                       double* hf) {
    int S = c->storage, H = c->hidden;
    std::vector<double> g(H), tmp(H);
    load_vec(w->g_final, H, S, g.data());
    for (int j = 1; j < gamma; ++j) {
        oracle_rmsnorm(x + (size_t)j * H, g.data(), H, c->rms_eps, tmp.data());
        for (int t = 0; t < H; ++t) hf[(size_t)(j - 1) * H + t] = R(tmp[t], S);
    }
}

// a3: embedding of [anchor, mask, ..., mask] (exact copies of table rows) into x [gamma][H].
void oracle_embed_block(const oracle_config* c, const oracle_weights* w, int anchor, int gamma, double* x) {
    int S = c->storage, H = c->hidden;
    for (int j = 0; j < gamma; ++j) {
        int tok = (j == 0) ? anchor : c->mask_id;
        for (int t = 0; t < H; ++t) x[(size_t)j * H + t] = load(w->embed, (long)tok * H + t, S);
    }
}

// ---------------------------------------------------------------------------
// a3..a7: draft one block of gamma positions in one forward pass: the embedding
// (position 0 holds the clean anchor token, positions 1..gamma-1 the mask
// token), every draft layer once (oracle_draft_layer), then the final norm and
// the shared LM head.  Mask position j predicts the token at len + j:
// drafts[j-1] = argmax of its logits (ties to the lowest index), j = 1..gamma-1.
// logits (optional): [(gamma-1), vocab], margin (optional): top1 - top2 per row.
// ---------------------------------------------------------------------------
void oracle_draft_block(const oracle_config* c, const oracle_weights* w,
                        const double* k_cache, const double* v_cache, int cap, int len,
                        int anchor, int gamma, int* drafts, double* logits, double* margin) {
    g_acc32 = c->acc32;
    int H = c->hidden;
    std::vector<double> x((size_t)gamma * H);
    oracle_embed_block(c, w, anchor, gamma, x.data());
    for (int l = 0; l < c->n_layers; ++l)
        oracle_draft_layer(c, w, l, k_cache, v_cache, cap, len, gamma, x.data());
    int nd = gamma - 1;
    if (nd <= 0) return;
    std::vector<double> hf((size_t)nd * H);
    oracle_final_norm(c, w, x.data(), gamma, hf.data());
    oracle_lm_head(c, w, hf.data(), nd, drafts, logits, margin);
}

// ---------------------------------------------------------------------------
// a8: greedy lossless acceptance for one request.
// a = largest k <= gamma-1 with drafts[i] == target[i] for all i < k;
// next_anchor = target[a]; committed += a + 1; len = min(len, committed).
// Returns 0, or -7 (token out of range: nothing is changed, outputs are -1).
// ---------------------------------------------------------------------------
int oracle_accept(int gamma, int vocab, const int* drafts, const int* target,
                  int* accept_len, int* next_anchor, int* len, int* committed) {
    for (int i = 0; i < gamma; ++i) {
        if (target[i] < 0 || target[i] >= vocab) {
            *accept_len = -1;
            *next_anchor = -1;
            return -7;
        }
    }
    int a = 0;
    while (a < gamma - 1 && drafts[a] == target[a]) ++a;
    *accept_len = a;
    *next_anchor = target[a];
    *committed += a + 1;
    if (*len > *committed) *len = *committed;
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

}  // extern "C"
