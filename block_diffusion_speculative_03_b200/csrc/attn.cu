// Block attention of the draft step (bf16 storage) on the 5th-generation
// tensor cores, split over the key axis across the CTAs of one cluster.
//
// For request b and kv head g, the R = G*gamma query rows (G = query heads per
// kv head) attend to every cached row [0, len) plus the gamma block rows the
// QKV epilogue wrote at [len, len+gamma): no mask.  CTA `rank` of the cluster
// (b, g) takes keys [rank*chunk, (rank+1)*chunk).
//
// The R <= 128 query rows fill CS = 1 (R > 64), 2 (R > 32) or 4 copies of a
// window of RW = 128/CS lanes of an M = 128 tile: TMEM lane l holds query row
// l % RW and takes key slice l / RW (64/CS keys) of every 64-key tile.  Q and P are MMA
// operands in tensor memory, so the tensor cores read only K and V from
// shared memory.
//
//   warps 2-5  softmax, one TMEM lane per thread: first write the lane's Q row
//            into TMEM; per tile read the lane's S slice, keep a base-2 running
//            maximum with an integer base B per row, write P = bf16(2^(t - B))
//            for the slice into a P buffer in TMEM (the lane's other columns
//            stay zero), and rescale the lane's O by an exact power of two when
//            B grows.  The lanes of a row agree on B through shared memory
//            whenever one of them would move it.
//   warp 0   TMA: K/V tiles of 64 keys into a kAttnStages-deep ring.
//   warp 1   tcgen05.mma (one thread): S_i = Q K_i^T into one of three TMEM
//            buffers (N = 64 keys), issued up to three tiles ahead of the
//            softmax, and O += P_i V_i (N = head_dim, V an MN-major operand
//            straight from the TMA tile) once P_i is written.
//
// Lane l of O so holds the P.V sum over key slice l / RW only; the CS lanes of
// a row are added when the split's partial (B, l, O) is written to shared
// memory.  After a cluster barrier every CTA merges a slice of the rows by
// reading all partials through distributed shared memory, and writes the bf16
// output.
#include <cooperative_groups.h>

#include "attn.cuh"

namespace cg = cooperative_groups;

namespace df {

// Largest lag (in powers of two) of a row's running integer base behind its maximum.
constexpr float kAttnBaseLag = 8.0f;

template <int D>
struct AttnCfg {
    static constexpr int HALVES = D / 64;
    static constexpr int KV_BYTES = HALVES * 64 * 128;       // 64 keys x D
    static constexpr int RING = 2 * kAttnStages * KV_BYTES;  // K ring, V ring
    // + barriers, + row exchange [128]; at least half an SM's shared memory, so two of
    // these CTAs (each allocating all 512 TMEM columns) never share an SM
    static constexpr int SMEM = (1024 + RING + 768) > 117 * 1024 ? (1024 + RING + 768) : 117 * 1024;
    static constexpr int NS = 3;                             // S buffers in TMEM
    static constexpr int PO_LD = D + 4;   // partial row stride (floats): 16-byte skew per row
    // TMEM columns: S[NS] (NS x 64), Q (D/2 bf16 pairs), O (D), P[2] (2 x 32 bf16 pairs)
    static constexpr uint32_t T_S = 0, T_Q = 192, T_O = 256, T_P = 384, TMEM_COLS = 512;
    static_assert(T_S + NS * 64 <= T_Q && T_Q + D / 2 <= T_O && T_O + D <= T_P && T_P + 64 <= TMEM_COLS, "TMEM");
    // the split's partial, written over the ring once the key loop is done
    static_assert(128 * PO_LD * 4 + 128 * 8 + 3 * 128 * kAttnMaxSplits * 4 <= RING, "partial");
};

template <int D, int CS>
__global__ void __launch_bounds__(kAttnThreads, 1) k_attn_tc(const __grid_constant__ AttnParams p) {
    using C = AttnCfg<D>;
    constexpr int S = kAttnStages;
    constexpr int RW = 128 / CS;   // rows per window of the M = 128 tile
    constexpr int KC = 64 / CS;    // keys of a tile per softmax thread
    constexpr int PO_LD = C::PO_LD;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_align_up<uint8_t>(smem_raw, 1024);
    uint8_t* sK = smem;                            // [S][KV_BYTES]
    uint8_t* sV = sK + S * C::KV_BYTES;            // [S][KV_BYTES]
    uint64_t* bars = (uint64_t*)(smem + C::RING);
    uint64_t* q_full = bars;
    uint64_t* kv_full = q_full + 1;                // [S]
    uint64_t* kv_empty = kv_full + S;              // [S]
    uint64_t* s_full = kv_empty + S;               // [NS]
    uint64_t* p_full = s_full + C::NS;             // [2]
    uint64_t* o_done = p_full + 2;                 // [2]
    uint64_t* drain = o_done + 2;
    uint32_t* tmem_slot = (uint32_t*)(drain + 1);
    volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
    float* xch = (float*)(smem + C::RING + 256);   // [128] per TMEM lane: running max, then row sum
    // After the key loop the ring holds this CTA's partial.
    float* po = (float*)smem;                      // [128][PO_LD] lanes' O, then rows 0..RW-1 summed
    float2* pml = (float2*)(po + 128 * PO_LD);     // [128] (integer base, row sum)

    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int nsplit = p.splits;
    const int g = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    long long* trace = p.trace ? p.trace + (((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 8
                               : nullptr;
    if (trace && tid == 0) trace[0] = (long long)globaltimer_ns();
    if (tid == 0) tma_prefetch_desc(&p.tmap);
    // The kernel runs right after the QKV GEMM, which writes q and the block's own
    // K/V rows [len, len + gamma).  len and the committed context rows [0, len)
    // are older (the previous step's calls, complete before this step's first
    // kernel passed its own dependency wait), so the committed-context tiles are
    // loaded before this kernel's dependency wait, overlapping the GEMM's tail.
    // q, the tiles holding block rows and req_ok (written by the embedding, which
    // may still be running when this kernel starts) are read after it.  A skipped
    // request (req_ok = 0) is attended over zero tiles: its output rows are zero.

    const int R = p.G * p.gamma;
    const int rows_per = (R + nsplit - 1) / nsplit;
    const int r_lo = rank * rows_per, r_hi = min(R, r_lo + rows_per);
    const int len_b = p.len[b];
    const int n = len_b + p.gamma;
    const int kv0 = rank * p.chunk;
    const int kv1 = min(n, kv0 + p.chunk);
    const int ntiles_all = kv1 > kv0 ? (kv1 - kv0 + 63) / 64 : 0;
    // leading tiles made of committed context rows only (independent of the QKV GEMM)
    const int n_early = min(min(ntiles_all, S), len_b > kv0 ? (len_b - kv0) / 64 : 0);
    const long long rowK = (long long)b * p.rows_req + (long long)p.layer * p.rows_layer + (long long)g * p.rows_kv;
    const long long rowV = rowK + p.rows_kind;

    if (tid == 0) {
        mbar_init(q_full, 128);
        for (int i = 0; i < S; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        for (int i = 0; i < C::NS; ++i) mbar_init(&s_full[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&p_full[i], 128);
            mbar_init(&o_done[i], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The next kernel may start only once this CTA holds its TMEM: a dependent CTA
    // on this SM that allocated first and then waited for this grid would never
    // let the allocation above succeed.
    griddep_launch();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem + C::T_S, tQ = tmem + C::T_Q, tO = tmem + C::T_O, tP = tmem + C::T_P;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // first use of each ring stage: no free-slot wait needed
            for (int it = 0; it < n_early; ++it) {
                mbar_arrive_expect_tx(&kv_full[it], 2 * C::KV_BYTES);
                for (int h = 0; h < C::HALVES; ++h) {
                    tma_load_2d(sK + it * C::KV_BYTES + h * 8192, &p.tmap, &kv_full[it], h * 64,
                                (int)(rowK + kv0 + it * 64));
                    tma_load_2d(sV + it * C::KV_BYTES + h * 8192, &p.tmap, &kv_full[it], h * 64,
                                (int)(rowV + kv0 + it * 64));
                }
            }
        }
        griddep_wait();
        if (trace && lane == 0) trace[1] = (long long)globaltimer_ns();
        const int ntiles = p.req_ok[b] ? ntiles_all : 0;
        if (lane == 0) {
            for (int it = n_early; it < ntiles; ++it) {
                const int st = it % S;
                if (!mbar_wait(&kv_empty[st], (uint32_t)(((it / S) & 1) ^ 1), abort_flag, p.status)) break;
                mbar_arrive_expect_tx(&kv_full[st], 2 * C::KV_BYTES);
                for (int h = 0; h < C::HALVES; ++h) {
                    tma_load_2d(sK + st * C::KV_BYTES + h * 8192, &p.tmap, &kv_full[st], h * 64,
                                (int)(rowK + kv0 + it * 64));
                    tma_load_2d(sV + st * C::KV_BYTES + h * 8192, &p.tmap, &kv_full[st], h * 64,
                                (int)(rowV + kv0 + it * 64));
                }
            }
            // a skipped request consumes none of its early tiles: let them land
            // before the CTA can exit
            for (int it = ntiles; it < n_early; ++it) {
                volatile int never = 0;
                mbar_wait(&kv_full[it], 0, &never, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        griddep_wait();
        const int ntiles = p.req_ok[b] ? ntiles_all : 0;
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64);
            constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
            bool ok = mbar_wait(q_full, 0, abort_flag, p.status);   // Q (and zeroed P) in TMEM
            tc_fence_after();
            if (trace) trace[2] = (long long)globaltimer_ns();
            // S_j = Q K_j^T into S buffer j % NS (free: the softmax has read S_{j-NS}).
            auto issue_s = [&](int j) -> bool {
                const int st = j % S;
                if (!mbar_wait(&kv_full[st], (uint32_t)((j / S) & 1), abort_flag, p.status)) return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(sK + st * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tc_mma_bf16_ts(tS + (j % C::NS) * 64, tQ + kk * 8,
                                   umma_desc_sw128(ka + (kk >> 2) * 8192) + 2 * (kk & 3), IDESC_S, kk > 0 ? 1u : 0u);
                tc_commit(&s_full[j % C::NS]);
                return true;
            };
            for (int j = 0; j < C::NS && j < ntiles && ok; ++j) ok = issue_s(j);
            for (int it = 0; it < ntiles && ok; ++it) {
                // O += P_it V_it once the softmax has written P_it (and so read S_it)
                const int pb = it & 1;
                if (!mbar_wait(&p_full[pb], (uint32_t)((it >> 1) & 1), abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t va = smem_u32(sV + (it % S) * C::KV_BYTES);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_bf16_ts(tO, tP + pb * 32 + kk * 8, umma_desc_sw128_mn(va + kk * 2048, 8192, 1024),
                                   IDESC_PV, (it > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&o_done[pb]);
                tc_commit(&kv_empty[it % S]);
                if (it + C::NS < ntiles) ok = issue_s(it + C::NS);
            }
            if (*abort_flag) {
                tc_commit(drain);   // let the issued MMAs finish before TMEM is released
                volatile int never = 0;
                mbar_wait(drain, 0, &never, nullptr);
            }
        }
    } else {
        // ------------------------------------------------------------ softmax (KC keys of a row per thread)
        const int q4 = warp & 3;
        const int rl = q4 * 32 + lane;                 // this thread's TMEM lane
        const int row = rl % RW, cs = rl / RW;         // query row, key slice (warp-uniform)
        const int e = tid - 64;                        // 0..127
        const uint32_t lanes = (uint32_t)(q4 * 32) << 16;
        const int jrow = row < R ? row / p.G : 0;      // block position of this thread's query row
        griddep_wait();                                // q comes from the QKV GEMM
        const int ntiles = p.req_ok[b] ? ntiles_all : 0;
        {
            // The lane's Q row (zero past R) into the Q operand, and zeros into the
            // lane's columns of both P buffers (other slices' keys stay zero).
            const __nv_bfloat16* qsrc =
                row < R ? p.q + ((size_t)(b * p.gamma + row / p.G) * p.nq + (size_t)(g * p.G + row % p.G)) * D
                        : nullptr;
            // the whole row in one batch of independent loads (one memory round trip),
            // then into tensor memory 16 columns (32 elements) at a time
            uint4 qv[D / 8];
#pragma unroll
            for (int k = 0; k < D / 8; ++k)
                qv[k] = qsrc ? *reinterpret_cast<const uint4*>(qsrc + 8 * k) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c0 = 0; c0 < D / 2; c0 += 16) {   // columns c0..c0+15 = elements 2*c0..2*c0+31
                float v[16];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint4 u = qv[c0 / 4 + k];
                    v[4 * k + 0] = __uint_as_float(u.x);
                    v[4 * k + 1] = __uint_as_float(u.y);
                    v[4 * k + 2] = __uint_as_float(u.z);
                    v[4 * k + 3] = __uint_as_float(u.w);
                }
                tmem_st16(tQ + lanes + c0, v);
            }
            float z[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 16) tmem_st16(tP + lanes + c0, z);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(q_full);
        }
        float base = -INFINITY, mt = -INFINITY, l = 0.f;
        bool ok = true;
        for (int it = 0; it < ntiles; ++it) {
            const int sb = it & 1;           // P buffer
            const int sbuf = it % C::NS;     // S buffer
            ok = mbar_wait(&s_full[sbuf], (uint32_t)((it / C::NS) & 1), abort_flag, p.status);
            tc_fence_after();
            if (trace && it == 0 && e == 0) trace[3] = (long long)globaltimer_ns();
            const int kvb = kv0 + it * 64 + cs * KC;   // first key of this thread's slice
            const uint32_t ts = tS + lanes + sbuf * 64 + cs * KC;
            // the slice's raw scores, masked past the last key, and their maximum over 8
            // independent partial maxima (exact in any order).  The scale to log2 units
            // is applied to the maximum (rounding is monotonic, so this equals the
            // maximum of the scaled scores) and inside the exponent's FMA.
            float t[KC];
            if constexpr (KC == 64) {
                tmem_ld32w(ts, t);
                tmem_ld32w(ts + 32, t + 32);
            } else if constexpr (KC == 32) {
                tmem_ld32w(ts, t);
            } else {
                tmem_ld16w(ts, t);
            }
            // keys past the split's end, and with a causal mask past the row's own position
            const int nvalid = (p.causal ? min(kv1, len_b + jrow + 1) : kv1) - kvb;
            if (nvalid < KC) {
#pragma unroll
                for (int i = 0; i < KC; ++i) t[i] = (i < nvalid) ? t[i] : -INFINITY;
            }
            float m8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = t[k];
#pragma unroll
            for (int i = 8; i < KC; ++i) m8[i & 7] = fmaxf(m8[i & 7], t[i]);
            const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                   fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
            mt = fmaxf(mt, mx * p.scale_log2);   // running maximum of this slice, log2 units
            if (ok && it >= 2)   // the P.V of tile it-2 read this P buffer: wait for it
                ok = mbar_wait(&o_done[sb], (uint32_t)(((it - 2) >> 1) & 1), abort_flag, p.status);
            // The integer base may lag the running maximum by up to kAttnBaseLag: P is
            // then at most 2^(kAttnBaseLag + 1), and every P and the row sum are the
            // oracle's times one exact power of two, so nothing rounds differently; the
            // O rescale (a wait for the previous P.V plus a TMEM round trip) becomes rare.
            // A row's base moves only if one of its slices' maxima passes base + lag, so
            // one barrier per tile ORs "a wait failed" and "a slice would move its base";
            // only then do the slices exchange maxima (and the first tile always does).
            const bool growl = floorf(mt) > base + kAttnBaseLag;
            if (named_bar_or(1, 128, !ok || growl)) {
                if (named_bar_or(1, 128, !ok)) { ok = false; break; }
                xch[rl] = mt;
                named_bar_sync(1, 128);
                float mrow = mt;
#pragma unroll
                for (int k = 1; k < CS; ++k) mrow = fmaxf(mrow, xch[(rl + k * RW) & 127]);
                const float nb = floorf(mrow);
                const bool grow = nb > base + kAttnBaseLag;
                if (it >= 1) {
                    // Rescale the lane's O and l by 2^(base - nb), an exact power of two
                    // (the TMEM accesses are warp-collective, so all 128 threads take
                    // part; rows whose base did not grow scale by 1).
                    ok = mbar_wait(&o_done[(it - 1) & 1], (uint32_t)(((it - 1) >> 1) & 1), abort_flag, p.status);
                    if (named_bar_or(1, 128, !ok)) { ok = false; break; }
                    tc_fence_after();
                    const float f = grow ? exp2f(base - nb) : 1.0f;
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 16) {
                        float v[16];
                        tmem_ld16w(tO + lanes + c0, v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] *= f;
                        tmem_st16(tO + lanes + c0, v);
                    }
                    tmem_wait_st();
                    l *= f;
                }
                if (grow) base = nb;
            }
            // The last tile of a split may extend past the last key: zero those V
            // rows (P is 0 there, but 0 * NaN from never-written cache slack is NaN).
            const int valid = kv1 - (kv0 + it * 64);
            if (valid < 64) {
                uint8_t* vs = sV + (it % S) * C::KV_BYTES;
                for (int idx = e; idx < (64 - valid) * C::HALVES * 8; idx += 128) {
                    const int r = valid + idx / (C::HALVES * 8), rem = idx % (C::HALVES * 8);
                    *reinterpret_cast<uint4*>(vs + (rem / 8) * 8192 + r * 128 + (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();   // the P.V MMA reads these rows through the async proxy
            }
            // P = bf16(2^(t - base)) of the slice's keys, two per TMEM column, into
            // this lane's columns cs*KC/2 .. of P buffer sb.
            const float bb = (base == -INFINITY) ? 0.f : base;
            uint32_t pk[KC / 2];
            float ls[KC / 16];   // independent partial sums, one per 16 keys
#pragma unroll
            for (int c0 = 0; c0 < KC; c0 += 16) {
                float s2 = 0.f;
#pragma unroll
                for (int i = 0; i < 16; i += 2) {
                    const float e0 = ex2_fast(fmaf(t[c0 + i], p.scale_log2, -bb));
                    const float e1 = ex2_fast(fmaf(t[c0 + i + 1], p.scale_log2, -bb));
                    s2 += e0 + e1;
                    pk[(c0 + i) / 2] = pack_bf16(e0, e1);
                }
                ls[c0 >> 4] = s2;
            }
            const uint32_t tp = tP + lanes + sb * 32 + cs * (KC / 2);
            if constexpr (KC == 64) {
                float pv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pv[i] = __uint_as_float(pk[i]);
                tmem_st16(tp, pv);
#pragma unroll
                for (int i = 0; i < 16; ++i) pv[i] = __uint_as_float(pk[16 + i]);
                tmem_st16(tp + 16, pv);
                l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            } else if constexpr (KC == 32) {
                float pv[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) pv[i] = __uint_as_float(pk[i]);
                tmem_st16(tp, pv);
                l += ls[0] + ls[1];
            } else {
                tmem_st8u(tp, pk);
                l += ls[0];
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&p_full[sb]);
        }
        // O of the whole split, once its last P.V has landed.
        if (ok && ntiles >= 1) {
            ok = mbar_wait(&o_done[(ntiles - 1) & 1], (uint32_t)(((ntiles - 1) >> 1) & 1), abort_flag, p.status);
            ok = !named_bar_or(1, 128, !ok);
            tc_fence_after();
        }
        if (trace && e == 0) trace[4] = (long long)globaltimer_ns();
        xch[rl] = l;              // the slices' partial row sums (same base)
        named_bar_sync(1, 128);   // every softmax thread is past the key loop before the ring is reused
        float lrow = l;
#pragma unroll
        for (int k = 1; k < CS; ++k) lrow += xch[(rl + k * RW) & 127];
        // the lane's O (its key slice's share of the row) into po[rl], 32 columns per
        // tensor-memory load
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
            float v[32];
            if (ok && ntiles >= 1) {
                tmem_ld32w(tO + lanes + c0, v);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(po + rl * PO_LD + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
        named_bar_sync(1, 128);
        // add the CS slices of each row into its first-window lane; the row's CS
        // threads take D/CS columns each (loads of several columns in flight at once)
#pragma unroll 4
        for (int c = cs * (D / CS); c < (cs + 1) * (D / CS); c += 4) {
            float4 a = *reinterpret_cast<const float4*>(po + row * PO_LD + c);
#pragma unroll
            for (int k = 1; k < CS; ++k) {
                const float4 o2 = *reinterpret_cast<const float4*>(po + (row + k * RW) * PO_LD + c);
                a.x += o2.x;
                a.y += o2.y;
                a.z += o2.z;
                a.w += o2.w;
            }
            *reinterpret_cast<float4*>(po + row * PO_LD + c) = a;
        }
        if (cs == 0) pml[row] = make_float2(base, ok ? lrow : 0.f);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
    if (trace && tid == 0) trace[5] = (long long)globaltimer_ns();

    // ---- merge the cluster's partials through distributed shared memory
    cluster.sync();
    if (trace && tid == 0) trace[6] = (long long)globaltimer_ns();
    const float* rpo[kAttnMaxSplits];
    const float2* rpml[kAttnMaxSplits];
#pragma unroll
    for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
        rpo[s2] = s2 < nsplit ? cluster.map_shared_rank(po, s2) : po;
        rpml[s2] = s2 < nsplit ? cluster.map_shared_rank(pml, s2) : pml;
    }
    // One round of distributed-shared-memory reads per output piece: columns
    // [c, c+4) and [c + D/2, c + D/2 + 4) of a row, so the lanes of a half-warp read
    // contiguous 256-byte runs.  Each thread fetches every split's (base, sum) of its
    // row and its 8 O columns together, and forms the row's merge weights itself
    // (exact powers of two times 1 / the merged sum).  At up to 16 rows per CTA every
    // thread has one piece.
    const int nr = r_hi - r_lo;
    for (int idx = tid; idx < nr * (D / 8); idx += kAttnThreads) {
        const int rr = idx / (D / 8), c = (idx % (D / 8)) * 4, r = r_lo + rr;
        float2 ml[kAttnMaxSplits];
        float4 va[kAttnMaxSplits], vb[kAttnMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
            if (s2 < nsplit) {
                ml[s2] = rpml[s2][r];
                va[s2] = *reinterpret_cast<const float4*>(rpo[s2] + r * PO_LD + c);
                vb[s2] = *reinterpret_cast<const float4*>(rpo[s2] + r * PO_LD + c + D / 2);
            } else {
                ml[s2] = make_float2(0.f, 0.f);
                va[s2] = vb[s2] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < kAttnMaxSplits; ++s2)
            if (s2 < nsplit && ml[s2].y > 0.f) M = fmaxf(M, ml[s2].x);
        const float bm = (M == -INFINITY) ? 0.f : M;
        float wv[kAttnMaxSplits];
        float L = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
            wv[s2] = (s2 < nsplit && ml[s2].y > 0.f) ? exp2f(ml[s2].x - bm) : 0.f;
            L += wv[s2] * ml[s2].y;
        }
        const float inv = L > 0.f ? 1.0f / L : 0.f;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s2 = 0; s2 < kAttnMaxSplits; ++s2) {
            if (s2 < nsplit) {
                const float w = wv[s2] * inv;
                acc[0] += w * va[s2].x;
                acc[1] += w * va[s2].y;
                acc[2] += w * va[s2].z;
                acc[3] += w * va[s2].w;
                acc[4] += w * vb[s2].x;
                acc[5] += w * vb[s2].y;
                acc[6] += w * vb[s2].z;
                acc[7] += w * vb[s2].w;
            }
        }
        const int j = r / p.G, hh = r % p.G;
        __nv_bfloat16* dst = p.out + ((size_t)(b * p.gamma + j) * p.nq + (size_t)(g * p.G + hh)) * D + c;
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]));
        *reinterpret_cast<uint2*>(dst + D / 2) = make_uint2(pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
    }
    if (trace && tid == 0) trace[7] = (long long)globaltimer_ns();
    cluster.sync();   // keep this CTA's shared memory alive until every peer has read it
}

int attn_smem_bytes(int d) { return d == 128 ? AttnCfg<128>::SMEM : AttnCfg<64>::SMEM; }

int attn_max_cluster(int d) {
    static int cached[2] = {0, 0};
    int& c = cached[d == 128 ? 1 : 0];
    if (c) return c;
    // both row-copy variants use the same resources
    void (*kern)(AttnParams) = (d == 128) ? k_attn_tc<128, 2> : k_attn_tc<64, 2>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(d));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kAttnMaxSplits, 1, 1);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = attn_smem_bytes(d);
    int size = 0;
    if (cudaOccupancyMaxPotentialClusterSize(&size, kern, &cfg) != cudaSuccess || size < 1) size = 1;
    cudaGetLastError();
    c = size < kAttnMaxSplits ? size : kAttnMaxSplits;
    return c;
}

// One wave: at most one CTA per SM over all clusters, clusters of <= max_cluster.
void attn_plan(int B, int nkv, int cap, int num_sms, int max_cluster, int& splits, int& chunk) {
    const int tiles = (cap + 63) / 64;
    int s = num_sms / (B * nkv);
    s = s < 1 ? 1 : (s > max_cluster ? max_cluster : s);
    if (s > tiles) s = tiles;
    chunk = ((tiles + s - 1) / s) * 64;
    splits = (cap + chunk - 1) / chunk;
}

int launch_attention(const AttnParams& p, int d, int B, cudaStream_t stream, long long* launches) {
    const int smem = attn_smem_bytes(d);
    // Row copies: 4 when the R = G * gamma query rows fit 32 lanes, 2 when they fit
    // 64, else 1 (R <= 128: one lane per row, each softmax thread takes all 64 keys).
    const int R = p.G * p.gamma;
    const int cs = R <= 32 ? 4 : (R <= 64 ? 2 : 1);
    void (*kern)(AttnParams) = (d == 128) ? (cs == 4 ? k_attn_tc<128, 4> : cs == 2 ? k_attn_tc<128, 2> : k_attn_tc<128, 1>)
                                          : (cs == 4 ? k_attn_tc<64, 4> : cs == 2 ? k_attn_tc<64, 2> : k_attn_tc<64, 1>);
    static bool done_v[2][3] = {{false, false, false}, {false, false, false}};
    bool& done = done_v[d == 128 ? 1 : 0][cs == 4 ? 2 : cs - 1];
    if (!done) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return (int)e;
        ensure_carveout((const void*)kern);
        done = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.splits, p.nkv, B);
    cfg.blockDim = dim3(kAttnThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    *launches += 1;
    return (int)e;
}

}  // namespace df
